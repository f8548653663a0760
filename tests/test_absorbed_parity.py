"""GPU parity of the fully absorbed decode from hidden states (mla_fold_query_weights,
mla_fold_output_weights, mla_decode_absorbed) against the fp64 oracle's unfolded chain:
query_from_hidden -> decode (unabsorbed) -> output_projection."""
import numpy as np
import pytest
import torch

import oracle
from workloads import DECODE_CASES, make_decode_inputs, make_query_path_inputs
from helpers import check_close, device_pool, dims_of, tiled_ok

pytestmark = pytest.mark.gpu


def _gpu(mla, inp, qp, layout=None):
    d = inp["dims"]
    bs = inp["block_size"]
    if layout is None:
        layout = 1 if tiled_ok(d, bs) else 0
    dims = dims_of(mla, d, bs, layout)
    dev = {k: v.cuda() for k, v in qp.items()}
    dev.update({k: inp[k].cuda() for k in ("block_table", "seqlens", "w_uk", "w_uv")})
    B, n_q = qp["h"].shape[:2]
    H, d_cq = d.n_heads, qp["w_dq"].shape[1]
    w_uqk = torch.empty((H, d_cq, d.d_c), dtype=d.torch_dtype, device="cuda")
    w_uvo = torch.empty((H, d.d_c, d.d_model), dtype=d.torch_dtype, device="cuda")
    mla.mla_fold_query_weights(dims, dev["w_uq"], dev["w_uk"], w_uqk)
    mla.mla_fold_output_weights(dims, dev["w_uv"], dev["w_o"], w_uvo)
    c_kv, k_pe, _keep = device_pool(mla, d, bs, inp["pool"], layout)
    max_seqlen = int(inp["seqlens"].max())
    out = torch.full((B, n_q, d.d_model), float("nan"), dtype=d.torch_dtype, device="cuda")
    lse = torch.full((B, n_q, H), float("nan"), dtype=torch.float32, device="cuda")
    ws = mla.alloc_workspace(mla.mla_decode_absorbed_workspace_size(dims, d_cq, B, n_q, max_seqlen))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    bt = dev["block_table"] if inp["case"].paged else None
    mla.mla_decode_absorbed(dims, dev["h"], dev["w_dq"], w_uqk, dev["w_qr"], c_kv, k_pe, bt, inp["max_blocks_per_seq"],
                            inp["num_blocks"], dev["seqlens"], max_seqlen, w_uvo, out, lse, ws, st)
    torch.cuda.synchronize()
    return out.float().cpu().numpy(), lse.cpu().numpy(), int(st.item())


def _oracle(inp, qp):
    d = inp["dims"]
    qn, qpe = oracle.query_from_hidden(qp["h"], qp["w_dq"], qp["w_uq"], qp["w_qr"])
    out, lse = oracle.decode(d, qn, qpe, inp["pool"], inp["block_table"], inp["block_size"], inp["seqlens"],
                             inp["w_uk"], inp["w_uv"])
    return oracle.output_projection(out, qp["w_o"]), lse


@pytest.mark.parametrize("name,d_cq,layout", [("small_v3_nq2_bf16", 1536, None), ("small_v3_bf16", 1536, 0),
                                             ("small_v2lite_bf16", 2048, None), ("small_f32_nq2", 48, None)])
def test_absorbed_decode_from_hidden(lib, name, d_cq, layout):
    inp = make_decode_inputs(DECODE_CASES[name])
    qp = make_query_path_inputs(DECODE_CASES[name], d_cq, seed=77)
    out, lse, st = _gpu(lib, inp, qp, layout)
    assert st == 0
    ref, ref_lse = _oracle(inp, qp)
    check_close(out, ref, inp["dims"].dtype, f"{name} absorbed decode")
    assert np.max(np.abs(lse - ref_lse)) <= (1e-4 if inp["dims"].dtype == "f32" else 3e-2)
