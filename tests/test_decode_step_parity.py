"""GPU parity of mla_decode_step (the append of a step's new tokens and the decode in one call;
on the tensor-core shapes the append and the query absorption are one kernel launch) against the
fp64 oracle: append_latent of the same hidden states, then the unabsorbed decode.  The cache rows
it writes are also compared bit for bit with those of mla_append_latent."""
import numpy as np
import pytest
import torch

import oracle
from workloads import DECODE_CASES, make_decode_step_inputs
from helpers import check_close, device_pool, dims_of, tiled_ok

pytestmark = pytest.mark.gpu


def _run_step(mla, inp, layout):
    d = inp["dims"]
    bs = inp["block_size"]
    dims = dims_of(mla, d, bs, layout)
    dev = {k: inp[k].cuda() for k in ("q_nope", "q_pe", "block_table", "seqlens", "w_uk", "w_uv", "h_new", "w_dkv",
                                      "w_kr", "gamma")}
    B, n_q, H = inp["q_nope"].shape[:3]
    c_kv, k_pe, keep = device_pool(mla, d, bs, inp["pool"], layout)
    max_seqlen = int(inp["seqlens"].max())
    out = torch.full((B, n_q, H, d.d_v), float("nan"), dtype=d.torch_dtype, device="cuda")
    lse = torch.full((B, n_q, H), float("nan"), dtype=torch.float32, device="cuda")
    ws = mla.alloc_workspace(mla.mla_decode_step_workspace_size(dims, B, n_q, max_seqlen))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    bt = dev["block_table"] if inp["case"].paged else None
    for _ in range(2):   # twice: the second call reuses the workspace (and its completion counter)
        mla.mla_decode_step(dims, dev["h_new"], dev["w_dkv"], dev["w_kr"], dev["gamma"], dev["q_nope"], dev["q_pe"],
                            c_kv, k_pe, bt, inp["max_blocks_per_seq"], inp["num_blocks"], dev["seqlens"], max_seqlen,
                            dev["w_uk"], dev["w_uv"], out, lse, ws, st)
    torch.cuda.synchronize()
    return out.float().cpu().numpy(), lse.cpu().numpy(), int(st.item()), keep


def _run_append(mla, inp, layout):
    """The same new tokens through mla_append_latent (tensor-core projection where it applies)."""
    d = inp["dims"]
    bs = inp["block_size"]
    dims = dims_of(mla, d, bs, layout)
    c_kv, k_pe, keep = device_pool(mla, d, bs, inp["pool"], layout)
    T = inp["h_new"].shape[0]
    nws = mla.mla_append_workspace_size(dims, T)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    B = inp["q_nope"].shape[0]
    mla.mla_append_latent(dims, inp["h_new"].cuda(), inp["w_dkv"].cuda(), inp["w_kr"].cuda(), inp["gamma"].cuda(),
                          inp["seq_idx"].cuda(), inp["pos"].cuda(), c_kv, k_pe,
                          inp["block_table"].cuda() if inp["case"].paged else None, B, inp["max_blocks_per_seq"],
                          inp["num_blocks"], st, workspace=mla.alloc_workspace(nws) if nws else None)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return keep


def _oracle(inp):
    d = inp["dims"]
    bs = inp["block_size"]
    c, k = oracle.append_latent(inp["h_new"], inp["w_dkv"], inp["w_kr"], inp["gamma"], inp["pos"], d.rms_eps,
                                d.rope_base)
    pool = inp["pool"].clone()
    rows = (inp["block_table"][inp["seq_idx"].long(), (inp["pos"] // bs).long()].long() * bs
            + (inp["pos"] % bs).long())
    pool[rows] = torch.from_numpy(np.concatenate([c, k], 1)).to(d.torch_dtype)
    return oracle.decode(d, inp["q_nope"], inp["q_pe"], pool, inp["block_table"], bs, inp["seqlens"], inp["w_uk"],
                         inp["w_uv"])


@pytest.mark.parametrize("name,layout", [("small_v3_nq2_bf16", 1), ("small_v3_bf16", 0), ("small_v2lite_bf16", 1),
                                        ("small_f32_nq2", 0), ("small_v3_many_bf16", 1), ("v3_bf16", 1)])
def test_decode_step(lib, name, layout):
    inp = make_decode_step_inputs(DECODE_CASES[name])
    d = inp["dims"]
    if layout == 1 and not tiled_ok(d, inp["block_size"]):
        pytest.skip("tiled layout needs bf16 and 64-token pages")
    out, lse, st, pool_step = _run_step(lib, inp, layout)
    assert st == 0
    ref, ref_lse = _oracle(inp)
    check_close(out, ref, d.dtype, f"{name} decode step")
    assert np.max(np.abs(lse - ref_lse)) <= (1e-4 if d.dtype == "f32" else 3e-2)
    pool_app = _run_append(lib, inp, layout)
    a = pool_step.view(torch.int16 if d.dtype == "bf16" else torch.int32)
    b = pool_app.view(torch.int16 if d.dtype == "bf16" else torch.int32)
    assert torch.equal(a, b), "cache rows of mla_decode_step differ from mla_append_latent's"
