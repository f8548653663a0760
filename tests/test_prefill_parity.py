"""GPU parity of mla_prefill (decompressed causal MHA form) against the oracle."""
import numpy as np
import pytest
import torch

import oracle
from workloads import PREFILL_CASES, make_prefill_inputs
from helpers import check_close, dims_of

pytestmark = pytest.mark.gpu


def build_cache(inp):
    """Cache rows from the oracle's append (rounded to the storage dtype), so the
    prefill check does not depend on the GPU append."""
    d = inp["dims"]
    bs = inp["block_size"]
    c, k = oracle.append_latent(inp["h"], inp["w_dkv"], inp["w_kr"], inp["gamma"], inp["pos"], d.rms_eps, d.rope_base)
    pool = torch.full((inp["num_blocks"] * bs, d.d_c + d.d_rope), float("nan"), dtype=d.torch_dtype)
    rows = (inp["block_table"][inp["seq_idx"].long(), (inp["pos"] // bs).long()].long() * bs + (inp["pos"] % bs).long())
    pool[rows] = torch.from_numpy(np.concatenate([c, k], axis=1)).to(d.torch_dtype)
    return pool


def gpu_prefill(mla, inp, pool):
    d = inp["dims"]
    dims = dims_of(mla, d, inp["block_size"])
    dev = {k: inp[k].cuda() for k in ("cu_seqlens", "q_nope", "q_pe", "block_table", "w_uk", "w_uv")}
    pool = pool.cuda()
    total, H = inp["q_nope"].shape[:2]
    out = torch.full((total, H, d.d_v), float("nan"), dtype=d.torch_dtype, device="cuda")
    lse = torch.full((total, H), float("nan"), dtype=torch.float32, device="cuda")
    max_seqlen = int(inp["seqlens"].max())
    B = inp["seqlens"].numel()
    ws = mla.alloc_workspace(mla.mla_prefill_workspace_size(dims, B, total, max_seqlen))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    mla.mla_prefill(dims, dev["cu_seqlens"], max_seqlen, dev["q_nope"], dev["q_pe"], pool, pool[:, d.d_c:],
                    dev["block_table"], inp["max_blocks_per_seq"], inp["num_blocks"], dev["w_uk"], dev["w_uv"],
                    out, lse, ws, st)
    torch.cuda.synchronize()
    return out.float().cpu().numpy(), lse.cpu().numpy(), int(st.item())


@pytest.mark.parametrize("name", ["small_prefill_f32", "small_prefill_bf16"])
def test_prefill_small_all_rows(lib, name):
    inp = make_prefill_inputs(PREFILL_CASES[name])
    pool = build_cache(inp)
    out, lse, st = gpu_prefill(lib, inp, pool)
    assert st == 0
    ref, ref_lse = oracle.prefill(inp["dims"], inp["q_nope"], inp["q_pe"], pool, inp["block_table"],
                                  inp["block_size"], inp["cu_seqlens"], inp["w_uk"], inp["w_uv"])
    check_close(out, ref, inp["dims"].dtype, name)
    assert np.max(np.abs(lse - ref_lse)) <= (1e-4 if inp["dims"].dtype == "f32" else 3e-2)


def test_prefill_full_size_sampled_rows(lib):
    """Batch 2 x 8192, 128 heads: every 512th row plus the last rows of each sequence."""
    inp = make_prefill_inputs(PREFILL_CASES["v3_prefill_bf16"])
    pool = build_cache(inp)
    out, lse, st = gpu_prefill(lib, inp, pool)
    assert st == 0 and np.all(np.isfinite(out))
    cu = inp["cu_seqlens"].tolist()
    pick = set()
    for b in range(len(cu) - 1):
        pick |= set(range(cu[b], cu[b + 1], 997)) | {cu[b + 1] - 1, cu[b + 1] - 2}
    ref, ref_lse = oracle.prefill(inp["dims"], inp["q_nope"], inp["q_pe"], pool, inp["block_table"],
                                  inp["block_size"], inp["cu_seqlens"], inp["w_uk"], inp["w_uv"], rows_pick=pick)
    rows = sorted(pick)
    check_close(out[rows], ref[rows], "bf16", "prefill v3 sampled")
