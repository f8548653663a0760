"""GPU parity of mla_prefill (decompressed causal MHA form) against the oracle."""
import functools

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


def _v3_rows(inp):
    """Every 16th query row plus the last 128 rows of each sequence."""
    cu = inp["cu_seqlens"].tolist()
    pick = set()
    for b in range(len(cu) - 1):
        pick |= set(range(cu[b], cu[b + 1], 16)) | set(range(max(cu[b], cu[b + 1] - 128), cu[b + 1]))
    return sorted(pick)


@functools.lru_cache(maxsize=1)
def _v3_reference():
    """Inputs of config 5 (V3, 2 x 8192 tokens), the cache from the oracle's append, and the
    oracle's output and lse on the checked rows."""
    inp = make_prefill_inputs(PREFILL_CASES["v3_prefill_bf16"])
    pool = build_cache(inp)
    rows = _v3_rows(inp)
    ref, ref_lse = oracle.prefill(inp["dims"], inp["q_nope"], inp["q_pe"], pool, inp["block_table"],
                                  inp["block_size"], inp["cu_seqlens"], inp["w_uk"], inp["w_uv"], rows_pick=set(rows))
    return inp, pool, rows, ref, ref_lse


def test_prefill_full_size_sampled_rows(lib):
    """Config 5 (batch 2 x 8192, 128 heads): every 16th row plus the last 128 rows of each
    sequence, every head, output and lse."""
    inp, pool, rows, ref, ref_lse = _v3_reference()
    out, lse, st = gpu_prefill(lib, inp, pool)
    assert st == 0 and np.all(np.isfinite(out))
    check_close(out[rows], ref[rows], "bf16", "prefill v3 sampled rows")
    assert np.max(np.abs(lse[rows] - ref_lse[rows])) <= 3e-2


def test_prefill_on_cache_built_by_gpu_append(lib):
    """Config 5 end to end on the GPU: mla_append_latent writes all 16,384 tokens' cache rows
    (the down-projection at prefill size, T = 16,384) and mla_prefill reads them.  The appended
    rows are checked against the oracle's append, and the prefill output against the oracle's
    prefill over the oracle-built cache."""
    inp, pool_ref, rows, ref, ref_lse = _v3_reference()
    d = inp["dims"]
    bs = inp["block_size"]
    dims = dims_of(lib, d, bs)
    T = inp["h"].shape[0]
    dev = {k: inp[k].cuda() for k in ("h", "w_dkv", "w_kr", "gamma", "seq_idx", "pos", "block_table")}
    pool = torch.full((inp["num_blocks"] * bs, d.d_c + d.d_rope), float("nan"), dtype=d.torch_dtype, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    nws = lib.mla_append_workspace_size(dims, T)
    assert nws > 0   # the tensor-core projection runs at this size
    lib.mla_append_latent(dims, dev["h"], dev["w_dkv"], dev["w_kr"], dev["gamma"], dev["seq_idx"], dev["pos"],
                          pool, pool[:, d.d_c:], dev["block_table"], inp["seqlens"].numel(),
                          inp["max_blocks_per_seq"], inp["num_blocks"], st, workspace=lib.alloc_workspace(nws))
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    gpu_pool = pool.cpu()
    # Content against the oracle's fp64 append (not its bf16-rounded copy), row by row through the table.
    c, k = oracle.append_latent(inp["h"], inp["w_dkv"], inp["w_kr"], inp["gamma"], inp["pos"], d.rms_eps,
                                d.rope_base)
    tok_rows = (inp["block_table"][inp["seq_idx"].long(), (inp["pos"] // bs).long()].long() * bs
                + (inp["pos"] % bs).long())
    got = gpu_pool[tok_rows].float().numpy()
    check_close(got[:, :d.d_c], c, "bf16", "append c_KV at T=16384")
    check_close(got[:, d.d_c:], k, "bf16", "append k_pe at T=16384")
    untouched = torch.ones(gpu_pool.shape[0], dtype=torch.bool)
    untouched[tok_rows] = False
    assert torch.isnan(gpu_pool[untouched].float()).all()
    out, lse, st2 = gpu_prefill(lib, inp, gpu_pool)
    assert st2 == 0
    check_close(out[rows], ref[rows], "bf16", "prefill on the GPU-built cache")
    assert np.max(np.abs(lse[rows] - ref_lse[rows])) <= 3e-2
