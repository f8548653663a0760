"""GPU parity of mla_decode_sparse (decode over a per-query-token selection of cached tokens)
against the fp64 oracle's sparse decode."""
import numpy as np
import pytest
import torch

import oracle
from workloads import DECODE_CASES, make_decode_inputs
from helpers import check_close, device_pool, dims_of, tiled_ok

pytestmark = pytest.mark.gpu


def make_selection(inp, topk, seed, pad_every=5):
    """Per query token, up to topk distinct tokens from 0 .. its causal limit, in random order, with
    -1 padding sprinkled in (every pad_every-th slot) and at the end."""
    g = np.random.default_rng(seed)
    B, n_q = inp["q_nope"].shape[:2]
    sl = inp["seqlens"].numpy()
    sel = np.full((B, n_q, topk), -1, dtype=np.int32)
    for b in range(B):
        for j in range(n_q):
            p = int(sl[b]) - n_q + j
            slots = [k for k in range(topk) if pad_every == 0 or k % pad_every != pad_every - 1]
            n = min(len(slots), p + 1)
            toks = g.permutation(p + 1)[:n]
            for k, t in zip(slots[:n], toks):
                sel[b, j, k] = t
    return torch.from_numpy(sel)


def gpu_sparse(mla, inp, sel, layout=None):
    d = inp["dims"]
    bs = inp["block_size"]
    if layout is None:
        layout = 1 if tiled_ok(d, bs) else 0
    dims = dims_of(mla, d, bs, layout)
    dev = {k: inp[k].cuda() for k in ("q_nope", "q_pe", "block_table", "seqlens", "w_uk", "w_uv")}
    B, n_q, H = inp["q_nope"].shape[:3]
    c_kv, k_pe, _keep = device_pool(mla, d, bs, inp["pool"], layout)
    out = torch.full((B, n_q, H, d.d_v), float("nan"), dtype=d.torch_dtype, device="cuda")
    lse = torch.full((B, n_q, H), float("nan"), dtype=torch.float32, device="cuda")
    ws = mla.alloc_workspace(mla.mla_decode_sparse_workspace_size(dims, B, n_q, sel.shape[2]))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    bt = dev["block_table"] if inp["case"].paged else None
    mla.mla_decode_sparse(dims, dev["q_nope"], dev["q_pe"], c_kv, k_pe, bt, inp["max_blocks_per_seq"],
                          inp["num_blocks"], dev["seqlens"], int(inp["seqlens"].max()), sel.cuda(), dev["w_uk"],
                          dev["w_uv"], out, lse, ws, st)
    torch.cuda.synchronize()
    return out.float().cpu().numpy(), lse.cpu().numpy(), int(st.item())


def _oracle(inp, sel, picks=None):
    return oracle.decode_sparse(inp["dims"], inp["q_nope"], inp["q_pe"], inp["pool"], inp["block_table"],
                                inp["block_size"], inp["seqlens"], sel.numpy(), inp["w_uk"], inp["w_uv"], picks=picks)


def _tol(dtype):
    return 1e-4 if dtype == "f32" else 3e-2


@pytest.mark.parametrize("name,topk,layout", [("small_v3_bf16", 100, None), ("small_v3_bf16", 300, 0),
                                             ("small_v3_nq2_bf16", 130, None), ("small_v2lite_bf16", 64, None),
                                             ("small_f32_nq2", 40, None), ("small_v3_many_bf16", 257, None)])
def test_sparse_small_all_outputs(lib, name, topk, layout):
    inp = make_decode_inputs(DECODE_CASES[name])
    sel = make_selection(inp, topk, seed=topk)
    out, lse, st = gpu_sparse(lib, inp, sel, layout)
    assert st == 0
    ref, ref_lse = _oracle(inp, sel)
    check_close(out, ref, inp["dims"].dtype, f"{name} sparse top{topk}")
    assert np.max(np.abs(lse - ref_lse)) <= _tol(inp["dims"].dtype)


def test_sparse_full_selection_matches_dense_decode(lib):
    """Listing every visible token in order gives mla_decode's output."""
    from helpers import gpu_decode
    inp = make_decode_inputs(DECODE_CASES["small_v3_nq2_bf16"])
    B, n_q = inp["q_nope"].shape[:2]
    sl = inp["seqlens"].numpy()
    k = int(sl.max())
    sel = torch.full((B, n_q, k), -1, dtype=torch.int32)
    for b in range(B):
        for j in range(n_q):
            p = int(sl[b]) - n_q + j
            sel[b, j, :p + 1] = torch.arange(p + 1, dtype=torch.int32)
    out, lse, st = gpu_sparse(lib, inp, sel)
    dense, dense_lse, st2 = gpu_decode(lib, inp)
    assert st == 0 and st2 == 0
    check_close(out, dense, "bf16", "sparse(all) vs dense")
    assert np.max(np.abs(lse - dense_lse)) <= 3e-2


def test_sparse_entries_past_the_causal_limit_are_reported(lib):
    inp = make_decode_inputs(DECODE_CASES["small_v3_bf16"])
    sel = make_selection(inp, 64, seed=3)
    sel[2, 0, 0] = int(inp["seqlens"][2])          # one past the last visible token
    _, _, st = gpu_sparse(lib, inp, sel)
    assert st == -6


def test_sparse_v3_batch64_top2048(lib):
    """V3 shapes, batch 64 x 4096 keys, 2048 selected tokens per query (the V3.2 top-k size):
    every head of sequences 0 and 63 and of four seeded random sequences."""
    inp = make_decode_inputs(DECODE_CASES["v3_bf16"])
    sel = make_selection(inp, 2048, seed=11, pad_every=0)
    out, lse, st = gpu_sparse(lib, inp, sel)
    assert st == 0 and np.all(np.isfinite(out))
    g = np.random.default_rng(5)
    seqs = sorted({0, 63} | set(int(x) for x in g.choice(64, 4, replace=False)))
    picks = [(b, 0, s) for b in seqs for s in range(inp["dims"].n_heads)]
    ref, ref_lse = _oracle(inp, sel, picks)
    idx = tuple(np.array(picks).T)
    check_close(out[idx], ref[idx], "bf16", "v3 sparse top2048")
    assert np.max(np.abs(lse[idx] - ref_lse[idx])) <= 3e-2
