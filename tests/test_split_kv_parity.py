"""GPU parity of the key-range split of a decode (mla_decode_partial + mla_merge_partials), with
N devices emulated one after another on one GPU: every range's partial is computed on the same
device, the partials are stacked as an all-gather would leave them, and merged.  Checked against
the fp64 oracle: each partial against the oracle's decode over that range's visible keys, the
merge against the oracle's decode over all keys."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from workloads import DECODE_CASES, make_decode_inputs
from helpers import check_close, device_pool, dims_of, tiled_ok
from test_sharding import _partials, _sharded

pytestmark = pytest.mark.gpu


def _run(mla, inp, world, layout=None):
    d = inp["dims"]
    bs = inp["block_size"]
    if layout is None:
        layout = 1 if tiled_ok(d, bs) else 0
    dims = dims_of(mla, d, bs, layout)
    dev = {k: inp[k].cuda() for k in ("q_nope", "q_pe", "block_table", "seqlens", "w_uk", "w_uv")}
    B, n_q, H = inp["q_nope"].shape[:3]
    max_seqlen = int(inp["seqlens"].max())
    c_kv, k_pe, _keep = device_pool(mla, d, bs, inp["pool"], layout)
    ranges = _sharded().kv_shard_ranges(max_seqlen, world)
    ws = mla.alloc_workspace(mla.mla_decode_workspace_size(dims, B, n_q, max_seqlen))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    o_parts = torch.empty((world, B, n_q, H, d.d_c), dtype=d.torch_dtype, device="cuda")
    l_parts = torch.empty((world, B, n_q, H), dtype=torch.float32, device="cuda")
    bt = dev["block_table"] if inp["case"].paged else None
    for r, (k0, k1) in enumerate(ranges):
        if k1 <= k0:
            o_parts[r].zero_()
            l_parts[r].fill_(float("-inf"))
            continue
        mla.mla_decode_partial(dims, dev["q_nope"], dev["q_pe"], c_kv, k_pe, bt, inp["max_blocks_per_seq"],
                               inp["num_blocks"], dev["seqlens"], max_seqlen, k0, k1, dev["w_uk"], o_parts[r],
                               l_parts[r], ws, st)
    out = torch.full((B, n_q, H, d.d_v), float("nan"), dtype=d.torch_dtype, device="cuda")
    lse = torch.full((B, n_q, H), float("nan"), dtype=torch.float32, device="cuda")
    mws = mla.alloc_workspace(mla.mla_merge_workspace_size(dims, B, n_q, world))
    mla.mla_merge_partials(dims, o_parts, l_parts, dev["w_uv"], out, lse, mws)
    torch.cuda.synchronize()
    return (ranges, o_parts.float().cpu().numpy(), l_parts.cpu().numpy(), out.float().cpu().numpy(),
            lse.cpu().numpy(), int(st.item()))


@pytest.mark.parametrize("name,world,layout", [("small_v3_nq2_bf16", 2, None), ("small_v3_nq2_bf16", 3, 0),
                                              ("small_v3_many_bf16", 4, None), ("small_f32_nq2", 3, None)])
def test_split_kv_small(lib, name, world, layout):
    inp = make_decode_inputs(DECODE_CASES[name])
    ranges, o_parts, l_parts, out, lse, st = _run(lib, inp, world, layout)
    assert st == 0
    dt = inp["dims"].dtype
    tol = 1e-4 if dt == "f32" else 3e-2
    # each partial against the oracle's decode over its range (heads 0 and H-1 for the 24-sequence case)
    H = inp["dims"].n_heads
    heads = [0, H - 1] if inp["q_nope"].shape[0] > 8 else None
    o_ref, l_ref = _partials(inp, ranges, heads)
    chk = ~np.isnan(l_ref)
    has = chk & np.isfinite(l_ref)
    assert np.array_equal(np.isfinite(l_parts)[chk], has[chk])
    check_close(o_parts[has], o_ref[has], dt, f"{name} partials")
    assert np.max(np.abs(l_parts[has] - l_ref[has])) <= tol
    # the merge against the decode over all keys
    ref, ref_lse = oracle.decode(inp["dims"], inp["q_nope"], inp["q_pe"], inp["pool"], inp["block_table"],
                                 inp["block_size"], inp["seqlens"], inp["w_uk"], inp["w_uv"])
    check_close(out, ref, dt, f"{name} merged over {world} ranges")
    assert np.max(np.abs(lse - ref_lse)) <= tol


def test_split_kv_128k_sequence_over_four_ranges(lib):
    """Config 4b (4 sequences of 131,072 keys, two causal query tokens) split into 4 key ranges of
    32,768: sequence 0 at every head, heads 0 and H-1 of the other sequences."""
    inp = make_decode_inputs(DECODE_CASES["v3_long_bf16"])
    _, _, _, out, lse, st = _run(lib, inp, 4)
    assert st == 0 and np.all(np.isfinite(out))
    B, n_q, H = inp["q_nope"].shape[:3]
    picks = [(0, j, s) for j in range(n_q) for s in range(H)] + \
            [(b, j, s) for b in range(1, B) for j in range(n_q) for s in (0, H - 1)]
    ref, ref_lse = oracle.decode(inp["dims"], inp["q_nope"], inp["q_pe"], inp["pool"], inp["block_table"],
                                 inp["block_size"], inp["seqlens"], inp["w_uk"], inp["w_uv"], picks=picks)
    idx = tuple(np.array(picks).T)
    check_close(out[idx], ref[idx], "bf16", "v3_long split over 4 ranges")
    assert np.max(np.abs(lse[idx] - ref_lse[idx])) <= 3e-2
