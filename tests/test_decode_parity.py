"""GPU parity of mla_decode / mla_decode_latent against the fp64 oracle.

Small cases run every output element; the full-size workloads run in the
same launch configuration bench.py times and are checked on sampled
(sequence, query token, head) outputs the oracle computes one by one.
"""
import numpy as np
import pytest
import torch

import oracle
from workloads import DECODE_CASES, make_decode_inputs
from helpers import check_close, gpu_decode

pytestmark = pytest.mark.gpu

SMALL = ["small_f32", "small_f32_nq2", "tiny_fp32", "small_v3_bf16", "small_v3_nq2_bf16", "small_v2lite_bf16",
         "small_v3_contig_bf16", "small_v3_b128_bf16", "small_v3_many_bf16"]


def _oracle(inp, picks=None, latent=False):
    d = inp["dims"]
    w_uv = inp["w_uv"]
    if latent:
        w_uv = torch.eye(d.d_c, dtype=torch.float64)[None].expand(d.n_heads, d.d_c, d.d_c)
        import dataclasses
        d = dataclasses.replace(d, d_v=d.d_c)
    return oracle.decode(d, inp["q_nope"], inp["q_pe"], inp["pool"], inp["block_table"], inp["block_size"],
                         inp["seqlens"], inp["w_uk"], w_uv, picks=picks)


def _lse_tol(dtype):
    return 1e-4 if dtype == "f32" else 3e-2


@pytest.mark.parametrize("name", SMALL)
def test_decode_small_all_outputs(lib, name):
    inp = make_decode_inputs(DECODE_CASES[name])
    out, lse, st = gpu_decode(lib, inp)
    assert st == 0
    ref, ref_lse = _oracle(inp)
    check_close(out, ref, inp["dims"].dtype, name)
    assert np.max(np.abs(lse - ref_lse)) <= _lse_tol(inp["dims"].dtype)


@pytest.mark.parametrize("name", ["small_v3_bf16", "small_v3_nq2_bf16", "small_v2lite_bf16", "small_v3_contig_bf16"])
def test_decode_small_row_pool(lib, name):
    """The same outputs from a row-layout pool (2-D TMA path of the tensor-core kernel)."""
    inp = make_decode_inputs(DECODE_CASES[name])
    out, lse, st = gpu_decode(lib, inp, layout=0)
    assert st == 0
    ref, ref_lse = _oracle(inp)
    check_close(out, ref, inp["dims"].dtype, name + " rows")
    assert np.max(np.abs(lse - ref_lse)) <= _lse_tol(inp["dims"].dtype)


@pytest.mark.parametrize("name", ["small_f32", "small_v3_nq2_bf16", "small_v2lite_bf16"])
def test_decode_latent_small(lib, name):
    inp = make_decode_inputs(DECODE_CASES[name])
    out, lse, st = gpu_decode(lib, inp, latent=True)
    assert st == 0
    ref, ref_lse = _oracle(inp, latent=True)
    check_close(out, ref, inp["dims"].dtype, name + " latent")
    assert np.max(np.abs(lse - ref_lse)) <= _lse_tol(inp["dims"].dtype)


def test_decode_reads_no_unused_rows(lib):
    """Unused pool rows and the tails of partly filled pages hold NaN: any read of
    them would poison the output, so finite parity proves they are masked."""
    inp = make_decode_inputs(DECODE_CASES["small_v3_bf16"])
    assert torch.isnan(inp["pool"].float()).any()
    out, _, st = gpu_decode(lib, inp)
    assert st == 0 and np.all(np.isfinite(out))


def test_decode_bad_block_id_is_reported(lib):
    """A block id outside the pool is caught on the device and reported, not read."""
    inp = make_decode_inputs(DECODE_CASES["small_f32"])
    inp["block_table"] = inp["block_table"].clone()
    inp["block_table"][2, 0] = inp["num_blocks"] + 5
    _, _, st = gpu_decode(lib, inp)
    assert st == -6  # MLA_ERR_BAD_INDEX


def _sample_picks(inp, n_seq, heads, seed):
    g = np.random.default_rng(seed)
    B, n_q, H = inp["q_nope"].shape[:3]
    sl = inp["seqlens"].numpy()
    seqs = {int(np.argmin(sl)), int(np.argmax(sl))}
    while len(seqs) < min(n_seq, B):
        seqs.add(int(g.integers(B)))
    picks = []
    for b in sorted(seqs):
        for s in sorted(set([0, H - 1] + list(g.integers(0, H, size=heads)))):
            for j in range(n_q):
                picks.append((b, j, int(s)))
    return picks


@pytest.mark.parametrize("name,n_seq,heads", [("tiny_fp32", 1, 8), ("v2lite_bf16", 32, 16), ("v3_bf16", 6, 4),
                                              ("v3_long_bf16", 1, 3), ("v3_ragged_bf16", 8, 2)])
def test_decode_full_size_sampled(lib, name, n_seq, heads):
    inp = make_decode_inputs(DECODE_CASES[name])
    out, lse, st = gpu_decode(lib, inp)
    assert st == 0
    assert np.all(np.isfinite(out))
    picks = _sample_picks(inp, n_seq, heads, 7)
    ref, ref_lse = _oracle(inp, picks=picks)
    idx = tuple(np.array(picks).T)
    got = out[idx[0], idx[1], idx[2]]
    check_close(got, ref[idx[0], idx[1], idx[2]], inp["dims"].dtype, name)
    assert np.max(np.abs(lse[idx] - ref_lse[idx])) <= _lse_tol(inp["dims"].dtype)
