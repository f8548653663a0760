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
from helpers import check_close, dims_of, gpu_decode

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
    """A block id outside the pool is caught on the device and reported, not read (CUDA-core path)."""
    inp = make_decode_inputs(DECODE_CASES["small_f32"])
    inp["block_table"] = inp["block_table"].clone()
    inp["block_table"][2, 0] = inp["num_blocks"] + 5
    _, _, st = gpu_decode(lib, inp)
    assert st == -6  # MLA_ERR_BAD_INDEX


@pytest.mark.parametrize("layout", [0, 1])
def test_decode_tc_bad_block_id_is_reported(lib, layout):
    """The tensor-core kernel reports a block id outside the pool (and reads pool row 0 in its
    place, which is inside the pool); the other sequences' outputs are unaffected."""
    inp = make_decode_inputs(DECODE_CASES["small_v3_bf16"])
    bad = inp["block_table"].clone()
    bad[2, 0] = inp["num_blocks"] + 5
    good_ref, good_lse = _oracle(inp, picks=[(b, 0, s) for b in (0, 1) for s in range(inp["dims"].n_heads)])
    inp["block_table"] = bad
    out, lse, st = gpu_decode(lib, inp, layout=layout)
    assert st == -6
    check_close(out[:2], good_ref[:2], "bf16", "sequences with valid tables")
    assert np.max(np.abs(lse[:2] - good_lse[:2])) <= 3e-2


def _check_picks(inp, out, lse, picks, what):
    ref, ref_lse = _oracle(inp, picks=picks)
    idx = tuple(np.array(picks).T)
    check_close(out[idx], ref[idx], inp["dims"].dtype, what)
    assert np.max(np.abs(lse[idx] - ref_lse[idx])) <= _lse_tol(inp["dims"].dtype), what


def _all_heads(inp, seqs):
    _, n_q, H = inp["q_nope"].shape[:3]
    return [(b, j, s) for b in seqs for j in range(n_q) for s in range(H)]


@pytest.mark.parametrize("name", ["tiny_fp32", "v2lite_bf16", "v3_bf16"])
def test_decode_full_size_every_output(lib, name):
    """Configs 1-3 at full size, every (sequence, query token, head) output and its lse.  The
    V3 batch-64 x 4096 step runs in the launch configuration bench.py times: its 4096 key
    tiles are cut evenly over the persistent clusters, so most sequences are split
    between two clusters and merged by the combine kernel."""
    inp = make_decode_inputs(DECODE_CASES[name])
    out, lse, st = gpu_decode(lib, inp)
    assert st == 0 and np.all(np.isfinite(out))
    ref, ref_lse = _oracle(inp)
    check_close(out, ref, inp["dims"].dtype, name)
    assert np.max(np.abs(lse - ref_lse)) <= _lse_tol(inp["dims"].dtype)


def test_decode_ragged_long_sampled_sequences(lib):
    """Config 4a (batch 128, seqlens uniform in [512, 32768], two causal query tokens): the
    shortest and the longest sequence plus six seeded random ones, every head and token;
    heads 0 and H-1 of every other sequence."""
    inp = make_decode_inputs(DECODE_CASES["v3_ragged_bf16"])
    out, lse, st = gpu_decode(lib, inp)
    assert st == 0 and np.all(np.isfinite(out))
    sl = inp["seqlens"].numpy()
    B, n_q, H = inp["q_nope"].shape[:3]
    g = np.random.default_rng(41)
    full = {int(np.argmin(sl)), int(np.argmax(sl))}
    while len(full) < 8:
        full.add(int(g.integers(B)))
    picks = _all_heads(inp, sorted(full))
    picks += [(b, j, s) for b in range(B) if b not in full for j in range(n_q) for s in (0, H - 1)]
    _check_picks(inp, out, lse, picks, "v3_ragged_bf16")


def test_decode_long_128k_sequence(lib):
    """Config 4b (batch 4 at 131072 keys, two causal query tokens): sequence 0 at every head
    and token; heads 0 and H-1 of the other three."""
    inp = make_decode_inputs(DECODE_CASES["v3_long_bf16"])
    out, lse, st = gpu_decode(lib, inp)
    assert st == 0 and np.all(np.isfinite(out))
    B, n_q, H = inp["q_nope"].shape[:3]
    picks = _all_heads(inp, [0]) + [(b, j, s) for b in range(1, B) for j in range(n_q) for s in (0, H - 1)]
    _check_picks(inp, out, lse, picks, "v3_long_bf16")


def test_decode_tiny_on_cache_built_by_gpu_append(lib):
    """Config 1 end to end: the cache of all 256 tokens is written by mla_append_latent from
    h (RMSNorm(h W_DKV), RoPE(h W_KR)), then decoded; the oracle appends and decodes the same
    h on the CPU."""
    from workloads import make_append_inputs
    case = DECODE_CASES["tiny_fp32"]
    d = case.dims
    S = int(case.seqlens[1])
    base = make_decode_inputs(case)
    app = make_append_inputs(d, S, torch.tensor([S], dtype=torch.int32), case.block_size, False, seed=case.seed + 7,
                             gamma_random=True, tokens=[(0, p) for p in range(S)])
    dims = dims_of(lib, d, case.block_size)
    pool = torch.full_like(base["pool"], float("nan")).cuda()
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    dev = {k: app[k].cuda() for k in ("h", "w_dkv", "w_kr", "gamma", "seq_idx", "pos")}
    lib.mla_append_latent(dims, dev["h"], dev["w_dkv"], dev["w_kr"], dev["gamma"], dev["seq_idx"], dev["pos"],
                          pool, pool[:, d.d_c:], None, 1, base["max_blocks_per_seq"], base["num_blocks"], st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    inp = dict(base)
    inp["pool"] = pool.cpu()
    out, lse, st2 = gpu_decode(lib, inp)
    assert st2 == 0
    c, k = oracle.append_latent(app["h"], app["w_dkv"], app["w_kr"], app["gamma"], app["pos"], d.rms_eps,
                                d.rope_base)
    ref_inp = dict(base)
    ref_inp["pool"] = torch.from_numpy(np.concatenate([c, k], 1))
    ref, ref_lse = _oracle(ref_inp)
    check_close(out, ref, "f32", "tiny fp32, cache from the GPU append")
    assert np.max(np.abs(lse - ref_lse)) <= 1e-4
