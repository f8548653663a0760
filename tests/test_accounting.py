"""Algorithmic work accounting (the numerators of every roofline the bench reports).

Each count is checked against an independent construction: visible (query,
key) pairs come from an explicit causal mask built from token positions, and
the per-pair operation counts from the shapes of the products the absorbed and
decompressed forms perform.  The cached row is the latent c_KV (width d_c)
plus the shared RoPE key (width d_R) ("DeepSeek-V3 解读 1: MLA", §MLA
高层次的思路 and §解耦 RoPE).  Queries are absorbed through W_UK and outputs
projected through W_UV in decode; prefill decompresses per head
("Transformer升级之路：21、MLA好在哪里?（下）", §双重投影).
"""
import numpy as np
import pytest

from workloads import (DECODE_CASES, PREFILL_CASES, Dims, V3, append_flops, decode_flops, latent_bytes,
                       prefill_flops)


def _visible_pairs_decode(seqlens, n_q):
    """Pairs (query token, key) allowed by causality: the n_q newest tokens of a
    sequence of length S sit at positions S-n_q .. S-1 and see every key at a
    position not after their own."""
    total = 0
    for S in seqlens:
        key_pos = np.arange(S)
        q_pos = np.arange(S - n_q, S)
        total += int((key_pos[None, :] <= q_pos[:, None]).sum())
    return total


def _matmul_flops(m, k, n):
    return 2 * m * k * n


@pytest.mark.parametrize("seqlens,n_q", [((1, 77, 300), 1), ((2, 65, 130), 2), ((5,), 3), ((4096,) * 3, 1)])
def test_decode_flops_by_explicit_products(seqlens, n_q):
    d = Dims(8, 64, 16, 32, 32, 256, "f32")
    got = decode_flops(d, seqlens, n_q)
    pairs = _visible_pairs_decode(seqlens, n_q)
    H = d.n_heads
    # Per head and query token: scores = q_abs [1, d_c+d_R] @ K^T [d_c+d_R, visible];
    # latent output = P [1, visible] @ C [visible, d_c].
    att = H * (_matmul_flops(1, d.d_c + d.d_rope, pairs) + _matmul_flops(1, pairs, d.d_c))
    tokens = len(seqlens) * n_q
    absorb = H * _matmul_flops(tokens, d.d_nope, d.d_c)      # q_nope [tokens, d_nope] @ W_UK[h] [d_nope, d_c]
    up = H * _matmul_flops(tokens, d.d_c, d.d_v)             # o_lat [tokens, d_c] @ W_UV[h] [d_c, d_v]
    assert got == dict(attention=att, absorb=absorb, up=up, total=att + absorb + up)


def test_v3_decode_workload_figures():
    """V3 shapes at batch 64 x 4096 keys, one query token: 2176 FLOPs per
    (head, key) of attention, 73.0 GFLOP, and one 576-wide bf16 row per key."""
    case = DECODE_CASES["v3_bf16"]
    d = case.dims
    seqlens = [4096] * 64
    assert d.latent_width == 576
    assert latent_bytes(d, seqlens) == 64 * 4096 * 576 * 2 == 301_989_888
    f = decode_flops(d, seqlens, 1)
    assert f["attention"] == 64 * 4096 * 128 * 2176
    assert round(f["attention"] / 1e9, 1) == 73.0


def test_latent_bytes_fp32_and_ragged():
    d = Dims(8, 64, 16, 32, 32, 256, "f32")
    assert latent_bytes(d, [1, 77, 300]) == (1 + 77 + 300) * 80 * 4
    assert latent_bytes(d, []) == 0


@pytest.mark.parametrize("seqlens", [(1,), (5, 70), (1, 130, 257)])
def test_prefill_flops_by_explicit_mask(seqlens):
    d = Dims(8, 64, 16, 32, 32, 256, "f32")
    got = prefill_flops(d, seqlens)
    H = d.n_heads
    pairs = sum(int(np.tril(np.ones((s, s), dtype=bool)).sum()) for s in seqlens)
    # Per head: S = Q [., d_nope+d_R] K^T over visible pairs, O = P V over d_v.
    att = H * (_matmul_flops(1, d.d_nope + d.d_rope, pairs) + _matmul_flops(1, pairs, d.d_v))
    tok = sum(seqlens)
    # Per head: k_nope = C W_UK[h]^T and v = C W_UV[h] for every cached token.
    decomp = H * (_matmul_flops(tok, d.d_c, d.d_nope) + _matmul_flops(tok, d.d_c, d.d_v))
    assert got == dict(attention=att, decompress=decomp, total=att + decomp)


def test_v3_prefill_workload_is_two_by_8192():
    case = PREFILL_CASES["v3_prefill_bf16"]
    f = prefill_flops(case.dims, case.seqlens)
    assert f["attention"] == 2 * (8192 * 8193 // 2) * 128 * 2 * (128 + 64 + 128)


def test_append_flops_is_one_projection():
    d = Dims(**V3)
    # h [T, D] @ [W_DKV | W_KR] [D, d_c + d_R]
    assert append_flops(d, 64) == _matmul_flops(64, 7168, 576)
