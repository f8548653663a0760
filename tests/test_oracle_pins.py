"""Pins of the fp64 oracle to facts that do not come from the oracle itself.

Each test names what fixes the expected value: a worked example from the
pages (tests/golden), a closed form, an invariant, a textbook special case
computed by a library routine, or brute force on tiny inputs.  Planted-
mistake tests at the end patch the oracle on the CPU and check that a pin
catches the mistake.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from oracle import mla_oracle as O
from workloads import Dims, DECODE_CASES, make_decode_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")

TINY = Dims(n_heads=2, d_c=4, d_rope=2, d_nope=3, d_v=3, d_model=5, dtype="f32")


def _rng(seed):
    return np.random.default_rng(seed)


# ------------------------------------------------------------------ RoPE (I2)

def test_rope_worked_example_from_pages():
    """DeepSeek-V3 解读 1: MLA, section RoPE: consecutive pairs, second pair at twice the angle."""
    g = json.load(open(os.path.join(GOLDEN, "rope_4d_example.json")))
    for c in g["cases"]:
        th = c["theta0"]
        got = O.rope_rotate(np.array(c["x"]), 1, freqs=[th, 2 * th])
        np.testing.assert_allclose(got, c["expected"], atol=1e-15)
        # Same numbers read as "pair k sits at position k" with one frequency theta_0.
        a = O.rope_rotate(np.array(c["x"][:2]), 1, freqs=[th])
        b = O.rope_rotate(np.array(c["x"][2:]), 2, freqs=[th])
        np.testing.assert_allclose(np.concatenate([a, b]), c["expected"], atol=1e-15)


def test_rope_relative_position_property():
    """<R_p q, R_p' k> depends only on p - p' (the property the page says RoPE keeps)."""
    r = _rng(1)
    q, k = r.standard_normal(64), r.standard_normal(64)
    base = 10000.0
    ref = O.rope_rotate(q, 7, base) @ O.rope_rotate(k, 3, base)
    for shift in (0, 1, 100, 4093, 131000):
        got = O.rope_rotate(q, 7 + shift, base) @ O.rope_rotate(k, 3 + shift, base)
        assert abs(got - ref) < 1e-9 * (1 + abs(ref))


def test_rope_norm_and_zero_position():
    r = _rng(2)
    x = r.standard_normal((5, 16))
    y = O.rope_rotate(x, np.arange(5) * 37, 10000.0)
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-14)
    np.testing.assert_array_equal(O.rope_rotate(x, 0, 10000.0), x)


def test_rope_frequency_schedule_special_cases():
    """Reading theta_i = base^(-2i/d): pair 0 turns by exactly p radians; with base 1 every pair does."""
    f = O.rope_frequencies(64, 10000.0)
    assert f[0] == 1.0 and f.shape == (32,)
    assert np.all(np.diff(f) < 0)
    x = np.array([1.0, 0.0])
    np.testing.assert_allclose(O.rope_rotate(x, 3, 10000.0), [math.cos(3), math.sin(3)], atol=1e-15)
    np.testing.assert_allclose(O.rope_frequencies(8, 1.0), np.ones(4))
    # Geometric: consecutive ratios all equal base^(-2/d).
    np.testing.assert_allclose(f[1:] / f[:-1], np.full(31, 10000.0 ** (-2 / 64)), rtol=1e-13)


def test_rope_composes_as_rotation():
    """R_a R_b = R_{a+b} and R_p applied to the pair basis gives (cos, sin) columns."""
    r = _rng(3)
    x = r.standard_normal(8)
    np.testing.assert_allclose(O.rope_rotate(O.rope_rotate(x, 5, 500.0), 9, 500.0), O.rope_rotate(x, 14, 500.0),
                               atol=1e-13)


# ------------------------------------------------------------------ RMSNorm / append

def test_rms_norm_closed_forms():
    r = _rng(4)
    c = r.standard_normal((6, 32)) * 3.0
    y = O.rms_norm(c, np.ones(32), 0.0)
    np.testing.assert_allclose(np.sqrt(np.mean(y * y, axis=-1)), 1.0, rtol=1e-14)
    # Scale invariance (eps = 0) and the per-channel gain.
    np.testing.assert_allclose(O.rms_norm(7.5 * c, np.ones(32), 0.0), y, rtol=1e-13)
    g = r.standard_normal(32)
    np.testing.assert_allclose(O.rms_norm(c, g, 0.0), y * g, rtol=1e-13)
    # A constant row a*1 maps to sign(a)*gamma when eps = 0.
    np.testing.assert_allclose(O.rms_norm(np.full((1, 4), -2.0), np.array([1, 2, 3, 4.0]), 0.0), [[-1, -2, -3, -4.0]])
    # eps enters under the root: row of zeros stays zero, tiny rows are damped.
    np.testing.assert_array_equal(O.rms_norm(np.zeros((1, 4)), np.ones(4), 1e-6), np.zeros((1, 4)))


def test_append_brute_force_tiny():
    """c_KV = RMSNorm(h W_DKV) and k_pe = RoPE(h W_KR), checked with plain Python loops."""
    r = _rng(5)
    T, D, dc, dr = 3, 5, 4, 2
    h, wd, wk = r.standard_normal((T, D)), r.standard_normal((D, dc)), r.standard_normal((D, dr))
    g = r.standard_normal(dc)
    pos = [0, 4, 11]
    c_kv, k_pe = O.append_latent(h, wd, wk, g, np.array(pos), 1e-6, 10000.0)
    for t in range(T):
        c = [sum(h[t][i] * wd[i][j] for i in range(D)) for j in range(dc)]
        rms = math.sqrt(sum(v * v for v in c) / dc + 1e-6)
        for j in range(dc):
            assert abs(c_kv[t][j] - c[j] / rms * g[j]) < 1e-12
        k = [sum(h[t][i] * wk[i][j] for i in range(D)) for j in range(dr)]
        a = pos[t] * 1.0  # d_R = 2: single pair, theta_0 = 1
        assert abs(k_pe[t][0] - (k[0] * math.cos(a) - k[1] * math.sin(a))) < 1e-12
        assert abs(k_pe[t][1] - (k[0] * math.sin(a) + k[1] * math.cos(a))) < 1e-12


# ------------------------------------------------------------------ cache accounting (I3)

def test_cache_size_numbers_from_pages():
    g = json.load(open(os.path.join(GOLDEN, "kv_cache_sizes.json")))
    gp = g["gpt3"]
    per_tok = O.kv_cache_bytes_mha(gp["layers"], gp["heads"], gp["head_dim"], 1, gp["bytes"])
    assert per_tok // gp["bytes"] == gp["values_per_token"]
    assert round(per_tok / 1e6, 1) == gp["mb_per_token_printed"]
    gb_128k = O.kv_cache_bytes_mha(gp["layers"], gp["heads"], gp["head_dim"], 128 * 1024, gp["bytes"]) / 1e9
    assert 0.5 * gp["context_128k_gb_order"] < gb_128k < 1.5 * gp["context_128k_gb_order"]
    m = g["mla_vs_gqa"]
    assert O.latent_elems_per_token(m["d_c"], m["d_rope"]) == 576
    assert O.latent_elems_per_token(m["d_c"], m["d_rope"]) / (2 * m["head_dim"]) == m["gqa_groups_equivalent"]
    m8 = g["mla_vs_gqa8"]
    assert O.latent_elems_per_token(512, 64) / (2 * m8["gqa_groups"] * m8["head_dim"]) == m8["ratio"]


def test_workload_pool_holds_exactly_latent_width():
    inp = make_decode_inputs(DECODE_CASES["small_f32"])
    d = inp["dims"]
    assert inp["pool"].shape[1] == O.latent_elems_per_token(d.d_c, d.d_rope)


# ------------------------------------------------------------------ softmax (I4)

def test_attend_probabilities_and_one_hot():
    r = _rng(6)
    K, V = r.standard_normal((50, 8)), r.standard_normal((50, 5))
    q = r.standard_normal(8)
    o, lse, p = O.attend(q, K, V, 50, 0.3)
    assert abs(p.sum() - 1.0) < 1e-15
    assert np.all(p >= 0)
    z = K @ q * 0.3
    assert abs(lse - math.log(sum(math.exp(v) for v in z))) < 1e-12
    np.testing.assert_allclose(o, sum(p[i] * V[i] for i in range(50)), rtol=1e-13)
    # A key aligned with a huge query wins outright: the output is exactly its value row.
    K2 = np.zeros((4, 3)); K2[2, 0] = 1.0
    o2, _, p2 = O.attend(np.array([2000.0, 0, 0]), K2, V[:4, :], 4, 1.0)
    np.testing.assert_array_equal(o2, V[2])
    # Only the first n_visible keys count (causal cut).
    o3, _, p3 = O.attend(q, K, V, 10, 0.3)
    o3b, _, _ = O.attend(q, K[:10], V[:10], 10, 0.3)
    np.testing.assert_array_equal(o3, o3b)


def test_attend_matches_library_sdpa():
    """Textbook attention via torch's scaled_dot_product_attention in float64."""
    r = _rng(7)
    S, dk, dv = 37, 12, 9
    K, V, q = r.standard_normal((S, dk)), r.standard_normal((S, dv)), r.standard_normal(dk)
    for n_vis in (1, 17, 37):
        o, _, _ = O.attend(q, K, V, n_vis, 1 / math.sqrt(dk))
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q)[None, None, None], torch.from_numpy(K[:n_vis])[None, None],
            torch.from_numpy(V[:n_vis])[None, None])[0, 0, 0].numpy()
        np.testing.assert_allclose(o, ref, rtol=1e-12, atol=1e-14)


# ------------------------------------------------------------------ absorption identity (I1)

def _absorbed_decode(dims, q_nope, q_pe, pool, bt, bs, seqlens, w_uk, w_uv):
    """Decoding column of the double-projection display: the query is folded with
    W_UK into the latent space, keys are the cached rows themselves, and W_UV is
    applied after the softmax-weighted sum of latents."""
    B, n_q, H, _ = q_nope.shape
    out = np.zeros((B, n_q, H, dims.d_v))
    scale = 1 / math.sqrt(dims.d_nope + dims.d_rope)
    for b in range(B):
        S = int(seqlens[b])
        rows = O.gather_rows(pool, bt, bs, b, S)
        C, R = rows[:, :dims.d_c], rows[:, dims.d_c:]
        for s in range(H):
            for j in range(n_q):
                p = S - n_q + j
                q_lat = np.asarray(w_uk[s], dtype=np.float64) @ np.asarray(q_nope[b, j, s], dtype=np.float64)
                q_r = O.rope_rotate(np.asarray(q_pe[b, j, s], dtype=np.float64), p, dims.rope_base)
                z = (C[:p + 1] @ q_lat + R[:p + 1] @ q_r) * scale
                w = np.exp(z - z.max()); w /= w.sum()
                out[b, j, s] = (w @ C[:p + 1]) @ np.asarray(w_uv[s], dtype=np.float64)
    return out


@pytest.mark.parametrize("name", ["small_f32", "small_f32_nq2"])
def test_absorbed_equals_unabsorbed(name):
    inp = make_decode_inputs(DECODE_CASES[name])
    d = inp["dims"]
    ref, _ = oracle.decode(d, inp["q_nope"], inp["q_pe"], inp["pool"], inp["block_table"], inp["block_size"],
                           inp["seqlens"], inp["w_uk"], inp["w_uv"])
    f = lambda t: t.to(torch.float64).numpy()
    got = _absorbed_decode(d, f(inp["q_nope"]), f(inp["q_pe"]), f(inp["pool"]), inp["block_table"].numpy(),
                           inp["block_size"], inp["seqlens"].numpy(), f(inp["w_uk"]), f(inp["w_uv"]))
    rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert rel < 1e-12, rel


# ------------------------------------------------------------------ MQA reduction (I5)

def test_mqa_reduction_with_identity_projections():
    """W_UK = W_UV = I, d_R = 0, d_nope = d_v = d_c: MLA decode is MQA with K = V = c."""
    dc, H, S = 6, 3, 9
    dims = Dims(n_heads=H, d_c=dc, d_rope=0, d_nope=dc, d_v=dc, d_model=8, dtype="f32")
    r = _rng(8)
    pool = r.standard_normal((S, dc))
    bt = np.arange(S).reshape(1, S)
    q_nope = r.standard_normal((1, 1, H, dc))
    q_pe = np.zeros((1, 1, H, 0))
    eye = np.stack([np.eye(dc)] * H)
    out, _ = oracle.decode(dims, q_nope, q_pe, pool, bt, 1, np.array([S]), eye, eye)
    q = torch.from_numpy(q_nope[0, 0])[:, None, :]          # [H, 1, dc]
    kv = torch.from_numpy(pool)[None].expand(H, S, dc)     # one shared K = V head
    ref = torch.nn.functional.scaled_dot_product_attention(q, kv, kv)[:, 0].numpy()
    np.testing.assert_allclose(out[0, 0], ref, rtol=1e-12, atol=1e-14)


# ------------------------------------------------------------------ brute force tiny (I6)

def _bf_exp(x):
    return math.exp(x)


def test_decode_brute_force_tiny():
    """H = 2, d_c = 4, d_R = 2, S = 3, paged with block size 2: pure-Python loops."""
    r = _rng(9)
    d = TINY
    S, n_q = 3, 1
    pool = r.standard_normal((6, d.d_c + d.d_rope))
    bt = np.array([[2, 0]])          # token 0,1 in block 2 (rows 4,5); token 2 in block 0 (row 0)
    q_nope = r.standard_normal((1, n_q, d.n_heads, d.d_nope))
    q_pe = r.standard_normal((1, n_q, d.n_heads, d.d_rope))
    w_uk = r.standard_normal((d.n_heads, d.d_c, d.d_nope))
    w_uv = r.standard_normal((d.n_heads, d.d_c, d.d_v))
    out, lse = oracle.decode(d, q_nope, q_pe, pool, bt, 2, np.array([S]), w_uk, w_uv)
    rows = [4, 5, 0]
    p = S - 1
    a = p * 1.0
    for s in range(d.n_heads):
        qr = [q_pe[0, 0, s, 0] * math.cos(a) - q_pe[0, 0, s, 1] * math.sin(a),
              q_pe[0, 0, s, 0] * math.sin(a) + q_pe[0, 0, s, 1] * math.cos(a)]
        zs, vs = [], []
        for i in range(S):
            c = pool[rows[i]][:4]
            kn = [sum(c[x] * w_uk[s][x][y] for x in range(4)) for y in range(3)]
            kr = pool[rows[i]][4:]
            z = sum(q_nope[0, 0, s, y] * kn[y] for y in range(3)) + qr[0] * kr[0] + qr[1] * kr[1]
            zs.append(z / math.sqrt(3 + 2))
            vs.append([sum(c[x] * w_uv[s][x][y] for x in range(4)) for y in range(3)])
        den = sum(_bf_exp(z) for z in zs)
        for y in range(3):
            want = sum(_bf_exp(zs[i]) * vs[i][y] for i in range(S)) / den
            assert abs(out[0, 0, s, y] - want) < 1e-12
        assert abs(lse[0, 0, s] - math.log(den)) < 1e-12


def test_softmax_exact_rational_tiny():
    """Weights exp(z_i)/sum exp(z_j) with z = ln(1), ln(2), ln(5) are exactly 1/8, 2/8, 5/8."""
    K = np.array([[math.log(1.0)], [math.log(2.0)], [math.log(5.0)]])
    V = np.eye(3)
    o, lse, p = O.attend(np.array([1.0]), K, V, 3, 1.0)
    for i, want in enumerate([Fraction(1, 8), Fraction(2, 8), Fraction(5, 8)]):
        assert abs(p[i] - float(want)) < 1e-15
        assert abs(o[i] - float(want)) < 1e-15
    assert abs(lse - math.log(8.0)) < 1e-15


# ------------------------------------------------------------------ prefill consistency

def test_prefill_row_equals_decode_of_prefix():
    """Row t of causal prefill equals a one-token decode over the first t+1 tokens."""
    r = _rng(10)
    d = Dims(n_heads=3, d_c=8, d_rope=4, d_nope=5, d_v=6, d_model=8, dtype="f32")
    L = 7
    pool = r.standard_normal((8, d.d_c + d.d_rope))
    bt = np.array([[1, 0]])
    qn, qp = r.standard_normal((L, d.n_heads, d.d_nope)), r.standard_normal((L, d.n_heads, d.d_rope))
    w_uk, w_uv = r.standard_normal((3, 8, 5)), r.standard_normal((3, 8, 6))
    out, lse = oracle.prefill(d, qn, qp, pool, bt, 4, np.array([0, L]), w_uk, w_uv)
    for t in range(L):
        o2, l2 = oracle.decode(d, qn[t][None, None], qp[t][None, None], pool, bt, 4, np.array([t + 1]), w_uk, w_uv)
        np.testing.assert_allclose(out[t], o2[0, 0], rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(lse[t], l2[0, 0], rtol=1e-13)


def test_prefill_matches_library_causal_sdpa():
    r = _rng(11)
    d = Dims(n_heads=2, d_c=8, d_rope=4, d_nope=6, d_v=5, d_model=8, dtype="f32")
    L = 11
    pool = r.standard_normal((L, d.d_c + d.d_rope))
    bt = np.arange(L).reshape(1, L)
    qn, qp = r.standard_normal((L, 2, 6)), r.standard_normal((L, 2, 4))
    w_uk, w_uv = r.standard_normal((2, 8, 6)), r.standard_normal((2, 8, 5))
    out, _ = oracle.prefill(d, qn, qp, pool, bt, 1, np.array([0, L]), w_uk, w_uv)
    for s in range(2):
        K = np.concatenate([pool[:, :8] @ w_uk[s], pool[:, 8:]], axis=1)
        V = pool[:, :8] @ w_uv[s]
        Q = np.concatenate([qn[:, s], O.rope_rotate(qp[:, s], np.arange(L), 10000.0)], axis=1)
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(Q)[None], torch.from_numpy(K)[None], torch.from_numpy(V)[None], is_causal=True)[0]
        np.testing.assert_allclose(out[:, s], ref.numpy(), rtol=1e-12, atol=1e-13)


# ------------------------------------------------------------------ paged gather

def test_paged_gather_equals_contiguous_after_permutation():
    r = _rng(12)
    bs, nblk, W = 4, 6, 3
    cont = r.standard_normal((nblk * bs, W))
    perm = np.array([3, 5, 0, 1, 4, 2])
    pool = np.empty_like(cont)
    for logical, phys in enumerate(perm):
        pool[phys * bs:(phys + 1) * bs] = cont[logical * bs:(logical + 1) * bs]
    got = O.gather_rows(pool, perm.reshape(1, -1), bs, 0, 22)
    np.testing.assert_array_equal(got, cont[:22])


# ------------------------------------------------------------------ planted mistakes

def _assert_some_pin_fails(monkeypatch, target, replacement, tests):
    monkeypatch.setattr(O, target, replacement)
    failed = 0
    for t in tests:
        try:
            t()
        except AssertionError:
            failed += 1
    assert failed > 0, f"no pin caught a planted mistake in {target}"


def test_planted_rope_sign_is_caught(monkeypatch):
    orig = O.rope_rotate

    def wrong(x, positions, base=10000.0, freqs=None):
        return orig(x, -np.asarray(positions, dtype=np.float64), base, freqs)   # rotates the other way
    _assert_some_pin_fails(monkeypatch, "rope_rotate", wrong, [test_rope_worked_example_from_pages])


def test_planted_half_split_pairs_are_caught(monkeypatch):
    orig = O.rope_rotate

    def wrong(x, positions, base=10000.0, freqs=None):
        x = np.asarray(x, dtype=np.float64)
        d = x.shape[-1]
        perm = np.concatenate([np.arange(d // 2), np.arange(d // 2, d)]).reshape(2, -1).T.reshape(-1)
        inv = np.argsort(perm)
        return orig(x[..., perm], positions, base, freqs)[..., inv]           # pairs (i, i + d/2)
    _assert_some_pin_fails(monkeypatch, "rope_rotate", wrong, [test_rope_worked_example_from_pages])


def test_planted_dropped_rope_key_is_caught(monkeypatch):
    orig = O.decompress_head

    def wrong(c, kpe, wuk, wuv):
        K, V = orig(c, kpe, wuk, wuv)
        K[:, wuk.shape[1]:] = 0.0                                            # forget the shared RoPE key
        return K, V
    _assert_some_pin_fails(monkeypatch, "decompress_head", wrong,
                           [test_decode_brute_force_tiny, lambda: test_absorbed_equals_unabsorbed("small_f32")])


def test_planted_causal_off_by_one_is_caught(monkeypatch):
    orig = O.attend

    def wrong(q, K, V, n_visible, scale):
        return orig(q, K, V, min(n_visible + 1, K.shape[0]), scale)          # lets a query see one key too many
    _assert_some_pin_fails(monkeypatch, "attend", wrong,
                           [test_prefill_matches_library_causal_sdpa, test_attend_probabilities_and_one_hot])


def test_planted_wrong_scale_is_caught(monkeypatch):
    orig = O.attend

    def wrong(q, K, V, n_visible, scale):
        return orig(q, K, V, n_visible, scale * 2.0)
    _assert_some_pin_fails(monkeypatch, "attend", wrong, [test_decode_brute_force_tiny])


# ------------------------------------------------------------------ sparse decode over selected tokens

def _sparse_tiny_inputs(seed):
    r = _rng(seed)
    d = TINY
    S, n_q = 6, 2
    pool = r.standard_normal((8, d.d_c + d.d_rope))
    bt = np.array([[3, 1, 2]])       # block size 2: tokens 0,1 -> rows 6,7; 2,3 -> rows 2,3; 4,5 -> rows 4,5
    q_nope = r.standard_normal((1, n_q, d.n_heads, d.d_nope))
    q_pe = r.standard_normal((1, n_q, d.n_heads, d.d_rope))
    w_uk = r.standard_normal((d.n_heads, d.d_c, d.d_nope))
    w_uv = r.standard_normal((d.n_heads, d.d_c, d.d_v))
    return d, S, n_q, pool, bt, q_nope, q_pe, w_uk, w_uv


def test_sparse_decode_brute_force_tiny():
    """Two query tokens at positions 4 and 5, each with its own selection (padding included):
    pure-Python loops over the listed tokens only, RoPE at the query's own position."""
    d, S, n_q, pool, bt, q_nope, q_pe, w_uk, w_uv = _sparse_tiny_inputs(21)
    sel = np.array([[[4, -1, 0, 2], [5, 1, -1, 3]]])
    out, lse = O.decode_sparse(d, q_nope, q_pe, pool, bt, 2, np.array([S]), sel, w_uk, w_uv)
    row_of = {0: 6, 1: 7, 2: 2, 3: 3, 4: 4, 5: 5}
    for j in range(n_q):
        p = S - n_q + j
        toks = [t for t in sel[0, j] if t != -1]
        for s in range(d.n_heads):
            qr = [q_pe[0, j, s, 0] * math.cos(p) - q_pe[0, j, s, 1] * math.sin(p),
                  q_pe[0, j, s, 0] * math.sin(p) + q_pe[0, j, s, 1] * math.cos(p)]
            zs, vs = [], []
            for t in toks:
                row = pool[row_of[t]]
                c = row[:4]
                kn = [sum(c[x] * w_uk[s][x][y] for x in range(4)) for y in range(3)]
                z = sum(q_nope[0, j, s, y] * kn[y] for y in range(3)) + qr[0] * row[4] + qr[1] * row[5]
                zs.append(z / math.sqrt(5))
                vs.append([sum(c[x] * w_uv[s][x][y] for x in range(4)) for y in range(3)])
            den = sum(math.exp(z) for z in zs)
            for y in range(3):
                want = sum(math.exp(zs[i]) * vs[i][y] for i in range(len(toks))) / den
                assert abs(out[0, j, s, y] - want) < 1e-12
            assert abs(lse[0, j, s] - math.log(den)) < 1e-12


def test_sparse_decode_full_selection_is_dense_decode():
    """Selecting every token up to each query's causal limit, in order, is the dense decode."""
    inp = make_decode_inputs(DECODE_CASES["small_f32_nq2"])
    B, n_q, H = inp["q_nope"].shape[:3]
    sl = inp["seqlens"].numpy()
    k = int(sl.max())
    sel = np.full((B, n_q, k), -1, dtype=np.int64)
    for b in range(B):
        for j in range(n_q):
            p = int(sl[b]) - n_q + j
            sel[b, j, :p + 1] = np.arange(p + 1)
    args = (inp["dims"], inp["q_nope"], inp["q_pe"], inp["pool"], inp["block_table"], inp["block_size"], inp["seqlens"])
    o1, l1 = oracle.decode_sparse(*args, sel, inp["w_uk"], inp["w_uv"])
    o2, l2 = oracle.decode(*args, inp["w_uk"], inp["w_uv"])
    np.testing.assert_allclose(o1, o2, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(l1, l2, rtol=1e-12)


def test_sparse_decode_is_a_set_function_and_ignores_padding():
    """Softmax over a set: shuffling the listed tokens and moving the padding changes nothing."""
    d, S, n_q, pool, bt, q_nope, q_pe, w_uk, w_uv = _sparse_tiny_inputs(22)
    a = np.array([[[0, 2, 4, -1, -1], [1, 3, 5, 0, -1]]])
    b = np.array([[[-1, 4, -1, 0, 2], [-1, 5, 0, 3, 1]]])
    o1, l1 = oracle.decode_sparse(d, q_nope, q_pe, pool, bt, 2, np.array([S]), a, w_uk, w_uv)
    o2, l2 = oracle.decode_sparse(d, q_nope, q_pe, pool, bt, 2, np.array([S]), b, w_uk, w_uv)
    np.testing.assert_allclose(o1, o2, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(l1, l2, rtol=1e-13)


def test_sparse_decode_single_token_returns_its_value_row():
    """One listed token: its softmax weight is exactly 1, so the output is that token's
    value c W_UV and the lse is its scaled logit."""
    d, S, n_q, pool, bt, q_nope, q_pe, w_uk, w_uv = _sparse_tiny_inputs(23)
    sel = np.array([[[3], [2]]])
    out, lse = oracle.decode_sparse(d, q_nope, q_pe, pool, bt, 2, np.array([S]), sel, w_uk, w_uv)
    row_of = {2: 2, 3: 3}
    for j, t in ((0, 3), (1, 2)):
        c = pool[row_of[t]][:4]
        for s in range(d.n_heads):
            np.testing.assert_allclose(out[0, j, s], c @ w_uv[s], rtol=1e-13, atol=1e-14)


def test_sparse_decode_rejects_tokens_past_the_causal_limit():
    d, S, n_q, pool, bt, q_nope, q_pe, w_uk, w_uv = _sparse_tiny_inputs(24)
    with pytest.raises(ValueError):
        oracle.decode_sparse(d, q_nope, q_pe, pool, bt, 2, np.array([S]), np.array([[[5], [5]]]), w_uk, w_uv)
    with pytest.raises(ValueError):
        oracle.decode_sparse(d, q_nope, q_pe, pool, bt, 2, np.array([S]), np.array([[[-1], [1]]]), w_uk, w_uv)


def _sparse_variant(mistake):
    """decode_sparse rewritten with one planted mistake: "position" rotates the query by the list
    length instead of its position; "prefix" attends to the first tokens instead of the listed ones."""
    def run(dims, q_nope, q_pe, pool, block_table, block_size, seqlens, topk_idx, w_uk, w_uv, picks=None):
        q_nope, q_pe, pool = np.asarray(q_nope, float), np.asarray(q_pe, float), np.asarray(pool, float)
        B, n_q, H, _ = q_nope.shape
        out = np.full((B, n_q, H, dims.d_v), np.nan)
        lse = np.full((B, n_q, H), np.nan)
        for b in range(B):
            for j in range(n_q):
                listed = [int(i) for i in topk_idx[b, j] if int(i) != -1]
                p = int(seqlens[b]) - n_q + j
                if mistake == "prefix":
                    listed = list(range(len(listed)))
                if mistake == "position":
                    p = len(listed) - 1
                tok = np.asarray(listed)
                rows = np.asarray(block_table)[b, tok // block_size] * block_size + tok % block_size
                for s in range(H):
                    K, V = O.decompress_head(pool[rows, :dims.d_c], pool[rows, dims.d_c:], w_uk[s], w_uv[s])
                    q = np.concatenate([q_nope[b, j, s], O.rope_rotate(q_pe[b, j, s], p, dims.rope_base)])
                    out[b, j, s], lse[b, j, s], _ = O.attend(q, K, V, len(listed),
                                                             1 / math.sqrt(dims.d_nope + dims.d_rope))
        return out, lse
    return run


@pytest.mark.parametrize("mistake", ["position", "prefix"])
def test_planted_sparse_mistakes_are_caught(monkeypatch, mistake):
    _assert_some_pin_fails(monkeypatch, "decode_sparse", _sparse_variant(mistake),
                           [test_sparse_decode_brute_force_tiny])


# ------------------------------------------------------------------ query latent path and output projection

def test_query_from_hidden_brute_force_tiny():
    r = _rng(31)
    D, d_cq, H, d_nope, d_R = 5, 3, 2, 4, 2
    h = r.standard_normal((2, D))
    w_dq, w_uq, w_qr = r.standard_normal((D, d_cq)), r.standard_normal((d_cq, H, d_nope)), r.standard_normal((d_cq, H, d_R))
    qn, qp = oracle.query_from_hidden(h, w_dq, w_uq, w_qr)
    for t in range(2):
        c = [sum(h[t][x] * w_dq[x][y] for x in range(D)) for y in range(d_cq)]
        for s in range(H):
            for k in range(d_nope):
                assert abs(qn[t, s, k] - sum(c[y] * w_uq[y][s][k] for y in range(d_cq))) < 1e-12
            for k in range(d_R):
                assert abs(qp[t, s, k] - sum(c[y] * w_qr[y][s][k] for y in range(d_cq))) < 1e-12


def test_output_projection_brute_force_tiny():
    """u_j = sum over heads s and value dims v of o[s, v] * W_O[s * d_v + v, j]."""
    r = _rng(32)
    H, d_v, D = 3, 2, 4
    o = r.standard_normal((2, H, d_v))
    w_o = r.standard_normal((H * d_v, D))
    u = oracle.output_projection(o, w_o)
    for t in range(2):
        for j in range(D):
            want = sum(o[t, s, v] * w_o[s * d_v + v, j] for s in range(H) for v in range(d_v))
            assert abs(u[t, j] - want) < 1e-12


def _folded_block_output(d, h, w_dq, w_uq, w_qr, pool, bt, bs, seqlens, n_q, w_uk, w_uv, w_o):
    """The decode written with the weights folded offline, in fp64: W_UQK^(s) = W_UQ^(s) W_UK^(s)T
    turns c_Q straight into the latent query; W_UVO^(s) = W_UV^(s) W_O^(s) turns each head's latent
    output straight into its share of u ("DeepSeek-V3 解读 1: MLA", section "为什么需要解耦 RoPE": W^UK
    absorbed into W^Q; "Transformer升级之路：21", section 键值共享: the c -> v map absorbed on the W_o side)."""
    H, d_c, d_v = d.n_heads, d.d_c, d.d_v
    w_uqk = np.einsum("chn,hln->hcl", w_uq, w_uk)                  # [H, d_cq, d_c]
    w_uvo = np.einsum("hlv,hvj->hlj", w_uv, w_o.reshape(H, d_v, -1))  # [H, d_c, D]
    B = h.shape[0]
    u = np.zeros((B, n_q, w_o.shape[1]))
    scale = 1 / math.sqrt(d.d_nope + d.d_rope)
    for b in range(B):
        S = int(seqlens[b])
        rows = bt[b, np.arange(S) // bs] * bs + np.arange(S) % bs
        c, kpe = pool[rows, :d_c], pool[rows, d_c:]
        for j in range(n_q):
            p = S - n_q + j
            c_q = h[b, j] @ w_dq
            for s in range(H):
                q_lat = c_q @ w_uqk[s]
                q_rot = O.rope_rotate(c_q @ w_qr[:, s, :], p, d.rope_base)
                z = (c[:p + 1] @ q_lat + kpe[:p + 1] @ q_rot) * scale
                e = np.exp(z - z.max())
                o_lat = (e / e.sum()) @ c[:p + 1]
                u[b, j] += o_lat @ w_uvo[s]
    return u


def test_folded_weights_equal_the_unfolded_chain():
    """Decode from hidden states with folded weights equals query_from_hidden -> decode (unabsorbed)
    -> output_projection to 1e-12 (two causal query tokens, paged)."""
    r = _rng(33)
    d = Dims(n_heads=3, d_c=8, d_rope=4, d_nope=5, d_v=6, d_model=7, dtype="f32")
    d_cq, n_q, B, bs = 6, 2, 2, 4
    seqlens = np.array([7, 10])
    pool = r.standard_normal((16, d.d_c + d.d_rope))
    bt = np.array([[3, 0, 1], [2, 1, 0]])
    h = r.standard_normal((B, n_q, d.d_model))
    w_dq = r.standard_normal((d.d_model, d_cq))
    w_uq = r.standard_normal((d_cq, d.n_heads, d.d_nope))
    w_qr = r.standard_normal((d_cq, d.n_heads, d.d_rope))
    w_uk = r.standard_normal((d.n_heads, d.d_c, d.d_nope))
    w_uv = r.standard_normal((d.n_heads, d.d_c, d.d_v))
    w_o = r.standard_normal((d.n_heads * d.d_v, d.d_model))
    qn, qp = oracle.query_from_hidden(h, w_dq, w_uq, w_qr)
    out, _ = oracle.decode(d, qn, qp, pool, bt, bs, seqlens, w_uk, w_uv)
    u = oracle.output_projection(out, w_o)
    u2 = _folded_block_output(d, h, w_dq, w_uq, w_qr, pool, bt, bs, seqlens, n_q, w_uk, w_uv, w_o)
    np.testing.assert_allclose(u, u2, rtol=1e-12, atol=1e-12)


def test_planted_output_projection_layout_is_caught(monkeypatch):
    """Concatenating the head outputs dimension-major instead of head-major fails the pin."""
    def wrong(out_heads, w_o):
        o = np.asarray(out_heads, dtype=np.float64)
        return np.swapaxes(o, -1, -2).reshape(o.shape[:-2] + (-1,)) @ np.asarray(w_o, dtype=np.float64)
    monkeypatch.setattr(oracle, "output_projection", wrong)
    with pytest.raises(AssertionError):
        test_output_projection_brute_force_tiny()
