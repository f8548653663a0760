"""Plain fp64 reference for MLA (test infrastructure; see the package docstring).

Sources (the pages this follows, by title and section):

* [SU21] "Transformer升级之路：21、MLA好在哪里?（下）" (spaces.ac.cn/archives/11111),
  section 双重投影, the two-column display: in training/prefill form every head s
  has k_i^(s) = c_i W_k^(s), v_i^(s) = c_i W_v^(s) and
  o_t^(s) = sum_{i<=t} exp(q_t^(s) k_i^(s)T) v_i^(s) / sum_{i<=t} exp(q_t^(s) k_i^(s)T);
  in decoding form W_k is folded into the query and K = V = c.
* [V3-MLA] "DeepSeek-V3 解读 1: MLA" (dtcms.com translation), sections
  "Multi-head Latent Attention" (only the latent c^KV and the RoPE key are
  cached; keys and values are rebuilt by W^UK and W^UV), "为什么需要解耦 RoPE"
  (one extra key shared by all heads carries RoPE; the compressed key is not
  rotated), "RoPE（旋转式位置编码）" (4-d example: consecutive dimension pairs
  are rotated, theta(p) = p * theta_0), and the Figure 1 caption (RMSNorm).
* [MEM] "现代 LLM 的 Memory-Compute Trade-off：从 MHA 到 MLA" (blog.niina.fun),
  section "MHA 与 KV Cache": cache size = 2 x layers x heads x head_dim x bytes
  per token.

Readings where the pages are silent (each is listed with its reason in the
design notes of the repository):

* RoPE frequencies theta_i = base^(-2i/d_R), pair (2i, 2i+1) at position p is
  rotated by p*theta_i with [[cos, -sin], [sin, cos]]; positions are 0-based.
* The softmax scale is 1/sqrt(d_nope + d_R).
* c_KV = gamma * c / sqrt(mean(c^2) + eps) over the d_c latent dims only.
* k_pe = RoPE(h W_KR), one key of width d_R shared by every head.
* Query token j of a sequence whose cache holds S tokens (the n_q new ones
  included) sits at position S - n_q + j and sees keys 0..S - n_q + j.
* lse is the natural-log log-sum-exp of the scaled logits.

Everything is float64 numpy.  Inputs that arrive in bf16 or fp32 are widened
exactly before use.
"""
from __future__ import annotations

import math

import numpy as np


def _f64(x) -> np.ndarray:
    """Widen a numpy array or torch tensor (any float dtype) to float64 exactly."""
    if hasattr(x, "detach"):
        import torch
        x = x.detach().to("cpu")
        if x.dtype in (torch.bfloat16, torch.float16):
            x = x.to(torch.float32)
        x = x.numpy()
    return np.asarray(x, dtype=np.float64)


def _i64(x) -> np.ndarray:
    if hasattr(x, "detach"):
        x = x.detach().to("cpu").numpy()
    return np.asarray(x, dtype=np.int64)


# ---------------------------------------------------------------- RoPE [V3-MLA §RoPE]

def rope_frequencies(d_rope: int, base: float) -> np.ndarray:
    """Per-pair angular frequencies theta_i = base^(-2i/d_rope), i = 0 .. d_rope/2 - 1."""
    assert d_rope % 2 == 0
    i = np.arange(d_rope // 2, dtype=np.float64)
    return np.power(float(base), -2.0 * i / d_rope)


def rope_rotate(x, positions, base: float = 10000.0, freqs=None) -> np.ndarray:
    """Rotate consecutive pairs (x[2i], x[2i+1]) of the last axis by positions * freqs[i].

    x: [..., d]; positions: broadcastable to x.shape[:-1].
    [x'; y'] = [[cos a, -sin a], [sin a, cos a]] [x; y],  a = p * theta_i.
    """
    x = _f64(x)
    d = x.shape[-1]
    if freqs is None:
        freqs = rope_frequencies(d, base)
    freqs = np.asarray(freqs, dtype=np.float64)
    p = np.asarray(_f64(positions), dtype=np.float64)
    ang = p[..., None] * freqs            # [..., d/2]
    c, s = np.cos(ang), np.sin(ang)
    xe, xo = x[..., 0::2], x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = xe * c - xo * s
    out[..., 1::2] = xe * s + xo * c
    return out


# ---------------------------------------------------------------- RMSNorm [V3-MLA Fig. 1]

def rms_norm(c, gamma, eps: float) -> np.ndarray:
    """gamma * c / sqrt(mean(c^2) + eps) over the last axis."""
    c = _f64(c)
    g = _f64(gamma)
    ms = np.mean(c * c, axis=-1, keepdims=True)
    return c / np.sqrt(ms + eps) * g


# ---------------------------------------------------------------- cache append [V3-MLA §MLA 高层次的思路, §解耦 RoPE]

def append_latent(h, w_dkv, w_kr, gamma, pos, eps: float, base: float):
    """Cache rows for new tokens: c_KV = RMSNorm(h W_DKV), k_pe = RoPE(h W_KR, pos).

    h [T, D], w_dkv [D, d_c], w_kr [D, d_R], gamma [d_c], pos [T].
    Returns (c_kv [T, d_c], k_pe [T, d_R]) in float64.
    """
    h = _f64(h)
    c = h @ _f64(w_dkv)
    k = h @ _f64(w_kr)
    return rms_norm(c, gamma, eps), rope_rotate(k, _i64(pos), base)


# ---------------------------------------------------------------- paged gather

def gather_rows(pool, block_table, block_size: int, b: int, n_tokens: int) -> np.ndarray:
    """Rows of tokens 0..n_tokens-1 of sequence b: token i lives in pool row
    block_table[b][i // block_size] * block_size + i % block_size."""
    bt = _i64(block_table)
    i = np.arange(n_tokens, dtype=np.int64)
    rows = bt[b, i // block_size] * block_size + (i % block_size)
    if hasattr(pool, "detach"):
        import torch
        return _f64(pool[torch.from_numpy(rows)])
    return _f64(np.asarray(pool)[rows])


# ---------------------------------------------------------------- decompression [SU21 §双重投影, left column]

def decompress_head(c_kv_seq, k_pe_seq, w_uk_h, w_uv_h):
    """Per-head key and value of every cached token.

    k_i = [c_i W_UK^(s) | kpe_i]   (d_nope + d_R; kpe_i is already rotated in the cache)
    v_i = c_i W_UV^(s)             (d_v)
    """
    c = _f64(c_kv_seq)
    K = np.concatenate([c @ _f64(w_uk_h), _f64(k_pe_seq)], axis=-1)
    V = c @ _f64(w_uv_h)
    return K, V


def attend(q, K, V, n_visible: int, scale: float):
    """Naive softmax attention of one query over keys 0..n_visible-1.

    Returns (o [d_v], lse, p [n_visible]) with z_i = scale * q.k_i,
    p = exp(z - max z) / sum exp(z - max z), lse = ln sum exp(z_i).
    """
    q = _f64(q)
    z = (K[:n_visible] @ q) * scale
    m = np.max(z)
    e = np.exp(z - m)
    den = np.sum(e)
    p = e / den
    o = p @ V[:n_visible]
    return o, m + math.log(den), p


# ---------------------------------------------------------------- decode (unabsorbed form)

def decode_one(dims, b: int, j: int, s: int, q_nope, q_pe, c_seq, kpe_seq, seqlen: int, n_q: int,
               w_uk, w_uv, K=None, V=None):
    """One output row (sequence b, query token j, head s) of a decode step.

    c_seq / kpe_seq: the sequence's cached rows (float64).  K, V may be passed in
    when the caller already decompressed head s for this sequence.
    """
    if K is None:
        K, V = decompress_head(c_seq, kpe_seq, _f64(w_uk[s]), _f64(w_uv[s]))
    p_j = seqlen - n_q + j
    q = np.concatenate([_f64(q_nope[b, j, s]), rope_rotate(_f64(q_pe[b, j, s]), p_j, dims.rope_base)])
    scale = 1.0 / math.sqrt(dims.d_nope + dims.d_rope)
    o, lse, _ = attend(q, K, V, p_j + 1, scale)
    return o, lse


def decode(dims, q_nope, q_pe, pool, block_table, block_size: int, seqlens, w_uk, w_uv,
           picks=None):
    """Decode step in unabsorbed form.

    pool [rows, d_c + d_R] holds c_KV in columns [0, d_c) and the rotated k_pe in
    [d_c, d_c + d_R).  q_nope [B, n_q, H, d_nope], q_pe [B, n_q, H, d_R] (not yet
    rotated).  Returns (out [B, n_q, H, d_v], lse [B, n_q, H]) as float64; with
    ``picks`` = list of (b, j, s) only those entries are computed (the rest NaN).
    """
    q_nope = _f64(q_nope)
    q_pe = _f64(q_pe)
    w_uk = _f64(w_uk)
    w_uv = _f64(w_uv)
    sl = _i64(seqlens)
    B, n_q, H, _ = q_nope.shape
    out = np.full((B, n_q, H, dims.d_v), np.nan)
    lse = np.full((B, n_q, H), np.nan)
    if picks is None:
        picks = [(b, j, s) for b in range(B) for s in range(H) for j in range(n_q)]
    by_seq = {}
    for (b, j, s) in picks:
        by_seq.setdefault(b, []).append((j, s))
    for b, items in by_seq.items():
        S = int(sl[b])
        rows = gather_rows(pool, block_table, block_size, b, S)
        c_seq, kpe_seq = rows[:, :dims.d_c], rows[:, dims.d_c:dims.d_c + dims.d_rope]
        by_head = {}
        for (j, s) in items:
            by_head.setdefault(s, []).append(j)
        for s, js in by_head.items():
            K, V = decompress_head(c_seq, kpe_seq, w_uk[s], w_uv[s])
            for j in js:
                out[b, j, s], lse[b, j, s] = decode_one(dims, b, j, s, q_nope, q_pe, c_seq, kpe_seq, S, n_q,
                                                         w_uk, w_uv, K, V)
    return out, lse


# ---------------------------------------------------------------- query latent path and output projection

def query_from_hidden(h, w_dq, w_uq, w_qr):
    """Queries from the compressed query latent ("DeepSeek-V3 解读 1: MLA", section "MLA：高层次的思路":
    queries too are projected into a low-dimensional latent space and restored from it; section
    "为什么需要解耦 RoPE": an extra RoPE query per head, taken from the same latent).

    c_Q = h W_DQ;  q_nope^(s) = c_Q W_UQ^(s);  q_pe^(s) = c_Q W_QR^(s) (not rotated: the decode
    rotates it at the query's position).
    h [..., D], w_dq [D, d_cq], w_uq [d_cq, H, d_nope], w_qr [d_cq, H, d_R].
    Returns (q_nope [..., H, d_nope], q_pe [..., H, d_R]) in float64.
    """
    c_q = _f64(h) @ _f64(w_dq)
    q_nope = np.einsum("...c,chd->...hd", c_q, _f64(w_uq))
    q_pe = np.einsum("...c,chd->...hd", c_q, _f64(w_qr))
    return q_nope, q_pe


def output_projection(out_heads, w_o):
    """The attention block's output u = [o^(1), ..., o^(H)] W^O ("DeepSeek-V3 解读 1: MLA": W^O maps the
    concatenated head outputs, n_h d_h wide, back to the model width d).
    out_heads [..., H, d_v], w_o [H d_v, D] -> [..., D] in float64."""
    o = _f64(out_heads)
    return o.reshape(o.shape[:-2] + (-1,)) @ _f64(w_o)


# ---------------------------------------------------------------- sparse decode over selected tokens

def decode_sparse(dims, q_nope, q_pe, pool, block_table, block_size: int, seqlens, topk_idx, w_uk, w_uv,
                  picks=None):
    """Decode step in unabsorbed form over a selected subset of each query token's cached tokens.

    The MQA-mode MLA of V3.2 (developer.cloud.tencent.com search results for
    "MLA", the snippet "MHA版MLA VS MQA版MLA": every head attends to the one
    shared latent key/value) restricted, for query token j of sequence b, to
    the cached tokens listed in topk_idx[b, j, :].  Entries equal to -1 are
    padding; every other entry is a token index in 0 .. S_b - n_q + j (the
    causal limit of that query token).  The listed tokens are attended to as
    listed: z_i = scale * q . k_i over the list, softmax over the list,
    output sum_i p_i v_i, per head, with keys and values decompressed from the
    cache exactly as in ``decode``.

    topk_idx [B, n_q, k] (int).  Returns (out [B, n_q, H, d_v], lse [B, n_q, H])
    as float64; with ``picks`` = list of (b, j, s) only those entries are computed.
    """
    q_nope = _f64(q_nope)
    q_pe = _f64(q_pe)
    w_uk = _f64(w_uk)
    w_uv = _f64(w_uv)
    sl = _i64(seqlens)
    idx = _i64(topk_idx)
    bt = _i64(block_table)
    B, n_q, H, _ = q_nope.shape
    out = np.full((B, n_q, H, dims.d_v), np.nan)
    lse = np.full((B, n_q, H), np.nan)
    if picks is None:
        picks = [(b, j, s) for b in range(B) for s in range(H) for j in range(n_q)]
    scale = 1.0 / math.sqrt(dims.d_nope + dims.d_rope)
    for (b, j, s) in picks:
        p_j = int(sl[b]) - n_q + j
        listed = [int(i) for i in idx[b, j] if int(i) != -1]
        if not listed or min(listed) < 0 or max(listed) > p_j:
            raise ValueError(f"selection of ({b}, {j}) must be non-empty and within 0..{p_j}")
        tok = np.asarray(listed, dtype=np.int64)
        rows = bt[b, tok // block_size] * block_size + tok % block_size
        if hasattr(pool, "detach"):
            import torch
            sel = _f64(pool[torch.from_numpy(rows)])
        else:
            sel = _f64(np.asarray(pool)[rows])
        K, V = decompress_head(sel[:, :dims.d_c], sel[:, dims.d_c:dims.d_c + dims.d_rope], w_uk[s], w_uv[s])
        q = np.concatenate([q_nope[b, j, s], rope_rotate(q_pe[b, j, s], p_j, dims.rope_base)])
        out[b, j, s], lse[b, j, s], _ = attend(q, K, V, len(listed), scale)
    return out, lse


# ---------------------------------------------------------------- prefill (decompressed MHA form)

def prefill(dims, q_nope, q_pe, pool, block_table, block_size: int, cu_seqlens, w_uk, w_uv,
            rows_pick=None):
    """Causal prefill in decompressed MHA form [SU21 §双重投影 left column].

    q_nope [total, H, d_nope], q_pe [total, H, d_R] (not yet rotated; token t of a
    sequence is at position t).  The cache holds every token of every sequence.
    Returns (out [total, H, d_v], lse [total, H]); with rows_pick (a set of global
    row indices) only those rows are computed.
    """
    q_nope = _f64(q_nope)
    q_pe = _f64(q_pe)
    w_uk = _f64(w_uk)
    w_uv = _f64(w_uv)
    cu = _i64(cu_seqlens)
    total, H, _ = q_nope.shape
    out = np.full((total, H, dims.d_v), np.nan)
    lse = np.full((total, H), np.nan)
    scale = 1.0 / math.sqrt(dims.d_nope + dims.d_rope)
    for b in range(len(cu) - 1):
        start, L = int(cu[b]), int(cu[b + 1] - cu[b])
        ts = [t for t in range(L) if rows_pick is None or (start + t) in rows_pick]
        if not ts:
            continue
        rows = gather_rows(pool, block_table, block_size, b, L)
        c_seq, kpe_seq = rows[:, :dims.d_c], rows[:, dims.d_c:dims.d_c + dims.d_rope]
        for s in range(H):
            K, V = decompress_head(c_seq, kpe_seq, w_uk[s], w_uv[s])
            for t in ts:
                q = np.concatenate([q_nope[start + t, s], rope_rotate(q_pe[start + t, s], t, dims.rope_base)])
                out[start + t, s], lse[start + t, s], _ = attend(q, K, V, t + 1, scale)
    return out, lse


# ---------------------------------------------------------------- cache accounting [MEM §MHA 与 KV Cache]

def kv_cache_bytes_mha(layers: int, heads: int, head_dim: int, tokens: int, bytes_per_elem: int) -> int:
    """Per-token K and V of every head in every layer: 2 * L * h * d_h * N * bytes."""
    return 2 * layers * heads * head_dim * tokens * bytes_per_elem


def latent_elems_per_token(d_c: int, d_rope: int) -> int:
    """MLA caches only c_KV (d_c) and the shared RoPE key (d_R) per token per layer."""
    return d_c + d_rope
