"""Seeded synthetic workloads for MLA latent-KV decode and prefill.

This module only draws random numbers and builds index structures (block
tables, sequence lengths, NaN sentinels).  It holds none of the method's
arithmetic, so both the fp64 oracle and the CUDA library can consume its
output without sharing any computation.

Shapes follow the DeepSeek-V2-Lite / DeepSeek-V3 attention dimensions used
by the workloads below (latent width d_c, shared RoPE key width d_R, per-head
no-RoPE width d_nope, value width d_v).  Values are N(0,1)/sqrt(fan_in) for
weights and N(0,1) for activations and cache rows, drawn from a CPU
``torch.Generator`` so every run with the same seed sees the same bits.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

__all__ = [
    "Dims", "DecodeCase", "PrefillCase", "DECODE_CASES", "PREFILL_CASES",
    "make_decode_inputs", "make_prefill_inputs", "make_append_inputs",
    "cache_row_of", "latent_bytes", "decode_flops", "prefill_flops", "make_decode_step_inputs", "append_flops",
    "make_decode_inputs_device", "make_query_path_inputs",
]


@dataclasses.dataclass(frozen=True)
class Dims:
    n_heads: int
    d_c: int
    d_rope: int
    d_nope: int
    d_v: int
    d_model: int
    dtype: str = "bf16"          # "bf16" or "f32": element type of every float tensor
    rope_base: float = 10000.0
    rms_eps: float = 1e-6

    @property
    def latent_width(self) -> int:
        """Elements cached per token per layer: the latent plus the shared RoPE key."""
        return self.d_c + self.d_rope

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    @property
    def elem_bytes(self) -> int:
        return 2 if self.dtype == "bf16" else 4


V2_LITE = dict(n_heads=16, d_c=512, d_rope=64, d_nope=128, d_v=128, d_model=2048)
V3 = dict(n_heads=128, d_c=512, d_rope=64, d_nope=128, d_v=128, d_model=7168)


@dataclasses.dataclass(frozen=True)
class DecodeCase:
    name: str
    dims: Dims
    batch: int
    n_q: int
    seqlens: tuple            # ("uniform", S) or ("range", lo, hi) or ("list", (...))
    block_size: int
    paged: bool               # False: identity block table (contiguous rows per sequence)
    seed: int

    def draw_seqlens(self, gen: torch.Generator) -> torch.Tensor:
        kind = self.seqlens[0]
        if kind == "uniform":
            return torch.full((self.batch,), int(self.seqlens[1]), dtype=torch.int32)
        if kind == "range":
            lo, hi = int(self.seqlens[1]), int(self.seqlens[2])
            return torch.randint(lo, hi + 1, (self.batch,), generator=gen, dtype=torch.int64).to(torch.int32)
        if kind == "list":
            vals = list(self.seqlens[1])
            assert len(vals) == self.batch
            return torch.tensor(vals, dtype=torch.int32)
        raise ValueError(kind)


@dataclasses.dataclass(frozen=True)
class PrefillCase:
    name: str
    dims: Dims
    seqlens: tuple            # tokens per sequence
    block_size: int
    paged: bool
    seed: int


# The five workloads, plus smaller cases that the oracle finishes in seconds.
DECODE_CASES = {
    # Tiny fp32: batch 1, 8 heads, d_c 64, d_R 16, d_nope 32, d_v 32, d_model 256, seqlen 256, contiguous.
    "tiny_fp32": DecodeCase("tiny_fp32", Dims(8, 64, 16, 32, 32, 256, "f32"), 1, 1, ("uniform", 256), 64, False, 1001),
    # V2-Lite-shaped: batch 32, 16 heads, seqlen 2048, page 64, permuted block table.
    "v2lite_bf16": DecodeCase("v2lite_bf16", Dims(**V2_LITE), 32, 1, ("uniform", 2048), 64, True, 1002),
    # V3-shaped: batch 64, 128 heads, seqlen 4096, page 64, permuted block table.
    "v3_bf16": DecodeCase("v3_bf16", Dims(**V3), 64, 1, ("uniform", 4096), 64, True, 1003),
    # V3-shaped ragged: batch 128, seqlens uniform in [512, 32768], 2 query tokens, page 64.
    "v3_ragged_bf16": DecodeCase("v3_ragged_bf16", Dims(**V3), 128, 2, ("range", 512, 32768), 64, True, 1004),
    # V3-shaped long: batch 4 at 131072, 2 query tokens, page 64.
    "v3_long_bf16": DecodeCase("v3_long_bf16", Dims(**V3), 4, 2, ("uniform", 131072), 64, True, 1014),
    # Small parity cases: several tiles, ragged tails, partially filled last pages.
    "small_f32": DecodeCase("small_f32", Dims(8, 64, 16, 32, 32, 256, "f32"), 3, 1, ("list", (1, 77, 300)), 16, True, 2001),
    "small_f32_nq2": DecodeCase("small_f32_nq2", Dims(8, 64, 16, 32, 32, 256, "f32"), 3, 2, ("list", (2, 65, 130)), 16, True, 2002),
    "small_v3_bf16": DecodeCase("small_v3_bf16", Dims(**V3), 3, 1, ("list", (1, 200, 700)), 64, True, 2003),
    "small_v3_nq2_bf16": DecodeCase("small_v3_nq2_bf16", Dims(**V3), 4, 2, ("list", (2, 64, 129, 1000)), 64, True, 2004),
    "small_v2lite_bf16": DecodeCase("small_v2lite_bf16", Dims(**V2_LITE), 5, 1, ("list", (63, 64, 65, 511, 2048)), 64, True, 2005),
    "small_v3_contig_bf16": DecodeCase("small_v3_contig_bf16", Dims(**V3), 2, 1, ("list", (300, 1024)), 64, False, 2006),
    # 128-token blocks (two 64-token pages per block in the tiled pool).
    "small_v3_b128_bf16": DecodeCase("small_v3_b128_bf16", Dims(**V3), 3, 1, ("list", (100, 128, 513)), 128, True, 2007),
    # Many short units: clusters cross unit boundaries, page boundaries at every offset class.
    "small_v3_many_bf16": DecodeCase("small_v3_many_bf16", Dims(**V3), 24, 1,
                                     ("list", (1, 5, 64, 65, 127, 128, 129, 200, 255, 256, 257, 300, 383, 384, 385,
                                               448, 511, 512, 513, 600, 640, 700, 768, 1000)), 64, True, 2008),
}

PREFILL_CASES = {
    # V3-shaped causal prefill: batch 2 x 8192 tokens, 128 heads.
    "v3_prefill_bf16": PrefillCase("v3_prefill_bf16", Dims(**V3), (8192, 8192), 64, True, 1005),
    "small_prefill_f32": PrefillCase("small_prefill_f32", Dims(8, 64, 16, 32, 32, 256, "f32"), (5, 70), 16, True, 2101),
    "small_prefill_bf16": PrefillCase("small_prefill_bf16", Dims(**V3), (1, 130, 257), 64, True, 2102),
}


def _randn(gen: torch.Generator, shape, scale: float = 1.0) -> torch.Tensor:
    t = torch.randn(*shape, generator=gen, dtype=torch.float32)
    if scale != 1.0:
        t.mul_(scale)
    return t


def _block_table(gen: torch.Generator, seqlens: torch.Tensor, block_size: int, paged: bool,
                 spare_blocks: int = 0):
    """Block table [B, max_blocks] and the pool size.

    Paged: every block id in [0, num_blocks) is used at most once, in a seeded
    random permutation, plus ``spare_blocks`` never referenced.  Contiguous:
    sequence b owns blocks b*max_blocks ... (b+1)*max_blocks-1 in order.
    """
    B = seqlens.numel()
    need = [(int(s) + block_size - 1) // block_size for s in seqlens.tolist()]
    mbps = max(need) if need else 1
    if not paged:
        num_blocks = B * mbps
        bt = torch.arange(num_blocks, dtype=torch.int32).reshape(B, mbps)
        return bt, num_blocks, mbps
    used = sum(need)
    num_blocks = used + spare_blocks
    perm = torch.randperm(num_blocks, generator=gen).to(torch.int32)
    bt = torch.full((B, mbps), -1, dtype=torch.int32)
    k = 0
    for b, n in enumerate(need):
        bt[b, :n] = perm[k:k + n]
        k += n
    return bt, num_blocks, mbps


def cache_row_of(block_table: torch.Tensor, block_size: int, b: int, i: int) -> int:
    """Pool row that holds token i of sequence b."""
    return int(block_table[b, i // block_size]) * block_size + (i % block_size)


def make_decode_inputs(case: DecodeCase, fill: str = "random", nan_sentinel: bool = True) -> dict:
    """CPU tensors for one decode step.

    fill="random": cache rows c_KV ~ N(0,1), k_pe ~ N(0,1) (unit RMS, like a
    normalised latent).  Unused pool rows hold NaN so a kernel that reads past a
    sequence's end poisons its output.
    """
    d = case.dims
    gen = torch.Generator().manual_seed(case.seed)
    seqlens = case.draw_seqlens(gen)
    assert int(seqlens.min()) >= case.n_q
    bt, num_blocks, mbps = _block_table(gen, seqlens, case.block_size, case.paged, spare_blocks=2 if case.paged else 0)
    W = d.latent_width
    dt = d.torch_dtype
    pool = torch.full((num_blocks * case.block_size, W), float("nan") if nan_sentinel else 0.0, dtype=dt)
    if fill == "random":
        for b in range(case.batch):
            S = int(seqlens[b])
            rows = _rows_of(bt, case.block_size, b, S)
            pool[rows] = _randn(gen, (S, W)).to(dt)
    else:
        raise ValueError(fill)
    q_nope = _randn(gen, (case.batch, case.n_q, d.n_heads, d.d_nope)).to(dt)
    q_pe = _randn(gen, (case.batch, case.n_q, d.n_heads, d.d_rope)).to(dt)
    w_uk = _randn(gen, (d.n_heads, d.d_c, d.d_nope), 1.0 / math.sqrt(d.d_c)).to(dt)
    w_uv = _randn(gen, (d.n_heads, d.d_c, d.d_v), 1.0 / math.sqrt(d.d_c)).to(dt)
    return dict(case=case, dims=d, seqlens=seqlens, block_table=bt, num_blocks=num_blocks,
                max_blocks_per_seq=mbps, block_size=case.block_size, pool=pool,
                q_nope=q_nope, q_pe=q_pe, w_uk=w_uk, w_uv=w_uv)


def _rows_of(bt: torch.Tensor, block_size: int, b: int, S: int) -> torch.Tensor:
    i = torch.arange(S, dtype=torch.int64)
    return bt[b, (i // block_size)].to(torch.int64) * block_size + (i % block_size)


def make_append_inputs(dims: Dims, T: int, seqlens: torch.Tensor, block_size: int, paged: bool,
                       seed: int, gamma_random: bool = True, tokens: Optional[list] = None) -> dict:
    """Hidden states h [T, D], projection weights and the (sequence, position) of each new token.

    ``tokens`` lists (seq, pos) pairs; by default the last T positions of the
    sequences are spread round-robin (the tokens a decode step appends).
    """
    gen = torch.Generator().manual_seed(seed)
    bt, num_blocks, mbps = _block_table(gen, seqlens, block_size, paged, spare_blocks=1 if paged else 0)
    dt = dims.torch_dtype
    h = _randn(gen, (T, dims.d_model)).to(dt)
    w_dkv = _randn(gen, (dims.d_model, dims.d_c), 1.0 / math.sqrt(dims.d_model)).to(dt)
    w_kr = _randn(gen, (dims.d_model, dims.d_rope), 1.0 / math.sqrt(dims.d_model)).to(dt)
    if gamma_random:
        gamma = (1.0 + 0.5 * _randn(gen, (dims.d_c,))).to(dt)
    else:
        gamma = torch.ones(dims.d_c).to(dt)
    if tokens is None:
        tokens = []
        B = seqlens.numel()
        per = [0] * B
        b = 0
        while len(tokens) < T:
            S = int(seqlens[b])
            if per[b] < S:
                tokens.append((b, S - 1 - per[b]))
                per[b] += 1
            b = (b + 1) % B
    seq_idx = torch.tensor([t[0] for t in tokens], dtype=torch.int32)
    pos = torch.tensor([t[1] for t in tokens], dtype=torch.int32)
    return dict(dims=dims, h=h, w_dkv=w_dkv, w_kr=w_kr, gamma=gamma, seq_idx=seq_idx, pos=pos,
                block_table=bt, num_blocks=num_blocks, max_blocks_per_seq=mbps, block_size=block_size,
                seqlens=seqlens)


def make_prefill_inputs(case: PrefillCase) -> dict:
    """Hidden states for every token of every sequence, plus queries and weights.

    The cache for prefill is built from h by the append step (c_KV =
    RMSNorm(h W_DKV), k_pe = RoPE(h W_KR)); this function returns h and the
    weights, not the cache.
    """
    d = case.dims
    gen = torch.Generator().manual_seed(case.seed)
    seqlens = torch.tensor(case.seqlens, dtype=torch.int32)
    total = int(seqlens.sum())
    cu = torch.zeros(len(case.seqlens) + 1, dtype=torch.int32)
    cu[1:] = torch.cumsum(seqlens, 0)
    bt, num_blocks, mbps = _block_table(gen, seqlens, case.block_size, case.paged, spare_blocks=1 if case.paged else 0)
    dt = d.torch_dtype
    h = _randn(gen, (total, d.d_model)).to(dt)
    w_dkv = _randn(gen, (d.d_model, d.d_c), 1.0 / math.sqrt(d.d_model)).to(dt)
    w_kr = _randn(gen, (d.d_model, d.d_rope), 1.0 / math.sqrt(d.d_model)).to(dt)
    gamma = torch.ones(d.d_c).to(dt)
    q_nope = _randn(gen, (total, d.n_heads, d.d_nope)).to(dt)
    q_pe = _randn(gen, (total, d.n_heads, d.d_rope)).to(dt)
    w_uk = _randn(gen, (d.n_heads, d.d_c, d.d_nope), 1.0 / math.sqrt(d.d_c)).to(dt)
    w_uv = _randn(gen, (d.n_heads, d.d_c, d.d_v), 1.0 / math.sqrt(d.d_c)).to(dt)
    seq_idx = torch.repeat_interleave(torch.arange(len(case.seqlens), dtype=torch.int32), seqlens.to(torch.int64))
    pos = torch.cat([torch.arange(int(s), dtype=torch.int32) for s in case.seqlens])
    return dict(case=case, dims=d, seqlens=seqlens, cu_seqlens=cu, block_table=bt, num_blocks=num_blocks,
                max_blocks_per_seq=mbps, block_size=case.block_size, h=h, w_dkv=w_dkv, w_kr=w_kr,
                gamma=gamma, q_nope=q_nope, q_pe=q_pe, w_uk=w_uk, w_uv=w_uv, seq_idx=seq_idx, pos=pos)


# ---- algorithmic work accounting (what a roofline divides by) ----

def latent_bytes(dims: Dims, seqlens) -> int:
    """Bytes of latent cache a decode step must read: one (d_c + d_R)-wide row per cached token."""
    total = int(sum(int(s) for s in seqlens))
    return total * dims.latent_width * dims.elem_bytes


def decode_flops(dims: Dims, seqlens, n_q: int) -> dict:
    """FLOPs of one absorbed-form decode step, split by stage.

    attention: per (query token, visible key, head) 2(d_c+d_R) for the score and
    2 d_c for P*c_KV; query token j of a sequence of length S sees S-n_q+j+1 keys.
    absorb: 2 d_nope d_c per (query token, head).  up: 2 d_c d_v per (query token, head).
    """
    H = dims.n_heads
    vis = 0
    for s in seqlens:
        s = int(s)
        for j in range(n_q):
            vis += s - n_q + j + 1
    att = vis * H * (2 * (dims.d_c + dims.d_rope) + 2 * dims.d_c)
    nq_tot = len(list(seqlens)) * n_q
    absorb = nq_tot * H * 2 * dims.d_nope * dims.d_c
    up = nq_tot * H * 2 * dims.d_c * dims.d_v
    return dict(attention=att, absorb=absorb, up=up, total=att + absorb + up)


def prefill_flops(dims: Dims, seqlens) -> dict:
    """FLOPs of causal prefill in decompressed form: QK over d_nope+d_R, PV over d_v,
    counted on the causal triangle (row t sees t+1 keys); plus the per-head K/V decompression."""
    H = dims.n_heads
    vis = sum(int(s) * (int(s) + 1) // 2 for s in seqlens)
    att = vis * H * 2 * (dims.d_nope + dims.d_rope + dims.d_v)
    tok = sum(int(s) for s in seqlens)
    decomp = tok * H * 2 * dims.d_c * (dims.d_nope + dims.d_v)
    return dict(attention=att, decompress=decomp, total=att + decomp)


def make_decode_step_inputs(case: DecodeCase, fill: str = "random") -> dict:
    """Decode inputs plus the append of this step's new tokens.

    The n_q newest tokens of every sequence (positions S_b - n_q .. S_b - 1) get
    hidden states h [B*n_q, D] and are appended through the same block table
    before attention; weights W_DKV, W_KR ~ N(0,1)/sqrt(D), gamma = 1.
    """
    inp = make_decode_inputs(case, fill=fill)
    d = case.dims
    gen = torch.Generator().manual_seed(case.seed + 500)
    dt = d.torch_dtype
    T = case.batch * case.n_q
    inp["h_new"] = _randn(gen, (T, d.d_model)).to(dt)
    inp["w_dkv"] = _randn(gen, (d.d_model, d.d_c), 1.0 / math.sqrt(d.d_model)).to(dt)
    inp["w_kr"] = _randn(gen, (d.d_model, d.d_rope), 1.0 / math.sqrt(d.d_model)).to(dt)
    inp["gamma"] = torch.ones(d.d_c).to(dt)
    sl = inp["seqlens"].to(torch.int64)
    inp["seq_idx"] = torch.arange(case.batch, dtype=torch.int32).repeat_interleave(case.n_q)
    inp["pos"] = (sl.repeat_interleave(case.n_q) - case.n_q
                  + torch.arange(case.n_q).repeat(case.batch)).to(torch.int32)
    return inp


def append_flops(dims: Dims, T: int) -> int:
    """FLOPs of appending T tokens: the [T, D] x [D, d_c + d_R] projection."""
    return 2 * T * dims.d_model * (dims.d_c + dims.d_rope)


def make_decode_inputs_device(case: DecodeCase, device="cuda") -> dict:
    """The inputs of ``make_decode_inputs`` for timing runs at full size, drawn on the device.

    Sequence lengths and the block table come from the same CPU generator and
    seed as ``make_decode_inputs`` (the same structure); the values (cache rows,
    queries, weights) come from a device generator seeded with the case seed, so
    they are not the CPU draws' bits but follow the same distributions.  Unused
    pool rows hold NaN.
    """
    d = case.dims
    gen = torch.Generator().manual_seed(case.seed)
    seqlens = case.draw_seqlens(gen)
    bt, num_blocks, mbps = _block_table(gen, seqlens, case.block_size, case.paged, spare_blocks=2 if case.paged else 0)
    W = d.latent_width
    dt = d.torch_dtype
    g = torch.Generator(device=device).manual_seed(case.seed)
    pool = torch.full((num_blocks * case.block_size, W), float("nan"), dtype=dt, device=device)
    rows = torch.cat([_rows_of(bt, case.block_size, b, int(seqlens[b])) for b in range(case.batch)]).to(device)
    pool[rows] = torch.randn(rows.numel(), W, generator=g, device=device).to(dt)
    q_nope = torch.randn(case.batch, case.n_q, d.n_heads, d.d_nope, generator=g, device=device).to(dt)
    q_pe = torch.randn(case.batch, case.n_q, d.n_heads, d.d_rope, generator=g, device=device).to(dt)
    w_uk = (torch.randn(d.n_heads, d.d_c, d.d_nope, generator=g, device=device) / math.sqrt(d.d_c)).to(dt)
    w_uv = (torch.randn(d.n_heads, d.d_c, d.d_v, generator=g, device=device) / math.sqrt(d.d_c)).to(dt)
    return dict(case=case, dims=d, seqlens=seqlens, block_table=bt, num_blocks=num_blocks,
                max_blocks_per_seq=mbps, block_size=case.block_size, pool=pool,
                q_nope=q_nope, q_pe=q_pe, w_uk=w_uk, w_uv=w_uv)


def make_query_path_inputs(case: DecodeCase, d_cq: int, seed: int) -> dict:
    """Hidden states and the query-side and output weights of the attention block, for the decode from
    hidden states: h [B, n_q, D] ~ N(0,1); W_DQ [D, d_cq], W_UQ [d_cq, H, d_nope], W_QR [d_cq, H, d_R]
    and W^O [H d_v, D], each ~ N(0,1)/sqrt(fan_in)."""
    d = case.dims
    gen = torch.Generator().manual_seed(seed)
    dt = d.torch_dtype
    return dict(
        h=_randn(gen, (case.batch, case.n_q, d.d_model)).to(dt),
        w_dq=_randn(gen, (d.d_model, d_cq), 1.0 / math.sqrt(d.d_model)).to(dt),
        w_uq=_randn(gen, (d_cq, d.n_heads, d.d_nope), 1.0 / math.sqrt(d_cq)).to(dt),
        w_qr=_randn(gen, (d_cq, d.n_heads, d.d_rope), 1.0 / math.sqrt(d_cq)).to(dt),
        w_o=_randn(gen, (d.n_heads * d.d_v, d.d_model), 1.0 / math.sqrt(d.n_heads * d.d_v)).to(dt),
    )
