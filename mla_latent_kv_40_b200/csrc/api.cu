// C-ABI entry points of libmla: argument validation, workspace carving and
// kernel dispatch.  Every step of every call runs in this library's kernels;
// there is no host-side compute and no CPU fallback.
#include <cuda_runtime.h>

#include "decode_tc.cuh"
#include "kernels.cuh"

using namespace mla;

namespace {

constexpr int kSimtChunk = 1024;   // keys per split in the CUDA-core decode path

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

bool dims_ok(const mla_dims *d) {
  if (!d) return false;
  if (d->n_heads <= 0 || d->d_c <= 0 || d->d_rope < 0 || (d->d_rope & 1) || d->d_nope <= 0 ||
      d->d_v <= 0 || d->block_size <= 0)
    return false;
  if (d->cache_layout == MLA_CACHE_TILED) {
    // Tiled pages: bf16, 64-token pages inside blocks, rows a whole number of 64-dim chunks.
    if (d->dtype != MLA_BF16 || d->block_size % 64 != 0 || (d->d_c + d->d_rope) % 64 != 0) return false;
  } else if (d->cache_layout == MLA_CACHE_ROWS) {
    if (d->ckv_stride < d->d_c || d->kpe_stride < d->d_rope) return false;
  } else {
    return false;
  }
  if (d->dtype != MLA_F32 && d->dtype != MLA_BF16) return false;
  if (!(d->rope_base > 0.f)) return false;
  return true;
}

size_t elem(const mla_dims *d) { return d->dtype == MLA_BF16 ? 2 : 4; }

struct DecodeLayout {
  size_t q_off, o_off, lse_off, tc_off, total;
  int max_chunks;
  bool use_tc;
};

DecodeLayout decode_layout(const mla_dims *d, int B, int n_q, int max_seqlen) {
  DecodeLayout L{};
  const size_t W = (size_t)d->d_c + d->d_rope;
  const size_t R = (size_t)n_q * d->n_heads;
  L.use_tc = tc_decode_supported(*d, n_q);
  L.q_off = 0;
  size_t off = align256((size_t)B * R * W * elem(d));
  if (L.use_tc) {
    L.max_chunks = 0;
    L.o_off = L.lse_off = off;
    L.tc_off = off;
    off += align256(tc_decode_workspace_bytes(*d, B, n_q));
  } else {
    L.max_chunks = (max_seqlen + kSimtChunk - 1) / kSimtChunk;
    L.o_off = off;
    off += align256((size_t)B * L.max_chunks * R * d->d_c * sizeof(float));
    L.lse_off = off;
    off += align256((size_t)B * L.max_chunks * R * sizeof(float));
    L.tc_off = off;
  }
  L.total = off;
  return L;
}

int check_decode_args(const mla_dims *dims, int B, int n_q, const void *c_kv, const void *k_pe,
                      int max_blocks_per_seq, int num_blocks, const int32_t *seqlens, int max_seqlen) {
  if (!dims_ok(dims)) return MLA_ERR_INVALID_ARG;
  if (B <= 0 || n_q <= 0 || max_seqlen < n_q || max_blocks_per_seq <= 0 || num_blocks <= 0)
    return MLA_ERR_INVALID_ARG;
  if (!c_kv || (!k_pe && dims->d_rope && dims->cache_layout == MLA_CACHE_ROWS) || !seqlens) return MLA_ERR_INVALID_ARG;
  if ((int64_t)max_blocks_per_seq * dims->block_size < max_seqlen) return MLA_ERR_INVALID_ARG;
  if (n_q * dims->n_heads > 256) return MLA_ERR_UNSUPPORTED;
  return MLA_OK;
}

int check_ws(const DecodeLayout &L, const void *workspace, size_t ws_bytes) {
  if (!workspace || ws_bytes < L.total || (reinterpret_cast<uintptr_t>(workspace) & 255)) return MLA_ERR_WORKSPACE;
  return MLA_OK;
}

constexpr int kAllKeys = 0x7fffffff;   // kv_end of a decode over every cached key

int attention_impl(const mla_dims *dims, int B, int n_q, const void *q_abs, const void *c_kv, const void *k_pe,
                   const int32_t *block_table, int max_blocks_per_seq, int num_blocks, const int32_t *seqlens,
                   int max_seqlen, const DecodeLayout &L, char *ws, int *dev_status, cudaStream_t st,
                   int kv_begin = 0, int kv_end = kAllKeys) {
  const bool bf16 = dims->dtype == MLA_BF16;
  CacheView cv{c_kv, k_pe, dims->ckv_stride, dims->kpe_stride, block_table, max_blocks_per_seq,
               num_blocks, dims->block_size, dims->cache_layout, dims->d_c, dims->d_c + dims->d_rope};
  if (L.use_tc)
    return launch_tc_attention(*dims, B, n_q, q_abs, cv, seqlens, max_seqlen, ws + L.tc_off, dev_status, st,
                               kv_begin, kv_end);
  AttnArgs at{B, n_q, dims->n_heads, dims->d_c, dims->d_rope, q_abs, cv, seqlens, default_scale(*dims),
              kSimtChunk, L.max_chunks, reinterpret_cast<float *>(ws + L.o_off),
              reinterpret_cast<float *>(ws + L.lse_off), dev_status, kv_begin, kv_end};
  return launch_attn_simt(at, bf16, st);
}

int combine_impl(const mla_dims *dims, int B, int n_q, const int32_t *seqlens, int max_seqlen, const void *w_uv,
                 void *out, float *lse, const DecodeLayout &L, char *ws, int *dev_status, cudaStream_t st) {
  const bool bf16 = dims->dtype == MLA_BF16;
  if (L.use_tc)
    return launch_tc_combine(*dims, B, n_q, seqlens, max_seqlen, w_uv, out, lse, ws + L.tc_off, dev_status, st);
  CombineArgs cb{B, n_q, dims->n_heads, dims->d_c, dims->d_v, seqlens, kSimtChunk, L.max_chunks,
                 reinterpret_cast<const float *>(ws + L.o_off), reinterpret_cast<const float *>(ws + L.lse_off),
                 w_uv, out, lse};
  return launch_combine(cb, bf16, st);
}

// Query absorption: tcgen05 where the shape and alignment allow, else warp MMAs, else CUDA cores.
int absorb_dispatch(const AbsorbArgs &ab, bool bf16, int *dev_status, cudaStream_t st) {
  if (absorb_tc_supported(ab, bf16)) return launch_absorb_tc(ab, dev_status, st);
  if (absorb_mma_supported(ab, bf16)) return launch_absorb_mma(ab, st);
  return launch_absorb(ab, bf16, st);
}

int decode_impl(const mla_dims *dims, int B, int n_q, const void *q_nope, const void *q_pe,
                const void *c_kv, const void *k_pe, const int32_t *block_table, int max_blocks_per_seq,
                int num_blocks, const int32_t *seqlens, int max_seqlen, const void *w_uk,
                const void *w_uv, void *out, float *lse, void *workspace, size_t ws_bytes,
                int *dev_status, cudaStream_t st, int kv_begin = 0, int kv_end = kAllKeys) {
  int rc = check_decode_args(dims, B, n_q, c_kv, k_pe, max_blocks_per_seq, num_blocks, seqlens, max_seqlen);
  if (rc) return rc;
  if (!q_nope || (!q_pe && dims->d_rope) || !w_uk || !out) return MLA_ERR_INVALID_ARG;
  const DecodeLayout L = decode_layout(dims, B, n_q, max_seqlen);
  if ((rc = check_ws(L, workspace, ws_bytes))) return rc;
  char *ws = static_cast<char *>(workspace);
  void *qbuf = ws + L.q_off;
  AbsorbArgs ab{B, n_q, dims->n_heads, dims->d_c, dims->d_rope, dims->d_nope,
                q_nope, q_pe, w_uk, seqlens, qbuf, dims->rope_base};
  if ((rc = absorb_dispatch(ab, dims->dtype == MLA_BF16, dev_status, st))) return rc;
  if ((rc = attention_impl(dims, B, n_q, qbuf, c_kv, k_pe, block_table, max_blocks_per_seq, num_blocks, seqlens,
                           max_seqlen, L, ws, dev_status, st, kv_begin, kv_end)))
    return rc;
  return combine_impl(dims, B, n_q, seqlens, max_seqlen, w_uv, out, lse, L, ws, dev_status, st);
}

// Sparse decode: the gathered pool holds B * n_q short "sequences" (one per query token) of
// 64-token pages, in the tiled layout where the tensor-core path takes the shape, else fused rows.
struct SparseLayout {
  mla_dims inner;               // dims of the gathered pool and of the attention over it
  int units, pages;             // B * n_q query tokens, pages per token
  size_t counts_off, pool_off, dec_off, total;
  DecodeLayout dec;             // decode workspace of the inner call (B * n_q sequences, one query each)
};

SparseLayout sparse_layout(const mla_dims *d, int B, int n_q, int topk) {
  SparseLayout L{};
  L.inner = *d;
  L.inner.block_size = 64;
  const int W = d->d_c + d->d_rope;
  const bool tiled = d->dtype == MLA_BF16 && W % 64 == 0;
  L.inner.cache_layout = tiled ? MLA_CACHE_TILED : MLA_CACHE_ROWS;
  L.inner.ckv_stride = L.inner.kpe_stride = W;
  L.units = B * n_q;
  L.pages = (topk + 63) / 64;
  L.counts_off = 0;
  L.pool_off = align256((size_t)L.units * sizeof(int32_t));
  L.dec_off = L.pool_off + align256((size_t)L.units * L.pages * 64 * W * elem(d));
  L.dec = decode_layout(&L.inner, L.units, 1, L.pages * 64);
  L.total = L.dec_off + L.dec.total;
  return L;
}

// K-split of a CUDA-core product so that about two CTAs per SM get work.
int gemm_ksplit(int M, int N, int K) {
  const int tiles = ((M + 63) / 64) * ((N + 63) / 64);
  int ks = (296 + tiles - 1) / tiles;
  ks = ks < 1 ? 1 : ks;
  const int kmax = (K + 255) / 256;          // keep at least 256 of K per split
  return ks > kmax ? kmax : ks;
}

GemmArgs gemm_args(int M, int N, int K, int batch, const void *A, int64_t sa_b, int64_t sa_m, int64_t sa_k,
                   const void *B, int64_t sb_b, int64_t sb_k, int64_t sb_n, void *C, int64_t sc_b, int64_t sc_m,
                   int64_t sc_n, bool split) {
  return GemmArgs{M, N, K, batch, split ? gemm_ksplit(M, N, K) : 1, A, sa_b, sa_m, sa_k, B, sb_b, sb_k, sb_n,
                  C, sc_b, sc_m, sc_n, nullptr};
}

// Decode from hidden states with folded weights: the workspace holds the decode workspace (whose
// query region receives the absorbed queries), c_Q, the raw RoPE queries, o_lat and the K-split
// partials of the products.
struct AbsorbedLayout {
  DecodeLayout dec;
  size_t cq_off, qpe_off, olat_off, part_off, total;
  GemmArgs g_cq, g_qlat, g_qpe, g_out;
};

AbsorbedLayout absorbed_layout(const mla_dims *d, int d_cq, int B, int n_q, int max_seqlen) {
  AbsorbedLayout L{};
  const int T = B * n_q, H = d->n_heads, W = d->d_c + d->d_rope, D = d->d_model;
  const size_t e = elem(d);
  L.dec = decode_layout(d, B, n_q, max_seqlen);
  L.cq_off = L.dec.total;
  L.qpe_off = L.cq_off + align256((size_t)T * d_cq * e);
  L.olat_off = L.qpe_off + align256((size_t)T * H * d->d_rope * e + 16);
  L.part_off = L.olat_off + align256((size_t)T * H * d->d_c * e);
  // c_Q = h W_DQ;  q_lat^(s) = c_Q W_UQK^(s) into q_abs;  q_pe = c_Q W_QR;  u = o_lat W_UVO.
  L.g_cq = gemm_args(T, d_cq, D, 1, nullptr, 0, D, 1, nullptr, 0, d_cq, 1, nullptr, 0, d_cq, 1, true);
  L.g_qlat = gemm_args(T, d->d_c, d_cq, H, nullptr, 0, d_cq, 1, nullptr, (int64_t)d_cq * d->d_c, d->d_c, 1, nullptr, W,
                       (int64_t)H * W, 1, false);
  L.g_qpe = gemm_args(T, H * d->d_rope, d_cq, 1, nullptr, 0, d_cq, 1, nullptr, 0, (int64_t)H * d->d_rope, 1, nullptr,
                      0, (int64_t)H * d->d_rope, 1, true);
  L.g_out = gemm_args(T, D, H * d->d_c, 1, nullptr, 0, (int64_t)H * d->d_c, 1, nullptr, 0, D, 1, nullptr, 0, D, 1, true);
  size_t part = 0;
  for (const GemmArgs *g : {&L.g_cq, &L.g_qlat, &L.g_qpe, &L.g_out}) {
    const size_t p = gemm_simt_workspace(*g);
    part = p > part ? p : part;
  }
  L.total = L.part_off + align256(part);
  return L;
}

// Sequence and position of each new token of a decode step: token t = b n_q + j sits at
// seqlens[b] - n_q + j.
__global__ void step_positions_kernel(int B, int n_q, const int32_t *seqlens, int32_t *seq_idx, int32_t *pos) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= B * n_q) return;
  const int b = t / n_q;
  seq_idx[t] = b;
  pos[t] = seqlens[b] - n_q + t % n_q;
}

// Decode step workspace: the fused kernel's completion counter, the append's split-K partials, the
// new tokens' (sequence, position) for the unfused path, then the decode workspace.
struct StepLayout {
  size_t counter_off, part_off, idx_off, dec_off, total;
  int nsplit, kps;
  DecodeLayout dec;
};

StepLayout step_layout(const mla_dims *d, int B, int n_q, int max_seqlen) {
  StepLayout L{};
  const int T = B * n_q, W = d->d_c + d->d_rope;
  L.counter_off = 0;
  L.part_off = 256;
  L.nsplit = 1;
  L.kps = d->d_model;
  const size_t part = append_mma_workspace(T, d->d_model, W, &L.nsplit, &L.kps);
  L.idx_off = L.part_off + align256(part);
  L.dec_off = L.idx_off + align256((size_t)2 * T * sizeof(int32_t));
  L.dec = decode_layout(d, B, n_q, max_seqlen);
  L.total = L.dec_off + L.dec.total;
  return L;
}

}  // namespace

extern "C" {

int mla_fold_query_weights(const mla_dims *dims, int d_cq, const void *w_uq, const void *w_uk, void *w_uqk,
                           mla_stream_t stream) {
  if (!dims_ok(dims) || d_cq <= 0 || !w_uq || !w_uk || !w_uqk) return MLA_ERR_INVALID_ARG;
  const int H = dims->n_heads, dn = dims->d_nope, dc = dims->d_c;
  // W_UQK[s] [d_cq x d_c] = W_UQ[:, s, :] [d_cq x d_nope] . W_UK[s]^T [d_nope x d_c]
  GemmArgs g{d_cq, dc, dn, H, 1, w_uq, dn, (int64_t)H * dn, 1, w_uk, (int64_t)dc * dn, 1, dn, w_uqk,
             (int64_t)d_cq * dc, dc, 1, nullptr};
  return launch_gemm_simt(g, dims->dtype == MLA_BF16, reinterpret_cast<cudaStream_t>(stream));
}

int mla_fold_output_weights(const mla_dims *dims, const void *w_uv, const void *w_o, void *w_uvo, mla_stream_t stream) {
  if (!dims_ok(dims) || dims->d_model <= 0 || !w_uv || !w_o || !w_uvo) return MLA_ERR_INVALID_ARG;
  const int H = dims->n_heads, dv = dims->d_v, dc = dims->d_c, D = dims->d_model;
  // W_UVO[s] [d_c x D] = W_UV[s] [d_c x d_v] . W_O[s d_v .. (s+1) d_v - 1, :] [d_v x D]
  GemmArgs g{dc, D, dv, H, 1, w_uv, (int64_t)dc * dv, dv, 1, w_o, (int64_t)dv * D, D, 1, w_uvo, (int64_t)dc * D, D, 1,
             nullptr};
  return launch_gemm_simt(g, dims->dtype == MLA_BF16, reinterpret_cast<cudaStream_t>(stream));
}

int mla_decode_absorbed_workspace_size(const mla_dims *dims, int d_cq, int B, int n_q, int max_seqlen, size_t *bytes) {
  if (!dims_ok(dims) || d_cq <= 0 || dims->d_model <= 0 || B <= 0 || n_q <= 0 || max_seqlen < n_q || !bytes)
    return MLA_ERR_INVALID_ARG;
  if (n_q * dims->n_heads > 256) return MLA_ERR_UNSUPPORTED;
  *bytes = absorbed_layout(dims, d_cq, B, n_q, max_seqlen).total;
  return MLA_OK;
}

int mla_decode_absorbed(const mla_dims *dims, int d_cq, int B, int n_q, const void *h, const void *w_dq,
                        const void *w_uqk, const void *w_qr, const void *c_kv, const void *k_pe,
                        const int32_t *block_table, int max_blocks_per_seq, int num_blocks, const int32_t *seqlens,
                        int max_seqlen, const void *w_uvo, void *out, float *lse, void *workspace, size_t ws_bytes,
                        int *dev_status, mla_stream_t stream) {
  int rc = check_decode_args(dims, B, n_q, c_kv, k_pe, max_blocks_per_seq, num_blocks, seqlens, max_seqlen);
  if (rc) return rc;
  if (d_cq <= 0 || dims->d_model <= 0 || !h || !w_dq || !w_uqk || (!w_qr && dims->d_rope) || !w_uvo || !out)
    return MLA_ERR_INVALID_ARG;
  AbsorbedLayout L = absorbed_layout(dims, d_cq, B, n_q, max_seqlen);
  if (!workspace || ws_bytes < L.total || (reinterpret_cast<uintptr_t>(workspace) & 255)) return MLA_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const bool bf16 = dims->dtype == MLA_BF16;
  char *ws = static_cast<char *>(workspace);
  void *q_abs = ws + L.dec.q_off, *c_q = ws + L.cq_off, *q_pe = ws + L.qpe_off, *o_lat = ws + L.olat_off;
  float *part = reinterpret_cast<float *>(ws + L.part_off);
  // (1) c_Q = h W_DQ.
  L.g_cq.A = h; L.g_cq.B = w_dq; L.g_cq.C = c_q; L.g_cq.part = part;
  if ((rc = launch_gemm(L.g_cq, bf16, st))) return rc;
  // (2) latent queries q_lat^(s) = c_Q W_UQK^(s), straight into the absorbed query buffer.
  L.g_qlat.A = c_q; L.g_qlat.B = w_uqk; L.g_qlat.C = q_abs; L.g_qlat.part = part;
  if ((rc = launch_gemm(L.g_qlat, bf16, st))) return rc;
  // (3) RoPE queries q_pe^(s) = RoPE(c_Q W_QR^(s), position), into the query buffer's RoPE slots.
  if (dims->d_rope) {
    L.g_qpe.A = c_q; L.g_qpe.B = w_qr; L.g_qpe.C = q_pe; L.g_qpe.part = part;
    if ((rc = launch_gemm(L.g_qpe, bf16, st))) return rc;
    if ((rc = launch_rope_into_query(B, n_q, dims->n_heads, dims->d_c, dims->d_rope, q_pe, seqlens, q_abs,
                                     dims->rope_base, bf16, st)))
      return rc;
  }
  // (4) split-KV attention and the merge of its partials into o_lat.
  if ((rc = attention_impl(dims, B, n_q, q_abs, c_kv, k_pe, block_table, max_blocks_per_seq, num_blocks, seqlens,
                           max_seqlen, L.dec, ws, dev_status, st)))
    return rc;
  if ((rc = combine_impl(dims, B, n_q, seqlens, max_seqlen, nullptr, o_lat, lse, L.dec, ws, dev_status, st))) return rc;
  // (5) u = sum_s o_lat^(s) W_UVO^(s).
  L.g_out.A = o_lat; L.g_out.B = w_uvo; L.g_out.C = out; L.g_out.part = part;
  return launch_gemm(L.g_out, bf16, st);
}

int mla_decode_sparse_workspace_size(const mla_dims *dims, int B, int n_q, int topk, size_t *bytes) {
  if (!dims_ok(dims) || B <= 0 || n_q <= 0 || topk <= 0 || !bytes) return MLA_ERR_INVALID_ARG;
  if (dims->n_heads > 256) return MLA_ERR_UNSUPPORTED;
  *bytes = sparse_layout(dims, B, n_q, topk).total;
  return MLA_OK;
}

int mla_decode_sparse(const mla_dims *dims, int B, int n_q, const void *q_nope, const void *q_pe, const void *c_kv,
                      const void *k_pe, const int32_t *block_table, int max_blocks_per_seq, int num_blocks,
                      const int32_t *seqlens, int max_seqlen, const int32_t *topk_idx, int topk, const void *w_uk,
                      const void *w_uv, void *out, float *lse, void *workspace, size_t ws_bytes, int *dev_status,
                      mla_stream_t stream) {
  if (!dims_ok(dims) || B <= 0 || n_q <= 0 || topk <= 0 || max_seqlen < n_q || max_blocks_per_seq <= 0 ||
      num_blocks <= 0)
    return MLA_ERR_INVALID_ARG;
  if (!q_nope || (!q_pe && dims->d_rope) || !c_kv || (!k_pe && dims->d_rope && dims->cache_layout == MLA_CACHE_ROWS) ||
      !seqlens || !topk_idx || !w_uk || !w_uv || !out)
    return MLA_ERR_INVALID_ARG;
  if ((int64_t)max_blocks_per_seq * dims->block_size < max_seqlen) return MLA_ERR_INVALID_ARG;
  if (dims->n_heads > 256) return MLA_ERR_UNSUPPORTED;
  const SparseLayout L = sparse_layout(dims, B, n_q, topk);
  if (!workspace || ws_bytes < L.total || (reinterpret_cast<uintptr_t>(workspace) & 255)) return MLA_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  char *ws = static_cast<char *>(workspace);
  int32_t *counts = reinterpret_cast<int32_t *>(ws + L.counts_off);
  char *pool = ws + L.pool_off;
  char *dws = ws + L.dec_off;
  // (1) Query absorption at each token's own position (the real sequence lengths).
  void *qbuf = dws + L.dec.q_off;
  AbsorbArgs ab{B, n_q, dims->n_heads, dims->d_c, dims->d_rope, dims->d_nope,
                q_nope, q_pe, w_uk, seqlens, qbuf, dims->rope_base};
  int rc = absorb_dispatch(ab, dims->dtype == MLA_BF16, dev_status, st);
  if (rc) return rc;
  // (2) The listed rows of every query token into its own pages of the gathered pool.
  CacheView src{c_kv, k_pe, dims->ckv_stride, dims->kpe_stride, block_table, max_blocks_per_seq, num_blocks,
                dims->block_size, dims->cache_layout, dims->d_c, dims->d_c + dims->d_rope};
  if ((rc = launch_sparse_gather(B, n_q, topk, topk_idx, seqlens, max_seqlen, src, pool,
                                 L.inner.cache_layout == MLA_CACHE_TILED, (int)elem(dims), counts, dev_status, st)))
    return rc;
  // (3) + (4) Attention over the gathered pool (every listed key visible to its own query) and combine.
  const mla_dims *in = &L.inner;
  const int W = dims->d_c + dims->d_rope;
  if ((rc = attention_impl(in, L.units, 1, qbuf, pool, pool + (size_t)dims->d_c * elem(dims), nullptr, L.pages,
                           L.units * L.pages, counts, L.pages * 64, L.dec, dws, dev_status, st)))
    return rc;
  (void)W;
  return combine_impl(in, L.units, 1, counts, L.pages * 64, w_uv, out, lse, L.dec, dws, dev_status, st);
}

const char *mla_status_string(int s) {
  switch (s) {
    case MLA_OK: return "ok";
    case MLA_ERR_INVALID_ARG: return "invalid argument";
    case MLA_ERR_UNSUPPORTED: return "unsupported shape";
    case MLA_ERR_WORKSPACE: return "workspace missing, too small or misaligned";
    case MLA_ERR_CUDA: return "CUDA error";
    case MLA_ERR_TIMEOUT: return "device wait timed out";
    case MLA_ERR_BAD_INDEX: return "block id, sequence index or position out of range";
    case MLA_ERR_STATIC_WS: return "shape needs more scratch than the built-in no-allocation buffer";
    default: return "unknown status";
  }
}

static AppendArgs append_args(const mla_dims *dims, int T, const void *h, const void *w_dkv, const void *w_kr,
                              const void *rms_gamma, const int32_t *seq_idx, const int32_t *pos, void *c_kv, void *k_pe,
                              const int32_t *block_table, int num_seqs, int max_blocks_per_seq, int num_blocks,
                              int *dev_status) {
  return AppendArgs{T, dims->d_model, dims->d_c, dims->d_rope, h, w_dkv, w_kr, rms_gamma, seq_idx, pos,
                    c_kv, k_pe, dims->ckv_stride, dims->kpe_stride, block_table, num_seqs,
                    max_blocks_per_seq, num_blocks, dims->block_size, dims->cache_layout, dims->rms_eps,
                    dims->rope_base, dev_status};
}

int mla_append_workspace_size(const mla_dims *dims, int T, size_t *bytes) {
  if (!dims_ok(dims) || dims->d_model <= 0 || T < 0 || !bytes) return MLA_ERR_INVALID_ARG;
  AppendArgs a = append_args(dims, T, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr,
                             nullptr, 1, 1, 1, nullptr);
  *bytes = (T > 0 && append_mma_supported(a, dims->dtype == MLA_BF16))
               ? append_mma_workspace(T, dims->d_model, dims->d_c + dims->d_rope, nullptr, nullptr)
               : 0;
  return MLA_OK;
}

int mla_append_latent(const mla_dims *dims, int T, const void *h, const void *w_dkv, const void *w_kr,
                      const void *rms_gamma, const int32_t *seq_idx, const int32_t *pos, void *c_kv,
                      void *k_pe, const int32_t *block_table, int num_seqs, int max_blocks_per_seq,
                      int num_blocks, void *workspace, size_t ws_bytes, int *dev_status, mla_stream_t stream) {
  if (!dims_ok(dims) || dims->d_model <= 0 || T < 0) return MLA_ERR_INVALID_ARG;
  if (T == 0) return MLA_OK;
  if (!h || !w_dkv || (!w_kr && dims->d_rope) || !seq_idx || !pos || !c_kv ||
      (!k_pe && dims->d_rope && dims->cache_layout == MLA_CACHE_ROWS))
    return MLA_ERR_INVALID_ARG;
  if (num_seqs <= 0 || max_blocks_per_seq <= 0 || num_blocks <= 0) return MLA_ERR_INVALID_ARG;
  const AppendArgs a = append_args(dims, T, h, w_dkv, w_kr, rms_gamma, seq_idx, pos, c_kv, k_pe, block_table,
                                   num_seqs, max_blocks_per_seq, num_blocks, dev_status);
  const bool bf16 = dims->dtype == MLA_BF16;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int nsplit = 1, kps = dims->d_model;
  if (workspace && append_mma_supported(a, bf16) && !(reinterpret_cast<uintptr_t>(workspace) & 15) &&
      ws_bytes >= append_mma_workspace(T, dims->d_model, dims->d_c + dims->d_rope, &nsplit, &kps)) {
    if (append_tc_supported(a, bf16)) {
      const int rc = launch_append_tc(a, workspace, nsplit, kps, st);
      return rc ? rc : launch_append_finish(a, workspace, nsplit, st);
    }
    return launch_append_mma(a, workspace, st);
  }
  return launch_append(a, bf16, st);
}

int mla_decode_step_workspace_size(const mla_dims *dims, int B, int n_q, int max_seqlen, size_t *bytes) {
  if (!dims_ok(dims) || dims->d_model <= 0 || B <= 0 || n_q <= 0 || max_seqlen < n_q || !bytes)
    return MLA_ERR_INVALID_ARG;
  if (n_q * dims->n_heads > 256) return MLA_ERR_UNSUPPORTED;
  *bytes = step_layout(dims, B, n_q, max_seqlen).total;
  return MLA_OK;
}

int mla_decode_step(const mla_dims *dims, int B, int n_q, const void *h_new, const void *w_dkv, const void *w_kr,
                    const void *rms_gamma, const void *q_nope, const void *q_pe, void *c_kv, void *k_pe,
                    const int32_t *block_table, int max_blocks_per_seq, int num_blocks, const int32_t *seqlens,
                    int max_seqlen, const void *w_uk, const void *w_uv, void *out, float *lse, void *workspace,
                    size_t ws_bytes, int *dev_status, mla_stream_t stream) {
  int rc = check_decode_args(dims, B, n_q, c_kv, k_pe, max_blocks_per_seq, num_blocks, seqlens, max_seqlen);
  if (rc) return rc;
  if (dims->d_model <= 0 || !h_new || !w_dkv || (!w_kr && dims->d_rope) || !q_nope || (!q_pe && dims->d_rope) ||
      !w_uk || !w_uv || !out)
    return MLA_ERR_INVALID_ARG;
  const StepLayout L = step_layout(dims, B, n_q, max_seqlen);
  if (!workspace || ws_bytes < L.total || (reinterpret_cast<uintptr_t>(workspace) & 255)) return MLA_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  char *ws = static_cast<char *>(workspace);
  const int T = B * n_q;
  int32_t *seq_idx = reinterpret_cast<int32_t *>(ws + L.idx_off), *pos = seq_idx + T;
  char *dws = ws + L.dec_off;
  void *qbuf = dws + L.dec.q_off;
  const bool bf16 = dims->dtype == MLA_BF16;
  AppendArgs ap = append_args(dims, T, h_new, w_dkv, w_kr, rms_gamma, seq_idx, pos, c_kv, k_pe, block_table, B,
                              max_blocks_per_seq, num_blocks, dev_status);
  AbsorbArgs ab{B, n_q, dims->n_heads, dims->d_c, dims->d_rope, dims->d_nope,
                q_nope, q_pe, w_uk, seqlens, qbuf, dims->rope_base};
  if (bf16 && L.dec.use_tc && decode_prep_supported(ap, ab)) {
    // One launch: append of the new tokens and the query absorption.
    if ((rc = launch_decode_prep(ap, ab, ws + L.part_off, L.nsplit, L.kps, reinterpret_cast<unsigned *>(ws + L.counter_off),
                                 st)))
      return rc;
  } else {
    step_positions_kernel<<<(T + 255) / 256, 256, 0, st>>>(B, n_q, seqlens, seq_idx, pos);
    if (cudaGetLastError() != cudaSuccess) return MLA_ERR_CUDA;
    if ((rc = mla_append_latent(dims, T, h_new, w_dkv, w_kr, rms_gamma, seq_idx, pos, c_kv, k_pe, block_table, B,
                                max_blocks_per_seq, num_blocks, ws + L.part_off, L.idx_off - L.part_off, dev_status,
                                stream)))
      return rc;
    if ((rc = absorb_dispatch(ab, bf16, dev_status, st))) return rc;
  }
  if ((rc = attention_impl(dims, B, n_q, qbuf, c_kv, k_pe, block_table, max_blocks_per_seq, num_blocks, seqlens,
                           max_seqlen, L.dec, dws, dev_status, st)))
    return rc;
  return combine_impl(dims, B, n_q, seqlens, max_seqlen, w_uv, out, lse, L.dec, dws, dev_status, st);
}

int mla_absorb_q(const mla_dims *dims, int B, int n_q, const void *q_nope, const void *q_pe,
                 const void *w_uk, const int32_t *seqlens, void *q_out, mla_stream_t stream) {
  if (!dims_ok(dims) || B <= 0 || n_q <= 0) return MLA_ERR_INVALID_ARG;
  if (!q_nope || (!q_pe && dims->d_rope) || !w_uk || !seqlens || !q_out) return MLA_ERR_INVALID_ARG;
  AbsorbArgs ab{B, n_q, dims->n_heads, dims->d_c, dims->d_rope, dims->d_nope,
                q_nope, q_pe, w_uk, seqlens, q_out, dims->rope_base};
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return absorb_dispatch(ab, dims->dtype == MLA_BF16, nullptr, st);
}

int mla_decode_workspace_size(const mla_dims *dims, int B, int n_q, int max_seqlen, size_t *bytes) {
  if (!dims_ok(dims) || B <= 0 || n_q <= 0 || max_seqlen < n_q || !bytes) return MLA_ERR_INVALID_ARG;
  if (n_q * dims->n_heads > 256) return MLA_ERR_UNSUPPORTED;
  *bytes = decode_layout(dims, B, n_q, max_seqlen).total;
  return MLA_OK;
}

int mla_decode(const mla_dims *dims, int B, int n_q, const void *q_nope, const void *q_pe,
               const void *c_kv, const void *k_pe, const int32_t *block_table, int max_blocks_per_seq,
               int num_blocks, const int32_t *seqlens, int max_seqlen, const void *w_uk,
               const void *w_uv, void *out, float *lse, void *workspace, size_t ws_bytes,
               int *dev_status, mla_stream_t stream) {
  if (!w_uv) return MLA_ERR_INVALID_ARG;
  return decode_impl(dims, B, n_q, q_nope, q_pe, c_kv, k_pe, block_table, max_blocks_per_seq,
                     num_blocks, seqlens, max_seqlen, w_uk, w_uv, out, lse, workspace, ws_bytes,
                     dev_status, reinterpret_cast<cudaStream_t>(stream));
}

int mla_decode_latent(const mla_dims *dims, int B, int n_q, const void *q_nope, const void *q_pe,
                      const void *c_kv, const void *k_pe, const int32_t *block_table,
                      int max_blocks_per_seq, int num_blocks, const int32_t *seqlens, int max_seqlen,
                      const void *w_uk, void *o_lat, float *lse, void *workspace, size_t ws_bytes,
                      int *dev_status, mla_stream_t stream) {
  return decode_impl(dims, B, n_q, q_nope, q_pe, c_kv, k_pe, block_table, max_blocks_per_seq,
                     num_blocks, seqlens, max_seqlen, w_uk, nullptr, o_lat, lse, workspace, ws_bytes,
                     dev_status, reinterpret_cast<cudaStream_t>(stream));
}

int mla_decode_attention(const mla_dims *dims, int B, int n_q, const void *q_abs, const void *c_kv,
                         const void *k_pe, const int32_t *block_table, int max_blocks_per_seq, int num_blocks,
                         const int32_t *seqlens, int max_seqlen, void *workspace, size_t ws_bytes,
                         int *dev_status, mla_stream_t stream) {
  int rc = check_decode_args(dims, B, n_q, c_kv, k_pe, max_blocks_per_seq, num_blocks, seqlens, max_seqlen);
  if (rc) return rc;
  if (!q_abs) return MLA_ERR_INVALID_ARG;
  const DecodeLayout L = decode_layout(dims, B, n_q, max_seqlen);
  if ((rc = check_ws(L, workspace, ws_bytes))) return rc;
  return attention_impl(dims, B, n_q, q_abs, c_kv, k_pe, block_table, max_blocks_per_seq, num_blocks, seqlens,
                        max_seqlen, L, static_cast<char *>(workspace), dev_status,
                        reinterpret_cast<cudaStream_t>(stream));
}

int mla_decode_combine(const mla_dims *dims, int B, int n_q, const int32_t *seqlens, int max_seqlen,
                       const void *w_uv, void *out, float *lse, void *workspace, size_t ws_bytes,
                       mla_stream_t stream) {
  if (!dims_ok(dims) || B <= 0 || n_q <= 0 || max_seqlen < n_q || !seqlens || !out) return MLA_ERR_INVALID_ARG;
  if (n_q * dims->n_heads > 256) return MLA_ERR_UNSUPPORTED;
  const DecodeLayout L = decode_layout(dims, B, n_q, max_seqlen);
  int rc = check_ws(L, workspace, ws_bytes);
  if (rc) return rc;
  return combine_impl(dims, B, n_q, seqlens, max_seqlen, w_uv, out, lse, L, static_cast<char *>(workspace), nullptr,
                      reinterpret_cast<cudaStream_t>(stream));
}

int mla_decode_launches(const mla_dims *dims, int n_q, int *count) {
  if (!dims_ok(dims) || n_q <= 0 || !count) return MLA_ERR_INVALID_ARG;
  *count = tc_decode_supported(*dims, n_q) ? 1 + tc_decode_kernel_launches() : 3;
  return MLA_OK;
}

int mla_decode_path(const mla_dims *dims, int n_q, int *path) {
  if (!dims_ok(dims) || n_q <= 0 || !path) return MLA_ERR_INVALID_ARG;
  *path = tc_decode_supported(*dims, n_q) ? MLA_PATH_TCGEN05 : MLA_PATH_CUDA_CORES;
  return MLA_OK;
}

int mla_decode_partial(const mla_dims *dims, int B, int n_q, const void *q_nope, const void *q_pe, const void *c_kv,
                       const void *k_pe, const int32_t *block_table, int max_blocks_per_seq, int num_blocks,
                       const int32_t *seqlens, int max_seqlen, int kv_begin, int kv_end, const void *w_uk,
                       void *o_lat, float *lse, void *workspace, size_t ws_bytes, int *dev_status,
                       mla_stream_t stream) {
  if (kv_begin < 0 || kv_begin % 64 || kv_end <= kv_begin || !lse) return MLA_ERR_INVALID_ARG;
  return decode_impl(dims, B, n_q, q_nope, q_pe, c_kv, k_pe, block_table, max_blocks_per_seq, num_blocks, seqlens,
                     max_seqlen, w_uk, nullptr, o_lat, lse, workspace, ws_bytes, dev_status,
                     reinterpret_cast<cudaStream_t>(stream), kv_begin, kv_end);
}

int mla_merge_workspace_size(const mla_dims *dims, int B, int n_q, int n_parts, size_t *bytes) {
  if (!dims_ok(dims) || B <= 0 || n_q <= 0 || n_parts <= 0 || !bytes) return MLA_ERR_INVALID_ARG;
  const size_t rows = (size_t)B * n_parts * n_q * dims->n_heads;
  *bytes = align256(rows * dims->d_c * sizeof(float)) + align256(rows * sizeof(float));
  return MLA_OK;
}

int mla_merge_partials(const mla_dims *dims, int B, int n_q, int n_parts, const void *o_lat_parts,
                       const float *lse_parts, const void *w_uv, void *out, float *lse, void *workspace,
                       size_t ws_bytes, mla_stream_t stream) {
  size_t need = 0;
  int rc = mla_merge_workspace_size(dims, B, n_q, n_parts, &need);
  if (rc) return rc;
  if (!o_lat_parts || !lse_parts || !out) return MLA_ERR_INVALID_ARG;
  if (!workspace || ws_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255)) return MLA_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // bf16 rows of 512: merged by log-sum-exp into bf16 rows and, with W_UV, multiplied by it on the
  // tensor cores in the same kernel (the workspace is not used).
  if (tc_merge_parts_supported(*dims, o_lat_parts, w_uv, out))
    return launch_tc_merge_parts(*dims, B, n_q, n_parts, o_lat_parts, lse_parts, w_uv, out, lse, st);
  if ((size_t)16 * (dims->d_c + n_parts) * sizeof(float) > 220 * 1024) return MLA_ERR_UNSUPPORTED;
  const size_t rows = (size_t)B * n_parts * n_q * dims->n_heads;
  float *o_part = static_cast<float *>(workspace);
  float *lse_part = reinterpret_cast<float *>(static_cast<char *>(workspace) + align256(rows * dims->d_c * sizeof(float)));
  const bool bf16 = dims->dtype == MLA_BF16;
  if ((rc = launch_partials_to_splits(n_parts, B, n_q, dims->n_heads, dims->d_c, o_lat_parts, lse_parts, bf16, o_part,
                                      lse_part, st)))
    return rc;
  CombineArgs cb{B, n_q, dims->n_heads, dims->d_c, dims->d_v, nullptr, 1, n_parts, o_part, lse_part, w_uv, out, lse};
  return launch_combine(cb, bf16, st);
}

int mla_prefill_workspace_size(const mla_dims *dims, int B, int total_tokens, int max_seqlen,
                               size_t *bytes) {
  if (!dims_ok(dims) || B <= 0 || total_tokens <= 0 || max_seqlen <= 0 || !bytes)
    return MLA_ERR_INVALID_ARG;
  const size_t dqk = (size_t)dims->d_nope + dims->d_rope;
  const size_t rows = (size_t)total_tokens * dims->n_heads;
  const size_t row_layout = 2 * align256(rows * dqk * elem(dims)) + align256(rows * dims->d_v * elem(dims));
  // The tensor-core path keeps its Q/K/V in per-(head, sequence) tiles padded to max_seqlen.
  const size_t tiled = dims->dtype == MLA_BF16 ? prefill_tiled_bytes(B, dims->n_heads, max_seqlen) : 0;
  *bytes = row_layout > tiled ? row_layout : tiled;
  return MLA_OK;
}

int mla_prefill(const mla_dims *dims, int B, const int32_t *cu_seqlens, int max_seqlen, int total_tokens,
                const void *q_nope, const void *q_pe, const void *c_kv, const void *k_pe,
                const int32_t *block_table, int max_blocks_per_seq, int num_blocks, const void *w_uk,
                const void *w_uv, void *out, float *lse, void *workspace, size_t ws_bytes, int *dev_status,
                mla_stream_t stream) {
  if (!dims_ok(dims) || B <= 0 || total_tokens <= 0 || max_seqlen <= 0 || max_blocks_per_seq <= 0 ||
      num_blocks <= 0)
    return MLA_ERR_INVALID_ARG;
  if (!cu_seqlens || !q_nope || (!q_pe && dims->d_rope) || !c_kv ||
      (!k_pe && dims->d_rope && dims->cache_layout == MLA_CACHE_ROWS) || !w_uk ||
      !w_uv || !out)
    return MLA_ERR_INVALID_ARG;
  size_t need = 0;
  mla_prefill_workspace_size(dims, B, total_tokens, max_seqlen, &need);
  if (!workspace || ws_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255)) return MLA_ERR_WORKSPACE;
  const size_t dqk = (size_t)dims->d_nope + dims->d_rope;
  const size_t rows = (size_t)total_tokens * dims->n_heads;
  char *ws = static_cast<char *>(workspace);
  void *qbuf = ws;
  void *kbuf = ws + align256(rows * dqk * elem(dims));
  void *vbuf = ws + 2 * align256(rows * dqk * elem(dims));
  PrefillArgs a{B, total_tokens, max_seqlen, dims->n_heads, dims->d_c, dims->d_rope, dims->d_nope, dims->d_v,
                cu_seqlens, q_nope, q_pe, w_uk, w_uv,
                CacheView{c_kv, k_pe, dims->ckv_stride, dims->kpe_stride, block_table, max_blocks_per_seq,
                          num_blocks, dims->block_size, dims->cache_layout, dims->d_c, dims->d_c + dims->d_rope},
                qbuf, kbuf, vbuf, out, lse, default_scale(*dims), dims->rope_base, dev_status, 0, 0, 0,
                static_cast<unsigned char *>(workspace), nullptr};
  return launch_prefill_simt(a, dims->dtype == MLA_BF16, reinterpret_cast<cudaStream_t>(stream));
}

static int cache_convert(const mla_dims *dims, const void *src, void *dst, int64_t num_rows, bool to_tiled,
                         mla_stream_t stream) {
  if (!dims || dims->dtype != MLA_BF16 || dims->d_c <= 0 || dims->d_rope < 0 || (dims->d_c + dims->d_rope) % 64)
    return MLA_ERR_INVALID_ARG;
  if (!src || !dst || num_rows < 0 || num_rows % 64) return MLA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst)) & 15) return MLA_ERR_INVALID_ARG;
  const int W = dims->d_c + dims->d_rope;
  const uintptr_t bytes = (uintptr_t)num_rows * W * 2;
  const uintptr_t a = reinterpret_cast<uintptr_t>(src), b = reinterpret_cast<uintptr_t>(dst);
  if (a < b + bytes && b < a + bytes) return MLA_ERR_INVALID_ARG;   // overlapping buffers
  return launch_cache_convert(src, dst, num_rows, W, to_tiled, reinterpret_cast<cudaStream_t>(stream));
}

int mla_cache_pack(const mla_dims *dims, const void *rows, void *tiled, int64_t num_rows, mla_stream_t stream) {
  return cache_convert(dims, rows, tiled, num_rows, true, stream);
}

int mla_cache_unpack(const mla_dims *dims, const void *tiled, void *rows, int64_t num_rows, mla_stream_t stream) {
  return cache_convert(dims, tiled, rows, num_rows, false, stream);
}

}  // extern "C"
