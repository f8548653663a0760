// Causal prefill in the decompressed multi-head form, on CUDA cores.
//
// "Transformer升级之路：21、MLA好在哪里?（下）", section 双重投影, training /
// prefill column: per head s, k_i = c_i W_k^(s), v_i = c_i W_v^(s) and
// o_t = softmax_{i<=t}(q_t k_i^T) v; with the decoupled RoPE of "DeepSeek-V3
// 解读 1: MLA" (section "为什么需要解耦 RoPE") the key is [c_i W_UK^(s) | kpe_i]
// and the query [q_nope | RoPE(q_pe, t)].
//
// Three steps: (1) build the rotated queries, (2) decompress K and V of every
// cached token per head into the workspace, (3) flash-style causal attention.
#include <math_constants.h>

#include "kernels.cuh"

namespace mla {

constexpr int kPfThreads = 256;

// (1) qbuf[t, s, :] = [q_nope | RoPE(q_pe, position of t)]
// One CTA per query token: the token's position and its d_R/2 rotation angles are computed once
// and shared by every head; then one element per thread, in row order (coalesced).
template <typename T>
__global__ void __launch_bounds__(kPfThreads) prefill_q_kernel(PrefillArgs a) {
  extern __shared__ float rot[];          // [d_rope / 2][2]: cos, sin
  __shared__ int pos_s, seq_s;
  const int t = blockIdx.x;
  if (threadIdx.x == 0) {                 // position of row t within its sequence
    int lo = 0, hi = a.B;                 // find b with cu[b] <= t < cu[b+1]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (a.cu_seqlens[mid] <= t) lo = mid; else hi = mid;
    }
    pos_s = t - a.cu_seqlens[lo];
    seq_s = lo;
  }
  __syncthreads();
  const int pos = pos_s, seq = seq_s;
  for (int i = threadIdx.x; i < (a.d_rope >> 1); i += blockDim.x)
    rope_cos_sin(pos, i, a.d_rope, a.rope_base, &rot[2 * i], &rot[2 * i + 1]);
  __syncthreads();
  const int dqk = a.d_nope + a.d_rope;
  const T *qn = static_cast<const T *>(a.q_nope) + (int64_t)t * a.H * a.d_nope;
  const T *qp = static_cast<const T *>(a.q_pe) + (int64_t)t * a.H * a.d_rope;
  T *qb = static_cast<T *>(a.qbuf) + (int64_t)t * a.H * dqk;
  // Tiled workspace: row pos % 128 of tile pos / 128 of (head s, sequence seq).
  for (int e = threadIdx.x; e < a.H * dqk; e += blockDim.x) {
    const int s = e / dqk, d = e % dqk;
    T v;
    if (d < a.d_nope) {
      v = qn[s * a.d_nope + d];
    } else {
      const int dr = d - a.d_nope, i = dr >> 1;
      const float x = to_f32(qp[s * a.d_rope + 2 * i]), y = to_f32(qp[s * a.d_rope + 2 * i + 1]);
      const float c = rot[2 * i], sn = rot[2 * i + 1];
      v = from_f32<T>((dr & 1) ? (x * sn + y * c) : (x * c - y * sn));
    }
    if (a.tiled)
      *reinterpret_cast<T *>(a.q_tiles + (((int64_t)s * a.B + seq) * a.nqt + pos / 128) * kPfQTileBytes +
                             swz_tile_offset(128, pos % 128, d)) = v;
    else
      qb[e] = v;
  }
}

// (2) kbuf[t, s, :] = [c_t W_UK[s] | kpe_t], vbuf[t, s, :] = c_t W_UV[s]
constexpr int kDecRows = 16;
template <typename T>
__global__ void __launch_bounds__(kPfThreads)
prefill_decompress_kernel(PrefillArgs a) {
  extern __shared__ float smem[];
  float *cs = smem;                        // [kDecRows][d_c]
  const int s = blockIdx.x;
  const int t0 = blockIdx.y * kDecRows;
  const int tid = threadIdx.x;
  const int dqk = a.d_nope + a.d_rope;
  __shared__ int64_t rows[kDecRows];
  if (tid < kDecRows) {
    const int t = t0 + tid;
    int64_t row = -1;
    if (t < a.total) {
      int lo = 0, hi = a.B;
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (a.cu_seqlens[mid] <= t) lo = mid; else hi = mid;
      }
      row = cache_row(a.cache.block_table, a.cache.max_blocks_per_seq, a.cache.num_blocks,
                      a.cache.block_size, lo, t - a.cu_seqlens[lo]);
      if (row < 0) report(a.dev_status, MLA_ERR_BAD_INDEX);
    }
    rows[tid] = row;
  }
  __syncthreads();
  for (int e = tid; e < kDecRows * a.d_c; e += kPfThreads) {
    const int r = e / a.d_c, c = e % a.d_c;
    cs[e] = rows[r] >= 0 ? a.cache.load<T>(rows[r], c) : 0.f;
  }
  __syncthreads();
  T *kb = static_cast<T *>(a.kbuf);
  T *vb = static_cast<T *>(a.vbuf);
  const T *wuk = static_cast<const T *>(a.w_uk) + (int64_t)s * a.d_c * a.d_nope;
  const T *wuv = static_cast<const T *>(a.w_uv) + (int64_t)s * a.d_c * a.d_v;
  for (int col = tid; col < a.d_nope + a.d_v; col += kPfThreads) {
    const bool isk = col < a.d_nope;
    const T *w = isk ? wuk + col : wuv + (col - a.d_nope);
    const int ldw = isk ? a.d_nope : a.d_v;
    float acc[kDecRows];
#pragma unroll
    for (int r = 0; r < kDecRows; ++r) acc[r] = 0.f;
    for (int c = 0; c < a.d_c; ++c) {
      const float wv = to_f32(w[(int64_t)c * ldw]);
#pragma unroll
      for (int r = 0; r < kDecRows; ++r) acc[r] = fmaf(cs[r * a.d_c + c], wv, acc[r]);
    }
#pragma unroll
    for (int r = 0; r < kDecRows; ++r) {
      const int t = t0 + r;
      if (t >= a.total) break;
      if (isk) kb[((int64_t)t * a.H + s) * dqk + col] = from_f32<T>(acc[r]);
      else vb[((int64_t)t * a.H + s) * a.d_v + (col - a.d_nope)] = from_f32<T>(acc[r]);
    }
  }
  for (int e = tid; e < kDecRows * a.d_rope; e += kPfThreads) {
    const int r = e / a.d_rope, d = e % a.d_rope;
    const int t = t0 + r;
    if (t < a.total && rows[r] >= 0)
      kb[((int64_t)t * a.H + s) * dqk + a.d_nope + d] = from_f32<T>(a.cache.load<T>(rows[r], a.d_c + d));
  }
}

// (3) causal attention: CTA (b, s, 16-row query tile), keys in tiles of 32.
constexpr int kPfRows = 16, kPfKeys = 32;
template <typename T>
__global__ void __launch_bounds__(kPfThreads)
prefill_attn_kernel(PrefillArgs a) {
  extern __shared__ float smem[];
  const int dqk = a.d_nope + a.d_rope;
  const int ldk = dqk + 1, ldv = a.d_v + 1;
  float *qs = smem;                         // [kPfRows][dqk]
  float *ks = qs + kPfRows * dqk;           // [kPfKeys][dqk+1]
  float *vs = ks + kPfKeys * ldk;           // [kPfKeys][d_v+1]
  float *ps = vs + kPfKeys * ldv;           // [kPfRows][kPfKeys]
  float *alpha = ps + kPfRows * kPfKeys;
  float *mrow = alpha + kPfRows;
  float *lrow = mrow + kPfRows;
  const int b = blockIdx.x, s = blockIdx.y;
  const int start = a.cu_seqlens[b], L = a.cu_seqlens[b + 1] - start;
  const int q0 = blockIdx.z * kPfRows;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (start < 0 || L < 0 || start + L > a.total || L > a.max_seqlen) {
    if (tid == 0 && s == 0 && blockIdx.z == 0) report(a.dev_status, MLA_ERR_BAD_INDEX);
    return;
  }
  if (q0 >= L) return;
  const T *qb = static_cast<const T *>(a.qbuf);
  const T *kb = static_cast<const T *>(a.kbuf);
  const T *vb = static_cast<const T *>(a.vbuf);
  for (int e = tid; e < kPfRows * dqk; e += kPfThreads) {
    const int r = e / dqk, d = e % dqk;
    qs[e] = q0 + r < L ? to_f32(qb[((int64_t)(start + q0 + r) * a.H + s) * dqk + d]) : 0.f;
  }
  if (tid < kPfRows) { mrow[tid] = -CUDART_INF_F; lrow[tid] = 0.f; }
  constexpr int kVPerThr = 8;               // d_v <= 8 * 32 columns, 16 rows / 8 warps = 2 rows per warp
  float acc[2][kVPerThr];
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int c = 0; c < kVPerThr; ++c) acc[i][c] = 0.f;
  const int kmax = min(L, q0 + kPfRows);    // causal: the tile's last row sees keys < q0 + 16
  for (int k0 = 0; k0 < kmax; k0 += kPfKeys) {
    __syncthreads();
    for (int e = tid; e < kPfKeys * dqk; e += kPfThreads) {
      const int kk = e / dqk, d = e % dqk;
      ks[kk * ldk + d] = k0 + kk < L ? to_f32(kb[((int64_t)(start + k0 + kk) * a.H + s) * dqk + d]) : 0.f;
    }
    for (int e = tid; e < kPfKeys * a.d_v; e += kPfThreads) {
      const int kk = e / a.d_v, d = e % a.d_v;
      vs[kk * ldv + d] = k0 + kk < L ? to_f32(vb[((int64_t)(start + k0 + kk) * a.H + s) * a.d_v + d]) : 0.f;
    }
    __syncthreads();
    {
      const int r = tid / 16, kk = tid % 16;
      float s0 = 0.f, s1 = 0.f;
      for (int d = 0; d < dqk; ++d) {
        const float qv = qs[r * dqk + d];
        s0 = fmaf(qv, ks[kk * ldk + d], s0);
        s1 = fmaf(qv, ks[(kk + 16) * ldk + d], s1);
      }
      const int t = q0 + r;
      ps[r * kPfKeys + kk] = (k0 + kk <= t && t < L) ? s0 * a.scale : -CUDART_INF_F;
      ps[r * kPfKeys + kk + 16] = (k0 + kk + 16 <= t && t < L) ? s1 * a.scale : -CUDART_INF_F;
    }
    __syncthreads();
    for (int rr = 0; rr < 2; ++rr) {
      const int r = warp * 2 + rr;
      const float sc = ps[r * kPfKeys + lane];
      float m = sc;
#pragma unroll
      for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      const float m_old = mrow[r], m_new = fmaxf(m_old, m);
      const float p = m_new == -CUDART_INF_F ? 0.f : __expf(sc - m_new);
      float sum = p;
#pragma unroll
      for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      ps[r * kPfKeys + lane] = p;
      __syncwarp();
      if (lane == 0) {
        const float al = m_old == -CUDART_INF_F ? 0.f : __expf(m_old - m_new);
        alpha[r] = al;
        lrow[r] = lrow[r] * al + sum;
        mrow[r] = m_new;
      }
    }
    __syncthreads();
    // warp w owns rows 2w, 2w+1; lane owns value columns lane + 32 c.
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int r = warp * 2 + i;
      const float al = alpha[r];
#pragma unroll
      for (int c = 0; c < kVPerThr; ++c) acc[i][c] *= al;
      for (int kk = 0; kk < kPfKeys; ++kk) {
        const float p = ps[r * kPfKeys + kk];
#pragma unroll
        for (int c = 0; c < kVPerThr; ++c) {
          const int col = lane + 32 * c;
          if (col < a.d_v) acc[i][c] = fmaf(p, vs[kk * ldv + col], acc[i][c]);
        }
      }
    }
  }
  __syncthreads();
  T *out = static_cast<T *>(a.out);
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int r = warp * 2 + i, t = q0 + r;
    if (t >= L) continue;
    const float l = lrow[r], inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
    for (int c = 0; c < kVPerThr; ++c) {
      const int col = lane + 32 * c;
      if (col < a.d_v) out[((int64_t)(start + t) * a.H + s) * a.d_v + col] = from_f32<T>(acc[i][c] * inv);
    }
    if (lane == 0 && a.lse) a.lse[(int64_t)(start + t) * a.H + s] = mrow[r] + logf(l);
  }
}

template <typename T>
static int launch_prefill_t(PrefillArgs a, cudaStream_t st) {
  const int dqk = a.d_nope + a.d_rope;
  // Both tensor-core steps available: Q, K and V go to the tiled workspace (one bulk copy per tile).
  if (sizeof(T) == 2 && decompress_tc_supported(a, true) && prefill_tc_supported(a, true)) {
    a.tiled = 1;
    a.nqt = (a.max_seqlen + 127) / 128;
    a.nkt = 2 * a.nqt;
    const size_t qbytes = (size_t)a.H * a.B * a.nqt * kPfQTileBytes;
    a.kv_tiles = a.q_tiles + ((qbytes + 255) & ~size_t(255));
  }
  prefill_q_kernel<T><<<a.total, kPfThreads, sizeof(float) * a.d_rope, st>>>(a);
  const size_t smem_dec = sizeof(float) * kDecRows * a.d_c;
  if (cudaFuncSetAttribute(prefill_decompress_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_dec))
    return MLA_ERR_CUDA;
  if (decompress_tc_supported(a, sizeof(T) == 2)) {
    if (const int rc = launch_decompress_tc(a, st)) return rc;
  } else {
    prefill_decompress_kernel<T><<<dim3(a.H, (a.total + kDecRows - 1) / kDecRows), kPfThreads, smem_dec, st>>>(a);
  }
  if (cudaGetLastError() != cudaSuccess) return MLA_ERR_CUDA;
  // Step (3) on the tensor cores where the shape allows it (bf16, 192-wide keys, 128-wide values).
  if (prefill_tc_supported(a, sizeof(T) == 2)) return launch_prefill_tc_attention(a, st);
  const size_t smem_att = sizeof(float) * (kPfRows * dqk + kPfKeys * (dqk + 1) + kPfKeys * (a.d_v + 1) +
                                           kPfRows * kPfKeys + 3 * kPfRows);
  if (cudaFuncSetAttribute(prefill_attn_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_att))
    return MLA_ERR_CUDA;
  prefill_attn_kernel<T><<<dim3(a.B, a.H, (a.max_seqlen + kPfRows - 1) / kPfRows), kPfThreads, smem_att, st>>>(a);
  return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

int launch_prefill_simt(const PrefillArgs &a, bool bf16, cudaStream_t st) {
  if (a.d_v > 256) return MLA_ERR_UNSUPPORTED;
  return bf16 ? launch_prefill_t<__nv_bfloat16>(a, st) : launch_prefill_t<float>(a, st);
}

}  // namespace mla
