// Split-KV attention over the latent cache on CUDA cores (fp32 arithmetic).
//
// The absorbed decode form of "Transformer升级之路：21、MLA好在哪里?（下）",
// section 双重投影, decoding column: every head of a sequence scores the same
// cached row [c_i | kpe_i] with its own latent query, and the output is the
// softmax-weighted sum of the latents c_i.
//
// This kernel is the fp32 path (exact to fp32 rounding) and the general
// fallback for shapes the tensor-core kernel does not take.  CTA (b, split,
// row-group) stages kRowGrp query rows and kKeyTile cached rows at a time and
// keeps an online softmax per row; each split writes its output normalised by
// its own sum, plus its log-sum-exp, for the combine step.
#include <math_constants.h>

#include "kernels.cuh"

namespace mla {

constexpr int kAttnThreads = 256;
constexpr int kRowGrp = 16;     // query rows per CTA
constexpr int kKeyTile = 32;    // cached rows per pass (one per lane in the softmax)
constexpr int kMaxDcPerThr = 2; // d_c <= 512

template <typename T>
__global__ void __launch_bounds__(kAttnThreads)
attn_simt_kernel(AttnArgs a) {
  extern __shared__ float smem[];
  const int W = a.d_c + a.d_rope;
  const int ldk = W + 1;
  float *qs = smem;                              // [kRowGrp][W]
  float *ks = qs + kRowGrp * W;                  // [kKeyTile][W+1]
  float *ps = ks + kKeyTile * ldk;               // [kRowGrp][kKeyTile]
  float *alpha = ps + kRowGrp * kKeyTile;        // [kRowGrp]
  float *mrow = alpha + kRowGrp;                 // [kRowGrp]
  float *lrow = mrow + kRowGrp;                  // [kRowGrp]

  const int b = blockIdx.x, split = blockIdx.y;
  const int R = a.n_q * a.H;
  const int r0 = blockIdx.z * kRowGrp;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int S = a.seqlens[b];
  const int max_keys = a.max_chunks * a.chunk;
  const int64_t prow = ((int64_t)b * a.max_chunks + split) * R;
  if (S < a.n_q || S > max_keys) {
    if (tid == 0 && split == 0 && blockIdx.z == 0) report(a.dev_status, MLA_ERR_BAD_INDEX);
    // Leave finite, neutral partials so the combine stays well defined.
    for (int r = r0 + warp; r < min(r0 + kRowGrp, R); r += 8) {
      for (int c = lane; c < a.d_c; c += 32) a.o_part[(prow + r) * a.d_c + c] = 0.f;
      if (lane == 0) a.lse_part[prow + r] = -CUDART_INF_F;
    }
    return;
  }
  const int k_begin = max(split * a.chunk, a.kv_begin);
  const int k_end = min(min(S, split * a.chunk + a.chunk), a.kv_end);

  const T *q = static_cast<const T *>(a.q);
  for (int e = tid; e < kRowGrp * W; e += kAttnThreads) {
    const int r = e / W, d = e % W;
    qs[e] = (r0 + r < R) ? to_f32(q[((int64_t)b * R + r0 + r) * W + d]) : 0.f;
  }
  if (tid < kRowGrp) {
    mrow[tid] = -CUDART_INF_F;
    lrow[tid] = 0.f;
  }
  float acc[kRowGrp][kMaxDcPerThr];
#pragma unroll
  for (int r = 0; r < kRowGrp; ++r)
#pragma unroll
    for (int i = 0; i < kMaxDcPerThr; ++i) acc[r][i] = 0.f;

  for (int k0 = k_begin; k0 < k_end; k0 += kKeyTile) {
    __syncthreads();
    // Stage the tile's rows; rows past the end are zero (and masked below).
    for (int kk = warp; kk < kKeyTile; kk += 8) {
      const int key = k0 + kk;
      int64_t row = -1;
      if (key < k_end) {
        row = cache_row(a.cache.block_table, a.cache.max_blocks_per_seq, a.cache.num_blocks,
                        a.cache.block_size, b, key);
        if (row < 0 && lane == 0) report(a.dev_status, MLA_ERR_BAD_INDEX);
      }
      for (int d = lane; d < W; d += 32) {
        float v = 0.f;
        if (row >= 0) v = a.cache.load<T>(row, d);
        ks[kk * ldk + d] = v;
      }
    }
    __syncthreads();
    // Scores: thread -> (row, two keys).
    {
      const int r = tid / 16, kk = tid % 16;
      float s0 = 0.f, s1 = 0.f;
      for (int d = 0; d < W; ++d) {
        const float qv = qs[r * W + d];
        s0 = fmaf(qv, ks[kk * ldk + d], s0);
        s1 = fmaf(qv, ks[(kk + 16) * ldk + d], s1);
      }
      const int j = (r0 + r) / a.H;                   // query token of this row
      const int visible = S - a.n_q + j + 1;          // keys 0 .. visible-1
      ps[r * kKeyTile + kk] = (k0 + kk < visible && k0 + kk < k_end) ? s0 * a.scale : -CUDART_INF_F;
      ps[r * kKeyTile + kk + 16] = (k0 + kk + 16 < visible && k0 + kk + 16 < k_end) ? s1 * a.scale : -CUDART_INF_F;
    }
    __syncthreads();
    // Online softmax: warp w owns rows 2w, 2w+1; lane = key.
    for (int rr = 0; rr < 2; ++rr) {
      const int r = warp * 2 + rr;
      const float s = ps[r * kKeyTile + lane];
      float m = s;
#pragma unroll
      for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      const float m_old = mrow[r];
      const float m_new = fmaxf(m_old, m);
      const float p = (m_new == -CUDART_INF_F) ? 0.f : __expf(s - m_new);
      float sum = p;
#pragma unroll
      for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      ps[r * kKeyTile + lane] = p;
      __syncwarp();
      if (lane == 0) {
        const float al = (m_old == -CUDART_INF_F) ? 0.f : __expf(m_old - m_new);
        alpha[r] = al;
        lrow[r] = lrow[r] * al + sum;
        mrow[r] = m_new;
      }
    }
    __syncthreads();
    // O = alpha * O + P C: thread owns latent columns tid, tid + 256.
#pragma unroll
    for (int i = 0; i < kMaxDcPerThr; ++i) {
      const int c = tid + i * kAttnThreads;
      if (c < a.d_c) {
#pragma unroll
        for (int r = 0; r < kRowGrp; ++r) acc[r][i] *= alpha[r];
        for (int kk = 0; kk < kKeyTile; ++kk) {
          const float cv = ks[kk * ldk + c];
#pragma unroll
          for (int r = 0; r < kRowGrp; ++r) acc[r][i] = fmaf(ps[r * kKeyTile + kk], cv, acc[r][i]);
        }
      }
    }
  }
  __syncthreads();
#pragma unroll
  for (int r = 0; r < kRowGrp; ++r) {
    if (r0 + r >= R) break;
    const float l = lrow[r];
    const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
    for (int i = 0; i < kMaxDcPerThr; ++i) {
      const int c = tid + i * kAttnThreads;
      if (c < a.d_c) a.o_part[(prow + r0 + r) * a.d_c + c] = acc[r][i] * inv;
    }
    if (tid == 0) a.lse_part[prow + r0 + r] = l > 0.f ? mrow[r] + logf(l) : -CUDART_INF_F;
  }
}

int launch_attn_simt(const AttnArgs &a, bool bf16, cudaStream_t st) {
  if (a.d_c > kMaxDcPerThr * kAttnThreads) return MLA_ERR_UNSUPPORTED;
  const int W = a.d_c + a.d_rope;
  const size_t smem = sizeof(float) * (kRowGrp * W + kKeyTile * (W + 1) + kRowGrp * kKeyTile + 3 * kRowGrp);
  const int R = a.n_q * a.H;
  const dim3 grid(a.B, a.max_chunks, (R + kRowGrp - 1) / kRowGrp);
  if (bf16) {
    if (cudaFuncSetAttribute(attn_simt_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem))
      return MLA_ERR_CUDA;
    attn_simt_kernel<__nv_bfloat16><<<grid, kAttnThreads, smem, st>>>(a);
  } else {
    if (cudaFuncSetAttribute(attn_simt_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem))
      return MLA_ERR_CUDA;
    attn_simt_kernel<float><<<grid, kAttnThreads, smem, st>>>(a);
  }
  return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

}  // namespace mla
