// Combine of split-KV partials and the per-head value up-projection.
//
// Each split k of a query row carries (O_k normalised by its own softmax sum,
// lse_k).  The exact softmax over the whole sequence is
//   LSE = log sum_k exp(lse_k),  o_lat = sum_k exp(lse_k - LSE) O_k,
// and the decode output of head s is out^(s) = o_lat W_UV^(s)
// ("Transformer升级之路：21、MLA好在哪里?（下）", section 双重投影, decoding
// column: o_t = [o^(1) W_v^(1), ..., o^(h) W_v^(h)]).
//
// CTA (s, row-group) merges kCombRows (b, j) rows of head s into shared memory
// and multiplies them by W_UV[s], so W_UV[s] is read once per row group.
#include <math_constants.h>

#include "kernels.cuh"

namespace mla {

constexpr int kCombThreads = 256;
constexpr int kCombRows = 16;

template <typename T>
__global__ void __launch_bounds__(kCombThreads)
combine_kernel(CombineArgs a) {
  extern __shared__ float smem[];
  float *ol = smem;                            // [kCombRows][d_c]
  float *wgt = ol + kCombRows * a.d_c;         // [kCombRows][max_chunks]
  const int s = blockIdx.x;
  const int g0 = blockIdx.y * kCombRows;       // first (b, j) row
  const int rows = a.B * a.n_q;
  const int R = a.n_q * a.H;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // Split weights: warp w handles rows w and w + 8.
  for (int rr = warp; rr < kCombRows; rr += 8) {
    const int g = g0 + rr;
    float *wr = wgt + rr * a.max_chunks;
    if (g >= rows) {
      for (int k = lane; k < a.max_chunks; k += 32) wr[k] = 0.f;
      continue;
    }
    const int b = g / a.n_q, j = g % a.n_q;
    const int S = a.seqlens[b];
    int nsplit = (S + a.chunk - 1) / a.chunk;
    nsplit = max(0, min(nsplit, a.max_chunks));
    const int64_t base = (int64_t)b * a.max_chunks * R + (int64_t)j * a.H + s;
    float m = -CUDART_INF_F;
    for (int k = lane; k < nsplit; k += 32) m = fmaxf(m, a.lse_part[base + (int64_t)k * R]);
#pragma unroll
    for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float sum = 0.f;
    for (int k = lane; k < a.max_chunks; k += 32) {
      const float e = (k < nsplit && m != -CUDART_INF_F) ? __expf(a.lse_part[base + (int64_t)k * R] - m) : 0.f;
      wr[k] = e;
      sum += e;
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    const float inv = sum > 0.f ? 1.f / sum : 0.f;
    for (int k = lane; k < a.max_chunks; k += 32) wr[k] *= inv;
    if (lane == 0 && a.lse) a.lse[(int64_t)g * a.H + s] = sum > 0.f ? m + logf(sum) : -CUDART_INF_F;
  }
  __syncthreads();
  for (int e = tid; e < kCombRows * a.d_c; e += kCombThreads) {
    const int rr = e / a.d_c, c = e % a.d_c;
    const int g = g0 + rr;
    float v = 0.f;
    if (g < rows) {
      const int b = g / a.n_q, j = g % a.n_q;
      const int64_t base = (int64_t)b * a.max_chunks * R + (int64_t)j * a.H + s;
      const float *wr = wgt + rr * a.max_chunks;
      for (int k = 0; k < a.max_chunks; ++k) {
        const float w = wr[k];
        if (w != 0.f) v = fmaf(w, a.o_part[(base + (int64_t)k * R) * a.d_c + c], v);
      }
    }
    ol[e] = v;
  }
  __syncthreads();
  T *out = static_cast<T *>(a.out);
  if (!a.w_uv) {
    for (int e = tid; e < kCombRows * a.d_c; e += kCombThreads) {
      const int rr = e / a.d_c, c = e % a.d_c;
      const int g = g0 + rr;
      if (g < rows) out[((int64_t)g * a.H + s) * a.d_c + c] = from_f32<T>(ol[e]);
    }
    return;
  }
  const T *w = static_cast<const T *>(a.w_uv) + (int64_t)s * a.d_c * a.d_v;
  for (int v = tid; v < a.d_v; v += kCombThreads) {
    float acc[kCombRows];
#pragma unroll
    for (int r = 0; r < kCombRows; ++r) acc[r] = 0.f;
    for (int c = 0; c < a.d_c; ++c) {
      const float wv = to_f32(w[(int64_t)c * a.d_v + v]);
#pragma unroll
      for (int r = 0; r < kCombRows; ++r) acc[r] = fmaf(ol[r * a.d_c + c], wv, acc[r]);
    }
#pragma unroll
    for (int r = 0; r < kCombRows; ++r) {
      const int g = g0 + r;
      if (g < rows) out[((int64_t)g * a.H + s) * a.d_v + v] = from_f32<T>(acc[r]);
    }
  }
}

int launch_combine(const CombineArgs &a, bool bf16, cudaStream_t st) {
  const size_t smem = sizeof(float) * (kCombRows * a.d_c + kCombRows * a.max_chunks);
  if (smem > 220 * 1024) return MLA_ERR_UNSUPPORTED;
  const dim3 grid(a.H, (a.B * a.n_q + kCombRows - 1) / kCombRows);
  if (bf16) {
    if (cudaFuncSetAttribute(combine_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem))
      return MLA_ERR_CUDA;
    combine_kernel<__nv_bfloat16><<<grid, kCombThreads, smem, st>>>(a);
  } else {
    if (cudaFuncSetAttribute(combine_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem))
      return MLA_ERR_CUDA;
    combine_kernel<float><<<grid, kCombThreads, smem, st>>>(a);
  }
  return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

}  // namespace mla
