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
    int nsplit = a.max_chunks;
    if (a.seqlens) {
      const int S = a.seqlens[b];
      nsplit = max(0, min((S + a.chunk - 1) / a.chunk, a.max_chunks));
    }
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

// Partials of N devices (each normalised over its own key range, with its lse) laid out as the N
// splits of every query row, in fp32.
template <typename T>
__global__ void partials_to_splits_kernel(int N, int B, int R, int d_c, const T *o_parts, const float *lse_parts,
                                          float *o_part, float *lse_part) {
  const int64_t per = (int64_t)B * R;                 // query rows of one device's partial
  const int64_t n = (int64_t)N * per * d_c;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
    const int c = (int)(e % d_c);
    const int64_t row = e / d_c;                      // r * per + b * R + q
    const int r = (int)(row / per);
    const int64_t rem = row % per;
    const int b = (int)(rem / R), q = (int)(rem % R);
    const int64_t dst = ((int64_t)b * N + r) * R + q;
    o_part[dst * d_c + c] = to_f32(o_parts[e]);
    if (c == 0) lse_part[dst] = lse_parts[row];
  }
}

int launch_partials_to_splits(int N, int B, int n_q, int H, int d_c, const void *o_parts, const float *lse_parts,
                              bool bf16, float *o_part, float *lse_part, cudaStream_t st) {
  const int R = n_q * H;
  if (bf16)
    partials_to_splits_kernel<<<1184, 256, 0, st>>>(N, B, R, d_c, static_cast<const __nv_bfloat16 *>(o_parts),
                                                   lse_parts, o_part, lse_part);
  else
    partials_to_splits_kernel<<<1184, 256, 0, st>>>(N, B, R, d_c, static_cast<const float *>(o_parts), lse_parts,
                                                   o_part, lse_part);
  return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
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
