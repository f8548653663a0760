// Query absorption: q_lat = W_UK q_nope (d_nope -> d_c) and the RoPE of q_pe.
//
// "Transformer升级之路：21、MLA好在哪里?（下）", section 双重投影, decoding
// column: the per-head key up-projection is folded into the query, which then
// lives in the d_c-wide latent space.  "DeepSeek-V3 解读 1: MLA", section
// "为什么需要解耦 RoPE": the RoPE part of the query is rotated separately.
//
// The step reads W_UK once ([H, d_c, d_nope], 16.8 MB at V3 shapes): CTA
// (s, c-slice) keeps a 64 x d_nope slice of W_UK[s] in shared memory and runs
// every (b, j) query row of head s against it.
#include "kernels.cuh"

namespace mla {

constexpr int kAbsThreads = 256;
constexpr int kAbsCols = 64;     // latent columns per CTA
constexpr int kAbsRows = 16;     // query rows staged per pass

template <typename T>
__global__ void __launch_bounds__(kAbsThreads)
absorb_q_kernel(AbsorbArgs a) {
  extern __shared__ float smem[];
  const int s = blockIdx.x;                 // head
  const int c0 = blockIdx.y * kAbsCols;     // first latent column
  const int dn = a.d_nope;
  const int ld = dn + 1;                    // padded row of the W slice
  float *ws = smem;                         // [kAbsCols][dn+1]
  float *qs = smem + kAbsCols * ld;         // [kAbsRows][dn]
  const T *wuk = static_cast<const T *>(a.w_uk) + (int64_t)s * a.d_c * dn;
  const T *qn = static_cast<const T *>(a.q_nope);
  T *qo = static_cast<T *>(a.q_out);
  const int W = a.d_c + a.d_rope;
  const int rows = a.B * a.n_q;
  const int tid = threadIdx.x;
  const int ncols = min(kAbsCols, a.d_c - c0);

  for (int e = tid; e < kAbsCols * dn; e += kAbsThreads) {
    const int c = e / dn, n = e % dn;
    ws[c * ld + n] = c < ncols ? to_f32(wuk[(int64_t)(c0 + c) * dn + n]) : 0.f;
  }
  const int c = tid % kAbsCols;
  const int rg = tid / kAbsCols;            // 0..3
  for (int r0 = 0; r0 < rows; r0 += kAbsRows) {
    __syncthreads();
    for (int e = tid; e < kAbsRows * dn; e += kAbsThreads) {
      const int r = e / dn, n = e % dn;
      qs[e] = (r0 + r < rows) ? to_f32(qn[((int64_t)(r0 + r) * a.H + s) * dn + n]) : 0.f;
    }
    __syncthreads();
    float acc[kAbsRows / 4];
#pragma unroll
    for (int i = 0; i < kAbsRows / 4; ++i) acc[i] = 0.f;
    for (int n = 0; n < dn; ++n) {
      const float w = ws[c * ld + n];
#pragma unroll
      for (int i = 0; i < kAbsRows / 4; ++i) acc[i] = fmaf(qs[(rg + 4 * i) * dn + n], w, acc[i]);
    }
    if (c < ncols) {
#pragma unroll
      for (int i = 0; i < kAbsRows / 4; ++i) {
        const int r = r0 + rg + 4 * i;
        if (r < rows) qo[((int64_t)r * a.H + s) * W + c0 + c] = from_f32<T>(acc[i]);
      }
    }
  }

  // RoPE part: the CTAs of the first latent slice also rotate q_pe of head s.
  if (blockIdx.y != 0) return;
  const T *qp = static_cast<const T *>(a.q_pe);
  const int half = a.d_rope / 2;
  for (int e = tid; e < rows * half; e += kAbsThreads) {
    const int r = e / half, i = e % half;
    const int b = r / a.n_q, j = r % a.n_q;
    const int p = a.seqlens[b] - a.n_q + j;
    float cs, sn;
    rope_cos_sin(p < 0 ? 0 : p, i, a.d_rope, a.rope_base, &cs, &sn);
    const int64_t src = ((int64_t)r * a.H + s) * a.d_rope + 2 * i;
    const float x = to_f32(qp[src]), y = to_f32(qp[src + 1]);
    T *dst = qo + ((int64_t)r * a.H + s) * W + a.d_c + 2 * i;
    dst[0] = from_f32<T>(x * cs - y * sn);
    dst[1] = from_f32<T>(x * sn + y * cs);
  }
}

int launch_absorb(const AbsorbArgs &a, bool bf16, cudaStream_t st) {
  const size_t smem = sizeof(float) * (kAbsCols * (a.d_nope + 1) + kAbsRows * a.d_nope);
  const dim3 grid(a.H, (a.d_c + kAbsCols - 1) / kAbsCols);
  if (bf16) {
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(absorb_q_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem))
      return MLA_ERR_CUDA;
    absorb_q_kernel<__nv_bfloat16><<<grid, kAbsThreads, smem, st>>>(a);
  } else {
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(absorb_q_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem))
      return MLA_ERR_CUDA;
    absorb_q_kernel<float><<<grid, kAbsThreads, smem, st>>>(a);
  }
  return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

}  // namespace mla
