// General strided, batched matrix product on CUDA cores (fp32 accumulation), and the RoPE of the
// query-latent path.  Used by the decode from hidden states with folded weights and by the
// offline weight folds:
//   c_Q = h W_DQ,  q_lat^(s) = c_Q W_UQK^(s),  q_pe^(s) = RoPE(c_Q W_QR^(s)),
//   u = sum_s o_lat^(s) W_UVO^(s),  W_UQK^(s) = W_UQ^(s) W_UK^(s)T,  W_UVO^(s) = W_UV^(s) W_O^(s)
// ("DeepSeek-V3 解读 1: MLA", sections "MLA：高层次的思路" and "为什么需要解耦 RoPE";
// "Transformer升级之路：21、MLA好在哪里?（下）", section 键值共享).
#include "kernels.cuh"

namespace mla {
namespace {

constexpr int kBM = 64, kBN = 64, kBK = 16, kGemmThreads = 256;

// C tile (64 x 64) of batch b and K-split ks: thread (ty, tx) owns rows ty + 16i, columns tx + 16j.
template <typename T>
__global__ void __launch_bounds__(kGemmThreads) gemm_simt_kernel(GemmArgs g) {
  __shared__ float As[kBK][kBM + 1];
  __shared__ float Bs[kBK][kBN + 1];
  const int n0 = blockIdx.x * kBN, m0 = blockIdx.y * kBM;
  const int b = blockIdx.z / g.ksplit, ks = blockIdx.z % g.ksplit;
  const int kc = ((g.K + g.ksplit - 1) / g.ksplit + kBK - 1) / kBK * kBK;
  const int k_lo = ks * kc, k_hi = min(g.K, k_lo + kc);
  const int tid = threadIdx.x, tx = tid % 16, ty = tid / 16;
  const T *A = static_cast<const T *>(g.A) + b * g.sa_b;
  const T *Bm = static_cast<const T *>(g.B) + b * g.sb_b;
  float acc[4][4] = {};
  for (int k0 = k_lo; k0 < k_hi; k0 += kBK) {
    for (int e = tid; e < kBK * kBM; e += kGemmThreads) {
      const int kk = e / kBM, mm = e % kBM;       // consecutive threads: consecutive rows of A
      const int m = m0 + mm, k = k0 + kk;
      As[kk][mm] = (m < g.M && k < k_hi) ? to_f32(A[m * g.sa_m + k * g.sa_k]) : 0.f;
    }
    for (int e = tid; e < kBK * kBN; e += kGemmThreads) {
      const int kk = e / kBN, nn = e % kBN;       // consecutive threads: consecutive columns of B
      const int n = n0 + nn, k = k0 + kk;
      Bs[kk][nn] = (n < g.N && k < k_hi) ? to_f32(Bm[k * g.sb_k + n * g.sb_n]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kBK; ++kk) {
      float a[4], bv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty + 16 * i];
#pragma unroll
      for (int j = 0; j < 4; ++j) bv[j] = Bs[kk][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int m = m0 + ty + 16 * i, n = n0 + tx + 16 * j;
      if (m >= g.M || n >= g.N) continue;
      if (g.ksplit == 1)
        static_cast<T *>(g.C)[b * g.sc_b + m * g.sc_m + n * g.sc_n] = from_f32<T>(acc[i][j]);
      else
        g.part[(((int64_t)b * g.ksplit + ks) * g.M + m) * g.N + n] = acc[i][j];
    }
}

template <typename T>
__global__ void gemm_reduce_kernel(GemmArgs g) {
  const int64_t n = (int64_t)g.batch * g.M * g.N;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
    const int col = (int)(e % g.N);
    const int64_t rest = e / g.N;
    const int m = (int)(rest % g.M), b = (int)(rest / g.M);
    float v = 0.f;
    for (int ks = 0; ks < g.ksplit; ++ks) v += g.part[(((int64_t)b * g.ksplit + ks) * g.M + m) * g.N + col];
    static_cast<T *>(g.C)[b * g.sc_b + m * g.sc_m + col * g.sc_n] = from_f32<T>(v);
  }
}

// q_abs[t, s, d_c + 2i, 2i+1] = RoPE(q_pe_raw[t, s, 2i .. 2i+1], seqlens[b] - n_q + j), t = b n_q + j.
template <typename T>
__global__ void rope_into_query_kernel(int B, int n_q, int H, int d_c, int d_rope, const T *q_pe_raw,
                                       const int32_t *seqlens, T *q_abs, float rope_base) {
  const int half = d_rope / 2;
  const int64_t n = (int64_t)B * n_q * H * half;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
    const int i = (int)(e % half);
    const int64_t ts = e / half;                  // t * H + s
    const int t = (int)(ts / H);
    const int pos = max(0, seqlens[t / n_q] - n_q + t % n_q);
    float c, sn;
    rope_cos_sin(pos, i, d_rope, rope_base, &c, &sn);
    const float x = to_f32(q_pe_raw[ts * d_rope + 2 * i]), y = to_f32(q_pe_raw[ts * d_rope + 2 * i + 1]);
    T *dst = q_abs + ts * (d_c + d_rope) + d_c + 2 * i;
    dst[0] = from_f32<T>(x * c - y * sn);
    dst[1] = from_f32<T>(x * sn + y * c);
  }
}

}  // namespace

size_t gemm_simt_workspace(const GemmArgs &g) {
  return g.ksplit > 1 ? (size_t)g.batch * g.ksplit * g.M * g.N * sizeof(float) : 0;
}

int launch_gemm_simt(const GemmArgs &g, bool bf16, cudaStream_t st) {
  if (g.M <= 0 || g.N <= 0 || g.K <= 0 || g.batch <= 0 || g.ksplit <= 0) return MLA_ERR_INVALID_ARG;
  if (g.ksplit > 1 && !g.part) return MLA_ERR_WORKSPACE;
  const dim3 grid((g.N + kBN - 1) / kBN, (g.M + kBM - 1) / kBM, g.batch * g.ksplit);
  if (bf16) gemm_simt_kernel<__nv_bfloat16><<<grid, kGemmThreads, 0, st>>>(g);
  else gemm_simt_kernel<float><<<grid, kGemmThreads, 0, st>>>(g);
  if (g.ksplit > 1) {
    if (bf16) gemm_reduce_kernel<__nv_bfloat16><<<592, 256, 0, st>>>(g);
    else gemm_reduce_kernel<float><<<592, 256, 0, st>>>(g);
  }
  return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

int launch_gemm_reduce(const GemmArgs &g, bool bf16, cudaStream_t st) {
  if (bf16) gemm_reduce_kernel<__nv_bfloat16><<<592, 256, 0, st>>>(g);
  else gemm_reduce_kernel<float><<<592, 256, 0, st>>>(g);
  return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

int launch_gemm(const GemmArgs &g, bool bf16, cudaStream_t st) {
  const int rc = launch_gemm_tc(g, bf16, st);
  return rc == MLA_ERR_UNSUPPORTED ? launch_gemm_simt(g, bf16, st) : rc;
}

int launch_rope_into_query(int B, int n_q, int H, int d_c, int d_rope, const void *q_pe_raw, const int32_t *seqlens,
                           void *q_abs, float rope_base, bool bf16, cudaStream_t st) {
  if (d_rope == 0) return MLA_OK;
  if (bf16)
    rope_into_query_kernel<<<592, 256, 0, st>>>(B, n_q, H, d_c, d_rope, static_cast<const __nv_bfloat16 *>(q_pe_raw),
                                                seqlens, static_cast<__nv_bfloat16 *>(q_abs), rope_base);
  else
    rope_into_query_kernel<<<592, 256, 0, st>>>(B, n_q, H, d_c, d_rope, static_cast<const float *>(q_pe_raw), seqlens,
                                                static_cast<float *>(q_abs), rope_base);
  return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

}  // namespace mla
