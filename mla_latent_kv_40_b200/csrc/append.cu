// Latent-cache append: c_KV = RMSNorm(h W_DKV), k_pe = RoPE(h W_KR, pos),
// scattered into the paged pool.
//
// "DeepSeek-V3 解读 1: MLA", section "MLA：高层次的思路" (down-projection to the
// cached latent) and section "为什么需要解耦 RoPE" (a separate RoPE key shared
// by all heads; the latent itself is not rotated).
//
// One CTA handles kTok tokens against all d_c + d_R output columns, so each
// weight element read from L2 serves kTok tokens.  The weights (d_model x 576
// bf16 = 8.3 MB at V3 shapes) dominate the traffic of a decode-size append.
#include "kernels.cuh"

namespace mla {

constexpr int kAppendTok = 8;        // tokens per CTA (one warp per token in the epilogue)
constexpr int kAppendThreads = 256;
constexpr int kAppendKChunk = 128;   // d_model slice staged in shared memory
constexpr int kAppendMaxCols = 4;    // columns per thread: d_c + d_R <= 1024

template <typename T>
__global__ void __launch_bounds__(kAppendThreads)
append_latent_kernel(AppendArgs a) {
  extern __shared__ float smem[];
  const int W = a.d_c + a.d_rope;
  float *hs = smem;                                   // [kAppendTok][kAppendKChunk]
  float *cs = smem + kAppendTok * kAppendKChunk;      // [kAppendTok][W]
  const T *h = static_cast<const T *>(a.h);
  const T *wd = static_cast<const T *>(a.w_dkv);
  const T *wk = static_cast<const T *>(a.w_kr);
  const int t0 = blockIdx.x * kAppendTok;
  const int ntok = min(kAppendTok, a.T - t0);
  const int tid = threadIdx.x;

  float acc[kAppendMaxCols][kAppendTok];
#pragma unroll
  for (int i = 0; i < kAppendMaxCols; ++i)
#pragma unroll
    for (int t = 0; t < kAppendTok; ++t) acc[i][t] = 0.f;

  for (int k0 = 0; k0 < a.d_model; k0 += kAppendKChunk) {
    const int kn = min(kAppendKChunk, a.d_model - k0);
    for (int e = tid; e < kAppendTok * kAppendKChunk; e += kAppendThreads) {
      const int t = e / kAppendKChunk, k = e % kAppendKChunk;
      hs[e] = (t < ntok && k < kn) ? to_f32(h[(int64_t)(t0 + t) * a.d_model + k0 + k]) : 0.f;
    }
    __syncthreads();
    for (int k = 0; k < kn; ++k) {
#pragma unroll
      for (int i = 0; i < kAppendMaxCols; ++i) {
        const int col = tid + i * kAppendThreads;
        if (col < W) {
          const float w = col < a.d_c ? to_f32(wd[(int64_t)(k0 + k) * a.d_c + col])
                                      : to_f32(wk[(int64_t)(k0 + k) * a.d_rope + (col - a.d_c)]);
#pragma unroll
          for (int t = 0; t < kAppendTok; ++t) acc[i][t] = fmaf(hs[t * kAppendKChunk + k], w, acc[i][t]);
        }
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < kAppendMaxCols; ++i) {
    const int col = tid + i * kAppendThreads;
    if (col < W)
#pragma unroll
      for (int t = 0; t < kAppendTok; ++t) cs[t * W + col] = acc[i][t];
  }
  __syncthreads();

  // Epilogue: warp w normalises and scatters token t0 + w.
  const int warp = tid >> 5, lane = tid & 31;
  if (warp >= ntok) return;
  const int tok = t0 + warp;
  const float *c = cs + warp * W;
  float ss = 0.f;
  for (int j = lane; j < a.d_c; j += 32) ss += c[j] * c[j];
#pragma unroll
  for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float inv = rsqrtf(ss / (float)a.d_c + a.rms_eps);
  const int b = a.seq_idx[tok], p = a.pos[tok];
  if (b < 0 || b >= a.num_seqs || p < 0 || (int64_t)p >= (int64_t)a.max_blocks_per_seq * a.block_size) {
    if (lane == 0) report(a.dev_status, MLA_ERR_BAD_INDEX);
    return;
  }
  const int64_t row = cache_row(a.block_table, a.max_blocks_per_seq, a.num_blocks, a.block_size, b, p);
  if (row < 0) {
    if (lane == 0) report(a.dev_status, MLA_ERR_BAD_INDEX);
    return;
  }
  auto at = [&](int d) {
    return latent_elem<T>(a.c_kv, a.k_pe, a.ckv_stride, a.kpe_stride, a.layout, a.d_c, W, row, d);
  };
  const T *g = static_cast<const T *>(a.gamma);
  for (int j = lane; j < a.d_c; j += 32) {
    const float gj = g ? to_f32(g[j]) : 1.f;
    *at(j) = from_f32<T>(c[j] * inv * gj);
  }
  for (int i = lane; i < a.d_rope / 2; i += 32) {
    float cs_, sn_;
    rope_cos_sin(p, i, a.d_rope, a.rope_base, &cs_, &sn_);
    const float x = c[a.d_c + 2 * i], y = c[a.d_c + 2 * i + 1];
    *at(a.d_c + 2 * i) = from_f32<T>(x * cs_ - y * sn_);
    *at(a.d_c + 2 * i + 1) = from_f32<T>(x * sn_ + y * cs_);
  }
}

int launch_append(const AppendArgs &a, bool bf16, cudaStream_t st) {
  if (a.T == 0) return MLA_OK;
  if (a.d_c + a.d_rope > kAppendMaxCols * kAppendThreads) return MLA_ERR_UNSUPPORTED;
  const size_t smem = sizeof(float) * (kAppendTok * kAppendKChunk + kAppendTok * (a.d_c + a.d_rope));
  const dim3 grid((a.T + kAppendTok - 1) / kAppendTok);
  if (bf16) {
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(append_latent_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem))
      return MLA_ERR_CUDA;
    append_latent_kernel<__nv_bfloat16><<<grid, kAppendThreads, smem, st>>>(a);
  } else {
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(append_latent_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem))
      return MLA_ERR_CUDA;
    append_latent_kernel<float><<<grid, kAppendThreads, smem, st>>>(a);
  }
  return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

}  // namespace mla
