// The last step of appending one new token's cache row: sum the split-K partials of
// h [W_DKV | W_KR], RMSNorm the d_c latent dims ("DeepSeek-V3 解读 1: MLA", Figure 1 caption),
// RoPE the shared key at the token's position (section "为什么需要解耦 RoPE") and scatter both
// into the paged pool.  Shared by the append finish kernel and the fused decode-step kernel.
#pragma once

#include "kernels.cuh"

namespace mla {

// Shared scratch of append_finish_token, in floats: the latent pairs' squares and the total.
constexpr int kFinishScratch = 577;

// One CTA of kThreads threads finishes token `tok` of sequence b at position p; `red` is shared
// scratch of kFinishScratch floats.  The partials are read through L2 (ld.global.cg): in the fused
// kernel they were written by other CTAs of the same grid.  The sum of squares of the RMSNorm is
// added in one fixed order whatever kThreads is, so every caller writes the same bits.  Rows up to
// 2 * 2 * 288 wide.
template <int kThreads>
__device__ __forceinline__ void append_finish_token(const AppendArgs &a, const float *part, int nsplit, int tok,
                                                    int b, int p, float *red) {
  constexpr int kMaxPairsPerThr = (576 + kThreads - 1) / kThreads;
  const int W = a.d_c + a.d_rope, npair = W / 2;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t split_stride = (int64_t)a.T * W / 2;   // in float2
  const float2 *pp = reinterpret_cast<const float2 *>(part) + (int64_t)tok * npair;
  float2 v[kMaxPairsPerThr];
  const int npc = a.d_c / 2;                          // latent pairs
#pragma unroll
  for (int i = 0; i < kMaxPairsPerThr; ++i) {
    const int j2 = tid + i * kThreads;
    float2 acc = make_float2(0.f, 0.f);
    if (j2 < npair) {
      // Up to 32 partials' loads in flight at once, then added in split order (the same order for
      // every caller, so the bits do not depend on the batching).
      for (int s0 = 0; s0 < nsplit; s0 += 32) {
        float2 xs[32];
#pragma unroll
        for (int k = 0; k < 32; ++k)
          xs[k] = s0 + k < nsplit ? __ldcg(pp + (int64_t)(s0 + k) * split_stride + j2) : make_float2(0.f, 0.f);
#pragma unroll
        for (int k = 0; k < 32; ++k)
          if (s0 + k < nsplit) {
            acc.x += xs[k].x;
            acc.y += xs[k].y;
          }
      }
      if (j2 < npc) red[j2] = acc.x * acc.x + acc.y * acc.y;
    }
    v[i] = acc;
  }
  __syncthreads();
  if (warp == 0) {                                    // lane l: pairs l, l + 32, ... in order, then a fixed tree
    float ss = 0.f;
    for (int k = lane; k < npc; k += 32) ss += red[k];
#pragma unroll
    for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if (lane == 0) red[kFinishScratch - 1] = ss;
  }
  __syncthreads();
  const float tot = red[kFinishScratch - 1];
  const float inv = rsqrtf(tot / (float)a.d_c + a.rms_eps);
  if (b < 0 || b >= a.num_seqs || p < 0 || (int64_t)p >= (int64_t)a.max_blocks_per_seq * a.block_size) {
    if (tid == 0) report(a.dev_status, MLA_ERR_BAD_INDEX);
    return;
  }
  const int64_t row = cache_row(a.block_table, a.max_blocks_per_seq, a.num_blocks, a.block_size, b, p);
  if (row < 0) {
    if (tid == 0) report(a.dev_status, MLA_ERR_BAD_INDEX);
    return;
  }
  auto at = [&](int d) {
    return latent_elem<__nv_bfloat16>(a.c_kv, a.k_pe, a.ckv_stride, a.kpe_stride, a.layout, a.d_c, W, row, d);
  };
  const __nv_bfloat16 *gm = static_cast<const __nv_bfloat16 *>(a.gamma);
#pragma unroll
  for (int i = 0; i < kMaxPairsPerThr; ++i) {
    const int j2 = tid + i * kThreads, j = 2 * j2;
    if (j2 >= npair) continue;
    if (j < a.d_c) {
      const float g0 = gm ? __bfloat162float(gm[j]) : 1.f, g1 = gm ? __bfloat162float(gm[j + 1]) : 1.f;
      *at(j) = __float2bfloat16_rn(v[i].x * inv * g0);
      *at(j + 1) = __float2bfloat16_rn(v[i].y * inv * g1);
    } else {
      float cs_, sn_;
      rope_cos_sin(p, (j - a.d_c) / 2, a.d_rope, a.rope_base, &cs_, &sn_);
      *at(j) = __float2bfloat16_rn(v[i].x * cs_ - v[i].y * sn_);
      *at(j + 1) = __float2bfloat16_rn(v[i].x * sn_ + v[i].y * cs_);
    }
  }
}

}  // namespace mla
