// Weight-streaming batched product on 5th-generation tensor cores for the decode from hidden
// states with folded weights ("DeepSeek-V3 解读 1: MLA", sections "MLA：高层次的思路" and
// "为什么需要解耦 RoPE"; "Transformer升级之路：21、MLA好在哪里?（下）", section 键值共享):
//   c_Q = h W_DQ,  q_lat^(s) = c_Q W_UQK^(s),  q_pe = c_Q W_QR,  u = o_lat W_UVO,
// i.e. C[b][t][n] = sum_k A[t][k] B[b][k][n] with few rows t (the step's tokens) and a wide
// weight B.  Like the append projection, the weight supplies the 128-row M side of each MMA
// (M-major, read once by TMA), the activation rows are the N side (64 per CTA, K-major), and K is
// split so that about two CTAs per SM get work; the split partials (fp32) are added in order by
// the reduce kernel of the CUDA-core product.  Shapes outside its layout rules return
// MLA_ERR_UNSUPPORTED and run on the CUDA-core product instead.
#include "kernels.cuh"
#include "sm100.cuh"
#include "tmap.cuh"

namespace mla {
namespace {

using namespace sm100;

constexpr int kGThreads = 128;
constexpr int kGN = 64;                                  // activation rows per CTA (MMA N)
constexpr int kGStages = 4;
constexpr uint32_t kGAChunk = 128 * 128;                 // weight tile: 2 M-chunks of [64 K rows x 128 B]
constexpr uint32_t kGBChunk = kGN * 128;                 // activation tile: [64 rows x 64 K] bf16
constexpr uint32_t kGStageBytes = kGAChunk + kGBChunk;   // 24 KB
constexpr uint64_t kGWaitNs = 2000000000ull;

struct GemmTcParams {
  int M, N, K, batch, ksplit, kc;   // kc: K per split, a multiple of 64
  int64_t K_rows_per_batch;         // weight rows of one batch in the weight map (= K)
  float *part;                      // [batch][ksplit][M][N] when ksplit > 1
  __nv_bfloat16 *C;
  int64_t sc_b, sc_m;
  int *dev_status;
};

__device__ __forceinline__ bool gwait(uint32_t bar, uint32_t parity, int *dev_status) {
  if (mbar_wait(bar, parity, kGWaitNs)) return true;
  report(dev_status, MLA_ERR_TIMEOUT);
  return false;
}

// CTA = (128 output columns n0.., K-split ks, batch b x 64 activation rows t0..).
__global__ void __launch_bounds__(kGThreads)
gemm_tc_kernel(const __grid_constant__ CUtensorMap map_b, const __grid_constant__ CUtensorMap map_a,
               const GemmTcParams g) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char *sm = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t bar_full[kGStages], bar_empty[kGStages], bar_mma;
  __shared__ uint32_t tmem_slot;
  const int n0 = blockIdx.x * 128, ks = blockIdx.y;
  const int mtiles = (g.M + kGN - 1) / kGN;
  const int b = blockIdx.z / mtiles, t0 = (blockIdx.z % mtiles) * kGN;
  const int kbeg = ks * g.kc, kend = min(g.K, kbeg + g.kc);
  const int nst = kend > kbeg ? (kend - kbeg) / 64 : 0;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  grid_dep_launch();   // weights are inputs; the activations and outputs follow grid_dep_wait()

  if (tid == 0) {
    for (int i = 0; i < kGStages; ++i) {
      mbar_init(smem_u32(&bar_full[i]), 1);
      mbar_init(smem_u32(&bar_empty[i]), 1);
    }
    mbar_init(smem_u32(&bar_mma), 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(&tmem_slot), kGN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  grid_dep_wait();   // the activation rows may come from the previous kernel

  int ok = 1;
  if (tid == 0) {
    // Producer: stage i = K rows kbeg + 64 i ..; weight chunk c holds output columns n0 + 64 c ..
    tma_prefetch_desc(&map_b);
    tma_prefetch_desc(&map_a);
    const int64_t wrow0 = (int64_t)b * g.K_rows_per_batch;
    for (int i = 0; i < nst; ++i) {
      const int st = i % kGStages;
      if (i >= kGStages && !gwait(smem_u32(&bar_empty[st]), ((i / kGStages) - 1) & 1, g.dev_status)) { ok = 0; break; }
      unsigned char *base = sm + st * kGStageBytes;
      const int k0 = kbeg + 64 * i;
      mbar_expect_tx(smem_u32(&bar_full[st]), kGStageBytes);
      tma_load_2d(smem_u32(base), &map_b, n0, (int32_t)(wrow0 + k0), smem_u32(&bar_full[st]));
      tma_load_2d(smem_u32(base + kGAChunk / 2), &map_b, n0 + 64, (int32_t)(wrow0 + k0), smem_u32(&bar_full[st]));
      tma_load_2d(smem_u32(base + kGAChunk), &map_a, k0, t0, smem_u32(&bar_full[st]));
    }
  } else if (tid == 32) {
    // MMA issuer: D [128 output columns x 64 rows] += B^T . A^T, four K = 16 steps per stage.
    const uint32_t idesc = idesc_bf16_f32(128, kGN, true, false);
    for (int i = 0; i < nst; ++i) {
      const int st = i % kGStages;
      if (!gwait(smem_u32(&bar_full[st]), (i / kGStages) & 1, g.dev_status)) { ok = 0; break; }
      tc_fence_after();
      const uint32_t a = smem_u32(sm + st * kGStageBytes), bb = a + kGAChunk;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_ss(tmem, smem_desc_sw128(a + kk * 2048, kGAChunk / 2, 1024), smem_desc_sw128(bb + kk * 32, 16, 1024), idesc,
               (i | kk) ? 1u : 0u);
      tc_commit(smem_u32(&bar_empty[st]));
    }
    tc_commit(smem_u32(&bar_mma));   // with no stage: completes at once
  }
  ok = __syncthreads_and(ok);
  if (ok && lane == 0) ok = gwait(smem_u32(&bar_mma), 0, g.dev_status) ? 1 : 0;
  ok = __shfl_sync(0xffffffffu, ok, 0);
  if (ok) mbar_wait(smem_u32(&bar_mma), 0, kGWaitNs);
  tc_fence_after();
  // Thread = output column n0 + 32 w + lane; for each activation row its value goes to the split's
  // partial (fp32) or, without a split, to C (bf16).  A split with no K range writes zeros.
  {
    const int n = n0 + warp * 32 + lane;
    uint32_t v[32];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      if (nst > 0) {
        tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + 32 * h, v);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = 0u;
      }
      if (ok && n < g.N)
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int t = t0 + 32 * h + i;
          if (t >= g.M) continue;
          if (g.ksplit > 1)
            g.part[(((int64_t)b * g.ksplit + ks) * g.M + t) * g.N + n] = __uint_as_float(v[i]);
          else
            g.C[(int64_t)b * g.sc_b + (int64_t)t * g.sc_m + n] = __float2bfloat16_rn(__uint_as_float(v[i]));
        }
    }
  }
  // Every issued load was consumed by an MMA that completed (the commit above) before the CTA leaves.
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kGN);
  }
}

}  // namespace

// Runs the product on the tensor cores when its layout allows, else returns MLA_ERR_UNSUPPORTED
// (and launches nothing): bf16; A [M rows x K] with unit K stride and shared by all batches (or a
// single batch); B [K x N] with unit N stride, batches K rows apart; C with unit N stride; N a
// multiple of 128, K of 64; row strides multiples of 8 elements and 16-byte aligned bases.
int launch_gemm_tc(const GemmArgs &g, bool bf16, cudaStream_t st) {
  if (!bf16 || g.M <= 0 || g.N <= 0 || g.K <= 0 || g.batch <= 0 || g.ksplit <= 0) return MLA_ERR_UNSUPPORTED;
  if (g.sa_k != 1 || g.sb_n != 1 || g.sc_n != 1) return MLA_ERR_UNSUPPORTED;
  if (g.N % 128 || g.K % 64 || g.sa_m % 8 || g.sb_k % 8) return MLA_ERR_UNSUPPORTED;
  if (g.batch > 1 && (g.sa_b != 0 || g.sb_b != (int64_t)g.K * g.sb_k)) return MLA_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(g.A) & 15) || (reinterpret_cast<uintptr_t>(g.B) & 15)) return MLA_ERR_UNSUPPORTED;
  if (g.ksplit > 1 && !g.part) return MLA_ERR_WORKSPACE;
  CUtensorMap mb, ma;
  if (!make_tmap_bf16(&mb, g.B, (uint64_t)g.N, (uint64_t)g.batch * g.K, (uint64_t)g.sb_k * 2, 64) ||
      !make_tmap_bf16(&ma, g.A, (uint64_t)g.K, (uint64_t)g.M, (uint64_t)g.sa_m * 2, kGN))
    return MLA_ERR_UNSUPPORTED;
  GemmTcParams p;
  p.M = g.M;
  p.N = g.N;
  p.K = g.K;
  p.batch = g.batch;
  p.ksplit = g.ksplit;
  p.kc = ((g.K + g.ksplit - 1) / g.ksplit + 63) / 64 * 64;
  p.K_rows_per_batch = g.K;
  p.part = g.part;
  p.C = static_cast<__nv_bfloat16 *>(g.C);
  p.sc_b = g.sc_b;
  p.sc_m = g.sc_m;
  p.dev_status = nullptr;
  const size_t smem = 1024 + (size_t)kGStages * kGStageBytes;
  static std::atomic<int> smem_set[kSmemCacheDevs];
  if (smem_limit(gemm_tc_kernel, smem, smem_set) != cudaSuccess)
    return MLA_ERR_CUDA;
  const dim3 grid(g.N / 128, g.ksplit, g.batch * ((g.M + kGN - 1) / kGN));
  if (launch_pdl(gemm_tc_kernel, grid, dim3(kGThreads), smem, st, mb, ma, p) != cudaSuccess) return MLA_ERR_CUDA;
  return g.ksplit > 1 ? launch_gemm_reduce(g, true, st) : MLA_OK;
}

}  // namespace mla
