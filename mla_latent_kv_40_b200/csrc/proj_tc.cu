// bf16 projections around the attention kernel on 5th-generation tensor cores.
//
//  * query absorption, q_lat^(s) = q_nope^(s) W_UK^(s)T per head, plus the RoPE
//    of q_pe ("Transformer升级之路：21、MLA好在哪里?（下）", section 双重投影,
//    decoding column);
//  * append down-projection [h W_DKV | h W_KR] over a K-split, reduced and
//    finished (RMSNorm, RoPE, scatter) by the append finish kernel
//    ("DeepSeek-V3 解读 1: MLA", sections "MLA：高层次的思路" and
//    "为什么需要解耦 RoPE").
//
// Both are weight-streaming GEMMs with few activation rows, so they run
// transposed: the weight supplies the 128-row M side of a tcgen05 MMA (read
// once, by TMA), the activation rows are the N side (N = 64 per CTA), and the
// fp32 accumulator sits in 64 tensor-memory columns.  One elected thread
// issues the TMA loads and the MMAs; all warps drain tensor memory.
#include "append_finish.cuh"
#include "kernels.cuh"
#include "sm100.cuh"
#include "tmap.cuh"

namespace mla {

using namespace sm100;

namespace {

constexpr int kTcThreads = 128;
constexpr int kTcN = 64;                      // activation rows (tokens / query rows) per CTA
constexpr uint32_t kAChunk = 128 * 128;       // [128 rows x 64 K] bf16, 128B-swizzled: 16 KB
constexpr uint32_t kBChunk = kTcN * 128;      // [64 rows x 64 K] bf16: 8 KB
constexpr uint64_t kWaitNs = 2000000000ull;
// The absorption's output staging tile reuses its operand tiles (one K-chunk at least).
static_assert(sizeof(__nv_bfloat16) * kTcN * (128 + 8) <= kAChunk + kBChunk, "staging fits the operand tiles");

// Bounded wait: on expiry report a timeout and let the caller skip its work.
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, int *dev_status) {
  if (mbar_wait(bar, parity, kWaitNs)) return true;
  report(dev_status, MLA_ERR_TIMEOUT);
  return false;
}

// ------------------------------------------------------------------ absorb
// CTA = (head s, 128 latent columns m0.., 64 query rows r0..):
//   D[m][r] = sum_k W_UK[s][m0 + m][k] q_nope[r0 + r][s][k]   (A and B both K-major)
// The CTAs with blockIdx.y == 0 .. 3 share the RoPE of their 64 rows.
// (s, by, bz) play the roles of (blockIdx.x, blockIdx.y, blockIdx.z) of a grid (H, d_c / 128, rows / 64)
// whose y extent is ny; sm is the CTA's 1024-byte aligned dynamic shared memory.
__device__ __forceinline__ void absorb_tc_body(const CUtensorMap &map_w, const CUtensorMap &map_q, const AbsorbArgs &a,
                                               int *dev_status, int s, int by, int bz, int ny, unsigned char *sm) {
  __shared__ __align__(8) uint64_t bar_full, bar_mma;
  __shared__ uint32_t tmem_slot;
  const int nkc = a.d_nope / 64;
  unsigned char *As = sm;                                  // [nkc][128 x 128 B]
  unsigned char *Bs = As + nkc * kAChunk;                  // [nkc][64 x 128 B]
  // [64][128 + 8] output staging over the operand tiles, which are dead once the MMAs completed:
  // 48 KB per CTA instead of 65 KB, so four CTAs fit on an SM and the grid runs in one wave.
  __nv_bfloat16 *Os = reinterpret_cast<__nv_bfloat16 *>(sm);
  constexpr int ldo = 128 + 8;
  const int m0 = by * 128, r0 = bz * kTcN;
  const int R = a.B * a.n_q, W = a.d_c + a.d_rope;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  grid_dep_launch();   // reads below touch inputs only; q_out is written after grid_dep_wait()

  if (tid == 0) {
    mbar_init(smem_u32(&bar_full), 1);
    mbar_init(smem_u32(&bar_mma), 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(&tmem_slot), kTcN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;

  if (tid == 0) {
    tma_prefetch_desc(&map_w);
    tma_prefetch_desc(&map_q);
    mbar_expect_tx(smem_u32(&bar_full), nkc * (kAChunk + kBChunk));
    for (int kc = 0; kc < nkc; ++kc) {
      tma_load_2d(smem_u32(As + kc * kAChunk), &map_w, 64 * kc, s * a.d_c + m0, smem_u32(&bar_full));
      tma_load_2d(smem_u32(Bs + kc * kBChunk), &map_q, s * a.d_nope + 64 * kc, r0, smem_u32(&bar_full));
    }
  }

  // RoPE of q_pe by warps 1-3 while the tiles stream in (thread 0 goes straight on to the MMAs):
  // rows r0 + y, y + gridDim.y, ... of this CTA; a warp takes whole rows, a lane one (x, y) pair,
  // and every row's loads are issued before any of its arithmetic.
  if (warp > 0) {
    __shared__ double theta[32];                           // pair frequencies, once per CTA
    const __nv_bfloat16 *qp = static_cast<const __nv_bfloat16 *>(a.q_pe);
    __nv_bfloat16 *qo = static_cast<__nv_bfloat16 *>(a.q_out);
    const int half = a.d_rope / 2;
    if (tid - 32 < half) theta[tid - 32] = rope_theta(tid - 32, a.d_rope, a.rope_base);
    asm volatile("bar.sync 1, 96;" ::: "memory");       // warps 1-3 only
    grid_dep_wait();                                       // q_out may still be read by an earlier kernel
    constexpr int kRowsPerWarp = 8;
    const int nr = (kTcN - by + ny - 1) / ny;
    for (int w0 = (warp - 1) * kRowsPerWarp; w0 < nr; w0 += 3 * kRowsPerWarp) {
      int pos[kRowsPerWarp];
      __nv_bfloat162 xy[kRowsPerWarp];
#pragma unroll
      for (int k = 0; k < kRowsPerWarp; ++k) {
        const int gr = r0 + by + ny * (w0 + k);
        const bool live = w0 + k < nr && gr < R && lane < half;
        pos[k] = live ? max(0, a.seqlens[gr / a.n_q] - a.n_q + gr % a.n_q) : -1;   // -1: nothing to do
        xy[k] = live ? *reinterpret_cast<const __nv_bfloat162 *>(qp + ((int64_t)gr * a.H + s) * a.d_rope + 2 * lane)
                     : __floats2bfloat162_rn(0.f, 0.f);
      }
#pragma unroll
      for (int k = 0; k < kRowsPerWarp; ++k) {
        if (pos[k] < 0) continue;
        const int gr = r0 + by + ny * (w0 + k);
        float cs, sn;
        rope_cos_sin_theta(pos[k], theta[lane], &cs, &sn);
        const float x = __low2float(xy[k]), y = __high2float(xy[k]);
        *reinterpret_cast<__nv_bfloat162 *>(qo + ((int64_t)gr * a.H + s) * W + a.d_c + 2 * lane) =
            __floats2bfloat162_rn(x * cs - y * sn, x * sn + y * cs);
      }
    }
  }

  int ok = 1;
  if (tid == 0) {
    ok = wait_bar(smem_u32(&bar_full), 0, dev_status) ? 1 : 0;
    if (ok) {
      tc_fence_after();
      const uint32_t idesc = idesc_bf16_f32(128, kTcN, false, false);
      for (int kc = 0; kc < nkc; ++kc)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_ss(tmem, smem_desc_sw128(smem_u32(As + kc * kAChunk) + kk * 32, 16, 1024),
                 smem_desc_sw128(smem_u32(Bs + kc * kBChunk) + kk * 32, 16, 1024), idesc, (kc | kk) ? 1u : 0u);
      tc_commit(smem_u32(&bar_mma));
    }
  }
  ok = __syncthreads_and(ok);
  if (ok && lane == 0) ok = wait_bar(smem_u32(&bar_mma), 0, dev_status) ? 1 : 0;
  ok = __shfl_sync(0xffffffffu, ok, 0);
  if (ok) mbar_wait(smem_u32(&bar_mma), 0, kWaitNs);
  tc_fence_after();
  // Warp w drains latent rows 32w..32w+31 (its lane quadrant): thread = one latent column m,
  // 64 query rows -> the staging tile, transposed to [query row][m].
  {
    uint32_t v[32];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + 32 * h, v);
      tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < 32; ++i) Os[(32 * h + i) * ldo + warp * 32 + lane] = __float2bfloat16_rn(__uint_as_float(v[i]));
    }
  }
  tc_fence_before();
  __syncthreads();
  grid_dep_wait();
  if (ok) {
    __nv_bfloat16 *qo = static_cast<__nv_bfloat16 *>(a.q_out);
    for (int c = tid; c < kTcN * 16; c += kTcThreads) {
      const int r = c >> 4, q8 = c & 15, gr = r0 + r;
      if (gr < R)
        *reinterpret_cast<uint4 *>(qo + ((int64_t)gr * a.H + s) * W + m0 + q8 * 8) =
            *reinterpret_cast<const uint4 *>(Os + r * ldo + q8 * 8);
    }
  }
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTcN);
  }
}

__device__ __forceinline__ unsigned char *align1024(unsigned char *p) {
  return reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

__global__ void __launch_bounds__(kTcThreads)
absorb_tc_kernel(const __grid_constant__ CUtensorMap map_w, const __grid_constant__ CUtensorMap map_q, AbsorbArgs a,
                 int *dev_status) {
  extern __shared__ unsigned char smem_raw[];
  absorb_tc_body(map_w, map_q, a, dev_status, blockIdx.x, blockIdx.y, blockIdx.z, gridDim.y, align1024(smem_raw));
}

// ------------------------------------------------------------------ append projection
// CTA = (128 output columns m0.. of [W_DKV | W_KR], K-split ks, 64 tokens t0..):
//   D[m][t] = sum_{k in split} W[k][m0 + m] h[t0 + t][k]     (A = W^T is M-major, B = h is K-major)
// Stages of 64 K rows stream through a ring; the partial goes to part[ks][t][m] (fp32).
constexpr int kApStages = 4;
constexpr uint32_t kApStageBytes = kAChunk + kBChunk;      // A: 2 M-chunks of [64 K x 128 B]; B: [64 x 128 B]

// (bx, ks, bz) play the roles of (blockIdx.x, blockIdx.y, blockIdx.z) of a grid (columns / 128, splits, T / 64).
__device__ __forceinline__ void append_tc_body(const CUtensorMap &map_wd, const CUtensorMap &map_wr,
                                               const CUtensorMap &map_h, int T, int d_c, int d_rope, int k_per_split,
                                               int D, float *part, int *dev_status, int bx, int ks, int bz,
                                               unsigned char *sm) {
  __shared__ __align__(8) uint64_t bar_full[kApStages], bar_empty[kApStages], bar_mma;
  __shared__ uint32_t tmem_slot;
  const int W = d_c + d_rope;
  const int m0 = bx * 128, t0 = bz * kTcN;
  const int kbeg = ks * k_per_split, kend = min(D, kbeg + k_per_split);
  const int nst = (kend - kbeg + 63) / 64;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool rope_tile = m0 >= d_c;
  grid_dep_launch();   // h and the weights are inputs; the partials are written after grid_dep_wait()

  if (tid == 0) {
    for (int i = 0; i < kApStages; ++i) {
      mbar_init(smem_u32(&bar_full[i]), 1);
      mbar_init(smem_u32(&bar_empty[i]), 1);
    }
    mbar_init(smem_u32(&bar_mma), 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(&tmem_slot), kTcN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;

  int ok = 1;
  if (tid == 0) {
    // Producer: stage i = K rows kbeg + 64i ..; the weight chunk c holds output columns m0 + 64c ..
    // (the RoPE tile reads W_KR, whose second chunk lies outside it and arrives as zeros).
    const CUtensorMap *mw = rope_tile ? &map_wr : &map_wd;
    const int mx = rope_tile ? m0 - d_c : m0;
    tma_prefetch_desc(mw);
    tma_prefetch_desc(&map_h);
    for (int i = 0; i < nst; ++i) {
      const int st = i % kApStages;
      if (i >= kApStages && !wait_bar(smem_u32(&bar_empty[st]), ((i / kApStages) - 1) & 1, dev_status)) { ok = 0; break; }
      unsigned char *base = sm + st * kApStageBytes;
      const int k0 = kbeg + 64 * i;
      mbar_expect_tx(smem_u32(&bar_full[st]), kApStageBytes);
      tma_load_2d(smem_u32(base), mw, mx, k0, smem_u32(&bar_full[st]));
      tma_load_2d(smem_u32(base + kAChunk / 2), mw, mx + 64, k0, smem_u32(&bar_full[st]));
      tma_load_2d(smem_u32(base + kAChunk), &map_h, k0, t0, smem_u32(&bar_full[st]));
    }
  } else if (tid == 32) {
    // MMA issuer.
    const uint32_t idesc = idesc_bf16_f32(128, kTcN, true, false);
    for (int i = 0; i < nst; ++i) {
      const int st = i % kApStages;
      if (!wait_bar(smem_u32(&bar_full[st]), (i / kApStages) & 1, dev_status)) { ok = 0; break; }
      tc_fence_after();
      const uint32_t a = smem_u32(sm + st * kApStageBytes), b = a + kAChunk;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_ss(tmem, smem_desc_sw128(a + kk * 2048, kAChunk / 2, 1024), smem_desc_sw128(b + kk * 32, 16, 1024), idesc,
               (i | kk) ? 1u : 0u);
      tc_commit(smem_u32(&bar_empty[st]));
    }
    tc_commit(smem_u32(&bar_mma));
  }
  ok = __syncthreads_and(ok);
  if (ok && lane == 0) ok = wait_bar(smem_u32(&bar_mma), 0, dev_status) ? 1 : 0;
  ok = __shfl_sync(0xffffffffu, ok, 0);
  if (ok) mbar_wait(smem_u32(&bar_mma), 0, kWaitNs);
  tc_fence_after();
  grid_dep_wait();
  // Thread = output column m0 + 32w + lane; for each token its value goes to part[ks][t][m]:
  // consecutive lanes write consecutive columns.
  {
    const int m = m0 + warp * 32 + lane;
    float *dst = part + ((int64_t)ks * T) * W + m;
    uint32_t v[32];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + 32 * h, v);
      tmem_wait_ld();
      if (ok && m < W)
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int t = t0 + 32 * h + i;
          if (t < T) dst[(int64_t)t * W] = __uint_as_float(v[i]);
        }
    }
  }
  // Every issued load has landed (the MMA consumed it) before the CTA may leave.
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTcN);
  }
}

__global__ void __launch_bounds__(kTcThreads)
append_tc_kernel(const __grid_constant__ CUtensorMap map_wd, const __grid_constant__ CUtensorMap map_wr,
                 const __grid_constant__ CUtensorMap map_h, int T, int d_c, int d_rope, int k_per_split, int D,
                 float *part, int *dev_status) {
  extern __shared__ unsigned char smem_raw[];
  append_tc_body(map_wd, map_wr, map_h, T, d_c, d_rope, k_per_split, D, part, dev_status, blockIdx.x, blockIdx.y,
                 blockIdx.z, align1024(smem_raw));
}

// ------------------------------------------------------------------ fused decode-step preparation
// One launch does the work that precedes the attention of a decode step: the append of the step's
// new tokens (projection, then RMSNorm / RoPE / scatter) and the query absorption.  Its CTAs take
// three roles by block index:
//   [0, nA)            append projection CTAs (split-K partials); each signals the counter when done;
//   [nA, nA + nB)      absorption CTAs (independent of the append);
//   [nA + nB, + T)     append finish CTAs, one per new token: they wait (bounded) until all nA
//                      projection CTAs have signalled, then finish their token.
// The finish CTAs come last, so every CTA they wait for is dispatched before them.
struct PrepParams {
  AppendArgs ap;
  AbsorbArgs ab;
  float *part;
  int nsplit, k_per_split;
  int nA, a_nx, a_ny;                 // append grid (columns / 128, splits, tokens / 64)
  int nB, b_ny, b_nz;                 // absorb grid (H, d_c / 128, rows / 64)
  unsigned *counter;                  // zeroed before the launch
};

__global__ void __launch_bounds__(kTcThreads)
decode_prep_kernel(const __grid_constant__ CUtensorMap map_wd, const __grid_constant__ CUtensorMap map_wr,
                   const __grid_constant__ CUtensorMap map_h, const __grid_constant__ CUtensorMap map_w,
                   const __grid_constant__ CUtensorMap map_q, const PrepParams pp) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char *sm = align1024(smem_raw);
  int id = blockIdx.x;
  if (id < pp.nA) {
    const int bx = id % pp.a_nx, ks = (id / pp.a_nx) % pp.a_ny, bz = id / (pp.a_nx * pp.a_ny);
    append_tc_body(map_wd, map_wr, map_h, pp.ap.T, pp.ap.d_c, pp.ap.d_rope, pp.k_per_split, pp.ap.d_model, pp.part,
                   pp.ap.dev_status, bx, ks, bz, sm);
    __threadfence();                  // this CTA's partials, then its signal (release at GPU scope)
    __syncthreads();
    if (threadIdx.x == 0) asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(pp.counter) : "memory");
    return;
  }
  id -= pp.nA;
  if (id < pp.nB) {
    const int s = id % pp.ab.H, by = (id / pp.ab.H) % pp.b_ny, bz = id / (pp.ab.H * pp.b_ny);
    absorb_tc_body(map_w, map_q, pp.ab, pp.ap.dev_status, s, by, bz, pp.b_ny, sm);
    return;
  }
  const int tok = id - pp.nB;
  __shared__ float red[kFinishScratch];
  __shared__ int ready;
  grid_dep_launch();
  grid_dep_wait();                    // earlier kernels may still read the cache rows written below
  if (threadIdx.x == 0) {
    int ok = 1;
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
      unsigned v;
      asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(pp.counter) : "memory");
      if ((int)v >= pp.nA) break;
      if (globaltimer_ns() - t0 > kWaitNs) {
        report(pp.ap.dev_status, MLA_ERR_TIMEOUT);
        ok = 0;
        break;
      }
      __nanosleep(200);
    }
    ready = ok;
  }
  __syncthreads();
  if (!ready) return;
  const int n_q = pp.ab.n_q;
  const int b = tok / n_q;
  const int p = pp.ab.seqlens[b] - n_q + tok % n_q;
  append_finish_token<kTcThreads>(pp.ap, pp.part, pp.nsplit, tok, b, p, red);
}

}  // namespace

// ------------------------------------------------------------------ host side
bool absorb_tc_supported(const AbsorbArgs &a, bool bf16) {
  return bf16 && a.d_nope % 64 == 0 && a.d_nope <= 256 && a.d_c % 128 == 0 && a.d_rope <= 64 && a.d_rope % 2 == 0 &&
         !(reinterpret_cast<uintptr_t>(a.q_nope) & 15) && !(reinterpret_cast<uintptr_t>(a.w_uk) & 15) &&
         !(reinterpret_cast<uintptr_t>(a.q_pe) & 3) && !(reinterpret_cast<uintptr_t>(a.q_out) & 15) &&
         ((a.d_c + a.d_rope) % 8) == 0;
}

int launch_absorb_tc(const AbsorbArgs &a, int *dev_status, cudaStream_t st) {
  const int R = a.B * a.n_q;
  CUtensorMap mw, mq;
  if (!make_tmap_bf16(&mw, a.w_uk, a.d_nope, (uint64_t)a.H * a.d_c, (uint64_t)a.d_nope * 2, 128) ||
      !make_tmap_bf16(&mq, a.q_nope, (uint64_t)a.H * a.d_nope, R, (uint64_t)a.H * a.d_nope * 2, kTcN))
    return MLA_ERR_CUDA;
  const int nkc = a.d_nope / 64;
  const size_t smem = 1024 + nkc * (kAChunk + kBChunk);
  static std::atomic<int> smem_set[kSmemCacheDevs];
  if (smem_limit(absorb_tc_kernel, smem, smem_set) != cudaSuccess)
    return MLA_ERR_CUDA;
  const dim3 grid(a.H, a.d_c / 128, (R + kTcN - 1) / kTcN);
  return launch_pdl(absorb_tc_kernel, grid, dim3(kTcThreads), smem, st, mw, mq, a, dev_status) == cudaSuccess
             ? MLA_OK
             : MLA_ERR_CUDA;
}

bool append_tc_supported(const AppendArgs &a, bool bf16) {
  return bf16 && a.d_model % 64 == 0 && a.d_c % 128 == 0 && a.d_rope <= 128 && a.d_rope % 8 == 0 &&
         !(reinterpret_cast<uintptr_t>(a.h) & 15) && !(reinterpret_cast<uintptr_t>(a.w_dkv) & 15) &&
         !(reinterpret_cast<uintptr_t>(a.w_kr) & 15);
}

int launch_append_tc(const AppendArgs &a, void *ws, int nsplit, int k_per_split, cudaStream_t st) {
  const int W = a.d_c + a.d_rope;
  CUtensorMap mwd, mwr, mh;
  if (!make_tmap_bf16(&mwd, a.w_dkv, a.d_c, a.d_model, (uint64_t)a.d_c * 2, 64) ||
      !make_tmap_bf16(&mwr, a.w_kr, a.d_rope, a.d_model, (uint64_t)a.d_rope * 2, 64) ||
      !make_tmap_bf16(&mh, a.h, a.d_model, a.T, (uint64_t)a.d_model * 2, kTcN))
    return MLA_ERR_CUDA;
  const size_t smem = 1024 + kApStages * kApStageBytes;
  static std::atomic<int> smem_set[kSmemCacheDevs];
  if (smem_limit(append_tc_kernel, smem, smem_set) != cudaSuccess)
    return MLA_ERR_CUDA;
  const dim3 grid((W + 127) / 128, nsplit, (a.T + kTcN - 1) / kTcN);
  return launch_pdl(append_tc_kernel, grid, dim3(kTcThreads), smem, st, mwd, mwr, mh, a.T, a.d_c, a.d_rope,
                    k_per_split, a.d_model, static_cast<float *>(ws), a.dev_status) == cudaSuccess
             ? MLA_OK
             : MLA_ERR_CUDA;
}

bool decode_prep_supported(const AppendArgs &ap, const AbsorbArgs &ab) {
  return append_tc_supported(ap, true) && append_mma_supported(ap, true) && absorb_tc_supported(ab, true);
}

int launch_decode_prep(const AppendArgs &ap, const AbsorbArgs &ab, void *part, int nsplit, int k_per_split,
                       unsigned *counter, cudaStream_t st) {
  const int W = ap.d_c + ap.d_rope, R = ab.B * ab.n_q;
  CUtensorMap mwd, mwr, mh, mw, mq;
  if (!make_tmap_bf16(&mwd, ap.w_dkv, ap.d_c, ap.d_model, (uint64_t)ap.d_c * 2, 64) ||
      !make_tmap_bf16(&mwr, ap.w_kr, ap.d_rope, ap.d_model, (uint64_t)ap.d_rope * 2, 64) ||
      !make_tmap_bf16(&mh, ap.h, ap.d_model, ap.T, (uint64_t)ap.d_model * 2, kTcN) ||
      !make_tmap_bf16(&mw, ab.w_uk, ab.d_nope, (uint64_t)ab.H * ab.d_c, (uint64_t)ab.d_nope * 2, 128) ||
      !make_tmap_bf16(&mq, ab.q_nope, (uint64_t)ab.H * ab.d_nope, R, (uint64_t)ab.H * ab.d_nope * 2, kTcN))
    return MLA_ERR_CUDA;
  PrepParams pp;
  pp.ap = ap;
  pp.ab = ab;
  pp.part = static_cast<float *>(part);
  pp.nsplit = nsplit;
  pp.k_per_split = k_per_split;
  pp.a_nx = (W + 127) / 128;
  pp.a_ny = nsplit;
  pp.nA = pp.a_nx * nsplit * ((ap.T + kTcN - 1) / kTcN);
  pp.b_ny = ab.d_c / 128;
  pp.b_nz = (R + kTcN - 1) / kTcN;
  pp.nB = ab.H * pp.b_ny * pp.b_nz;
  pp.counter = counter;
  const int nkc = ab.d_nope / 64;
  const size_t smem_ab = 1024 + nkc * (kAChunk + kBChunk);
  const size_t smem_ap = 1024 + kApStages * kApStageBytes;
  const size_t smem = smem_ab > smem_ap ? smem_ab : smem_ap;
  static std::atomic<int> smem_set[kSmemCacheDevs];
  if (smem_limit(decode_prep_kernel, smem, smem_set) != cudaSuccess)
    return MLA_ERR_CUDA;
  if (cudaMemsetAsync(counter, 0, sizeof(unsigned), st) != cudaSuccess) return MLA_ERR_CUDA;
  return launch_pdl(decode_prep_kernel, dim3(pp.nA + pp.nB + ap.T), dim3(kTcThreads), smem, st, mwd, mwr, mh, mw, mq,
                    pp) == cudaSuccess
             ? MLA_OK
             : MLA_ERR_CUDA;
}

}  // namespace mla
