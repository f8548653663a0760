// Causal prefill attention on 5th-generation tensor cores (tcgen05, sm_100a).
//
// "Transformer升级之路：21、MLA好在哪里?（下）", section 双重投影, training /
// prefill column: per head s the keys are decompressed, k_i = [c_i W_UK^(s) |
// kpe_i] (192 wide), the values v_i = c_i W_UV^(s) (128 wide), and
// o_t = softmax_{i<=t}(q_t k_i^T / sqrt(192)) V.  The query, key and value rows
// come from the prefill workspace (built by the first two prefill steps); this
// kernel is the third step, the attention itself.
//
// CTA = (sequence b, head s, 128 query rows q0..).  Q [128 x 192] stays in
// shared memory; keys and values stream in stages of 64 tokens (K [64 x 192],
// V [64 x 128]) by TMA.  One thread issues the MMAs:
//   S = Q . K^T      M = 128, N = 64, K = 192   into one of two 64-column
//                    tensor-memory buffers, so the next tile's S overlaps this
//                    tile's softmax;
//   O += P . V       M = 128, N = 128, K = 64   into 128 tensor-memory columns.
// Eight softmax warps (lane quadrant x half of the 64 columns) read S, keep a
// lazy reference maximum per row (log2 units; O is rescaled in tensor memory
// only when a row's maximum moves up by more than 8), write P (bf16) into one
// of two shared tiles and finally normalise O and write out and lse.  Query
// tiles are launched longest-first (causal work grows with the tile index).
// Every wait is bounded; on expiry the kernel reports MLA_ERR_TIMEOUT and
// finishes without waiting further.
#include <math_constants.h>

#include "kernels.cuh"
#include "sm100.cuh"
#include "tmap.cuh"

namespace mla {
namespace {

using namespace sm100;

constexpr int kPq = 128;                       // query rows per CTA (M of every MMA)
constexpr int kPk = 64;                        // keys per stage
constexpr int kDqk = 192, kDvp = 128;          // key / value widths this kernel takes
constexpr int kPStages = 3;
constexpr int kPThreads = 384;
constexpr uint32_t kQBytes = kPq * kDqk * 2;                 // 3 chunks of [128 x 128 B]
constexpr uint32_t kKChunk = kPk * 128;                      // [64 x 64] bf16
constexpr uint32_t kStageBytes = 3 * kKChunk + 2 * kKChunk;  // K (3 chunks) + V (2 chunks): 40 KB
constexpr uint32_t kPTile = kPq * kPk * 2;                   // P [128 x 64] bf16: 16 KB
constexpr uint32_t kOffStages = kQBytes;
constexpr uint32_t kOffP = kOffStages + kPStages * kStageBytes;
constexpr uint32_t kTiles = kOffP + 2 * kPTile;
constexpr uint32_t kSCols = 0, kOCols = 128;                 // TMEM: S buffers at 0 and 64, O at 128
constexpr float kRescale = 8.f;
constexpr uint64_t kWait = 2000000000ull;

enum PBar { P_QFULL = 0, P_KVFULL = 1, P_KVEMPTY = P_KVFULL + kPStages, P_SFULL = P_KVEMPTY + kPStages,
            P_SEMPTY = P_SFULL + 2, P_PFULL = P_SEMPTY + 2, P_PVDONE = P_PFULL + 2, P_COUNT = P_PVDONE + 2 };
// P_PVDONE + b completes when the product O += P V that read P buffer b has completed.

struct PfSmem {
  uint64_t bars[P_COUNT];
  float xmax[2][2][kPq];        // the two column halves' tile maxima (double-buffered)
  float xl[2][kPq];             // the two halves' row sums at the end
  uint32_t tmem_base;
  int abort;
};
constexpr size_t kPfSmem = 1024 + kTiles + sizeof(PfSmem);
static_assert(kPfSmem <= 232448, "prefill shared memory budget");

struct PfParams {
  int B, H, max_seqlen, total;
  int tiled, nqt, nkt;          // tiled workspace: Q and K|V tiles per (head, sequence), one bulk copy each
  const unsigned char *q_tiles, *kv_tiles;
  const int32_t *cu_seqlens;
  float scale_log2;
  __nv_bfloat16 *out;           // [total, H, 128]
  float *lse;                   // [total, H] or NULL
  int *dev_status;
};

// Bounded wait; after the first expiry in the CTA every wait returns at once.
__device__ __forceinline__ bool pwait(PfSmem &sb, uint32_t bar, uint32_t parity, int *dev_status) {
  if (*(volatile int *)&sb.abort) return false;
  if (mbar_wait(bar, parity, kWait)) return true;
  *(volatile int *)&sb.abort = 1;
  report(dev_status, MLA_ERR_TIMEOUT);
  return false;
}

// Warp-uniform bounded wait: lane 0 waits, the verdict is broadcast, and on success every lane
// observes the completed phase itself (acquire for its own reads).
__device__ __forceinline__ bool pwarp_wait(PfSmem &sb, uint32_t bar, uint32_t parity, int *dev_status) {
  int ok = 0;
  if ((threadIdx.x & 31) == 0) ok = pwait(sb, bar, parity, dev_status) ? 1 : 0;
  ok = __shfl_sync(0xffffffffu, ok, 0);
  if (ok) mbar_wait(bar, parity, kWait);
  return ok != 0;
}

__global__ void __launch_bounds__(kPThreads, 1)
prefill_tc_kernel(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mk,
                  const __grid_constant__ CUtensorMap mv, const PfParams p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char *tiles = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  PfSmem &sb = *reinterpret_cast<PfSmem *>(tiles + kTiles);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.z, s = blockIdx.y;
  const int qt = gridDim.x - 1 - blockIdx.x;                   // longest causal rows first
  const int start = p.cu_seqlens[b], L = p.cu_seqlens[b + 1] - start;
  const int q0 = qt * kPq;
  if (start < 0 || L < 0 || start + L > p.total || L > p.max_seqlen) {
    if (threadIdx.x == 0 && s == 0 && qt == 0) report(p.dev_status, MLA_ERR_BAD_INDEX);
    return;
  }
  if (q0 >= L) return;                                         // CTA-uniform
  const int nk = (min(L, q0 + kPq) + kPk - 1) / kPk;          // key tiles this query tile sees
  auto bar = [&](int i) { return smem_u32(&sb.bars[i]); };

  if (threadIdx.x == 0) {
    for (int i = 0; i < P_COUNT; ++i) mbar_init(bar(i), 1);
    mbar_init(bar(P_SEMPTY), 8);
    mbar_init(bar(P_SEMPTY + 1), 8);
    mbar_init(bar(P_PFULL), 8);
    mbar_init(bar(P_PFULL + 1), 8);
    sb.abort = 0;
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc(smem_u32(&sb.tmem_base), 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = sb.tmem_base;
  grid_dep_launch();

  if (warp == 0 && lane == 0) {
    // ---- producer: Q once, then one stage (K and V of 64 tokens) per key tile
    grid_dep_wait();
    if (!p.tiled) {
      tma_prefetch_desc(&mq);
      tma_prefetch_desc(&mk);
      tma_prefetch_desc(&mv);
    }
    mbar_expect_tx(bar(P_QFULL), kQBytes);
    const int64_t hs = (int64_t)s * p.B + b;   // (head, sequence) of the tiled workspace
    if (p.tiled)
      bulk_load(smem_u32(tiles), p.q_tiles + (hs * p.nqt + qt) * kPfQTileBytes, kQBytes, bar(P_QFULL));
    else
      for (int c = 0; c < 3; ++c)
        tma_load_2d(smem_u32(tiles + c * (kPq * 128)), &mq, s * kDqk + 64 * c, start + q0, bar(P_QFULL));
    int kt = 0;
    for (; kt < nk; ++kt) {
      const int st = kt % kPStages;
      if (kt >= kPStages && !pwait(sb, bar(P_KVEMPTY + st), ((kt / kPStages) - 1) & 1, p.dev_status)) break;
      unsigned char *stg = tiles + kOffStages + st * kStageBytes;
      mbar_expect_tx(bar(P_KVFULL + st), kStageBytes);
      if (p.tiled) {   // K (3 chunks) and V (2 chunks) of 64 tokens: one 40 KB copy
        bulk_load(smem_u32(stg), p.kv_tiles + (hs * p.nkt + kt) * kPfKVTileBytes, kStageBytes, bar(P_KVFULL + st));
      } else {
        for (int c = 0; c < 3; ++c)
          tma_load_2d(smem_u32(stg + c * kKChunk), &mk, s * kDqk + 64 * c, start + kPk * kt, bar(P_KVFULL + st));
        for (int c = 0; c < 2; ++c)
          tma_load_2d(smem_u32(stg + (3 + c) * kKChunk), &mv, s * kDvp + 64 * c, start + kPk * kt, bar(P_KVFULL + st));
      }
    }
    // Every issued load lands before the CTA may leave.
    for (int j = max(0, kt - kPStages); j < kt; ++j) pwait(sb, bar(P_KVFULL + j % kPStages), (j / kPStages) & 1, p.dev_status);
    pwait(sb, bar(P_QFULL), 0, p.dev_status);
  } else if (warp == 1 && lane == 0) {
    // ---- MMA issuer: S(kt), then O += P(kt-1) V(kt-1), so each softmax overlaps the next S.
    const uint32_t idS = idesc_bf16_f32(kPq, kPk, false, false);
    const uint32_t idO = idesc_bf16_f32(kPq, kDvp, false, true);
    pwait(sb, bar(P_QFULL), 0, p.dev_status);
    tc_fence_after();
    const uint32_t qa = smem_u32(tiles);
    for (int kt = 0; kt <= nk; ++kt) {
      if (kt < nk) {
        const int st = kt % kPStages, sbuf = kt & 1;
        if (kt >= 2) pwait(sb, bar(P_SEMPTY + sbuf), ((kt >> 1) - 1) & 1, p.dev_status);
        pwait(sb, bar(P_KVFULL + st), (kt / kPStages) & 1, p.dev_status);
        tc_fence_after();
        const uint32_t kb = smem_u32(tiles + kOffStages + st * kStageBytes);
        for (int c = 0; c < 3; ++c)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ss(tbase + kSCols + kPk * sbuf, smem_desc_sw128(qa + c * (kPq * 128) + kk * 32, 16, 1024),
                   smem_desc_sw128(kb + c * kKChunk + kk * 32, 16, 1024), idS, (c | kk) ? 1u : 0u);
        tc_commit(bar(P_SFULL + sbuf));
      }
      if (kt >= 1) {
        const int j = kt - 1, st = j % kPStages, pb = j & 1;
        pwait(sb, bar(P_PFULL + pb), (j >> 1) & 1, p.dev_status);
        tc_fence_after();
        fence_proxy_async_smem();
        const uint32_t pa = smem_u32(tiles + kOffP + pb * kPTile);
        const uint32_t vb = smem_u32(tiles + kOffStages + st * kStageBytes + 3 * kKChunk);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_ss(tbase + kOCols, smem_desc_sw128(pa + kk * 32, 16, 1024), smem_desc_sw128(vb + kk * 2048, kKChunk, 1024),
                 idO, (j | kk) ? 1u : 0u);
        tc_commit(bar(P_KVEMPTY + st));
        tc_commit(bar(P_PVDONE + pb));
      }
    }
  } else if (warp >= 4) {
    // ---- softmax: warp (quadrant q, half h) owns rows 32q.. and S columns 32h..32h+31, O columns 64h..
    const int q4 = warp & 3, h = (warp - 4) >> 2;
    const int r = q4 * 32 + lane;
    const int qp = q0 + r;                                     // query position in the sequence
    const bool real = qp < L;
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    float m_ref = -CUDART_INF_F, l = 0.f;
    for (int kt = 0; kt < nk; ++kt) {
      const int sbuf = kt & 1;
      pwarp_wait(sb, bar(P_SFULL + sbuf), (kt >> 1) & 1, p.dev_status);
      tc_fence_after();
      uint32_t sc[32];
      tmem_ld32(tbase + lane_off + kSCols + kPk * sbuf + 32 * h, sc);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(P_SEMPTY + sbuf));
      // keys 64kt + 32h + i, visible while <= qp
      const int nvalid = real ? min(32, qp - (kPk * kt + 32 * h) + 1) : 0;
      float mx = -CUDART_INF_F;
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (i < nvalid) mx = fmaxf(mx, __uint_as_float(sc[i]) * p.scale_log2);
      sb.xmax[kt & 1][h][r] = mx;
      asm volatile("bar.sync 1, 256;" ::: "memory");
      mx = fmaxf(mx, sb.xmax[kt & 1][h ^ 1][r]);
      float alpha = 1.f;
      const bool need = mx > m_ref + kRescale;
      if (need) {
        alpha = exp2f(m_ref - mx);
        l *= alpha;
        m_ref = mx;
      }
      uint32_t pk[16];
      float psum = 0.f;
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const float p0 = (2 * e < nvalid) ? exp2f(__uint_as_float(sc[2 * e]) * p.scale_log2 - m_ref) : 0.f;
        const float p1 = (2 * e + 1 < nvalid) ? exp2f(__uint_as_float(sc[2 * e + 1]) * p.scale_log2 - m_ref) : 0.f;
        pk[e] = pack_bf16x2(p0, p1);
        psum += __uint_as_float(pk[e] << 16) + __uint_as_float(pk[e] & 0xffff0000u);
      }
      l += psum;
      // P buffer kt & 1 is free once its last reader, the product of tile kt - 2, has completed; the
      // products of the previous tile may still run.  Only when a row's reference moved must O
      // hold every earlier product (tile kt - 1) before it is rescaled.
      if (kt >= 2) pwarp_wait(sb, bar(P_PVDONE + (kt & 1)), ((kt - 2) >> 1) & 1, p.dev_status);
      if (kt >= 1 && __any_sync(0xffffffffu, need)) {
        pwarp_wait(sb, bar(P_PVDONE + ((kt - 1) & 1)), ((kt - 1) >> 1) & 1, p.dev_status);
        tc_fence_after();
        {
#pragma unroll 1
          for (int c = 0; c < 2; ++c) {
            uint32_t v[32];
            tmem_ld32(tbase + lane_off + kOCols + 64 * h + 32 * c, v);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * alpha);
            tmem_st32(tbase + lane_off + kOCols + 64 * h + 32 * c, v);
          }
          tmem_wait_st();
        }
      }
      // P row r, keys 32h.. -> 16-byte groups 4h..4h+3 of the row, 128B-swizzled K-major tile.
      unsigned char *prow = tiles + kOffP + (kt & 1) * kPTile + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
      for (int c = 0; c < 4; ++c)
        *reinterpret_cast<uint4 *>(prow + (((4 * h + c) ^ (r & 7)) << 4)) =
            make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(P_PFULL + (kt & 1)));
    }
    // Row sums of both halves, then O / l and lse after the last product.
    sb.xl[h][r] = l;
    asm volatile("bar.sync 1, 256;" ::: "memory");
    l += sb.xl[h ^ 1][r];
    pwarp_wait(sb, bar(P_PVDONE + ((nk - 1) & 1)), ((nk - 1) >> 1) & 1, p.dev_status);
    tc_fence_after();
    grid_dep_wait();   // the outputs may still be read by an earlier kernel
    const float inv = l > 0.f ? 1.f / l : 0.f;
    __nv_bfloat16 *dst = p.out + ((int64_t)(start + qp) * p.H + s) * kDvp + 64 * h;
#pragma unroll 1
    for (int c = 0; c < 2; ++c) {
      uint32_t v[32];
      tmem_ld32(tbase + lane_off + kOCols + 64 * h + 32 * c, v);
      tmem_wait_ld();
      if (real && !*(volatile int *)&sb.abort)
#pragma unroll
        for (int i = 0; i < 32; i += 8)
          *reinterpret_cast<uint4 *>(dst + 32 * c + i) =
              make_uint4(pack_bf16x2(__uint_as_float(v[i]) * inv, __uint_as_float(v[i + 1]) * inv),
                         pack_bf16x2(__uint_as_float(v[i + 2]) * inv, __uint_as_float(v[i + 3]) * inv),
                         pack_bf16x2(__uint_as_float(v[i + 4]) * inv, __uint_as_float(v[i + 5]) * inv),
                         pack_bf16x2(__uint_as_float(v[i + 6]) * inv, __uint_as_float(v[i + 7]) * inv));
    }
    if (h == 0 && real && p.lse)
      p.lse[(int64_t)(start + qp) * p.H + s] = l > 0.f ? (m_ref + __log2f(l)) * 0.69314718055994531f : -CUDART_INF_F;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tbase, 256);
  }
}

// ------------------------------------------------------------ decompression
// CTA = (sequence b, head s, 128 tokens p0.. of the sequence):
//   D [128 tokens x 256] = C [128 x d_c] . [W_UK^(s) | W_UV^(s)] [d_c x 256]
// A = the tokens' latent rows (K-major, two 64-token pages per K chunk, TMA boxes from the
// row pool through the block table), B = the two weights side by side (N-major: output
// columns contiguous, 64-column chunks), streamed over d_c in stages of 64.
// Columns 0..127 are k_nope -> kbuf[t][s][0..127], columns 128..255 are v -> vbuf[t][s][..];
// the token's RoPE key is copied to kbuf[t][s][128..191].
constexpr int kDcTok = 128;                    // tokens per CTA
constexpr int kDcStages = 4;
constexpr uint32_t kDcA = kDcTok * 128;        // [128 tokens x 64 dims]: 16 KB
constexpr uint32_t kDcB = 4 * kKChunk;         // [64 dims x 256 outputs]: 4 chunks of [64 x 64]
constexpr uint32_t kDcStage = kDcA + kDcB;     // 48 KB
constexpr size_t kDcSmem = 1024 + kDcStages * kDcStage + 64;

struct DcParams {
  int H, d_c, block_size, max_blocks_per_seq, num_blocks, total;
  int tiled, B, nkt;            // tiled workspace: write K|V tiles per (head, sequence, 64-token page)
  unsigned char *kv_tiles;
  const int32_t *cu_seqlens, *block_table;
  const __nv_bfloat16 *k_pe;
  int64_t kpe_stride;
  __nv_bfloat16 *kbuf, *vbuf;
  int *dev_status;
};

__device__ __forceinline__ int64_t dc_row(const DcParams &p, int b, int pos) {
  const int lb = pos / p.block_size;
  if (lb >= p.max_blocks_per_seq) return -1;
  const int blk = p.block_table ? p.block_table[(int64_t)b * p.max_blocks_per_seq + lb] : b * p.max_blocks_per_seq + lb;
  if (blk < 0 || blk >= p.num_blocks) return -1;
  return (int64_t)blk * p.block_size + pos % p.block_size;
}

__global__ void __launch_bounds__(128, 1)
decompress_tc_kernel(const __grid_constant__ CUtensorMap mc, const __grid_constant__ CUtensorMap mwk,
                     const __grid_constant__ CUtensorMap mwv, const DcParams p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char *tiles = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t full[kDcStages], empty[kDcStages], done;
  __shared__ uint32_t tmem_slot;
  __shared__ int page_row[2];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.z, s = blockIdx.y;
  const int start = p.cu_seqlens[b], L = p.cu_seqlens[b + 1] - start;
  const int p0 = blockIdx.x * kDcTok;
  if (start < 0 || L < 0 || start + L > p.total) {
    if (threadIdx.x == 0 && s == 0 && blockIdx.x == 0) report(p.dev_status, MLA_ERR_BAD_INDEX);
    return;
  }
  if (p0 >= L) return;                                          // CTA-uniform
  const int nkc = p.d_c / 64;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kDcStages; ++i) {
      mbar_init(smem_u32(&full[i]), 1);
      mbar_init(smem_u32(&empty[i]), 1);
    }
    mbar_init(smem_u32(&done), 1);
    fence_mbar_init();
  }
  if (threadIdx.x < 2) {
    // first pool row of each 64-token page of the tile (-1: past the end or a bad block id)
    const int pos = p0 + 64 * threadIdx.x;
    page_row[threadIdx.x] = pos < L ? (int)dc_row(p, b, pos) : -1;
  }
  if (warp == 2) {
    tmem_alloc(smem_u32(&tmem_slot), 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = tmem_slot;
  grid_dep_launch();
  int ok = 1;
  if (warp == 0 && lane == 0) {
    grid_dep_wait();
    for (int kc = 0; kc < nkc; ++kc) {
      const int st = kc % kDcStages;
      if (kc >= kDcStages && !mbar_wait(smem_u32(&empty[st]), ((kc / kDcStages) - 1) & 1, kWait)) {
        report(p.dev_status, MLA_ERR_TIMEOUT);
        ok = 0;
        break;
      }
      unsigned char *stg = tiles + st * kDcStage;
      mbar_expect_tx(smem_u32(&full[st]), kDcStage);
      for (int pg = 0; pg < 2; ++pg)   // a page past the end (or invalid) reads row 0: masked on output
        tma_load_2d(smem_u32(stg + pg * (64 * 128)), &mc, 64 * kc, max(page_row[pg], 0), smem_u32(&full[st]));
      for (int c = 0; c < 2; ++c) {
        tma_load_2d(smem_u32(stg + kDcA + c * kKChunk), &mwk, 64 * c, s * p.d_c + 64 * kc, smem_u32(&full[st]));
        tma_load_2d(smem_u32(stg + kDcA + (2 + c) * kKChunk), &mwv, 64 * c, s * p.d_c + 64 * kc, smem_u32(&full[st]));
      }
    }
  } else if (warp == 1 && lane == 0) {
    const uint32_t idesc = idesc_bf16_f32(128, 256, false, true);
    for (int kc = 0; kc < nkc; ++kc) {
      const int st = kc % kDcStages;
      if (!mbar_wait(smem_u32(&full[st]), (kc / kDcStages) & 1, kWait)) {
        report(p.dev_status, MLA_ERR_TIMEOUT);
        ok = 0;
        break;
      }
      tc_fence_after();
      const uint32_t a = smem_u32(tiles + st * kDcStage), bb = a + kDcA;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_ss(tbase, smem_desc_sw128(a + kk * 32, 16, 1024), smem_desc_sw128(bb + kk * 2048, kKChunk, 1024), idesc,
               (kc | kk) ? 1u : 0u);
      tc_commit(smem_u32(&empty[st]));
    }
    tc_commit(smem_u32(&done));
  }
  ok = __syncthreads_and(ok);
  int ok2 = 0;
  if (lane == 0 && ok) ok2 = mbar_wait(smem_u32(&done), 0, kWait) ? 1 : 0;
  ok2 = __shfl_sync(0xffffffffu, ok2, 0);
  if (ok2) mbar_wait(smem_u32(&done), 0, kWait);
  tc_fence_after();
  grid_dep_wait();
  // Thread = token p0 + 32w + lane (its tensor-memory lane): 256 outputs -> kbuf / vbuf rows, or
  // its row of the K|V tile of its 64-token page (rows past the sequence end are zeroed there, so
  // the attention's masked products meet finite values).
  const int tok = 32 * warp + lane, pos = p0 + tok;
  const bool real = ok2 && pos < L && page_row[tok >> 6] >= 0;
  const int64_t t = start + pos;
  unsigned char *tile = p.tiled ? p.kv_tiles + (((int64_t)s * p.B + b) * p.nkt + pos / 64) * kPfKVTileBytes : nullptr;
  const int prow = pos & 63;
#pragma unroll 1
  for (int c = 0; c < 8; ++c) {
    uint32_t v[32];
    tmem_ld32(tbase + ((uint32_t)(32 * warp) << 16) + 32 * c, v);
    tmem_wait_ld();
    if (p.tiled) {
      // columns 32c .. 32c+31: K dims 32c.. (c < 4) or V dims 32(c-4).. (V follows the 3 K chunks)
      unsigned char *base = c < 4 ? tile : tile + 3 * kKChunk;
      const int d0 = c < 4 ? 32 * c : 32 * (c - 4);
#pragma unroll
      for (int i = 0; i < 32; i += 8)
        *reinterpret_cast<uint4 *>(base + swz_tile_offset(64, prow, d0 + i)) =
            real ? make_uint4(pack_bf16x2(__uint_as_float(v[i]), __uint_as_float(v[i + 1])),
                              pack_bf16x2(__uint_as_float(v[i + 2]), __uint_as_float(v[i + 3])),
                              pack_bf16x2(__uint_as_float(v[i + 4]), __uint_as_float(v[i + 5])),
                              pack_bf16x2(__uint_as_float(v[i + 6]), __uint_as_float(v[i + 7])))
                 : make_uint4(0, 0, 0, 0);
    } else if (real) {
      __nv_bfloat16 *dst = c < 4 ? p.kbuf + (t * p.H + s) * kDqk + 32 * c : p.vbuf + (t * p.H + s) * kDvp + 32 * (c - 4);
#pragma unroll
      for (int i = 0; i < 32; i += 8)
        *reinterpret_cast<uint4 *>(dst + i) =
            make_uint4(pack_bf16x2(__uint_as_float(v[i]), __uint_as_float(v[i + 1])),
                       pack_bf16x2(__uint_as_float(v[i + 2]), __uint_as_float(v[i + 3])),
                       pack_bf16x2(__uint_as_float(v[i + 4]), __uint_as_float(v[i + 5])),
                       pack_bf16x2(__uint_as_float(v[i + 6]), __uint_as_float(v[i + 7])));
    }
  }
  // the shared RoPE key, already rotated in the cache (zeros past the end in the tiled layout)
  const int64_t row = real ? (int64_t)page_row[tok >> 6] + (tok & 63) : 0;
  const uint4 *src = reinterpret_cast<const uint4 *>(p.k_pe + row * p.kpe_stride);
  if (p.tiled) {
#pragma unroll
    for (int i = 0; i < 8; ++i)
      *reinterpret_cast<uint4 *>(tile + swz_tile_offset(64, prow, 128 + 8 * i)) = real ? src[i] : make_uint4(0, 0, 0, 0);
  } else if (real) {
    uint4 *dst = reinterpret_cast<uint4 *>(p.kbuf + (t * p.H + s) * kDqk + 128);
#pragma unroll
    for (int i = 0; i < 8; ++i) dst[i] = src[i];
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tbase, 256);
  }
}

}  // namespace

bool prefill_tc_supported(const PrefillArgs &a, bool bf16) {
  return bf16 && a.d_nope + a.d_rope == kDqk && a.d_v == kDvp && a.cache.d_c > 0 &&
         !(reinterpret_cast<uintptr_t>(a.qbuf) & 15) && !(reinterpret_cast<uintptr_t>(a.kbuf) & 15) &&
         !(reinterpret_cast<uintptr_t>(a.vbuf) & 15) && !(reinterpret_cast<uintptr_t>(a.out) & 15);
}

bool decompress_tc_supported(const PrefillArgs &a, bool bf16) {
  const CacheView &c = a.cache;
  return bf16 && a.d_nope == 128 && a.d_v == kDvp && a.d_rope == 64 && a.d_c % 64 == 0 && c.layout == MLA_CACHE_ROWS &&
         c.block_size % 64 == 0 && !(reinterpret_cast<uintptr_t>(c.c_kv) & 15) &&
         !(reinterpret_cast<uintptr_t>(c.k_pe) & 15) && (c.ckv_stride * 2) % 16 == 0 && (c.kpe_stride * 2) % 16 == 0 &&
         !(reinterpret_cast<uintptr_t>(a.w_uk) & 15) && !(reinterpret_cast<uintptr_t>(a.w_uv) & 15) &&
         !(reinterpret_cast<uintptr_t>(a.kbuf) & 15) && !(reinterpret_cast<uintptr_t>(a.vbuf) & 15);
}

int launch_decompress_tc(const PrefillArgs &a, cudaStream_t st) {
  const CacheView &c = a.cache;
  CUtensorMap mc, mwk, mwv;
  const uint64_t pool_rows = (uint64_t)c.num_blocks * c.block_size;
  if (!make_tmap_bf16(&mc, c.c_kv, a.d_c, pool_rows, (uint64_t)c.ckv_stride * 2, 64) ||
      !make_tmap_bf16(&mwk, a.w_uk, a.d_nope, (uint64_t)a.H * a.d_c, (uint64_t)a.d_nope * 2, 64) ||
      !make_tmap_bf16(&mwv, a.w_uv, a.d_v, (uint64_t)a.H * a.d_c, (uint64_t)a.d_v * 2, 64))
    return MLA_ERR_CUDA;
  if (cudaFuncSetAttribute(decompress_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kDcSmem))
    return MLA_ERR_CUDA;
  DcParams p;
  p.H = a.H;
  p.d_c = a.d_c;
  p.block_size = c.block_size;
  p.max_blocks_per_seq = c.max_blocks_per_seq;
  p.num_blocks = c.num_blocks;
  p.total = a.total;
  p.cu_seqlens = a.cu_seqlens;
  p.block_table = c.block_table;
  p.k_pe = static_cast<const __nv_bfloat16 *>(c.k_pe);
  p.kpe_stride = c.kpe_stride;
  p.kbuf = static_cast<__nv_bfloat16 *>(a.kbuf);
  p.vbuf = static_cast<__nv_bfloat16 *>(a.vbuf);
  p.dev_status = a.dev_status;
  p.tiled = a.tiled;
  p.B = a.B;
  p.nkt = a.nkt;
  p.kv_tiles = a.kv_tiles;
  const dim3 grid((a.max_seqlen + kDcTok - 1) / kDcTok, a.H, a.B);
  return launch_pdl(decompress_tc_kernel, grid, dim3(128), kDcSmem, st, mc, mwk, mwv, p) == cudaSuccess ? MLA_OK
                                                                                                    : MLA_ERR_CUDA;
}

int launch_prefill_tc_attention(const PrefillArgs &a, cudaStream_t st) {
  CUtensorMap mq, mk, mv;
  const uint64_t rows = a.total;
  if (!make_tmap_bf16(&mq, a.qbuf, (uint64_t)a.H * kDqk, rows, (uint64_t)a.H * kDqk * 2, kPq) ||
      !make_tmap_bf16(&mk, a.kbuf, (uint64_t)a.H * kDqk, rows, (uint64_t)a.H * kDqk * 2, kPk) ||
      !make_tmap_bf16(&mv, a.vbuf, (uint64_t)a.H * kDvp, rows, (uint64_t)a.H * kDvp * 2, kPk))
    return MLA_ERR_CUDA;
  if (cudaFuncSetAttribute(prefill_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kPfSmem))
    return MLA_ERR_CUDA;
  PfParams p;
  p.B = a.B;
  p.H = a.H;
  p.tiled = a.tiled;
  p.nqt = a.nqt;
  p.nkt = a.nkt;
  p.q_tiles = a.q_tiles;
  p.kv_tiles = a.kv_tiles;
  p.max_seqlen = a.max_seqlen;
  p.total = a.total;
  p.cu_seqlens = a.cu_seqlens;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  p.out = static_cast<__nv_bfloat16 *>(a.out);
  p.lse = a.lse;
  p.dev_status = a.dev_status;
  const dim3 grid((a.max_seqlen + kPq - 1) / kPq, a.H, a.B);
  return launch_pdl(prefill_tc_kernel, grid, dim3(kPThreads), kPfSmem, st, mq, mk, mv, p) == cudaSuccess
             ? MLA_OK
             : MLA_ERR_CUDA;
}

}  // namespace mla
