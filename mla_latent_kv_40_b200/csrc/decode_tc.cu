// Split-KV MLA decode on 5th-generation tensor cores (tcgen05, sm_100a).
//
// The absorbed decode form of "Transformer升级之路：21、MLA好在哪里?（下）",
// section 双重投影, decoding column: all heads of a sequence attend to the same
// cached rows [c_i | kpe_i] (576 wide), so one 128-row block of queries
// (head x query token) against a 64-key tile is a dense contraction:
//   S = Q [128 x 576] . K^T [576 x 64]        (scores)
//   O += P [128 x 64] . C [64 x 512]          (softmax-weighted latents)
//
// Resources decide the shape of the kernel.  O is 128 x 512 fp32 = 256 KB, the
// whole tensor memory of one SM, and Q is 147 KB of bf16.  So each work unit
// runs on a cluster of two CTAs on two SMs:
//   * the score CTA (rank 0) keeps the latent part of Q in its tensor memory
//     (A operand of TS-form MMAs) and the RoPE part in shared memory, streams
//     the unit's pages as half-page stages (one 32-40 KB contiguous bulk copy
//     each from the tiled pool), computes S for two pages at a time into one
//     of two tensor-memory buffers, runs the online softmax in registers, and
//     sends each page of P (bf16, staged in shared memory) to the value CTA
//     with one shared-to-peer bulk copy (distributed shared memory);
//   * the value CTA (rank 1) streams the 512-wide latent part of the same
//     pages and accumulates O = P . C in all 512 tensor-memory columns, then
//     normalises and writes the unit's partial output.
// The score CTA does 53% of the MMA work and the value CTA 47%.
//
// One thread issues a tcgen05.mma about every 128 cycles, whatever N is: enough
// to keep the tensor pipe busy at N = 256, a quarter of its rate at N = 64.  So
// each CTA issues from two threads on different SM sub-partitions, each with its
// own accumulator: in the score CTA one thread per page of a score tile (N = 64
// each), in the value CTA one thread per 256-column half of O (N = 256), served
// by its own group of four epilogue warps.
//
// Online softmax uses a lazy reference maximum (kept in log2 units): P is
// exp2(s - m_ref) and m_ref only moves when a tile's maximum exceeds it by more
// than 8, so the O accumulator is rescaled (tcgen05.ld / st by the value CTA)
// only on those rare tiles.  The row sum adds P in fp32 (before its rounding to bf16), and O is
// divided by it once, at the end.
//
// Work is split over the persistent clusters by 64-key tiles across all
// (sequence, 128-row block) units, at about equal cost (a unit start costs a few
// tiles: see Split); a unit cut between clusters leaves one partial (O / l, lse)
// per piece, merged by the merge kernel.  Every wait on
// an mbarrier is bounded in time: on expiry the kernel reports MLA_ERR_TIMEOUT,
// drains its in-flight copies, frees its tensor memory and returns.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math_constants.h>
#include <type_traits>

#include <atomic>
#include <cstring>
#include <mutex>

#include "decode_tc.cuh"
#include "mma_tile.cuh"
#include "sm100.cuh"

namespace mla {
namespace {

using namespace sm100;

constexpr int kTileKeys = 64;                      // one cache page of keys (a "page tile")
constexpr int kSuper = 2;                          // page tiles per score tile: N = 128 keys per MMA
constexpr int kDc = 512, kDr = 64, kW = kDc + kDr;
constexpr int kRows = 128;                         // M of every MMA: query rows per unit
constexpr int kKStages = 4;                        // score CTA: half-page stages in flight (two pages)
static_assert(kKStages == 2 * 2, "one stage pair per page position of a score tile");
constexpr int kVStages = 4;                        // value CTA: [64 keys x 256 dims] half-page stages in flight
constexpr int kThreads = 384;
constexpr int kLaunchRegs = 168;                   // per thread (65536 / 384, rounded down to 8)
constexpr uint32_t kChunkBytes = kTileKeys * 128;  // one [64 keys x 64 dims] bf16 TMA box, 128B-swizzled
// A score-CTA stage is half a page, brought in by ONE contiguous bulk copy: chunks 0-3 (the
// first 256 latent dims, 32 KB) or chunks 4-8 (the other 256 latent dims and the RoPE key, 40 KB).
// One SM's copy engine sustains about 5 M bulk copies a second, so 8 KB copies cap an SM near
// 42 GB/s while 32-40 KB copies run it at 90+ GB/s.
__host__ __device__ constexpr int half_chunks(int half) { return half ? 5 : 4; }
constexpr uint32_t kKStageBytes = 5 * kChunkBytes;                 // 40960 (room for the larger half)
constexpr uint32_t kVStageBytes = 4 * kChunkBytes;                 // 32768
constexpr uint32_t kPBytes = kRows * kTileKeys * 2;                // 16384
constexpr int kPSlots = 5;                         // P page tiles in flight from the score CTA to the value CTA
constexpr uint32_t kPWriters = 4;                 // softmax warps that write one P page (one per lane quadrant)
constexpr uint32_t kPaWords = 36;                  // per writer warp: 32 row rescale factors, a flag word, padding
constexpr uint32_t kStgBytes = 4096 + kPaWords * 4;                // score CTA: one warp's P rows + factors, staged
constexpr uint32_t kPTxBytes = kPWriters * kStgBytes;              // bytes that fill one P slot
// A P slot (value CTA) and a P staging tile (score CTA) hold a page of P (16 KB) followed by its
// rescale factors, so that ONE bulk copy moves both; the stride keeps every P page 1024-aligned.
constexpr uint32_t kPSlotBytes = ((kPTxBytes + 1023) / 1024) * 1024;   // 17408
constexpr uint32_t kQpeOff = 0;                                    // score CTA: Q rope part, [128 x 64] bf16
constexpr uint32_t kKOff = kRows * 128;                            // score CTA: key stages
constexpr uint32_t kPOff = kVStages * kVStageBytes;                // value CTA: P slots
constexpr uint32_t kStgOff = kKOff + kKStages * kKStageBytes;      // score CTA: P pages of both halves, factors
constexpr uint32_t kScoreEnd = kStgOff + 2 * kPSlotBytes, kValueEnd = kPOff + kPSlots * kPSlotBytes;
constexpr uint32_t kRegionA = ((kScoreEnd > kValueEnd ? kScoreEnd : kValueEnd) + 1023) & ~1023u;   // 214016
static_assert(kPOff + kPSlots * kPSlotBytes <= kRegionA, "value-CTA tiles must fit the shared region");
constexpr float kRescaleLog2 = 8.f;
constexpr uint64_t kWaitNs = 2000000000ull;        // 2 s per wait
constexpr int kMaxClusters = 128;
constexpr int kTimeoutRecInts = 1 + 6 * 2 * (kThreads / 32);

// TMEM columns
constexpr uint32_t kQCol = 0;      // score CTA: latent part of Q, 256 columns (2 bf16 per column)
constexpr uint32_t kSCol = 256;    // score CTA: S, two buffers of 128 columns (one score tile each)
// value CTA: O in columns 0..511

// Barrier slots (same indices in both CTAs).
enum Bar {
  B_KFULL = 0, B_KEMPTY = B_KFULL + kKStages, B_SFULL = B_KEMPTY + kKStages, B_SEMPTY = B_SFULL + 2,
  B_QREADY = B_SEMPTY + 2, B_PEMPTY = B_QREADY + 1, B_STATSEMPTY = B_PEMPTY + kPSlots,
  B_VFULL = B_STATSEMPTY + 1, B_VEMPTY = B_VFULL + kVStages, B_PFULL = B_VEMPTY + kVStages,
  B_PVDONE = B_PFULL + kPSlots, B_REQ = B_PVDONE + kPSlots, B_REQDONE = B_REQ + 2, B_STATSFULL = B_REQDONE + 2,
  B_OFREE = B_STATSFULL + 1, B_COUNT = B_OFREE + 1
};

// A request from the value CTA's MMA thread to its epilogue warps.
struct Req {
  int kind;        // 0: fix up a tile before its MMA, 1: unit epilogue
  int vstage, slot, nvalid, tail, rescale, segid, last_slot, last_parity;
};

struct SmemB {                       // small region after the tiles
  float stat_l[kRows], stat_m[kRows];// value CTA: row sum and reference max of a finished unit
  float xmax[2][2][kRows];           // score CTA: the two softmax halves' tile maxima (double-buffered)
  float xl[2][kRows];                // score CTA: the two halves' row sums at the end of a unit
  uint64_t bars[B_COUNT];
  Req req[2];                        // value CTA: one request channel per O half (issuer -> epilogue group)
  uint32_t tmem_base;
  int abort;
  int plan_u0, plan_p0, plan_s0;     // first unit of this cluster, its tile prefix and segment prefix
  int plan_k0;                       // non-empty units before the first unit
  int plan_C;                        // clusters that get work: min(launched clusters, total tiles)
  int plan_beta;                     // cost of a unit start, in tiles (see Split)
  long long plan_W;                  // total cost
  int prog[kThreads / 32];           // per-warp progress (tiles handled), kept for timeout records
  long long plan_start, plan_end, plan_total;
};
constexpr size_t kSmemBytes = 1024 + kRegionA + sizeof(SmemB);
static_assert(kSmemBytes <= 232448, "shared memory budget");

// Value CTA: shared address of the rescale factors that arrived with P slot pb, per writer warp: its
// 32 rows' factors, a flag word ("some row of this tile rescaled") and padding.
__device__ __forceinline__ uint32_t slot_factors(uint32_t tiles_s, int pb) {
  return tiles_s + kPOff + pb * kPSlotBytes + kPBytes;
}

__device__ __forceinline__ uint32_t ld_shared_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}

struct TcParams {
  int B, n_q, H, n_rb, U, max_seqlen;
  int kv_begin, kv_end;              // attend to keys in [kv_begin, kv_end) only (kv_begin a multiple of 64)
  const __nv_bfloat16 *q;            // [B, n_q, H, 576]
  const int32_t *seqlens, *block_table;
  int max_blocks_per_seq, num_blocks, block_size;
  float scale_log2;
  __nv_bfloat16 *o_part;             // [seg][128][512], O / l of each segment
  float *lse_part;                   // [seg][128]
  int *seg_info;                     // [U][2]
  int *timeout_rec;                  // [kTimeoutRecInts]: where bounded waits gave up (diagnostics)
  int *dev_status;
  const unsigned char *tiled;        // tiled page pool (pages move by bulk copy), or NULL: row pool via TMA maps
  const unsigned char *row_pool;     // row pool base (c_kv) for L2 prefetch
  int rows_contig;                   // row pool with fused 576-wide rows: a page is 73728 contiguous bytes
};

__device__ __forceinline__ int seq_len_clamped(const TcParams &p, int b) {
  const int S = p.seqlens[b];
  return S < 0 ? 0 : (S > p.max_seqlen ? p.max_seqlen : S);
}

// End of the keys a unit reads: the sequence's end or the key range's, whichever comes first.
__device__ __forceinline__ int key_end(const TcParams &p, int b) {
  const int S = seq_len_clamped(p, b);
  return S < p.kv_end ? S : p.kv_end;
}

// Tiles (64-key pages) of a unit inside the key range; tile t holds keys kv_begin + 64 t ...
__device__ __forceinline__ int unit_tiles(const TcParams &p, int u) {
  const int e = key_end(p, u / p.n_rb) - p.kv_begin;
  return e > 0 ? (e + kTileKeys - 1) / kTileKeys : 0;
}

// Work split.  The units' 64-key tiles, in unit order, are cut into C ranges of about equal cost.
// A tile costs 1, and every unit start after the first costs kBoundaryCost more: a cluster that
// moves on to a new unit drains and refills its pipeline there (the next query block goes into
// tensor memory, the finished unit's O is written out).  On V3 shapes at batch 64 x 4096, cluster
// end times fit ~1.56 us per tile plus ~12.5 us per segment, so a unit start costs ~8 tiles.
// Tile t of unit u costs t + beta k_u (k_u: non-empty units before u); cluster c owns the tiles
// whose cost lies in [floor(c W / C), floor((c+1) W / C)).  beta is used only while one unit start
// cannot jump over a whole cluster's share, (beta + 1) C <= W.
constexpr int kBoundaryCost = 8;
struct Split {
  long long W;   // total cost: tiles + beta (non-empty units - 1)
  int beta, C;
};

__device__ __forceinline__ int cluster_of(long long t, int k, const Split &sp) {
  const long long cost = t + (long long)sp.beta * k;
  return (int)(((cost + 1) * sp.C + sp.W - 1) / sp.W - 1);
}

// Warp-level plan: total tiles and cost, this cluster's tile range, its first unit and the tile,
// non-empty-unit and segment prefixes of that unit.  Every CTA computes the same values.
__device__ __forceinline__ void make_plan(const TcParams &p, SmemB &sb, int cid, int C) {
  const int lane = threadIdx.x & 31;
  long long total = 0;
  int une = 0;
  for (int u0 = 0; u0 < p.U; u0 += 32) {
    const int u = u0 + lane;
    int nt = u < p.U ? unit_tiles(p, u) : 0;
    une += __popc(__ballot_sync(0xffffffffu, nt > 0));
#pragma unroll
    for (int o = 16; o; o >>= 1) nt += __shfl_xor_sync(0xffffffffu, nt, o);
    total += nt;
  }
  // With fewer tiles than clusters only the first `total` clusters get work, so
  // that every active range is non-empty and segment ids have no gaps.
  C = (int)(total < C ? total : C);
  Split sp;
  sp.C = C > 0 ? C : 1;
  sp.beta = kBoundaryCost;
  sp.W = total + (long long)sp.beta * (une > 0 ? une - 1 : 0);
  if ((long long)(sp.beta + 1) * sp.C > sp.W) {
    sp.beta = 0;
    sp.W = total;
  }
  if (sp.W <= 0) sp.W = 1;
  // Cluster c's range is [x_c, x_{c+1}) with x_c the first tile of cost >= floor(c W / C); inside
  // unit u that is max(P_u, floor(c W / C) - beta k_u), in the first unit whose last tile reaches it.
  const long long Ls = cid < C ? (long long)cid * sp.W / sp.C : 0;
  const long long Le = cid < C ? (long long)(cid + 1) * sp.W / sp.C : 0;
  const bool last_c = cid + 1 >= C;
  long long tp = 0, sp_seg = 0;   // running tile / segment prefix
  int kp = 0;                     // running count of non-empty units
  int found = -1;
  long long fp = 0, fs = 0, start = 0, end = last_c ? total : -1;
  int fk = 0;
  for (int u0 = 0; u0 < p.U && (found < 0 || end < 0); u0 += 32) {
    const int u = u0 + lane;
    const int nt = u < p.U ? unit_tiles(p, u) : 0;
    // inclusive scans of nt and of (nt > 0)
    int inc = nt, kinc = nt > 0 ? 1 : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, inc, o);
      const int kv = __shfl_up_sync(0xffffffffu, kinc, o);
      if (lane >= o) {
        inc += v;
        kinc += kv;
      }
    }
    const long long my_p = tp + inc - nt;
    const int my_k = kp + kinc - (nt > 0 ? 1 : 0);
    int ns = 0;
    if (nt > 0 && total > 0) ns = cluster_of(my_p + nt - 1, my_k, sp) - cluster_of(my_p, my_k, sp) + 1;
    int sinc = ns;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, sinc, o);
      if (lane >= o) sinc += v;
    }
    const long long my_s = sp_seg + sinc - ns;
    const long long last_cost = my_p + nt - 1 + (long long)sp.beta * my_k;
    if (found < 0) {
      const unsigned m = __ballot_sync(0xffffffffu, u < p.U && nt > 0 && last_cost >= Ls);
      if (m) {
        const int src = __ffs(m) - 1;
        found = u0 + src;
        fp = __shfl_sync(0xffffffffu, my_p, src);
        fs = __shfl_sync(0xffffffffu, my_s, src);
        fk = __shfl_sync(0xffffffffu, my_k, src);
        const long long x = Ls - (long long)sp.beta * fk;
        start = x > fp ? x : fp;
      }
    }
    if (end < 0) {
      const unsigned m = __ballot_sync(0xffffffffu, u < p.U && nt > 0 && last_cost >= Le);
      if (m) {
        const int src = __ffs(m) - 1;
        const long long ep = __shfl_sync(0xffffffffu, my_p, src);
        const long long x = Le - (long long)sp.beta * __shfl_sync(0xffffffffu, my_k, src);
        end = x > ep ? x : ep;
      }
    }
    tp += __shfl_sync(0xffffffffu, inc, 31);
    kp += __shfl_sync(0xffffffffu, kinc, 31);
    sp_seg += __shfl_sync(0xffffffffu, sinc, 31);
  }
  if (end < 0) end = total;
  if (lane == 0) {
    sb.plan_C = sp.C;
    sb.plan_beta = sp.beta;
    sb.plan_W = sp.W;
    sb.plan_total = total;
    sb.plan_start = start;
    sb.plan_end = (found < 0 || cid >= C) ? start : end;
    sb.plan_u0 = found < 0 ? 0 : found;
    sb.plan_p0 = (int)fp;
    sb.plan_s0 = (int)fs;
    sb.plan_k0 = fk;
  }
}

// Iterates the (unit, tile range) segments of this cluster.
struct SegIter {
  int u, prefix, seg_prefix, k;   // k: non-empty units before u
  long long pos, end;
  Split sp;
  __device__ __forceinline__ bool next(const TcParams &p, int cid, int &b, int &rb, int &t0, int &t1, int &segid, bool &first_of_unit,
                       int &nseg_unit) {
    while (pos < end && u < p.U) {
      const int nt = unit_tiles(p, u);
      const long long lo = pos > prefix ? pos : prefix;
      const long long hi = end < (long long)prefix + nt ? end : (long long)prefix + nt;
      const int c0 = nt > 0 ? cluster_of(prefix, k, sp) : 0;
      const int ns = nt > 0 ? cluster_of((long long)prefix + nt - 1, k, sp) - c0 + 1 : 0;
      if (lo < hi) {
        b = u / p.n_rb;
        rb = u % p.n_rb;
        t0 = (int)(lo - prefix);
        t1 = (int)(hi - prefix);
        segid = seg_prefix + (cid - c0);
        first_of_unit = (lo == prefix);
        nseg_unit = ns;
        const int cur_u = u;
        // advance
        pos = hi;
        if (hi == (long long)prefix + nt) {
          prefix += nt;
          seg_prefix += ns;
          k += nt > 0 ? 1 : 0;
          u = cur_u + 1;
        }
        return true;
      }
      prefix += nt;
      seg_prefix += ns;
      k += nt > 0 ? 1 : 0;
      ++u;
    }
    return false;
  }
};

// Bounded wait that turns a timeout into the CTA-wide abort state.  The first
// timeout of each (CTA rank, warp) in the grid is recorded in rec[1 + 6 * (12 * rank + warp) ..]:
// cluster, barrier slot, parity, source line, the warp's progress counter.  The record is
// written out of line (it only runs after a timeout), which keeps the many inlined waits small.
__device__ __noinline__ bool wait_timed_out(SmemB &sb, uint32_t bar, uint32_t parity, int *dev_status, int *rec,
                                            int tag) {
  *(volatile int *)&sb.abort = 1;
  report(dev_status, MLA_ERR_TIMEOUT);
  if (rec) {
    const int w = (int)(threadIdx.x >> 5);
    int *e = rec + 1 + 6 * ((kThreads / 32) * (int)cluster_ctarank() + w);
    if (atomicCAS(e, 0, 1) == 0) {
      e[1] = (int)cluster_id_x();
      e[2] = (int)((bar - smem_u32(&sb.bars[0])) / 8);
      e[3] = (int)parity;
      e[4] = tag;
      e[5] = sb.prog[w];
    }
    atomicAdd(rec, 1);
  }
  return false;
}

__device__ __forceinline__ bool wait_or_abort(SmemB &sb, uint32_t bar, uint32_t parity, int *dev_status,
                                              bool cluster_scope = false, int *rec = nullptr, int tag = 0) {
  if (*(volatile int *)&sb.abort) return false;
  if (mbar_wait(bar, parity, kWaitNs, cluster_scope)) return true;
  return wait_timed_out(sb, bar, parity, dev_status, rec, tag);
}

// Warp-uniform bounded wait: lane 0 waits, the verdict is broadcast, and then
// every lane observes the completed phase itself (acquire for its own reads).
// The phase cannot move on in between: the next completion of the same
// barrier needs an arrival from this warp.
__device__ __forceinline__ bool warp_wait(SmemB &sb, uint32_t bar, uint32_t parity, int *dev_status,
                                          bool cluster_scope = false, int *rec = nullptr, int tag = 0) {
  int ok = 0;
  if ((threadIdx.x & 31) == 0) ok = wait_or_abort(sb, bar, parity, dev_status, cluster_scope, rec, tag) ? 1 : 0;
  ok = __shfl_sync(0xffffffffu, ok, 0);
  if (ok) mbar_wait(bar, parity, kWaitNs, cluster_scope);
  return ok != 0;
}

__device__ __forceinline__ int64_t tile_row(const TcParams &p, int b, int t) {
  const int key = p.kv_begin + t * kTileKeys;
  const int lb = key / p.block_size;
  if (lb >= p.max_blocks_per_seq) return -1;
  const int blk = p.block_table ? p.block_table[(int64_t)b * p.max_blocks_per_seq + lb]
                                : b * p.max_blocks_per_seq + lb;
  if (blk < 0 || blk >= p.num_blocks) return -1;
  return (int64_t)blk * p.block_size + (key % p.block_size);
}

// Pool rows of a sequence's pages, looked up a warp-load at a time: lane l keeps the
// rows of pages base + l and base + 32 + l.  Warp-collective; pages must be asked
// for in non-decreasing order per sequence, at most 32 pages behind the newest.
struct PageRows {
  int b = -1, base = 0;
  int64_t r0 = -1, r1 = -1;
  __device__ __forceinline__ void load(const TcParams &p) {
    const int lane = threadIdx.x & 31;
    r0 = tile_row(p, b, base + lane);
    r1 = tile_row(p, b, base + 32 + lane);
  }
  __device__ __forceinline__ int64_t get(const TcParams &p, int seq, int page) {
    if (seq != b || page < base || page >= base + 96) {
      b = seq;
      base = page;
      load(p);
    } else if (page >= base + 64) {
      base += 32;
      r0 = r1;
      r1 = tile_row(p, b, base + 32 + (threadIdx.x & 31));
    }
    const int k = page - base;
    return __shfl_sync(0xffffffffu, k < 32 ? r0 : r1, k & 31);
  }
};

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
mla_decode_tc_kernel(const __grid_constant__ CUtensorMap map_c, const __grid_constant__ CUtensorMap map_pe,
                     const __grid_constant__ TcParams p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char *tiles = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  SmemB &sb = *reinterpret_cast<SmemB *>(tiles + kRegionA);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int cid = (int)cluster_id_x();
  const int C = (int)nclusters_x();
  auto bar = [&](int i) { return smem_u32(&sb.bars[i]); };
  const uint32_t peer = rank ^ 1u;

  // The next kernel on the stream may start its prologue now.  Roles that read what an earlier
  // kernel of this library writes (queries, pool pages) or that write global memory call
  // grid_dep_wait() first; the prologue below touches inputs only.
  grid_dep_launch();
  if (threadIdx.x < 8) sb.prog[threadIdx.x] = 0;
  if (threadIdx.x == 0) {
    uint32_t counts[B_COUNT];
    for (int i = 0; i < B_COUNT; ++i) counts[i] = 1;
    counts[B_SEMPTY] = counts[B_SEMPTY + 1] = 8;      // one per softmax warp
    counts[B_QREADY] = 8;
    counts[B_SFULL] = counts[B_SFULL + 1] = 2;      // one commit per score-MMA issuer
    counts[B_STATSEMPTY] = 8;                         // remote, one per value-CTA epilogue warp
    for (int i = 0; i < kPSlots; ++i) counts[B_PVDONE + i] = 2;   // one commit per value-MMA issuer
    // P full: the relay's arrival, which also arms the bytes the four writer warps' bulk copies bring.
    counts[B_REQDONE] = counts[B_REQDONE + 1] = kRows;   // the four warps of one epilogue group
    counts[B_STATSFULL] = kRows;                      // remote, every softmax thread
    counts[B_OFREE] = 2 * kRows;                      // both epilogue groups
    for (int i = 0; i < B_COUNT; ++i) mbar_init(bar(i), counts[i]);
    if (rank == 1)
      for (int i = 0; i < kPSlots; ++i) mbar_expect_tx(bar(B_PFULL + i), kPTxBytes);
    sb.abort = 0;
    fence_mbar_init();
  }
  if (warp == 3) {
    tmem_alloc(smem_u32(&sb.tmem_base), 512);
    tmem_relinquish();
  }
  if (warp == 0) make_plan(p, sb, cid, C);
  if (threadIdx.x == 32 && !p.tiled) {
    tma_prefetch_desc(&map_c);
    tma_prefetch_desc(&map_pe);
  }
  tc_fence_before();
  cluster_sync();   // barriers initialised in both CTAs before any remote arrive
  tc_fence_after();
  const uint32_t tbase = sb.tmem_base;

  SegIter it0;
  it0.u = sb.plan_u0;
  it0.prefix = sb.plan_p0;
  it0.seg_prefix = sb.plan_s0;
  it0.k = sb.plan_k0;
  it0.pos = sb.plan_start;
  it0.end = sb.plan_end;
  it0.sp.W = sb.plan_W;
  it0.sp.beta = sb.plan_beta;
  it0.sp.C = sb.plan_C;

  int b, rb, t0, t1, segid, nseg;
  bool first_u;

  // Every role runs with the launch's kLaunchRegs registers.  No setmaxnreg split: a producer or
  // issuer squeezed into fewer registers spills, and with the shared-memory carve-out at its
  // maximum, L1 is too small to hold the spills, so they cost L2 round trips per stage.
  if (warp < 4) {
    if (rank == 0) {
      if (warp == 0) {
      // ---- key producer (whole warp: page lookups in warp-wide batches; lane 0 issues): a score
      // tile is up to 2 pages (128 keys); each page is streamed as two stages, one bulk copy each
      // (chunks 0-3, then chunks 4-8).  Page pg of a tile always goes to stages 2 pg and 2 pg + 1,
      // which only its MMA issuer reads, so each stage's uses are consumed in order.
      grid_dep_wait();
      SegIter it = it0;
      PageRows pr;
      uint32_t u[kKStages] = {};   // loads issued so far into each stage
      while (it.next(p, cid, b, rb, t0, t1, segid, first_u, nseg)) {
        for (int T = t0; T < t1; T += kSuper) {
          const int npg = min(kSuper, t1 - T);
          int32_t rows[kSuper];
#pragma unroll
          for (int pg = 0; pg < kSuper; ++pg) {
            int64_t row = pg < npg ? pr.get(p, b, T + pg) : 0;
            if (row < 0) {
              if (lane == 0) report(p.dev_status, MLA_ERR_BAD_INDEX);
              row = 0;
            }
            rows[pg] = (int32_t)row;
          }
          // Lane 0 streams the tile's pages, two stages per page: chunks 0-3, then chunks 4-8.
          int ok = 1;
          if (lane == 0) {
            for (int pg = 0; pg < npg && ok; ++pg) {
              sb.prog[warp] = (int)(u[0] + u[2]);
              for (int half = 0; half < 2; ++half) {
                const int s = 2 * pg + half;
                if (u[s] > 0 &&
                    !wait_or_abort(sb, bar(B_KEMPTY + s), (u[s] - 1) & 1, p.dev_status, false, p.timeout_rec, __LINE__)) {
                  ok = 0;
                  break;
                }
                const uint32_t dst = smem_u32(tiles + kKOff + s * kKStageBytes);
                const int c0 = 4 * half, nc = half_chunks(half);
                mbar_expect_tx(bar(B_KFULL + s), nc * kChunkBytes);
                if (p.tiled)   // chunks c0 .. c0+nc-1 of a page are contiguous, already in the order the MMA reads them
                  bulk_load(dst, p.tiled + (int64_t)(rows[pg] / kTileKeys) * (9 * kChunkBytes) + c0 * kChunkBytes,
                            nc * kChunkBytes, bar(B_KFULL + s));
                else
                  for (int c = 0; c < nc; ++c) {
                    if (c0 + c < 8) tma_load_2d(dst + c * kChunkBytes, &map_c, 64 * (c0 + c), rows[pg], bar(B_KFULL + s));
                    else tma_load_2d(dst + c * kChunkBytes, &map_pe, 0, rows[pg], bar(B_KFULL + s));
                  }
                ++u[s];
              }
            }
          }
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) goto prod_done0;
        }
      }
    prod_done0:
      // Drain: the last load issued on each stage must have landed before exit.
      if (lane == 0)
        for (int s = 0; s < kKStages; ++s)
          if (u[s]) mbar_wait(bar(B_KFULL + s), (u[s] - 1) & 1, kWaitNs);
      } else if ((warp == 1 || warp == 2) && lane == 0) {
      // ---- MMA issuers: S [128 x 64 per page] = Q . K^T for the tile's pages side by side, into
      // one of two tensor-memory buffers so that the next tile's MMAs overlap this tile's softmax.
      // The latent part of Q is the A operand from tensor memory; the RoPE part is in shared memory.
      // One thread issues a tcgen05.mma only every ~120 cycles whatever N is, well below the tensor
      // pipe's rate for N = 64, so each page of a tile has its own issuing thread (page 0: warp 1,
      // page 1: warp 2, on different SM sub-partitions); both commit the tile's S-full barrier.
      const int my_pg = warp - 1;
      SegIter it = it0;
      uint32_t u = 0, ns = 0, uc = 0;   // u: pages this issuer has consumed (uses of its stage pair)
      bool ok = true;
      while (ok && it.next(p, cid, b, rb, t0, t1, segid, first_u, nseg)) {
        if (!wait_or_abort(sb, bar(B_QREADY), uc & 1, p.dev_status, false, p.timeout_rec, __LINE__)) break;
        tc_fence_after();
        for (int T = t0; T < t1; T += kSuper, ++ns) {
          const int npg = min(kSuper, t1 - T);
          const uint32_t idesc = idesc_bf16_f32(kRows, kTileKeys, false, false);
          const uint32_t sbuf = ns & 1, dcol = tbase + kSCol + 128 * sbuf;
          if (ns >= 2 && !wait_or_abort(sb, bar(B_SEMPTY + sbuf), ((ns >> 1) - 1) & 1, p.dev_status, false, p.timeout_rec, __LINE__)) { ok = false; break; }
          tc_fence_after();
          // This issuer's page of the tile fills S columns 64 pg .. 64 pg + 63 (N = 64 MMAs), one
          // half-page stage at a time.
          if (my_pg < npg) {
            sb.prog[warp] = (int)u;
            for (int half = 0; half < 2; ++half) {
              const int s = 2 * my_pg + half;
              if (!wait_or_abort(sb, bar(B_KFULL + s), u & 1, p.dev_status, false, p.timeout_rec, __LINE__)) { ok = false; break; }
              tc_fence_after();
              const uint32_t kt = smem_u32(tiles + kKOff + s * kKStageBytes);
              const uint32_t dcol_pg = dcol + 64 * my_pg;
              for (int c = 0; c < half_chunks(half); ++c) {
                const int j = 4 * half + c;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                  const uint64_t bd = smem_desc_sw128(kt + c * kChunkBytes + kk * 32, 16, 1024);
                  if (j < 8)
                    mma_ts(dcol_pg, tbase + kQCol + 32 * j + 8 * kk, bd, idesc, (j | kk) ? 1u : 0u);
                  else
                    mma_ss(dcol_pg, smem_desc_sw128(smem_u32(tiles + kQpeOff) + kk * 32, 16, 1024), bd, idesc, 1u);
                }
              }
              tc_commit(bar(B_KEMPTY + s));
            }
            ++u;
          }
          if (!ok) break;
          tc_commit(bar(B_SFULL + sbuf));
        }
        ++uc;
      }
      }
    } else {
      if (warp == 0) {
      // ---- latent producer (whole warp: lookups in warp-wide batches, lane 0 issues): each page's
      // c_KV part is streamed as two half-page stages [64 keys x 256 dims], one per PV MMA group.
      grid_dep_wait();
      if (cid == 0) {
        for (int i = lane; i < kTimeoutRecInts; i += 32) p.timeout_rec[i] = 0;
        // Units with no tiles get an empty segment list (their rows combine to zero).
        for (int u = lane; u < p.U; u += 32)
          if (unit_tiles(p, u) == 0) {
            p.seg_info[2 * u] = 0;
            p.seg_info[2 * u + 1] = 0;
          }
        for (int bb = lane; bb < p.B; bb += 32) {
          const int S = p.seqlens[bb];
          if (S < p.n_q || S > p.max_seqlen) report(p.dev_status, MLA_ERR_BAD_INDEX);
        }
      }
      SegIter it = it0;
      PageRows pr;
      uint32_t n = 0;
      while (it.next(p, cid, b, rb, t0, t1, segid, first_u, nseg)) {
        if (first_u && lane == 0) {
          // This cluster holds the unit's first tile: publish where its partials live.
          p.seg_info[2 * (b * p.n_rb + rb)] = segid;
          p.seg_info[2 * (b * p.n_rb + rb) + 1] = nseg;
        }
        for (int t = t0; t < t1; ++t) {
          int64_t row = pr.get(p, b, t);
          if (row < 0) row = 0;   // reported by the score CTA
          for (int h = 0; h < 2; ++h, ++n) {
            if (lane == 0) sb.prog[warp] = (int)n;
            const int s = n % kVStages;
            if (n >= kVStages && !warp_wait(sb, bar(B_VEMPTY + s), ((n / kVStages) - 1) & 1, p.dev_status, false, p.timeout_rec, __LINE__)) goto prod_done1;
            if (lane == 0) {
              const uint32_t dst = smem_u32(tiles + s * kVStageBytes);
              mbar_expect_tx(bar(B_VFULL + s), kVStageBytes);
              if (p.tiled)   // latent chunks 4h .. 4h+3 of the page: 32 contiguous KB
                bulk_load(dst, p.tiled + (row / kTileKeys) * (9 * kChunkBytes) + h * kVStageBytes, kVStageBytes,
                          bar(B_VFULL + s));
              else
                for (int j = 0; j < 4; ++j)
                  tma_load_2d(dst + j * kChunkBytes, &map_c, 64 * (4 * h + j), (int32_t)row, bar(B_VFULL + s));
            }
          }
        }
      }
    prod_done1:
      if (lane == 0)
        for (int s = 0; s < kVStages; ++s)
          if (const uint32_t uses = n / kVStages + (s < (int)(n % kVStages) ? 1u : 0u))
            mbar_wait(bar(B_VFULL + s), (uses - 1) & 1, kWaitNs);
      } else if ((warp == 1 || warp == 3) && lane == 0) {
      // ---- MMA issuers: O += P . C.  Issuer hv (warp 1: hv = 0, warp 3: hv = 1) owns O columns
      // 256 hv .. 256 hv + 255 and reads only the page's latent half hv (stage hv of every stage
      // pair), so the two issue streams and their fix-up requests run independently.
      const int hv = warp == 1 ? 0 : 1;
      SegIter it = it0;
      uint32_t n = 0, np = 0, uc = 0, nfix = 0;
      const uint32_t idesc = idesc_bf16_f32(kRows, 256, false, true);
      bool ok = true;
      while (ok && it.next(p, cid, b, rb, t0, t1, segid, first_u, nseg)) {
        if (uc > 0 && !wait_or_abort(sb, bar(B_OFREE), (uc - 1) & 1, p.dev_status, false, p.timeout_rec, __LINE__)) break;
        const int S = seq_len_clamped(p, b);
        for (int t = t0; t < t1; ++t, n += 2, ++np) {
          sb.prog[warp] = (int)n;
          const int pb = np % kPSlots;
          const int sv = (int)((n + hv) % kVStages);
          const uint32_t pv = ((n + hv) / kVStages) & 1;
          if (!wait_or_abort(sb, bar(B_PFULL + pb), (np / kPSlots) & 1, p.dev_status, true, p.timeout_rec, __LINE__)) {
            ok = false;
            break;
          }
          const bool tail = p.kv_begin + (t + 1) * kTileKeys > S;
          const uint32_t fa = slot_factors(smem_u32(tiles), pb);
          const bool resc = t != t0 && (ld_shared_u32(fa + 4 * 32) | ld_shared_u32(fa + 4 * (kPaWords + 32)) |
                                        ld_shared_u32(fa + 4 * (2 * kPaWords + 32)) |
                                        ld_shared_u32(fa + 4 * (3 * kPaWords + 32))) != 0;
          if (!wait_or_abort(sb, bar(B_VFULL + sv), pv, p.dev_status, false, p.timeout_rec, __LINE__)) {
            ok = false;
            break;
          }
          if (tail || resc) {
            // Rare: this half's epilogue group zeroes the latent rows past the end and/or rescales
            // its O columns first.  A rescale reads O back, so the previous page's MMAs (both
            // halves: the slot's P.V barrier counts both issuers) must have completed.
            if (resc && !wait_or_abort(sb, bar(B_PVDONE + (np - 1) % kPSlots), ((np - 1) / kPSlots) & 1, p.dev_status,
                                       false, p.timeout_rec, __LINE__)) { ok = false; break; }
            sb.req[hv] = Req{0, sv, pb, S - p.kv_begin - t * kTileKeys, tail ? 1 : 0, resc ? 1 : 0, 0, 0, 0};
            mbar_arrive(bar(B_REQ + hv));
            if (!wait_or_abort(sb, bar(B_REQDONE + hv), nfix & 1, p.dev_status, false, p.timeout_rec, __LINE__)) { ok = false; break; }
            ++nfix;
          }
          tc_fence_after();
          const uint32_t pt = smem_u32(tiles + kPOff + pb * kPSlotBytes);
          const uint32_t vt = smem_u32(tiles + sv * kVStageBytes);
          // O[:, 256 hv ..] += P . C[:, 256 hv ..]: four K = 16 steps over the page's 64 keys.
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {
            const uint64_t ad = smem_desc_sw128(pt + ks * 32, 16, 1024);
            const uint64_t bd = smem_desc_sw128(vt + ks * 2048, kChunkBytes, 1024);
            mma_ss(tbase + 256 * hv, ad, bd, idesc, (t != t0 || ks > 0) ? 1u : 0u);
          }
          tc_commit(bar(B_VEMPTY + sv));
          tc_commit(bar(B_PVDONE + pb));
        }
        if (!ok) break;
        // Unit epilogue request: the epilogue group waits for the last MMAs itself.
        const uint32_t last = np - 1;
        sb.req[hv] = Req{1, 0, 0, 0, 0, 0, segid, (int)(last % kPSlots), (int)((last / kPSlots) & 1)};
        mbar_arrive(bar(B_REQ + hv));
        ++uc;
      }
      } else if (warp == 2 && lane == 0) {
      // ---- relay: a P slot is free once the MMAs that read it completed
      // Each slot's next P-full phase is armed with the bytes the score CTA will copy
      // before that CTA may copy them (at start-up, then whenever the slot frees up).
      SegIter it = it0;
      uint32_t np = 0;
      const uint32_t pempty_remote = mapa(bar(B_PEMPTY), peer);
      bool ok = true;
      while (ok && it.next(p, cid, b, rb, t0, t1, segid, first_u, nseg)) {
        for (int t = t0; t < t1; ++t, ++np) {
          sb.prog[warp] = (int)np;
          const int pb = np % kPSlots;
          if (!wait_or_abort(sb, bar(B_PVDONE + pb), (np / kPSlots) & 1, p.dev_status, false, p.timeout_rec, __LINE__)) {
            ok = false;
            break;
          }
          mbar_expect_tx(bar(B_PFULL + pb), kPTxBytes);
          mbar_arrive_cluster(pempty_remote + 8 * pb);
        }
      }
      }
    }
  } else {
    if (rank == 0) {
      // ---- softmax: 8 warps; warp (quadrant q, half h) owns rows 32q..32q+31 (its TMEM lanes)
      // and page h (score columns 64h..64h+63) of each two-page score tile.
      const int q4 = warp & 3, h = (warp - 4) >> 2;
      const int r = q4 * 32 + lane;
      const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
      grid_dep_wait();
      SegIter it = it0;
      uint32_t ns = 0, np = 0, uc = 0;
      const uint32_t pbuf_remote = mapa(smem_u32(tiles + kPOff), peer);
      // Staging of this half's P page (all four lane quadrants) and of its rescale factors.
      unsigned char *stgp = tiles + kStgOff + h * kPSlotBytes;
      unsigned char *stga = stgp + kPBytes;
      const uint32_t statl_remote = mapa(smem_u32(&sb.stat_l[0]), peer);
      const uint32_t statm_remote = mapa(smem_u32(&sb.stat_m[0]), peer);
      const uint32_t pfull_remote = mapa(bar(B_PFULL), peer);
      const uint32_t statsfull_remote = mapa(bar(B_STATSFULL), peer);
      const int nrows = p.n_q * p.H;
      // No early exit in this region: the eight warps meet at named barriers, so on a timeout they
      // keep walking the same (now wait-free: every wait returns at once) loop to the end.
      while (it.next(p, cid, b, rb, t0, t1, segid, first_u, nseg)) {
        // Q rows -> half h loads latent dims 256h..256h+255 of its warp's 32 rows into TMEM columns
        // 128h..; half 0 also puts the RoPE dims into the shared [128 x 64] A tile.  The previous
        // unit's MMAs are complete (its last S was consumed), so both may be overwritten.  The loads
        // are coalesced (eight lanes per 128-byte row segment) and pass through the warp's 4 KB of
        // the half's P staging tile, 128-byte swizzled, from which each thread reads its own row for
        // the tensor-memory store; the last P copy out of that tile must have read it first.
        const int gr = rb * kRows + r;
        const bool real = gr < nrows;
        {
          if (q4 == 0 && lane == 0) bulk_wait_read_all();
          asm volatile("bar.sync %0, 128;" ::"r"(2 + h) : "memory");
          unsigned char *stg_w = stgp + q4 * 4096;
          const int j = lane & 7;
          const uint4 *rowp[8];
          bool live[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const int g = rb * kRows + q4 * 32 + 4 * k + (lane >> 3);
            live[k] = g < nrows;
            rowp[k] = reinterpret_cast<const uint4 *>(p.q + ((int64_t)b * nrows + (live[k] ? g : 0)) * kW);
          }
#pragma unroll 1
          for (int cb = 0; cb < 4; cb += 2) {
            uint4 x[2][8];
#pragma unroll
            for (int rr = 0; rr < 2; ++rr)
#pragma unroll
              for (int k = 0; k < 8; ++k)
                x[rr][k] = live[k] ? __ldg(rowp[k] + h * 32 + (cb + rr) * 8 + j) : make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) {
#pragma unroll
              for (int k = 0; k < 8; ++k) {
                const int lr = 4 * k + (lane >> 3);
                *reinterpret_cast<uint4 *>(stg_w + (lr >> 3) * 1024 + (lr & 7) * 128 + ((j ^ (lr & 7)) << 4)) = x[rr][k];
              }
              __syncwarp();
              uint32_t v[32];
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const uint4 y = *reinterpret_cast<const uint4 *>(stg_w + (lane >> 3) * 1024 + (lane & 7) * 128 + ((i ^ (lane & 7)) << 4));
                v[4 * i] = y.x; v[4 * i + 1] = y.y; v[4 * i + 2] = y.z; v[4 * i + 3] = y.w;
              }
              tmem_st32(tbase + lane_off + kQCol + 128 * h + 32 * (cb + rr), v);
              __syncwarp();
            }
          }
          if (h == 0) {
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const int rq = q4 * 32 + 4 * k + (lane >> 3);
              *reinterpret_cast<uint4 *>(tiles + kQpeOff + (rq >> 3) * 1024 + (rq & 7) * 128 + ((j ^ (rq & 7)) << 4)) =
                  live[k] ? __ldg(rowp[k] + 64 + j) : make_uint4(0, 0, 0, 0);
            }
            fence_proxy_async_smem();
          }
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(B_QREADY));
        }
        const int S = seq_len_clamped(p, b);
        const int j = real ? gr / p.H : 0;
        // Keys this row may see, counted from the key range's first key.
        const int vis_end = (real ? min(S - p.n_q + j + 1, p.kv_end) : 0) - p.kv_begin;
        float m_ref = -CUDART_INF_F, l = 0.f;
        for (int T = t0; T < t1; T += kSuper, ++ns) {
          if (lane == 0) sb.prog[warp] = (int)np;
          const int npg = min(kSuper, t1 - T);
          const uint32_t sbuf = ns & 1;
          warp_wait(sb, bar(B_SFULL + sbuf), (ns >> 1) & 1, p.dev_status, false, p.timeout_rec, __LINE__);
          tc_fence_after();
          // My page of the tile is page h: keys 64T + 64h + k, k < 64.  Its scores are read from
          // tensor memory twice, 32 columns at a time (for the maximum, then for P), so that at most
          // 32 of them are live in registers; the buffer is released after the last read.
          const uint32_t scol = tbase + lane_off + kSCol + 128 * sbuf + 64 * h;
          auto release_s = [&]() {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_SEMPTY + sbuf));
          };
          // Valid while below the row's causal limit and inside the pages this tile holds.
          const int nvalid = min(vis_end - (T + h) * kTileKeys, (npg - h) * kTileKeys);
          // Only a sequence's last page has keys past some row's limit: warps whose rows all see
          // the whole page skip the per-key mask.
          const bool whole = __all_sync(0xffffffffu, nvalid >= kTileKeys);
          float mx = -CUDART_INF_F;
#pragma unroll 1
          for (int c2 = 0; c2 < 2; ++c2) {
            uint32_t v[32];
            tmem_ld32(scol + 32 * c2, v);
            tmem_wait_ld();
            if (whole) {
#pragma unroll
              for (int k = 0; k < 32; k += 2) mx = max3f(mx, __uint_as_float(v[k]), __uint_as_float(v[k + 1]));
            } else {
#pragma unroll
              for (int k = 0; k < 32; ++k)   // a select, not a branch: nvalid differs between rows
                mx = fmaxf(mx, 32 * c2 + k < nvalid ? __uint_as_float(v[k]) : -CUDART_INF_F);
            }
          }
          // The scale is positive: the scaled maximum is the maximum of the scaled scores.
          mx *= p.scale_log2;
          if (h >= npg) release_s();   // no page here: nothing more to read
          sb.xmax[ns & 1][h][r] = mx;
          asm volatile("bar.sync 1, 256;" ::: "memory");
          mx = fmaxf(mx, sb.xmax[ns & 1][h ^ 1][r]);
          float alpha = 1.f;
          const bool need = mx > m_ref + kRescaleLog2;
          if (need) {
            alpha = exp2f(m_ref - mx);
            l *= alpha;
            m_ref = mx;
          }
          if (h < npg) {
            const uint32_t pn = np + h;
            const int pb = pn % kPSlots;
            const bool issuer = q4 == 0 && lane == 0;   // sends the half's page for all four warps
            // The page's staging buffer is free once the previous copies out of it have read it.
            if (issuer) bulk_wait_read_all();
            asm volatile("bar.sync %0, 128;" ::"r"(2 + h) : "memory");
            // My 32 P rows, K-major and 128B-swizzled like the value CTA's [128 x 64] P tile (rows
            // 32q..32q+31 are its bytes 4096q..4096q+4095), then the rows' rescale factors (the first
            // page of a score tile carries the tile's factors) and the warp's flag word.
            unsigned char *prow = stgp + 4096 * q4 + (lane >> 3) * 1024 + (lane & 7) * 128;
            float psum0 = 0.f, psum1 = 0.f;   // the row sum, from P before its rounding to bf16
#pragma unroll 1
            for (int c2 = 0; c2 < 2; ++c2) {
              uint32_t v[32];
              tmem_ld32(scol + 32 * c2, v);
              tmem_wait_ld();
              if (c2 == 1) release_s();
              // Keys past the row's limit get exponent -inf: exp2 gives exactly 0, without a branch.
              auto p_half = [&](auto masked) {
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                  uint32_t pk[4];
#pragma unroll
                  for (int e = 0; e < 4; ++e) {
                    const int k = 8 * c + 2 * e, kk = 32 * c2 + k;
                    float x0 = __uint_as_float(v[k]) * p.scale_log2 - m_ref;
                    float x1 = __uint_as_float(v[k + 1]) * p.scale_log2 - m_ref;
                    if (decltype(masked)::value) {
                      x0 = kk < nvalid ? x0 : -CUDART_INF_F;
                      x1 = kk + 1 < nvalid ? x1 : -CUDART_INF_F;
                    }
                    const float p0 = exp2f(x0), p1 = exp2f(x1);
                    pk[e] = pack_bf16x2(p0, p1);
                    psum0 += p0;
                    psum1 += p1;
                  }
                  *reinterpret_cast<uint4 *>(prow + (((4 * c2 + c) ^ (lane & 7)) << 4)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                }
              };
              if (whole) p_half(std::false_type{});
              else p_half(std::true_type{});
            }
            l += psum0 + psum1;
            float *pa = reinterpret_cast<float *>(stga) + q4 * kPaWords;
            pa[lane] = h == 0 ? alpha : 1.f;
            const unsigned moved = __ballot_sync(0xffffffffu, need && h == 0 && T != t0);
            if (lane < 4) reinterpret_cast<uint32_t *>(pa + 32)[lane] = (lane == 0 && moved) ? 1u : 0u;
            fence_proxy_async_smem();
            asm volatile("bar.sync %0, 128;" ::"r"(2 + h) : "memory");
            // Into the value CTA's slot once the MMAs that read its previous contents completed: two
            // bulk copies (the page, its factors) that complete on the slot's P-full barrier.
            if (issuer && (pn < kPSlots || wait_or_abort(sb, bar(B_PEMPTY + pb), ((pn / kPSlots) - 1) & 1, p.dev_status,
                                                         true, p.timeout_rec, __LINE__))) {
              const uint32_t pfull = pfull_remote + 8 * pb;
              bulk_copy_to_peer(pbuf_remote + pb * kPSlotBytes, smem_u32(stgp), kPTxBytes, pfull);
              bulk_commit();
            }
          }
          np += npg;
        }
        // Unit statistics: combine the halves' row sums, then send them to the value CTA.
        sb.xl[h][r] = l;
        asm volatile("bar.sync 1, 256;" ::: "memory");
        if (h == 0) {
          l += sb.xl[1][r];
          if (uc > 0) warp_wait(sb, bar(B_STATSEMPTY), (uc - 1) & 1, p.dev_status, true, p.timeout_rec, __LINE__);
          st_cluster_f32(statl_remote + r * 4, l);
          st_cluster_f32(statm_remote + r * 4, m_ref);
          mbar_arrive_cluster(statsfull_remote);
        }
        asm volatile("bar.sync 1, 256;" ::: "memory");   // xl may be reused by the next unit
        ++uc;
      }
      if (lane == 0) bulk_wait_all();   // the staged copies have landed before this CTA may exit
    } else {
      // ---- epilogue warps, two groups of four: group g (warps 4 + 4g .. 7 + 4g) serves the MMA
      // issuer of O half g (columns 256 g .. 256 g + 255): tile fix-ups on request, then each
      // unit's epilogue for those columns.  Warp w owns rows (TMEM lanes) 32 (w & 3) ...
      const int g = (warp - 4) >> 2;
      const int r = (warp & 3) * 32 + lane;
      const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
      const uint32_t ocol = 256 * g;
      grid_dep_wait();
      SegIter it = it0;
      uint32_t nreq = 0, uc = 0;
      const uint32_t statsempty_remote = mapa(bar(B_STATSEMPTY), peer);
      bool ok = true;
      while (ok && it.next(p, cid, b, rb, t0, t1, segid, first_u, nseg)) {
        for (;;) {
          if (lane == 0) sb.prog[warp] = (int)nreq;
          if (!warp_wait(sb, bar(B_REQ + g), nreq & 1, p.dev_status, false, p.timeout_rec, __LINE__)) { ok = false; break; }
          ++nreq;
          const Req q = sb.req[g];
          if (q.kind == 0) {
            if (q.tail) {
              // Rows past the sequence end may hold anything (NaN): zero them in this half's latent
              // stage so that 0 * row stays 0.
              const int nrow = kTileKeys - q.nvalid;
              unsigned char *vt = tiles + q.vstage * kVStageBytes;
              for (int e = r; e < nrow * 32; e += kRows) {
                const int row = q.nvalid + e / 32, rest = e % 32, ch = rest / 8, piece = rest % 8;
                *reinterpret_cast<uint4 *>(vt + ch * kChunkBytes + row * 128 + piece * 16) = make_uint4(0, 0, 0, 0);
              }
              fence_proxy_async_smem();
            }
            if (q.rescale) {
              tc_fence_after();
              const float a = __uint_as_float(ld_shared_u32(slot_factors(smem_u32(tiles), q.slot) +
                                                            4 * ((r >> 5) * kPaWords + (r & 31))));
#pragma unroll 1
              for (int c = 0; c < 8; ++c) {
                uint32_t v[32];
                tmem_ld32(tbase + lane_off + ocol + 32 * c, v);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * a);
                tmem_st32(tbase + lane_off + ocol + 32 * c, v);
              }
              tmem_wait_st();
              tc_fence_before();
            }
            mbar_arrive(bar(B_REQDONE + g));
            continue;
          }
          // Unit epilogue: the unit's last MMAs and the row statistics.
          if (!warp_wait(sb, bar(B_PVDONE + q.last_slot), q.last_parity, p.dev_status, false, p.timeout_rec, __LINE__) ||
              !warp_wait(sb, bar(B_STATSFULL), uc & 1, p.dev_status, true, p.timeout_rec, __LINE__)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const float l = sb.stat_l[r], m = sb.stat_m[r];
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(statsempty_remote);
          const float inv = l > 0.f ? 1.f / l : 0.f;
          __nv_bfloat16 *dst = p.o_part + ((int64_t)q.segid * kRows + r) * kDc + ocol;
#pragma unroll 1
          for (int c = 0; c < 8; ++c) {
            uint32_t v[32];
            tmem_ld32(tbase + lane_off + ocol + 32 * c, v);
            tmem_wait_ld();
            // 32-byte stores: the row's 64 bytes leave in two whole sectors (rows are 1 KB apart, the
            // O halves start at 512 bytes, so every store is 32-byte aligned).
#pragma unroll
            for (int i = 0; i < 32; i += 16) {
              const uint4 lo = make_uint4(pack_bf16x2(__uint_as_float(v[i]) * inv, __uint_as_float(v[i + 1]) * inv),
                                          pack_bf16x2(__uint_as_float(v[i + 2]) * inv, __uint_as_float(v[i + 3]) * inv),
                                          pack_bf16x2(__uint_as_float(v[i + 4]) * inv, __uint_as_float(v[i + 5]) * inv),
                                          pack_bf16x2(__uint_as_float(v[i + 6]) * inv, __uint_as_float(v[i + 7]) * inv));
              const uint4 hi = make_uint4(pack_bf16x2(__uint_as_float(v[i + 8]) * inv, __uint_as_float(v[i + 9]) * inv),
                                          pack_bf16x2(__uint_as_float(v[i + 10]) * inv, __uint_as_float(v[i + 11]) * inv),
                                          pack_bf16x2(__uint_as_float(v[i + 12]) * inv, __uint_as_float(v[i + 13]) * inv),
                                          pack_bf16x2(__uint_as_float(v[i + 14]) * inv, __uint_as_float(v[i + 15]) * inv));
              st_global_v8(dst + 32 * c + i, lo, hi);
            }
          }
          if (g == 0) p.lse_part[(int64_t)q.segid * kRows + r] = l > 0.f ? (m + __log2f(l)) * 0.69314718055994531f : -CUDART_INF_F;
          tc_fence_before();
          mbar_arrive(bar(B_OFREE));
          ++uc;
          break;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 3) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
  cluster_sync();   // no CTA leaves while its peer may still touch its shared memory
}

// ------------------------------------------------------------ merge of the split partials
// One warp merges the ns pieces of one (query row, head) by their log-sum-exps: piece k is the bf16
// row part[k * part_stride][0 .. 512) with log-sum-exp lse[k * lse_stride].  It writes the merged
// row (bf16) and, if lse_dst is non-null, the log of the summed exp (-inf, with a zero row, where no
// piece saw a key).  Each lane owns 16 latent columns (8 in each half of the row), and the loads of
// up to kMergeUnroll pieces are in flight together, so a row cut into a few pieces costs one round
// of loads.
constexpr int kMergeThreads = 256;
constexpr int kMergeUnroll = 4;
constexpr int kMaxSegPerUnit = kMaxClusters + 1;

__device__ __forceinline__ void merge_row(int lane, int ns, const __nv_bfloat16 *part, int64_t part_stride,
                                          const float *lse, int64_t lse_stride, __nv_bfloat16 *dst,
                                          float *lse_dst) {
  float m = -CUDART_INF_F;
  for (int k = lane; k < ns; k += 32) m = fmaxf(m, lse[(int64_t)k * lse_stride]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  float sum = 0.f;
  if (m != -CUDART_INF_F)
    for (int k = lane; k < ns; k += 32) sum += __expf(lse[(int64_t)k * lse_stride] - m);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  const float inv = sum > 0.f ? 1.f / sum : 0.f;
  float v[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) v[e] = 0.f;
  for (int k0 = 0; k0 < ns; k0 += kMergeUnroll) {
    uint4 x[kMergeUnroll][2];
    float wk[kMergeUnroll];
#pragma unroll
    for (int i = 0; i < kMergeUnroll; ++i) {
      const int k = k0 + i;
      const bool have = k < ns;
      const __nv_bfloat16 *src = part + (int64_t)(have ? k : 0) * part_stride + 8 * lane;
      x[i][0] = have ? *reinterpret_cast<const uint4 *>(src) : make_uint4(0, 0, 0, 0);
      x[i][1] = have ? *reinterpret_cast<const uint4 *>(src + 256) : make_uint4(0, 0, 0, 0);
      wk[i] = have && m != -CUDART_INF_F ? __expf(lse[(int64_t)k * lse_stride] - m) * inv : 0.f;
    }
#pragma unroll
    for (int i = 0; i < kMergeUnroll; ++i)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const __nv_bfloat162 *xh = reinterpret_cast<const __nv_bfloat162 *>(&x[i][hh]);
#pragma unroll
        for (int e2 = 0; e2 < 4; ++e2) {
          const float2 f = __bfloat1622float2(xh[e2]);
          v[8 * hh + 2 * e2] = fmaf(wk[i], f.x, v[8 * hh + 2 * e2]);
          v[8 * hh + 2 * e2 + 1] = fmaf(wk[i], f.y, v[8 * hh + 2 * e2 + 1]);
        }
      }
  }
  dst += 8 * lane;
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    uint4 packed;
    __nv_bfloat162 *ph = reinterpret_cast<__nv_bfloat162 *>(&packed);
#pragma unroll
    for (int e2 = 0; e2 < 4; ++e2) ph[e2] = __floats2bfloat162_rn(v[8 * hh + 2 * e2], v[8 * hh + 2 * e2 + 1]);
    *reinterpret_cast<uint4 *>(dst + 256 * hh) = packed;
  }
  if (lane == 0 && lse_dst) *lse_dst = sum > 0.f ? m + logf(sum) : -CUDART_INF_F;
}

// One warp per (query row g = (b, j), head s): the pieces of g's unit, listed by the attention
// kernel's segment table, merged into o_lat[g][s] and lse_out[g][s].
__global__ void __launch_bounds__(kMergeThreads)
tc_merge_kernel(int B, int n_q, int H, int n_rb, int max_segs, const int *seg_info, const __nv_bfloat16 *o_part,
                const float *lse_part, __nv_bfloat16 *o_lat, float *lse_out) {
  sm100::grid_dep_launch();
  sm100::grid_dep_wait();   // the partials and the segment table come from the attention kernel
  const int lane = threadIdx.x & 31;
  const int64_t item = (int64_t)blockIdx.x * (kMergeThreads / 32) + (threadIdx.x >> 5);
  if (item >= (int64_t)B * n_q * H) return;
  const int g = (int)(item / H), s = (int)(item % H);
  const int b = g / n_q, j = g % n_q;
  const int gr = j * H + s;
  const int u = b * n_rb + gr / kRows, lr = gr % kRows;
  int s0 = seg_info[2 * u], ns = seg_info[2 * u + 1];
  ns = ns < 0 ? 0 : (ns > kMaxSegPerUnit ? kMaxSegPerUnit : ns);
  if (s0 < 0 || s0 + ns > max_segs) {
    s0 = 0;
    ns = 0;
  }
  merge_row(lane, ns, o_part + ((int64_t)s0 * kRows + lr) * kDc, (int64_t)kRows * kDc,
            lse_part + (int64_t)s0 * kRows + lr, kRows, o_lat + item * kDc, lse_out ? lse_out + item : nullptr);
}

// One warp per row r = ((b, j), s) of n_parts stacked partials (one per key range, e.g. gathered
// from the devices that each decoded one range): o_parts [n_parts][rows][512], lse_parts
// [n_parts][rows], merged into o_lat[r] and lse_out[r].
__global__ void __launch_bounds__(kMergeThreads)
parts_merge_kernel(int64_t rows, int n_parts, const __nv_bfloat16 *o_parts, const float *lse_parts,
                   __nv_bfloat16 *o_lat, float *lse_out) {
  sm100::grid_dep_launch();
  sm100::grid_dep_wait();
  const int lane = threadIdx.x & 31;
  const int64_t r = (int64_t)blockIdx.x * (kMergeThreads / 32) + (threadIdx.x >> 5);
  if (r >= rows) return;
  merge_row(lane, n_parts, o_parts + r * kDc, rows * kDc, lse_parts + r, rows, o_lat + r * kDc,
            lse_out ? lse_out + r : nullptr);
}

// ------------------------------------------------------------ merge + W_UV product
// Where the pieces of output row (g, s) live: the attention kernel's per-unit segment list
// (seg_info != NULL: piece k is row (s0 + k) * 128 + lr of the segment partials), or n_parts stacked
// partials (piece k is row k * rows * H + g * H + s).
struct Pieces {
  const __nv_bfloat16 *part;   // rows of 512 bf16
  const float *lse;            // one log-sum-exp per row of `part`
  const int *seg_info;         // [units][2], or NULL for stacked partials
  int n_q, H, n_rb, max_segs, n_parts;
};

// Number of pieces of row (g, s) and the index of its first piece row; pieces are `stride` rows apart.
__device__ __forceinline__ int piece_rows(const Pieces &pc, int rows, int g, int s, int64_t &first, int64_t &stride) {
  if (!pc.seg_info) {
    first = (int64_t)g * pc.H + s;
    stride = (int64_t)rows * pc.H;
    return pc.n_parts;
  }
  const int b = g / pc.n_q, j = g % pc.n_q;
  const int gr = j * pc.H + s;
  const int u = b * pc.n_rb + gr / kRows;
  int s0 = pc.seg_info[2 * u], ns = pc.seg_info[2 * u + 1];
  ns = ns < 0 ? 0 : (ns > kMaxSegPerUnit ? kMaxSegPerUnit : ns);
  if (s0 < 0 || s0 + ns > pc.max_segs) return 0;
  first = (int64_t)s0 * kRows + gr % kRows;
  stride = kRows;
  return ns;
}

// CTA = (head s, 64 query rows (b, j)): the rows' pieces are merged by their log-sum-exps straight
// into the B operand tile of the W_UV product (o_lat [64 rows x 512], K-major, 128-byte swizzled,
// bf16), then out^T [d_v x 64] = W_UV^(s)T . o_lat^T on the tensor cores, with W_UV supplying the
// 128-row M side (A = W_UV^T, M-major; fp32 accumulator in 64 tensor-memory columns).  All of
// W_UV[s] (128 KB) is requested by TMA before the kernel waits for the attention kernel, so its
// transfer overlaps that kernel's tail.  The merge runs on all 256 threads at once: four threads
// per row, each owning 16 of the row's 64 16-byte column blocks (blocks 4 i + q), so that the four
// threads of a row read 64 contiguous bytes per load.
constexpr int kCombRows = 64;
constexpr int kCombThreads = 256;
constexpr int kDv = 128;                                   // the W_UV tile width this kernel takes
constexpr uint32_t kOlBytes = kCombRows * kDc * 2;         // o_lat: [8 K-chunks][64 rows][128 B]
constexpr uint32_t kWuvBytes = kDc * kDv * 2;              // W_UV^T: [8 K-chunks][2 M-chunks][64 K rows][128 B]
static_assert(kCombThreads == 4 * kCombRows, "four merging threads per row");

__global__ void __launch_bounds__(kCombThreads)
tc_combine_kernel(const __grid_constant__ CUtensorMap map_w, const Pieces pc, int rows, float *lse_out,
                  __nv_bfloat16 *out, int *dev_status) {
  extern __shared__ unsigned char csm_raw[];
  unsigned char *csm = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(csm_raw) + 1023) & ~uintptr_t(1023));
  unsigned char *ol = csm;                                                          // o_lat, K-major, swizzled
  unsigned char *wa = csm + kOlBytes;                                               // W_UV^T, M-major, swizzled
  __shared__ __align__(8) uint64_t bar_w, bar_mma;
  __shared__ uint32_t tmem_slot;
  __shared__ int s_loaded;
  const int s = blockIdx.x, H = pc.H;
  const int g0 = blockIdx.y * kCombRows;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  sm100::grid_dep_launch();
  // W_UV[s] (an input: no need to wait), as 16 TMA boxes of [64 K rows x 64 output columns] in the
  // MMA's M-major, 128-byte-swizzled layout: box (K-chunk kc, M-chunk mc) at (kc * 2 + mc) * 8 KB.
  if (tid == 0) {
    mbar_init(smem_u32(&bar_w), 1);
    mbar_init(smem_u32(&bar_mma), 1);
    fence_mbar_init();
    tma_prefetch_desc(&map_w);
    mbar_expect_tx(smem_u32(&bar_w), kWuvBytes);
    for (int kc = 0; kc < kDc / 64; ++kc)
      for (int mc = 0; mc < 2; ++mc)
        tma_load_2d(smem_u32(wa + (kc * 2 + mc) * 8192), &map_w, 64 * mc, s * kDc + 64 * kc, smem_u32(&bar_w));
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(&tmem_slot), kCombRows);
    tmem_relinquish();
  }
  sm100::grid_dep_wait();   // the partials and the segment list come from the attention kernel
  {
    // Merge of row rr (output row g = g0 + rr); rows past the end become zero rows of the tile.
    const int rr = tid >> 2, q = tid & 3, g = g0 + rr;
    int64_t first = 0, stride = 0;
    const int ns = g < rows ? piece_rows(pc, rows, g, s, first, stride) : 0;
    float m = -CUDART_INF_F;
    for (int k = 0; k < ns; ++k) m = fmaxf(m, pc.lse[first + k * stride]);
    float sum = 0.f;
    if (m != -CUDART_INF_F)
      for (int k = 0; k < ns; ++k) sum += __expf(pc.lse[first + k * stride] - m);
    const float inv = sum > 0.f ? 1.f / sum : 0.f;
#pragma unroll 1
    for (int hh = 0; hh < 2; ++hh) {
      // this round: column blocks cb = 4 (8 hh + i) + q, i < 8 (8 bf16 each)
      float acc[8][8];
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[i][e] = 0.f;
      for (int k0 = 0; k0 < ns; k0 += 2) {
        uint4 x[2][8];
        float wk[2];
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
          const bool have = k0 + kk < ns;
          const __nv_bfloat16 *src = pc.part + (first + (int64_t)(have ? k0 + kk : 0) * stride) * kDc;
#pragma unroll
          for (int i = 0; i < 8; ++i)
            x[kk][i] = have ? *reinterpret_cast<const uint4 *>(src + 8 * (4 * (8 * hh + i) + q)) : make_uint4(0, 0, 0, 0);
          wk[kk] = have && m != -CUDART_INF_F ? __expf(pc.lse[first + (int64_t)(k0 + kk) * stride] - m) * inv : 0.f;
        }
#pragma unroll
        for (int kk = 0; kk < 2; ++kk)
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const __nv_bfloat162 *xh = reinterpret_cast<const __nv_bfloat162 *>(&x[kk][i]);
#pragma unroll
            for (int e2 = 0; e2 < 4; ++e2) {
              const float2 f = __bfloat1622float2(xh[e2]);
              acc[i][2 * e2] = fmaf(wk[kk], f.x, acc[i][2 * e2]);
              acc[i][2 * e2 + 1] = fmaf(wk[kk], f.y, acc[i][2 * e2 + 1]);
            }
          }
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int cb = 4 * (8 * hh + i) + q, kc = cb >> 3, jj = cb & 7;
        uint4 packed;
        packed.x = pack_bf16x2(acc[i][0], acc[i][1]);
        packed.y = pack_bf16x2(acc[i][2], acc[i][3]);
        packed.z = pack_bf16x2(acc[i][4], acc[i][5]);
        packed.w = pack_bf16x2(acc[i][6], acc[i][7]);
        *reinterpret_cast<uint4 *>(ol + kc * 8192 + (rr >> 3) * 1024 + (rr & 7) * 128 + ((jj ^ (rr & 7)) << 4)) = packed;
      }
    }
    if (q == 0 && lse_out && g < rows) lse_out[(int64_t)g * H + s] = sum > 0.f ? m + logf(sum) : -CUDART_INF_F;
    fence_proxy_async_smem();   // the merged tile is read by the MMA (async proxy)
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  int loaded = 1;
  if (tid == 0) {
    if (!mbar_wait(smem_u32(&bar_w), 0, kWaitNs)) {
      report(dev_status, MLA_ERR_TIMEOUT);
      loaded = 0;
    }
    s_loaded = loaded;
  }
  // Without its operands the MMA is skipped; its barrier is still completed (commit with nothing issued).
  if (tid == 0) {
    tc_fence_after();
    const uint32_t idesc = idesc_bf16_f32(128, kCombRows, true, false);
    for (int kc = 0; kc < kDc / 64 && loaded; ++kc)
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_ss(tmem, smem_desc_sw128(smem_u32(wa + kc * 16384) + kk * 2048, 8192, 1024),
               smem_desc_sw128(smem_u32(ol + kc * 8192) + kk * 32, 16, 1024), idesc, (kc | kk) ? 1u : 0u);
    tc_commit(smem_u32(&bar_mma));
  }
  int ok = 1;
  if (lane == 0 && !mbar_wait(smem_u32(&bar_mma), 0, kWaitNs)) {
    report(dev_status, MLA_ERR_TIMEOUT);
    ok = 0;
  }
  ok = __shfl_sync(0xffffffffu, ok, 0);
  if (ok) mbar_wait(smem_u32(&bar_mma), 0, kWaitNs);
  tc_fence_after();
  // Warp w drains output columns 32(w%4).. (its lane quadrant) for query rows 32(w/4)..: each thread
  // holds one output column of 32 rows -> a [64 rows x 128] bf16 staging tile over o_lat's space.
  __nv_bfloat16 *stg = reinterpret_cast<__nv_bfloat16 *>(ol);
  constexpr int lds = kDv + 8;
  {
    uint32_t v[32];
    tmem_ld32(tmem + ((uint32_t)((warp & 3) * 32) << 16) + 32 * (warp >> 2), v);
    tmem_wait_ld();
    __syncthreads();   // every thread is past its reads of o_lat (the MMAs completed before the loads)
    ok = ok && s_loaded;
#pragma unroll
    for (int i = 0; i < 32; ++i)
      stg[(32 * (warp >> 2) + i) * lds + (warp & 3) * 32 + lane] = __float2bfloat16_rn(__uint_as_float(v[i]));
  }
  tc_fence_before();
  __syncthreads();
  if (ok)
    for (int c = tid; c < kCombRows * (kDv / 8); c += kCombThreads) {
      const int rr = c >> 4, q8 = c & 15, g = g0 + rr;
      if (g < rows)
        *reinterpret_cast<uint4 *>(out + ((int64_t)g * H + s) * kDv + q8 * 8) =
            *reinterpret_cast<const uint4 *>(stg + rr * lds + q8 * 8);
    }
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kCombRows);
  }
  if (tid == 0 && !loaded)   // the copies must have landed before this CTA's shared memory goes away
    mbar_wait(smem_u32(&bar_w), 0, kWaitNs);
}

// ------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

int make_map(CUtensorMap *m, const void *base, uint64_t inner, uint64_t rows, uint64_t row_bytes) {
  auto fn = encode_fn();
  if (!fn) return MLA_ERR_CUDA;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {64, 64};
  cuuint32_t es[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MLA_OK : MLA_ERR_CUDA;
}

struct WsLayout {
  size_t seg_info, o_part, lse_part, total;
};

int clusters_for_device();

// Partials: one per (unit, cluster) piece, at most U + C - 1 pieces for C clusters.
WsLayout ws_layout(int B, int n_rb) {
  auto a256 = [](size_t x) { return (x + 255) & ~size_t(255); };
  const size_t U = (size_t)B * n_rb;
  const int C = clusters_for_device();
  const size_t segs = U + (C > 0 ? C : kMaxClusters);
  WsLayout L;
  L.seg_info = 0;
  L.o_part = a256(U * 2 * sizeof(int) + kTimeoutRecInts * sizeof(int));
  L.lse_part = L.o_part + a256(segs * kRows * kDc * sizeof(__nv_bfloat16));
  L.total = L.lse_part + a256(segs * kRows * sizeof(float));
  return L;
}

// Clusters of two CTAs that fit on the current device at once (0 without a device).  The
// answer is cached per device; the first query on a device computes it under a mutex, so
// concurrent first calls from several host threads are safe.
int clusters_for_device() {
  static std::atomic<int> cached[128];
  static std::mutex mu;
  int dev = 0, ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || ndev <= 0) {
    cudaGetLastError();
    return 0;
  }
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return 0;
  if (const int c = cached[dev].load(std::memory_order_acquire)) return c;
  std::lock_guard<std::mutex> lock(mu);
  if (const int c = cached[dev].load(std::memory_order_acquire)) return c;
  if (cudaFuncSetAttribute(mla_decode_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes))
    return 0;
  // One CTA of kThreads per SM needs at most kLaunchRegs registers per thread.
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, mla_decode_tc_kernel) != cudaSuccess || fa.numRegs > kLaunchRegs) return 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * kMaxClusters);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, mla_decode_tc_kernel, &cfg) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    int sms = 0;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    n = sms / 2;
  }
  if (n > kMaxClusters) n = kMaxClusters;
  cached[dev].store(n, std::memory_order_release);
  return n;
}

}  // namespace

bool tc_decode_supported(const mla_dims &d, int n_q) {
  const bool layout_ok = d.cache_layout == MLA_CACHE_TILED || (d.ckv_stride % 8 == 0 && d.kpe_stride % 8 == 0);
  return d.dtype == MLA_BF16 && d.d_c == kDc && d.d_rope == kDr && d.block_size % kTileKeys == 0 && layout_ok &&
         d.d_v == 128 && n_q * d.n_heads <= 2 * kRows;
}

int tc_decode_kernel_launches() { return 2; }   // attention; merge (+ W_UV product)

size_t tc_decode_workspace_bytes(const mla_dims &d, int B, int n_q) {
  const int n_rb = (n_q * d.n_heads + kRows - 1) / kRows;
  return ws_layout(B, n_rb).total;
}

int launch_tc_attention(const mla_dims &d, int B, int n_q, const void *q_abs, const CacheView &cache,
                        const int32_t *seqlens, int max_seqlen, void *ws, int *dev_status, cudaStream_t st,
                        int kv_begin, int kv_end) {
  if (kv_begin < 0 || kv_begin % kTileKeys) return MLA_ERR_INVALID_ARG;
  const bool tiled = cache.layout == MLA_CACHE_TILED;
  if ((reinterpret_cast<uintptr_t>(cache.c_kv) & 15) || (!tiled && (reinterpret_cast<uintptr_t>(cache.k_pe) & 15)) ||
      (reinterpret_cast<uintptr_t>(q_abs) & 15))
    return MLA_ERR_INVALID_ARG;
  const int n_rb = (n_q * d.n_heads + kRows - 1) / kRows;
  const WsLayout L = ws_layout(B, n_rb);
  char *w = static_cast<char *>(ws);
  CUtensorMap mc, mpe;
  memset(&mc, 0, sizeof(mc));
  memset(&mpe, 0, sizeof(mpe));
  if (!tiled) {   // row pool: 2-D TMA boxes of [64 rows x 64 dims]
    const uint64_t rows = (uint64_t)cache.num_blocks * cache.block_size;
    int rc = make_map(&mc, cache.c_kv, kDc, rows, (uint64_t)cache.ckv_stride * 2);
    if (rc) return rc;
    if ((rc = make_map(&mpe, cache.k_pe, kDr, rows, (uint64_t)cache.kpe_stride * 2))) return rc;
  }
  const int C = clusters_for_device();
  if (C <= 0) return MLA_ERR_CUDA;
  TcParams p;
  p.B = B;
  p.n_q = n_q;
  p.H = d.n_heads;
  p.n_rb = n_rb;
  p.U = B * n_rb;
  p.max_seqlen = max_seqlen;
  p.q = static_cast<const __nv_bfloat16 *>(q_abs);
  p.seqlens = seqlens;
  p.block_table = cache.block_table;
  p.max_blocks_per_seq = cache.max_blocks_per_seq;
  p.num_blocks = cache.num_blocks;
  p.block_size = cache.block_size;
  p.scale_log2 = default_scale(d) * 1.4426950408889634f;
  p.tiled = tiled ? static_cast<const unsigned char *>(cache.c_kv) : nullptr;
  p.row_pool = static_cast<const unsigned char *>(cache.c_kv);
  p.rows_contig = !tiled && cache.ckv_stride == kW && cache.kpe_stride == kW &&
                  static_cast<const char *>(cache.k_pe) == static_cast<const char *>(cache.c_kv) + 2 * kDc;
  p.o_part = reinterpret_cast<__nv_bfloat16 *>(w + L.o_part);
  p.lse_part = reinterpret_cast<float *>(w + L.lse_part);
  p.seg_info = reinterpret_cast<int *>(w + L.seg_info);
  p.timeout_rec = p.seg_info + 2 * p.U;
  p.dev_status = dev_status;
  p.kv_begin = kv_begin;
  p.kv_end = kv_end;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * C);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, mla_decode_tc_kernel, mc, mpe, p) != cudaSuccess) return MLA_ERR_CUDA;
  return MLA_OK;
}

namespace {

// out [rows][H][128] = (pieces of each row, merged) . W_UV^(s) per head s, on the tensor cores;
// lse (if non-null) gets the merged log-sum-exps.
int launch_merge_wuv(const mla_dims &d, int rows, const Pieces &pc, const void *w_uv, void *out, float *lse,
                     int *dev_status, cudaStream_t st) {
  // W_UV as [H * 512 rows][128] (boxes of 64 rows x 64 columns).
  CUtensorMap mw;
  int rc = make_map(&mw, w_uv, kDv, (uint64_t)d.n_heads * kDc, (uint64_t)kDv * 2);
  if (rc) return rc;
  const size_t smem = 1024 + kOlBytes + kWuvBytes;
  static std::atomic<int> smem_set[kSmemCacheDevs];
  if (smem_limit(tc_combine_kernel, smem, smem_set) != cudaSuccess)
    return MLA_ERR_CUDA;
  const dim3 grid(d.n_heads, (rows + kCombRows - 1) / kCombRows);
  return launch_pdl(tc_combine_kernel, grid, dim3(kCombThreads), smem, st, mw, pc, rows, lse,
                    static_cast<__nv_bfloat16 *>(out), dev_status) == cudaSuccess
             ? MLA_OK
             : MLA_ERR_CUDA;
}

}  // namespace

int launch_tc_combine(const mla_dims &d, int B, int n_q, const int32_t *seqlens, int max_seqlen, const void *w_uv,
                      void *out, float *lse, void *ws, int *dev_status, cudaStream_t st) {
  (void)seqlens;
  (void)max_seqlen;
  const int n_rb = (n_q * d.n_heads + kRows - 1) / kRows;
  const WsLayout L = ws_layout(B, n_rb);
  char *w = static_cast<char *>(ws);
  if (w_uv && (d.d_v != kDv || (reinterpret_cast<uintptr_t>(w_uv) & 15))) return MLA_ERR_UNSUPPORTED;
  const int rows = B * n_q;
  const int max_segs = B * n_rb + clusters_for_device();
  if (w_uv) {   // merge and W_UV product in one kernel
    const Pieces pc{reinterpret_cast<const __nv_bfloat16 *>(w + L.o_part), reinterpret_cast<const float *>(w + L.lse_part),
                    reinterpret_cast<const int *>(w + L.seg_info), n_q, d.n_heads, n_rb, max_segs, 0};
    return launch_merge_wuv(d, rows, pc, w_uv, out, lse, dev_status, st);
  }
  // Without W_UV the merged rows are the output.
  const int64_t warps = (int64_t)rows * d.n_heads;
  const dim3 mgrid((unsigned)((warps + kMergeThreads / 32 - 1) / (kMergeThreads / 32)));
  return launch_pdl(tc_merge_kernel, mgrid, dim3(kMergeThreads), 0, st, B, n_q, d.n_heads, n_rb, max_segs,
                    reinterpret_cast<const int *>(w + L.seg_info), reinterpret_cast<const __nv_bfloat16 *>(w + L.o_part),
                    reinterpret_cast<const float *>(w + L.lse_part), static_cast<__nv_bfloat16 *>(out), lse) == cudaSuccess
             ? MLA_OK
             : MLA_ERR_CUDA;
}

bool tc_merge_parts_supported(const mla_dims &d, const void *o_parts, const void *w_uv, const void *out) {
  const bool aligned = !(reinterpret_cast<uintptr_t>(o_parts) & 15) && !(reinterpret_cast<uintptr_t>(out) & 15) &&
                       !(reinterpret_cast<uintptr_t>(w_uv) & 15);
  return d.dtype == MLA_BF16 && d.d_c == kDc && (!w_uv || d.d_v == kDv) && aligned;
}

int launch_tc_merge_parts(const mla_dims &d, int B, int n_q, int n_parts, const void *o_parts, const float *lse_parts,
                          const void *w_uv, void *out, float *lse, cudaStream_t st) {
  if (!tc_merge_parts_supported(d, o_parts, w_uv, out) || n_parts <= 0) return MLA_ERR_UNSUPPORTED;
  const int rows = B * n_q;
  if (w_uv) {
    const Pieces pc{static_cast<const __nv_bfloat16 *>(o_parts), lse_parts, nullptr, n_q, d.n_heads, 0, 0, n_parts};
    return launch_merge_wuv(d, rows, pc, w_uv, out, lse, nullptr, st);
  }
  const int64_t R = (int64_t)rows * d.n_heads;
  const dim3 mgrid((unsigned)((R + kMergeThreads / 32 - 1) / (kMergeThreads / 32)));
  return launch_pdl(parts_merge_kernel, mgrid, dim3(kMergeThreads), 0, st, R, n_parts,
                    static_cast<const __nv_bfloat16 *>(o_parts), lse_parts, static_cast<__nv_bfloat16 *>(out), lse) ==
                 cudaSuccess
             ? MLA_OK
             : MLA_ERR_CUDA;
}

}  // namespace mla
