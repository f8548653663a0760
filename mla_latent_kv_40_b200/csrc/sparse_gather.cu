// Gather of selected cache rows for the sparse decode: every query token (b, j) lists the
// tokens it attends to; its valid entries are compacted, in list order, into a private run of
// 64-token pages, which the regular split-KV attention then reads as one short sequence.
#include "kernels.cuh"

namespace mla {
namespace {

constexpr int kPage = 64;
constexpr int kThreads = 256;

// Byte address of the 16-byte group holding dims d .. d + 16/elem - 1 of row r.
__device__ __forceinline__ const unsigned char *src_group(const CacheView &c, int64_t r, int d, int elem) {
  if (c.layout == MLA_CACHE_TILED)
    return static_cast<const unsigned char *>(c.c_kv) + tiled_byte_offset(r, d, c.W);
  return d < c.d_c ? static_cast<const unsigned char *>(c.c_kv) + (r * c.ckv_stride + d) * elem
                   : static_cast<const unsigned char *>(c.k_pe) + (r * c.kpe_stride + (d - c.d_c)) * elem;
}

__device__ __forceinline__ unsigned char *dst_group(unsigned char *pool, bool tiled, int64_t r, int d, int W,
                                                    int elem) {
  return tiled ? pool + tiled_byte_offset(r, d, W) : pool + (r * W + d) * elem;
}

// grid (units = B * n_q, pages per unit); a CTA compacts and copies one page of its unit's list.
__global__ void __launch_bounds__(kThreads)
sparse_gather_kernel(int n_q, int topk, int pages, const int32_t *idx, const int32_t *seqlens, int max_seqlen,
                     CacheView c, unsigned char *pool, bool dst_tiled, bool vec16, int elem, int32_t *counts,
                     int *dev_status) {
  __shared__ int64_t src_row[kPage];
  __shared__ int slot[kPage];
  __shared__ int warp_valid[kPage / 32];
  const int u = blockIdx.x, pg = blockIdx.y;
  const int b = u / n_q, j = u % n_q;
  const int tid = threadIdx.x;
  int S = seqlens[b];
  S = S < 0 ? 0 : (S > max_seqlen ? max_seqlen : S);
  const int limit = S - n_q + j;                       // last position this query token may see
  const int32_t *list = idx + (int64_t)u * topk;

  // A listed token is valid when it is not padding (-1), lies in 0 .. limit and its block id is in the pool.
  auto row_of = [&](int e, bool report_bad) -> int64_t {
    if (e >= topk) return -1;
    const int t = list[e];
    if (t == -1) return -1;
    const int64_t r = t >= 0 && t <= limit
                          ? cache_row(c.block_table, c.max_blocks_per_seq, c.num_blocks, c.block_size, b, t)
                          : -1;
    if (r < 0 && report_bad) report(dev_status, MLA_ERR_BAD_INDEX);
    return r;
  };

  // Valid entries before this page: the page's first slot.
  int before = 0;
  for (int base = 0; base < kPage * pg; base += kThreads) {
    const int e = base + tid;
    before += __syncthreads_count(e < kPage * pg && row_of(e, false) >= 0);
  }
  // This page's entries: ranks by ballot, in list order.
  if (tid < kPage) {
    const int64_t r = row_of(kPage * pg + tid, true);
    const unsigned m = __ballot_sync(0xffffffffu, r >= 0);
    if ((tid & 31) == 0) warp_valid[tid >> 5] = __popc(m);
    src_row[tid] = r;
    slot[tid] = r >= 0 ? __popc(m & ((1u << (tid & 31)) - 1)) : -1;
  }
  __syncthreads();
  if (tid < kPage && (tid >> 5) == 1 && slot[tid] >= 0) slot[tid] += warp_valid[0];
  __syncthreads();
  const int mine = warp_valid[0] + warp_valid[1];
  if (pg == pages - 1 && tid == 0) {
    counts[u] = before + mine;
    if (before + mine == 0) report(dev_status, MLA_ERR_BAD_INDEX);   // nothing to attend to
  }
  // Copy: row by row, each thread one 16-byte group (or one element where the rows are not
  // 16-byte granular).
  const int per = vec16 ? 16 / elem : 1;               // elements per item
  const int items = c.W / per;
  const int64_t row0 = (int64_t)u * pages * kPage;
  for (int e = tid; e < kPage * items; e += kThreads) {
    const int k = e / items, d = (e % items) * per;
    if (slot[k] < 0) continue;
    const int64_t dst_row = row0 + before + slot[k];
    const unsigned char *s = src_group(c, src_row[k], d, elem);
    unsigned char *t = dst_group(pool, dst_tiled, dst_row, d, c.W, elem);
    if (vec16) *reinterpret_cast<uint4 *>(t) = *reinterpret_cast<const uint4 *>(s);
    else if (elem == 2) *reinterpret_cast<uint16_t *>(t) = *reinterpret_cast<const uint16_t *>(s);
    else *reinterpret_cast<uint32_t *>(t) = *reinterpret_cast<const uint32_t *>(s);
  }
}

}  // namespace

int launch_sparse_gather(int B, int n_q, int topk, const int32_t *idx, const int32_t *seqlens, int max_seqlen,
                         const CacheView &src, void *pool, bool dst_tiled, int elem, int32_t *counts,
                         int *dev_status, cudaStream_t st) {
  const int pages = (topk + kPage - 1) / kPage;
  // 16-byte items need every 16-byte group of a row to lie inside one contiguous, aligned piece.
  const int per = 16 / elem;
  bool vec16 = src.W % per == 0 && (src.d_c % per == 0) &&
               !(reinterpret_cast<uintptr_t>(pool) & 15) && !(reinterpret_cast<uintptr_t>(src.c_kv) & 15);
  if (src.layout == MLA_CACHE_ROWS)
    vec16 = vec16 && (src.ckv_stride * elem) % 16 == 0 && (src.kpe_stride * elem) % 16 == 0 &&
            !(reinterpret_cast<uintptr_t>(src.k_pe) & 15);
  if (dst_tiled && !vec16) return MLA_ERR_UNSUPPORTED;   // the tiled layout moves whole 16-byte groups
  sparse_gather_kernel<<<dim3(B * n_q, pages), kThreads, 0, st>>>(n_q, topk, pages, idx, seqlens, max_seqlen, src,
                                                                  static_cast<unsigned char *>(pool), dst_tiled,
                                                                  vec16, elem, counts, dev_status);
  return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

}  // namespace mla
