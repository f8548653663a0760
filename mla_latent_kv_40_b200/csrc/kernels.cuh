// Argument bundles and launchers of every libmla kernel (host side).
#pragma once

#include <atomic>

#include "common.cuh"

namespace mla {

// Launch with programmatic stream serialisation: the kernel may start while the previous kernel
// on the stream is still running, and orders itself with grid_dep_wait().
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args &&>(args)...);
}

// Raises a kernel's dynamic shared-memory limit to `bytes` on the current device.  The driver is
// called only the first time a launcher asks for that size (or more) on that device, since the
// limit then stays set for the process; `cache` is the launcher's own record of the sizes set per
// device.  Devices past the table's end always call the driver.
constexpr int kSmemCacheDevs = 64;
template <typename... KArgs>
inline cudaError_t smem_limit(void (*kernel)(KArgs...), size_t bytes, std::atomic<int> (&cache)[kSmemCacheDevs]) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  const bool tracked = dev >= 0 && dev < kSmemCacheDevs;
  if (tracked && cache[dev].load(std::memory_order_acquire) >= (int)bytes) return cudaSuccess;
  const cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess && tracked) {
    int cur = cache[dev].load(std::memory_order_relaxed);
    while (cur < (int)bytes && !cache[dev].compare_exchange_weak(cur, (int)bytes, std::memory_order_release)) {
    }
  }
  return e;
}

struct AppendArgs {
  int T, d_model, d_c, d_rope;
  const void *h, *w_dkv, *w_kr, *gamma;
  const int32_t *seq_idx, *pos;
  void *c_kv, *k_pe;
  int64_t ckv_stride, kpe_stride;
  const int32_t *block_table;
  int num_seqs, max_blocks_per_seq, num_blocks, block_size;
  int layout;
  float rms_eps, rope_base;
  int *dev_status;
};

struct AbsorbArgs {
  int B, n_q, H, d_c, d_rope, d_nope;
  const void *q_nope, *q_pe, *w_uk;
  const int32_t *seqlens;
  void *q_out;  // [B, n_q, H, d_c + d_rope]
  float rope_base;
};

// Paged-cache view shared by the decode kernels.
struct CacheView {
  const void *c_kv, *k_pe;
  int64_t ckv_stride, kpe_stride;
  const int32_t *block_table;
  int max_blocks_per_seq, num_blocks, block_size;
  int layout;                    // mla_cache_layout
  int d_c, W;                    // latent width and full row width d_c + d_rope

  template <typename T>
  __device__ __forceinline__ float load(int64_t row, int d) const {
    return to_f32(*latent_elem<const T>(const_cast<void *>(c_kv), const_cast<void *>(k_pe), ckv_stride, kpe_stride,
                                        layout, d_c, W, row, d));
  }
};

// Split-KV attention over the latent cache (the absorbed decode core).
struct AttnArgs {
  int B, n_q, H, d_c, d_rope;
  const void *q;            // [B, n_q, H, d_c + d_rope]: [q_lat | rotated q_pe]
  CacheView cache;
  const int32_t *seqlens;
  float scale;
  int chunk;                // keys per split
  int max_chunks;           // splits allocated per sequence
  float *o_part;            // [B, max_chunks, n_q*H, d_c], normalised by the split's own sum
  float *lse_part;          // [B, max_chunks, n_q*H]
  int *dev_status;
  int kv_begin, kv_end;     // only keys in [kv_begin, kv_end) are read
};

// Merge of the split partials and the per-head up-projection.
struct CombineArgs {
  int B, n_q, H, d_c, d_v;
  const int32_t *seqlens;   // NULL: every one of the max_chunks splits holds a partial
  int chunk, max_chunks;
  const float *o_part, *lse_part;
  const void *w_uv;         // [H, d_c, d_v], NULL: write o_lat instead
  void *out;                // [B, n_q, H, d_v] or o_lat [B, n_q, H, d_c]
  float *lse;               // [B, n_q, H] or NULL
};

struct PrefillArgs {
  int B, total, max_seqlen, H, d_c, d_rope, d_nope, d_v;
  const int32_t *cu_seqlens;
  const void *q_nope, *q_pe, *w_uk, *w_uv;
  CacheView cache;
  void *qbuf, *kbuf, *vbuf;   // workspace: [total, H, d_nope+d_rope] x2, [total, H, d_v]
  void *out;
  float *lse;
  float scale, rope_base;
  int *dev_status;
  // Tiled workspace of the tensor-core prefill (set by the launcher): per head s and sequence b,
  // Q in tiles of 128 query rows [3 chunks][128 rows x 128 B] (48 KB) at q_tiles, and K with V in
  // tiles of 64 tokens [3 K chunks | 2 V chunks][64 rows x 128 B] (40 KB) at kv_tiles; chunks
  // 128-byte swizzled like the tiled latent pool, so each tile moves as one bulk copy.
  int tiled, nqt, nkt;        // tiles per (head, sequence): nqt = ceil(max_seqlen / 128), nkt = 2 nqt
  unsigned char *q_tiles, *kv_tiles;
};

// Byte offset of element (row, dim) inside a tile of `rows` rows and 64-dim chunks.
__host__ __device__ __forceinline__ int64_t swz_tile_offset(int rows, int row, int dim) {
  const int c = dim >> 6, g = (dim >> 3) & 7, e = dim & 7;
  return (int64_t)c * rows * 128 + row * 128 + ((g ^ (row & 7)) << 4) + e * 2;
}
constexpr int64_t kPfQTileBytes = 128 * 192 * 2;     // 49152
constexpr int64_t kPfKVTileBytes = 64 * (192 + 128) * 2;   // 40960
// Workspace bytes of the tiled prefill layout.
inline size_t prefill_tiled_bytes(int B, int H, int max_seqlen) {
  const size_t nqt = (size_t)(max_seqlen + 127) / 128;
  const size_t q = (size_t)H * B * nqt * kPfQTileBytes;
  return ((q + 255) & ~size_t(255)) + (size_t)H * B * 2 * nqt * kPfKVTileBytes;
}

int launch_append(const AppendArgs &a, bool bf16, cudaStream_t st);
int launch_absorb(const AbsorbArgs &a, bool bf16, cudaStream_t st);
int launch_attn_simt(const AttnArgs &a, bool bf16, cudaStream_t st);
int launch_combine(const CombineArgs &a, bool bf16, cudaStream_t st);
int launch_prefill_simt(const PrefillArgs &a, bool bf16, cudaStream_t st);
// Step (3) of the prefill, causal attention over the decompressed rows, on tcgen05.
bool prefill_tc_supported(const PrefillArgs &a, bool bf16);
// Step (2) of the prefill, per-head decompression of K and V, on tcgen05 (row pools).
bool decompress_tc_supported(const PrefillArgs &a, bool bf16);
int launch_decompress_tc(const PrefillArgs &a, cudaStream_t st);
int launch_prefill_tc_attention(const PrefillArgs &a, cudaStream_t st);
// bf16 tensor-core (mma.sync) projections.
size_t append_mma_workspace(int T, int d_model, int W, int *nsplit, int *k_per_split);
bool append_mma_supported(const AppendArgs &a, bool bf16);
int launch_append_mma(const AppendArgs &a, void *ws, cudaStream_t st);
bool absorb_mma_supported(const AbsorbArgs &a, bool bf16);
int launch_absorb_mma(const AbsorbArgs &a, cudaStream_t st);
// tcgen05 versions (TMA-fed, weights on the M side); the append one writes the same partials
// as launch_append_mma and leaves them to its finish kernel.
bool absorb_tc_supported(const AbsorbArgs &a, bool bf16);
int launch_absorb_tc(const AbsorbArgs &a, int *dev_status, cudaStream_t st);
bool append_tc_supported(const AppendArgs &a, bool bf16);
int launch_append_tc(const AppendArgs &a, void *ws, int nsplit, int k_per_split, cudaStream_t st);
int launch_append_finish(const AppendArgs &a, const void *ws, int nsplit, cudaStream_t st);
// Fused decode-step preparation: the append of the step's new tokens and the query absorption in
// one launch (tensor-core shapes only).  `counter` is 4 bytes of workspace, zeroed by the launcher.
bool decode_prep_supported(const AppendArgs &ap, const AbsorbArgs &ab);
int launch_decode_prep(const AppendArgs &ap, const AbsorbArgs &ab, void *part, int nsplit, int k_per_split,
                       unsigned *counter, cudaStream_t st);
int launch_cache_convert(const void *src, void *dst, int64_t num_rows, int W, bool to_tiled, cudaStream_t st);
// Cross-device merge: partials [N][B][n_q][H][d_c] (dtype) and lses [N][B][n_q][H] -> the split
// layout launch_combine reads (o_part [B][N][n_q*H][d_c] fp32, lse_part [B][N][n_q*H]).
int launch_partials_to_splits(int N, int B, int n_q, int H, int d_c, const void *o_parts, const float *lse_parts,
                              bool bf16, float *o_part, float *lse_part, cudaStream_t st);
// C[b] = A[b] B[b] with element strides (any transposition), fp32 accumulation on CUDA cores,
// optionally split over K (fp32 partials in `part`, then summed into C).
struct GemmArgs {
  int M, N, K, batch, ksplit;
  const void *A;
  int64_t sa_b, sa_m, sa_k;
  const void *B;
  int64_t sb_b, sb_k, sb_n;
  void *C;
  int64_t sc_b, sc_m, sc_n;
  float *part;              // [batch][ksplit][M][N] when ksplit > 1
};
size_t gemm_simt_workspace(const GemmArgs &g);
int launch_gemm_simt(const GemmArgs &g, bool bf16, cudaStream_t st);
// The tensor-core product for weight-streaming shapes (MLA_ERR_UNSUPPORTED, nothing launched, when
// the layout does not fit); the in-order sum of K-split partials into C; and the dispatcher that tries
// the tensor cores first.  All use the same partial buffer (gemm_simt_workspace).
int launch_gemm_tc(const GemmArgs &g, bool bf16, cudaStream_t st);
int launch_gemm_reduce(const GemmArgs &g, bool bf16, cudaStream_t st);
int launch_gemm(const GemmArgs &g, bool bf16, cudaStream_t st);
// RoPE of the query-latent path's q_pe [T, H, d_R] into the RoPE slots of q_abs [T, H, d_c + d_R].
int launch_rope_into_query(int B, int n_q, int H, int d_c, int d_rope, const void *q_pe_raw, const int32_t *seqlens,
                           void *q_abs, float rope_base, bool bf16, cudaStream_t st);
// Sparse decode: compact each query token's listed cache rows into its own run of 64-token pages.
int launch_sparse_gather(int B, int n_q, int topk, const int32_t *idx, const int32_t *seqlens, int max_seqlen,
                         const CacheView &src, void *pool, bool dst_tiled, int elem, int32_t *counts,
                         int *dev_status, cudaStream_t st);

}  // namespace mla
