/*
 * mla.h — C ABI of libmla.so: Multi-head Latent Attention (MLA) over a paged
 * latent KV cache, for NVIDIA B200 (sm_100a).
 *
 * The method (sources by page title and section):
 *  - "DeepSeek-V3 解读 1: MLA", section "MLA：高层次的思路": each token's hidden
 *    state h is compressed to a latent c_KV of width d_c; only the latent is
 *    cached and per-head keys/values are rebuilt from it by W_UK and W_UV.
 *  - same page, section "为什么需要解耦 RoPE": one extra key k_pe of width d_R,
 *    shared by every head, carries RoPE; the latent part is never rotated.
 *  - "Transformer升级之路：21、MLA好在哪里?（下）", section 双重投影: decode may
 *    fold W_UK into the query (q_lat = q_nope W_UK^T, width d_c) and apply
 *    W_UV after attention, so every head attends to the same cached rows
 *    (MQA with K = V = c); prefill uses the decompressed multi-head form.
 *
 * Conventions shared by every entry point
 *  - All tensor pointers are DEVICE pointers, row-major, owned by the caller.
 *    The library allocates no device memory; scratch space is the caller's
 *    `workspace`, sized by the matching *_workspace_size call.
 *  - Float tensors use the element type dims->dtype (MLA_F32: float,
 *    MLA_BF16: __nv_bfloat16).  lse outputs are always float.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *    stream).  Argument errors are returned before anything is launched.
 *    Errors found on the device (a block id outside [0, num_blocks), a
 *    bounded wait that timed out) are written to *dev_status (if non-NULL) with
 *    an atomic compare-and-swap from 0, so the first error wins; the caller
 *    zeroes it beforehand and reads it after synchronising.
 *  - Concurrent calls on different streams with disjoint outputs and
 *    workspaces are safe, with one exception: mla_decode_noalloc, whose calls
 *    share one library-owned scratch buffer per GPU (see there).  Besides that
 *    buffer, the library's only global state is per-device host-side caches
 *    filled on first use and read-only afterwards: the number of attention
 *    clusters that fit on the device, the driver's tensor-map encoder, the
 *    device address of the no-allocation scratch buffer, and, per kernel, the
 *    dynamic shared-memory size already requested from the driver.  Each is
 *    guarded (a mutex or atomics), so first calls from several host threads
 *    are safe.
 *  - There is no CPU fallback: a shape the CUDA kernels do not handle returns
 *    MLA_ERR_UNSUPPORTED.
 *
 * Paged latent cache
 *  Token i of sequence b lives in pool row r = blk * block_size + i % block_size
 *  with blk = block_table[b * max_blocks_per_seq + i / block_size]
 *  (block_table == NULL means the identity table: blk = b * max_blocks_per_seq
 *  + i / block_size, i.e. each sequence owns a contiguous run of rows).
 *  Two pool layouts (mla_dims.cache_layout):
 *  - MLA_CACHE_ROWS: c_KV of row r is at c_kv + r * ckv_stride (d_c elements),
 *    the rotated RoPE key at k_pe + r * kpe_stride (d_R elements).  One pool of
 *    rows of d_c + d_R elements has k_pe = c_kv + d_c and both strides d_c + d_R.
 *  - MLA_CACHE_TILED: one pool at c_kv (k_pe and the strides are ignored), in
 *    pages of 64 tokens; block_size must be a multiple of 64 and block blk
 *    holds pages blk*block_size/64 .. +block_size/64-1, i.e. row r lies in page
 *    r / 64 as token t = r % 64.  A page is W/64 chunks (W = d_c + d_R, a
 *    multiple of 64) of 8 KB; chunk c holds dims 64c .. 64c+63 of its 64 tokens,
 *    token t at byte 128 t of the chunk, and its 16-byte group g (dims 8g ..
 *    8g+7 of the chunk) at byte 16 * (g XOR (t mod 8)) of that 128-byte line.
 *    c_KV dims come first, then the RoPE key.  This is the order in which the
 *    tensor cores read a page (128-byte swizzled, K-major), so a page moves
 *    with plain contiguous bulk copies.  bf16 only.  mla_cache_pack /
 *    mla_cache_unpack convert between a row pool and this layout.
 *
 * Positions and RoPE
 *  Positions are 0-based.  Pair (2i, 2i+1) of a RoPE vector at position p is
 *  rotated by p * theta_i, theta_i = rope_base^(-2i/d_R), with
 *  [x'; y'] = [[cos, -sin], [sin, cos]] [x; y].  In decode, seqlens[b] counts
 *  the cached tokens INCLUDING the n_q new ones (already appended), and query
 *  token j of sequence b sits at position seqlens[b] - n_q + j and attends to
 *  keys 0 .. seqlens[b] - n_q + j (causal among the new tokens).
 */
#ifndef MLA_H_
#define MLA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define MLA_API __attribute__((visibility("default")))
#else
#define MLA_API
#endif

typedef struct CUstream_st *mla_stream_t; /* the same type as cudaStream_t */

typedef enum {
  MLA_OK = 0,
  MLA_ERR_INVALID_ARG = -1, /* a NULL required pointer, a non-positive size, inconsistent dims */
  MLA_ERR_UNSUPPORTED = -2, /* a valid shape the kernels do not implement */
  MLA_ERR_WORKSPACE = -3,   /* workspace NULL or smaller than *_workspace_size reports */
  MLA_ERR_CUDA = -4,        /* a CUDA runtime/driver call or a kernel launch failed */
  MLA_ERR_TIMEOUT = -5,     /* device only: a bounded wait inside a kernel gave up */
  MLA_ERR_BAD_INDEX = -6,   /* device only: a block id outside [0, num_blocks) or a bad position */
  MLA_ERR_STATIC_WS = -7    /* the shape needs more scratch than mla_decode_noalloc's built-in buffer */
} mla_status;

typedef enum { MLA_F32 = 0, MLA_BF16 = 1 } mla_dtype;

typedef enum { MLA_CACHE_ROWS = 0, MLA_CACHE_TILED = 1 } mla_cache_layout;

typedef struct {
  int n_heads;        /* H: query heads */
  int d_c;            /* latent width (c_KV) */
  int d_rope;         /* d_R: width of the shared RoPE key and of q_pe; even */
  int d_nope;         /* per-head query/key width without RoPE */
  int d_v;            /* per-head value width */
  int d_model;        /* D: hidden width of h (append only) */
  int block_size;     /* tokens per cache page, >= 1 */
  int ckv_stride;     /* elements between consecutive rows of the c_KV pool, >= d_c */
  int kpe_stride;     /* elements between consecutive rows of the k_pe pool, >= d_rope */
  float rope_base;    /* RoPE base, e.g. 10000 */
  float softmax_scale;/* <= 0 selects 1/sqrt(d_nope + d_rope) */
  float rms_eps;      /* epsilon of the RMSNorm on c_KV, e.g. 1e-6 */
  int dtype;          /* mla_dtype of every float tensor */
  int cache_layout;   /* mla_cache_layout of the latent pool */
} mla_dims;

/*
 * mla_append_latent — write the cache rows of T new tokens.
 *   "DeepSeek-V3 解读 1: MLA", sections "MLA：高层次的思路" (c_KV = h W_DKV) and
 *   "为什么需要解耦 RoPE" (k_pe = RoPE(h W_KR), shared by all heads), with an
 *   RMSNorm over the d_c latent dims: c_KV = gamma * c / sqrt(mean(c^2) + eps).
 *   h [T, D]; w_dkv [D, d_c]; w_kr [D, d_R]; rms_gamma [d_c] or NULL (= all ones);
 *   seq_idx [T], pos [T] (int32): sequence and 0-based position of each token.
 *   Writes c_kv/k_pe rows of (seq_idx[t], pos[t]) through block_table
 *   ([num_seqs, max_blocks_per_seq] or NULL, see above).  On the device,
 *   seq_idx outside [0, num_seqs), pos outside [0, max_blocks_per_seq *
 *   block_size) and block ids outside [0, num_blocks) report
 *   MLA_ERR_BAD_INDEX and skip that token.
 *   T == 0 is a no-op.  Rows not named by (seq_idx, pos) are not touched.
 */
MLA_API int mla_append_latent(const mla_dims *dims, int T, const void *h, const void *w_dkv,
                      const void *w_kr, const void *rms_gamma, const int32_t *seq_idx,
                      const int32_t *pos, void *c_kv, void *k_pe, const int32_t *block_table,
                      int num_seqs, int max_blocks_per_seq, int num_blocks, void *workspace,
                      size_t ws_bytes, int *dev_status, mla_stream_t stream);

/*
 * mla_append_workspace_size — scratch bytes that let mla_append_latent run
 *   the down-projection on tensor cores, split over d_model (bf16 shapes with
 *   d_model a multiple of 64, d_c a multiple of 64, d_R <= 64).  0 when the
 *   shape has no such path.  mla_append_latent with workspace == NULL (or a
 *   smaller one) runs the CUDA-core path instead; both give the same rows up
 *   to the order of fp32 additions.
 */
MLA_API int mla_append_workspace_size(const mla_dims *dims, int T, size_t *bytes);

/*
 * mla_decode_step_workspace_size / mla_decode_step — one whole decode step:
 *   the append of the step's n_q new tokens of every sequence, then mla_decode.
 *   "DeepSeek-V3 解读 1: MLA", section "Key-Value 缓存": every generated token's
 *   key and value enter the cache before it is attended to; here its latent
 *   row c_KV = RMSNorm(h W_DKV) and its RoPE key (as mla_append_latent) are
 *   written at positions seqlens[b] - n_q .. seqlens[b] - 1 of sequence b, and
 *   the decode of mla_decode reads them.  On the tensor-core shapes the append
 *   and the query absorption run as ONE kernel launch ahead of the attention
 *   (its append-finish CTAs wait, with a bounded wait, for its projection CTAs);
 *   other shapes run the same steps as separate launches.
 *   h_new [B, n_q, D] (the new tokens' hidden states, token j of sequence b at
 *   row b n_q + j); w_dkv, w_kr, rms_gamma as mla_append_latent; seqlens count
 *   the cached tokens including the new ones; the other arguments as
 *   mla_decode.  The cache rows of the new tokens are written (c_kv, k_pe).
 *   workspace: >= mla_decode_step_workspace_size bytes, 256-byte aligned.
 */
MLA_API int mla_decode_step_workspace_size(const mla_dims *dims, int B, int n_q, int max_seqlen, size_t *bytes);
MLA_API int mla_decode_step(const mla_dims *dims, int B, int n_q, const void *h_new, const void *w_dkv,
                            const void *w_kr, const void *rms_gamma, const void *q_nope, const void *q_pe, void *c_kv,
                            void *k_pe, const int32_t *block_table, int max_blocks_per_seq, int num_blocks,
                            const int32_t *seqlens, int max_seqlen, const void *w_uk, const void *w_uv, void *out,
                            float *lse, void *workspace, size_t ws_bytes, int *dev_status, mla_stream_t stream);

/*
 * mla_absorb_q — the decode query in latent space.
 *   "Transformer升级之路：21、MLA好在哪里?（下）", section 双重投影, decoding
 *   column: q^(s) = x W_q^(s) W_k^(s)T lies in R^{d_c}; here
 *   q_lat[b,j,s,:] = W_UK[s] q_nope[b,j,s,:] and q_rot = RoPE(q_pe, seqlens[b] - n_q + j).
 *   q_nope [B, n_q, H, d_nope], q_pe [B, n_q, H, d_R] (not rotated),
 *   w_uk [H, d_c, d_nope], seqlens [B] (int32, device).
 *   Writes q_out [B, n_q, H, d_c + d_R] = [q_lat | q_rot] in dims->dtype
 *   (rounded once, after fp32 accumulation).
 */
MLA_API int mla_absorb_q(const mla_dims *dims, int B, int n_q, const void *q_nope, const void *q_pe,
                 const void *w_uk, const int32_t *seqlens, void *q_out, mla_stream_t stream);

/*
 * mla_decode_workspace_size — bytes of scratch mla_decode / mla_decode_latent
 *   need for B sequences of n_q query tokens whose seqlens are <= max_seqlen.
 *   Depends on the current device's SM count.
 */
MLA_API int mla_decode_workspace_size(const mla_dims *dims, int B, int n_q, int max_seqlen, size_t *bytes);

/*
 * mla_decode — one batched decode step in matrix-absorbed form.
 *   Same section 双重投影, decoding column, with the shared RoPE key:
 *   z_i = scale * (q_lat . c_i + q_rot . kpe_i), softmax over keys
 *   0 .. seqlens[b] - n_q + j, o_lat = sum_i p_i c_i, out^(s) = o_lat W_UV^(s).
 *   q_nope [B, n_q, H, d_nope], q_pe [B, n_q, H, d_R] (not rotated);
 *   cache as described above; seqlens [B] (int32, device, >= n_q, <= max_seqlen);
 *   w_uk [H, d_c, d_nope]; w_uv [H, d_c, d_v].
 *   Writes out [B, n_q, H, d_v] and, if non-NULL, lse [B, n_q, H] (float,
 *   natural log of sum_i exp(z_i)).  workspace: >= mla_decode_workspace_size bytes,
 *   256-byte aligned.  Errors: INVALID_ARG, UNSUPPORTED (n_q * H > 256),
 *   WORKSPACE, CUDA; on the device BAD_INDEX, TIMEOUT.
 */
MLA_API int mla_decode(const mla_dims *dims, int B, int n_q, const void *q_nope, const void *q_pe,
               const void *c_kv, const void *k_pe, const int32_t *block_table,
               int max_blocks_per_seq, int num_blocks, const int32_t *seqlens, int max_seqlen,
               const void *w_uk, const void *w_uv, void *out, float *lse, void *workspace,
               size_t ws_bytes, int *dev_status, mla_stream_t stream);

/*
 * mla_decode_latent — mla_decode without the W_UV up-projection: writes the
 *   softmax-weighted latent o_lat [B, n_q, H, d_c] (dims->dtype) and lse.  For
 *   callers that fold W_UV into their output projection (same page, section
 *   键值共享: the c -> v map is absorbed on the W_o side).  w_uv is not read.
 */
MLA_API int mla_decode_latent(const mla_dims *dims, int B, int n_q, const void *q_nope, const void *q_pe,
                      const void *c_kv, const void *k_pe, const int32_t *block_table,
                      int max_blocks_per_seq, int num_blocks, const int32_t *seqlens,
                      int max_seqlen, const void *w_uk, void *o_lat, float *lse, void *workspace,
                      size_t ws_bytes, int *dev_status, mla_stream_t stream);

/*
 * mla_decode_attention / mla_decode_combine — the two halves of mla_decode
 *   after mla_absorb_q, for callers that schedule the stages themselves.
 *   mla_decode_attention: q_abs [B, n_q, H, d_c + d_R] is mla_absorb_q's output;
 *   runs the split-KV attention over the latent cache (scores
 *   scale * q_abs . [c_i | kpe_i], online softmax, sum_i p_i c_i) and leaves
 *   per-split partial outputs and log-sum-exps in `workspace` (layout private
 *   to the library; same size rule as mla_decode).
 *   mla_decode_combine: merges those partials by their log-sum-exps and, when
 *   w_uv is non-NULL, applies out^(s) = o_lat W_UV^(s) (out [B, n_q, H, d_v]);
 *   with w_uv == NULL it writes o_lat [B, n_q, H, d_c].  It must see the same
 *   dims, B, n_q, seqlens, max_seqlen and workspace as the attention call.
 */
MLA_API int mla_decode_attention(const mla_dims *dims, int B, int n_q, const void *q_abs, const void *c_kv,
                                 const void *k_pe, const int32_t *block_table, int max_blocks_per_seq,
                                 int num_blocks, const int32_t *seqlens, int max_seqlen, void *workspace,
                                 size_t ws_bytes, int *dev_status, mla_stream_t stream);
MLA_API int mla_decode_combine(const mla_dims *dims, int B, int n_q, const int32_t *seqlens, int max_seqlen,
                               const void *w_uv, void *out, float *lse, void *workspace, size_t ws_bytes,
                               mla_stream_t stream);

/*
 * mla_decode_noalloc — mla_decode for callers that cannot allocate device
 *   memory.  The source pages have no counterpart: this is a deployment
 *   variant, not part of the method.  Some callers cannot call cudaMalloc or
 *   hold a workspace of their own: code embedded in a host runtime that owns
 *   every device allocation and forbids side allocations, or plain C callers
 *   with no allocator at hand.  This entry point takes the same arguments as
 *   mla_decode minus the workspace, and uses instead one scratch buffer of
 *   MLA_NOALLOC_SCRATCH_BYTES (16 MiB) that the library reserves statically
 *   in device memory; every GPU that loads the library holds it until the
 *   process exits.  It allocates nothing: no cudaMalloc, no cudaFree, no
 *   allocating library routine.
 *   - The first call on each device looks up that device's address of the
 *     buffer (once per device, with that device current); make that first
 *     call before any stream capture.
 *   - Every call on a device shares the one buffer, which keeps the last
 *     call's contents.  Calls whose executions overlap on the GPU (different
 *     streams, or several host threads) race on it: serialise them.
 *   - Shapes whose mla_decode_workspace_size exceeds the buffer return
 *     MLA_ERR_STATIC_WS before anything is launched.
 *   Output and errors are otherwise those of mla_decode.
 */
#define MLA_NOALLOC_SCRATCH_BYTES (16u << 20)
MLA_API int mla_decode_noalloc(const mla_dims *dims, int B, int n_q, const void *q_nope, const void *q_pe,
                               const void *c_kv, const void *k_pe, const int32_t *block_table,
                               int max_blocks_per_seq, int num_blocks, const int32_t *seqlens, int max_seqlen,
                               const void *w_uk, const void *w_uv, void *out, float *lse, int *dev_status,
                               mla_stream_t stream);

/*
 * mla_decode_partial — one device's share of a decode whose keys are split
 *   between devices: mla_decode_latent restricted to the cached keys in
 *   [kv_begin, kv_end) of every sequence (each query token still sees only
 *   keys up to its own position seqlens[b] - n_q + j).
 *   "现代 LLM 的 Memory-Compute Trade-off：从 MHA 到 MLA", section "MHA 与 KV
 *   Cache": the cache of one long sequence grows linearly with its length, so
 *   a 128k-token sequence may be spread over several GPUs; and "Transformer
 *   升级之路：21", section 总而言之: MQA-form decoding cannot be split by head,
 *   so the split is by key range.  Each device's partial is merged exactly by
 *   mla_merge_partials.
 *   kv_begin: a multiple of 64, >= 0; kv_end > kv_begin.  seqlens are the full
 *   sequence lengths (they fix the query positions).
 *   Writes o_lat [B, n_q, H, d_c] (dims->dtype): the softmax-weighted latent
 *   over the range's visible keys, normalised by their own sum; and lse
 *   [B, n_q, H] (float, required): their log-sum-exp, -inf (with o_lat 0)
 *   where none is visible.  Workspace as mla_decode_workspace_size.
 */
MLA_API int mla_decode_partial(const mla_dims *dims, int B, int n_q, const void *q_nope, const void *q_pe,
                               const void *c_kv, const void *k_pe, const int32_t *block_table, int max_blocks_per_seq,
                               int num_blocks, const int32_t *seqlens, int max_seqlen, int kv_begin, int kv_end,
                               const void *w_uk, void *o_lat, float *lse, void *workspace, size_t ws_bytes,
                               int *dev_status, mla_stream_t stream);

/*
 * mla_merge_workspace_size / mla_merge_partials — the exact merge of n_parts
 *   partials of one decode (e.g. gathered from n_parts devices):
 *   LSE = ln sum_r exp(lse_r), o_lat = sum_r exp(lse_r - LSE) o_lat_r, then
 *   out^(s) = o_lat^(s) W_UV^(s) ("Transformer升级之路：21", section 双重投影,
 *   decoding column); with w_uv == NULL it writes o_lat [B, n_q, H, d_c].
 *   o_lat_parts [n_parts, B, n_q, H, d_c] (dims->dtype), lse_parts
 *   [n_parts, B, n_q, H] (float), both device memory (the caller gathers them,
 *   e.g. with an all-gather over NCCL).  Writes out [B, n_q, H, d_v] and, if
 *   non-NULL, lse [B, n_q, H].  bf16 with d_c = 512 (and d_v = 128 when w_uv
 *   is given) and 16-byte aligned buffers: one kernel merges the rows,
 *   rounds them to bf16 as mla_decode does, and applies W_UV on the tensor
 *   cores; other shapes merge in fp32 on CUDA cores (two kernels).
 */
MLA_API int mla_merge_workspace_size(const mla_dims *dims, int B, int n_q, int n_parts, size_t *bytes);
MLA_API int mla_merge_partials(const mla_dims *dims, int B, int n_q, int n_parts, const void *o_lat_parts,
                               const float *lse_parts, const void *w_uv, void *out, float *lse, void *workspace,
                               size_t ws_bytes, mla_stream_t stream);

/*
 * mla_fold_query_weights / mla_fold_output_weights — the offline folds of the
 *   fully absorbed decode.
 *   "DeepSeek-V3 解读 1: MLA", section "为什么需要解耦 RoPE": W^UK can be absorbed
 *   into the query projection, W_UQK^(s) = W_UQ^(s) W_UK^(s)T [d_cq x d_c], so the
 *   query latent c_Q maps straight to the latent query.  "Transformer升级之路：
 *   21", section 键值共享: the c -> v map is absorbed on the W_o side,
 *   W_UVO^(s) = W_UV^(s) W_O^(s) [d_c x D], with W_O^(s) the d_v rows of the
 *   output projection W^O [H d_v, D] that belong to head s.
 *   w_uq [d_cq, H, d_nope], w_uk [H, d_c, d_nope] -> w_uqk [H, d_cq, d_c];
 *   w_uv [H, d_c, d_v], w_o [H d_v, D] -> w_uvo [H, d_c, D]; dims->dtype,
 *   fp32 accumulation, rounded once.  CUDA cores (run once per model).
 *   Note the sizes: at V3 shapes (d_cq 1536, H 128, d_c 512, D 7168) the folded
 *   W_UQK holds 201 MB and W_UVO 940 MB, against 67 MB for W_UQ and W_UK and
 *   134 MB for W_UV and W^O: folding trades the per-step W_UK / W_UV products
 *   for larger weights.
 */
MLA_API int mla_fold_query_weights(const mla_dims *dims, int d_cq, const void *w_uq, const void *w_uk, void *w_uqk,
                                   mla_stream_t stream);
MLA_API int mla_fold_output_weights(const mla_dims *dims, const void *w_uv, const void *w_o, void *w_uvo,
                                    mla_stream_t stream);

/*
 * mla_decode_absorbed_workspace_size / mla_decode_absorbed — one decode step of
 *   the attention block from the hidden states, in the fully absorbed form:
 *   c_Q = h W_DQ ("DeepSeek-V3 解读 1: MLA", section "MLA：高层次的思路": queries
 *   are compressed to a latent too), q_lat^(s) = c_Q W_UQK^(s),
 *   q_pe^(s) = RoPE(c_Q W_QR^(s), seqlens[b] - n_q + j), the split-KV attention
 *   of mla_decode over the latent cache, and u = sum_s o_lat^(s) W_UVO^(s).
 *   h [B, n_q, D], w_dq [D, d_cq], w_uqk [H, d_cq, d_c] and w_uvo [H, d_c, D]
 *   (from the folds above), w_qr [d_cq, H, d_R]; cache, seqlens, lse as
 *   mla_decode.  Writes out [B, n_q, D] (dims->dtype; D = dims->d_model).
 *   The four products run on CUDA cores; the attention on the same kernels as
 *   mla_decode.  c_Q, the queries and o_lat are rounded to dims->dtype between
 *   the steps.
 */
MLA_API int mla_decode_absorbed_workspace_size(const mla_dims *dims, int d_cq, int B, int n_q, int max_seqlen,
                                               size_t *bytes);
MLA_API int mla_decode_absorbed(const mla_dims *dims, int d_cq, int B, int n_q, const void *h, const void *w_dq,
                                const void *w_uqk, const void *w_qr, const void *c_kv, const void *k_pe,
                                const int32_t *block_table, int max_blocks_per_seq, int num_blocks,
                                const int32_t *seqlens, int max_seqlen, const void *w_uvo, void *out, float *lse,
                                void *workspace, size_t ws_bytes, int *dev_status, mla_stream_t stream);

/*
 * mla_decode_sparse_workspace_size — scratch bytes of mla_decode_sparse for B
 *   sequences of n_q query tokens with lists of topk entries.
 */
MLA_API int mla_decode_sparse_workspace_size(const mla_dims *dims, int B, int n_q, int topk, size_t *bytes);

/*
 * mla_decode_sparse — the decode of mla_decode restricted, per query token, to a
 *   selected subset of its sequence's cached tokens.
 *   The MQA-mode MLA that V3.2 moved to (developer.cloud.tencent.com search
 *   results for "MLA", the snippet "MHA版MLA VS MQA版MLA": every head attends to
 *   the one shared latent key/value), with the attended tokens chosen per query
 *   token by the caller (the selection itself is not computed here).
 *   topk_idx [B, n_q, topk] (int32, device): the token indices query token j of
 *   sequence b attends to.  -1 is padding.  Every other entry must lie in
 *   0 .. seqlens[b] - n_q + j (the query's causal limit) and its block id in
 *   [0, num_blocks); entries that do not are reported as MLA_ERR_BAD_INDEX and
 *   skipped.  The valid entries are attended to as listed (softmax over the
 *   list, no deduplication); a query token with none reports MLA_ERR_BAD_INDEX
 *   and gets zeros.  The query's RoPE position is its own, seqlens[b] - n_q + j.
 *   Other arguments and outputs as mla_decode.  workspace: >=
 *   mla_decode_sparse_workspace_size bytes, 256-byte aligned; it holds the
 *   gathered rows (topk rows per query token, rounded up to 64).
 */
MLA_API int mla_decode_sparse(const mla_dims *dims, int B, int n_q, const void *q_nope, const void *q_pe,
                              const void *c_kv, const void *k_pe, const int32_t *block_table, int max_blocks_per_seq,
                              int num_blocks, const int32_t *seqlens, int max_seqlen, const int32_t *topk_idx,
                              int topk, const void *w_uk, const void *w_uv, void *out, float *lse, void *workspace,
                              size_t ws_bytes, int *dev_status, mla_stream_t stream);

/*
 * mla_prefill_workspace_size — scratch bytes of mla_prefill for total_tokens
 *   query tokens in B sequences of at most max_seqlen tokens.
 */
MLA_API int mla_prefill_workspace_size(const mla_dims *dims, int B, int total_tokens, int max_seqlen,
                               size_t *bytes);

/*
 * mla_prefill — causal prefill in the decompressed multi-head form.
 *   Same page, section 双重投影, training/prefill column: per head
 *   k_i = [c_i W_UK^(s) | kpe_i] (width d_nope + d_R), v_i = c_i W_UV^(s) (d_v),
 *   o_t = softmax_{i<=t}(scale * q_t . k_i) v.
 *   cu_seqlens [B+1] (int32, device): sequence b owns query rows
 *   cu_seqlens[b] .. cu_seqlens[b+1]-1, its token t at position t; its cache
 *   (already appended) holds tokens 0 .. len-1.  q_nope [total, H, d_nope],
 *   q_pe [total, H, d_R] (not rotated).  Writes out [total, H, d_v] and, if
 *   non-NULL, lse [total, H].
 */
MLA_API int mla_prefill(const mla_dims *dims, int B, const int32_t *cu_seqlens, int max_seqlen,
                int total_tokens, const void *q_nope, const void *q_pe, const void *c_kv,
                const void *k_pe, const int32_t *block_table, int max_blocks_per_seq,
                int num_blocks, const void *w_uk, const void *w_uv, void *out, float *lse,
                void *workspace, size_t ws_bytes, int *dev_status, mla_stream_t stream);

/*
 * mla_decode_launches — how many kernels one mla_decode call launches for this
 *   shape (query absorption, attention, and the combine: on the tensor-core
 *   path one kernel that merges the split partials and applies W_UV, on the
 *   CUDA-core path one kernel); for launch accounting in profilers and
 *   benchmarks.
 *   Writes *count; no device work.
 */
MLA_API int mla_decode_launches(const mla_dims *dims, int n_q, int *count);

/*
 * mla_decode_path — which kernels mla_decode / mla_decode_attention run for
 *   this shape: MLA_PATH_TCGEN05 (the tensor-core split-KV kernel and its
 *   combine: bf16, d_c 512, d_R 64, d_v 128, 64-token-multiple pages,
 *   n_q * H <= 256) or MLA_PATH_CUDA_CORES (fp32 and every other shape).
 *   Host-side logic only; no device work.  Writes *path.
 */
#define MLA_PATH_CUDA_CORES 0
#define MLA_PATH_TCGEN05 1
MLA_API int mla_decode_path(const mla_dims *dims, int n_q, int *path);

/*
 * mla_cache_pack / mla_cache_unpack — convert a latent pool between the row
 *   layout and the tiled page layout (see "Paged latent cache" above).
 *   rows: [num_rows, d_c + d_R] bf16, row-major (c_KV then the RoPE key);
 *   tiled: num_rows / 64 pages.  num_rows must be a multiple of 64; dims->dtype
 *   must be MLA_BF16 and d_c + d_R a multiple of 64.  The two buffers must not
 *   overlap.  Pure data movement: unpack(pack(x)) == x bit for bit.
 */
MLA_API int mla_cache_pack(const mla_dims *dims, const void *rows, void *tiled, int64_t num_rows,
                           mla_stream_t stream);
MLA_API int mla_cache_unpack(const mla_dims *dims, const void *tiled, void *rows, int64_t num_rows,
                             mla_stream_t stream);

/*
 * mla_wait_selftest — exercise the bounded device wait used by every
 *   tensor-core kernel of this library.  One thread waits on a barrier that
 *   nothing completes; after limit_ns nanoseconds of device time
 *   (globaltimer) it gives up, writes MLA_ERR_TIMEOUT into *dev_status (if it
 *   still holds MLA_OK) and exits normally.  It causes no fault and leaves
 *   the context usable.  This is a diagnostic with no counterpart on the
 *   pages.
 *   limit_ns: 1 .. 10^10.  dev_status: device int, required.
 *   Returns MLA_ERR_INVALID_ARG for a bad limit or a NULL status, MLA_ERR_CUDA
 *   if the launch fails, else MLA_OK (asynchronous; read *dev_status after a
 *   synchronisation).
 */
MLA_API int mla_wait_selftest(long long limit_ns, int *dev_status, mla_stream_t stream);

/* Human-readable text of an mla_status value (static storage). */
MLA_API const char *mla_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* MLA_H_ */
