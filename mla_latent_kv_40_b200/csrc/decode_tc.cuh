// Tensor-core (tcgen05) split-KV decode over the latent cache: host interface.
#pragma once

#include "kernels.cuh"

namespace mla {

// True when the shape runs on the tcgen05 path (bf16, fused 576-wide rows, ...).
bool tc_decode_supported(const mla_dims &d, int n_q);
// Kernels the tcgen05 attention + combine launch per call.
int tc_decode_kernel_launches();
// Scratch bytes the tcgen05 path needs beyond the absorbed query buffer.
size_t tc_decode_workspace_bytes(const mla_dims &d, int B, int n_q);
// Split-KV attention from an absorbed query buffer; partials stay in ws.  Only keys in
// [kv_begin, kv_end) are read (kv_begin a multiple of 64); the full decode passes 0, INT_MAX.
int launch_tc_attention(const mla_dims &d, int B, int n_q, const void *q_abs, const CacheView &cache,
                        const int32_t *seqlens, int max_seqlen, void *ws, int *dev_status, cudaStream_t st,
                        int kv_begin, int kv_end);
// Merge of the partials, and the W_UV product in the same kernel when w_uv != NULL.
int launch_tc_combine(const mla_dims &d, int B, int n_q, const int32_t *seqlens, int max_seqlen, const void *w_uv,
                      void *out, float *lse, void *ws, int *dev_status, cudaStream_t st);
// True when stacked partials of this shape merge on the path below (bf16, d_c 512, d_v 128 with
// W_UV, 16-byte aligned rows).
bool tc_merge_parts_supported(const mla_dims &d, const void *o_parts, const void *w_uv, const void *out);
// Merge of n_parts stacked partials o_parts [n_parts][B*n_q*H][512] (+ W_UV when w_uv != NULL, in
// the same kernel).
int launch_tc_merge_parts(const mla_dims &d, int B, int n_q, int n_parts, const void *o_parts, const float *lse_parts,
                          const void *w_uv, void *out, float *lse, cudaStream_t st);

}  // namespace mla
