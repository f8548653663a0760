// Shared device helpers of libmla: element conversion, status reporting,
// paged-row addressing and the RoPE angle.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/mla.h"

namespace mla {

// ---- element types ---------------------------------------------------------
__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// ---- device-side error reporting -------------------------------------------
// First error wins: the word moves from 0 to the code once.
__device__ __forceinline__ void report(int *dev_status, int code) {
  if (dev_status) atomicCAS(dev_status, 0, code);
}

// ---- paged latent cache ----------------------------------------------------
// Row of token i of sequence b, or -1 if the block id is out of range.
__device__ __forceinline__ int64_t cache_row(const int32_t *block_table, int max_blocks_per_seq,
                                             int num_blocks, int block_size, int b, int i) {
  if (i < 0) return -1;
  const int lb = i / block_size;
  if (lb >= max_blocks_per_seq) return -1;
  const int blk = block_table ? block_table[(int64_t)b * max_blocks_per_seq + lb]
                              : b * max_blocks_per_seq + lb;
  if (blk < 0 || blk >= num_blocks) return -1;
  return (int64_t)blk * block_size + (i % block_size);
}

// ---- latent pool layouts -----------------------------------------------------
// Byte offset of element (row r, dim d) in a tiled pool whose rows are W
// elements wide: 64-token pages of W/64 chunks; chunk c = d / 64 holds token t
// at byte 128 t and its 16-byte group g = (d / 8) % 8 at 16 * (g ^ (t % 8)).
__host__ __device__ __forceinline__ int64_t tiled_byte_offset(int64_t r, int d, int W) {
  const int64_t page = r >> 6;
  const int t = (int)(r & 63);
  const int c = d >> 6, g = (d >> 3) & 7, e = d & 7;
  return page * (int64_t)W * 128 + (int64_t)c * 8192 + t * 128 + ((g ^ (t & 7)) << 4) + e * 2;
}

// Address of element (row r, dim d), d in [0, d_c + d_rope): c_KV dims first,
// then the RoPE key, in either pool layout.
template <typename T>
__device__ __forceinline__ T *latent_elem(void *c_kv, void *k_pe, int64_t ckv_stride, int64_t kpe_stride, int layout,
                                          int d_c, int W, int64_t r, int d) {
  if (layout == MLA_CACHE_TILED)
    return reinterpret_cast<T *>(static_cast<char *>(c_kv) + tiled_byte_offset(r, d, W));
  return d < d_c ? static_cast<T *>(c_kv) + r * ckv_stride + d : static_cast<T *>(k_pe) + r * kpe_stride + (d - d_c);
}

// ---- RoPE ------------------------------------------------------------------
// cos/sin of p * base^(-2i/d).  The angle is formed and reduced modulo 2*pi in
// double so that positions up to 2^31 keep full fp32 accuracy in the result.
// theta_i = base^(-2i / d_R), in double so that pos * theta_i keeps its fractional turns.
__device__ __forceinline__ double rope_theta(int pair, int d_rope, float base) {
  return pow((double)base, -2.0 * (double)pair / (double)d_rope);
}

__device__ __forceinline__ void rope_cos_sin_theta(int pos, double theta, float *c, float *s) {
  double a = (double)pos * theta;
  const double two_pi = 6.283185307179586476925286766559, inv_two_pi = 0.15915494309189533576888376337251;
  a = fma(-two_pi, floor(a * inv_two_pi), a);   // reduced to [0, 2*pi) up to one ulp of a at the ends
  float sf, cf;
  sincosf((float)a, &sf, &cf);
  *c = cf;
  *s = sf;
}

__device__ __forceinline__ void rope_cos_sin(int pos, int pair, int d_rope, float base, float *c,
                                             float *s) {
  rope_cos_sin_theta(pos, rope_theta(pair, d_rope, base), c, s);
}

__host__ __device__ inline float default_scale(const mla_dims &d) {
  return d.softmax_scale > 0.f ? d.softmax_scale : 1.0f / sqrtf((float)(d.d_nope + d.d_rope));
}

}  // namespace mla
