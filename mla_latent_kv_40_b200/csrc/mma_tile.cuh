// Warp-level bf16 tensor-core tiles (mma.sync m16n8k16, fp32 accumulation)
// for the small projections around the attention kernel: the append
// down-projection, the W_UK query absorption and the W_UV up-projection.
// These are weight-streaming GEMMs whose time is the weight read; warp-level
// MMAs keep them off the CUDA cores without tying up tensor memory.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace mla {
namespace mma {

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// 16-byte asynchronous global -> shared copy (zero-filled when !valid).
__device__ __forceinline__ void cp16(void *dst, const void *src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_addr(dst)), "l"(src),
               "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Four 8x8 b16 matrices; lane i supplies the address of row i % 8 of matrix i / 8.
__device__ __forceinline__ void ldsm_x4(const void *p, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(smem_addr(p)));
}
__device__ __forceinline__ void ldsm_x4_t(const void *p, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(smem_addr(p)));
}

// D += A (16x16, row-major) * B (16x8, column-major), bf16 in, fp32 accumulate.
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// A fragment of rows r0..r0+15, cols k0..k0+15 of a row-major smem tile (ld elements per row).
__device__ __forceinline__ void load_a(const __nv_bfloat16 *tile, int ld, int r0, int k0, uint32_t (&a)[4]) {
  const int lane = threadIdx.x & 31;
  const __nv_bfloat16 *p = tile + (r0 + (lane & 7) + 8 * ((lane >> 3) & 1)) * ld + k0 + 8 * (lane >> 4);
  ldsm_x4(p, a[0], a[1], a[2], a[3]);
}

// B fragments of two n8 tiles (n0..n0+15) over k0..k0+15.
// kn: the smem tile is [K][N] (N contiguous); otherwise it is [N][K] (K contiguous).
__device__ __forceinline__ void load_b2(const __nv_bfloat16 *tile, int ld, int k0, int n0, bool kn, uint32_t (&b)[4]) {
  const int lane = threadIdx.x & 31;
  if (kn) {
    const __nv_bfloat16 *p = tile + (k0 + (lane & 7) + 8 * ((lane >> 3) & 1)) * ld + n0 + 8 * (lane >> 4);
    ldsm_x4_t(p, b[0], b[1], b[2], b[3]);
  } else {
    const __nv_bfloat16 *p = tile + (n0 + (lane & 7) + 8 * (lane >> 4)) * ld + k0 + 8 * ((lane >> 3) & 1);
    ldsm_x4(p, b[0], b[1], b[2], b[3]);
  }
}

}  // namespace mma
}  // namespace mla
