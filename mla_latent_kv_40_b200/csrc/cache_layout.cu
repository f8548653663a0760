// Conversion of the latent pool between the row layout and the tiled page
// layout (64-token pages of 8 KB chunks, 128-byte swizzled), 16 bytes at a time.
#include "kernels.cuh"

namespace mla {

__global__ void cache_convert_kernel(const uint4 *src, uint4 *dst, int64_t num_rows, int W, bool to_tiled) {
  const int groups = W / 8;                       // 16-byte groups per row
  const int64_t n = num_rows * groups;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = e / groups;
    const int q = (int)(e % groups);
    const int64_t tiled = tiled_byte_offset(r, 8 * q, W) / 16;
    if (to_tiled) dst[tiled] = src[e];
    else dst[e] = src[tiled];
  }
}

int launch_cache_convert(const void *src, void *dst, int64_t num_rows, int W, bool to_tiled, cudaStream_t st) {
  if (num_rows <= 0) return MLA_OK;
  cache_convert_kernel<<<1184, 256, 0, st>>>(static_cast<const uint4 *>(src), static_cast<uint4 *>(dst), num_rows, W,
                                             to_tiled);
  return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

}  // namespace mla
