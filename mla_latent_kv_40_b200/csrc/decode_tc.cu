#include "decode_tc.cuh"

namespace mla {

bool tc_decode_supported(const mla_dims &, int) { return false; }
int tc_decode_kernel_launches() { return 2; }
size_t tc_decode_workspace_bytes(const mla_dims &, int, int) { return 0; }
int launch_tc_attention(const mla_dims &, int, int, const void *, const CacheView &, const int32_t *, int, void *,
                        int *, cudaStream_t) {
  return MLA_ERR_UNSUPPORTED;
}
int launch_tc_combine(const mla_dims &, int, int, const int32_t *, int, const void *, void *, float *, void *,
                      cudaStream_t) {
  return MLA_ERR_UNSUPPORTED;
}

}  // namespace mla
