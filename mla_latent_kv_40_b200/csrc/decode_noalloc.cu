// mla_decode_noalloc: mla_decode with library-owned static scratch, for
// callers that cannot allocate device memory (see include/mla.h).
//
// The scratch is one file-scope __device__ array.  In host code its name is
// only a host-side stand-in, not a device address, so each device's address is
// looked up once with cudaGetSymbolAddress (that device current) and cached.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/mla.h"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[MLA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 128;
std::mutex g_mu;
void *g_scratch_addr[kMaxDevices];  // per device; nullptr until the first call there

int scratch_for_current_device(void **addr) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MLA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_addr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return MLA_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *addr = g_scratch_addr[dev];
  return MLA_OK;
}

}  // namespace

extern "C" int mla_decode_noalloc(const mla_dims *dims, int B, int n_q, const void *q_nope, const void *q_pe,
                                  const void *c_kv, const void *k_pe, const int32_t *block_table,
                                  int max_blocks_per_seq, int num_blocks, const int32_t *seqlens, int max_seqlen,
                                  const void *w_uk, const void *w_uv, void *out, float *lse, int *dev_status,
                                  mla_stream_t stream) {
  size_t need = 0;
  int rc = mla_decode_workspace_size(dims, B, n_q, max_seqlen, &need);
  if (rc) return rc;
  if (need > MLA_NOALLOC_SCRATCH_BYTES) return MLA_ERR_STATIC_WS;
  void *scratch = nullptr;
  if ((rc = scratch_for_current_device(&scratch))) return rc;
  return mla_decode(dims, B, n_q, q_nope, q_pe, c_kv, k_pe, block_table, max_blocks_per_seq, num_blocks, seqlens,
                    max_seqlen, w_uk, w_uv, out, lse, scratch, MLA_NOALLOC_SCRATCH_BYTES, dev_status, stream);
}
