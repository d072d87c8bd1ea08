// attn_decode_paged_noalloc: the paged decode for callers that cannot
// allocate device memory. Its split partials live in a file-scope static
// device array instead of a caller workspace; the kernels are those of
// attn_decode_paged, reached through that entry point.

#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>
#include <mutex>

#include "internal.h"

// ----------------------------------------------------------------------------
// Decode without a caller workspace: the split partials live in a static
// device array. In host code `g_decode_scratch` names a host-side stand-in,
// not device memory, so its device address is looked up once per device
// (with that device current) and passed to the kernels as a plain pointer.
// ----------------------------------------------------------------------------
static __device__ __align__(256) unsigned char g_decode_scratch[ATTN_DECODE_NOALLOC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void* g_scratch_addr[kMaxDevices] = {};

int scratch_for_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return ATTN_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr) return ATTN_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return ATTN_OK;
}
}  // namespace

extern "C" ATTN_API int attn_decode_paged_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                                  const int32_t* block_table, const int32_t* seq_lens, void* o,
                                                  float* lse, int B, int Hq, int Hkv, int d, int num_blocks,
                                                  int block_size, int max_blocks_per_seq, int max_seq_len,
                                                  float scale, int32_t* status, attn_stream_t stream) {
  void* scratch = nullptr;
  const int rc = scratch_for_current_device(&scratch);
  if (rc != ATTN_OK) return rc;
  // Same validation and kernels as attn_decode_paged; a request that needs more
  // than the static array gets ATTN_ERR_WORKSPACE before any launch.
  return attn_decode_paged(q, k_cache, v_cache, block_table, seq_lens, o, lse, B, Hq, Hkv, d, num_blocks,
                           block_size, max_blocks_per_seq, max_seq_len, scale, scratch,
                           static_cast<size_t>(ATTN_DECODE_NOALLOC_SCRATCH_BYTES), status, stream);
}
