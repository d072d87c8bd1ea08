// The extern "C" boundary: argument validation, the decode split plan and
// dispatch to the kernels. Nothing here allocates device memory.

#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <mutex>

#include "internal.h"

namespace attn {

void* tensor_map_encode_fn() {
  static void* fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = f;
  });
  return fn;
}

long long wait_budget_cycles() {
  const char* s = std::getenv("ATTN_WAIT_BUDGET_CYCLES");
  const long long v = s ? std::atoll(s) : 0;
  return v > 0 ? v : 1000000000LL;
}

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int current_sm_count(int* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_CUDA;
  if (cudaDeviceGetAttribute(out, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return ATTN_ERR_CUDA;
  return ATTN_OK;
}

}  // namespace
}  // namespace attn

using namespace attn;

extern "C" {

int attn_version(void) { return 100; }

const char* attn_status_string(int status) {
  switch (status) {
    case ATTN_OK:
      return "ok";
    case ATTN_ERR_INVALID_ARG:
      return "invalid argument";
    case ATTN_ERR_UNSUPPORTED:
      return "unsupported configuration (head dimension must be 64 or 128)";
    case ATTN_ERR_CUDA:
      return "CUDA runtime or driver call failed";
    case ATTN_ERR_DEVICE_CHECK:
      return "device check failed: block-table entry or seq_len out of range";
    case ATTN_ERR_TIMEOUT:
      return "a bounded pipeline wait expired";
    case ATTN_ERR_WORKSPACE:
      return "workspace missing or too small";
    default:
      return "unknown status";
  }
}

int attn_prefill(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int N,
                 int d, int mask_kind, int window, float scale, int32_t* status, attn_stream_t stream) {
  if (!q || !k || !v || !o) return ATTN_ERR_INVALID_ARG;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || N <= 0 || d <= 0) return ATTN_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return ATTN_ERR_INVALID_ARG;
  if (mask_kind != ATTN_MASK_FULL && mask_kind != ATTN_MASK_CAUSAL && mask_kind != ATTN_MASK_SLIDING_WINDOW)
    return ATTN_ERR_INVALID_ARG;
  if (mask_kind == ATTN_MASK_SLIDING_WINDOW && window < 1) return ATTN_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return ATTN_ERR_INVALID_ARG;
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  // TMA coordinates and the persistent kernel's item indices are int32
  if (static_cast<long long>(B) * Hq * N > (1LL << 31) - 1) return ATTN_ERR_UNSUPPORTED;
  if (mask_kind == ATTN_MASK_SLIDING_WINDOW && window >= N) mask_kind = ATTN_MASK_CAUSAL;
  return launch_prefill(q, k, v, o, lse, B, Hq, Hkv, N, d, mask_kind, window, scale, status,
                        reinterpret_cast<cudaStream_t>(stream));
}

int attn_prefill_paged(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_table,
                       const int32_t* seq_lens, void* o, float* lse, int B, int Hq, int Hkv, int Nq, int d,
                       int num_blocks, int block_size, int max_blocks_per_seq, int max_seq_len, int mask_kind,
                       int window, float scale, int32_t* status, attn_stream_t stream) {
  if (!q || !k_cache || !v_cache || !block_table || !seq_lens || !o) return ATTN_ERR_INVALID_ARG;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Nq <= 0 || d <= 0 || num_blocks <= 0 || block_size <= 0 ||
      max_blocks_per_seq <= 0 || max_seq_len < Nq)
    return ATTN_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return ATTN_ERR_INVALID_ARG;
  if (static_cast<long long>(max_blocks_per_seq) * block_size < max_seq_len) return ATTN_ERR_INVALID_ARG;
  if (mask_kind != ATTN_MASK_FULL && mask_kind != ATTN_MASK_CAUSAL && mask_kind != ATTN_MASK_SLIDING_WINDOW)
    return ATTN_ERR_INVALID_ARG;
  if (mask_kind == ATTN_MASK_SLIDING_WINDOW && window < 1) return ATTN_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o)) return ATTN_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(block_table) & 3u) || (reinterpret_cast<uintptr_t>(seq_lens) & 3u))
    return ATTN_ERR_INVALID_ARG;
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (block_size != 16 && block_size != 32 && block_size != 64 && block_size != 128) return ATTN_ERR_UNSUPPORTED;
  if (static_cast<long long>(B) * Hq * Nq > (1LL << 31) - 1) return ATTN_ERR_UNSUPPORTED;
  if (mask_kind == ATTN_MASK_SLIDING_WINDOW && window >= max_seq_len) mask_kind = ATTN_MASK_CAUSAL;
  return launch_prefill_paged(q, k_cache, v_cache, block_table, seq_lens, o, lse, B, Hq, Hkv, Nq, d, num_blocks,
                              block_size, max_blocks_per_seq, max_seq_len, mask_kind, window, scale, status,
                              reinterpret_cast<cudaStream_t>(stream));
}

int attn_decode_plan(int B, int Hq, int Hkv, int max_seq_len, int num_sms, int* chunk_tokens, int* num_splits) {
  DecodePlan plan;
  const int rc = plan_decode(B, Hq, Hkv, max_seq_len, num_sms, &plan);
  if (rc != ATTN_OK) return rc;
  if (chunk_tokens) *chunk_tokens = plan.chunk;
  if (num_splits) *num_splits = plan.splits;
  return ATTN_OK;
}

}  // extern "C"

namespace {

// Workspace bytes of a (possibly windowed) decode, 0 for invalid sizes.
size_t decode_bytes(int B, int Hq, int Hkv, int d, int max_seq_len, int block_size, int window, int n_sink) {
  if (d != 64 && d != 128) return 0;
  if (block_size <= 0 || block_size % 16 != 0) return 0;
  if (window < 0 || n_sink < 0 || max_seq_len <= 0) return 0;
  int sms = 0;
  if (current_sm_count(&sms) != ATTN_OK) return 0;
  DecodePlan plan;
  if (plan_decode(B, Hq, Hkv, decode_plan_length(max_seq_len, window, n_sink), sms, &plan) != ATTN_OK) return 0;
  return decode_workspace_bytes(B, Hq, Hkv, d, plan);
}

int decode_common(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_table,
                  const int32_t* seq_lens, const float* sinks, void* o, float* lse, int B, int Hq, int Hkv, int d,
                  int num_blocks, int block_size, int max_blocks_per_seq, int max_seq_len, int window, int n_sink,
                  float scale, void* workspace, size_t workspace_bytes, int32_t* status, attn_stream_t stream) {
  if (!q || !k_cache || !v_cache || !block_table || !seq_lens || !o) return ATTN_ERR_INVALID_ARG;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || d <= 0 || num_blocks <= 0 || block_size <= 0 || max_blocks_per_seq <= 0 ||
      max_seq_len <= 0)
    return ATTN_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return ATTN_ERR_INVALID_ARG;
  if (static_cast<long long>(max_blocks_per_seq) * block_size < max_seq_len) return ATTN_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;
  // sinks: the first n_sink positions, only beside a finite window, 0 <= n_sink <= n
  if (window < 0 || n_sink < 0 || n_sink > max_seq_len || (n_sink > 0 && window == 0)) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o)) return ATTN_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(block_table) & 3u) || (reinterpret_cast<uintptr_t>(seq_lens) & 3u))
    return ATTN_ERR_INVALID_ARG;
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return ATTN_ERR_INVALID_ARG;
  if (sinks && (reinterpret_cast<uintptr_t>(sinks) & 3u)) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (block_size % 16 != 0) return ATTN_ERR_UNSUPPORTED;
  if (B > 65535 || static_cast<long long>(Hkv) * ((Hq / Hkv + 15) / 16) > 65535) return ATTN_ERR_UNSUPPORTED;
  // a window that covers every position hides nothing: the sink positions are inside it
  if (window >= max_seq_len) window = n_sink = 0;
  int sms = 0;
  if (current_sm_count(&sms) != ATTN_OK) return ATTN_ERR_CUDA;
  DecodePlan plan;
  if (plan_decode(B, Hq, Hkv, decode_plan_length(max_seq_len, window, n_sink), sms, &plan) != ATTN_OK)
    return ATTN_ERR_INVALID_ARG;
  if (!workspace || !aligned16(workspace) || workspace_bytes < decode_workspace_bytes(B, Hq, Hkv, d, plan))
    return ATTN_ERR_WORKSPACE;
  const cudaError_t e = launch_decode(q, k_cache, v_cache, block_table, seq_lens, sinks, o, lse, B, Hq, Hkv, d,
                                      num_blocks, block_size, max_blocks_per_seq, max_seq_len, window, n_sink, scale,
                                      workspace, plan, status, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // namespace

extern "C" {

size_t attn_decode_workspace_bytes(int B, int Hq, int Hkv, int d, int max_seq_len, int block_size) {
  return decode_bytes(B, Hq, Hkv, d, max_seq_len, block_size, 0, 0);
}

size_t attn_decode_window_workspace_bytes(int B, int Hq, int Hkv, int d, int max_seq_len, int block_size, int window,
                                          int n_sink) {
  if (window >= max_seq_len) window = n_sink = 0;
  return decode_bytes(B, Hq, Hkv, d, max_seq_len, block_size, window, n_sink);
}

int attn_decode_paged(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_table,
                      const int32_t* seq_lens, void* o, float* lse, int B, int Hq, int Hkv, int d,
                      int num_blocks, int block_size, int max_blocks_per_seq, int max_seq_len, float scale,
                      void* workspace, size_t workspace_bytes, int32_t* status, attn_stream_t stream) {
  return decode_common(q, k_cache, v_cache, block_table, seq_lens, nullptr, o, lse, B, Hq, Hkv, d, num_blocks,
                       block_size, max_blocks_per_seq, max_seq_len, 0, 0, scale, workspace, workspace_bytes, status,
                       stream);
}

int attn_decode_paged_window(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_table,
                             const int32_t* seq_lens, const float* sinks, void* o, float* lse, int B, int Hq, int Hkv,
                             int d, int num_blocks, int block_size, int max_blocks_per_seq, int max_seq_len,
                             int window, int n_sink, float scale, void* workspace, size_t workspace_bytes,
                             int32_t* status, attn_stream_t stream) {
  return decode_common(q, k_cache, v_cache, block_table, seq_lens, sinks, o, lse, B, Hq, Hkv, d, num_blocks,
                       block_size, max_blocks_per_seq, max_seq_len, window, n_sink, scale, workspace,
                       workspace_bytes, status, stream);
}

size_t attn_prefill_backward_workspace_bytes(int B, int Hq, int N) {
  if (B <= 0 || Hq <= 0 || N <= 0) return 0;
  return backward_workspace_bytes(B, Hq, N);
}

int attn_prefill_backward(const void* q, const void* k, const void* v, const void* o, const void* d_o,
                          const float* lse, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int N, int d,
                          int mask_kind, int window, float scale, void* workspace, size_t workspace_bytes,
                          int32_t* status, attn_stream_t stream) {
  if (!q || !k || !v || !o || !d_o || !lse || !dq || !dk || !dv) return ATTN_ERR_INVALID_ARG;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || N <= 0 || d <= 0) return ATTN_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return ATTN_ERR_INVALID_ARG;
  if (mask_kind != ATTN_MASK_FULL && mask_kind != ATTN_MASK_CAUSAL && mask_kind != ATTN_MASK_SLIDING_WINDOW)
    return ATTN_ERR_INVALID_ARG;
  if (mask_kind == ATTN_MASK_SLIDING_WINDOW && window < 1) return ATTN_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(d_o) || !aligned16(dq) ||
      !aligned16(dk) || !aligned16(dv) || (reinterpret_cast<uintptr_t>(lse) & 3u))
    return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (B > 65535 || Hq > 65535 || static_cast<long long>(B) * Hq * N > (1LL << 31) - 1) return ATTN_ERR_UNSUPPORTED;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 15u) ||
      workspace_bytes < backward_workspace_bytes(B, Hq, N))
    return ATTN_ERR_WORKSPACE;
  if (mask_kind == ATTN_MASK_SLIDING_WINDOW && window >= N) mask_kind = ATTN_MASK_CAUSAL;
  return launch_backward(q, k, v, o, d_o, lse, dq, dk, dv, B, Hq, Hkv, N, d, mask_kind, window, scale, workspace,
                         status, reinterpret_cast<cudaStream_t>(stream));
}

size_t attn_mla_decode_workspace_bytes(int B, int H, int d_latent, int d_rope, int max_seq_len) {
  if (d_latent != 512 || d_rope != 64) return 0;
  int sms = 0;
  if (current_sm_count(&sms) != ATTN_OK) return 0;
  MlaPlan plan;
  if (plan_mla(B, H, max_seq_len, sms, &plan) != ATTN_OK) return 0;
  return mla_workspace_bytes(B, H, plan);
}

int attn_mla_decode_paged(const void* q, const void* cache, const int32_t* block_table, const int32_t* seq_lens,
                          void* o, float* lse, int B, int H, int d_latent, int d_rope, int num_blocks, int block_size,
                          int max_blocks_per_seq, int max_seq_len, float scale, void* workspace,
                          size_t workspace_bytes, int32_t* status, attn_stream_t stream) {
  if (!q || !cache || !block_table || !seq_lens || !o) return ATTN_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0 || d_latent <= 0 || d_rope <= 0 || num_blocks <= 0 || block_size <= 0 ||
      max_blocks_per_seq <= 0 || max_seq_len <= 0)
    return ATTN_ERR_INVALID_ARG;
  if (static_cast<long long>(max_blocks_per_seq) * block_size < max_seq_len) return ATTN_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(cache) || !aligned16(o)) return ATTN_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(block_table) & 3u) || (reinterpret_cast<uintptr_t>(seq_lens) & 3u))
    return ATTN_ERR_INVALID_ARG;
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return ATTN_ERR_INVALID_ARG;
  if (d_latent != 512 || d_rope != 64) return ATTN_ERR_UNSUPPORTED;
  if (block_size != 16 && block_size != 32 && block_size != 64 && block_size != 128) return ATTN_ERR_UNSUPPORTED;
  if (B > 65535 || (H + 63) / 64 > 65535) return ATTN_ERR_UNSUPPORTED;
  int sms = 0;
  if (current_sm_count(&sms) != ATTN_OK) return ATTN_ERR_CUDA;
  MlaPlan plan;
  if (plan_mla(B, H, max_seq_len, sms, &plan) != ATTN_OK) return ATTN_ERR_INVALID_ARG;
  if (!workspace || !aligned16(workspace) || workspace_bytes < mla_workspace_bytes(B, H, plan))
    return ATTN_ERR_WORKSPACE;
  return launch_mla_decode(q, cache, block_table, seq_lens, o, lse, B, H, num_blocks, block_size,
                           max_blocks_per_seq, max_seq_len, scale, workspace, plan, status,
                           reinterpret_cast<cudaStream_t>(stream));
}

int attn_paged_gather(const void* cache, const int32_t* block_table, const int32_t* seq_lens, void* out, int B,
                      int Hkv, int d, int num_blocks, int block_size, int max_blocks_per_seq, int max_seq_len,
                      int32_t* status, attn_stream_t stream) {
  if (!cache || !block_table || !seq_lens || !out) return ATTN_ERR_INVALID_ARG;
  if (B <= 0 || Hkv <= 0 || d <= 0 || num_blocks <= 0 || block_size <= 0 || max_blocks_per_seq <= 0 ||
      max_seq_len <= 0)
    return ATTN_ERR_INVALID_ARG;
  if (static_cast<long long>(max_blocks_per_seq) * block_size < max_seq_len) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(cache) || !aligned16(out)) return ATTN_ERR_INVALID_ARG;
  if (d % 8 != 0) return ATTN_ERR_UNSUPPORTED;
  const cudaError_t e = launch_paged_gather(cache, block_table, seq_lens, out, B, Hkv, d, num_blocks, block_size,
                                            max_blocks_per_seq, max_seq_len, status,
                                            reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // extern "C"
