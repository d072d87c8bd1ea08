// Library-internal declarations shared by the C-ABI layer and the kernels.
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda_runtime.h>

#include "../../include/attn.h"

namespace attn {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// Bounded waits: clock64 cycles before a pipeline wait gives up (~0.5 s at
// the B200's boost clock). Read per call from ATTN_WAIT_BUDGET_CYCLES when set.
long long wait_budget_cycles();
// Waits that drain in-flight copies and MMAs before a CTA exits use their own,
// larger bound, so that a short pipeline budget never cuts a drain short.
constexpr long long kDrainBudgetCycles = 4000000000LL;

// The driver's cuTensorMapEncodeTiled, looked up once through the runtime
// (no link against libcuda); nullptr when unavailable.
void* tensor_map_encode_fn();

struct DecodePlan {
  int chunk;        // tokens per split (multiple of 16, at most 16 * kDecodeMaxChunkSubs)
  int splits;       // ceil(planning length / chunk)
  int cta_rows;     // query heads a split CTA covers: 16, or 32 (warp pairs) when 16 < Hq / Hkv
  int hchunks;      // split CTAs per (sequence, K/V head, split): ceil(Hq / Hkv / cta_rows)
  int merge_in_launch;  // 1: every partial of a row fits one CTA's staging (the last CTA merges)
  int dyn;          // 1: few (sequence, K/V head) units, whole waves: grains handed out at run time
};
// Split plan constants: resident decode CTAs of 16 query heads per SM (two
// fit in shared memory at d = 128; one CTA of 32 heads takes both places), the
// most 16-token sub-blocks per split, and the partials one merge staging holds
// for one query-head row (divided by the rows merged).
constexpr int kDecodeCtasPerSm = 2;
constexpr int kDecodeMaxChunkSubs = 256;
constexpr int kDecodeMergeSlots = 192;

int plan_decode(int B, int Hq, int Hkv, int max_seq_len, int num_sms, DecodePlan* out);
// Length the split plan is made for: max_seq_len without a window, else the
// most tokens a windowed query's visible sub-block list can span.
int decode_plan_length(int max_seq_len, int window, int n_sink);
// Workspace: partial outputs [B, Hq, splits, d] fp32, partial LSEs
// [B, Hq, splits] fp32, then (16-byte aligned) the merge's ticket counter and
// the grain counter, two uint64 per (sequence, K/V head, head chunk).
struct DecodeWorkspace {
  size_t o_part_offset, lse_part_offset, counters_offset, bytes;
};
DecodeWorkspace decode_workspace_layout(int B, int Hq, int Hkv, int d, const DecodePlan& plan);
size_t decode_workspace_bytes(int B, int Hq, int Hkv, int d, const DecodePlan& plan);

// Kernel launchers (defined next to their kernels). Return cudaError_t.
// window 0 = every cached token visible (n_sink must then be 0); sinks may be nullptr.
cudaError_t launch_decode(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_table,
                          const int32_t* seq_lens, const float* sinks, void* o, float* lse, int B, int Hq, int Hkv,
                          int d, int num_blocks, int block_size, int max_blocks_per_seq, int max_seq_len, int window,
                          int n_sink, float scale, void* workspace, const DecodePlan& plan, int32_t* status,
                          cudaStream_t stream);

cudaError_t launch_paged_gather(const void* cache, const int32_t* block_table, const int32_t* seq_lens, void* out,
                                int B, int Hkv, int d, int num_blocks, int block_size, int max_blocks_per_seq,
                                int max_seq_len, int32_t* status, cudaStream_t stream);

// Returns ATTN_OK / ATTN_ERR_CUDA (tensor-map encoding or launch failure).
int launch_prefill(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int N,
                   int d, int mask_kind, int window, float scale, int32_t* status, cudaStream_t stream);

// Prefill of the newest Nq positions of each sequence against its paged context.
// Absorbed MLA decode: split kernel + log-sum-exp merge (mla_sm100.cu).
struct MlaPlan {
  int chunk;   // tokens per split (multiple of 128)
  int splits;  // ceil(max_seq_len / chunk)
};
int plan_mla(int B, int H, int max_seq_len, int num_sms, MlaPlan* out);
size_t mla_workspace_bytes(int B, int H, const MlaPlan& plan);
int launch_mla_decode(const void* q, const void* cache, const int32_t* block_table, const int32_t* seq_lens, void* o,
                      float* lse, int B, int H, int num_blocks, int block_size, int max_blocks_per_seq,
                      int max_seq_len, float scale, void* workspace, const MlaPlan& plan, int32_t* status,
                      cudaStream_t stream);
// The split-merge kernel of the paged decode, for head widths 64, 128 and 512.
// after_split_grid: launched right after a decode split grid that let its
// dependents launch early (programmatic dependent launch). all_splits: every
// split wrote a partial (the decode's run-time grains), not just the splits
// that hold the sequence's sub-blocks.
cudaError_t launch_decode_merge(const float* o_part, const float* lse_part, const int32_t* seq_lens,
                                const float* sinks, void* o, float* lse, int B, int Hq, int d, int splits, int chunk,
                                int max_seq_len, int window, int n_sink, int32_t* status, cudaStream_t stream,
                                bool after_split_grid = false, bool all_splits = false);

// Backward pass (backward_sm100.cu): workspace = D = rowsum(dO * O), fp32 [B, Hq, N].
size_t backward_workspace_bytes(int B, int Hq, int N);
int launch_backward(const void* q, const void* k, const void* v, const void* o, const void* d_o, const float* lse,
                    void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int N, int d, int mask_kind, int window,
                    float scale, void* workspace, int32_t* status, cudaStream_t stream);

int launch_prefill_paged(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_table,
                         const int32_t* seq_lens, void* o, float* lse, int B, int Hq, int Hkv, int Nq, int d,
                         int num_blocks, int block_size, int max_blocks_per_seq, int max_seq_len, int mask_kind,
                         int window, float scale, int32_t* status, cudaStream_t stream);

}  // namespace attn
