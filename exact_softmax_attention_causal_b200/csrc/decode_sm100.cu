// Paged single-token decode: split-KV partials + log-sum-exp merge, and the
// bit-exact block-table gather.
//
// What it computes ("Module 09: Efficient Attention", "Code: A Paged KV Cache
// from Scratch"; "USAAIO Lesson 90", part 2): for every sequence b and query
// head h, softmax(scale * q_{b,h} . K_b^T) V_b over all seq_lens[b] cached
// tokens, where token t of sequence b lives in slot t % block_size of physical
// block block_table[b][t / block_size] of the pool
// [num_blocks, block_size, Hkv, d].
//
// How ("Inference attention" post, "FlashDecoding"): the sequence is cut into
// chunks of `chunk` tokens. One CTA handles one (chunk, K/V head, query-head
// chunk of <= 16, sequence). Its 4 warps each stream 16-token sub-blocks of
// K and V through a private 3-stage cp.async ring in shared memory (16-byte
// loads of whole 256-byte head rows), score the <= 16 query heads of the
// group against them with mma.sync m16n8k16 (bf16 in, fp32 accumulate), and
// keep FlashAttention's running (max, sum, output) per query head. With 17 to
// 32 query heads per K/V head (MQA) a CTA takes 32 heads with 8 warps: each
// pair of warps streams the sub-blocks through one shared 6-stage ring and
// scores 16 heads per warp, so the tiles are read once for all the heads.
// The warps combine in shared memory and write one normalised partial output
// and its log-sum-exp per (sequence, head, chunk). The CTA that finishes last among
// the chunks of a (sequence, K/V head, head chunk) combines them with the
// online softmax's rescaling and writes the output, in the same launch (a
// ticket counter in the workspace tells each CTA whether it is the last);
// more chunks than one CTA stages at once are combined by a merge kernel that
// spreads the rows over the GPU. When every CTA of a sequence is resident at
// once (few sequences, 16-head CTAs, no window) the chunks' 32-token grains
// are handed out at run time, so that SMs served faster by HBM take more.
//
// The kernel is HBM-bound: each K/V byte of a (sequence, K/V head) is read
// once and shared by the whole query-head group.
//
// Sliding window and sinks ("Module 5. Modern Attention Mechanisms", sections
// 9, 10 and 12): with a window of W positions the query at position n - 1
// sees positions max(0, n - W) .. n - 1, plus the first n_sink positions
// (StreamingLLM). The kernels walk a list of the 16-token sub-blocks that
// hold a visible token (the sink sub-blocks, then the window's), so the
// splits, the loads and the merge only ever touch visible sub-blocks; rows of
// a listed sub-block that are not visible are zero-filled instead of loaded
// and masked to -inf. A learned per-head sink logit s_h (gpt-oss) is one more
// score column with no value; the merge folds it in:
// lse = log(exp(lse_tokens) + exp(s_h)), O = O_tokens * exp(lse_tokens - lse).

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>

#include "internal.h"
#include "ptx.cuh"

namespace attn {
namespace {

constexpr int kGroups = 4;  // token groups of a split CTA: group t streams sub-blocks t, t + 4, ...
constexpr int kSub = 16;    // tokens per sub-block
// Lazy rescaling (FlashAttention-4): a row's running maximum, and with it the
// rescaling of its output accumulator, is only moved when a new score exceeds
// it by more than this many factors of 2; until then the probabilities are
// taken against the stale maximum (at most 2^8, exact in the final
// normalisation, which divides by a sum taken against the same maximum).
constexpr float kDecRescaleLog2 = 8.0f;
// Run-time work split (one-wave plans without a window, 16 heads per CTA):
// the sequence's sub-blocks form grains of kDecGrainSubs; every warp starts
// with two fixed grains and then takes the next free one from a counter, so
// that warps on SMs that stream faster take more of the sequence.
constexpr int kDecGrainSubs = 2;

// A split CTA covers HC chunks of 16 query heads of one K/V head. HC = 1: one
// warp per token group, each with a private 3-stage ring (two CTAs per SM).
// HC = 2 (17 to 32 query heads per K/V head, e.g. MQA): a pair of warps per
// token group shares one 6-stage ring, each warp scoring its own 16 heads
// against the same K/V tiles, so every tile crosses into the SM once for all
// 32 heads (one CTA of 8 warps per SM).
template <int HC>
struct DecShape {
  static constexpr int kWarps = kGroups * HC;
  static constexpr int kThreads = kWarps * 32;
  static constexpr int kStages = HC == 1 ? 3 : 6;
  static constexpr int kRows = 16 * HC;  // query-head rows of a CTA
};

struct DecodeParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k_cache;
  const __nv_bfloat16* v_cache;
  const int32_t* block_table;
  const int32_t* seq_lens;
  float* o_part;    // [B, Hq, splits, D]
  float* lse_part;  // [B, Hq, splits]
  // Counters, two per (sequence, K/V head, head chunk): [0] counts the
  // finished chunks (the merge in the launch), [1] hands out grains (DYN).
  unsigned long long* counters;
  // Sequences whose visible sub-blocks fit one split are written directly by
  // that split's CTA (normalised, learned sink folded in); the others by the
  // CTA that merges their chunks.
  __nv_bfloat16* o;  // [B, Hq, D]
  float* lse;        // [B, Hq] or nullptr
  const float* sinks;
  int32_t* status;
  int B, Hq, Hkv, group, hchunks;
  int num_blocks, block_size, max_blocks_per_seq, max_seq_len;
  int chunk, splits;
  int merge_in_launch;       // 1: the last CTA merges; 0: every CTA leaves its partial to a merge kernel
  int early_dependents;      // 1: let the merge kernel's CTAs launch now (they wait for this grid to finish)
  int window, n_sink;  // window 0: every cached token is visible (n_sink is then 0)
  int dyn;             // 1: grains of kDecGrainSubs sub-blocks handed out at run time (DYN kernels)
  uint32_t token;      // this call's tag for the ticket and grain counters (never 0)
  float scale_log2;  // scale * log2(e): scores live in the base-2 domain
};

// The visible tokens of a query at position seq_len - 1, as a list of
// 16-token sub-blocks: sub-blocks 0 .. a-1 hold the sink positions [0, s) not
// already inside the window, sub-blocks w0 .. ceil(seq_len / 16) - 1 the
// window [lo, seq_len). Every listed sub-block holds at least one visible
// token, and a pool block none of whose tokens is visible is never listed.
struct VisibleList {
  int lo;   // first window position
  int s;    // sink positions below lo: [0, s)
  int a;    // sink sub-blocks
  int w0;   // first window sub-block (after the sink ones)
  int nsb;  // listed sub-blocks
  __device__ __forceinline__ VisibleList(int seq_len, int window, int n_sink) {
    lo = window > 0 ? max(0, seq_len - window) : 0;
    s = min(n_sink, lo);
    a = (s + kSub - 1) / kSub;
    w0 = max(lo / kSub, a);
    nsb = a + max(0, (seq_len + kSub - 1) / kSub - w0);
  }
  // first token of listed sub-block u
  __device__ __forceinline__ int token0(int u) const { return kSub * (u < a ? u : w0 + (u - a)); }
  __device__ __forceinline__ bool visible(int t, int seq_len) const { return t < seq_len && (t >= lo || t < s); }
};

__device__ __forceinline__ void flag_status(int32_t* status, int bit) {
  if (status != nullptr) atomicOr(status, bit);
}

// Warp reduce-scatter of 32 columns: on entry lane l holds v[c] for its own
// row; on exit the returned value on lane l is the sum of column l over the 32 lanes.
__device__ __forceinline__ float warp_reduce_scatter_sum32(float (&v)[32], int lane) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    const bool upper = (lane & o) != 0;
#pragma unroll
    for (int k = 0; k < o; ++k) {
      const float keep = upper ? v[k + o] : v[k];
      const float send = upper ? v[k] : v[k + o];
      v[k] = keep + __shfl_xor_sync(0xffffffffu, send, o);
    }
  }
  return v[0];
}

// Shared memory: Q tile [16 * HC][D], then per token group kStages x (K [16][D],
// V [16][D]), then the split's block-table entries (one per listed sub-block),
// the merge's staged log-sum-exps and two flags.
// Rows are 16-byte-chunk swizzled: chunk c of row r lives at chunk c ^ (r & 7),
// which makes every ldmatrix phase hit 8 distinct bank groups.
// After the main loop the ring holds the warps' partial results and then the
// partial outputs a merge reads: kMergeFloats floats, i.e. kMergeFloats / (rows * D)
// chunks of `rows` query heads at a time (192 / rows, whatever D is).
template <int D, int HC>
struct DecSmem {
  using S = DecShape<HC>;
  static constexpr int kRowBytes = D * 2;
  static constexpr int kChunks = kRowBytes / 16;
  static constexpr int kTile = kSub * kRowBytes;
  static constexpr int kQBytes = S::kRows * kRowBytes;
  static constexpr int kRing = kGroups * S::kStages * 2 * kTile;
  static constexpr int kMergeFloats = kDecodeMergeSlots * D;
  static constexpr int kCombineFloats = kGroups * S::kRows * (2 + D);  // per token group: m, l, O rows
  static constexpr int kPhysOff = kQBytes + kRing;
  static constexpr int kLseOff = kPhysOff + kDecodeMaxChunkSubs * 4;
  static constexpr int kFlagOff = kLseOff + kDecodeMergeSlots * 4;
  static constexpr int kTotal = kFlagOff + 16;
  static_assert(kMergeFloats * 4 <= kRing && kCombineFloats * 4 <= kRing,
                "the ring holds the combine area and one merge staging");
};
static_assert(kDecodeCtasPerSm * (DecSmem<128, 1>::kTotal + 1024) <= 228 * 1024,
              "the split plan counts on two resident CTAs per SM at d = 128");
static_assert(DecSmem<128, 2>::kTotal <= 227 * 1024, "a paired CTA fits one SM at d = 128");

__device__ __forceinline__ uint32_t swz(int row, int chunk, int row_bytes) {
  return static_cast<uint32_t>(row * row_bytes + ((chunk ^ (row & 7)) << 4));
}

// Final output of one row from its unnormalised sum (already divided by the
// token sum: `inv`) and the tokens' log-sum-exp; folds a learned sink logit
// into the normaliser. Returns the natural-log LSE written for the row.
__device__ __forceinline__ float sink_fold_value(float sk, float lse_tok, float& scale_out, bool& bad) {
  if (!(fabsf(sk) <= 3.0e38f)) bad = true;  // NaN or infinite sink logit
  const float hi = fmaxf(lse_tok, sk), lo = fminf(lse_tok, sk);
  const float lse_all = hi + log1pf(__expf(lo - hi));
  scale_out *= __expf(lse_tok - lse_all);
  return lse_all;
}
__device__ __forceinline__ float sink_fold(const float* sinks, int h, float lse_tok, float& scale_out, bool& bad) {
  return sinks == nullptr ? lse_tok : sink_fold_value(sinks[h], lse_tok, scale_out, bad);
}

// One ticket on a counter this call has claimed (claim_counter), shared by
// `expected` CTAs of this launch: true for the CTA that takes the last one.
// A single atomic add, whatever the number of CTAs finishing at once.
__device__ __forceinline__ bool take_ticket(unsigned long long* c, int expected) {
  const unsigned long long old = atomicAdd(c, 1ull);
  return static_cast<int>(old & 0xffffffffull) + 1 == expected;
}

// Makes a workspace counter this call's before the CTA counts on it. The
// counter's high 32 bits hold the tag of the call that last claimed it: a
// different tag (another call, or memory that was never a counter) is
// replaced by (tag, 0), so the workspace needs no clearing, and once any CTA
// of this call has claimed it the others leave it as it is (their counts are
// never lost). A compare-and-swap fails only when another CTA of this call
// claimed or counted in between, after which the tag is this call's, so the
// loop ends within two tries; its bound is a guard, on expiry the timeout bit
// is set and the CTA does not count on the counter.
__device__ __forceinline__ bool claim_counter(unsigned long long* c, uint32_t token, int32_t* status) {
  const unsigned long long tag = static_cast<unsigned long long>(token) << 32;
  unsigned long long cur = atomicAdd(c, 0ull);
  for (int i = 0; i < 64; ++i) {
    if ((cur >> 32) == token) return true;
    const unsigned long long prev = atomicCAS(c, cur, tag);
    if (prev == cur) return true;
    cur = prev;
  }
  flag_status(status, ATTN_STATUS_BIT_TIMEOUT);
  return false;
}

// Merge the `count` partial results (slots 0 .. count - 1) of `rows`
// query-head rows into the output: lse = log sum_s exp(lse_s), O = sum_s
// exp(lse_s - lse) O_s ("Inference attention" post, "FlashDecoding"). The
// partials are staged in shared memory with cp.async (L2 only: they were
// written by other CTAs of this launch), kDecodeMergeSlots / rows slots at a
// time, and combined with the online softmax's rescaling between stagings;
// the row is then normalised, the learned sink folded in and O (bf16) and LSE
// written. Called by all NT threads of the CTA.
template <int D, int NT>
__device__ void merge_partials(const DecodeParams& p, int b, int h0, int rows, int count, float* stage,
                               float* lse_s) {
  constexpr int kMaxCpt = D / 8;
  int tpr = D / 4;  // threads per row: a power of two, at least 8
  while (tpr * rows > NT) tpr >>= 1;
  const int cpt = D / tpr;  // columns per thread, a multiple of 4
  const int r = threadIdx.x / tpr;
  const int part = threadIdx.x % tpr;
  const bool active = r < rows;
  const int col0 = part * cpt;
  const size_t rowg = static_cast<size_t>(b) * p.Hq + h0 + (active ? r : 0);
  const int cap = kDecodeMergeSlots / rows;
  constexpr int kQuads = D / 4;  // 16-byte pieces of one row

  float M = -INFINITY, L = 0.f;
  bool nan_seen = false;
  float acc[kMaxCpt];
#pragma unroll
  for (int e = 0; e < kMaxCpt; ++e) acc[e] = 0.f;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int c0 = 0; c0 < count; c0 += cap) {
    const int n = min(cap, count - c0);
    // one warp per (slot, row): the row's D floats are contiguous in the workspace
    for (int pi = warp; pi < n * rows; pi += NT / 32) {
      const int sl = pi / rows, rr = pi - sl * rows;
      const size_t src_row = (static_cast<size_t>(b) * p.Hq + h0 + rr) * p.splits + c0 + sl;
      const float* src = p.o_part + src_row * D;
      const uint32_t dst = smem_u32(stage + pi * D);
#pragma unroll
      for (int c4 = lane; c4 < kQuads; c4 += 32) cp_async_16(dst + c4 * 16, src + c4 * 4, 16u);
    }
    cp_async_commit();
    // the log-sum-exps: independent loads, one or two per thread, all in flight together
    for (int i = threadIdx.x; i < n * rows; i += NT) {
      const int sl = i / rows, rr = i - sl * rows;
      lse_s[i] = __ldcg(p.lse_part + (static_cast<size_t>(b) * p.Hq + h0 + rr) * p.splits + c0 + sl);
    }
    cp_async_wait<0>();
    __syncthreads();
    if (active) {
      float m_chunk = -INFINITY;
      for (int sl = 0; sl < n; ++sl) {
        const float x = lse_s[sl * rows + r];
        nan_seen |= (x != x);
        m_chunk = fmaxf(m_chunk, x);
      }
      const float m_new = fmaxf(M, m_chunk);
      const float keep = (M == -INFINITY) ? 0.f : fast_exp2((M - m_new) * kLog2e);
      L *= keep;
#pragma unroll
      for (int e = 0; e < kMaxCpt; ++e) acc[e] *= keep;
      for (int sl = 0; sl < n; ++sl) {
        const float x = lse_s[sl * rows + r];
        const float w = (x == -INFINITY || x != x) ? 0.f : fast_exp2((x - m_new) * kLog2e);
        L += w;
        const float* src = stage + (sl * rows + r) * D + col0;
#pragma unroll
        for (int e = 0; e < kMaxCpt; e += 4) {
          if (e < cpt) {
            const float4 v = *reinterpret_cast<const float4*>(src + e);
            acc[e] += w * v.x;
            acc[e + 1] += w * v.y;
            acc[e + 2] += w * v.z;
            acc[e + 3] += w * v.w;
          }
        }
      }
      M = m_new;
    }
    __syncthreads();  // the staging area is refilled by the next round
  }
  if (!active) return;
  float inv = 1.f / L;
  const float lse_tok = M + __logf(L);
  bool bad = nan_seen;
  bool bad_sink = false;
  const float lse_out = sink_fold(p.sinks, h0 + r, lse_tok, inv, bad_sink);
  if (bad_sink && part == 0) flag_status(p.status, ATTN_STATUS_BIT_DEVICE_CHECK);
  bad |= bad_sink;
  __nv_bfloat16* dst = p.o + rowg * D + col0;
#pragma unroll
  for (int e = 0; e < kMaxCpt; e += 2)
    if (e < cpt)
      *reinterpret_cast<uint32_t*>(dst + e) = pack_bf16x2(bad ? NAN : acc[e] * inv, bad ? NAN : acc[e + 1] * inv);
  if (part == 0 && p.lse != nullptr) p.lse[rowg] = bad ? NAN : lse_out;
}

// WIN: the sequence is read through the visible-sub-block list (sliding window,
// sink positions); without it every cached token is visible and the list
// arithmetic folds away at compile time. HC: 16-head chunks per CTA (DecShape).
// DYN: the split's sub-blocks are handed out as grains at run time (HC = 1,
// no window); every CTA of a (sequence, K/V head) then writes a partial.
template <int D, bool WIN, int HC, bool DYN>
__global__ void __launch_bounds__(DecShape<HC>::kThreads) decode_split_kernel(const DecodeParams p) {
  static_assert(!DYN || (HC == 1 && !WIN), "run-time grains: 16 heads per CTA, no window");
  using L = DecSmem<D, HC>;
  using Sh = DecShape<HC>;
  constexpr int NT = Sh::kThreads;
  constexpr int kStages = Sh::kStages;
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* q_s = smem;
  uint8_t* ring = smem + L::kQBytes;
  int* phys_s = reinterpret_cast<int*>(smem + L::kPhysOff);
  float* lse_s = reinterpret_cast<float*>(smem + L::kLseOff);
  int* cta_bad = reinterpret_cast<int*>(smem + L::kFlagOff);
  int* last_flag = cta_bad + 1;
  int* grain_ok = cta_bad + 2;
  int* dtok = reinterpret_cast<int*>(smem + L::kPhysOff);  // DYN: first token per (warp, stage), -1: no tile

  // One wave followed by the merge kernel: its CTAs may take the SMs' spare
  // room now and wait there for this grid, instead of being launched after it.
  if (p.early_dependents) asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
  const int split = blockIdx.x;
  const int kvh = blockIdx.y / p.hchunks;
  const int hc = blockIdx.y % p.hchunks;
  const int b = blockIdx.z;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int h0 = kvh * p.group + hc * Sh::kRows;
  const int rows = min(Sh::kRows, p.group - hc * Sh::kRows);
  // the learned sink logit of the row this thread finishes (row tid / 8 of the
  // combine below), requested now so that its latency hides behind the split
  const float sink_pre =
      (p.sinks != nullptr && static_cast<int>(threadIdx.x >> 3) < rows) ? __ldg(p.sinks + h0 + (threadIdx.x >> 3)) : 0.f;

  // Requests that do not depend on the sequence length go out with its read:
  // the Q rows and, without a window, the split's block-table entries (its
  // sub-blocks are then positions 16 u0 .. in order; entries past the
  // sequence are read but never used, and stay inside the table's row).
  const int per_split = p.chunk / kSub;
  const int u0 = split * per_split;  // this split's listed sub-blocks [u0, u0 + nsub)
  constexpr int kQPer = (Sh::kRows * L::kChunks + NT - 1) / NT;
  uint4 qv[kQPer];
#pragma unroll
  for (int k = 0; k < kQPer; ++k) {
    const int i = threadIdx.x + k * NT;
    const int r = i / L::kChunks, c = i % L::kChunks;
    qv[k] = make_uint4(0u, 0u, 0u, 0u);
    if (i < Sh::kRows * L::kChunks && r < rows)
      qv[k] = *reinterpret_cast<const uint4*>(p.q + (static_cast<size_t>(b) * p.Hq + h0 + r) * D + c * 8);
  }
  constexpr int kTabPer = (kDecodeMaxChunkSubs + NT - 1) / NT;
  int tab[kTabPer];
  // DYN: the block-table entries of this warp's two fixed grains, lane l < kDecGrainSubs
  // holding sub-block l of grain g_cur (ph_a) and of grain g_nxt (ph_b).
  const int n_fixed = p.splits * Sh::kWarps;  // fixed grains per round: one per warp of the sequence's CTAs
  int g_cur = split * Sh::kWarps + warp;
  int g_nxt = g_cur + n_fixed;
  int ph_a = -1, ph_b = -1;
  unsigned long long* grain_ctr = nullptr;
  if constexpr (DYN) {
    const int subs_max = (p.max_seq_len + kSub - 1) / kSub;
    const int32_t* trow = p.block_table + static_cast<size_t>(b) * p.max_blocks_per_seq;
    const int ua = g_cur * kDecGrainSubs + lane, ub = g_nxt * kDecGrainSubs + lane;
    if (lane < kDecGrainSubs && ua < subs_max) ph_a = __ldg(trow + ua * kSub / p.block_size);
    if (lane < kDecGrainSubs && ub < subs_max) ph_b = __ldg(trow + ub * kSub / p.block_size);
    grain_ctr = p.counters + (static_cast<size_t>(b) * gridDim.y + blockIdx.y) * 2 + 1;
    if (threadIdx.x == 64) *grain_ok = claim_counter(grain_ctr, p.token, p.status) ? 1 : 0;
  } else if constexpr (!WIN) {
    const int subs_max = (p.max_seq_len + kSub - 1) / kSub;
#pragma unroll
    for (int k = 0; k < kTabPer; ++k) {
      const int i = threadIdx.x + k * NT;
      tab[k] = (i < per_split && u0 + i < subs_max)
                   ? __ldg(p.block_table + static_cast<size_t>(b) * p.max_blocks_per_seq + (u0 + i) * kSub / p.block_size)
                   : -1;
    }
  }

  // The in-launch merge's ticket counter, claimed while the loads above are
  // in flight.
  unsigned long long* tickets = p.counters + (static_cast<size_t>(b) * gridDim.y + blockIdx.y) * 2;
  if (p.merge_in_launch && threadIdx.x == 0) *last_flag = claim_counter(tickets, p.token, p.status) ? 1 : 0;

  const int seq_len = p.seq_lens[b];
  if (seq_len < 1 || seq_len > p.max_seq_len) {
    // the first split's CTA writes the NaN rows of this head chunk
    if (split == 0) {
      for (int i = threadIdx.x; i < rows * D; i += NT)
        p.o[(static_cast<size_t>(b) * p.Hq + h0 + i / D) * D + i % D] = __float2bfloat16_rn(NAN);
      if (threadIdx.x < rows && p.lse != nullptr) p.lse[static_cast<size_t>(b) * p.Hq + h0 + threadIdx.x] = NAN;
      if (threadIdx.x == 0) flag_status(p.status, ATTN_STATUS_BIT_DEVICE_CHECK);
    }
    return;
  }
  const VisibleList vis(seq_len, WIN ? p.window : 0, WIN ? p.n_sink : 0);
  // split past the end of the list: nothing to read, no ticket to take (with
  // DYN every CTA may receive grains and writes a partial, empty or not)
  if (!DYN && u0 >= vis.nsb) return;
  const int nsub = DYN ? 0 : min(per_split, vis.nsb - u0);
  // partials of this sequence: the splits that hold its sub-blocks, or every split with DYN
  const int ns = DYN ? p.splits : (vis.nsb + per_split - 1) / per_split;
  const int n_grains = (vis.nsb + kDecGrainSubs - 1) / kDecGrainSubs;
  // one split: this CTA writes the output itself (only when no merge kernel
  // follows, which would otherwise merge this row's single partial)
  const bool direct = (ns == 1) && p.merge_in_launch;

  if (threadIdx.x == 0) *cta_bad = 0;
  // The split's block-table entries, one per listed sub-block, in shared
  // memory before any cache copy is issued (with a window they depend on the
  // sequence length and are requested now, all at once).
  if constexpr (DYN) {
  } else if constexpr (!WIN) {
#pragma unroll
    for (int k = 0; k < kTabPer; ++k) {
      const int i = threadIdx.x + k * NT;
      if (i < nsub) phys_s[i] = tab[k];
    }
  } else {
    for (int i = threadIdx.x; i < nsub; i += NT) {
      const int lblk = vis.token0(u0 + i) / p.block_size;
      phys_s[i] = __ldg(p.block_table + static_cast<size_t>(b) * p.max_blocks_per_seq + lblk);
    }
  }
  // Q rows of this head chunk -> swizzled shared tile; padding rows are zero.
#pragma unroll
  for (int k = 0; k < kQPer; ++k) {
    const int i = threadIdx.x + k * NT;
    if (i < Sh::kRows * L::kChunks)
      *reinterpret_cast<uint4*>(q_s + swz(i / L::kChunks, i % L::kChunks, L::kRowBytes)) = qv[k];
  }
  __syncthreads();

  // Token group tg streams sub-blocks tg, tg + 4, ... through its ring; with
  // HC = 2 its two warps (hw = 0, 1) each copy half of every tile and score
  // query-head rows 16 hw .. 16 hw + 15 of the CTA against all of it.
  const int tg = warp / HC;
  const int hw = warp % HC;
  uint8_t* my_ring = ring + tg * kStages * 2 * L::kTile;
  const int n_my = (nsub > tg) ? (nsub - tg + kGroups - 1) / kGroups : 0;
  bool bad = false;

  // Tile copies: the 32 * HC lanes of a token group copy 16-byte chunk c_l of
  // rows r_l, r_l + kRowStep, ... of each 16-row K and V tile.
  constexpr int kRowStep = 32 * HC / L::kChunks;
  constexpr int kCopies = kSub / kRowStep;
  static_assert(kRowStep * L::kChunks == 32 * HC && kCopies * kRowStep == kSub, "lanes tile the sub-block");
  const int r_l = (hw * 32 + lane) / L::kChunks, c_l = (hw * 32 + lane) % L::kChunks;
  const size_t row_elems = static_cast<size_t>(p.Hkv) * D;  // pool elements from one token to the next
  const size_t lane_src = static_cast<size_t>(r_l) * row_elems + static_cast<size_t>(kvh) * D + c_l * 8;

  auto issue = [&](int j, int stage) {
    const int i = tg + j * kGroups;  // sub-block of this split
    const int t = vis.token0(u0 + i);    // its first token
    const int lblk = t / p.block_size;
    const int off = t - lblk * p.block_size;  // multiple of 16, off + 15 < block_size
    const int phys = phys_s[i];
    const bool ok = (phys >= 0) && (phys < p.num_blocks);
    bad |= !ok;
    const size_t base = ok ? (static_cast<size_t>(phys) * p.block_size + off) * row_elems + lane_src : 0;
    const uint32_t kdst = smem_u32(my_ring + stage * 2 * L::kTile);
#pragma unroll
    for (int k = 0; k < kCopies; ++k) {
      const int r = r_l + k * kRowStep;
      const bool valid = ok && vis.visible(t + r, seq_len);  // hidden slots are zero-filled, never read
      const size_t src = valid ? base + static_cast<size_t>(k * kRowStep) * row_elems : 0;
      const uint32_t dst = kdst + swz(r, c_l, L::kRowBytes);
      cp_async_16(dst, p.k_cache + src, valid ? 16u : 0u);
      cp_async_16(dst + L::kTile, p.v_cache + src, valid ? 16u : 0u);
    }
  };

  // DYN: this warp's t-th tile is sub-block t % kDecGrainSubs of its
  // (t / kDecGrainSubs)-th grain: the two fixed grains, then one taken from
  // the counter per grain, two grains ahead of its use (lane 0 holds the
  // pending ticket), with its block-table entries read one grain ahead. A
  // grain at or past n_grains ends the warp's stream (the counter only grows,
  // so every later one would too).
  int grab = 0;
  const bool may_grab = DYN && (*grain_ok != 0);
  if (DYN && may_grab && lane == 0) grab = static_cast<int>(atomicAdd(grain_ctr, 1ull) & 0xffffffffull);
  auto issue_dyn = [&](int t, int stage) {
    const int off = t % kDecGrainSubs;
    if (off == 0 && t > 0) {  // next grain
      g_cur = g_nxt;
      ph_a = ph_b;
      const int taken = __shfl_sync(0xffffffffu, grab, 0);
      g_nxt = (may_grab && g_cur < n_grains) ? 2 * n_fixed + taken : n_grains;
      const int un = g_nxt * kDecGrainSubs + lane;
      ph_b = (lane < kDecGrainSubs && g_nxt < n_grains && un < vis.nsb)
                 ? __ldg(p.block_table + static_cast<size_t>(b) * p.max_blocks_per_seq + un * kSub / p.block_size)
                 : -1;
      if (may_grab && g_nxt < n_grains && lane == 0)
        grab = static_cast<int>(atomicAdd(grain_ctr, 1ull) & 0xffffffffull);
    }
    const int u = g_cur * kDecGrainSubs + off;
    const bool have = (g_cur < n_grains) && (u < vis.nsb);
    if (lane == 0) dtok[warp * kStages + stage] = have ? u * kSub : -1;
    if (!have) return;
    const int t0 = u * kSub;
    const int lblk = t0 / p.block_size;
    const int boff = t0 - lblk * p.block_size;
    const int phys = __shfl_sync(0xffffffffu, ph_a, off);
    const bool ok = (phys >= 0) && (phys < p.num_blocks);
    bad |= !ok;
    const size_t base = ok ? (static_cast<size_t>(phys) * p.block_size + boff) * row_elems + lane_src : 0;
    const uint32_t kdst = smem_u32(my_ring + stage * 2 * L::kTile);
#pragma unroll
    for (int k = 0; k < kCopies; ++k) {
      const int r = r_l + k * kRowStep;
      const bool valid = ok && (t0 + r < seq_len);
      const size_t src = valid ? base + static_cast<size_t>(k * kRowStep) * row_elems : 0;
      const uint32_t dst = kdst + swz(r, c_l, L::kRowBytes);
      cp_async_16(dst, p.k_cache + src, valid ? 16u : 0u);
      cp_async_16(dst + L::kTile, p.v_cache + src, valid ? 16u : 0u);
    }
  };

#pragma unroll
  for (int j = 0; j < kStages - 1; ++j) {
    if constexpr (DYN) {
      issue_dyn(j, j);
    } else {
      if (j < n_my) issue(j, j);
    }
    cp_async_commit();
  }

  // A fragments of Q for every 16-wide k step (rows = query heads).
  uint32_t qf[D / 16][4];
  {
    const uint32_t qb = smem_u32(q_s);
    const int r = hw * 16 + (lane & 15);
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const int c = kk * 2 + (lane >> 4);
      ldmatrix_x4(qb + swz(r, c, L::kRowBytes), qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3]);
    }
  }

  const float neg_inf = -INFINITY;
  float m_run[2] = {neg_inf, neg_inf};  // rows g and g + 8 of this lane (base-2 domain)
  float l_run[2] = {0.f, 0.f};          // per-lane partial sums; reduced over the quad at the end
  float o_acc[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n) o_acc[n][0] = o_acc[n][1] = o_acc[n][2] = o_acc[n][3] = 0.f;

  const int g = lane >> 2, tq = lane & 3;

  for (int j = 0; DYN || j < n_my; ++j) {
    if constexpr (DYN) {
      issue_dyn(j + kStages - 1, (j + kStages - 1) % kStages);
      cp_async_commit();
      cp_async_wait<kStages - 1>();
      __syncwarp();
      if (dtok[warp * kStages + j % kStages] < 0) break;  // no tile j: the stream has ended
    } else if constexpr (HC == 1) {
      const int jn = j + kStages - 1;
      if (jn < n_my) issue(jn, jn % kStages);
      cp_async_commit();
      cp_async_wait<kStages - 1>();
      __syncwarp();
    } else {
      // This thread's copies of tile j have landed; the pair barrier makes the
      // partner's half visible and tells that the partner is done with tile
      // j - 1, whose stage the next copy overwrites.
      cp_async_wait<kStages - 2>();
      asm volatile("bar.sync %0, %1;\n" ::"r"(1 + tg), "r"(32 * HC) : "memory");
      const int jn = j + kStages - 1;
      if (jn < n_my) issue(jn, jn % kStages);
      cp_async_commit();
    }

    const uint32_t kb = smem_u32(my_ring + (j % kStages) * 2 * L::kTile);
    const uint32_t vb = kb + L::kTile;
    const int tok0 = DYN ? dtok[warp * kStages + j % kStages] : vis.token0(u0 + tg + j * kGroups);

    // S = Q K^T for 16 tokens: two n-tiles of 8 tokens, each summed in two
    // independent accumulator chains (even and odd k steps).
    float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    float s_odd[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const int r = ((lane >> 4) << 3) + (lane & 7);
      const int c = kk * 2 + ((lane >> 3) & 1);
      uint32_t b00, b01, b10, b11;
      ldmatrix_x4(kb + swz(r, c, L::kRowBytes), b00, b01, b10, b11);
      mma_bf16_16816((kk & 1) ? s_odd[0] : s[0], qf[kk], b00, b01);
      mma_bf16_16816((kk & 1) ? s_odd[1] : s[1], qf[kk], b10, b11);
    }
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) s[nt][e] += s_odd[nt][e];
    // scale into base 2, mask slots that are not visible
    float mx[2] = {neg_inf, neg_inf};
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int tok = tok0 + nt * 8 + 2 * tq + (e & 1);
        const float x = vis.visible(tok, seq_len) ? s[nt][e] * p.scale_log2 : neg_inf;
        s[nt][e] = x;
        mx[e >> 1] = fmaxf(mx[e >> 1], x);
      }
    }
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      mx[rr] = fmaxf(mx[rr], __shfl_xor_sync(0xffffffffu, mx[rr], 1));
      mx[rr] = fmaxf(mx[rr], __shfl_xor_sync(0xffffffffu, mx[rr], 2));
    }
    // Every listed sub-block holds a visible token, so mx is finite. The
    // maxima move (and the accumulators are rescaled) only when a row's new
    // score exceeds its maximum by more than kDecRescaleLog2, always on the
    // first sub-block (m_run = -inf); the test is warp-wide so that the
    // rescaling stays one branch for the warp.
    const bool grow = (mx[0] > m_run[0] + kDecRescaleLog2) || (mx[1] > m_run[1] + kDecRescaleLog2);
    if (__any_sync(0xffffffffu, grow)) {
      float alpha[2];
#pragma unroll
      for (int rr = 0; rr < 2; ++rr) {
        const float m_new = fmaxf(m_run[rr], mx[rr]);
        alpha[rr] = fast_exp2(m_run[rr] - m_new);  // 0 on the first sub-block (m_run = -inf)
        m_run[rr] = m_new;
        l_run[rr] *= alpha[rr];
      }
#pragma unroll
      for (int n = 0; n < D / 8; ++n) {
        o_acc[n][0] *= alpha[0];
        o_acc[n][1] *= alpha[0];
        o_acc[n][2] *= alpha[1];
        o_acc[n][3] *= alpha[1];
      }
    }
    float pr[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        pr[nt][e] = fast_exp2(s[nt][e] - m_run[e >> 1]);
        l_run[e >> 1] += pr[nt][e];
      }
    uint32_t pa[4];
    pa[0] = pack_bf16x2(pr[0][0], pr[0][1]);
    pa[1] = pack_bf16x2(pr[0][2], pr[0][3]);
    pa[2] = pack_bf16x2(pr[1][0], pr[1][1]);
    pa[3] = pack_bf16x2(pr[1][2], pr[1][3]);
    // O += P V: V rows are tokens (k), columns are the head dim (n) -> trans loads.
#pragma unroll
    for (int n = 0; n < D / 8; n += 2) {
      const int r = (lane & 7) + (((lane >> 3) & 1) << 3);
      const int c = n + (lane >> 4);
      uint32_t b0a, b1a, b0b, b1b;
      ldmatrix_x4_trans(vb + swz(r, c, L::kRowBytes), b0a, b1a, b0b, b1b);
      mma_bf16_16816(o_acc[n], pa, b0a, b1a);
      mma_bf16_16816(o_acc[n + 1], pa, b0b, b1b);
    }
    __syncwarp();
  }
  cp_async_wait<0>();

#pragma unroll
  for (int rr = 0; rr < 2; ++rr) {
    l_run[rr] += __shfl_xor_sync(0xffffffffu, l_run[rr], 1);
    l_run[rr] += __shfl_xor_sync(0xffffffffu, l_run[rr], 2);
  }
  if (bad) atomicOr(cta_bad, 1);
  __syncthreads();  // every warp is done with its ring: reuse it for the combine

  // Combine the token groups: per group m[R], l[R], O[R][D] (unnormalised,
  // fp32) for the CTA's R = 16 * HC query-head rows.
  constexpr int R = Sh::kRows;
  float* wm = reinterpret_cast<float*>(ring);
  float* wl = wm + kGroups * R;
  float* wo = wl + kGroups * R;
  const int r0 = tg * R + hw * 16 + g;  // this lane's first row in the combine area
  if (tq == 0) {
    wm[r0] = m_run[0];
    wm[r0 + 8] = m_run[1];
    wl[r0] = l_run[0];
    wl[r0 + 8] = l_run[1];
  }
#pragma unroll
  for (int n = 0; n < D / 8; ++n) {
    const int col = n * 8 + 2 * tq;
    float* w0 = wo + r0 * D + col;
    float* w1 = wo + (r0 + 8) * D + col;
    w0[0] = o_acc[n][0];
    w0[1] = o_acc[n][1];
    w1[0] = o_acc[n][2];
    w1[1] = o_acc[n][3];
  }
  __syncthreads();

  const bool cta_is_bad = (*cta_bad != 0);
  if (cta_is_bad && threadIdx.x == 0) flag_status(p.status, ATTN_STATUS_BIT_DEVICE_CHECK);
  // thread -> (row = tid / 8, 8 threads per row, D / 8 columns each)
  {
    const int r = threadIdx.x >> 3;
    const int part = threadIdx.x & 7;
    if (r < rows) {
      float M = neg_inf;
#pragma unroll
      for (int w = 0; w < kGroups; ++w) M = fmaxf(M, wm[w * R + r]);
      float wsc[kGroups];
      float Lsum = 0.f;
#pragma unroll
      for (int w = 0; w < kGroups; ++w) {
        wsc[w] = (wm[w * R + r] == neg_inf) ? 0.f : fast_exp2(wm[w * R + r] - M);
        Lsum += wsc[w] * wl[w * R + r];
      }
      // a CTA that received no grain (DYN) leaves an empty partial: O = 0, LSE = -inf
      float inv = Lsum > 0.f ? 1.f / Lsum : 0.f;
      if (direct) {
        bool bad_row = cta_is_bad;
        const float lse_tok = (M + __log2f(Lsum)) * kLn2;
        const float lse_out = p.sinks != nullptr ? sink_fold_value(sink_pre, lse_tok, inv, bad_row) : lse_tok;
        if (bad_row && part == 0 && !cta_is_bad) flag_status(p.status, ATTN_STATUS_BIT_DEVICE_CHECK);
        __nv_bfloat16* dst = p.o + (static_cast<size_t>(b) * p.Hq + h0 + r) * D;
        for (int c = part * (D / 8); c < (part + 1) * (D / 8); c += 8) {
          uint32_t pk[4];
#pragma unroll
          for (int e = 0; e < 8; e += 2) {
            float v0 = 0.f, v1 = 0.f;
#pragma unroll
            for (int w = 0; w < kGroups; ++w) {
              v0 += wsc[w] * wo[(w * R + r) * D + c + e];
              v1 += wsc[w] * wo[(w * R + r) * D + c + e + 1];
            }
            pk[e >> 1] = pack_bf16x2(bad_row ? NAN : v0 * inv, bad_row ? NAN : v1 * inv);
          }
          *reinterpret_cast<uint4*>(dst + c) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
        if (part == 0 && p.lse != nullptr) p.lse[static_cast<size_t>(b) * p.Hq + h0 + r] = bad_row ? NAN : lse_out;
      } else {
        const size_t prow = (static_cast<size_t>(b) * p.Hq + h0 + r) * p.splits + split;
        float* dst = p.o_part + prow * D;
        for (int c = part * (D / 8); c < (part + 1) * (D / 8); c += 4) {
          float4 acc;
          float* a = &acc.x;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            float v = 0.f;
#pragma unroll
            for (int w = 0; w < kGroups; ++w) v += wsc[w] * wo[(w * R + r) * D + c + e];
            a[e] = cta_is_bad ? NAN : v * inv;
          }
          *reinterpret_cast<float4*>(dst + c) = acc;
        }
        if (part == 0) p.lse_part[prow] = cta_is_bad ? NAN : (Lsum > 0.f ? (M + __log2f(Lsum)) * kLn2 : -INFINITY);
      }
    }
  }
  if (direct || !p.merge_in_launch) return;

  // Split-KV merge in this launch (the plan leaves it to the merge kernel when
  // a sequence has more partials than one staging holds). Partial results are
  // published with a device-scope fence before the ticket and read after one
  // (through L2), so the merging CTA sees every other CTA's stores: the
  // barrier orders every thread's partial stores before thread 0's release
  // fence and ticket; the thread that takes the last ticket fences again
  // (acquire) before the barrier that releases the CTA into the merge.
  // *last_flag holds the counter claim's outcome (written before the barriers
  // above); a CTA whose claim ran out takes no ticket.
  float* stage = reinterpret_cast<float*>(ring);
  __syncthreads();  // also: the combine area was read above; the merge refills it
  if (threadIdx.x == 0) {
    fence_acq_rel_gpu();
    const bool last = (*last_flag != 0) && take_ticket(tickets, ns);
    if (last) fence_acq_rel_gpu();
    *last_flag = last ? 1 : 0;
  }
  __syncthreads();
  if (*last_flag == 0) return;
  merge_partials<D, NT>(p, b, h0, rows, ns, stage, lse_s);
}

struct MergeParams {
  const float* o_part;
  const float* lse_part;
  const int32_t* seq_lens;
  const float* sinks;  // [Hq] learned sink logits or nullptr
  __nv_bfloat16* o;
  float* lse;
  int32_t* status;
  int B, Hq, splits, chunk, max_seq_len, window, n_sink;
  int all_splits;  // every split wrote a partial (run-time grains)
};

// Rows with fewer than 32 splits: one CTA of 8 warps per (sequence, query
// head): lse = log sum_s exp(lse_s), O = sum_s exp(lse_s - lse) O_s over the
// chunks that hold tokens. Warp w takes chunks w, w + 8, ... four at a time
// (their loads are all in flight before the first is used) and the warps
// combine their partial sums in shared memory. A learned sink logit joins the
// normaliser last (it carries no value).
constexpr int kMergeWarps = 8;
constexpr int kMergeUnroll = 4;

template <int D>
__global__ void __launch_bounds__(kMergeWarps * 32) decode_merge_kernel(const MergeParams p) {
  constexpr int COLS = D;
  asm volatile("griddepcontrol.wait;\n" ::: "memory");  // the split grid has finished and its stores are visible
  constexpr int PER = COLS / 32;  // columns per lane
  __shared__ float s_max[kMergeWarps];
  __shared__ int s_nan[kMergeWarps];
  __shared__ float s_sum[kMergeWarps];
  __shared__ float s_acc[kMergeWarps][COLS];
  const size_t row = blockIdx.x;  // b * Hq + h
  const int b = static_cast<int>(row / p.Hq);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int seq_len = p.seq_lens[b];
  __nv_bfloat16* orow = p.o + row * D + lane * PER;
  if (seq_len < 1 || seq_len > p.max_seq_len) {
    if (threadIdx.x == 0) {
      flag_status(p.status, ATTN_STATUS_BIT_DEVICE_CHECK);
      if (p.lse) p.lse[row] = NAN;
    }
    if (warp == 0)
#pragma unroll
      for (int e = 0; e < PER; ++e) orow[e] = __float2bfloat16_rn(NAN);
    return;
  }
  const int per_split = p.chunk / kSub;
  const int ns =
      p.all_splits ? p.splits : (VisibleList(seq_len, p.window, p.n_sink).nsb + per_split - 1) / per_split;
  const float* lrow = p.lse_part + row * p.splits;
  // global max over the chunks
  float M = -INFINITY;
  bool nan_seen = false;
  for (int s = threadIdx.x; s < ns; s += kMergeWarps * 32) {
    const float x = lrow[s];
    nan_seen |= (x != x);
    M = fmaxf(M, x);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  nan_seen = __any_sync(0xffffffffu, nan_seen);
  if (lane == 0) {
    s_max[warp] = M;
    s_nan[warp] = nan_seen ? 1 : 0;
  }
  __syncthreads();
  M = s_max[0];
  int any_nan = s_nan[0];
#pragma unroll
  for (int w = 1; w < kMergeWarps; ++w) {
    M = fmaxf(M, s_max[w]);
    any_nan |= s_nan[w];
  }
  // this warp's chunks: weights relative to the global max
  float sum = 0.f;
  float acc[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) acc[e] = 0.f;
  const float* obase = p.o_part + row * p.splits * D + lane * PER;
  for (int base = warp; base < ns; base += kMergeUnroll * kMergeWarps) {
    float ls[kMergeUnroll];
    float v[kMergeUnroll][PER];
#pragma unroll
    for (int u = 0; u < kMergeUnroll; ++u) {
      const int s = base + u * kMergeWarps;
      ls[u] = -INFINITY;
#pragma unroll
      for (int e = 0; e < PER; ++e) v[u][e] = 0.f;
      if (s < ns) {
        ls[u] = lrow[s];
        const float* src = obase + static_cast<size_t>(s) * D;
        if constexpr (PER % 2 == 0) {
#pragma unroll
          for (int e = 0; e < PER; e += 2) {
            const float2 x = *reinterpret_cast<const float2*>(src + e);
            v[u][e] = x.x;
            v[u][e + 1] = x.y;
          }
        } else {
#pragma unroll
          for (int e = 0; e < PER; ++e) v[u][e] = src[e];
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kMergeUnroll; ++u) {
      const float w = (ls[u] == -INFINITY) ? 0.f : fast_exp2((ls[u] - M) * kLog2e);
      sum += w;
#pragma unroll
      for (int e = 0; e < PER; ++e) acc[e] += w * v[u][e];
    }
  }
  if (lane == 0) s_sum[warp] = sum;
#pragma unroll
  for (int e = 0; e < PER; ++e) s_acc[warp][lane * PER + e] = acc[e];
  __syncthreads();
  if (warp == 0) {
    float total = 0.f;
#pragma unroll
    for (int w = 0; w < kMergeWarps; ++w) total += s_sum[w];
    float inv = 1.f / total;
    // a learned sink: one more score column s_h with a zero value, log-added to
    // the normaliser; the output shrinks by the tokens' share of the mass
    bool bad_sink = false;
    const float lse_out = sink_fold(p.sinks, static_cast<int>(row % p.Hq), M + __logf(total), inv, bad_sink);
    if (bad_sink) {
      any_nan = 1;
      if (lane == 0) flag_status(p.status, ATTN_STATUS_BIT_DEVICE_CHECK);
    }
    float out[PER];
#pragma unroll
    for (int e = 0; e < PER; ++e) {
      float v = 0.f;
#pragma unroll
      for (int w = 0; w < kMergeWarps; ++w) v += s_acc[w][lane * PER + e];
      out[e] = any_nan ? NAN : v * inv;
    }
    if constexpr (PER % 2 == 0) {
#pragma unroll
      for (int e = 0; e < PER; e += 2)
        *reinterpret_cast<__nv_bfloat162*>(orow + e) = __floats2bfloat162_rn(out[e], out[e + 1]);
    } else {
#pragma unroll
      for (int e = 0; e < PER; ++e) orow[e] = __float2bfloat16_rn(out[e]);
    }
    if (lane == 0 && p.lse) p.lse[row] = any_nan ? NAN : lse_out;
  }
}

// Rows with many splits: one CTA of kMergeWarps warps per (sequence, query
// head, 32 columns). Every thread takes one split of a round of 256: its
// log-sum-exp and its 32 columns of the partial output are all requested at
// once, so a round costs one memory round trip. The round's maximum comes
// from a block reduction; each warp then sums its splits' weighted columns
// with a reduce-scatter (lane c ends with column c), and the warps' sums are
// added in shared memory onto the running result, rescaled between rounds
// as in the online softmax.
template <int D>
__global__ void __launch_bounds__(kMergeWarps * 32) decode_merge_wide_kernel(const MergeParams p) {
  asm volatile("griddepcontrol.wait;\n" ::: "memory");  // the split grid has finished and its stores are visible
  constexpr int kRound = kMergeWarps * 32;
  __shared__ float s_max[kMergeWarps];
  __shared__ int s_nan[kMergeWarps];
  __shared__ float s_w[kMergeWarps];
  __shared__ float s_acc[kMergeWarps][32];
  const size_t row = blockIdx.x;  // b * Hq + h
  const int c0 = static_cast<int>(blockIdx.y) * 32;
  const bool lead = (blockIdx.y == 0);  // writes the row's LSE and status bits
  const int b = static_cast<int>(row / p.Hq);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int seq_len = p.seq_lens[b];
  __nv_bfloat16* orow = p.o + row * D + c0;
  if (seq_len < 1 || seq_len > p.max_seq_len) {
    if (threadIdx.x == 0 && lead) {
      flag_status(p.status, ATTN_STATUS_BIT_DEVICE_CHECK);
      if (p.lse) p.lse[row] = NAN;
    }
    if (warp == 0) orow[lane] = __float2bfloat16_rn(NAN);
    return;
  }
  const int per_split = p.chunk / kSub;
  const int ns =
      p.all_splits ? p.splits : (VisibleList(seq_len, p.window, p.n_sink).nsb + per_split - 1) / per_split;
  const float* lrow = p.lse_part + row * p.splits;
  const float* obase = p.o_part + row * p.splits * D + c0;
  float M_run = -INFINITY, L_run = 0.f, acc_run = 0.f;  // acc_run: column `lane` (warp 0)
  bool any_nan = false;
  for (int s0 = 0; s0 < ns; s0 += kRound) {
    const int s = s0 + static_cast<int>(threadIdx.x);
    const bool valid = s < ns;
    float v[32];
    float x = -INFINITY;
    if (valid) {
      x = __ldcg(lrow + s);
      const float4* src = reinterpret_cast<const float4*>(obase + static_cast<size_t>(s) * D);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const float4 t = __ldcg(src + q);
        v[4 * q] = t.x;
        v[4 * q + 1] = t.y;
        v[4 * q + 2] = t.z;
        v[4 * q + 3] = t.w;
      }
    } else {
#pragma unroll
      for (int e = 0; e < 32; ++e) v[e] = 0.f;
    }
    // the round's maximum and NaN flag over all threads
    const bool is_nan = (x != x);
    float m = is_nan ? -INFINITY : x;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    const bool warp_nan = __any_sync(0xffffffffu, is_nan);
    if (lane == 0) {
      s_max[warp] = m;
      s_nan[warp] = warp_nan ? 1 : 0;
    }
    __syncthreads();
    float m_round = s_max[0];
    int nan_round = s_nan[0];
#pragma unroll
    for (int w = 1; w < kMergeWarps; ++w) {
      m_round = fmaxf(m_round, s_max[w]);
      nan_round |= s_nan[w];
    }
    any_nan |= (nan_round != 0);
    const float m_new = fmaxf(M_run, m_round);
    // this split's weight against the running maximum; empty or NaN splits weigh 0
    const float wgt = (x == -INFINITY || is_nan) ? 0.f : fast_exp2((x - m_new) * kLog2e);
#pragma unroll
    for (int e = 0; e < 32; ++e) v[e] *= wgt;
    const float col = warp_reduce_scatter_sum32(v, lane);  // column `lane` of this warp's splits
    float wsum = wgt;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, o);
    s_acc[warp][lane] = col;
    if (lane == 0) s_w[warp] = wsum;
    __syncthreads();
    if (warp == 0) {
      const float keep = (M_run == -INFINITY) ? 0.f : fast_exp2((M_run - m_new) * kLog2e);
      float csum = 0.f, wtot = 0.f;
#pragma unroll
      for (int w = 0; w < kMergeWarps; ++w) {
        csum += s_acc[w][lane];
        wtot += s_w[w];
      }
      acc_run = acc_run * keep + csum;
      L_run = L_run * keep + wtot;
    }
    M_run = m_new;
    __syncthreads();  // s_max / s_acc are rewritten by the next round
  }
  if (warp == 0) {
    float inv = 1.f / L_run;
    bool bad_sink = false;
    const float lse_out = sink_fold(p.sinks, static_cast<int>(row % p.Hq), M_run + __logf(L_run), inv, bad_sink);
    if (bad_sink) {
      any_nan = true;
      if (lane == 0 && lead) flag_status(p.status, ATTN_STATUS_BIT_DEVICE_CHECK);
    }
    orow[lane] = __float2bfloat16_rn(any_nan ? NAN : acc_run * inv);
    if (lane == 0 && lead && p.lse) p.lse[row] = any_nan ? NAN : lse_out;
  }
}

// Gather: out[b][h][t][:] = cache[block_table[b][t / bs]][t % bs][h][:] for
// t < seq_lens[b], zero for the rest of [0, max_seq_len). One thread per
// 16-byte chunk; consecutive threads walk (head, chunk) of one token, which
// is contiguous in the pool.
__global__ void paged_gather_kernel(const uint4* __restrict__ cache, const int32_t* __restrict__ table,
                                    const int32_t* __restrict__ seq_lens, uint4* __restrict__ out, int B, int Hkv,
                                    int chunks_per_row, int num_blocks, int block_size, int max_blocks_per_seq,
                                    int max_seq_len, int32_t* status) {
  const size_t per_seq = static_cast<size_t>(max_seq_len) * Hkv * chunks_per_row;
  const size_t total = per_seq * B;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int b = static_cast<int>(i / per_seq);
    size_t rem = i - static_cast<size_t>(b) * per_seq;
    const int t = static_cast<int>(rem / (static_cast<size_t>(Hkv) * chunks_per_row));
    rem -= static_cast<size_t>(t) * Hkv * chunks_per_row;
    const int h = static_cast<int>(rem / chunks_per_row);
    const int c = static_cast<int>(rem - static_cast<size_t>(h) * chunks_per_row);
    const int n = seq_lens[b];
    uint4 val = make_uint4(0u, 0u, 0u, 0u);
    const uint4 nan4 = make_uint4(0x7fc07fc0u, 0x7fc07fc0u, 0x7fc07fc0u, 0x7fc07fc0u);  // bf16 NaN pairs
    if (n < 0 || n > max_seq_len) {
      val = nan4;
      if (t == 0 && h == 0 && c == 0 && status) atomicOr(status, ATTN_STATUS_BIT_DEVICE_CHECK);
    } else if (t < n) {
      const int lblk = t / block_size;
      const int phys = table[static_cast<size_t>(b) * max_blocks_per_seq + lblk];
      if (phys < 0 || phys >= num_blocks) {
        val = nan4;
        if (h == 0 && c == 0 && status) atomicOr(status, ATTN_STATUS_BIT_DEVICE_CHECK);
      } else {
        val = cache[((static_cast<size_t>(phys) * block_size + (t - lblk * block_size)) * Hkv + h) * chunks_per_row +
                    c];
      }
    }
    out[((static_cast<size_t>(b) * Hkv + h) * max_seq_len + t) * chunks_per_row + c] = val;
  }
}

template <int D>
cudaError_t launch_decode_t(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_table,
                            const int32_t* seq_lens, const float* sinks, void* o, float* lse, int B, int Hq, int Hkv,
                            int num_blocks, int block_size, int max_blocks_per_seq, int max_seq_len, int window,
                            int n_sink, float scale, void* workspace, const DecodePlan& plan, uint32_t token,
                            int32_t* status, cudaStream_t stream) {
  DecodeParams p;
  const DecodeWorkspace ws = decode_workspace_layout(B, Hq, Hkv, D, plan);
  uint8_t* base = static_cast<uint8_t*>(workspace);
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k_cache = static_cast<const __nv_bfloat16*>(k_cache);
  p.v_cache = static_cast<const __nv_bfloat16*>(v_cache);
  p.block_table = block_table;
  p.seq_lens = seq_lens;
  p.o_part = reinterpret_cast<float*>(base + ws.o_part_offset);
  p.lse_part = reinterpret_cast<float*>(base + ws.lse_part_offset);
  p.counters = reinterpret_cast<unsigned long long*>(base + ws.counters_offset);
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.sinks = sinks;
  p.status = status;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.group = Hq / Hkv;
  p.hchunks = plan.hchunks;
  p.num_blocks = num_blocks;
  p.block_size = block_size;
  p.max_blocks_per_seq = max_blocks_per_seq;
  p.max_seq_len = max_seq_len;
  p.chunk = plan.chunk;
  p.splits = plan.splits;
  // The last CTA of a (sequence, head chunk) merges in this launch when one
  // staging holds all its partials; otherwise a separate merge kernel spreads
  // the rows over the whole GPU, which costs less than two in-launch levels.
  p.merge_in_launch = plan.merge_in_launch;
  const long long ctas = static_cast<long long>(plan.splits) * Hkv * plan.hchunks * B;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) !=
                                                 cudaSuccess)
    return cudaErrorUnknown;
  const long long resident = static_cast<long long>(kDecodeCtasPerSm) * sms * 16 / plan.cta_rows;
  p.early_dependents = (!p.merge_in_launch && ctas <= resident) ? 1 : 0;
  p.window = window;
  p.n_sink = n_sink;
  p.token = token;
  p.scale_log2 = scale * kLog2e;

  const bool paired = plan.cta_rows == 32;
  // run-time grains: one-wave plans of 16-head CTAs without a window (all the
  // CTAs of a sequence run at once, so the faster ones can take over work)
  p.dyn = (plan.dyn && !paired && window == 0 && plan.splits > 1 && ctas <= resident) ? 1 : 0;
  const int smem = paired ? DecSmem<D, 2>::kTotal : DecSmem<D, 1>::kTotal;
  const int threads = paired ? DecShape<2>::kThreads : DecShape<1>::kThreads;
  const auto kernel =
      paired ? (window > 0 ? decode_split_kernel<D, true, 2, false> : decode_split_kernel<D, false, 2, false>)
             : (window > 0 ? decode_split_kernel<D, true, 1, false>
                           : (p.dyn ? decode_split_kernel<D, false, 1, true> : decode_split_kernel<D, false, 1, false>));
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(plan.splits, Hkv * plan.hchunks, B);
  kernel<<<grid, threads, smem, stream>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess || p.merge_in_launch) return e;
  return launch_decode_merge(p.o_part, p.lse_part, seq_lens, sinks, o, lse, B, Hq, D, plan.splits, plan.chunk,
                             max_seq_len, window, n_sink, status, stream, p.early_dependents != 0, p.dyn != 0);
}

}  // namespace

cudaError_t launch_decode_merge(const float* o_part, const float* lse_part, const int32_t* seq_lens,
                                const float* sinks, void* o, float* lse, int B, int Hq, int d, int splits, int chunk,
                                int max_seq_len, int window, int n_sink, int32_t* status, cudaStream_t stream,
                                bool after_split_grid, bool all_splits) {
  MergeParams m;
  m.o_part = o_part;
  m.lse_part = lse_part;
  m.seq_lens = seq_lens;
  m.sinks = sinks;
  m.o = static_cast<__nv_bfloat16*>(o);
  m.lse = lse;
  m.status = status;
  m.B = B;
  m.Hq = Hq;
  m.splits = splits;
  m.chunk = chunk;
  m.max_seq_len = max_seq_len;
  m.window = window;
  m.n_sink = n_sink;
  m.all_splits = all_splits ? 1 : 0;
  // rows with many splits: 32 columns per CTA, one split per thread per round,
  // so that a single long sequence still spreads its merge over many SMs
  const bool wide = splits >= 32;
  const unsigned rows = static_cast<unsigned>(B) * static_cast<unsigned>(Hq);
  const dim3 grid(rows, wide ? static_cast<unsigned>(d / 32) : 1u);
  if (after_split_grid && wide && (d == 128 || d == 64)) {
    // programmatic dependent launch: the split grid let these CTAs launch early;
    // each waits (griddepcontrol.wait) until the split grid has completed
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(kMergeWarps * 32);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return d == 128 ? cudaLaunchKernelEx(&cfg, decode_merge_wide_kernel<128>, m)
                    : cudaLaunchKernelEx(&cfg, decode_merge_wide_kernel<64>, m);
  }
  if (d == 128)
    wide ? decode_merge_wide_kernel<128><<<grid, kMergeWarps * 32, 0, stream>>>(m)
         : decode_merge_kernel<128><<<grid, kMergeWarps * 32, 0, stream>>>(m);
  else if (d == 64)
    wide ? decode_merge_wide_kernel<64><<<grid, kMergeWarps * 32, 0, stream>>>(m)
         : decode_merge_kernel<64><<<grid, kMergeWarps * 32, 0, stream>>>(m);
  else if (d == 512)
    wide ? decode_merge_wide_kernel<512><<<grid, kMergeWarps * 32, 0, stream>>>(m)
         : decode_merge_kernel<512><<<grid, kMergeWarps * 32, 0, stream>>>(m);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

DecodeWorkspace decode_workspace_layout(int B, int Hq, int Hkv, int d, const DecodePlan& plan) {
  DecodeWorkspace w;
  const size_t rows = static_cast<size_t>(B) * Hq * plan.splits;
  w.o_part_offset = 0;
  w.lse_part_offset = rows * d * sizeof(float);
  w.counters_offset = (w.lse_part_offset + rows * sizeof(float) + 15) / 16 * 16;
  const size_t units = static_cast<size_t>(B) * Hkv * plan.hchunks;
  w.bytes = w.counters_offset + units * 2 * sizeof(unsigned long long);
  return w;
}

size_t decode_workspace_bytes(int B, int Hq, int Hkv, int d, const DecodePlan& plan) {
  return decode_workspace_layout(B, Hq, Hkv, d, plan).bytes;
}

int decode_plan_length(int max_seq_len, int window, int n_sink) {
  const long long whole = (static_cast<long long>(max_seq_len) + 15) / 16 * 16;
  if (window <= 0) return max_seq_len;
  // listed sub-blocks <= ceil(n_sink / 16) + ceil(window / 16) + 1
  const long long listed = 16LL * ((n_sink + 15LL) / 16 + (window + 15LL) / 16 + 1);
  return static_cast<int>(listed < whole ? listed : whole);
}

int plan_decode(int B, int Hq, int Hkv, int max_seq_len, int num_sms, DecodePlan* out) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || max_seq_len <= 0 || num_sms <= 0 || out == nullptr)
    return ATTN_ERR_INVALID_ARG;
  const int group = Hq / Hkv;
  // more than 16 query heads per K/V head: CTAs of 32 heads (warp pairs), one per SM
  const int cta_rows = group > 16 ? 32 : 16;
  const int hchunks = (group + cta_rows - 1) / cta_rows;
  const int rows = group < cta_rows ? group : cta_rows;
  const long long units = static_cast<long long>(B) * Hkv * hchunks;  // (sequence, K/V head, head chunk)
  const long long subs = (static_cast<long long>(max_seq_len) + 15) / 16;
  const long long slots = static_cast<long long>(kDecodeCtasPerSm) * num_sms * 16 / cta_rows;  // CTAs resident at once
  const long long cap = kDecodeMergeSlots / rows;  // partials one merge stages at a time
  long long splits;
  if (units >= slots) {
    // Enough (sequence, head) units to fill the GPU: 2048-token splits, so
    // that long sequences of a batch are cut and short ones take one split.
    splits = (subs + 127) / 128;
  } else {
    // Few units (a single long sequence, a small batch): whole waves of
    // resident CTAs, each split at most kDecodeMaxChunkSubs sub-blocks.
    const long long waves = (units * subs + slots * kDecodeMaxChunkSubs - 1) / (slots * kDecodeMaxChunkSubs);
    splits = waves * slots / units;
    const long long min_chunk_subs = 16;  // at least 256 tokens (4 sub-blocks per warp)
    splits = std::min(splits, (subs + min_chunk_subs - 1) / min_chunk_subs);
    splits = std::max(splits, (subs + kDecodeMaxChunkSubs - 1) / kDecodeMaxChunkSubs);
    splits = std::max(splits, 1LL);
  }
  // spread the 16-token sub-blocks evenly over the splits (no near-empty last split)
  const long long chunk_subs = (subs + splits - 1) / splits;
  out->chunk = static_cast<int>(16 * chunk_subs);
  out->splits = static_cast<int>((subs + chunk_subs - 1) / chunk_subs);
  out->cta_rows = cta_rows;
  out->hchunks = hchunks;
  out->dyn = units < slots ? 1 : 0;
  // the merge in the launch stages every partial of a row at once
  out->merge_in_launch = out->splits <= cap ? 1 : 0;
  return ATTN_OK;
}

cudaError_t launch_decode(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_table,
                          const int32_t* seq_lens, const float* sinks, void* o, float* lse, int B, int Hq, int Hkv,
                          int d, int num_blocks, int block_size, int max_blocks_per_seq, int max_seq_len, int window,
                          int n_sink, float scale, void* workspace, const DecodePlan& plan, int32_t* status,
                          cudaStream_t stream) {
  // A fresh tag per call for the ticket counters (never 0, the value a finished
  // call leaves behind).
  static std::atomic<uint32_t> next_token{0x9e3779b9u};
  uint32_t token = next_token.fetch_add(1u, std::memory_order_relaxed);
  if (token == 0u) token = next_token.fetch_add(1u, std::memory_order_relaxed);
  if (d == 128)
    return launch_decode_t<128>(q, k_cache, v_cache, block_table, seq_lens, sinks, o, lse, B, Hq, Hkv, num_blocks,
                                block_size, max_blocks_per_seq, max_seq_len, window, n_sink, scale, workspace, plan,
                                token, status, stream);
  return launch_decode_t<64>(q, k_cache, v_cache, block_table, seq_lens, sinks, o, lse, B, Hq, Hkv, num_blocks,
                             block_size, max_blocks_per_seq, max_seq_len, window, n_sink, scale, workspace, plan,
                             token, status, stream);
}

cudaError_t launch_paged_gather(const void* cache, const int32_t* block_table, const int32_t* seq_lens, void* out,
                                int B, int Hkv, int d, int num_blocks, int block_size, int max_blocks_per_seq,
                                int max_seq_len, int32_t* status, cudaStream_t stream) {
  const int chunks = d / 8;
  const size_t total = static_cast<size_t>(B) * max_seq_len * Hkv * chunks;
  const int threads = 256;
  const size_t want = (total + threads - 1) / threads;
  const int blocks = static_cast<int>(want < 65535 * 8 ? want : 65535 * 8);
  paged_gather_kernel<<<blocks, threads, 0, stream>>>(static_cast<const uint4*>(cache), block_table, seq_lens,
                                                      static_cast<uint4*>(out), B, Hkv, chunks, num_blocks,
                                                      block_size, max_blocks_per_seq, max_seq_len, status);
  return cudaGetLastError();
}

}  // namespace attn
