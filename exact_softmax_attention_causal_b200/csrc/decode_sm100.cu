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
// keep FlashAttention's running (max, sum, output) per query head. The warps
// combine in shared memory and write one normalised partial output and its
// log-sum-exp per (sequence, head, chunk). The merge kernel combines the
// chunks with the online softmax's rescaling.
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

#include <cmath>
#include <cstdint>

#include "internal.h"
#include "ptx.cuh"

namespace attn {
namespace {

constexpr int kDecWarps = 4;
constexpr int kDecThreads = kDecWarps * 32;
constexpr int kStages = 3;  // per-warp ring depth
constexpr int kSub = 16;    // tokens per sub-block

struct DecodeParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k_cache;
  const __nv_bfloat16* v_cache;
  const int32_t* block_table;
  const int32_t* seq_lens;
  float* o_part;    // [B, Hq, splits, D]
  float* lse_part;  // [B, Hq, splits]
  // One split per sequence: the split kernel writes the final output itself
  // (normalised, learned sink folded in) and no merge runs.
  __nv_bfloat16* o;  // [B, Hq, D]
  float* lse;        // [B, Hq] or nullptr
  const float* sinks;
  int32_t* status;
  int B, Hq, Hkv, group, hchunks;
  int num_blocks, block_size, max_blocks_per_seq, max_seq_len;
  int chunk, splits;
  int window, n_sink;  // window 0: every cached token is visible (n_sink is then 0)
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

// Shared memory: Q tile [16][D] then, per warp, kStages x (K [16][D], V [16][D]).
// Rows are 16-byte-chunk swizzled: chunk c of row r lives at chunk c ^ (r & 7),
// which makes every ldmatrix phase hit 8 distinct bank groups.
template <int D>
struct DecSmem {
  static constexpr int kRowBytes = D * 2;
  static constexpr int kChunks = kRowBytes / 16;
  static constexpr int kTile = kSub * kRowBytes;
  static constexpr int kRing = kDecWarps * kStages * 2 * kTile;
  static constexpr int kTotal = kTile + kRing + 64;
};

__device__ __forceinline__ uint32_t swz(int row, int chunk, int row_bytes) {
  return static_cast<uint32_t>(row * row_bytes + ((chunk ^ (row & 7)) << 4));
}

// Final output of one row from its unnormalised sum (already divided by the
// token sum: `inv`) and the tokens' log-sum-exp; folds a learned sink logit
// into the normaliser. Returns the natural-log LSE written for the row.
__device__ __forceinline__ float sink_fold(const float* sinks, int h, float lse_tok, float& scale_out, bool& bad) {
  if (sinks == nullptr) return lse_tok;
  const float sk = sinks[h];
  if (!(fabsf(sk) <= 3.0e38f)) bad = true;  // NaN or infinite sink logit
  const float hi = fmaxf(lse_tok, sk), lo = fminf(lse_tok, sk);
  const float lse_all = hi + log1pf(__expf(lo - hi));
  scale_out *= __expf(lse_tok - lse_all);
  return lse_all;
}

// WIN: the sequence is read through the visible-sub-block list (sliding window,
// sink positions); without it every cached token is visible and the list
// arithmetic folds away at compile time.
template <int D, bool WIN>
__global__ void __launch_bounds__(kDecThreads) decode_split_kernel(const DecodeParams p) {
  using L = DecSmem<D>;
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* q_s = smem;
  uint8_t* ring = smem + L::kTile;
  int* cta_bad = reinterpret_cast<int*>(smem + L::kTile + L::kRing);

  const int split = blockIdx.x;
  const int kvh = blockIdx.y / p.hchunks;
  const int hc = blockIdx.y % p.hchunks;
  const int b = blockIdx.z;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const int seq_len = p.seq_lens[b];
  const bool direct = (p.splits == 1);
  if (seq_len < 1 || seq_len > p.max_seq_len) {
    // the merge kernel flags this row; without a merge this CTA writes its NaN rows
    if (direct) {
      const int h0 = kvh * p.group + hc * 16, rows = min(16, p.group - hc * 16);
      for (int i = threadIdx.x; i < rows * D; i += kDecThreads)
        p.o[(static_cast<size_t>(b) * p.Hq + h0 + i / D) * D + i % D] = __float2bfloat16_rn(NAN);
      if (threadIdx.x < rows && p.lse != nullptr) p.lse[static_cast<size_t>(b) * p.Hq + h0 + threadIdx.x] = NAN;
      if (threadIdx.x == 0) flag_status(p.status, ATTN_STATUS_BIT_DEVICE_CHECK);
    }
    return;
  }
  const VisibleList vis(seq_len, WIN ? p.window : 0, WIN ? p.n_sink : 0);
  const int u0 = split * (p.chunk / kSub);  // this split's listed sub-blocks [u0, u0 + nsub)
  if (u0 >= vis.nsb) return;  // split past the end of the list: the merge never reads it
  const int nsub = min(p.chunk / kSub, vis.nsb - u0);
  const int h0 = kvh * p.group + hc * 16;
  const int rows = min(16, p.group - hc * 16);

  if (threadIdx.x == 0) *cta_bad = 0;
  // Q rows of this head chunk -> swizzled shared tile; padding rows are zero.
  for (int i = threadIdx.x; i < 16 * L::kChunks; i += kDecThreads) {
    const int r = i / L::kChunks, c = i % L::kChunks;
    uint4 val = make_uint4(0u, 0u, 0u, 0u);
    if (r < rows)
      val = *reinterpret_cast<const uint4*>(p.q + (static_cast<size_t>(b) * p.Hq + h0 + r) * D + c * 8);
    *reinterpret_cast<uint4*>(q_s + swz(r, c, L::kRowBytes)) = val;
  }
  __syncthreads();

  // A fragments of Q for every 16-wide k step (rows = query heads).
  uint32_t qf[D / 16][4];
  {
    const uint32_t qb = smem_u32(q_s);
    const int r = lane & 15;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const int c = kk * 2 + (lane >> 4);
      ldmatrix_x4(qb + swz(r, c, L::kRowBytes), qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3]);
    }
  }

  // Per-warp streaming over sub-blocks warp, warp + 4, ...
  uint8_t* my_ring = ring + warp * kStages * 2 * L::kTile;
  const int n_my = (nsub > warp) ? (nsub - warp + kDecWarps - 1) / kDecWarps : 0;
  bool bad = false;

  auto issue = [&](int j, int stage) {
    const int t = vis.token0(u0 + warp + j * kDecWarps);  // first token of the sub-block
    const int lblk = t / p.block_size;
    const int off = t - lblk * p.block_size;  // multiple of 16, off + 15 < block_size
    const int phys = __ldg(p.block_table + static_cast<size_t>(b) * p.max_blocks_per_seq + lblk);
    const bool ok = (phys >= 0) && (phys < p.num_blocks);
    bad |= !ok;
    const uint32_t kdst = smem_u32(my_ring + stage * 2 * L::kTile);
#pragma unroll
    for (int x = lane; x < kSub * L::kChunks; x += 32) {
      const int r = x / L::kChunks, c = x % L::kChunks;
      const bool valid = ok && vis.visible(t + r, seq_len);  // hidden slots are zero-filled, never read
      const size_t src = valid ? ((static_cast<size_t>(phys) * p.block_size + off + r) * p.Hkv + kvh) * D + c * 8
                               : 0;
      const uint32_t dst = kdst + swz(r, c, L::kRowBytes);
      cp_async_16(dst, p.k_cache + src, valid ? 16u : 0u);
      cp_async_16(dst + L::kTile, p.v_cache + src, valid ? 16u : 0u);
    }
  };

  const float neg_inf = -INFINITY;
  float m_run[2] = {neg_inf, neg_inf};  // rows g and g + 8 of this lane (base-2 domain)
  float l_run[2] = {0.f, 0.f};          // per-lane partial sums; reduced over the quad at the end
  float o_acc[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n) o_acc[n][0] = o_acc[n][1] = o_acc[n][2] = o_acc[n][3] = 0.f;

  const int g = lane >> 2, tq = lane & 3;

#pragma unroll
  for (int j = 0; j < kStages - 1; ++j) {
    if (j < n_my) issue(j, j);
    cp_async_commit();
  }
  for (int j = 0; j < n_my; ++j) {
    const int jn = j + kStages - 1;
    if (jn < n_my) issue(jn, jn % kStages);
    cp_async_commit();
    cp_async_wait<kStages - 1>();
    __syncwarp();

    const uint32_t kb = smem_u32(my_ring + (j % kStages) * 2 * L::kTile);
    const uint32_t vb = kb + L::kTile;
    const int tok0 = vis.token0(u0 + warp + j * kDecWarps);

    // S = Q K^T for 16 tokens: two n-tiles of 8 tokens.
    float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const int r = ((lane >> 4) << 3) + (lane & 7);
      const int c = kk * 2 + ((lane >> 3) & 1);
      uint32_t b00, b01, b10, b11;
      ldmatrix_x4(kb + swz(r, c, L::kRowBytes), b00, b01, b10, b11);
      mma_bf16_16816(s[0], qf[kk], b00, b01);
      mma_bf16_16816(s[1], qf[kk], b10, b11);
    }
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
    // every listed sub-block holds a visible token, so mx is finite
    float alpha[2];
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      const float m_new = fmaxf(m_run[rr], mx[rr]);
      alpha[rr] = fast_exp2(m_run[rr] - m_new);  // 0 on the first sub-block (m_run = -inf)
      m_run[rr] = m_new;
      l_run[rr] *= alpha[rr];
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
#pragma unroll
    for (int n = 0; n < D / 8; ++n) {
      o_acc[n][0] *= alpha[0];
      o_acc[n][1] *= alpha[0];
      o_acc[n][2] *= alpha[1];
      o_acc[n][3] *= alpha[1];
    }
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

  // Combine the 4 warps: per warp m[16], l[16], O[16][D] (unnormalised, fp32).
  float* wm = reinterpret_cast<float*>(ring);
  float* wl = wm + kDecWarps * 16;
  float* wo = wl + kDecWarps * 16;
  if (tq == 0) {
    wm[warp * 16 + g] = m_run[0];
    wm[warp * 16 + g + 8] = m_run[1];
    wl[warp * 16 + g] = l_run[0];
    wl[warp * 16 + g + 8] = l_run[1];
  }
#pragma unroll
  for (int n = 0; n < D / 8; ++n) {
    const int col = n * 8 + 2 * tq;
    float* w0 = wo + (warp * 16 + g) * D + col;
    float* w1 = wo + (warp * 16 + g + 8) * D + col;
    w0[0] = o_acc[n][0];
    w0[1] = o_acc[n][1];
    w1[0] = o_acc[n][2];
    w1[1] = o_acc[n][3];
  }
  __syncthreads();

  const bool cta_is_bad = (*cta_bad != 0);
  if (cta_is_bad && threadIdx.x == 0) flag_status(p.status, ATTN_STATUS_BIT_DEVICE_CHECK);
  // 128 threads: thread -> (row = tid / 8, 8 threads per row, D / 8 columns each)
  {
    const int r = threadIdx.x >> 3;
    const int part = threadIdx.x & 7;
    if (r < rows) {
      float M = neg_inf;
#pragma unroll
      for (int w = 0; w < kDecWarps; ++w) M = fmaxf(M, wm[w * 16 + r]);
      float wsc[kDecWarps];
      float Lsum = 0.f;
#pragma unroll
      for (int w = 0; w < kDecWarps; ++w) {
        wsc[w] = (wm[w * 16 + r] == neg_inf) ? 0.f : fast_exp2(wm[w * 16 + r] - M);
        Lsum += wsc[w] * wl[w * 16 + r];
      }
      float inv = 1.f / Lsum;
      if (direct) {
        bool bad_row = cta_is_bad;
        const float lse_out = sink_fold(p.sinks, h0 + r, (M + __log2f(Lsum)) * kLn2, inv, bad_row);
        if (bad_row && part == 0 && !cta_is_bad) flag_status(p.status, ATTN_STATUS_BIT_DEVICE_CHECK);
        __nv_bfloat16* dst = p.o + (static_cast<size_t>(b) * p.Hq + h0 + r) * D;
        for (int c = part * (D / 8); c < (part + 1) * (D / 8); c += 8) {
          uint32_t pk[4];
#pragma unroll
          for (int e = 0; e < 8; e += 2) {
            float v0 = 0.f, v1 = 0.f;
#pragma unroll
            for (int w = 0; w < kDecWarps; ++w) {
              v0 += wsc[w] * wo[(w * 16 + r) * D + c + e];
              v1 += wsc[w] * wo[(w * 16 + r) * D + c + e + 1];
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
            for (int w = 0; w < kDecWarps; ++w) v += wsc[w] * wo[(w * 16 + r) * D + c + e];
            a[e] = cta_is_bad ? NAN : v * inv;
          }
          *reinterpret_cast<float4*>(dst + c) = acc;
        }
        if (part == 0) p.lse_part[prow] = cta_is_bad ? NAN : (M + __log2f(Lsum)) * kLn2;
      }
    }
  }
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
};

// One CTA of 8 warps per (sequence, query head): lse = log sum_s exp(lse_s),
// O = sum_s exp(lse_s - lse) O_s over the chunks that hold tokens. Warp w
// takes chunks w, w + 8, ... four at a time (their loads are all in flight
// before the first is used) and the warps combine their partial sums in
// shared memory, so a single long sequence with hundreds of chunks still
// merges in parallel. A learned sink logit joins the normaliser last (it
// carries no value).
constexpr int kMergeWarps = 8;
constexpr int kMergeUnroll = 4;

// COLS < D: the row's columns are shared out over D / COLS CTAs (blockIdx.y),
// for rows with many splits; each reads every split's log-sum-exp and its
// own columns of the partial outputs.
template <int D, int COLS>
__global__ void __launch_bounds__(kMergeWarps * 32) decode_merge_kernel(const MergeParams p) {
  constexpr int PER = COLS / 32;  // columns per lane
  __shared__ float s_max[kMergeWarps];
  __shared__ int s_nan[kMergeWarps];
  __shared__ float s_sum[kMergeWarps];
  __shared__ float s_acc[kMergeWarps][COLS];
  const size_t row = blockIdx.x;  // b * Hq + h
  const int c0 = static_cast<int>(blockIdx.y) * COLS;
  const bool lead = (blockIdx.y == 0);  // writes the row's LSE and status bits
  const int b = static_cast<int>(row / p.Hq);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int seq_len = p.seq_lens[b];
  __nv_bfloat16* orow = p.o + row * D + c0 + lane * PER;
  if (seq_len < 1 || seq_len > p.max_seq_len) {
    if (threadIdx.x == 0 && lead) {
      flag_status(p.status, ATTN_STATUS_BIT_DEVICE_CHECK);
      if (p.lse) p.lse[row] = NAN;
    }
    if (warp == 0)
#pragma unroll
      for (int e = 0; e < PER; ++e) orow[e] = __float2bfloat16_rn(NAN);
    return;
  }
  const int per_split = p.chunk / kSub;
  const int ns = (VisibleList(seq_len, p.window, p.n_sink).nsb + per_split - 1) / per_split;
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
  const float* obase = p.o_part + row * p.splits * D + c0 + lane * PER;
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
      if (lane == 0 && lead) flag_status(p.status, ATTN_STATUS_BIT_DEVICE_CHECK);
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
                            int n_sink, float scale, void* workspace, const DecodePlan& plan, int32_t* status,
                            cudaStream_t stream) {
  DecodeParams p;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k_cache = static_cast<const __nv_bfloat16*>(k_cache);
  p.v_cache = static_cast<const __nv_bfloat16*>(v_cache);
  p.block_table = block_table;
  p.seq_lens = seq_lens;
  p.o_part = static_cast<float*>(workspace);
  p.lse_part = p.o_part + static_cast<size_t>(B) * Hq * plan.splits * D;
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
  p.window = window;
  p.n_sink = n_sink;
  p.scale_log2 = scale * kLog2e;

  const int smem = DecSmem<D>::kTotal;
  const auto kernel = window > 0 ? decode_split_kernel<D, true> : decode_split_kernel<D, false>;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(plan.splits, Hkv * plan.hchunks, B);
  kernel<<<grid, kDecThreads, smem, stream>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess || plan.splits == 1) return e;  // one split: the split kernel wrote the output

  return launch_decode_merge(p.o_part, p.lse_part, seq_lens, sinks, o, lse, B, Hq, D, plan.splits, plan.chunk,
                             max_seq_len, window, n_sink, status, stream);
}

}  // namespace

cudaError_t launch_decode_merge(const float* o_part, const float* lse_part, const int32_t* seq_lens,
                                const float* sinks, void* o, float* lse, int B, int Hq, int d, int splits, int chunk,
                                int max_seq_len, int window, int n_sink, int32_t* status, cudaStream_t stream) {
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
  // rows with many splits: 32 columns per CTA, so a single long sequence still
  // spreads its merge over many SMs
  const bool wide = splits >= 32;
  const unsigned rows = static_cast<unsigned>(B) * static_cast<unsigned>(Hq);
  const dim3 grid(rows, wide ? static_cast<unsigned>(d / 32) : 1u);
  if (d == 128)
    wide ? decode_merge_kernel<128, 32><<<grid, kMergeWarps * 32, 0, stream>>>(m)
         : decode_merge_kernel<128, 128><<<grid, kMergeWarps * 32, 0, stream>>>(m);
  else if (d == 64)
    wide ? decode_merge_kernel<64, 32><<<grid, kMergeWarps * 32, 0, stream>>>(m)
         : decode_merge_kernel<64, 64><<<grid, kMergeWarps * 32, 0, stream>>>(m);
  else if (d == 512)
    wide ? decode_merge_kernel<512, 32><<<grid, kMergeWarps * 32, 0, stream>>>(m)
         : decode_merge_kernel<512, 512><<<grid, kMergeWarps * 32, 0, stream>>>(m);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

size_t decode_workspace_bytes(int B, int Hq, int d, const DecodePlan& plan) {
  const size_t rows = static_cast<size_t>(B) * Hq * plan.splits;
  return rows * d * sizeof(float) + rows * sizeof(float);
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
  const int hchunks = (group + 15) / 16;
  const long long units = static_cast<long long>(B) * Hkv * hchunks;
  // CTAs: at least one per SM. More, shorter splits were measured slower on
  // single long sequences (per-CTA latency and merge work outweigh the fill).
  const long long target = 1LL * num_sms;
  int chunk = 2048;
  while (chunk > 256 && units * ((max_seq_len + chunk - 1) / chunk) < target) chunk >>= 1;
  // spread the 16-token sub-blocks evenly over the splits (no near-empty last split)
  const int subs = (max_seq_len + 15) / 16;
  const int nominal_splits = (max_seq_len + chunk - 1) / chunk;
  out->chunk = 16 * ((subs + nominal_splits - 1) / nominal_splits);
  out->splits = (max_seq_len + out->chunk - 1) / out->chunk;
  out->hchunks = hchunks;
  return ATTN_OK;
}

cudaError_t launch_decode(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_table,
                          const int32_t* seq_lens, const float* sinks, void* o, float* lse, int B, int Hq, int Hkv,
                          int d, int num_blocks, int block_size, int max_blocks_per_seq, int max_seq_len, int window,
                          int n_sink, float scale, void* workspace, const DecodePlan& plan, int32_t* status,
                          cudaStream_t stream) {
  if (d == 128)
    return launch_decode_t<128>(q, k_cache, v_cache, block_table, seq_lens, sinks, o, lse, B, Hq, Hkv, num_blocks,
                                block_size, max_blocks_per_seq, max_seq_len, window, n_sink, scale, workspace, plan,
                                status, stream);
  return launch_decode_t<64>(q, k_cache, v_cache, block_table, seq_lens, sinks, o, lse, B, Hq, Hkv, num_blocks,
                             block_size, max_blocks_per_seq, max_seq_len, window, n_sink, scale, workspace, plan,
                             status, stream);
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
