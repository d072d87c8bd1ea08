// Attention backward pass on the 5th-generation tensor cores (tcgen05 + TMEM
// + TMA): dQ, dK, dV of prefill attention.
//
// What it computes: the derivative of O = softmax(scale Q K^T + M) V
// ("Module 5. Modern Attention Mechanisms", section 4; grouped-query heads as
// in section 6) for an upstream gradient dO, by the chain rule:
//   P  = exp(scale S - LSE) (S = Q K^T, LSE the forward's log-sum-exp)
//   dV = P^T dO,  dP = dO V^T,  dS = P (dP - D),  D = rowsum(dO * O)
//   dQ = scale dS K,  dK = scale dS^T Q,
// with dK and dV of a K/V head summed over the query heads of its group.
// As the "Inference attention" post (section "FlashAttention") says of the
// backward pass, S and P are recomputed tile by tile from the saved LSE
// instead of being stored.
//
// How: three kernels, no atomics (the result does not depend on scheduling):
//   bwd_rowdot_kernel  D = rowsum(dO * O), one warp per row, fp32.
//   bwd_dkdv_kernel    one CTA per (batch, K/V head, 128-key tile): for every
//                      query head of the group and every 128-row query tile
//                      that sees the key tile, in two halves of 64 query rows,
//                      S^T = K Q^T and dP^T = V dO^T into TMEM (M = keys),
//                      P^T and dS^T (bf16) written back over them, then
//                      dV += P^T dO and dK += dS^T Q with the probabilities
//                      read from TMEM. The halves alternate between two TMEM
//                      regions, so the P / dS warps work on one half while the
//                      tensor cores run the other's products.
//   bwd_dq_kernel      one CTA per (batch, query head, 128-row query tile):
//                      S = Q K^T and dP = dO V^T per key tile, dS (bf16) over
//                      S, then dQ += dS K. K and V stream through rings of
//                      three and two stages; S is double-buffered and dP is
//                      released as soon as the dS warps have loaded it, so
//                      the next tile's scores are ready when they finish.
// Each recomputes S once more than a single fused kernel would (seven
// 128x128xd products per tile pair instead of five), in exchange for
// deterministic sums without a dQ accumulator shared between CTAs.
//
// Roles in both tile kernels (320 threads): warps 0-7 compute P and dS (warp w
// reads TMEM lanes 32 (w % 4) .. + 31, one key row (dK/dV) or query row (dQ)
// per lane; in the dQ kernel over the column half w / 4 of each tile, in the
// dK/dV kernel over the half-tiles of TMEM region w / 4), warp 8 is the TMA
// producer, warp 9 issues the MMAs and owns TMEM (the whole warp runs the issue
// loop and one elected lane issues each MMA and commit). Every pipeline wait is
// bounded; on expiry the CTA records ATTN_STATUS_BIT_TIMEOUT, writes NaN, drains
// and exits.

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>

#include "internal.h"
#include "ptx.cuh"

namespace attn {
namespace {

constexpr int kT = 128;             // rows per tile (TMEM lanes), keys per tile
constexpr int kBwdThreads = 320;
constexpr int kBwdTmaWarp = 8;
constexpr int kBwdMmaWarp = 9;
constexpr int kBwdSoftWarps = 8;  // TMEM sub-partition (w % 4) x column half (w / 4)
constexpr int kBox = 128 * 128;     // bytes of one 64-column, 128-row swizzled box

struct BwdParams {
  const __nv_bfloat16* o;
  const __nv_bfloat16* d_o;
  const float* lse;   // [B, Hq, N] natural log (forward output)
  // workspace, rows padded to whole tiles (npad = 128 * ntiles), 16-byte aligned:
  float* lse2;        // [B, Hq, npad] LSE * log2(e), +inf past N
  float* dvec;        // [B, Hq, npad] D = rowsum(dO * O), 0 past N
  __nv_bfloat16* dq;  // [B, Hq, N, d]
  __nv_bfloat16* dk;  // [B, Hkv, N, d]
  __nv_bfloat16* dv;  // [B, Hkv, N, d]
  int32_t* status;
  int B, Hq, Hkv, N, group, mask_kind, window, ntiles, npad;
  int chunk_kv, chunk_q;  // heads per scheduling chunk (dK/dV kernel: batch x K/V head; dQ: batch x query head)
  float scale, scale_log2;
  long long budget;
};

__device__ __forceinline__ void bwd_abort(volatile int* abort_flag, int32_t* status) {
  *abort_flag = 1;
  if (status != nullptr) atomicOr(status, ATTN_STATUS_BIT_TIMEOUT);
}

// key kpos visible to query qpos (both < N checked by the caller)
__device__ __forceinline__ bool bwd_visible(const BwdParams& p, int qpos, int kpos) {
  if (p.mask_kind == ATTN_MASK_FULL) return true;
  if (kpos > qpos) return false;
  return p.mask_kind != ATTN_MASK_SLIDING_WINDOW || qpos - kpos < p.window;
}

// Block order of both tile kernels: the (head, tile) blocks are taken in chunks of `chunk`
// heads whose shared operands fit in L2 together; inside a chunk the tile of rank 0 (the one
// with the most work under a causal or window mask) comes first for every head, then rank 1, ...
// Blocks are dispatched roughly in index order, so the longest run first (less idle time at the
// end) while the blocks in flight read the tiles of a few heads only.
__device__ __forceinline__ void block_order(int x, int units, int ntiles, int chunk, int& unit, int& rank) {
  const int per_chunk = chunk * ntiles;
  const int c = x / per_chunk;
  const int within = x - c * per_chunk;
  const int n = min(chunk, units - c * chunk);  // heads in this (possibly last, shorter) chunk
  rank = within / n;
  unit = c * chunk + (within - rank * n);
}

// Query tiles [lo, hi] that see key tile j, and key tiles that query tile i sees.
__device__ __forceinline__ void q_tiles_of_key_tile(const BwdParams& p, int j, int& lo, int& hi) {
  lo = 0;
  hi = p.ntiles - 1;
  if (p.mask_kind != ATTN_MASK_FULL) lo = j;
  if (p.mask_kind == ATTN_MASK_SLIDING_WINDOW) hi = min(hi, (j * kT + kT - 1 + p.window - 1) / kT);
}
__device__ __forceinline__ void k_tiles_of_q_tile(const BwdParams& p, int i, int& lo, int& hi) {
  lo = 0;
  hi = p.ntiles - 1;
  if (p.mask_kind != ATTN_MASK_FULL) hi = i;
  if (p.mask_kind == ATTN_MASK_SLIDING_WINDOW) lo = max(0, i * kT - p.window + 1) / kT;
}

// kind::f16 instruction descriptor (fp32 accumulate, bf16 inputs).
__host__ __device__ constexpr uint32_t idesc_bwd(int M, int N, int a_mn, int b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(a_mn) << 15) |
         (static_cast<uint32_t>(b_mn) << 16) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

// Both product helpers are warp-collective (the MMA warp runs them converged).
// D x d/16 steps of a product with both operands K-major in shared memory
// (K dimension = head dim: 64-column boxes of 16 KB hold 4 steps of 32 bytes).
template <int D>
__device__ __forceinline__ void mma_kmajor(uint32_t d_tmem, uint64_t da, uint64_t db, uint32_t idesc) {
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint64_t off = static_cast<uint64_t>(((kk >> 2) * kBox + (kk & 3) * 32) >> 4);
    tc_mma_ss_w(d_tmem, da + off, db + off, idesc, kk > 0 ? 1u : 0u);
  }
}
// 64 / 16 steps of the same product over half a tile (dK/dV kernel): A holds the bf16 pairs of
// 64 K rows, written in two 32-row chunks, each over the first half of its own 32 columns:
// K rows 16 kk .. 16 kk + 15 sit at column 32 (kk / 2) + 8 (kk % 2).
__device__ __forceinline__ void mma_tmem_a_half(uint32_t d_tmem, uint32_t a_tmem, uint64_t db, uint32_t idesc,
                                                bool first) {
#pragma unroll
  for (int kk = 0; kk < kT / 32; ++kk)
    tc_mma_ts_w(d_tmem, a_tmem + 32u * (kk >> 1) + 8u * (kk & 1), db + static_cast<uint64_t>((kk * 2048) >> 4),
                idesc, (!first || kk > 0) ? 1u : 0u);
}
// 128 / 16 steps of D (+)= A[tmem] * B[smem, MN-major, 16 rows per step]. A holds bf16 pairs
// written by two warps per TMEM sub-partition, each over the first half of its own 64 columns:
// K rows 16 kk .. 16 kk + 15 sit at column 64 (kk / 4) + 8 (kk % 4).
__device__ __forceinline__ void mma_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint64_t db, uint32_t idesc,
                                           bool first) {
#pragma unroll
  for (int kk = 0; kk < kT / 16; ++kk)
    tc_mma_ts_w(d_tmem, a_tmem + 64u * (kk >> 2) + 8u * (kk & 3), db + static_cast<uint64_t>((kk * 2048) >> 4), idesc,
                (!first || kk > 0) ? 1u : 0u);
}

// ---------------------------------------------------------------------------
// D = rowsum(dO * O) and LSE * log2(e), one warp per (batch, head, padded row)
// ---------------------------------------------------------------------------
template <int D>
__global__ void bwd_rowdot_kernel(const BwdParams p) {
  const size_t rows = static_cast<size_t>(p.B) * p.Hq * p.npad;
  const size_t prow = blockIdx.x * static_cast<size_t>(blockDim.x / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (prow >= rows) return;
  const size_t bh = prow / p.npad;
  const int q = static_cast<int>(prow - bh * p.npad);
  if (q >= p.N) {  // padding rows: no probability mass (exp2(x - inf) = 0) and D = 0
    if (lane == 0) {
      p.dvec[prow] = 0.f;
      p.lse2[prow] = INFINITY;
    }
    return;
  }
  const size_t row = bh * p.N + q;
  constexpr int PER = D / 32;
  const __nv_bfloat16* a = p.o + row * D + lane * PER;
  const __nv_bfloat16* g = p.d_o + row * D + lane * PER;
  float s = 0.f;
#pragma unroll
  for (int e = 0; e < PER; e += 2) {
    const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(a + e));
    const float2 y = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(g + e));
    s += x.x * y.x + x.y * y.y;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) {
    p.dvec[prow] = s;
    p.lse2[prow] = p.lse[row] * kLog2e;
  }
}

// Shared-memory plan of the dK/dV kernel (1024-byte aligned) and the TMEM columns of both
// tile kernels:
template <int D>
struct BwdCfg {
  static constexpr int kHalves = D / 64;
  static constexpr int kTile = kHalves * kBox;  // one 128 x D bf16 tile
  // dK/dV: K, V resident; two stages of (Q, dO) and their LSE / D rows.
  static constexpr int kKOff = 0;
  static constexpr int kVOff = kKOff + kTile;
  static constexpr int kQOff = kVOff + kTile;          // + stage * 2 * kTile
  static constexpr int kStageBytes = 2 * kTile;        // Q then dO
  static constexpr int kRowOff = kQOff + 2 * kStageBytes;  // [stage][LSE*log2e 128 | D 128] fp32 (dK/dV)
  static constexpr int kBarOff = kRowOff + 2 * 2 * kT * 4;
  static constexpr int kBytes = kBarOff + 256;
  static constexpr int kAlloc = kBytes + 1024;
  // TMEM columns. dQ kernel: S 128, dP 128, the dQ accumulator, a second S buffer in the
  // last 128 columns. dK/dV kernel: two regions of 128 columns, each holding one half-tile's
  // S^T (64 columns) and dP^T (64 columns), then the dV and dK accumulators.
  static constexpr uint32_t kColS = 0, kColDP = 128, kColAcc0 = 256, kColAcc1 = 256 + D, kColS2 = 384;
  static constexpr uint32_t kRegion = 128, kRegionDP = 64;
};

// Barriers of the dK/dV kernel.
enum : int {
  kBbKV = 0,       // K and V resident tiles landed
  kBbFull = 1,     // + stage (2)
  kBbEmpty = 3,    // + stage (2)
  kBbS = 5,        // S^T and dP^T of a half-tile in TMEM, + region (2)
  kBbP = 7,        // P^T / dS^T written back by the region's 4 softmax warps, + region (2)
  kBbAcc = 9,      // accumulators final
  kBbDrain = 10,
};
constexpr int kBwdTmemSlot = 128;
constexpr int kBwdAbort = 132;

// Shared-memory plan of the dQ kernel: Q and dO resident, K in a ring of three
// stages and V in a ring of two. V of key tile t is released once dP(t) has read
// it, K only after dQ(t), so the ring that is released later is the deeper one.
template <int D>
struct DqCfg {
  static constexpr int kTile = BwdCfg<D>::kTile;
  static constexpr int kKStages = 3, kVStages = 2;
  static constexpr int kQOff = 0;
  static constexpr int kDoOff = kTile;
  static constexpr int kKOff = 2 * kTile;                 // + stage * kTile
  static constexpr int kVOff = kKOff + kKStages * kTile;  // + stage * kTile
  static constexpr int kBarOff = kVOff + kVStages * kTile;
  static constexpr int kBytes = kBarOff + 256;
  static constexpr int kAlloc = kBytes + 1024;
  static_assert(kAlloc <= 227 * 1024, "dQ kernel shared memory");
};
enum : int {
  kDqQ = 0,                 // Q and dO landed
  kDqFullK = 1,             // + stage (3)
  kDqEmptyK = 4,            // + stage (3)
  kDqFullV = 7,             // + stage (2)
  kDqEmptyV = 9,            // + stage (2)
  kDqS = 11,                // S and dP of the current key tile are in TMEM
  kDqP = 12,                // dS of key tile t written back (8 arrivals), + t % 2 (2)
  kDqAcc = 14,
  kDqDrain = 15,
  kDqDPFree = 16,           // the dS warps have loaded dP (8 arrivals)
};
// kDqP alternates between two barriers: the MMA warp issues dP(t + 1), which lets the dS
// warps go on to key tile t + 1, before it waits for dS(t); on one barrier they could
// complete the phases of t and t + 1 before that wait looks, and the wait would then see
// the phase parity of t again and never return.
constexpr int kDqTmemSlot = 192;
constexpr int kDqAbort = 196;

// ---------------------------------------------------------------------------
// dK, dV: one CTA per (key tile, K/V head, batch)
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                    const BwdParams p) {
  using C = BwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  const uint32_t sbase = (raw_u32 + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (sbase - raw_u32);
  // key tile j sees the query tiles j, j + 1, ... under a causal or window mask: rank j
  int unit, j;
  block_order(static_cast<int>(blockIdx.x), p.B * p.Hkv, p.ntiles, p.chunk_kv, unit, j);
  const int kvh = unit % p.Hkv, b = unit / p.Hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int qlo, qhi;
  q_tiles_of_key_tile(p, j, qlo, qhi);
  const int nq = qhi - qlo + 1;
  const int iters = p.group * nq;  // (query head of the group, query tile) pairs, head-major

  const uint32_t bars = sbase + C::kBarOff;
  auto bar = [&](int i) -> uint32_t { return bars + 8u * static_cast<uint32_t>(i); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kBarOff + kBwdTmemSlot);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kBarOff + kBwdAbort);
  if (threadIdx.x == 0) {
    mbar_init(bar(kBbKV), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(kBbFull + s), 1);
      mbar_init(bar(kBbEmpty + s), 1);
    }
    for (int r = 0; r < 2; ++r) {
      mbar_init(bar(kBbS + r), 1);
      mbar_init(bar(kBbP + r), kBwdSoftWarps / 2);  // the warp group of region r
    }
    mbar_init(bar(kBbAcc), 1);
    mbar_init(bar(kBbDrain), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kBwdMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const long long budget = p.budget;

  if (warp == kBwdTmaWarp) {
    if (lane == 0) {
      // ---------------------------------------------------------- TMA producer
      const int zkv = b * p.Hkv + kvh;
      mbar_arrive_expect_tx(bar(kBbKV), 2 * C::kTile);
      for (int hh = 0; hh < C::kHalves; ++hh) {
        tma_load_3d(sbase + C::kKOff + hh * kBox, &tm_k, bar(kBbKV), hh * 64, j * kT, zkv);
        tma_load_3d(sbase + C::kVOff + hh * kBox, &tm_v, bar(kBbKV), hh * 64, j * kT, zkv);
      }
      int issued[2] = {0, 0};
      bool ok = true;
      for (int t = 0; t < iters && ok; ++t) {
        const int s = t & 1;
        if (t >= 2 && !mbar_wait_bounded(bar(kBbEmpty + s), ((t - 2) >> 1) & 1, budget, abort_flag)) {
          ok = false;
          break;
        }
        const int h = kvh * p.group + t / nq, i = qlo + t % nq;
        const int zq = b * p.Hq + h;
        const uint32_t st = sbase + C::kQOff + s * C::kStageBytes;
        const uint32_t rows = sbase + C::kRowOff + s * (2 * kT * 4);
        const size_t prow = static_cast<size_t>(zq) * p.npad + static_cast<size_t>(i) * kT;
        mbar_arrive_expect_tx(bar(kBbFull + s), 2 * C::kTile + 2 * kT * 4);
        for (int hh = 0; hh < C::kHalves; ++hh) {
          tma_load_3d(st + hh * kBox, &tm_q, bar(kBbFull + s), hh * 64, i * kT, zq);
          tma_load_3d(st + C::kTile + hh * kBox, &tm_do, bar(kBbFull + s), hh * 64, i * kT, zq);
        }
        bulk_load(rows, p.lse2 + prow, kT * 4, bar(kBbFull + s));
        bulk_load(rows + kT * 4, p.dvec + prow, kT * 4, bar(kBbFull + s));
        issued[s] = t / 2 + 1;
      }
      if (!ok) bwd_abort(abort_flag, p.status);
      volatile int never = 0;
      mbar_wait_bounded(bar(kBbKV), 0, kDrainBudgetCycles, &never);
      for (int s = 0; s < 2; ++s)
        if (issued[s] > 0) mbar_wait_bounded(bar(kBbFull + s), (issued[s] - 1) & 1, kDrainBudgetCycles, &never);
    }
  } else if (warp == kBwdMmaWarp) {
    // ------------------------------------------------------------ MMA issuer (whole warp)
    const uint64_t dk = desc_sw128(sbase + C::kKOff, 16, 1024);
    const uint64_t dvv = desc_sw128(sbase + C::kVOff, 16, 1024);
    constexpr uint32_t kIdS = idesc_bwd(kT, kT / 2, 0, 0);  // S^T = K Q^T, dP^T = V dO^T (64 query rows)
    constexpr uint32_t kIdAcc = idesc_bwd(kT, D, 0, 1);     // dV += P^T dO, dK += dS^T Q (B MN-major)
    constexpr uint32_t kHalfRows = (kT / 2) * 128;          // bytes of 64 rows in a 128-byte-swizzled box
    auto wait = [&](uint32_t b_, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait_bounded(b_, parity, budget, abort_flag));
    };
    // Half u covers query rows 64 (u % 2) .. + 63 of pair u / 2 and uses TMEM region u % 2.
    auto half_stage = [&](int u) -> uint32_t {
      return sbase + C::kQOff + ((u >> 1) & 1) * C::kStageBytes + (u & 1) * kHalfRows;
    };
    auto issue_s = [&](int u) {
      const uint32_t st = half_stage(u);
      const uint32_t reg = tmem + C::kRegion * (u & 1);
      mma_kmajor<D>(reg, dk, desc_sw128(st, 16, 1024), kIdS);
      mma_kmajor<D>(reg + C::kRegionDP, dvv, desc_sw128(st + C::kTile, 16, 1024), kIdS);
      tc_commit_w(bar(kBbS + (u & 1)));
    };
    const int halves = 2 * iters;
    bool ok = wait(bar(kBbKV), 0) && wait(bar(kBbFull), 0);
    if (ok) {
      tc_fence_after();
      issue_s(0);
      issue_s(1);
    }
    for (int u = 0; u < halves && ok; ++u) {
      const int r = u & 1, t = u >> 1;
      if (!wait(bar(kBbP + r), (u >> 1) & 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
      // B = dO (then Q) as an MN-major operand: N = head dim (64-column boxes kBox apart),
      // K = query rows (16 per step, 2 KB apart)
      const uint32_t st = half_stage(u);
      const uint32_t reg = tmem + C::kRegion * r;
      mma_tmem_a_half(tmem + C::kColAcc0, reg, desc_sw128(st + C::kTile, kBox, 1024), kIdAcc, u == 0);
      mma_tmem_a_half(tmem + C::kColAcc1, reg + C::kRegionDP, desc_sw128(st, kBox, 1024), kIdAcc, u == 0);
      if (r == 1) tc_commit_w(bar(kBbEmpty + (t & 1)));  // the pair's last read of its stage
      if (u + 2 < halves) {
        // the next half in this region, issued behind the products that read the region
        if (r == 0) {  // it opens pair t + 1
          if (!wait(bar(kBbFull + ((t + 1) & 1)), ((t + 1) >> 1) & 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
        }
        issue_s(u + 2);
      }
    }
    if (!ok && lane == 0) bwd_abort(abort_flag, p.status);
    tc_commit_w(bar(kBbAcc));
    tc_commit_w(bar(kBbDrain));
    volatile int never = 0;
    mbar_wait_bounded(bar(kBbDrain), 0, kDrainBudgetCycles, &never);
    __syncwarp();
  } else {
    // ------------------------------------------------------------ P / dS warps 0-7
    // Two warp groups in ping-pong: group g = w / 4 takes the half-tiles g, g + 2, ... (TMEM
    // region g), all 64 query rows of each, so one group computes while the other waits.
    const int r = (warp & 3) * 32 + lane;  // key row of the tile = TMEM lane
    const int ch = warp >> 2;              // warp group: TMEM region, and D-column half in the epilogue
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const uint32_t reg = lane_base + C::kRegion * ch;
    const int kpos = j * kT + r;
    const float sl2 = p.scale_log2;
    bool ok = true;
    int i = qlo;  // query tile of pair t: pairs run head-major, so i cycles through qlo .. qhi
    for (int t = 0; t < iters; ++t, i = (i == qhi) ? qlo : i + 1) {
      // the staged LSE / D rows first (the MMA warp releases stage t & 1 only after the pair's
      // last products, which wait for this group's P / dS), then this half's S^T and dP^T
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait_bounded(bar(kBbFull + (t & 1)), (t >> 1) & 1, budget, abort_flag));
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait_bounded(bar(kBbS + ch), t & 1, budget, abort_flag));
      if (!ok) break;  // no named barriers here: leaving early strands no other warp
      tc_fence_after();
      const float* srow = reinterpret_cast<const float*>(smem + C::kRowOff + (t & 1) * (2 * kT * 4));
      const bool full_tile = (p.mask_kind == ATTN_MASK_FULL || (i > j && (p.mask_kind == ATTN_MASK_CAUSAL ||
                                                                          (i * kT + kT - 1) - j * kT < p.window))) &&
                             (i * kT + kT <= p.N) && (j * kT + kT <= p.N);
#pragma unroll 1
      for (int cc = 0; cc < 2; ++cc) {
        const int c = 2 * ch + cc;  // 32-column chunk of the tile: query rows 32 c .. 32 c + 31
        uint32_t sv[32], dpv[32];
        tmem_ld_32x32b_x32(reg + 32u * cc, sv);
        tmem_ld_32x32b_x32(reg + C::kRegionDP + 32u * cc, dpv);
        // the 32 query columns' LSE (base 2) and D: broadcast shared-memory reads;
        // rows past N carry +inf and 0
        float l2[32], dd[32];
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          const float4 lv = *reinterpret_cast<const float4*>(srow + 32 * c + e);
          const float4 dv4 = *reinterpret_cast<const float4*>(srow + kT + 32 * c + e);
          l2[e] = lv.x;
          l2[e + 1] = lv.y;
          l2[e + 2] = lv.z;
          l2[e + 3] = lv.w;
          dd[e] = dv4.x;
          dd[e + 1] = dv4.y;
          dd[e + 2] = dv4.z;
          dd[e + 3] = dv4.w;
        }
        if (!full_tile) {
          // hidden (query, key) entries: LSE +inf makes the exponent -inf and P exactly 0
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int qpos = i * kT + 32 * c + e;
            if (!(qpos < p.N && kpos < p.N && bwd_visible(p, qpos, kpos))) l2[e] = INFINITY;
          }
        }
        tc_wait_ld();
        uint32_t pk[16], dsk[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const float p0 = exp2_approx(fmaf(__uint_as_float(sv[e]), sl2, -l2[e]));
          const float p1 = exp2_approx(fmaf(__uint_as_float(sv[e + 1]), sl2, -l2[e + 1]));
          pk[e >> 1] = pack_bf16x2(p0, p1);
          dsk[e >> 1] = pack_bf16x2(p0 * (__uint_as_float(dpv[e]) - dd[e]), p1 * (__uint_as_float(dpv[e + 1]) - dd[e + 1]));
        }
        // bf16 pairs over the first half of this chunk's own (already read) columns
        tmem_st_32x32b_x16(reg + 32u * cc, pk);
        tmem_st_32x32b_x16(reg + C::kRegionDP + 32u * cc, dsk);
      }
      tc_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kBbP + ch));
    }
    // ------------------------------------------------------------ epilogue
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait_bounded(bar(kBbAcc), 0, budget, abort_flag));
    if (!ok) bwd_abort(abort_flag, p.status);
    tc_fence_after();
    // TMEM loads are warp-collective: every lane runs them, only rows < N are stored
    const bool store = kpos < p.N;
    __nv_bfloat16* dvrow = p.dv + ((static_cast<size_t>(b) * p.Hkv + kvh) * p.N + (store ? kpos : 0)) * D;
    __nv_bfloat16* dkrow = p.dk + ((static_cast<size_t>(b) * p.Hkv + kvh) * p.N + (store ? kpos : 0)) * D;
#pragma unroll 1
    for (int c = ch * (D / 64); c < (ch + 1) * (D / 64); ++c) {  // this warp's half of the head dim
      uint32_t va[32], ka[32];
      tmem_ld_32x32b_x32(lane_base + C::kColAcc0 + 32u * c, va);
      tmem_ld_32x32b_x32(lane_base + C::kColAcc1 + 32u * c, ka);
      tc_wait_ld();
#pragma unroll
      for (int e = 0; e < 32; e += 8) {
        uint32_t pv[4], pkk[4];
#pragma unroll
        for (int u = 0; u < 8; u += 2) {
          pv[u >> 1] = pack_bf16x2(ok ? __uint_as_float(va[e + u]) : NAN, ok ? __uint_as_float(va[e + u + 1]) : NAN);
          pkk[u >> 1] = pack_bf16x2(ok ? __uint_as_float(ka[e + u]) * p.scale : NAN,
                                    ok ? __uint_as_float(ka[e + u + 1]) * p.scale : NAN);
        }
        if (store) {
          *reinterpret_cast<uint4*>(dvrow + 32 * c + e) = make_uint4(pv[0], pv[1], pv[2], pv[3]);
          *reinterpret_cast<uint4*>(dkrow + 32 * c + e) = make_uint4(pkk[0], pkk[1], pkk[2], pkk[3]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kBwdMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// dQ: one CTA per (query tile, query head, batch)
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                  const BwdParams p) {
  using C = BwdCfg<D>;  // TMEM columns
  using Q = DqCfg<D>;   // shared memory and barriers
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  const uint32_t sbase = (raw_u32 + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (sbase - raw_u32);
  // with a causal or window mask the last query tiles see the most keys: rank 0 is the last tile
  int unit, rank;
  block_order(static_cast<int>(blockIdx.x), p.B * p.Hq, p.ntiles, p.chunk_q, unit, rank);
  const int i = (p.mask_kind == ATTN_MASK_FULL) ? rank : p.ntiles - 1 - rank;
  const int h = unit % p.Hq, b = unit / p.Hq;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int klo, khi;
  k_tiles_of_q_tile(p, i, klo, khi);
  const int iters = khi - klo + 1;
  const int kvh = h / p.group;

  const uint32_t bars = sbase + Q::kBarOff;
  auto bar = [&](int x) -> uint32_t { return bars + 8u * static_cast<uint32_t>(x); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Q::kBarOff + kDqTmemSlot);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Q::kBarOff + kDqAbort);
  if (threadIdx.x == 0) {
    mbar_init(bar(kDqQ), 1);
    for (int s = 0; s < Q::kKStages; ++s) {
      mbar_init(bar(kDqFullK + s), 1);
      mbar_init(bar(kDqEmptyK + s), 1);
    }
    for (int s = 0; s < Q::kVStages; ++s) {
      mbar_init(bar(kDqFullV + s), 1);
      mbar_init(bar(kDqEmptyV + s), 1);
    }
    mbar_init(bar(kDqS), 1);
    for (int s = 0; s < 2; ++s) mbar_init(bar(kDqP + s), kBwdSoftWarps);
    mbar_init(bar(kDqAcc), 1);
    mbar_init(bar(kDqDrain), 1);
    mbar_init(bar(kDqDPFree), kBwdSoftWarps);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kBwdMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const long long budget = p.budget;

  if (warp == kBwdTmaWarp) {
    if (lane == 0) {
      // ---------------------------------------------------------- TMA producer
      const int zq = b * p.Hq + h, zkv = b * p.Hkv + kvh;
      mbar_arrive_expect_tx(bar(kDqQ), 2 * C::kTile);
      for (int hh = 0; hh < C::kHalves; ++hh) {
        tma_load_3d(sbase + Q::kQOff + hh * kBox, &tm_q, bar(kDqQ), hh * 64, i * kT, zq);
        tma_load_3d(sbase + Q::kDoOff + hh * kBox, &tm_do, bar(kDqQ), hh * 64, i * kT, zq);
      }
      int nk[Q::kKStages] = {}, nv[Q::kVStages] = {};  // loads issued per stage
      bool ok = true;
      for (int t = 0; t < iters && ok; ++t) {
        const int jt = klo + t;
        const int sk = t % Q::kKStages, sv = t % Q::kVStages;
        // K of key tile t: its stage held K(t - 3), released after dQ(t - 3)
        if (nk[sk] > 0 && !mbar_wait_bounded(bar(kDqEmptyK + sk), (nk[sk] - 1) & 1, budget, abort_flag)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(bar(kDqFullK + sk), C::kTile);
        for (int hh = 0; hh < C::kHalves; ++hh)
          tma_load_3d(sbase + Q::kKOff + sk * C::kTile + hh * kBox, &tm_k, bar(kDqFullK + sk), hh * 64, jt * kT, zkv);
        ++nk[sk];
        // V of key tile t: its stage held V(t - 2), released after dP(t - 2)
        if (nv[sv] > 0 && !mbar_wait_bounded(bar(kDqEmptyV + sv), (nv[sv] - 1) & 1, budget, abort_flag)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(bar(kDqFullV + sv), C::kTile);
        for (int hh = 0; hh < C::kHalves; ++hh)
          tma_load_3d(sbase + Q::kVOff + sv * C::kTile + hh * kBox, &tm_v, bar(kDqFullV + sv), hh * 64, jt * kT, zkv);
        ++nv[sv];
      }
      if (!ok) bwd_abort(abort_flag, p.status);
      // every issued copy has landed before the CTA can exit
      volatile int never = 0;
      mbar_wait_bounded(bar(kDqQ), 0, kDrainBudgetCycles, &never);
      for (int s = 0; s < Q::kKStages; ++s)
        if (nk[s] > 0) mbar_wait_bounded(bar(kDqFullK + s), (nk[s] - 1) & 1, kDrainBudgetCycles, &never);
      for (int s = 0; s < Q::kVStages; ++s)
        if (nv[s] > 0) mbar_wait_bounded(bar(kDqFullV + s), (nv[s] - 1) & 1, kDrainBudgetCycles, &never);
    }
  } else if (warp == kBwdMmaWarp) {
    // ------------------------------------------------------------ MMA issuer (whole warp)
    const uint64_t dq = desc_sw128(sbase + Q::kQOff, 16, 1024);
    const uint64_t ddo = desc_sw128(sbase + Q::kDoOff, 16, 1024);
    constexpr uint32_t kIdS = idesc_bwd(kT, kT, 0, 0);   // S = Q K^T, dP = dO V^T
    constexpr uint32_t kIdAcc = idesc_bwd(kT, D, 0, 1);  // dQ += dS K (K as an MN-major B)
    // Two S buffers (columns kColS and kColS2): S of key tile t + 1 is computed
    // while the dS warps work on tile t; dP has one buffer, refilled once they
    // have loaded it.
    auto col_s = [&](int t) -> uint32_t { return (t & 1) ? C::kColS2 : C::kColS; };
    auto k_at = [&](int t) -> uint32_t { return sbase + Q::kKOff + (t % Q::kKStages) * C::kTile; };
    auto v_at = [&](int t) -> uint32_t { return sbase + Q::kVOff + (t % Q::kVStages) * C::kTile; };
    auto wait = [&](uint32_t b_, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait_bounded(b_, parity, budget, abort_flag));
    };
    auto wait_k = [&](int t) -> bool {
      if (!wait(bar(kDqFullK + t % Q::kKStages), (t / Q::kKStages) & 1)) return false;
      tc_fence_after();
      return true;
    };
    auto wait_v = [&](int t) -> bool {
      if (!wait(bar(kDqFullV + t % Q::kVStages), (t / Q::kVStages) & 1)) return false;
      tc_fence_after();
      return true;
    };
    // dP of key tile t, then release its V stage
    auto issue_dp = [&](int t) {
      mma_kmajor<D>(tmem + C::kColDP, ddo, desc_sw128(v_at(t), 16, 1024), kIdS);
      tc_commit_w(bar(kDqEmptyV + t % Q::kVStages));
      tc_commit_w(bar(kDqS));
    };
    bool ok = wait(bar(kDqQ), 0) && wait_k(0) && wait_v(0);
    if (ok) {
      mma_kmajor<D>(tmem + col_s(0), dq, desc_sw128(k_at(0), 16, 1024), kIdS);
      issue_dp(0);
    }
    for (int t = 0; t < iters && ok; ++t) {
      const bool next = t + 1 < iters;
      // S of the next key tile into the other buffer (its previous dS was consumed by
      // the dQ MMA issued in the last iteration, in order)
      if (next) {
        if (!wait_k(t + 1)) {
          ok = false;
          break;
        }
        mma_kmajor<D>(tmem + col_s(t + 1), dq, desc_sw128(k_at(t + 1), 16, 1024), kIdS);
      }
      if (next) {  // dP of the next key tile, as soon as the dS warps have loaded this one
        if (!wait(bar(kDqDPFree), t & 1) || !wait_v(t + 1)) {
          ok = false;
          break;
        }
        issue_dp(t + 1);
      }
      if (!wait(bar(kDqP + (t & 1)), (t >> 1) & 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
      mma_tmem_a(tmem + C::kColAcc0, tmem + col_s(t), desc_sw128(k_at(t), kBox, 1024), kIdAcc, t == 0);
      tc_commit_w(bar(kDqEmptyK + t % Q::kKStages));
    }
    if (!ok && lane == 0) bwd_abort(abort_flag, p.status);
    tc_commit_w(bar(kDqAcc));
    tc_commit_w(bar(kDqDrain));
    volatile int never = 0;
    mbar_wait_bounded(bar(kDqDrain), 0, kDrainBudgetCycles, &never);
    __syncwarp();
  } else {
    // ------------------------------------------------------------ dS warps 0-7
    const int r = (warp & 3) * 32 + lane;  // query row of the tile = TMEM lane
    const int ch = warp >> 2;              // key columns 64 ch .. 64 ch + 63
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const int qpos = i * kT + r;
    const size_t row = (static_cast<size_t>(b) * p.Hq + h) * p.N + qpos;
    const size_t prow = (static_cast<size_t>(b) * p.Hq + h) * p.npad + qpos;
    const float l2 = p.lse2[prow];
    const float dr = p.dvec[prow];
    const float sl2 = p.scale_log2;
    bool ok = true;
    for (int t = 0; t < iters; ++t) {
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait_bounded(bar(kDqS), t & 1, budget, abort_flag));
      if (!ok) break;
      tc_fence_after();
      const int jt = klo + t;
      const uint32_t colS = (t & 1) ? C::kColS2 : C::kColS;  // this key tile's S buffer
      const bool full_tile = (p.mask_kind == ATTN_MASK_FULL || (i > jt && (p.mask_kind == ATTN_MASK_CAUSAL ||
                                                                           (i * kT + kT - 1) - jt * kT < p.window))) &&
                             (i * kT + kT <= p.N) && (jt * kT + kT <= p.N);
      // both chunks of dP and S at once: once dP is in registers the MMA warp may refill it
      uint32_t dpa[2][32], sva[2][32];
      tmem_ld_32x32b_x32(lane_base + C::kColDP + 32u * (2 * ch), dpa[0]);
      tmem_ld_32x32b_x32(lane_base + C::kColDP + 32u * (2 * ch + 1), dpa[1]);
      tmem_ld_32x32b_x32(lane_base + colS + 32u * (2 * ch), sva[0]);
      tmem_ld_32x32b_x32(lane_base + colS + 32u * (2 * ch + 1), sva[1]);
      tc_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kDqDPFree));
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        const int c = 2 * ch + cc;  // 32-column chunk of the tile
        uint32_t* sv = sva[cc];
        const uint32_t* dpv = dpa[cc];
        if (!full_tile) {
          // hidden (query, key) entries: a score of -inf makes P exactly 0 (scale_log2 > 0)
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int kpos = jt * kT + 32 * c + e;
            if (!(qpos < p.N && kpos < p.N && bwd_visible(p, qpos, kpos))) sv[e] = __float_as_uint(-INFINITY);
          }
        }
        // paired fp32 instructions, rounded as their scalar forms: P = 2^(s scale log2 e - LSE2),
        // dS = P (dP - D)
        const float2 sl2v = make_float2(sl2, sl2), nl2v = make_float2(-l2, -l2), ndr = make_float2(-dr, -dr);
        uint32_t dsk[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const float2 x = ffma2(make_float2(__uint_as_float(sv[e]), __uint_as_float(sv[e + 1])), sl2v, nl2v);
          const float2 pr = make_float2(exp2_approx(x.x), exp2_approx(x.y));
          const float2 ds = fmul2(pr, fadd2(make_float2(__uint_as_float(dpv[e]), __uint_as_float(dpv[e + 1])), ndr));
          dsk[e >> 1] = pack_bf16x2(ds.x, ds.y);
        }
        tmem_st_32x32b_x16(lane_base + colS + 64u * ch + 16u * cc, dsk);  // dS as bf16 pairs, own half
      }
      tc_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kDqP + (t & 1)));
    }
    // ------------------------------------------------------------ epilogue
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait_bounded(bar(kDqAcc), 0, budget, abort_flag));
    if (!ok) bwd_abort(abort_flag, p.status);
    tc_fence_after();
    // TMEM loads are warp-collective: every lane runs them, only rows < N are stored
    const bool store = qpos < p.N;
    __nv_bfloat16* dqrow = p.dq + (store ? row : 0) * D;
#pragma unroll 1
    for (int c = ch * (D / 64); c < (ch + 1) * (D / 64); ++c) {  // this warp's half of the head dim
      uint32_t qa[32];
      tmem_ld_32x32b_x32(lane_base + C::kColAcc0 + 32u * c, qa);
      tc_wait_ld();
#pragma unroll
      for (int e = 0; e < 32; e += 8) {
        uint32_t pq[4];
#pragma unroll
        for (int u = 0; u < 8; u += 2)
          pq[u >> 1] = pack_bf16x2(ok ? __uint_as_float(qa[e + u]) * p.scale : NAN,
                                   ok ? __uint_as_float(qa[e + u + 1]) * p.scale : NAN);
        if (store) *reinterpret_cast<uint4*>(dqrow + 32 * c + e) = make_uint4(pq[0], pq[1], pq[2], pq[3]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kBwdMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// [heads][n][d] bf16 as a rank-3 tensor (d innermost), 64-column x 128-row boxes, 128-byte swizzle.
bool encode_bwd(CUtensorMap* map, const void* base, int d, int n, int heads) {
  const auto enc = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(tensor_map_encode_fn());
  if (enc == nullptr) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(n),
                              static_cast<cuuint64_t>(heads)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(n) * d * 2};
  const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(kT), 1};
  const cuuint32_t estride[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estride,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
int launch_backward_t(const void* q, const void* k, const void* v, const void* o, const void* d_o, const float* lse,
                      void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int N, int mask_kind, int window,
                      float scale, void* workspace, int32_t* status, cudaStream_t stream) {
  CUtensorMap tq, tk, tv, tdo;
  if (!encode_bwd(&tq, q, D, N, B * Hq) || !encode_bwd(&tk, k, D, N, B * Hkv) || !encode_bwd(&tv, v, D, N, B * Hkv) ||
      !encode_bwd(&tdo, d_o, D, N, B * Hq))
    return ATTN_ERR_CUDA;
  BwdParams p;
  p.o = static_cast<const __nv_bfloat16*>(o);
  p.d_o = static_cast<const __nv_bfloat16*>(d_o);
  p.lse = lse;
  p.ntiles = (N + kT - 1) / kT;
  p.npad = p.ntiles * kT;
  p.dvec = static_cast<float*>(workspace);
  p.lse2 = p.dvec + static_cast<size_t>(B) * Hq * p.npad;
  p.dq = static_cast<__nv_bfloat16*>(dq);
  p.dk = static_cast<__nv_bfloat16*>(dk);
  p.dv = static_cast<__nv_bfloat16*>(dv);
  p.status = status;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.N = N;
  p.group = Hq / Hkv;
  p.mask_kind = mask_kind;
  p.window = window;
  p.scale = scale;
  p.scale_log2 = scale * kLog2e;
  p.budget = wait_budget_cycles();
  // Scheduling chunks of the dK/dV kernel: the K/V heads are split into as few equal chunks as
  // keep the Q and dO tiles that a chunk's blocks read (its query heads' rows; under a window
  // mask only the window's span of the sequence) within about 96 MB of L2. Its blocks differ
  // most in size (key tile 0 of a causal mask reads every query tile), so the longest first
  // pays; for the dQ kernel one head at a time (chunks of 1) measured as fast as any chunking.
  const int span = (mask_kind == ATTN_MASK_SLIDING_WINDOW) ? std::min(N, window + kT) : N;
  const double head_bytes = static_cast<double>(span) * D * 2, budget_bytes = 96.0 * 1024 * 1024;
  const int units_kv = B * Hkv;
  const double chunks = std::min(static_cast<double>(units_kv),
                                 std::max(1.0, std::ceil(units_kv * 2.0 * p.group * head_bytes / budget_bytes)));
  p.chunk_kv = std::max(1, static_cast<int>(std::ceil(units_kv / chunks)));
  p.chunk_q = 1;
  const size_t rows = static_cast<size_t>(B) * Hq * p.npad;
  bwd_rowdot_kernel<D><<<static_cast<unsigned>((rows + 7) / 8), 256, 0, stream>>>(p);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  constexpr int smem_dkdv = BwdCfg<D>::kAlloc, smem_dq = DqCfg<D>::kAlloc;
  if (cudaFuncSetAttribute(bwd_dkdv_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_dkdv) != cudaSuccess ||
      cudaFuncSetAttribute(bwd_dq_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_dq) != cudaSuccess)
    return ATTN_ERR_CUDA;
  bwd_dkdv_kernel<D><<<B * Hkv * p.ntiles, kBwdThreads, smem_dkdv, stream>>>(tq, tk, tv, tdo, p);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  bwd_dq_kernel<D><<<B * Hq * p.ntiles, kBwdThreads, smem_dq, stream>>>(tq, tk, tv, tdo, p);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // namespace

size_t backward_workspace_bytes(int B, int Hq, int N) {
  const size_t npad = static_cast<size_t>((N + kT - 1) / kT) * kT;
  return 2 * static_cast<size_t>(B) * Hq * npad * sizeof(float);  // D, then LSE * log2(e)
}

int launch_backward(const void* q, const void* k, const void* v, const void* o, const void* d_o, const float* lse,
                    void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int N, int d, int mask_kind, int window,
                    float scale, void* workspace, int32_t* status, cudaStream_t stream) {
  if (d == 128)
    return launch_backward_t<128>(q, k, v, o, d_o, lse, dq, dk, dv, B, Hq, Hkv, N, mask_kind, window, scale,
                                  workspace, status, stream);
  return launch_backward_t<64>(q, k, v, o, d_o, lse, dq, dk, dv, B, Hq, Hkv, N, mask_kind, window, scale, workspace,
                               status, stream);
}

}  // namespace attn
