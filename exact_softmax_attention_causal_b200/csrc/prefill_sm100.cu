// Prefill attention on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// What it computes ("Module 5. Modern Attention Mechanisms", section 4):
// O = softmax(scale * Q K^T + M) V per query head, M the full / causal /
// sliding-window mask (key j visible to query i iff j <= i, and i - j < W for
// the window), with query head h reading K/V head h / (Hq / Hkv) (section 6),
// and LSE = log sum_j exp(scale * q_i . k_j) over the visible keys.
//
// How: FlashAttention's online softmax (section 8 of the same page; the
// "Inference attention" post, section "FlashAttention"): one CTA owns a
// 128-row query tile of one (batch, head) and streams 128-key tiles of K and
// V, never writing scores to HBM. Tiles entirely above the diagonal or left
// of the window are never visited; only the tiles that straddle a mask edge
// evaluate the mask per element.
//
// Roles (192 threads, one CTA per SM):
//   warps 0-3  softmax: thread i owns query row i = TMEM lane i. Reads a
//              128-column score row from TMEM, applies scale (folded with
//              log2 e) and mask, updates the running max and sum, writes the
//              probabilities back to TMEM as bf16 and, when needed, rescales
//              the output accumulator in TMEM; finally O / l -> bf16 and LSE.
//   warp 4     TMA producer: Q once, then K and V tiles into a ring of
//              shared-memory stages (128-byte swizzle, 64-column boxes).
//   warp 5     MMA issuer: S_j = Q K_j^T (both operands in shared memory) into
//              one of two TMEM score buffers, and O += P_j V_j with P read
//              straight from TMEM. Allocates and frees the 512 TMEM columns.
// The score MMA of tile j+1 runs while the softmax works on tile j.
//
// Lazy rescaling: the running max used for the exponentials only moves when
// the true running max exceeds it by more than 8 (base 2). Every p stays
// <= 2^8 and both the output and the sum are taken relative to the same
// max, so the result is exact up to rounding (the FlashAttention-4 idea of
// skipping most rescales, as the "Inference attention" post describes it).
//
// All pipeline waits are bounded; on expiry the CTA records
// ATTN_STATUS_BIT_TIMEOUT, writes NaN rows, drains its copies and MMAs
// (bounded again), frees TMEM and exits.

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "internal.h"
#include "ptx.cuh"

namespace attn {
namespace {

constexpr int kBM = 128;  // query rows per tile (= TMEM lanes)
constexpr int kBN = 128;  // keys per tile
constexpr int kPfThreads = 192;
constexpr float kRescaleThreshold = 8.0f;

template <int D>
struct PfCfg {
  static constexpr int kHalf = 128 * 128;    // bytes of one 64-column box of 128 rows
  static constexpr int kHalves = D / 64;     // 128-byte swizzle columns per tile
  static constexpr int kTile = kHalves * kHalf;
  static constexpr int kStages = (D == 128) ? 2 : 4;
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kQOff + kTile;
  static constexpr int kVOff = kKOff + kStages * kTile;
  static constexpr int kBarOff = kVOff + kStages * kTile;
  static constexpr int kBytes = kBarOff + 256;
  static constexpr int kAlloc = kBytes + 1024;  // slack to align the base to 1024 bytes
  // TMEM column map (512 columns allocated)
  static constexpr uint32_t kColS0 = 0;
  static constexpr uint32_t kColS1 = 128;
  static constexpr uint32_t kColO = 256;
  static constexpr uint32_t kColP = 384;  // 128 bf16 probabilities = 64 columns
};

// Barrier slots inside the barrier block (8 bytes each).
enum : int {
  kBarQFull = 0,
  kBarKFull = 1,   // + stage (up to 4)
  kBarVFull = 5,   // + stage
  kBarKEmpty = 9,  // + stage
  kBarVEmpty = 13, // + stage
  kBarSFull = 17,  // + buffer (2)
  kBarPFull = 19,
  kBarODone = 20,
  kBarDrain = 21,
  kNumBars = 22,
};
constexpr int kTmemSlotOff = 192;
constexpr int kAbortOff = 196;

// Shared-memory matrix descriptor, 128-byte swizzle (tcgen05 format: start
// address, leading and stride byte offsets in 16-byte units, version 1,
// layout type 2 = SWIZZLE_128B).
__device__ __forceinline__ uint64_t desc_sw128(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) |
         (static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16) |
         (static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor for kind::f16: fp32 accumulate, bf16 A and B, A
// K-major, B K-major (0) or MN-major (1), N >> 3 at bit 17, M >> 4 at bit 24.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, int b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(b_mn_major) << 16) |
         (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

struct PrefillParams {
  __nv_bfloat16* o;
  float* lse;
  int32_t* status;
  int B, Hq, Hkv, N, group, mask_kind, window, num_q_tiles;
  float scale_log2;
  long long budget;
};

// Key tiles a query tile visits: [lo, hi], inclusive.
__device__ __forceinline__ void kv_tile_range(const PrefillParams& p, int q0, int& lo, int& hi) {
  hi = (p.N - 1) / kBN;
  lo = 0;
  if (p.mask_kind != ATTN_MASK_FULL) hi = min(hi, (q0 + kBM - 1) / kBN);
  if (p.mask_kind == ATTN_MASK_SLIDING_WINDOW) lo = max(0, q0 - p.window + 1) / kBN;
}

// True when every (row, key) pair of the tile is visible, so no per-element mask is needed.
__device__ __forceinline__ bool tile_is_full(const PrefillParams& p, int q0, int k0) {
  bool full = (k0 + kBN <= p.N);
  if (p.mask_kind != ATTN_MASK_FULL) full = full && (k0 + kBN - 1 <= q0);
  if (p.mask_kind == ATTN_MASK_SLIDING_WINDOW) full = full && (q0 + kBM - 1 - k0 < p.window);
  return full;
}

__device__ __forceinline__ bool key_visible(const PrefillParams& p, int qi, int kj) {
  if (kj >= p.N) return false;
  if (p.mask_kind == ATTN_MASK_FULL) return true;
  if (kj > qi) return false;
  return p.mask_kind != ATTN_MASK_SLIDING_WINDOW || (qi - kj < p.window);
}

__device__ __forceinline__ void raise_abort(volatile int* abort_flag, int32_t* status) {
  *abort_flag = 1;
  if (status != nullptr) atomicOr(status, ATTN_STATUS_BIT_TIMEOUT);
}

template <int D>
__global__ void __launch_bounds__(kPfThreads, 1)
    prefill_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const PrefillParams p) {
  using C = PfCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  const uint32_t sbase = (raw_u32 + 1023u) & ~1023u;  // swizzled tiles need 1024-byte alignment
  uint8_t* smem = smem_raw + (sbase - raw_u32);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int h = blockIdx.x;
  const int b = blockIdx.y;
  // heaviest query tiles first when the mask makes work grow with the tile index
  const int qt = (p.mask_kind == ATTN_MASK_FULL) ? blockIdx.z : (p.num_q_tiles - 1 - blockIdx.z);
  const int q0 = qt * kBM;
  const int kvh = h / p.group;
  int kt_lo, kt_hi;
  kv_tile_range(p, q0, kt_lo, kt_hi);
  const int T = kt_hi - kt_lo + 1;

  const uint32_t bars = sbase + C::kBarOff;
  auto bar = [&](int i) -> uint32_t { return bars + 8u * static_cast<uint32_t>(i); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kBarOff + kTmemSlotOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kBarOff + kAbortOff);

  if (threadIdx.x == 0) {
    mbar_init(bar(kBarQFull), 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(bar(kBarKFull + s), 1);
      mbar_init(bar(kBarVFull + s), 1);
      mbar_init(bar(kBarKEmpty + s), 1);
      mbar_init(bar(kBarVEmpty + s), 1);
    }
    mbar_init(bar(kBarSFull + 0), 1);
    mbar_init(bar(kBarSFull + 1), 1);
    mbar_init(bar(kBarPFull), kBM);
    mbar_init(bar(kBarODone), 1);
    mbar_init(bar(kBarDrain), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const long long budget = p.budget;

  if (warp == 4) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      const int zq = b * p.Hq + h;
      const int zkv = b * p.Hkv + kvh;
      mbar_arrive_expect_tx(bar(kBarQFull), C::kTile);
      for (int hh = 0; hh < C::kHalves; ++hh)
        tma_load_3d(sbase + C::kQOff + hh * C::kHalf, &tm_q, bar(kBarQFull), hh * 64, q0, zq);
      // K_i is issued before V_{i-1}: the score MMA needs K one tile earlier than PV needs V.
      int k_issued = 0, v_issued = 0;
      bool ok = true;
      for (int i = 0; i <= T && ok; ++i) {
        if (i < T) {
          const int s = i % C::kStages, round = i / C::kStages;
          if (round > 0 && !mbar_wait_bounded(bar(kBarKEmpty + s), (round - 1) & 1, budget, abort_flag)) {
            ok = false;
            break;
          }
          const int k0 = (kt_lo + i) * kBN;
          mbar_arrive_expect_tx(bar(kBarKFull + s), C::kTile);
          for (int hh = 0; hh < C::kHalves; ++hh)
            tma_load_3d(sbase + C::kKOff + s * C::kTile + hh * C::kHalf, &tm_k, bar(kBarKFull + s), hh * 64, k0,
                        zkv);
          k_issued = i + 1;
        }
        if (i >= 1) {
          const int jv = i - 1;
          const int s = jv % C::kStages, round = jv / C::kStages;
          if (round > 0 && !mbar_wait_bounded(bar(kBarVEmpty + s), (round - 1) & 1, budget, abort_flag)) {
            ok = false;
            break;
          }
          const int k0 = (kt_lo + jv) * kBN;
          mbar_arrive_expect_tx(bar(kBarVFull + s), C::kTile);
          for (int hh = 0; hh < C::kHalves; ++hh)
            tma_load_3d(sbase + C::kVOff + s * C::kTile + hh * C::kHalf, &tm_v, bar(kBarVFull + s), hh * 64, k0,
                        zkv);
          v_issued = jv + 1;
        }
      }
      if (!ok) raise_abort(abort_flag, p.status);
      // Drain: the newest copy of every stage has landed before the CTA may exit.
      volatile int never = 0;
      mbar_wait_bounded(bar(kBarQFull), 0, kDrainBudgetCycles, &never);
      for (int j = (k_issued > C::kStages ? k_issued - C::kStages : 0); j < k_issued; ++j)
        mbar_wait_bounded(bar(kBarKFull + j % C::kStages), (j / C::kStages) & 1, kDrainBudgetCycles, &never);
      for (int j = (v_issued > C::kStages ? v_issued - C::kStages : 0); j < v_issued; ++j)
        mbar_wait_bounded(bar(kBarVFull + j % C::kStages), (j / C::kStages) & 1, kDrainBudgetCycles, &never);
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16(kBM, kBN, 0);
      constexpr uint32_t idesc_pv = idesc_bf16(kBM, D, 1);
      const uint32_t sQ = sbase + C::kQOff;
      bool ok = mbar_wait_bounded(bar(kBarQFull), 0, budget, abort_flag);
      auto issue_s = [&](int j) -> bool {
        const int s = j % C::kStages;
        if (!mbar_wait_bounded(bar(kBarKFull + s), (j / C::kStages) & 1, budget, abort_flag)) return false;
        tc_fence_after();
        const uint32_t sK = sbase + C::kKOff + s * C::kTile;
        const uint32_t d_col = tmem + ((j & 1) ? C::kColS1 : C::kColS0);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t koff = (kk >> 2) * C::kHalf + (kk & 3) * 32;
          tc_mma_ss(d_col, desc_sw128(sQ + koff, 16, 1024), desc_sw128(sK + koff, 16, 1024), idesc_qk,
                    kk > 0 ? 1u : 0u);
        }
        tc_commit(bar(kBarSFull + (j & 1)));
        tc_commit(bar(kBarKEmpty + s));
        return true;
      };
      if (ok) ok = issue_s(0);
      for (int j = 0; j < T && ok; ++j) {
        if (j + 1 < T && !issue_s(j + 1)) {
          ok = false;
          break;
        }
        const int s = j % C::kStages;
        if (!mbar_wait_bounded(bar(kBarPFull), j & 1, budget, abort_flag) ||
            !mbar_wait_bounded(bar(kBarVFull + s), (j / C::kStages) & 1, budget, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sV = sbase + C::kVOff + s * C::kTile;
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {
          // 16 keys per step: P columns [8 kk, 8 kk + 8), V rows [16 kk, 16 kk + 16)
          tc_mma_ts(tmem + C::kColO, tmem + C::kColP + kk * 8, desc_sw128(sV + kk * 2048, C::kHalf, 1024), idesc_pv,
                    (j > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(bar(kBarODone));
        tc_commit(bar(kBarVEmpty + s));
      }
      if (!ok) raise_abort(abort_flag, p.status);
      // Drain: every MMA this thread issued has completed before TMEM is freed.
      tc_commit(bar(kBarDrain));
      volatile int never = 0;
      mbar_wait_bounded(bar(kBarDrain), 0, kDrainBudgetCycles, &never);
    }
  } else {
    // ------------------------------------------------------------ softmax warps 0-3
    const int r = threadIdx.x;  // tile row = TMEM lane
    const int qi = q0 + r;      // query position
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    float m_used = -INFINITY;   // max the exponentials are taken against (base 2)
    float l_sum = 0.f;          // running sum of 2^(x - m_used), fp32
    bool ok = true;
    for (int j = 0; j < T; ++j) {
      const int k0 = (kt_lo + j) * kBN;
      ok = __all_sync(0xffffffffu, mbar_wait_bounded(bar(kBarSFull + (j & 1)), (j >> 1) & 1, budget, abort_flag));
      if (!ok) break;
      tc_fence_after();
      uint32_t sr[kBN];
      const uint32_t scol = lane_base + ((j & 1) ? C::kColS1 : C::kColS0);
#pragma unroll
      for (int c = 0; c < kBN / 32; ++c)
        tmem_ld_32x32b_x32(scol + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]));
      tc_wait_ld();

      const bool full = tile_is_full(p, q0, k0);
      float mt = -INFINITY;
#pragma unroll
      for (int c = 0; c < kBN; ++c) {
        float x = __uint_as_float(sr[c]) * p.scale_log2;
        if (!full && !key_visible(p, qi, k0 + c)) x = -INFINITY;
        sr[c] = __float_as_uint(x);
        mt = fmaxf(mt, x);
      }
      const float m_new = fmaxf(m_used, mt);
      bool rescale_o = false;
      float factor = 1.f;
      if (m_new > m_used + kRescaleThreshold) {  // also true for the first visible key (m_used = -inf)
        const bool prev_finite = (m_used != -INFINITY);
        factor = prev_finite ? fast_exp2(m_used - m_new) : 0.f;
        l_sum *= factor;
        rescale_o = prev_finite;  // earlier tiles already put visible keys into O
        m_used = m_new;
      }
      if (j > 0) {  // PV_{j-1} done: O is stable and the P buffer is free
        ok = __all_sync(0xffffffffu, mbar_wait_bounded(bar(kBarODone), (j - 1) & 1, budget, abort_flag));
        if (!ok) break;
      }
      tc_fence_after();
      if (__any_sync(0xffffffffu, rescale_o)) {
        const float f = rescale_o ? factor : 1.f;
#pragma unroll
        for (int c = 0; c < D / 16; ++c) {
          uint32_t ov[16];
          tmem_ld_32x32b_x16(lane_base + C::kColO + c * 16, ov);
          tc_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * f);
          tmem_st_32x32b_x16(lane_base + C::kColO + c * 16, ov);
        }
      }
      const float mref = (m_used == -INFINITY) ? 0.f : m_used;  // a row with nothing visible yet gets p = 0
      float rs = 0.f;
#pragma unroll
      for (int cc = 0; cc < kBN / 32; ++cc) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float p0 = fast_exp2(__uint_as_float(sr[cc * 32 + 2 * e]) - mref);
          const float p1 = fast_exp2(__uint_as_float(sr[cc * 32 + 2 * e + 1]) - mref);
          rs += p0 + p1;
          pk[e] = pack_bf16x2(p0, p1);
        }
        tmem_st_32x32b_x16(lane_base + C::kColP + cc * 16, pk);
      }
      tc_wait_st();
      l_sum += rs;
      tc_fence_before();
      mbar_arrive(bar(kBarPFull));
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait_bounded(bar(kBarODone), (T - 1) & 1, budget, abort_flag));
    if (!ok) raise_abort(abort_flag, p.status);
    tc_fence_after();

    // ---- epilogue: O / l -> bf16, LSE (natural log)
    const bool row_valid = qi < p.N;
    __nv_bfloat16* orow = p.o + (static_cast<size_t>(b * p.Hq + h) * p.N + (row_valid ? qi : 0)) * D;
    const float inv_l = ok ? 1.f / l_sum : NAN;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      uint32_t ov[32];
      if (ok) {
        tmem_ld_32x32b_x32(lane_base + C::kColO + c * 32, ov);
        tc_wait_ld();
      }
      uint4 pk[4];
      uint32_t* pw = reinterpret_cast<uint32_t*>(pk);
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const float a0 = ok ? __uint_as_float(ov[2 * e]) * inv_l : NAN;
        const float a1 = ok ? __uint_as_float(ov[2 * e + 1]) * inv_l : NAN;
        pw[e] = pack_bf16x2(a0, a1);
      }
      if (row_valid) {
        uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
        for (int e = 0; e < 4; ++e) dst[e] = pk[e];
      }
    }
    if (row_valid && p.lse != nullptr)
      p.lse[static_cast<size_t>(b * p.Hq + h) * p.N + qi] = ok ? (m_used + __log2f(l_sum)) * kLn2 : NAN;
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

// [heads][n][d] bf16 viewed as a rank-3 tensor (d innermost); box = 64 columns
// x 128 rows x 1 head, 128-byte swizzle. Rows past n read as zero.
bool encode_bhnd(CUtensorMap* map, const void* base, int d, int n, int heads) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(n),
                              static_cast<cuuint64_t>(heads)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(n) * d * 2};
  const cuuint32_t box[3] = {64, 128, 1};
  const cuuint32_t estride[3] = {1, 1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
                         estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int D>
int launch_prefill_t(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int N,
                     int mask_kind, int window, float scale, int32_t* status, cudaStream_t stream) {
  CUtensorMap tq, tk, tv;
  if (!encode_bhnd(&tq, q, D, N, B * Hq) || !encode_bhnd(&tk, k, D, N, B * Hkv) ||
      !encode_bhnd(&tv, v, D, N, B * Hkv))
    return ATTN_ERR_CUDA;
  PrefillParams p;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.status = status;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.N = N;
  p.group = Hq / Hkv;
  p.mask_kind = mask_kind;
  p.window = window;
  p.num_q_tiles = (N + kBM - 1) / kBM;
  p.scale_log2 = scale * kLog2e;
  p.budget = wait_budget_cycles();
  constexpr int smem = PfCfg<D>::kAlloc;
  if (cudaFuncSetAttribute(prefill_fwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return ATTN_ERR_CUDA;
  const dim3 grid(Hq, B, p.num_q_tiles);
  prefill_fwd_kernel<D><<<grid, kPfThreads, smem, stream>>>(tq, tk, tv, p);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // namespace

int launch_prefill(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int N,
                   int d, int mask_kind, int window, float scale, int32_t* status, cudaStream_t stream) {
  if (d == 128) return launch_prefill_t<128>(q, k, v, o, lse, B, Hq, Hkv, N, mask_kind, window, scale, status, stream);
  return launch_prefill_t<64>(q, k, v, o, lse, B, Hq, Hkv, N, mask_kind, window, scale, status, stream);
}

}  // namespace attn
