// Prefill attention on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// What it computes ("Module 5. Modern Attention Mechanisms", section 4):
// O = softmax(scale * Q K^T + M) V per query head, M the full / causal /
// sliding-window mask (key j visible to query i iff j <= i, and i - j < W for
// the window), with query head h reading K/V head h / (Hq / Hkv) (section 6),
// and LSE = log sum_j exp(scale * q_i . k_j) over the visible keys.
//
// How: FlashAttention's online softmax (section 8 of the same page; the
// "Inference attention" post, section "FlashAttention"), never writing scores
// to HBM. A work item is 256 query rows (two 128-row tiles A and B) of one
// (batch, head); it streams 128-key tiles of K and V, each loaded once for
// both tiles. Key tiles entirely above the diagonal or left of the window are
// never visited; only tiles that straddle a mask edge evaluate the mask per
// element.
//
// Persistent schedule: one CTA per SM walks a share of the items, heaviest
// first, handed out in snake order so the per-CTA totals stay even. Across
// items the K/V ring keeps streaming, the next item's Q loads as soon as the
// current item's last score MMA has read Q, and its first score MMAs overlap
// the current item's epilogue.
//
// Roles (384 threads):
//   warps 0-3  softmax of tile A, warps 4-7 softmax of tile B: thread i owns
//              query row i of its tile = TMEM lane i. Reads the 128-column
//              score row from TMEM, applies scale (folded with log2 e) and,
//              on edge tiles only, the mask; updates the running max and sum;
//              rescales its output row in TMEM when the max moved; writes the
//              probabilities back as bf16 over the consumed score columns, in
//              two halves each announced on its own barrier; finally
//              O / l -> bf16 and LSE.
//   warp 8     TMA producer: both Q tiles per item, then K and V tiles into a
//              ring of shared-memory stages (128-byte swizzle, 64-column boxes).
//   warp 9     MMA issuer: S_X = Q_X K_j^T (both operands in shared memory) and
//              O_X += P_X V_j with P_X read straight from TMEM, alternating
//              between the tiles so the tensor core works on one tile while
//              the other tile's softmax runs. Allocates and frees TMEM.
//   warps 10-11 idle (they complete the register-donating warpgroup).
// A tile's score barrier is committed after its previous P.V, so when the
// softmax sees new scores its output accumulator is stable and may be
// rescaled in place.
//
// Lazy rescaling: the running max used for the exponentials only moves when
// the true running max exceeds it by more than 8 (base 2). Every p stays
// <= 2^8 and both the output and the sum are taken relative to the same
// max, so the result is exact up to rounding (the FlashAttention-4 idea of
// skipping most rescales, as the "Inference attention" post describes it).
//
// All pipeline waits are bounded; on expiry the CTA records
// ATTN_STATUS_BIT_TIMEOUT, writes NaN rows for every item it has left, drains
// its copies and MMAs (bounded again), frees TMEM and exits.

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "internal.h"
#include "ptx.cuh"

namespace attn {
namespace {

constexpr int kBM = 128;  // query rows per tile (= TMEM lanes)
constexpr int kBN = 128;  // keys per tile
constexpr int kTilesPerCta = 2;
constexpr int kRowsPerCta = kTilesPerCta * kBM;
constexpr int kPfThreads = 384;  // 8 softmax warps + a warpgroup holding the TMA and MMA warps
constexpr int kTmaWarp = 8;
constexpr int kMmaWarp = 9;
// Register split (per thread): launched with 168 (65536 / 384, rounded down to
// a multiple of 8 and capped by the 16K-register sub-partition holding three
// warps); the TMA/MMA warpgroup gives registers back, the softmax warpgroups
// take them: 256 x 224 + 128 x 56 = 384 x 168 = 64512.
constexpr uint32_t kRegsLaunch = 168;
constexpr uint32_t kRegsSoftmax = 224;
constexpr uint32_t kRegsControl = 56;
static_assert(256 * kRegsSoftmax + 128 * kRegsControl == kPfThreads * kRegsLaunch, "register split");
static_assert(2 * kRegsSoftmax * 32 + kRegsControl * 32 <= 16384, "per sub-partition register file");
constexpr float kRescaleThreshold = 8.0f;

template <int D>
struct PfCfg {
  static constexpr int kHalf = 128 * 128;    // bytes of one 64-column box of 128 rows
  static constexpr int kHalves = D / 64;     // 128-byte swizzle columns per tile
  static constexpr int kTile = kHalves * kHalf;
  static constexpr int kKStages = (D == 128) ? 2 : 4;  // K ring depth
  static constexpr int kVStages = (D == 128) ? 2 : 4;  // V ring depth
  static constexpr int kQOff = 0;            // Q tile A, then Q tile B
  static constexpr int kKOff = kQOff + kTilesPerCta * kTile;
  static constexpr int kVOff = kKOff + kKStages * kTile;
  // Epilogue staging: per softmax warp 32 rows x 64 columns of bf16 (4 KB, one
  // 128-byte-swizzled TMA store box), written once per 64-column half of O.
  static constexpr int kStageOff = kVOff + kVStages * kTile;
  static constexpr int kStageBytes = 8 * 32 * 128;
  static constexpr int kBarOff = kStageOff + kStageBytes;
  // Paged contexts: work classes (query tile pair, sequence) sorted by their
  // key-tile count, heaviest first (at most kOrderMax classes; else the fixed order).
  static constexpr int kOrderOff = kBarOff + 256;
  static constexpr int kOrderMax = 256;
  static constexpr int kBytes = kOrderOff + kOrderMax * 4;
  static constexpr int kAlloc = kBytes + 1024;  // slack to align the base to 1024 bytes
  static_assert(kAlloc <= 232448, "shared memory per CTA");
  // TMEM columns (512 allocated): scores of A and B (128 fp32 columns each;
  // the bf16 probabilities overwrite their first 64 columns), then outputs.
  __host__ __device__ static constexpr uint32_t col_s(int x) { return x ? 128u : 0u; }
  __host__ __device__ static constexpr uint32_t col_o(int x) { return 256u + static_cast<uint32_t>(x * D); }
};

// Barrier slots inside the barrier block (8 bytes each).
enum : int {
  kBarQFull = 0,
  kBarKFull = 1,    // + stage (up to 4)
  kBarVFull = 5,    // + stage
  kBarKEmpty = 9,   // + stage
  kBarVEmpty = 13,  // + stage
  kBarSFull = 17,   // + tile (2)
  kBarPLo = 19,     // + tile: probabilities of keys 0-63 written
  kBarPHi = 21,     // + tile: probabilities of keys 64-127 written
  kBarOFinal = 23,  // + tile
  kBarDrain = 25,
  kBarQEmpty = 26,  // both Q tiles consumed by the item's last score MMA
  kNumBars = 27,
};
constexpr int kTmemSlotOff = 224;
constexpr int kAbortOff = 228;

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
  int B, Hq, Hkv, N, group, mask_kind, window, num_cta_tiles;  // N = query rows per sequence
  int num_items;  // num_cta_tiles * Hq * B
  int ordered;    // paged: items follow the per-launch cost order in shared memory
  float scale_log2;
  long long budget;
  // Paged context (prefix prefill): the keys of sequence b are its seq_lens[b]
  // cached tokens, read through block_table; the N query rows are its newest N
  // positions. Unused (null) for the contiguous prefill, where keys = rows = N.
  const int32_t* block_table;  // [B, max_blocks]
  const int32_t* seq_lens;     // [B]
  int max_blocks, block_size, num_blocks, max_seq_len;
};

// One work item: 256 query rows of one (batch, head). Items are numbered
// heaviest first (for causal and window masks the work of a row tile grows
// with its index), heads of a K/V group adjacent so concurrently running CTAs
// share K/V tiles in L2.
struct WorkItem {
  int q0, h, b;
};
// Item w belongs to class w / Hq = rank * B + b (fixed order) or to class
// order[w / Hq] (paged, costs sorted at launch); head w % Hq.
__device__ __forceinline__ WorkItem item_at(const PrefillParams& p, int w, const int* order, bool use_order) {
  const int cls = use_order ? order[w / p.Hq] : w / p.Hq;
  const int rank = cls / p.B;
  const int ct = (p.mask_kind == ATTN_MASK_FULL) ? rank : (p.num_cta_tiles - 1 - rank);
  return WorkItem{ct * kRowsPerCta, w % p.Hq, cls - rank * p.B};
}
// Snake assignment of the heaviest-first list over the persistent CTAs:
// round r hands item r * G + c (r even) or r * G + G - 1 - c (r odd) to CTA c.
__device__ __forceinline__ int item_index(int round, int c, int G) {
  return round * G + ((round & 1) ? (G - 1 - c) : c);
}

// Geometry of one item: nk keys, query row i at position pos0 + i (bottom-right
// alignment: the rows are the newest positions of the sequence), and the key
// tiles [lo, lo + T) its 256 rows see. For a paged context with an out-of-range
// seq_len the item is computed over nk = N and its rows come out as NaN.
struct ItemGeom {
  int nk, pos0, lo, T;
  bool bad;
};
template <bool PAGED>
__device__ __forceinline__ ItemGeom item_geom(const PrefillParams& p, const WorkItem& wi) {
  int nk = p.N;
  bool bad = false;
  if (PAGED) {
    const int sl = __ldg(p.seq_lens + wi.b);
    bad = sl < p.N || sl > p.max_seq_len;
    nk = bad ? p.N : sl;
  }
  const int pos0 = nk - p.N;
  int hi = (nk - 1) / kBN, lo = 0;
  if (p.mask_kind != ATTN_MASK_FULL) hi = min(hi, (pos0 + wi.q0 + kRowsPerCta - 1) / kBN);
  if (p.mask_kind == ATTN_MASK_SLIDING_WINDOW) lo = max(0, pos0 + wi.q0 - p.window + 1) / kBN;
  return ItemGeom{nk, pos0, lo, hi - lo + 1, bad};
}

// Key tiles each query tile of an item needs, relative to the item's first
// key tile: tile A (x = 0) uses [0, a1), tile B (x = 1) uses [b0, T). Tile A's
// rows end one key tile earlier under a causal or window mask, and tile B's
// window starts up to one tile later, so each skips the tile only the other
// needs. A always uses the first key tile and B the last, and together they
// cover all T.
struct TileRanges {
  int a1, b0;
};
__device__ __forceinline__ TileRanges tile_ranges(const PrefillParams& p, const WorkItem& wi, const ItemGeom& gm) {
  int a1 = gm.T, b0 = 0;
  if (p.mask_kind != ATTN_MASK_FULL) {
    const int hi_a = min((gm.nk - 1) / kBN, (gm.pos0 + wi.q0 + kBM - 1) / kBN);
    a1 = hi_a - gm.lo + 1;
  }
  if (p.mask_kind == ATTN_MASK_SLIDING_WINDOW) b0 = max(0, gm.pos0 + wi.q0 + kBM - p.window + 1) / kBN - gm.lo;
  // a tile B wholly past the last row still runs the last key tile (its rows are
  // never stored), so that both tiles finish every item
  return TileRanges{a1, min(b0, gm.T - 1)};
}

// True when every (row, key) pair of a 128 x 128 tile is visible: rows at
// positions [qpos0, qpos0 + 128), keys [k0, k0 + 128) of nk.
__device__ __forceinline__ bool tile_is_full(const PrefillParams& p, int qpos0, int k0, int nk) {
  bool full = (k0 + kBN <= nk);
  if (p.mask_kind != ATTN_MASK_FULL) full = full && (k0 + kBN - 1 <= qpos0);
  if (p.mask_kind == ATTN_MASK_SLIDING_WINDOW) full = full && (qpos0 + kBM - 1 - k0 < p.window);
  return full;
}

__device__ __forceinline__ void raise_abort(volatile int* abort_flag, int32_t* status) {
  *abort_flag = 1;
  if (status != nullptr) atomicOr(status, ATTN_STATUS_BIT_TIMEOUT);
}

// One MMA step of S = Q K^T: descriptors are the operand bases plus a fixed
// offset (16-byte units) added inside the asm, so the compiler cannot hoist a
// descriptor per step into registers.
template <uint32_t OFF, uint32_t IDESC>
__device__ __forceinline__ void mma_ss_step(uint32_t d_tmem, uint64_t a_base, uint64_t b_base, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n .reg .b64 da, db;\n setp.ne.b32 p, %3, 0;\n add.s64 da, %1, %4;\n add.s64 db, %2, %4;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], da, db, %5, p;\n}\n" ::"r"(d_tmem),
      "l"(a_base), "l"(b_base), "r"(accumulate), "n"(OFF), "n"(IDESC)
      : "memory");
}
// One MMA step of O += P V with P in TMEM at column offset ACOL and V at OFF.
template <uint32_t ACOL, uint32_t OFF, uint32_t IDESC>
__device__ __forceinline__ void mma_ts_step(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_base, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n .reg .b32 ta;\n .reg .b64 db;\n setp.ne.b32 p, %3, 0;\n add.u32 ta, %1, %4;\n"
      " add.s64 db, %2, %5;\n tcgen05.mma.cta_group::1.kind::f16 [%0], [ta], db, %6, p;\n}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_base), "r"(accumulate), "n"(ACOL), "n"(OFF), "n"(IDESC)
      : "memory");
}
// All D/16 steps of one score MMA (K dimension = head dim; 64-column boxes of
// 16 KB hold 4 steps of 32 bytes each).
template <int D, int KK = 0>
__device__ __forceinline__ void mma_scores(uint32_t d_tmem, uint64_t dq, uint64_t dk) {
  constexpr uint32_t off = static_cast<uint32_t>(((KK >> 2) * (128 * 128) + (KK & 3) * 32) >> 4);
  mma_ss_step<off, idesc_bf16(kBM, kBN, 0)>(d_tmem, dq, dk, KK > 0 ? 1u : 0u);
  if constexpr (KK + 1 < D / 16) mma_scores<D, KK + 1>(d_tmem, dq, dk);
}
// Steps [KK, END) of one P.V MMA (16 keys per step: 8 TMEM columns of P, 2 KB of V).
template <int D, int KK, int END>
__device__ __forceinline__ void mma_pv(uint32_t d_tmem, uint32_t p_tmem, uint64_t dv, bool first) {
  constexpr uint32_t voff = static_cast<uint32_t>((KK * 2048) >> 4);
  mma_ts_step<KK * 8, voff, idesc_bf16(kBM, D, 1)>(d_tmem, p_tmem, dv, (!first || KK > 0) ? 1u : 0u);
  if constexpr (KK + 1 < END) mma_pv<D, KK + 1, END>(d_tmem, p_tmem, dv, first);
}

// Scale-and-shift and the running sums with paired fp32 instructions.
constexpr bool kPairedFma = true;

// Multiply this thread's TMEM output row by f (warp-collective).
template <int D>
__device__ __forceinline__ void rescale_row_t(uint32_t colO, float f) {
#pragma unroll
  for (int c = 0; c < D / 16; ++c) {
    uint32_t ov[16];
    tmem_ld_32x32b_x16(colO + c * 16, ov);
    tc_wait_ld();
#pragma unroll
    for (int e = 0; e < 16; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * f);
    tmem_st_32x32b_x16(colO + c * 16, ov);
  }
}

__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Persistent: one CTA per SM walks its share of the work items. Barrier phases
// run on across items: K/V stages and score/probability barriers count key
// tiles (g), Q and final-output barriers count items (it).
template <int D, bool PAGED>
__global__ void __launch_bounds__(kPfThreads, 1)
    prefill_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                       const __grid_constant__ CUtensorMap tm_kr, const __grid_constant__ CUtensorMap tm_vr,
                       const PrefillParams p) {
  using C = PfCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  const uint32_t sbase = (raw_u32 + 1023u) & ~1023u;  // swizzled tiles need 1024-byte alignment
  uint8_t* smem = smem_raw + (sbase - raw_u32);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int cta = blockIdx.x;
  const int G = gridDim.x;

  const uint32_t bars = sbase + C::kBarOff;
  auto bar = [&](int i) -> uint32_t { return bars + 8u * static_cast<uint32_t>(i); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kBarOff + kTmemSlotOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kBarOff + kAbortOff);

  if (threadIdx.x == 0) {
    mbar_init(bar(kBarQFull), 1);
    mbar_init(bar(kBarQEmpty), 1);
    for (int s = 0; s < 4; ++s) {  // every slot initialised; only kKStages / kVStages used
      mbar_init(bar(kBarKFull + s), 1);
      mbar_init(bar(kBarVFull + s), 1);
      mbar_init(bar(kBarKEmpty + s), 1);
      mbar_init(bar(kBarVEmpty + s), 1);
    }
    for (int x = 0; x < kTilesPerCta; ++x) {
      mbar_init(bar(kBarSFull + x), 1);
      mbar_init(bar(kBarPLo + x), kBM);
      mbar_init(bar(kBarPHi + x), kBM);
      mbar_init(bar(kBarOFinal + x), 1);
    }
    mbar_init(bar(kBarDrain), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  // Paged contexts: every CTA sorts the work classes by key-tile count (the
  // same order everywhere), so the snake deal starts from the heaviest items
  // of the longest contexts. The key ring, not yet written, holds the costs.
  int* order = reinterpret_cast<int*>(smem + C::kOrderOff);
  const bool use_order = PAGED && p.ordered;
  if (use_order && warp == 0) {
    const int classes = p.num_cta_tiles * p.B;
    int* cost = reinterpret_cast<int*>(smem + C::kKOff);
    for (int c = lane; c < classes; c += 32) {
      const int rank = c / p.B;
      const int ct = (p.mask_kind == ATTN_MASK_FULL) ? rank : (p.num_cta_tiles - 1 - rank);
      cost[c] = item_geom<PAGED>(p, WorkItem{ct * kRowsPerCta, 0, c - rank * p.B}).T;
    }
    __syncwarp();
    for (int c = lane; c < classes; c += 32) {
      int r = 0;
      for (int c2 = 0; c2 < classes; ++c2) r += (cost[c2] > cost[c]) || (cost[c2] == cost[c] && c2 < c);
      order[r] = c;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const long long budget = p.budget;

  if (warp >= kTmaWarp) {
    regs_dec<kRegsControl>();
    if (warp == kTmaWarp && (PAGED || lane == 0)) {
      // ---------------------------------------------------------- TMA producer
      // Lane 0 waits on the ring and arms the barriers; the copies of a paged
      // key tile (one box per pool block) go out from lanes 0 .. 128 / block_size - 1
      // at once, lane e issuing block e. The contiguous kernel runs lane 0 alone.
      if (lane == 0) {
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
      }
      int g = 0;             // key tiles issued before this item (K and V alike)
      int k_issued = 0, v_issued = 0, it = 0;
      bool ok = true;
      for (int round = 0; ok; ++round) {
        const int w = item_index(round, cta, G);
        if (w >= p.num_items) break;
        const WorkItem wi = item_at(p, w, order, use_order);
        const ItemGeom gm = item_geom<PAGED>(p, wi);
        const int kt_lo = gm.lo, T = gm.T;
        const int zq = wi.b * p.Hq + wi.h;
        const int kvh = wi.h / p.group;
        const int zkv = wi.b * p.Hkv + kvh;
        // One K or V tile: a 128-row box of the contiguous tensor, or, for a paged
        // context, 128 / block_size boxes of one block each, found through the
        // block table. A block past the sequence or with an entry outside the pool
        // is requested at block index num_blocks: TMA fills it with zeros (the
        // softmax masks those keys and flags the bad entry). The sequence's last,
        // partly filled block goes row by row (tm_row: one-row boxes) so that its
        // slots past seq_len arrive as zeros, never as stale pool contents: their
        // probabilities are 0, and 0 * NaN would still poison P.V.
        //
        // Each lane reads its block's table entry one key tile ahead and keeps it
        // for the V copy of the same tile, so no copy waits on a table read.
        const int bs = PAGED ? p.block_size : kBN;
        const int boxes = kBN / bs;
        auto fetch = [&](int kt) -> int {
          if (!PAGED) return 0;
          const int key = kt * kBN + lane * bs;
          return (lane < boxes && !gm.bad && key < gm.nk)
                     ? __ldg(p.block_table + static_cast<size_t>(wi.b) * p.max_blocks + key / bs)
                     : p.num_blocks;
        };
        auto load_kv = [&](const CUtensorMap* tm, const CUtensorMap* tm_row, uint32_t dst, uint32_t bar_full, int kt,
                           int ent) {
          if (!PAGED) {
            if (lane == 0)
              for (int hh = 0; hh < C::kHalves; ++hh)
                tma_load_3d(dst + hh * C::kHalf, tm, bar_full, hh * 64, kt * kBN, zkv);
          } else if (lane < boxes) {
            const int key = kt * kBN + lane * bs;
            const int phys = (ent >= 0 && ent < p.num_blocks) ? ent : p.num_blocks;
            const uint32_t bdst = dst + lane * bs * 128;
            if (key + bs <= gm.nk || phys == p.num_blocks) {
              for (int hh = 0; hh < C::kHalves; ++hh)
                tma_load_4d(bdst + hh * C::kHalf, tm, bar_full, hh * 64, kvh, 0, phys);
            } else {
              const int valid = gm.nk - key;  // 1 .. bs - 1 rows hold tokens
              for (int slot = 0; slot < bs; ++slot)
                for (int hh = 0; hh < C::kHalves; ++hh)
                  tma_load_4d(bdst + hh * C::kHalf + slot * 128, tm_row, bar_full, hh * 64, kvh, slot,
                              slot < valid ? phys : p.num_blocks);
            }
          }
        };
        int ent_k = fetch(kt_lo), ent_v = p.num_blocks;  // entries of key tiles i and i - 1
        // Q of this item once the previous item's last score MMA has read its Q
        bool armed = true;
        if (lane == 0) {
          armed = (it == 0) || mbar_wait_bounded(bar(kBarQEmpty), (it - 1) & 1, budget, abort_flag);
          if (armed) {
            mbar_arrive_expect_tx(bar(kBarQFull), kTilesPerCta * C::kTile);
            for (int x = 0; x < kTilesPerCta; ++x)
              for (int hh = 0; hh < C::kHalves; ++hh)
                tma_load_3d(sbase + C::kQOff + x * C::kTile + hh * C::kHalf, &tm_q, bar(kBarQFull), hh * 64,
                            wi.q0 + x * kBM, zq);
          }
        }
        ok = PAGED ? __shfl_sync(0xffffffffu, armed, 0) : armed;
        if (!ok) break;
        // K_i is issued before V_{i-1}: the score MMA needs K one tile earlier than P.V needs V.
        for (int i = 0; i <= T; ++i) {
          if (i < T) {
            const int gi = g + i, s = gi % C::kKStages, rnd = gi / C::kKStages;
            if (lane == 0) {
              armed = (rnd == 0) || mbar_wait_bounded(bar(kBarKEmpty + s), (rnd - 1) & 1, budget, abort_flag);
              if (armed) mbar_arrive_expect_tx(bar(kBarKFull + s), C::kTile);
            }
            ok = PAGED ? __shfl_sync(0xffffffffu, armed, 0) : armed;
            if (!ok) break;
            load_kv(&tm_k, &tm_kr, sbase + C::kKOff + s * C::kTile, bar(kBarKFull + s), kt_lo + i, ent_k);
            k_issued = gi + 1;
          }
          if (i >= 1) {
            const int gv = g + i - 1, s = gv % C::kVStages, rnd = gv / C::kVStages;
            if (lane == 0) {
              armed = (rnd == 0) || mbar_wait_bounded(bar(kBarVEmpty + s), (rnd - 1) & 1, budget, abort_flag);
              if (armed) mbar_arrive_expect_tx(bar(kBarVFull + s), C::kTile);
            }
            ok = PAGED ? __shfl_sync(0xffffffffu, armed, 0) : armed;
            if (!ok) break;
            load_kv(&tm_v, &tm_vr, sbase + C::kVOff + s * C::kTile, bar(kBarVFull + s), kt_lo + i - 1, ent_v);
            v_issued = gv + 1;
          }
          if (PAGED) {
            ent_v = ent_k;
            if (i + 1 < T) ent_k = fetch(kt_lo + i + 1);
          }
        }
        g += T;
        ++it;
      }
      if (lane == 0) {
        if (!ok) raise_abort(abort_flag, p.status);
        // Drain: the newest copy of every stage and of Q has landed before the CTA may exit.
        volatile int never = 0;
        if (it > 0) mbar_wait_bounded(bar(kBarQFull), (it - 1) & 1, kDrainBudgetCycles, &never);
        for (int j = (k_issued > C::kKStages ? k_issued - C::kKStages : 0); j < k_issued; ++j)
          mbar_wait_bounded(bar(kBarKFull + j % C::kKStages), (j / C::kKStages) & 1, kDrainBudgetCycles, &never);
        for (int j = (v_issued > C::kVStages ? v_issued - C::kVStages : 0); j < v_issued; ++j)
          mbar_wait_bounded(bar(kBarVFull + j % C::kVStages), (j / C::kVStages) & 1, kDrainBudgetCycles, &never);
      }
    } else if (warp == kMmaWarp && lane == 0) {
      // ---------------------------------------------------------- MMA issuer
      // Descriptors are built once; an operand at byte offset o from its base has
      // descriptor base + o / 16 (the start address is the low field, and every
      // tile lies below 256 KB, so the addition never carries out of it).
      const uint64_t dq0 = desc_sw128(sbase + C::kQOff, 16, 1024);
      const uint64_t dk0 = desc_sw128(sbase + C::kKOff, 16, 1024);
      const uint64_t dv0 = desc_sw128(sbase + C::kVOff, C::kHalf, 1024);
      constexpr uint64_t kTileUnits = C::kTile >> 4;
      // S_x = Q_x K^T of global key tile g into tile x's score columns
      auto issue_s = [&](int x, int g) {
        mma_scores<D>(tmem + C::col_s(x), dq0 + static_cast<uint64_t>(x) * kTileUnits,
                      dk0 + static_cast<uint64_t>(g % C::kKStages) * kTileUnits);
        tc_commit(bar(kBarSFull + x));
      };
      // O_x (+)= P_x V for keys [64 half, 64 half + 64) of global key tile g; P_x sits in
      // the first 64 score columns (16 keys = 8 columns per MMA step); `first` starts O_x.
      // c is tile x's count of score tiles so far (the parity of its S and P barriers).
      auto pv_half = [&](int x, int g, int c, int half, bool first) -> bool {
        if (!mbar_wait_bounded(bar((half ? kBarPHi : kBarPLo) + x), c & 1, budget, abort_flag)) return false;
        tc_fence_after();
        const uint64_t dv = dv0 + static_cast<uint64_t>(g % C::kVStages) * kTileUnits;
        if (half == 0)
          mma_pv<D, 0, 4>(tmem + C::col_o(x), tmem + C::col_s(x), dv, first);
        else
          mma_pv<D, 4, 8>(tmem + C::col_o(x), tmem + C::col_s(x), dv, first);
        return true;
      };
      int g = 0, it = 0;
      int cnt[kTilesPerCta] = {0, 0};  // score tiles computed per query tile
      bool ok = true;
      for (int round = 0; ok; ++round) {
        const int w = item_index(round, cta, G);
        if (w >= p.num_items) break;
        const WorkItem wi = item_at(p, w, order, use_order);
        const ItemGeom gm = item_geom<PAGED>(p, wi);
        const int T = gm.T;
        const TileRanges tr = tile_ranges(p, wi, gm);
        if (!mbar_wait_bounded(bar(kBarQFull), it & 1, budget, abort_flag) ||
            !mbar_wait_bounded(bar(kBarKFull + g % C::kKStages), (g / C::kKStages) & 1, budget, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        issue_s(0, g);
        if (tr.b0 == 0) issue_s(1, g);
        tc_commit(bar(kBarKEmpty + g % C::kKStages));
        if (T == 1) tc_commit(bar(kBarQEmpty));
        for (int j = 0; j < T; ++j) {
          const int gj = g + j, gn = gj + 1;
          const int s = gj % C::kVStages;  // V stage of key tile j
          if (!mbar_wait_bounded(bar(kBarVFull + s), (gj / C::kVStages) & 1, budget, abort_flag)) {
            ok = false;
            break;
          }
          // tile A: P.V of key tile j (as each half of P lands), then the scores of tile
          // j + 1 (in issue order, so the new scores overwrite P only after P.V read it)
          if (j < tr.a1) {
            if (!pv_half(0, gj, cnt[0], 0, j == 0) || !pv_half(0, gj, cnt[0], 1, j == 0)) {
              ok = false;
              break;
            }
            ++cnt[0];
            if (j == tr.a1 - 1) tc_commit(bar(kBarOFinal + 0));
          }
          if (j + 1 < T) {
            if (!mbar_wait_bounded(bar(kBarKFull + gn % C::kKStages), (gn / C::kKStages) & 1, budget, abort_flag)) {
              ok = false;
              break;
            }
            tc_fence_after();
            if (j + 1 < tr.a1) issue_s(0, gn);
          }
          // tile B
          if (j >= tr.b0) {
            if (!pv_half(1, gj, cnt[1], 0, j == tr.b0) || !pv_half(1, gj, cnt[1], 1, j == tr.b0)) {
              ok = false;
              break;
            }
            ++cnt[1];
            if (j == T - 1) tc_commit(bar(kBarOFinal + 1));
          }
          tc_commit(bar(kBarVEmpty + s));
          if (j + 1 < T) {
            if (j + 1 >= tr.b0) issue_s(1, gn);
            tc_commit(bar(kBarKEmpty + gn % C::kKStages));
            if (j + 2 == T) tc_commit(bar(kBarQEmpty));  // that was the item's last read of Q
          }
        }
        g += T;
        ++it;
      }
      if (!ok) raise_abort(abort_flag, p.status);
      // Drain: every MMA this thread issued has completed before TMEM is freed.
      tc_commit(bar(kBarDrain));
      volatile int never = 0;
      mbar_wait_bounded(bar(kBarDrain), 0, kDrainBudgetCycles, &never);
    }
  } else {
    regs_inc<kRegsSoftmax>();
    // ------------------------------------------------------------ softmax warps 0-7
    const int x = warp >> 2;                // query tile A (0) or B (1)
    const int r = threadIdx.x & (kBM - 1);  // row of the tile = TMEM lane
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const uint32_t colS = lane_base + C::col_s(x);
    const uint32_t colO = lane_base + C::col_o(x);
    const float sl2 = p.scale_log2;
    auto rescale_rows = [](uint32_t col, float f) { rescale_row_t<D>(col, f); };
    int cnt = 0, it = 0;  // this tile's score tiles so far, items so far
    bool ok = true;
    for (int round = 0;; ++round) {
      const int w = item_index(round, cta, G);
      if (w >= p.num_items) break;
      const WorkItem wi = item_at(p, w, order, use_order);
      const ItemGeom gm = item_geom<PAGED>(p, wi);
      const int kt_lo = gm.lo, T = gm.T;
      const int qr0 = wi.q0 + x * kBM;  // first query row of the tile
      const int qi = qr0 + r;           // this thread's query row
      const int qpos = gm.pos0 + qi;    // its position among the keys
      // A paged item whose seq_len is out of range, or that reads a block-table
      // entry outside the pool, yields NaN rows and the device-check status bit.
      bool item_bad = false;
      if (PAGED) {
        item_bad = gm.bad;
        if (!item_bad) {
          const int first = kt_lo * kBN / p.block_size;
          const int last = (min((kt_lo + T) * kBN, gm.nk) - 1) / p.block_size;
          bool bad_entry = false;
          for (int e = first + lane; e <= last; e += 32) {
            const int entry = __ldg(p.block_table + static_cast<size_t>(wi.b) * p.max_blocks + e);
            bad_entry |= entry < 0 || entry >= p.num_blocks;
          }
          item_bad = __any_sync(0xffffffffu, bad_entry);
        }
        if (item_bad && lane == 0 && p.status != nullptr) atomicOr(p.status, ATTN_STATUS_BIT_DEVICE_CHECK);
      }
      float m_used = -INFINITY;         // max the exponentials are taken against (base 2)
      float l_sum = 0.f;                // running sum of 2^(x - m_used), fp32
      const TileRanges tr = tile_ranges(p, wi, gm);
      const int j_end = x == 0 ? tr.a1 : T;
      for (int j = x == 0 ? 0 : tr.b0; j < j_end && ok; ++j, ++cnt) {
        const int k0 = (kt_lo + j) * kBN;
        ok = __all_sync(0xffffffffu, mbar_wait_bounded(bar(kBarSFull + x), cnt & 1, budget, abort_flag));
        if (!ok) break;
        tc_fence_after();
        uint32_t raw[kBN];
#pragma unroll
        for (int c = 0; c < kBN / 32; ++c)
          tmem_ld_32x32b_x32(colS + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&raw[c * 32]));
        tc_wait_ld();
        float sv[kBN];
#pragma unroll
        for (int c = 0; c < kBN; ++c) sv[c] = __uint_as_float(raw[c]);

        if (!tile_is_full(p, gm.pos0 + qr0, k0, gm.nk)) {
          // edge tile: visible keys of this row are columns [cmin, cmax]
          int cmax = gm.nk - 1 - k0;
          if (p.mask_kind != ATTN_MASK_FULL) cmax = min(cmax, qpos - k0);
          const int cmin = (p.mask_kind == ATTN_MASK_SLIDING_WINDOW) ? qpos - k0 - p.window + 1 : 0;
#pragma unroll
          for (int c = 0; c < kBN; ++c) sv[c] = (c >= cmin && c <= cmax) ? sv[c] : -INFINITY;
        }
        // row max of the raw scores (scale > 0 commutes with max): four independent chains
        float mx0 = -INFINITY, mx1 = -INFINITY, mx2 = -INFINITY, mx3 = -INFINITY;
#pragma unroll
        for (int c = 0; c < kBN; c += 8) {
          mx0 = max3f(mx0, sv[c], sv[c + 1]);
          mx1 = max3f(mx1, sv[c + 2], sv[c + 3]);
          mx2 = max3f(mx2, sv[c + 4], sv[c + 5]);
          mx3 = max3f(mx3, sv[c + 6], sv[c + 7]);
        }
        const float m_new = fmaxf(m_used, max3f(mx0, mx1, fmaxf(mx2, mx3)) * sl2);
        bool rescale_o = false;
        float factor = 1.f;
        if (m_new > m_used + kRescaleThreshold) {  // also true for the first visible key (m_used = -inf)
          const bool prev_finite = (m_used != -INFINITY);
          factor = prev_finite ? fast_exp2(m_used - m_new) : 0.f;
          l_sum *= factor;
          rescale_o = prev_finite;  // earlier tiles already put visible keys into O
          m_used = m_new;
        }
        // The score barrier was committed after this tile's previous P.V: O is stable.
        if (__any_sync(0xffffffffu, rescale_o)) rescale_rows(colO, rescale_o ? factor : 1.f);

        // p = 2^(s * scale * log2 e - m); a row with nothing visible yet uses m = 0.
        // P goes out in two halves, each announced on its own barrier, so the MMA
        // warp starts P.V on keys 0-63 while keys 64-127 are still being exponentiated.
        const float neg_m = (m_used == -INFINITY) ? 0.f : -m_used;
        float2 acc0 = make_float2(0.f, 0.f), acc1 = acc0, acc2 = acc0, acc3 = acc0;
#pragma unroll
        for (int cc = 0; cc < kBN / 32; ++cc) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int c = cc * 32 + 2 * e;
            float2 xv;
            if (kPairedFma) {
              xv = ffma2(make_float2(sv[c], sv[c + 1]), make_float2(sl2, sl2), make_float2(neg_m, neg_m));
            } else {
              xv.x = fmaf(sv[c], sl2, neg_m);
              xv.y = fmaf(sv[c + 1], sl2, neg_m);
            }
            float2 pv;
            pv.x = fast_exp2(xv.x);
            pv.y = fast_exp2(xv.y);
            float2& acc = (e & 3) == 0 ? acc0 : (e & 3) == 1 ? acc1 : (e & 3) == 2 ? acc2 : acc3;
            if (kPairedFma) {
              acc = fadd2(acc, pv);
            } else {
              acc.x += pv.x;
              acc.y += pv.y;
            }
            pk[e] = pack_bf16x2(pv.x, pv.y);
          }
          tmem_st_32x32b_x16(colS + cc * 16, pk);  // over score columns already consumed
          if (cc == 1 || cc == 3) {
            tc_wait_st();
            tc_fence_before();
            mbar_arrive(bar((cc == 1 ? kBarPLo : kBarPHi) + x));
          }
        }
        l_sum += ((acc0.x + acc0.y) + (acc1.x + acc1.y)) + ((acc2.x + acc2.y) + (acc3.x + acc3.y));
      }
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait_bounded(bar(kBarOFinal + x), it & 1, budget, abort_flag));
      if (!ok) raise_abort(abort_flag, p.status);
      tc_fence_after();

      // ---- epilogue: O / l -> bf16 through a swizzled shared staging box and a TMA
      // store per warp and 64-column half (rows past N are clipped by the store);
      // LSE (natural log) per thread. After a timeout every remaining row of this
      // CTA is written as NaN without touching TMEM.
      const bool row_valid = qi < p.N;
      const size_t row = static_cast<size_t>(wi.b * p.Hq + wi.h) * p.N + (row_valid ? qi : 0);
      const bool out_ok = ok && !item_bad;
      const float inv_l = out_ok ? 1.f / l_sum : NAN;
      const uint32_t stage = sbase + C::kStageOff + warp * 4096;
      const int wrow = r & 31;
#pragma unroll
      for (int hh = 0; hh < D / 64; ++hh) {
        if (lane == 0) bulk_wait_read_all();  // the previous store has read the staging box
        __syncwarp();
#pragma unroll
        for (int q32 = 0; q32 < 2; ++q32) {  // 32 columns at a time: 4 swizzled 16-byte chunks
          uint32_t ov[32];
          if (ok) {
            tmem_ld_32x32b_x32(colO + hh * 64 + q32 * 32, ov);
            tc_wait_ld();
          }
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {
            uint32_t w4[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float a0 = ok ? __uint_as_float(ov[c4 * 8 + 2 * e]) * inv_l : NAN;
              const float a1 = ok ? __uint_as_float(ov[c4 * 8 + 2 * e + 1]) * inv_l : NAN;
              w4[e] = pack_bf16x2(a0, a1);
            }
            const int c = q32 * 4 + c4;
            const uint32_t dst = stage + wrow * 128 + ((c ^ (wrow & 7)) << 4);
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};\n" ::"r"(dst), "r"(w4[0]), "r"(w4[1]),
                         "r"(w4[2]), "r"(w4[3])
                         : "memory");
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && qr0 + (warp & 3) * 32 < p.N) {  // a box wholly past N has nothing to write
          tma_store_3d(&tm_o, stage, hh * 64, qr0 + (warp & 3) * 32, wi.b * p.Hq + wi.h);
          bulk_commit();
        }
      }
      if (row_valid && p.lse != nullptr) p.lse[row] = out_ok ? (m_used + __log2f(l_sum)) * kLn2 : NAN;
      // The next item's first P.V overwrites O: its P is announced only after
      // these loads completed (tcgen05.wait::ld above, fence before the arrive).
      tc_fence_before();
      ++it;
    }
    if (lane == 0) bulk_wait_all();  // output stores complete before the CTA exits
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// [heads][n][d] bf16 viewed as a rank-3 tensor (d innermost); box = 64 columns
// x 128 rows x 1 head, 128-byte swizzle. Rows past n read as zero.
bool encode_bhnd(CUtensorMap* map, const void* base, int d, int n, int heads, int box_rows = 128) {
  const auto enc = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(tensor_map_encode_fn());
  if (enc == nullptr) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(n),
                              static_cast<cuuint64_t>(heads)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(n) * d * 2};
  const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
  const cuuint32_t estride[3] = {1, 1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
                         estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// The paged pool [num_blocks][block_size][Hkv][d] bf16 as a rank-4 tensor
// (d, Hkv, slot, block); box = 64 columns x 1 head x box_slots slots x 1
// block, 128-byte swizzle: box_slots = block_size loads one block of one head,
// box_slots = 1 one token row.
bool encode_pool(CUtensorMap* map, const void* base, int d, int hkv, int block_size, int num_blocks,
                 int box_slots) {
  const auto enc = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(tensor_map_encode_fn());
  if (enc == nullptr) return false;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(hkv),
                              static_cast<cuuint64_t>(block_size), static_cast<cuuint64_t>(num_blocks)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(hkv) * d * 2,
                                 static_cast<cuuint64_t>(block_size) * hkv * d * 2};
  const cuuint32_t box[4] = {64, 1, static_cast<cuuint32_t>(box_slots), 1};
  const cuuint32_t estride[4] = {1, 1, 1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box,
                         estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

struct PagedContext {
  const int32_t* block_table;
  const int32_t* seq_lens;
  int num_blocks, block_size, max_blocks, max_seq_len;
};

// N = query rows per sequence. Contiguous: k, v are [B, Hkv, N, d]. Paged
// (ctx != null): k, v are the pools and every sequence's keys come from its
// block-table row.
template <int D, bool PAGED>
int launch_prefill_t(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int N,
                     int mask_kind, int window, float scale, int32_t* status, cudaStream_t stream,
                     const PagedContext* ctx) {
  CUtensorMap tq, tk, tv, to, tkr, tvr;
  if (!encode_bhnd(&tq, q, D, N, B * Hq) || !encode_bhnd(&to, o, D, N, B * Hq, 32)) return ATTN_ERR_CUDA;
  if (PAGED) {
    if (!encode_pool(&tk, k, D, Hkv, ctx->block_size, ctx->num_blocks, ctx->block_size) ||
        !encode_pool(&tv, v, D, Hkv, ctx->block_size, ctx->num_blocks, ctx->block_size) ||
        !encode_pool(&tkr, k, D, Hkv, ctx->block_size, ctx->num_blocks, 1) ||
        !encode_pool(&tvr, v, D, Hkv, ctx->block_size, ctx->num_blocks, 1))
      return ATTN_ERR_CUDA;
  } else {
    if (!encode_bhnd(&tk, k, D, N, B * Hkv) || !encode_bhnd(&tv, v, D, N, B * Hkv)) return ATTN_ERR_CUDA;
    tkr = tk;  // unused without a paged context
    tvr = tv;
  }
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
  p.num_cta_tiles = (N + kRowsPerCta - 1) / kRowsPerCta;
  p.num_items = p.num_cta_tiles * Hq * B;
  p.ordered = (PAGED && p.num_cta_tiles * B <= PfCfg<D>::kOrderMax) ? 1 : 0;
  p.scale_log2 = scale * kLog2e;
  p.budget = wait_budget_cycles();
  p.block_table = PAGED ? ctx->block_table : nullptr;
  p.seq_lens = PAGED ? ctx->seq_lens : nullptr;
  p.max_blocks = PAGED ? ctx->max_blocks : 0;
  p.block_size = PAGED ? ctx->block_size : 0;
  p.num_blocks = PAGED ? ctx->num_blocks : 0;
  p.max_seq_len = PAGED ? ctx->max_seq_len : N;
  constexpr int smem = PfCfg<D>::kAlloc;
  if (cudaFuncSetAttribute(prefill_fwd_kernel<D, PAGED>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
      cudaSuccess)
    return ATTN_ERR_CUDA;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
    return ATTN_ERR_CUDA;
  const dim3 grid(p.num_items < sms ? p.num_items : sms);  // persistent: one CTA per SM
  prefill_fwd_kernel<D, PAGED><<<grid, kPfThreads, smem, stream>>>(tq, tk, tv, to, tkr, tvr, p);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // namespace

int launch_prefill(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int N,
                   int d, int mask_kind, int window, float scale, int32_t* status, cudaStream_t stream) {
  if (d == 128)
    return launch_prefill_t<128, false>(q, k, v, o, lse, B, Hq, Hkv, N, mask_kind, window, scale, status, stream,
                                        nullptr);
  return launch_prefill_t<64, false>(q, k, v, o, lse, B, Hq, Hkv, N, mask_kind, window, scale, status, stream,
                                     nullptr);
}

int launch_prefill_paged(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_table,
                         const int32_t* seq_lens, void* o, float* lse, int B, int Hq, int Hkv, int Nq, int d,
                         int num_blocks, int block_size, int max_blocks_per_seq, int max_seq_len, int mask_kind,
                         int window, float scale, int32_t* status, cudaStream_t stream) {
  const PagedContext ctx{block_table, seq_lens, num_blocks, block_size, max_blocks_per_seq, max_seq_len};
  if (d == 128)
    return launch_prefill_t<128, true>(q, k_cache, v_cache, o, lse, B, Hq, Hkv, Nq, mask_kind, window, scale, status,
                                       stream, &ctx);
  return launch_prefill_t<64, true>(q, k_cache, v_cache, o, lse, B, Hq, Hkv, Nq, mask_kind, window, scale, status,
                                    stream, &ctx);
}

}  // namespace attn
