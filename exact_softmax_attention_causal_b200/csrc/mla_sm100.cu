// Absorbed Multi-head Latent Attention (MLA) decode on the 5th-generation
// tensor cores (tcgen05 + TMEM + TMA), split along the cached sequence.
//
// What it computes ("Module 5. Modern Attention Mechanisms", section 7;
// "Module 09: Efficient Attention", the MLA section): every cached token is
// one row [c_t ; k^R_t] of d_c + d_R = 512 + 64 bf16 numbers shared by all
// heads; head h's query is the row [A_h^T q^C_h ; q^R_h] of the same width.
// The logit is their dot product times `scale` (1 / sqrt(d_head + d_R)), the
// softmax runs over the sequence's cached tokens, and the output is the
// latent sum_t p_t c_t (d_c numbers; the caller applies the value
// up-projection). So it is multi-query attention with K = the whole row and
// V = its first 512 columns.
//
// How. One CTA handles 64 heads of one sequence over one split of `chunk`
// tokens; the partial outputs and log-sum-exps of the splits are combined by
// the paged decode's merge kernel (online-softmax rescaling, "Inference
// attention" post, "FlashDecoding"). The 64 heads' 512-wide fp32 outputs fill
// 256 of the 512 TMEM columns, so the CTA works on the transposed problem:
//   S^T [64 tokens x 64 heads]   = K_tile [64 x 576] . Q^T          (M = 64 tokens)
//   O^T [512 latent x 64 heads] += V_tile^T [512 x 64] . P^T        (4 MMAs of M = 128)
// A tile is 64 cached rows in nine 64-column chunks (128-byte swizzle); its
// first eight chunks are V_tile, read a second time as an MN-major A operand.
// Two tiles are in flight: the shared memory holds the resident Q^T (72 KB)
// and two 72 KB tile slots, so the next tile streams in while the current one
// is scored, exponentiated and multiplied. P^T is written by the softmax into
// the ninth chunk's slot once the score MMAs have read it. An M = 64 score
// tile lives in TMEM lanes 0-15 of each 32-lane sub-partition (token
// 16 q + i in lane 32 q + i). The softmax runs over the token lanes of each
// score column, so its maxima and sums are reduced across lanes: shuffles
// inside a warp, shared memory across the four warps of a column half.
//
// Roles (320 threads):
//   warps 0-7  softmax: warp w reads TMEM lanes 32 (w % 4) .. + 31 (16 tokens
//              of the score tile, latent rows of each output block) and head
//              columns 32 (w / 4) .. + 31. Lazy rescaling as in the prefill:
//              the max a column's exponentials use moves only when the tile
//              max exceeds it by more than 8 (base 2).
//   warp 8     TMA producer: Q^T once (nine 8 KB chunks), then for every tile
//              the nine 8 KB chunks of its 64 cached rows into the tile's
//              slot, one box per pool block (64-row boxes inside blocks of
//              128), lane e issuing block e's boxes (block-table entries
//              fetched a tile ahead, one per lane). Rows past the split come
//              in as zeros (one-row boxes for a partly filled block,
//              out-of-range block index for whole blocks).
//   warp 9     MMA issuer; allocates and frees TMEM. It issues each tile's
//              score MMAs as soon as the tile has landed and a score buffer
//              is free, and each tile's output MMAs as soon as its P^T is
//              written, whichever is ready first, so the tensor core works
//              on the next tile's scores while the softmax runs.
// All pipeline waits are bounded; on expiry the CTA records
// ATTN_STATUS_BIT_TIMEOUT, writes NaN partials, drains and exits.

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <type_traits>

#include "internal.h"
#include "ptx.cuh"

namespace attn {
namespace {

constexpr int kDc = 512;             // latent width d_c (the value width)
constexpr int kDr = 64;              // positional-key width d_h^R
constexpr int kRow = kDc + kDr;      // cached row width
constexpr int kChunks = kRow / 64;   // 64-column chunks of a row (128-byte swizzle)
constexpr int kTok = 64;             // tokens per tile (the score MMA's M)
constexpr int kNH = 64;              // heads per CTA = MMA N
constexpr int kSlots = 2;            // tiles in flight
constexpr int kPSlot = kChunks - 1;  // the positional chunk's slot holds P^T after the score MMAs
constexpr int kMlaThreads = 320;
constexpr int kMlaTmaWarp = 8;
constexpr int kMlaMmaWarp = 9;
constexpr float kMlaRescaleThreshold = 8.0f;

constexpr int kQChunkBytes = kNH * 128;   // 64 heads x 64 columns
constexpr int kKChunkBytes = kTok * 128;  // 64 tokens x 64 columns
constexpr int kTileBytes = kChunks * kKChunkBytes;
constexpr int kQOff = 0;
constexpr int kKOff = kQOff + kChunks * kQChunkBytes;
constexpr int kRedOff = kKOff + kSlots * kTileBytes;  // cross-warp reductions: [2 halves][4 warps][32]
constexpr int kRedBytes = 2 * 4 * 32 * 4;
constexpr int kMOff = kRedOff + kRedBytes;  // running max per head column: [2 halves][32]
constexpr int kBarOff = kMOff + 2 * 32 * 4;
constexpr int kSmemBytes = kBarOff + 256;
constexpr int kSmemAlloc = kSmemBytes + 1024;  // slack to align the base to 1024 bytes
static_assert(kSmemAlloc <= 232448, "shared memory per CTA");

// TMEM columns: two score buffers, then the four 64-column output blocks.
constexpr uint32_t kColS = 0;     // + 64 * buffer
constexpr uint32_t kColO = 128;   // + 64 * latent block
constexpr uint32_t kTmemCols = 512;

enum : int {
  kMbQFull = 0,
  kMbKFull = 1,    // + slot (2): the tile's nine chunks landed
  kMbKEmpty = 3,   // + slot (2): the tile's output MMAs have read it
  kMbSFull = 5,    // + buffer (2)
  kMbSFree = 7,    // + buffer (2), one arrival per softmax warp
  kMbPFull = 9,    // + slot (2), one arrival per softmax warp
  kMbOReady = 11,  // the tile's output MMAs completed
  kMbDrain = 12,
  kMbCount = 13,
};
constexpr int kMlaTmemSlot = 224;
constexpr int kMlaAbort = 228;
constexpr int kMlaBad = 232;

// kind::f16 instruction descriptor: fp32 accumulate, bf16 A and B, A and B
// K-major (0) or MN-major (1), N >> 3 at bit 17, M >> 4 at bit 24.
constexpr uint32_t idesc_mla(int M, int N, int a_mn, int b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(a_mn) << 15) |
         (static_cast<uint32_t>(b_mn) << 16) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}
constexpr uint32_t kIdescScore = idesc_mla(kTok, kNH, 0, 0);  // S^T = K . Q^T, both K-major
constexpr uint32_t kIdescScore16 = idesc_mla(kTok, 16, 0, 0);  // the same for a block of <= 16 heads
constexpr uint32_t kIdescOut = idesc_mla(128, kNH, 1, 1);     // O^T += V^T . P^T, both MN-major

struct MlaParams {
  const int32_t* block_table;
  const int32_t* seq_lens;
  float* o_part;    // [B, H, splits, 512]
  float* lse_part;  // [B, H, splits]
  int32_t* status;
  int B, H, num_blocks, block_size, max_blocks, max_seq_len, chunk, splits;
  float scale_log2;
  long long budget;
};

__device__ __forceinline__ void mla_abort(volatile int* abort_flag, int32_t* status) {
  *abort_flag = 1;
  if (status != nullptr) atomicOr(status, ATTN_STATUS_BIT_TIMEOUT);
}

// Warp reduce-scatter of NC columns (16 or 32): on entry lane l holds v[c] for
// its token row; on exit lane l holds the max (or sum) of column l % NC over
// the 32 rows.
template <int NC, bool kMax>
__device__ __forceinline__ float warp_reduce_scatter(float (&v)[NC], int lane) {
#pragma unroll
  for (int o = NC / 2; o >= 1; o >>= 1) {
    const bool upper = (lane & o) != 0;
#pragma unroll
    for (int k = 0; k < o; ++k) {
      const float keep = upper ? v[k + o] : v[k];
      const float send = upper ? v[k] : v[k + o];
      const float recv = __shfl_xor_sync(0xffffffffu, send, o);
      v[k] = kMax ? fmaxf(keep, recv) : keep + recv;
    }
  }
#pragma unroll
  for (int o = NC; o < 32; o <<= 1) {  // the lane groups that held different rows
    const float recv = __shfl_xor_sync(0xffffffffu, v[0], o);
    v[0] = kMax ? fmaxf(v[0], recv) : v[0] + recv;
  }
  return v[0];
}

__device__ __forceinline__ void named_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;\n" ::"r"(id), "r"(threads) : "memory");
}

__global__ void __launch_bounds__(kMlaThreads, 1)
    mla_split_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_c,
                     const __grid_constant__ CUtensorMap tm_crow, const MlaParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  const uint32_t sbase = (raw_u32 + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (sbase - raw_u32);

  const int split = blockIdx.x, hb = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int seq_len = __ldg(p.seq_lens + b);
  if (seq_len < 1 || seq_len > p.max_seq_len) return;  // the merge kernel flags this row
  const int t0 = split * p.chunk;
  if (t0 >= seq_len) return;  // nothing cached in this split: the merge never reads it
  const int t1 = min(t0 + p.chunk, seq_len);
  const int ntiles = (t1 - t0 + kTok - 1) / kTok;
  // this block holds at most 16 heads (H = 16, or a last block of at most 16)
  const bool narrow = p.H - hb * kNH <= 16;

  const uint32_t bars = sbase + kBarOff;
  auto bar = [&](int i) -> uint32_t { return bars + 8u * static_cast<uint32_t>(i); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kBarOff + kMlaTmemSlot);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kBarOff + kMlaAbort);
  volatile int* bad_flag = reinterpret_cast<volatile int*>(smem + kBarOff + kMlaBad);

  if (threadIdx.x == 0) {
    mbar_init(bar(kMbQFull), 1);
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(bar(kMbKFull + s), 1);
      mbar_init(bar(kMbKEmpty + s), 1);
      mbar_init(bar(kMbSFull + s), 1);
      mbar_init(bar(kMbSFree + s), 8);
      mbar_init(bar(kMbPFull + s), 8);
    }
    mbar_init(bar(kMbOReady), 1);
    mbar_init(bar(kMbDrain), 1);
    *abort_flag = 0;
    *bad_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMlaMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const long long budget = p.budget;

  if (warp == kMlaTmaWarp) {
    // ------------------------------------------------------------ TMA producer
    // Lane 0 waits for the tile's slot and arms its barrier; lane e then issues
    // the boxes of the tile's e-th pool block (or, for 128-token blocks, the
    // tile's 64-row half of its block), so a tile's copies go out from several
    // threads at once.
    const int bs = p.block_size;
    const int box_rows = bs < kTok ? bs : kTok;
    const int boxes = kTok / box_rows;
    const int32_t* table = p.block_table + static_cast<size_t>(b) * p.max_blocks;
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_c);
      prefetch_tmap(&tm_crow);
      mbar_arrive_expect_tx(bar(kMbQFull), kChunks * kQChunkBytes);
      for (int j = 0; j < kChunks; ++j)
        tma_load_3d(sbase + kQOff + j * kQChunkBytes, &tm_q, bar(kMbQFull), 64 * j, hb * kNH, b);
    }
    // This lane's block of a tile: out-of-range or unneeded blocks become the
    // out-of-range index num_blocks (TMA fills zeros); a bad referenced entry
    // also marks the CTA's output as invalid.
    auto fetch = [&](int tile) -> int {
      const int key = t0 + tile * kTok + lane * box_rows;
      return (lane < boxes && key < t1) ? __ldg(table + key / bs) : p.num_blocks;
    };
    int ent = fetch(0);
    int issued = 0;  // tiles whose copies were all issued
    bool ok = true;
    for (int i = 0; i < ntiles && ok; ++i) {
      const int slot = i % kSlots;
      const int ent_next = (i + 1 < ntiles) ? fetch(i + 1) : p.num_blocks;
      const int key = t0 + i * kTok + lane * box_rows;
      int phys = ent;
      if (lane < boxes && key < t1 && (phys < 0 || phys >= p.num_blocks)) {
        *bad_flag = 1;
        phys = p.num_blocks;
      }
      if (key >= t1) phys = p.num_blocks;
      bool armed = true;
      if (lane == 0) {
        armed = (i < kSlots) ||
                mbar_wait_bounded(bar(kMbKEmpty + slot), ((i - kSlots) / kSlots) & 1, budget, abort_flag);
        if (armed) mbar_arrive_expect_tx(bar(kMbKFull + slot), kTileBytes);
      }
      ok = __shfl_sync(0xffffffffu, armed, 0);
      if (!ok) break;
      if (lane < boxes) {
        const int row0 = key % bs;  // first row of the box inside its block
        const uint32_t dst0 = sbase + kKOff + slot * kTileBytes + lane * box_rows * 128;
        if (key + box_rows <= t1 || phys == p.num_blocks) {
          for (int j = 0; j < kChunks; ++j)
            tma_load_3d(dst0 + j * kKChunkBytes, &tm_c, bar(kMbKFull + slot), 64 * j, row0, phys);
        } else {
          const int valid = t1 - key;  // 1 .. box_rows - 1 rows hold tokens of this split
          for (int j = 0; j < kChunks; ++j)
            for (int r = 0; r < box_rows; ++r)
              tma_load_3d(dst0 + j * kKChunkBytes + r * 128, &tm_crow, bar(kMbKFull + slot), 64 * j, row0 + r,
                          r < valid ? phys : p.num_blocks);
        }
      }
      issued = i + 1;
      ent = ent_next;
    }
    if (lane == 0) {
      if (!ok) mla_abort(abort_flag, p.status);
      // Drain: Q and the newest copy of every slot landed before the CTA may exit.
      volatile int never = 0;
      mbar_wait_bounded(bar(kMbQFull), 0, kDrainBudgetCycles, &never);
      for (int i = (issued > kSlots ? issued - kSlots : 0); i < issued; ++i)
        mbar_wait_bounded(bar(kMbKFull + i % kSlots), (i / kSlots) & 1, kDrainBudgetCycles, &never);
    }
  } else if (warp == kMlaMmaWarp) {
    if (lane == 0) {
      // ---------------------------------------------------------- MMA issuer
      const uint64_t dq = desc_sw128(sbase + kQOff, 16, 1024);
      const uint64_t dk = desc_sw128(sbase + kKOff, 16, 1024);
      // V^T block m: chunks 2m and 2m + 1 (64 latent columns each) as one MN-major
      // operand; P^T in the positional chunk's place, MN-major, one 64-head group.
      const uint64_t dv = desc_sw128(sbase + kKOff, kKChunkBytes, 1024);
      const uint64_t dp = desc_sw128(sbase + kKOff + kPSlot * kKChunkBytes, kKChunkBytes, 1024);
      constexpr uint64_t kTileUnits = kTileBytes >> 4;
      bool ok = mbar_wait_bounded(bar(kMbQFull), 0, budget, abort_flag);
      // Tile j's scores need its slot loaded and score buffer j % 2 released by
      // the softmax of tile j - 2; its output MMAs need its P^T. Each is issued
      // as soon as it is ready: the barriers are polled with test_wait, which
      // never suspends, so waiting on one never hides that another completed. Every barrier tested here is at most one phase
      // ahead of the phase tested (the next phase needs work issued after this
      // test), so the parity tests are unambiguous.
      int ns = 0, npv = 0;
      long long idle_since = clock64();
      // a block of at most 16 heads scores only its first 16 query columns
      const uint32_t idesc_s = narrow ? kIdescScore16 : kIdescScore;
      // O^T += V^T . P^T of tile npv when its P^T has been written (the softmax
      // rescaled O^T first where its max moved); its commit frees the tile's slot.
      auto try_pv = [&]() -> bool {
        if (npv >= ns) return false;
        const int sl = npv % kSlots;
        if (!mbar_test_wait(bar(kMbPFull + sl), (npv / kSlots) & 1)) return false;
        tc_fence_after();
        for (int m = 0; m < 4; ++m) {
#pragma unroll
          for (int kk = 0; kk < kTok / 16; ++kk) {
            const uint64_t a =
                dv + sl * kTileUnits + static_cast<uint64_t>((2 * m * kKChunkBytes + kk * 2048) >> 4);
            const uint64_t bp = dp + sl * kTileUnits + static_cast<uint64_t>((kk * 2048) >> 4);
            tc_mma_ss(tmem + kColO + 64u * m, a, bp, kIdescOut, (npv > 0 || kk > 0) ? 1u : 0u);
          }
        }
        tc_commit(bar(kMbKEmpty + sl));
        tc_commit(bar(kMbOReady));
        ++npv;
        return true;
      };
      while (ok && npv < ntiles) {
        bool progressed = false;
        if (ns < ntiles && ns < npv + kSlots) {
          const int sl = ns % kSlots;
          if (mbar_test_wait(bar(kMbKFull + sl), (ns / kSlots) & 1) &&
              (ns < kSlots || mbar_test_wait(bar(kMbSFree + sl), ((ns - kSlots) / kSlots) & 1))) {
            tc_fence_after();
            // S^T = K . Q^T over the nine chunks, 4 steps of 16 columns each. Issuing
            // MMAs blocks while the tensor pipe is busy, so between chunks a tile whose
            // P^T is ready gets its output MMAs first: they free its slot for the next
            // copy instead of waiting behind the whole score product.
            for (int j = 0; j < kChunks; ++j) {
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const uint64_t a = dk + sl * kTileUnits + static_cast<uint64_t>((j * kKChunkBytes + kk * 32) >> 4);
                const uint64_t bq = dq + static_cast<uint64_t>((j * kQChunkBytes + kk * 32) >> 4);
                tc_mma_ss(tmem + kColS + 64u * sl, a, bq, idesc_s, (j | kk) != 0 ? 1u : 0u);
              }
              try_pv();
            }
            tc_commit(bar(kMbSFull + sl));
            ++ns;
            progressed = true;
          }
        }
        if (!progressed) progressed = try_pv();
        if (progressed) {
          idle_since = clock64();
        } else if (*abort_flag || clock64() - idle_since > budget) {
          ok = false;
        }
      }
      if (!ok) mla_abort(abort_flag, p.status);
      tc_commit(bar(kMbDrain));
      volatile int never = 0;
      mbar_wait_bounded(bar(kMbDrain), 0, kDrainBudgetCycles, &never);
    }
  } else {
    // ------------------------------------------------------------ softmax warps 0-7
    const int sp = warp & 3;    // TMEM sub-partition: lanes 32 sp .. 32 sp + 31
    const int hh = warp >> 2;   // head columns 32 hh .. 32 hh + 31
    const int r = sp * 32 + lane;      // latent row of an output block
    const int tok = sp * 16 + lane;    // token of a score tile held by this lane (lanes 0-15)
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(sp * 32) << 16);
    float* red = reinterpret_cast<float*>(smem + kRedOff) + hh * 4 * 32;  // [4 warps][32]
    float* msm = reinterpret_cast<float*>(smem + kMOff) + hh * 32;        // running max per head column
    const float sl2 = p.scale_log2;
    if (sp == 0) msm[lane] = -INFINITY;
    float l_part[32];  // this thread's share (its token rows) of every column's sum
#pragma unroll
    for (int c = 0; c < 32; ++c) l_part[c] = 0.f;
    float m_lane = -INFINITY;  // lane c: the max head column 32 hh + c's exponentials use (base 2)
    named_sync(1 + hh, 128);
    // This half's head columns: 32 hh .. 32 hh + 31, or in a block of at most
    // 16 heads 8 hh .. 8 hh + 7. Each half writes its own 16-byte chunks of
    // every P^T row: its data chunk (4 hh .. 4 hh + 3, or hh) and, in a narrow
    // block, three of the six zero chunks 2 .. 7.
    const int cb = narrow ? 8 * hh : 32 * hh;
    auto chunk_of = [&](int q) { return narrow ? (q == 0 ? hh : 1 + 3 * hh + q) : 4 * hh + q; };
    if (hb * kNH + cb >= p.H) {
      // A column half with no head of this block: its P^T chunks are zero for
      // every tile, written once the score MMAs have read the tile's positional
      // chunk; nothing else is computed or stored.
      bool idle_ok = true;
      for (int i = 0; i < ntiles; ++i) {
        const int sb = i % kSlots;
        if (idle_ok)
          idle_ok =
              __all_sync(0xffffffffu, mbar_wait_bounded(bar(kMbSFull + sb), (i / kSlots) & 1, budget, abort_flag));
        if (!idle_ok) continue;
        if (lane == 0) mbar_arrive(bar(kMbSFree + sb));
        if (lane < 16) {
          uint8_t* pslot = smem + kKOff + sb * kTileBytes + kPSlot * kKChunkBytes;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int chunk = chunk_of(q);
            *reinterpret_cast<uint4*>(pslot + tok * 128 + ((chunk ^ (tok & 7)) << 4)) = make_uint4(0u, 0u, 0u, 0u);
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(kMbPFull + sb));
      }
      if (!idle_ok) mla_abort(abort_flag, p.status);
    } else {
    // Every softmax warp takes part in every named barrier of every tile, also
    // after a wait gave up (ok == false: it then skips its TMEM and mbarrier
    // work), so no warp can be left waiting at a barrier the others skipped.
    // NC: the head columns this warp scores (32, or 8 in a block of at most 16
    // heads, whose remaining columns of P^T are written as zeros).
    auto run = [&](auto nc_tag) {
    constexpr int NC = decltype(nc_tag)::value;
    bool ok = true;
    for (int i = 0; i < ntiles; ++i) {
      const int sb = i % kSlots;
      const uint32_t col_s = lane_base + kColS + 64u * sb + static_cast<uint32_t>(cb);
      if (ok)
        ok = __all_sync(0xffffffffu, mbar_wait_bounded(bar(kMbSFull + sb), (i / kSlots) & 1, budget, abort_flag));
      // lanes 16-31 of the sub-partition hold no score of an M = 64 tile
      const bool valid = ok && lane < 16 && (t0 + i * kTok + tok) < t1;
      float wmax = -INFINITY;
      if (ok) {
        tc_fence_after();
        uint32_t raw[NC];
        if constexpr (NC == 32) tmem_ld_32x32b_x32(col_s, raw);
        else tmem_ld_32x32b_x8(col_s, raw);
        tc_wait_ld();
        float v[NC];
#pragma unroll
        for (int c = 0; c < NC; ++c) v[c] = valid ? __uint_as_float(raw[c]) * sl2 : -INFINITY;
        wmax = warp_reduce_scatter<NC, true>(v, lane);  // lane c: column c % NC over this warp's 16 tokens
      }
      // tile max of every head column across the 4 warps; running max update
      red[sp * 32 + lane] = wmax;
      named_sync(1 + hh, 128);
      const float tmax = fmaxf(fmaxf(red[lane], red[32 + lane]), fmaxf(red[64 + lane], red[96 + lane]));
      const float m_old = msm[lane];
      named_sync(1 + hh, 128);  // red and msm are rewritten below / next tile
      const bool moved = tmax > m_old + kMlaRescaleThreshold;  // also the first tile (m_old = -inf)
      m_lane = moved ? tmax : m_old;
      const float a_lane = !moved ? 1.f : (m_old == -INFINITY ? 0.f : fast_exp2(m_old - tmax));
      if (sp == 0) msm[lane] = m_lane;
      if (!ok) continue;
      if (__any_sync(0xffffffffu, moved)) {
#pragma unroll
        for (int c = 0; c < NC; ++c) l_part[c] *= __shfl_sync(0xffffffffu, a_lane, c);
        if (i > 0) {
          // the previous tile's output MMAs must be complete before O^T is rescaled
          ok = __all_sync(0xffffffffu, mbar_wait_bounded(bar(kMbOReady), (i - 1) & 1, budget, abort_flag));
          if (!ok) continue;
          tc_fence_after();
#pragma unroll 1
          for (int m = 0; m < 4; ++m) {
            uint32_t ov[NC];  // only this half's columns: a narrow block's halves share a 32-column window
            const uint32_t col = lane_base + kColO + 64u * m + static_cast<uint32_t>(cb);
            if constexpr (NC == 32) tmem_ld_32x32b_x32(col, ov);
            else tmem_ld_32x32b_x8(col, ov);
            tc_wait_ld();
#pragma unroll
            for (int c = 0; c < NC; ++c)
              ov[c] = __float_as_uint(__uint_as_float(ov[c]) * __shfl_sync(0xffffffffu, a_lane, c));
            if constexpr (NC == 32) tmem_st_32x32b_x32(col, ov);
            else tmem_st_32x32b_x8(col, ov);
          }
          tc_wait_st();
        }
      }
      // probabilities from a second read of the scores (fewer live registers);
      // P^T row tok (lanes 0-15), head columns 32 hh .. + 31 -> 64 bytes of the
      // 128-byte swizzled row: 16-byte chunk q lands at chunk q ^ (tok & 7)
      uint32_t raw[NC];
      if constexpr (NC == 32) tmem_ld_32x32b_x32(col_s, raw);
      else tmem_ld_32x32b_x8(col_s, raw);
      tc_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kMbSFree + sb));
      uint32_t pk[16];
#pragma unroll
      for (int c = 0; c < 32; c += 2) {
        if (c < NC) {
          const float x0 = valid ? __uint_as_float(raw[c]) * sl2 : -INFINITY;
          const float x1 = valid ? __uint_as_float(raw[c + 1]) * sl2 : -INFINITY;
          const float p0 = fast_exp2(x0 - __shfl_sync(0xffffffffu, m_lane, c));
          const float p1 = fast_exp2(x1 - __shfl_sync(0xffffffffu, m_lane, c + 1));
          l_part[c] += p0;
          l_part[c + 1] += p1;
          pk[c >> 1] = pack_bf16x2(p0, p1);
        } else {
          pk[c >> 1] = 0u;  // the zero chunks of a narrow block
        }
      }
      if (lane < 16) {
        uint8_t* pslot = smem + kKOff + sb * kTileBytes + kPSlot * kKChunkBytes;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int chunk = chunk_of(q);
          *reinterpret_cast<uint4*>(pslot + tok * 128 + ((chunk ^ (tok & 7)) << 4)) =
              make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kMbPFull + sb));
    }
    // ------------------------------------------------------------ epilogue
    if (ok)
      ok = __all_sync(0xffffffffu, mbar_wait_bounded(bar(kMbOReady), (ntiles - 1) & 1, budget, abort_flag));
    if (!ok) mla_abort(abort_flag, p.status);
    tc_fence_after();
    // column sums of the probabilities over all 64 token rows
    float l_nc[NC];
#pragma unroll
    for (int c = 0; c < NC; ++c) l_nc[c] = l_part[c];
    const float wsum = warp_reduce_scatter<NC, false>(l_nc, lane);
    red[sp * 32 + lane] = wsum;
    named_sync(1 + hh, 128);
    const float csum = (red[lane] + red[32 + lane]) + (red[64 + lane] + red[96 + lane]);
    const bool out_ok = ok && (*bad_flag == 0);
    if (threadIdx.x == 0 && *bad_flag != 0 && p.status != nullptr) atomicOr(p.status, ATTN_STATUS_BIT_DEVICE_CHECK);
    const float inv_lane = 1.f / csum;
    const int head0 = hb * kNH + cb;
    if (sp == 0 && lane < NC && head0 + lane < p.H)  // one warp per column half writes the partial log-sum-exps
      p.lse_part[(static_cast<size_t>(b) * p.H + head0 + lane) * p.splits + split] =
          out_ok ? (m_lane + __log2f(csum)) * kLn2 : NAN;
#pragma unroll 1
    for (int m = 0; m < 4; ++m) {
      uint32_t ov[32];
      tmem_ld_32x32b_x32(lane_base + kColO + 64u * m + static_cast<uint32_t>(cb), ov);
      tc_wait_ld();
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        const float inv = __shfl_sync(0xffffffffu, inv_lane, c);
        if (c < NC && head0 + c < p.H)
          p.o_part[((static_cast<size_t>(b) * p.H + head0 + c) * p.splits + split) * kDc + m * 128 + r] =
              out_ok ? __uint_as_float(ov[c]) * inv : NAN;
      }
    }
    };
    if (narrow) run(std::integral_constant<int, 8>{});
    else run(std::integral_constant<int, 32>{});
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMlaMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// A rank-3 bf16 tensor (cols innermost) with 64-column boxes of box_rows x 1,
// 128-byte swizzle; out-of-range rows and blocks read as zero.
bool encode_rank3(CUtensorMap* map, const void* base, int cols, int rows, int depth, int box_rows) {
  const auto enc = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(tensor_map_encode_fn());
  if (enc == nullptr) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows),
                              static_cast<cuuint64_t>(depth)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(cols) * 2, static_cast<cuuint64_t>(rows) * cols * 2};
  const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
  const cuuint32_t estride[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estride,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

int plan_mla(int B, int H, int max_seq_len, int num_sms, MlaPlan* out) {
  if (B <= 0 || H <= 0 || max_seq_len <= 0 || num_sms <= 0 || out == nullptr) return ATTN_ERR_INVALID_ARG;
  // One CTA per SM (its shared memory): aim for two waves of (sequence, head
  // block, split) CTAs; long splits keep the fp32 partials small next to the
  // cache bytes they summarise.
  const long long units = static_cast<long long>(B) * ((H + kNH - 1) / kNH);
  int chunk = 4096;
  while (chunk > 512 && units * ((max_seq_len + chunk - 1) / chunk) < 2LL * num_sms) chunk >>= 1;
  const int tiles = (max_seq_len + kTok - 1) / kTok;
  const int nominal = (max_seq_len + chunk - 1) / chunk;
  out->chunk = kTok * ((tiles + nominal - 1) / nominal);  // tiles spread evenly over the splits
  out->splits = (max_seq_len + out->chunk - 1) / out->chunk;
  return ATTN_OK;
}

size_t mla_workspace_bytes(int B, int H, const MlaPlan& plan) {
  const size_t rows = static_cast<size_t>(B) * H * plan.splits;
  return rows * kDc * sizeof(float) + rows * sizeof(float);
}

int launch_mla_decode(const void* q, const void* cache, const int32_t* block_table, const int32_t* seq_lens, void* o,
                      float* lse, int B, int H, int num_blocks, int block_size, int max_blocks_per_seq,
                      int max_seq_len, float scale, void* workspace, const MlaPlan& plan, int32_t* status,
                      cudaStream_t stream) {
  CUtensorMap tq, tc, tcr;
  const int box_rows = block_size < kTok ? block_size : kTok;  // 64-row boxes inside 128-token blocks
  if (!encode_rank3(&tq, q, kRow, H, B, kNH) || !encode_rank3(&tc, cache, kRow, block_size, num_blocks, box_rows) ||
      !encode_rank3(&tcr, cache, kRow, block_size, num_blocks, 1))
    return ATTN_ERR_CUDA;
  MlaParams p;
  p.block_table = block_table;
  p.seq_lens = seq_lens;
  p.o_part = static_cast<float*>(workspace);
  p.lse_part = p.o_part + static_cast<size_t>(B) * H * plan.splits * kDc;
  p.status = status;
  p.B = B;
  p.H = H;
  p.num_blocks = num_blocks;
  p.block_size = block_size;
  p.max_blocks = max_blocks_per_seq;
  p.max_seq_len = max_seq_len;
  p.chunk = plan.chunk;
  p.splits = plan.splits;
  p.scale_log2 = scale * kLog2e;
  p.budget = wait_budget_cycles();
  if (cudaFuncSetAttribute(mla_split_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemAlloc) !=
      cudaSuccess)
    return ATTN_ERR_CUDA;
  const dim3 grid(plan.splits, (H + kNH - 1) / kNH, B);
  mla_split_kernel<<<grid, kMlaThreads, kSmemAlloc, stream>>>(tq, tc, tcr, p);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  const cudaError_t e = launch_decode_merge(p.o_part, p.lse_part, seq_lens, nullptr, o, lse, B, H, kDc, plan.splits,
                                            plan.chunk, max_seq_len, 0, 0, status, stream);
  return e == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // namespace attn
