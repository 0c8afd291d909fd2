// hca_attn.cu -- HCA attention forward on sm_100a (tcgen05 + TMEM + TMA).
//
// Method: the mirrorspeed page, section "Hybrid sparse attention, 1/7 full context
// access" (and the besthub page, "Core Architectural Innovations", item 1): the cache
// keeps one entry per 128 tokens, and a query attends to those entries together with the
// latest raw tokens; HCA heads are 512 wide (ai-club.cn page,
// section "混合注意力（MLA + HCA）").  Visible set of a query at t (this library's
// reading): raw positions [max(0,t-W+1), t] and entries j < n_c(t) = max(0,(t-W+1)/blk).
//
// Kernel design (persistent: a CTA walks row tiles T = blockIdx.x + i*gridDim.x):
//   * A row tile = 128 rows = (128/g) consecutive tokens x the g query heads sharing one K/V
//     head, so every K/V tile is shared by the whole tile and the window band of 128/g
//     tokens spans only 128/g + W - 1 keys.
//   * d = 512 makes a 128 x 512 fp32 O accumulator fill all of TMEM, so O is built one
//     256-wide half of d_v at a time: TMEM = O half [0,256) + two S buffers [256,384),
//     [384,512).  Phase A of a tile computes S_j = Q K_j^T, the online softmax and
//     O[:, 0:256] += P_j V_j[:, 0:256]; it also writes each P_j (bf16) and the rescale
//     factor it applied to a per-CTA scratch (L2-resident).  Phase B reloads those P_j into
//     TMEM and runs only O[:, 256:512] += P_j V_j[:, 256:512] with the same rescales, so the
//     second half costs no QK^T and no exponentials, and Q's buffer is free to take the
//     next tile's Q while phase B runs.
//   * warp 0: TMA producer (Q per tile; K and V through a ring of two 32 KB groups, in exactly
//     the order the MMA warp consumes them: a K group is 128 d-columns of a key tile (two 16 KB
//     chunks of 128 rows), a V group 64 keys x one 256-column half of d_v (four 8 KB chunks);
//     key tiles of at most 32 keys use 32-row boxes); warp 1: TMEM allocation and the single
//     MMA-issuing thread.  One barrier wait per group: a wait costs the issuing thread a few
//     hundred cycles, which only ~500 cycles of queued MMA work hide (8 QK^T MMAs of N = 128,
//     or 4 PV MMAs of N = 256); warps 2-5: softmax and the P reloads, one thread per row (TMEM
//     lane); warps 6-9: the epilogues, which read each O half out of TMEM, hand it back to the
//     MMA warp and stage it through shared memory (64-byte swizzle, four 8 KB boxes) into TMA
//     tensor stores, while the softmax warps go on with the next half or row tile.
//   * S_j accumulates over eight 64-wide d chunks (SS MMA, K-major operands, 128B swizzle).
//     P_j is written in place over S_j in TMEM and PV runs as a TS MMA (A = P from TMEM,
//     B = V, MN-major, N = 256 over a V group's four chunks).  Online softmax with a lazy
//     rescale: the reference max only moves when the tile max exceeds it by 2^8.
//   * Key tiles: compressed entries [0, n_c(t_last)) in tiles of 128, then the window
//     band [max(0, t_first-W+1), t_last] in tiles of 128; per-row visibility is one
//     column interval per tile.  The band of 128/g tokens is 128/g + W - 1 keys long, so with
//     W = 128 it overhangs one tile by a few keys; when those fit beside the last, partial tile
//     of compressed entries, the two share one "merged" key tile (rows [0,16) = the band's
//     first 16 keys, rows [16,128) = the entries) instead of costing a QK^T of their own, and
//     that tile has two visible intervals per row.
//   * Barrier phases run on across tiles: p_ready / pv_done are per S buffer and follow a
//     key-tile counter that never resets (phase A and phase B tiles both count); s_full is per
//     S buffer too but only phase-A tiles complete it, so its consumer keeps one parity bit per
//     buffer; o_full / o_empty follow the O-half counter, q_full / q_empty the row-tile counter.
//     MMAs on different accumulators are not ordered, so an S buffer is rewritten (by QK^T
//     or by a P reload) only after the PV that read its previous P has completed.
#include <cuda_bf16.h>

#include <mutex>

#include "host_common.h"
#include "ptx.cuh"

namespace hcadsa {
namespace {

constexpr int kD = 512;      // value width (and score width of the standard head shape)
constexpr int kDHalf = 256;
constexpr int kKeyTile = 128;
constexpr int kSmallRows = 32;  // TMA box height for key tiles of at most 32 keys
constexpr int kMergeWinRows = 16;                       // window keys at the head of a merged tile
constexpr int kMergeEntRows = kKeyTile - kMergeWinRows;  // compressed entries after them
// Ring: 32 KB groups (a K group: two 16 KB chunks of 128 rows; a V group: four 8 KB chunks of 64
// rows).  Two groups; the third group's space is the epilogue's staging area, or a third group
// when key ranges are split (those epilogues write fp32 partials straight to global memory).
constexpr int kGroups = 2;
constexpr int kMaxGroups = 3;
constexpr int kChunkBytes = 128 * 128;  // 128 rows x 64 bf16
constexpr int kSmallChunkBytes = kSmallRows * 128;
constexpr int kVChunks = kDHalf / 64;  // 4
constexpr int kVRows = 64;             // keys per V ring group (4 chunks of 64 keys x 64 columns)
constexpr int kVChunkBytes = kVRows * 128;
constexpr int kOutCols = 32;                  // O columns per TMA store box
constexpr int kOutBufBytes = 128 * kOutCols * 2;  // 8 KB
constexpr int kGroupBytes = 2 * kChunkBytes;

// Shared-memory plan per score width DQK (the value width is always 512):
//   DQK = 512: Q 128 KB + two ring groups + a third 32 KB region that is the epilogue's staging
//              (four 32-column boxes = 128 columns of O per round) or, with split key ranges, a
//              third ring group.
//   DQK = 576 (FlashMask-4's qk 576 / v 512 shape: 512-wide latent + 64-wide positional slice):
//              Q 144 KB + two ring groups + a 16 KB staging area (two boxes = 64 columns per
//              round); split key ranges keep two ring groups.  225 KB either way.
template <int DQK>
struct Shape {
  static constexpr int kQChunks = DQK / 64;           // 8 or 9 chunks of 64 score columns
  static constexpr int kQBytes = kQChunks * kChunkBytes;
  static constexpr int kOutBufs = DQK == 512 ? 4 : 2;  // staging boxes per round
  static constexpr int kMaxGroups = DQK == 512 ? 3 : 2;
  static constexpr int kExtraBytes = DQK == 512 ? kGroupBytes : kOutBufs * kOutBufBytes;
  static constexpr int kSmemBytes = kQBytes + kGroups * kGroupBytes + kExtraBytes + 1024;
  static_assert(DQK == 512 || DQK == 576, "score width");
  static_assert(kOutBufs * kOutBufBytes <= kExtraBytes, "staging fits its region");
  static_assert((kMaxGroups - kGroups) * kGroupBytes <= kExtraBytes, "split-mode ring group fits");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory");
};
constexpr int kThreads = 320;
constexpr int kSoftmaxWarp0 = 2;   // warps 2-5: softmax and P reloads
constexpr int kEpilogueWarp0 = 6;  // warps 6-9: O read-out and stores
constexpr float kLazyRescale = 8.0f;  // log2 units
// per-CTA scratch per key tile: P (128 rows x 128 keys bf16) + one fp32 rescale factor per row
constexpr size_t kScratchPBytes = 128 * kKeyTile * 2;
constexpr size_t kScratchTileBytes = kScratchPBytes + 128 * 4;

struct Params {
  int Lq, q_offset, Hq, Hkv, g, TT, n_c, win_start, W, blk;
  int n_tiles;      // token tiles per (b, kv head)
  int total_tiles;  // B * Hkv * n_tiles
  int splits;       // work units per row tile (key tiles split among them) ...
  int split_extra;  // ... plus one more for the first split_extra row tiles
  int split_mode;   // units write partial results for the combine pass
  int total_units;  // total_tiles * splits + split_extra (stream_k: record slots, grid + total_tiles)
  int stream_k;     // split mode with equal row tiles: CTA c takes key tiles [c*Jtot/G, (c+1)*Jtot/G)
  int J_all;        // stream_k: key tiles of every row tile (Jtot = total_tiles * J_all)
  int sk_grid;      // stream_k: G, the attention kernel's grid
  int J_max;        // key tiles of the longest row tile (scratch capacity)
  float scale_log2;
  float* lse;
  uint8_t* scratch;  // gridDim.x * J_max * kScratchTileBytes
  float* part_o;     // split mode: [total_units][128][512] unnormalised O of each unit
  float2* part_ml;   // split mode: [total_units][128] (reference max in log2 units, row sum)
  uint16_t* O;       // the output (stored directly by the epilogue when deep_ring)
  int deep_ring;     // 512 shape, long rows: the staging region is a third ring group
  int* err;
};

// Q and O, then K and V over {compressed entries, window} x box heights, and the two boxes of
// each half of a merged key tile.
struct Maps {
  CUtensorMap q;
  CUtensorMap o;          // box 32 columns x 128 rows, 64-byte swizzle (stores)
  CUtensorMap k[2][2];    // [0 = compressed, 1 = window][0 = 128 rows, 1 = 32 rows]
  CUtensorMap v[2][2];    // [0 = compressed, 1 = window][0 = 64 rows, 1 = 32 rows]
  CUtensorMap kmerge[2];  // [0 = window 16 rows, 1 = compressed 112 rows]
  CUtensorMap vmerge[2];  // [0 = window 16 rows, 1 = compressed 48 rows]
};

__device__ __forceinline__ int n_compressed(int t, int W, int blk) {
  const int s = t - W + 1;
  return s > 0 ? s / blk : 0;
}
__device__ __forceinline__ int window_start(int t, int W) {
  const int s = t - W + 1;
  return s > 0 ? s : 0;
}

// tcgen05.wait::ld naming the 16 destination registers of the loads it completes, so the
// compiler cannot move their uses above the wait
__device__ __forceinline__ void tmem_wait_ld_regs16(uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.wait::ld.sync.aligned;"
      : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
        "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15])
      :
      : "memory");
}

__device__ __forceinline__ void softmax_bar_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_group_read1() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}

struct KeyTile {
  int kind;    // 0: compressed entries, 1: raw window positions, 2: merged (window keys, then entries)
  int start;   // first entry (kinds 0, 2) / position (kind 1)
  int n;       // MMA N (multiple of 16, <= 128)
  int wstart;  // kind 2: first window position (tile rows [0, 16))
  int wn;      // kind 2: window keys the tile owns (<= 16; the band's later keys are in window tiles)
};

__host__ __device__ inline int first_unit(int T, const Params& p) { return T * p.splits + min(T, p.split_extra); }
__host__ __device__ inline int n_splits(int T, const Params& p) { return p.splits + (T < p.split_extra ? 1 : 0); }

// Stream-K split (every row tile has J_all key tiles): all row tiles' key tiles laid end to end,
// Jtot = total_tiles * J_all of them, and CTA c takes [c*Jtot/G, (c+1)*Jtot/G).  Its piece of row
// tile T is the unit with record index c + T (unique: both grow along the key-tile order), so a
// CTA's units are consecutive records and so are a row tile's: CTAs c_first(T) .. c_last(T), the
// ones holding the row tile's first and last key tiles.
// (The host enables it only while Jtot * (G + 1) < 2^31, so 32-bit arithmetic is exact.)
__host__ __device__ inline int sk_cta_start(int c, const Params& p) {
  return (int)((unsigned)c * (unsigned)(p.total_tiles * p.J_all) / (unsigned)p.sk_grid);
}
__host__ __device__ inline int sk_cta_of(int x, const Params& p) {  // CTA holding global key tile x
  return (int)(((unsigned)(x + 1) * (unsigned)p.sk_grid - 1u) / (unsigned)(p.total_tiles * p.J_all));
}

// The units (record indices) this CTA processes: first, first + step, ... below end, with
// step = 1 (stream_k) or gridDim.x.  With stream_k the CTA also keeps its key-tile range
// [lo, hi).  Kept in shared memory (set once at kernel start) and read where needed, so the
// per-unit loops do not hold them in registers.
struct UnitInfo {
  int first, end;   // units
  int js_first;     // stream_k: first key tile of the first unit (later units start at 0)
  int je_last;      // stream_k: end key tile of the last unit (earlier units end at J_all)
};
__device__ __forceinline__ UnitInfo unit_info(const Params& p) {
  UnitInfo u;
  if (p.stream_k) {
    const int lo = sk_cta_start(blockIdx.x, p), hi = sk_cta_start(blockIdx.x + 1, p);
    const int T0 = lo / p.J_all, T1 = (hi - 1) / p.J_all;
    u.first = (int)blockIdx.x + T0;
    u.end = (int)blockIdx.x + T1 + 1;
    u.js_first = lo - T0 * p.J_all;
    u.je_last = hi - T1 * p.J_all;
  } else {
    u.first = (int)blockIdx.x;
    u.end = p.total_units;
    u.js_first = 0;
    u.je_last = 0;
  }
  return u;
}
__device__ __forceinline__ int unit_step(const Params& p) { return p.stream_k ? 1 : (int)gridDim.x; }
__shared__ UnitInfo s_units;  // this CTA's units, set once by thread 0 at kernel start

// The key tiles of one work unit: split s of row tile T (S = n_splits(T) units from
// first_unit(T)) takes the row tile's key tiles [s*Jt/S, (s+1)*Jt/S); with stream_k, unit
// c + T of CTA c takes the row tile's share of [c*Jtot/G, (c+1)*Jtot/G).
struct TileSet {
  int b, hk, tok0;  // batch, kv head, first token (relative to q_offset)
  int J_c, J;       // number of compressed tiles of the row tile, key tiles of this unit
  int js;           // first key tile of this unit
  int nc_hi;        // entries needed by the last token
  int ws_lo;        // window start of the first token
  int t_hi;         // last valid token position
  int w_part;       // keys of the band beyond its whole 128-key tiles (1..128)
  int merged;       // 1: the band's first w_part keys share the last compressed tile
  __device__ void init(int U, const Params& p) {
    int T, split = 0, S = 1;
    if (p.stream_k) {
      T = U - (int)blockIdx.x;
    } else {
      const int big = p.split_extra * (p.splits + 1);  // units of the row tiles with an extra split
      T = U < big ? U / (p.splits + 1) : p.split_extra + (U - big) / p.splits;
      split = U - first_unit(T, p);
      S = n_splits(T, p);
    }
    init_tile(T, p);
    const int Jt = J;
    if (p.stream_k) {  // Jt == J_all
      js = U == s_units.first ? s_units.js_first : 0;
      J = (U == s_units.end - 1 ? s_units.je_last : Jt) - js;
    } else {
      js = split * Jt / S;
      J = (split + 1) * Jt / S - js;
    }
  }
  // row tile T: everything but the key-tile range of the unit (J = all of the row tile's tiles)
  __device__ __forceinline__ void init_tile(int T, const Params& p) {
    const int bh = T / p.n_tiles, tile = T % p.n_tiles;
    b = bh / p.Hkv;
    hk = bh % p.Hkv;
    tok0 = tile * p.TT;
    t_hi = p.q_offset + min(tok0 + p.TT, p.Lq) - 1;
    nc_hi = n_compressed(t_hi, p.W, p.blk);
    ws_lo = window_start(p.q_offset + tok0, p.W);
    J_c = (nc_hi + kKeyTile - 1) / kKeyTile;
    const int w_span = t_hi - ws_lo + 1;
    const int n_wt = (w_span + kKeyTile - 1) / kKeyTile;
    w_part = w_span - (n_wt - 1) * kKeyTile;
    merged = J_c >= 1 && n_wt >= 2 && w_part <= kMergeWinRows && nc_hi - (J_c - 1) * kKeyTile <= kMergeEntRows;
    J = J_c + n_wt - merged;
    js = 0;
  }
  __device__ KeyTile get(int jl) const {
    KeyTile kt;
    const int j = js + jl;
    kt.wstart = 0;
    kt.wn = 0;
    if (j < J_c) {
      kt.kind = merged && j == J_c - 1 ? 2 : 0;
      kt.start = j * kKeyTile;
      const int rem = nc_hi - kt.start;
      if (kt.kind == 2) {
        kt.wstart = ws_lo;
        kt.wn = w_part;
        kt.n = kMergeWinRows + ((rem + 15) & ~15);
      } else {
        kt.n = (min(kKeyTile, rem) + 15) & ~15;
      }
    } else {
      kt.kind = 1;
      // after a merged tile the band continues at its (w_part+1)-th key in whole tiles
      kt.start = ws_lo + (merged ? w_part : 0) + (j - J_c) * kKeyTile;
      const int rem = min(kKeyTile, t_hi + 1 - kt.start);
      kt.n = (rem + 15) & ~15;
    }
    return kt;
  }
};

struct __align__(8) Barriers {
  uint64_t q_full, q_empty;
  uint64_t full[kMaxGroups];   // both chunks of a ring group landed
  uint64_t empty[kMaxGroups];  // the MMAs that read the group have completed
  uint64_t s_full[2];
  uint64_t p_ready[2];
  uint64_t pv_done[2];  // the PV that read P from S buffer i has completed
  uint64_t o_full;      // every PV of the current O half has completed
  uint64_t o_empty[2];  // the epilogue has read O columns [0,128) / [128,256)
  uint64_t l_ready[2];  // the softmax warps have written 1/l of row tile i (mod 2)
  uint64_t l_empty[2];  // the epilogue warps have stored both O halves of that row tile
};

// One thread's row of P_j in the scratch: key tile j owns kScratchTileBytes; inside it the
// 16-byte unit c16 (8 keys) of row r is unit c16*128 + r, so a warp's 32 rows are one
// contiguous 512-byte run; the 128 rescale factors follow the P units.
__device__ __forceinline__ uint4* scratch_p(uint8_t* base, int j, int r) {
  return reinterpret_cast<uint4*>(base + (size_t)j * kScratchTileBytes) + r;
}
__device__ __forceinline__ float* scratch_alpha(uint8_t* base, int j, int r) {
  return reinterpret_cast<float*>(base + (size_t)j * kScratchTileBytes + kScratchPBytes) + r;
}

// Loads row r of P_j (n keys) from the scratch into 16 registers of 8 keys each.
__device__ __forceinline__ void load_p_row(uint4 (&pr)[16], float& alpha, uint8_t* base, int j, int n, int r) {
  const uint4* src = scratch_p(base, j, r);
#pragma unroll
  for (int c = 0; c < 16; ++c)
    pr[c] = c * 8 < n ? __ldcg(src + c * 128) : make_uint4(0u, 0u, 0u, 0u);
  alpha = n > 0 ? __ldcg(scratch_alpha(base, j, r)) : 1.0f;
}

// Multiplies this thread's row of the O half by alpha.
__device__ __forceinline__ void rescale_o(uint32_t t_row, float alpha) {
  for (int oc = 0; oc < kDHalf; oc += 32) {
    uint32_t v[32];
    tmem_ld32_nowait(t_row + oc, v);
    tmem_wait_ld_regs(v);
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * alpha);
    tmem_st32(t_row + oc, v);
  }
  tmem_wait_st();
}

template <int DQK>
__global__ void __launch_bounds__(kThreads, 1) hca_attn_kernel(const __grid_constant__ Maps maps, const __grid_constant__ Params p) {
  using S = Shape<DQK>;
  constexpr int kQChunks = S::kQChunks;
  constexpr int kQBytes = S::kQBytes;
  constexpr int kOutBufs = S::kOutBufs;
  constexpr int kMaxGroups = S::kMaxGroups;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sRing = smem + kQBytes;
  uint8_t* sOut = sRing + kGroups * kGroupBytes;
  __shared__ Barriers bar;
  __shared__ float inv_l_sh[2][128];  // 1/l per row (1 in split mode), double-buffered by row tile
  UnitInfo& ui = s_units;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    mbar_init(&bar.q_full, 1);
    mbar_init(&bar.q_empty, 1);
    for (int s = 0; s < kMaxGroups; ++s) {
      mbar_init(&bar.full[s], 1);
      mbar_init(&bar.empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar.s_full[s], 1);
      mbar_init(&bar.p_ready[s], 128);
      mbar_init(&bar.pv_done[s], 1);
    }
    mbar_init(&bar.o_full, 1);
    mbar_init(&bar.o_empty[0], 128);
    mbar_init(&bar.o_empty[1], 128);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar.l_ready[s], 128);
      mbar_init(&bar.l_empty[s], 128);
    }
    abort_flag = 0;
    ui = unit_info(p);
    fence_mbarrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_sh, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&maps.q);
      const uint32_t ngroups = (p.split_mode || p.deep_ring) ? kMaxGroups : kGroups;
      uint32_t grp = 0, gph = 0;  // next ring group to fill and the phase of its use
      bool ok = true;
      auto next_group = [&]() {
        if (++grp == ngroups) {
          grp = 0;
          gph ^= 1;
        }
      };
      // K: all rows of key tile kt x columns col .. col + 64 nch - 1 (nch = 2 16 KB chunks, or 1 for
      // the last, odd chunk of a 576-wide score) into the next group
      auto load_k = [&](const KeyTile& kt, int col, int hk, int b, int nch) {
        ok = mbar_wait(&bar.empty[grp], gph ^ 1, &abort_flag, p.err);
        if (ok) {
          uint8_t* dst = sRing + grp * kGroupBytes;
          if (kt.kind == 2) {  // 16 window rows, then 112 entry rows: both boxes fill the chunk
            mbar_arrive_expect_tx(&bar.full[grp], nch * kChunkBytes);
            for (int cc = 0; cc < nch; ++cc) {
              tma_load_4d(dst + cc * kChunkBytes, &maps.kmerge[0], &bar.full[grp], col + cc * 64, hk,
                          kt.wstart - p.win_start, b);
              tma_load_4d(dst + cc * kChunkBytes + kMergeWinRows * 128, &maps.kmerge[1], &bar.full[grp],
                          col + cc * 64, hk, kt.start, b);
            }
          } else {
            const int small = kt.n <= kSmallRows ? 1 : 0;
            const CUtensorMap* m = &maps.k[kt.kind][small];
            const int row0 = kt.kind ? kt.start - p.win_start : kt.start;
            mbar_arrive_expect_tx(&bar.full[grp], nch * (small ? kSmallChunkBytes : kChunkBytes));
            tma_load_4d(dst, m, &bar.full[grp], col, hk, row0, b);
            if (nch == 2) tma_load_4d(dst + kChunkBytes, m, &bar.full[grp], col + 64, hk, row0, b);
          }
        }
        next_group();
      };
      // V: rows [64 gi, 64 gi + 64) of key tile kt x columns col0 .. col0+255 (four 8 KB chunks)
      // into the next group
      auto load_vgroup = [&](const KeyTile& kt, int gi, int col0, int hk, int b) {
        ok = mbar_wait(&bar.empty[grp], gph ^ 1, &abort_flag, p.err);
        if (ok) {
          uint8_t* dst = sRing + grp * kGroupBytes;
          if (kt.kind == 2 && gi == 0) {  // 16 window rows, then 48 entry rows
            mbar_arrive_expect_tx(&bar.full[grp], kVChunks * kVChunkBytes);
            for (int c = 0; c < kVChunks; ++c) {
              tma_load_4d(dst + c * kVChunkBytes, &maps.vmerge[0], &bar.full[grp], col0 + c * 64, hk,
                          kt.wstart - p.win_start, b);
              tma_load_4d(dst + c * kVChunkBytes + kMergeWinRows * 128, &maps.vmerge[1], &bar.full[grp],
                          col0 + c * 64, hk, kt.start, b);
            }
          } else {
            // tile row r of a merged tile (r >= 16) holds entry start + r - 16
            const int kind = kt.kind == 1 ? 1 : 0;
            const int small = kt.n <= kSmallRows ? 1 : 0;
            const int row0 = (kt.kind == 1 ? kt.start - p.win_start : kt.start) + gi * kVRows -
                             (kt.kind == 2 ? kMergeWinRows : 0);
            mbar_arrive_expect_tx(&bar.full[grp], kVChunks * (small ? kSmallRows : kVRows) * 128);
            for (int c = 0; c < kVChunks; ++c)
              tma_load_4d(dst + c * kVChunkBytes, &maps.v[kind][small], &bar.full[grp], col0 + c * 64, hk, row0, b);
          }
        }
        next_group();
      };
      auto load_v = [&](const TileSet& ts, int j, int col0) {
        const KeyTile kt = ts.get(j);
        const int ngv = kt.n > kVRows ? 2 : 1;
        for (int gi = 0; ok && gi < ngv; ++gi) load_vgroup(kt, gi, col0, ts.hk, ts.b);
      };
      if (ui.first < ui.end) {
        TileSet t0;
        t0.init(ui.first, p);
        mbar_arrive_expect_tx(&bar.q_full, kQBytes);
        for (int c = 0; c < kQChunks; ++c)
          tma_load_4d(sQ + c * kChunkBytes, &maps.q, &bar.q_full, c * 64, t0.hk * p.g, t0.tok0, t0.b);
      }
      uint32_t tcount = 0;
      for (int T = ui.first; ok && T < ui.end; T += unit_step(p), ++tcount) {
        TileSet ts;
        ts.init(T, p);
        if (ts.J > p.J_max) break;
        // phase A: step s loads the K chunks of key tile s, then the first-half V chunks of tile s-1
        for (int step = 0; ok && step <= ts.J; ++step) {
          if (step < ts.J) {
            const KeyTile kt = ts.get(step);
            for (int c = 0; ok && c < kQChunks; c += 2) load_k(kt, c * 64, ts.hk, ts.b, kQChunks - c >= 2 ? 2 : 1);
          }
          if (ok && step >= 1) load_v(ts, step - 1, 0);
        }
        if (!ok) break;
        // the next tile's Q, once this tile's last S MMA has read the buffer
        const int Tn = T + unit_step(p);
        if (Tn < ui.end) {
          TileSet tn;
          tn.init(Tn, p);
          ok = mbar_wait(&bar.q_empty, tcount & 1, &abort_flag, p.err);
          if (!ok) break;
          mbar_arrive_expect_tx(&bar.q_full, kQBytes);
          for (int c = 0; c < kQChunks; ++c)
            tma_load_4d(sQ + c * kChunkBytes, &maps.q, &bar.q_full, c * 64, tn.hk * p.g, tn.tok0, tn.b);
        }
        // phase B: second-half V chunks
        for (int j = 0; ok && j < ts.J; ++j) load_v(ts, j, kDHalf);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t sQa = smem_u32(sQ), sRa = smem_u32(sRing);
      const uint32_t ngroups = (p.split_mode || p.deep_ring) ? kMaxGroups : kGroups;
      uint32_t grp = 0, gph = 0;  // next ring group to consume and the phase of its use
      auto next_group = [&]() {
        if (++grp == ngroups) {
          grp = 0;
          gph ^= 1;
        }
      };
      uint32_t tcount = 0;  // row tiles
      uint32_t g = 0;       // key tiles of all earlier phases
      uint32_t it = 0;      // O halves
      bool ok = true;
      // N = 256: one PV MMA covers the whole O half, the four 64-column chunks of a V group
      // (LBO = one 8 KB chunk); its 64 keys take four MMAs of K = 16
      const uint32_t idesc_pv = idesc_bf16_f32(128, kDHalf, false, true);
      // descriptors of the ring groups and of Q; the start-address field counts 16-byte units
      const uint64_t dq0 = smem_desc_sw128(sQa, 16, 1024);
      const uint64_t dk0 = smem_desc_sw128(sRa, 16, 1024);
      const uint64_t dv0 = smem_desc_sw128(sRa, kVChunkBytes, 1024);
      constexpr uint64_t kGroupDesc = kGroupBytes >> 4;  // group offset in descriptor units
      // PV of key tile j (global counter gj) into the O half; V from one group per 64 keys
      auto pv = [&](const KeyTile& kt, int j, uint32_t gj) {
        const uint32_t tP = tmem + kDHalf + (gj & 1) * kKeyTile;
        if (j == 0) {  // the previous O half's epilogue must have read all of it
          for (int hh = 0; ok && hh < 2; ++hh) ok = mbar_wait(&bar.o_empty[hh], (it & 1) ^ 1, &abort_flag, p.err);
          if (!ok) return;
        }
        const int ngv = kt.n > kVRows ? 2 : 1;
        for (int gi = 0; ok && gi < ngv; ++gi, next_group()) {
          ok = mbar_wait(&bar.full[grp], gph, &abort_flag, p.err);
          if (!ok) break;
          tc_fence_after();
          const uint64_t db = dv0 + grp * kGroupDesc;
          const int nk = min(kVRows, kt.n - gi * kVRows) / 16;
          for (int kk = 0; kk < nk; ++kk)  // P columns of keys 64 gi + 16 kk .. +15 (bf16 pairs)
            mma_ts(tmem, tP + (gi * 4 + kk) * 8, db + (uint64_t)(kk * (2048 >> 4)), idesc_pv,
                   (j > 0 || gi > 0 || kk > 0) ? 1u : 0u);
          mma_commit(&bar.empty[grp]);
        }
      };
      for (int T = ui.first; ok && T < ui.end; T += unit_step(p), ++tcount) {
        TileSet ts;
        ts.init(T, p);
        if (ts.J > p.J_max) {
          raise_device_error(p.err, kErrDeviceBounds);
          break;
        }
        ok = mbar_wait(&bar.q_full, tcount & 1, &abort_flag, p.err);
        if (!ok) break;
        tc_fence_after();
        // ---- phase A: step s issues QK_s, then PV_{s-1} (first half of d_v)
        for (int step = 0; ok && step <= ts.J; ++step) {
          if (step < ts.J) {
            const uint32_t gs = g + step;
            const KeyTile kt = ts.get(step);
            const uint32_t tS = tmem + kDHalf + (gs & 1) * kKeyTile;
            const uint32_t idesc = idesc_bf16_f32(128, kt.n, false, false);
            if (gs >= 2) {  // S buffer gs&1 holds P_{gs-2}, the TMEM operand of PV_{gs-2}
              ok = mbar_wait(&bar.pv_done[gs & 1], ((gs >> 1) - 1) & 1, &abort_flag, p.err);
              if (!ok) break;
              tc_fence_after();
            }
            for (int c = 0; ok && c < kQChunks; c += 2, next_group()) {
              ok = mbar_wait(&bar.full[grp], gph, &abort_flag, p.err);
              if (!ok) break;
              tc_fence_after();
              const uint64_t da = dq0 + (uint64_t)((c * kChunkBytes) >> 4);
              const uint64_t db = dk0 + grp * kGroupDesc;
#pragma unroll
              for (int cc = 0; cc < 2; ++cc) {
                if (kQChunks % 2 == 1 && c + cc >= kQChunks) break;  // the odd last chunk (576 wide)
#pragma unroll
                for (int k = 0; k < 4; ++k)
                  mma_ss(tS, da + (uint64_t)((cc * kChunkBytes + k * 32) >> 4),
                         db + (uint64_t)((cc * kChunkBytes + k * 32) >> 4), idesc, (c | cc | k) != 0);
              }
              mma_commit(&bar.empty[grp]);
            }
            if (!ok) break;
            mma_commit(&bar.s_full[gs & 1]);
            if (step == ts.J - 1) mma_commit(&bar.q_empty);
          }
          if (step >= 1) {
            const int j = step - 1;
            const uint32_t gj = g + j;
            ok = mbar_wait(&bar.p_ready[gj & 1], (gj >> 1) & 1, &abort_flag, p.err);
            if (!ok) break;
            tc_fence_after();
            pv(ts.get(j), j, gj);
            if (!ok) break;
            mma_commit(&bar.pv_done[gj & 1]);
            if (j == ts.J - 1) mma_commit(&bar.o_full);
          }
        }
        if (!ok) break;
        g += ts.J;
        ++it;
        // ---- phase B: PV only (second half of d_v), P reloaded into TMEM by the softmax warps
        for (int j = 0; ok && j < ts.J; ++j) {
          const uint32_t gj = g + j;
          ok = mbar_wait(&bar.p_ready[gj & 1], (gj >> 1) & 1, &abort_flag, p.err);
          if (!ok) break;
          tc_fence_after();
          pv(ts.get(j), j, gj);
          if (!ok) break;
          mma_commit(&bar.pv_done[gj & 1]);
          if (j == ts.J - 1) mma_commit(&bar.o_full);
        }
        g += ts.J;
        ++it;
      }
    }
  } else if (warp >= kEpilogueWarp0) {
    // ------------------------------------------------------------ epilogue
    // Runs beside the softmax warps: while it reads out and stores one O half, they already
    // reload P for the next half or run the next row tile's softmax.
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // row of the tile == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const bool store_issuer = r == 0;
    uint32_t it = 0, tl = 0;  // O halves, row tiles
    bool ok = true;

    // One O half per call.  With split key ranges the unit's unnormalised fp32 O rows go
    // straight to part_o; otherwise they are normalised, staged and stored (below).
    auto epilogue = [&](const TileSet& ts, int col0, float inv_l, int U, bool row_valid) {
      ok = mbar_wait(&bar.o_full, it & 1, &abort_flag, p.err);
      if (!ok) return;
      tc_fence_after();
      if (p.split_mode) {
        for (int hh = 0; hh < 2; ++hh) {
          for (int oc = 0; oc < 128; oc += 32) {
            uint32_t v[32];
            tmem_ld32_nowait(tmem + lane_off + hh * 128 + oc, v);
            tmem_wait_ld_regs(v);
            if (row_valid) {
              float4* dst = reinterpret_cast<float4*>(p.part_o + ((size_t)U * 128 + r) * kD + col0 + hh * 128 + oc);
#pragma unroll
              for (int i = 0; i < 8; ++i)
                dst[i] = make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                                     __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
            }
          }
          tc_fence_before();
          mbar_arrive(&bar.o_empty[hh]);
        }
        ++it;
        return;
      }
      // O half -> normalised bf16 -> staging (128 columns = four 32-column SW64 boxes) -> TMA
      // tensor stores.  Columns [0,128) go to the staging while [128,256) are read, so O returns
      // to the MMA warp after 256 columns of TMEM loads while only 128 are held in registers.
      uint32_t ob[64];
      auto read_o = [&](int c0) {  // 16 columns per load keeps ob + v within the register budget
#pragma unroll
        for (int oc = 0; oc < 128; oc += 16) {
          uint32_t v[16];
          tmem_ld16(tmem + lane_off + c0 + oc, v);
          tmem_wait_ld_regs16(v);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            ob[oc / 2 + i] = pack_bf16x2(__uint_as_float(v[2 * i]) * inv_l, __uint_as_float(v[2 * i + 1]) * inv_l);
        }
      };
      // one staging round: the kOutBufs boxes of 32 columns starting at column 32 * kOutBufs * sub
      // of the 128 held in ob
      auto stage_o = [&](int sub) {  // the stores that last read the staging must be done with it
        if (store_issuer) bulk_wait_group_read0();
        softmax_bar_sync();
#pragma unroll
        for (int q = 0; q < kOutBufs; ++q)
#pragma unroll
          for (int i = 0; i < 4; ++i) {  // 64-byte swizzle: 16-byte unit i of row r at unit i ^ ((r >> 1) & 3)
            const int w = (sub * kOutBufs + q) * 16 + 4 * i;
            *reinterpret_cast<uint4*>(sOut + q * kOutBufBytes + r * 64 + ((i ^ ((r >> 1) & 3)) * 16)) =
                make_uint4(ob[w], ob[w + 1], ob[w + 2], ob[w + 3]);
          }
        fence_proxy_async_smem();
      };
      auto store_o = [&](int c0) {
        softmax_bar_sync();
        if (store_issuer) {
#pragma unroll
          for (int q = 0; q < kOutBufs; ++q)
            tma_store_4d(&maps.o, sOut + q * kOutBufBytes, col0 + c0 + q * kOutCols, ts.hk * p.g, ts.tok0, ts.b);
          bulk_commit_group();
        }
      };
      if (kOutBufs == 4 && p.deep_ring) {
        // long rows (many key tiles per row tile): the staging region is the ring's third group,
        // so the rows go straight from registers to global memory (16-byte stores)
        uint16_t* orow = nullptr;
        {
          const int tok_r = ts.tok0 + r / p.g;
          if (row_valid)
            orow = p.O + (((size_t)ts.b * p.Lq + tok_r) * p.Hq + ts.hk * p.g + r % p.g) * kD + col0;
        }
        auto store_row = [&](int c0) {
          if (orow) {
            uint4* dst = reinterpret_cast<uint4*>(orow + c0);
#pragma unroll
            for (int i = 0; i < 16; ++i) dst[i] = make_uint4(ob[4 * i], ob[4 * i + 1], ob[4 * i + 2], ob[4 * i + 3]);
          }
        };
        read_o(0);
        store_row(0);
        read_o(128);
        tc_fence_before();
        mbar_arrive(&bar.o_empty[0]);
        mbar_arrive(&bar.o_empty[1]);
        store_row(128);
      } else if constexpr (kOutBufs == 4) {  // one round per 128 columns
        read_o(0);
        stage_o(0);
        read_o(128);
        tc_fence_before();
        mbar_arrive(&bar.o_empty[0]);
        mbar_arrive(&bar.o_empty[1]);
        store_o(0);
        stage_o(0);
        store_o(128);
      } else {  // two rounds of 64 columns per 128 (smaller staging area)
        read_o(0);
        stage_o(0);
        store_o(0);
        stage_o(1);
        store_o(64);
        read_o(128);
        tc_fence_before();
        mbar_arrive(&bar.o_empty[0]);
        mbar_arrive(&bar.o_empty[1]);
        stage_o(0);
        store_o(128);
        stage_o(1);
        store_o(192);
      }
      ++it;
    };

    for (int T = ui.first; ok && T < ui.end; T += unit_step(p), ++tl) {
      TileSet ts;
      ts.init(T, p);
      if (ts.J > p.J_max) break;
      const bool row_valid = ts.tok0 + r / p.g < p.Lq;
      ok = mbar_wait(&bar.l_ready[tl & 1], (tl >> 1) & 1, &abort_flag, p.err);
      if (!ok) break;
      const float inv_l = inv_l_sh[tl & 1][r];
      epilogue(ts, 0, inv_l, T, row_valid);
      if (!ok) break;
      epilogue(ts, kDHalf, inv_l, T, row_valid);
      if (!ok) break;
      mbar_arrive(&bar.l_empty[tl & 1]);
    }
    if (store_issuer) bulk_wait_group0();
  } else {
    // ------------------------------------------------------------ softmax and P reloads
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // row of the tile == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    uint8_t* scratch = p.scratch + (size_t)blockIdx.x * p.J_max * kScratchTileBytes;
    uint32_t g = 0, tl = 0;  // key tiles, row tiles
    // s_full[b] completes once per phase-A key tile on S buffer b (phase B issues no QK^T), so
    // its parity is tracked per buffer here rather than derived from the key-tile counter
    uint32_t s_par = 0;
    bool ok = true;

    for (int T = ui.first; ok && T < ui.end; T += unit_step(p), ++tl) {
      TileSet ts;
      ts.init(T, p);
      if (ts.J > p.J_max) break;
      const int tok = ts.tok0 + r / p.g;  // relative token index
      const int h = ts.hk * p.g + r % p.g;
      const bool row_valid = tok < p.Lq;
      const int t = p.q_offset + min(tok, p.Lq - 1);
      const int nc_t = n_compressed(t, p.W, p.blk);
      const int ws_t = window_start(t, p.W);
      float m_ref = -INFINITY, l_run = 0.0f;
      // ---- phase A
      for (int j = 0; ok && j < ts.J; ++j) {
        const uint32_t gs = g + j;
        const KeyTile kt = ts.get(j);
        // visible columns: [lo, hi) and, in a merged tile, its window columns [lo2, hi2)
        int lo, hi, lo2 = 0, hi2 = 0;
        if (kt.kind == 1) {
          lo = max(ws_t, kt.start) - kt.start;
          hi = min(t + 1, kt.start + kt.n) - kt.start;
        } else if (kt.kind == 0) {
          lo = 0;
          hi = min(nc_t, kt.start + kt.n) - kt.start;
        } else {
          lo = kMergeWinRows;
          hi = kMergeWinRows + nc_t - kt.start;  // nc_t <= nc_hi: never past the tile's entries
          lo2 = max(ws_t - kt.wstart, 0);
          hi2 = min(t + 1 - kt.wstart, kt.wn);
        }
        // Padding rows (tokens past Lq: a partial last tile, 7 of the 8 token slots of a decode
        // tile) keep the last token's intervals.  Their Q rows are TMA zero fill, so their scores
        // are 0 and their P finite, and nothing of theirs is stored; an empty interval would only
        // push their warps off the all-visible fast paths below.
        const uint32_t tS = tmem + lane_off + kDHalf + (gs & 1) * kKeyTile;
        ok = mbar_wait(&bar.s_full[gs & 1], (s_par >> (gs & 1)) & 1, &abort_flag, p.err);
        if (!ok) break;
        s_par ^= 1u << (gs & 1);
        tc_fence_after();
        // pass 1: tile max over this row's visible columns.  An interval may be empty (hi < lo:
        // a token whose window starts past a band tile, or that needs fewer entries than a tile
        // holds when blk < 128/g), so the widths are clamped at 0.
        const uint32_t vis_n = hi > lo ? (uint32_t)(hi - lo) : 0u;  // c visible iff (c - lo) < vis_n
        const uint32_t vis_n2 = hi2 > lo2 ? (uint32_t)(hi2 - lo2) : 0u;  // ... or (c - lo2) < vis_n2
        float mx = -INFINITY;
        for (int c0 = 0; c0 < kt.n; c0 += 32) {
          uint32_t v[32];
          tmem_ld32_nowait(tS + c0, v);
          tmem_wait_ld_regs(v);
          if (__all_sync(0xffffffffu, lo <= c0 && c0 + 32 <= hi)) {  // chunk visible to every row
#pragma unroll
            for (int i = 0; i < 32; ++i) mx = fmaxf(mx, __uint_as_float(v[i]));
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if ((uint32_t)(c0 + i - lo) < vis_n || (uint32_t)(c0 + i - lo2) < vis_n2)
                mx = fmaxf(mx, __uint_as_float(v[i]));
          }
        }
        const float m_tile = mx * p.scale_log2;  // -inf stays -inf
        bool need = false;
        if (m_ref == -INFINITY) {
          m_ref = m_tile;
        } else if (m_tile > m_ref + kLazyRescale) {
          need = true;
        }
        float alpha = 1.0f;
        if (__any_sync(0xffffffffu, need)) {
          // O must hold every PV of this half up to key tile j-1 (j >= 1 here) before the rescale
          const uint32_t gp = gs - 1;
          ok = mbar_wait(&bar.pv_done[gp & 1], (gp >> 1) & 1, &abort_flag, p.err);
          if (!ok) break;
          tc_fence_after();
          if (need) {
            alpha = fast_exp2(m_ref - m_tile);
            m_ref = m_tile;
          }
          l_run *= alpha;
          rescale_o(tmem + lane_off, alpha);
        }
        // rows that belong to no token (a partial last tile, decode tiles) keep nothing in the
        // scratch: their P and O rows are never stored, so phase B leaves them unloaded
        if (row_valid) *scratch_alpha(scratch, j, r) = alpha;
        // pass 2: P = exp2(s*scale*log2e - m_ref) as bf16, in place over S and into the scratch
        const uint32_t vis_p = m_ref != -INFINITY ? vis_n : 0u;
        const uint32_t vis_p2 = m_ref != -INFINITY ? vis_n2 : 0u;
        uint4* prow = scratch_p(scratch, j, r);
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          if (q4 * 32 < kt.n) {
            uint32_t v[32];
            tmem_ld32_nowait(tS + q4 * 32, v);
            tmem_wait_ld_regs(v);
            uint32_t pk[16];
            const int c0 = q4 * 32;
            if (__all_sync(0xffffffffu, vis_p != 0u && lo <= c0 && c0 + 32 <= hi)) {  // chunk visible to every row
              float ls = 0.0f;
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const float p0 = fast_exp2(fmaf(__uint_as_float(v[2 * i]), p.scale_log2, -m_ref));
                const float p1 = fast_exp2(fmaf(__uint_as_float(v[2 * i + 1]), p.scale_log2, -m_ref));
                ls += p0 + p1;
                pk[i] = pack_bf16x2(p0, p1);
              }
              l_run += ls;
            } else {
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const int c = c0 + 2 * i;
                float p0 = 0.0f, p1 = 0.0f;
                if ((uint32_t)(c - lo) < vis_p || (uint32_t)(c - lo2) < vis_p2)
                  p0 = fast_exp2(fmaf(__uint_as_float(v[2 * i]), p.scale_log2, -m_ref));
                if ((uint32_t)(c + 1 - lo) < vis_p || (uint32_t)(c + 1 - lo2) < vis_p2)
                  p1 = fast_exp2(fmaf(__uint_as_float(v[2 * i + 1]), p.scale_log2, -m_ref));
                l_run += p0 + p1;
                pk[i] = pack_bf16x2(p0, p1);
              }
            }
            tmem_st16(tS + q4 * 16, pk);
            if (row_valid) {
#pragma unroll
              for (int u = 0; u < 4; ++u)
                __stcg(prow + (q4 * 4 + u) * 128, make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]));
            }
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bar.p_ready[gs & 1]);
      }
      if (!ok) break;
      float inv_l = l_run > 0.0f ? 1.0f / l_run : 0.0f;
      if (p.split_mode) {  // the combine pass normalises
        inv_l = 1.0f;
        if (row_valid) p.part_ml[(size_t)T * 128 + r] = make_float2(m_ref, l_run);
      } else if (p.lse && row_valid) {
        p.lse[((size_t)ts.b * p.Lq + tok) * p.Hq + h] = (m_ref + __log2f(l_run)) * 0.69314718055994531f;
      }
      // hand 1/l to the epilogue warps (their buffer of two row tiles ago must be consumed)
      if (tl >= 2) {
        ok = mbar_wait(&bar.l_empty[tl & 1], ((tl >> 1) - 1) & 1, &abort_flag, p.err);
        if (!ok) break;
      }
      inv_l_sh[tl & 1][r] = inv_l;
      mbar_arrive(&bar.l_ready[tl & 1]);
      g += ts.J;
      // ---- phase B: reload P_j into the S buffers, apply the same rescales
      for (int j = 0; ok && j < ts.J; ++j) {
        const uint32_t gs = g + j;
        const KeyTile kt = ts.get(j);
        uint4 pr[16];
        float alpha;
        load_p_row(pr, alpha, scratch, j, row_valid ? kt.n : 0, r);
        if (!row_valid) alpha = 1.0f;
        if (gs >= 2) {  // S buffer gs&1 is free once PV_{gs-2} has read its P
          ok = mbar_wait(&bar.pv_done[gs & 1], ((gs >> 1) - 1) & 1, &abort_flag, p.err);
          if (!ok) break;
          tc_fence_after();
        }
        if (__any_sync(0xffffffffu, alpha != 1.0f)) {
          const uint32_t gp = gs - 1;
          ok = mbar_wait(&bar.pv_done[gp & 1], (gp >> 1) & 1, &abort_flag, p.err);
          if (!ok) break;
          tc_fence_after();
          rescale_o(tmem + lane_off, alpha);
        }
        const uint32_t tS = tmem + lane_off + kDHalf + (gs & 1) * kKeyTile;
#pragma unroll
        for (int c0 = 0; c0 < kKeyTile; c0 += 32) {
          if (c0 < kt.n) {
            uint32_t pk[16];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              pk[4 * u] = pr[c0 / 8 + u].x;
              pk[4 * u + 1] = pr[c0 / 8 + u].y;
              pk[4 * u + 2] = pr[c0 / 8 + u].z;
              pk[4 * u + 3] = pr[c0 / 8 + u].w;
            }
            tmem_st16(tS + c0 / 2, pk);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bar.p_ready[gs & 1]);
      }
      if (!ok) break;
      g += ts.J;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

// Split key ranges: row r of row tile T gathers its units' partial results,
//     M = max_s m_s,  w_s = 2^(m_s - M),  O = sum_s w_s O_s / sum_s w_s l_s,
// (m_s in log2 units, O_s and l_s relative to 2^m_s; units with l_s = 0 saw no key and drop
// out) and writes O (bf16) and lse.  One warp per row (8 rows per CTA, blockIdx.y = row
// group) and 128-column slice (blockIdx.z), 4 columns per lane.  A row tile has at most 64
// units: lane i reads the (m, l) of units i and i + 32 in one round, the warp reduces M and
// L, and the O loads of all units are independent of one another.
__global__ void __launch_bounds__(256) hca_combine_kernel(const Params p, uint16_t* __restrict__ O) {
  const int T = blockIdx.x;
  const int bh = T / p.n_tiles, tile = T % p.n_tiles;
  const int b = bh / p.Hkv, hk = bh % p.Hkv;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int r = blockIdx.y * 8 + warp;
  const int tok = tile * p.TT + r / p.g;
  if (tok >= p.Lq) return;
  const int h = hk * p.g + r % p.g;
  int U0, S;
  if (p.stream_k) {
    const int cf = sk_cta_of(T * p.J_all, p), cl = sk_cta_of((T + 1) * p.J_all - 1, p);
    U0 = cf + T;
    S = cl - cf + 1;
  } else {
    U0 = first_unit(T, p);
    S = n_splits(T, p);
  }
  float2 ml0 = make_float2(-INFINITY, 0.0f), ml1 = make_float2(-INFINITY, 0.0f);
  if (lane < S) ml0 = p.part_ml[((size_t)U0 + lane) * 128 + r];
  if (lane + 32 < S) ml1 = p.part_ml[((size_t)U0 + lane + 32) * 128 + r];
  float M = fmaxf(ml0.y > 0.0f ? ml0.x : -INFINITY, ml1.y > 0.0f ? ml1.x : -INFINITY);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  const float w0 = ml0.y > 0.0f ? exp2f(ml0.x - M) : 0.0f;
  const float w1 = ml1.y > 0.0f ? exp2f(ml1.x - M) : 0.0f;
  float L = w0 * ml0.y + w1 * ml1.y;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
  const float inv_L = L > 0.0f ? 1.0f / L : 0.0f;
  uint16_t* orow = O + (((size_t)b * p.Lq + tok) * p.Hq + h) * kD;
  const int c = blockIdx.z * 128 + lane * 4;  // this CTA's 128-column slice of the row
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
  for (int sp = 0; sp < S; ++sp) {  // every unit wrote its valid rows (zeros where it saw no key)
    const float w = __shfl_sync(0xffffffffu, sp < 32 ? w0 : w1, sp & 31);
    const float4 o = *reinterpret_cast<const float4*>(p.part_o + (((size_t)U0 + sp) * 128 + r) * kD + c);
    acc.x += w * o.x;
    acc.y += w * o.y;
    acc.z += w * o.z;
    acc.w += w * o.w;
  }
  *reinterpret_cast<uint2*>(orow + c) =
      make_uint2(pack_bf16x2(acc.x * inv_L, acc.y * inv_L), pack_bf16x2(acc.z * inv_L, acc.w * inv_L));
  if (blockIdx.z == 0 && lane == 0 && p.lse)
    p.lse[((size_t)b * p.Lq + tok) * p.Hq + h] = (M + __log2f(L)) * 0.69314718055994531f;
}

// [B, rows, heads, pitch] bf16 tensor seen as its first d columns (d <= pitch)
bool make_map_4d_pitch(CUtensorMap* m, const void* base, int d, int pitch, int heads, int rows, int B, int box_cols,
                       int box_heads, int box_rows, int swizzle) {
  const uint64_t dims[4] = {(uint64_t)d, (uint64_t)heads, (uint64_t)rows, (uint64_t)B};
  const uint64_t strides[3] = {(uint64_t)pitch * 2, (uint64_t)heads * pitch * 2, (uint64_t)rows * heads * pitch * 2};
  const uint32_t box[4] = {(uint32_t)box_cols, (uint32_t)box_heads, (uint32_t)box_rows, 1};
  return encode_tmap_bf16_swizzle(m, 4, const_cast<void*>(base), dims, strides, box, swizzle);
}
bool make_map_4d(CUtensorMap* m, const void* base, int d, int heads, int rows, int B, int box_cols, int box_heads,
                 int box_rows, int swizzle) {
  return make_map_4d_pitch(m, base, d, d, heads, rows, B, box_cols, box_heads, box_rows, swizzle);
}

int num_sms() {
  static std::mutex mu;
  static int cache[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  std::lock_guard<std::mutex> lock(mu);
  if (!cache[dev] && cudaDeviceGetAttribute(&cache[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return 0;
  return cache[dev];
}

// Launch geometry shared by the workspace query and the launch: HCADSA_ERR_UNSUPPORTED for
// shapes the kernel does not take, HCADSA_ERR_CUDA if the device cannot be queried.
struct Geometry {
  int g, TT, n_tiles, total_tiles, splits, split_extra, total_units, grid, J_max;
  int stream_k, J_all;  // stream-K split of equal row tiles (see sk_cta_start)
  size_t scratch_bytes;   // probability tiles: grid * J_max * kScratchTileBytes
  size_t part_bytes;      // split mode: unnormalised O rows and (max, sum) of every unit
  size_t workspace_bytes;
};

long long host_n_compressed(long long t, int W, int blk) { return t - W + 1 > 0 ? (t - W + 1) / blk : 0; }
long long host_window_start(long long t, int W) { return t - W + 1 > 0 ? t - W + 1 : 0; }
// key tiles of the row tile with tokens [tok0, tok_hi] (relative to q_offset); the same rule as
// TileSet::init, merged tile included
long long host_tile_J(long long q_offset, long long tok0, long long tok_hi, int W, int blk) {
  const long long t_hi = q_offset + tok_hi;
  const long long nc = host_n_compressed(t_hi, W, blk);
  const long long J_c = (nc + kKeyTile - 1) / kKeyTile;
  const long long w_span = t_hi - host_window_start(q_offset + tok0, W) + 1;
  const long long n_wt = (w_span + kKeyTile - 1) / kKeyTile;
  const long long w_part = w_span - (n_wt - 1) * kKeyTile;
  const int merged = J_c >= 1 && n_wt >= 2 && w_part <= kMergeWinRows && nc - (J_c - 1) * kKeyTile <= kMergeEntRows;
  return J_c + n_wt - merged;
}

hcadsa_status geometry(Geometry* G, int B, int Lq, int q_offset, int Hq, int Hkv, int d, int blk, int W) {
  if (B <= 0 || Lq <= 0 || q_offset < 0 || Hq <= 0 || Hkv <= 0 || blk <= 0 || W <= 0 || Hq % Hkv != 0)
    return HCADSA_ERR_SHAPE;
  const int g = Hq / Hkv;
  if (d != kD || g > 128 || 128 % g != 0) return HCADSA_ERR_UNSUPPORTED;
  const long long t_last = (long long)q_offset + Lq - 1;
  if (t_last > 2147483647LL - 256) return HCADSA_ERR_UNSUPPORTED;
  const int TT = 128 / g;
  const long long n_tiles = (Lq + TT - 1) / TT;
  const long long total = (long long)B * Hkv * n_tiles;
  if (total > 2147483647LL) return HCADSA_ERR_UNSUPPORTED;
  const long long nc_last = t_last - W + 1 > 0 ? (t_last - W + 1) / blk : 0;
  // a tile's window band spans at most TT + W - 1 positions
  const long long J_max = (nc_last + kKeyTile - 1) / kKeyTile + ((long long)TT + W - 2 + kKeyTile) / kKeyTile;
  if (J_max > (1 << 20)) return HCADSA_ERR_UNSUPPORTED;
  const int sms = num_sms();
  if (sms <= 0) return HCADSA_ERR_CUDA;
  // Few row tiles (decode: one token per sequence) leave most SMs idle: split every row tile's
  // key tiles into `splits` units (each unit keeps at least one key tile) and combine after.
  long long splits = 1, extra = 0;
  int stream_k = 0;
  long long J_all = 0;
  if (2 * total <= sms) {
    long long J_min = J_max, J_hi = 0;
    for (long long t = 0; t < n_tiles; ++t) {
      const long long tok0 = t * TT, tok_hi = (tok0 + TT < Lq ? tok0 + TT : Lq) - 1;
      const long long J = host_tile_J(q_offset, tok0, tok_hi, W, blk);
      J_min = J < J_min ? J : J_min;
      J_hi = J > J_hi ? J : J_hi;
    }
    // Equal row tiles (decode: one token per sequence, all at the same position): stream-K, every
    // CTA an equal share of all key tiles, as long as each CTA gets one and no row tile is split
    // into more than 64 units (the combine pass's limit).  Units per row tile otherwise differ by
    // one (13 against 16.25 key tiles per unit at B = 32, t = 1M).
    if (J_min == J_hi && total * J_min >= sms && total * J_min * (sms + 1) < 2147483647LL) {
      Params q{};
      q.total_tiles = (int)total;
      q.J_all = (int)J_min;
      q.sk_grid = sms;
      int S_max = 0;
      for (long long T = 0; T < total; ++T) {
        const int S = sk_cta_of((int)((T + 1) * J_min - 1), q) - sk_cta_of((int)(T * J_min), q) + 1;
        S_max = S > S_max ? S : S_max;
      }
      if (S_max <= 64) {
        stream_k = 1;
        J_all = J_min;
      }
    }
    // one unit per SM: sms / total units per row tile, one more for the first sms % total
    // (two units per SM balance the key tiles better but measured slower at B = 32, t = 1M:
    // 148 us against 136 us, the per-unit fixed costs outweigh it)
    splits = sms / total;
    extra = sms % total;
    if (splits + (extra ? 1 : 0) > J_min) {
      splits = J_min;
      extra = 0;
    }
    if (splits + (extra ? 1 : 0) > 64) {  // the combine pass takes at most 64 units per row tile
      splits = 64;
      extra = 0;
    }
  }
  G->g = g;
  G->TT = TT;
  G->n_tiles = (int)n_tiles;
  G->total_tiles = (int)total;
  G->stream_k = stream_k;
  G->J_all = (int)J_all;
  if (stream_k) {  // records c + T: at most sms + total of them
    G->splits = 1;
    G->split_extra = 0;
    G->total_units = (int)(sms + total);
    G->grid = sms;
  } else {
    G->splits = (int)splits;
    G->split_extra = (int)extra;
    G->total_units = (int)(total * splits + extra);
    G->grid = G->total_units < sms ? G->total_units : sms;
  }
  G->J_max = (int)J_max;
  G->scratch_bytes = (size_t)G->grid * (size_t)J_max * kScratchTileBytes;
  G->part_bytes = G->total_units > G->total_tiles ? (size_t)G->total_units * 128 * (kD * 4 + 8) : 0;
  G->workspace_bytes = G->scratch_bytes + G->part_bytes;
  return HCADSA_OK;
}

}  // namespace
}  // namespace hcadsa

extern "C" size_t hca_attn_fwd_workspace_size(int B, int Lq, int q_offset, int Hq, int Hkv, int d, int n_c, int blk,
                                              int W) {
  (void)n_c;
  hcadsa::Geometry G;
  if (hcadsa::geometry(&G, B, Lq, q_offset, Hq, Hkv, d, blk, W) != HCADSA_OK) return 0;
  return G.workspace_bytes;
}

namespace hcadsa {
namespace {

// Checks shared by both entry points; returns HCADSA_OK and the launch geometry when the call is
// valid.  Score width dqk, value width kD (512).
hcadsa_status check_call(const void* Q, const void* Kc, const void* Vc, int n_c, const void* Kw, const void* Vw,
                         int win_start, int n_w, const void* O, const float* lse, int B, int Lq, int q_offset,
                         int Hq, int Hkv, int blk, int W, const void* workspace, size_t workspace_bytes,
                         Geometry* G) {
  if (!Q || !Kw || !Vw || !O) return HCADSA_ERR_NULL;
  if (n_c > 0 && (!Kc || !Vc)) return HCADSA_ERR_NULL;
  if (B < 0 || Lq < 0 || q_offset < 0 || Hq <= 0 || Hkv <= 0 || n_c < 0 || n_w < 0 || win_start < 0 || blk <= 0 ||
      W <= 0)
    return HCADSA_ERR_SHAPE;
  if (Hq % Hkv != 0) return HCADSA_ERR_SHAPE;
  const int g = Hq / Hkv;
  if (g > 128 || 128 % g != 0) return HCADSA_ERR_UNSUPPORTED;
  if (!aligned16(Q) || !aligned16(Kw) || !aligned16(Vw) || !aligned16(O) ||
      (n_c > 0 && (!aligned16(Kc) || !aligned16(Vc))) || (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)))
    return HCADSA_ERR_ALIGN;
  if (B == 0 || Lq == 0) return HCADSA_OK;
  // every query's visible set must be stored
  const long long t_first = q_offset, t_last = (long long)q_offset + Lq - 1;
  if (t_last > 2147483647LL - 256) return HCADSA_ERR_UNSUPPORTED;
  const long long ws_first = t_first - W + 1 > 0 ? t_first - W + 1 : 0;
  const long long nc_last = t_last - W + 1 > 0 ? (t_last - W + 1) / blk : 0;
  if (ws_first < win_start || t_last - win_start >= n_w || nc_last > n_c) return HCADSA_ERR_SHAPE;
  const hcadsa_status gs = geometry(G, B, Lq, q_offset, Hq, Hkv, kD, blk, W);
  if (gs != HCADSA_OK) return gs;
  if (!workspace || workspace_bytes < G->workspace_bytes) return HCADSA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return HCADSA_ERR_ALIGN;
  return HCADSA_OK;
}

// Builds the tensor maps and launches.  Score width DQK; K rows are DQK wide, V rows are read as
// the first kD columns of rows `vpitch` wide (vpitch = kD: separate V; vpitch = DQK: V is the
// latent part of K).
template <int DQK>
hcadsa_status launch_hca(const hcadsa_bf16* Q, const hcadsa_bf16* Kc, const hcadsa_bf16* Vc, int n_c,
                         const hcadsa_bf16* Kw, const hcadsa_bf16* Vw, int vpitch, int win_start, int n_w,
                         hcadsa_bf16* O, float* lse, int B, int Lq, int q_offset, int Hq, int Hkv, int blk, int W,
                         float scale, void* workspace, const Geometry& G, cudaStream_t stream) {
  using S = Shape<DQK>;
  const int g = Hq / Hkv;
  Maps maps;
  if (!make_map_4d(&maps.q, Q, DQK, Hq, Lq, B, 64, g, G.TT, 128)) return HCADSA_ERR_CUDA;
  if (!make_map_4d(&maps.o, O, kD, Hq, Lq, B, kOutCols, g, G.TT, 64)) return HCADSA_ERR_CUDA;
  {
    // entries of the merged tiles exist only when n_c > 0; otherwise those maps are never read
    const hcadsa_bf16* KcM = n_c > 0 ? Kc : Kw;
    const hcadsa_bf16* VcM = n_c > 0 ? Vc : Vw;
    const int rows_c = n_c > 0 ? n_c : n_w;
    if (!make_map_4d(&maps.kmerge[0], Kw, DQK, Hkv, n_w, B, 64, 1, kMergeWinRows, 128) ||
        !make_map_4d(&maps.kmerge[1], KcM, DQK, Hkv, rows_c, B, 64, 1, kMergeEntRows, 128) ||
        !make_map_4d_pitch(&maps.vmerge[0], Vw, kD, vpitch, Hkv, n_w, B, 64, 1, kMergeWinRows, 128) ||
        !make_map_4d_pitch(&maps.vmerge[1], VcM, kD, vpitch, Hkv, rows_c, B, 64, 1, kVRows - kMergeWinRows, 128))
      return HCADSA_ERR_CUDA;
    for (int small = 0; small < 2; ++small) {
      const int krows = small ? kSmallRows : kKeyTile, vrows = small ? kSmallRows : kVRows;
      if (!make_map_4d(&maps.k[1][small], Kw, DQK, Hkv, n_w, B, 64, 1, krows, 128) ||
          !make_map_4d_pitch(&maps.v[1][small], Vw, kD, vpitch, Hkv, n_w, B, 64, 1, vrows, 128) ||
          !make_map_4d(&maps.k[0][small], KcM, DQK, Hkv, rows_c, B, 64, 1, krows, 128) ||
          !make_map_4d_pitch(&maps.v[0][small], VcM, kD, vpitch, Hkv, rows_c, B, 64, 1, vrows, 128))
        return HCADSA_ERR_CUDA;
    }
  }
  Params p;
  p.Lq = Lq;
  p.q_offset = q_offset;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.g = g;
  p.TT = G.TT;
  p.n_c = n_c;
  p.win_start = win_start;
  p.W = W;
  p.blk = blk;
  p.n_tiles = G.n_tiles;
  p.total_tiles = G.total_tiles;
  p.splits = G.splits;
  p.split_extra = G.split_extra;
  p.split_mode = G.total_units > G.total_tiles ? 1 : 0;
  p.total_units = G.total_units;
  p.stream_k = G.stream_k;
  p.J_all = G.J_all;
  p.sk_grid = G.grid;
  p.J_max = G.J_max;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.lse = lse;
  p.scratch = static_cast<uint8_t*>(workspace);
  p.part_o = p.split_mode ? reinterpret_cast<float*>(p.scratch + G.scratch_bytes) : nullptr;
  p.part_ml = p.split_mode ? reinterpret_cast<float2*>(p.scratch + G.scratch_bytes + (size_t)G.total_units * 128 * kD * 4)
                           : nullptr;
  p.O = reinterpret_cast<uint16_t*>(O);
  // a third ring group pays off once row tiles have many key tiles (long contexts); with few
  // (L = 32768: 3-4) the TMA-stored epilogue is the better use of the region
  p.deep_ring = (DQK == 512 && !p.split_mode && G.J_max >= 6) ? 1 : 0;
  p.err = device_error_ptr();
  if (cudaFuncSetAttribute(hca_attn_kernel<DQK>, cudaFuncAttributeMaxDynamicSharedMemorySize, S::kSmemBytes) !=
      cudaSuccess)
    return HCADSA_ERR_CUDA;
  hca_attn_kernel<DQK><<<G.grid, kThreads, S::kSmemBytes, stream>>>(maps, p);
  if (p.split_mode) {
    const hcadsa_status st = launch_status();
    if (st != HCADSA_OK) return st;
    // only row groups holding a valid token: 8 rows per CTA
    const int valid_rows = Lq < G.TT ? Lq * g : 128;
    hca_combine_kernel<<<dim3((unsigned)G.total_tiles, (unsigned)((valid_rows + 7) / 8), kD / 128), 256, 0, stream>>>(
        p, reinterpret_cast<uint16_t*>(O));
  }
  return launch_status();
}

}  // namespace
}  // namespace hcadsa

extern "C" hcadsa_status hca_attn_fwd(const hcadsa_bf16* Q, const hcadsa_bf16* Kc, const hcadsa_bf16* Vc, int n_c,
                                      const hcadsa_bf16* Kw, const hcadsa_bf16* Vw, int win_start, int n_w,
                                      hcadsa_bf16* O, float* lse, int B, int Lq, int q_offset, int Hq, int Hkv,
                                      int d, int blk, int W, float scale, void* workspace, size_t workspace_bytes,
                                      hcadsa_stream stream) {
  using namespace hcadsa;
  Geometry G;
  if (d != kD && Q && Kw && Vw && O && (n_c == 0 || (Kc && Vc)) && B >= 0 && Lq >= 0 && Hq > 0 && Hkv > 0 &&
      Hq % Hkv == 0)
    return HCADSA_ERR_UNSUPPORTED;
  const hcadsa_status st = check_call(Q, Kc, Vc, n_c, Kw, Vw, win_start, n_w, O, lse, B, Lq, q_offset, Hq, Hkv, blk,
                                      W, workspace, workspace_bytes, &G);
  if (st != HCADSA_OK || B == 0 || Lq == 0) return st;
  return launch_hca<512>(Q, Kc, Vc, n_c, Kw, Vw, kD, win_start, n_w, O, lse, B, Lq, q_offset, Hq, Hkv, blk, W, scale,
                         workspace, G, as_stream(stream));
}

extern "C" size_t hca_attn_fwd_latent_workspace_size(int B, int Lq, int q_offset, int Hq, int Hkv, int dqk, int dv,
                                                     int n_c, int blk, int W) {
  if (dqk != 576 || dv != 512) return 0;
  return hca_attn_fwd_workspace_size(B, Lq, q_offset, Hq, Hkv, dv, n_c, blk, W);
}

extern "C" hcadsa_status hca_attn_fwd_latent(const hcadsa_bf16* Q, const hcadsa_bf16* Kc, int n_c,
                                             const hcadsa_bf16* Kw, int win_start, int n_w, hcadsa_bf16* O,
                                             float* lse, int B, int Lq, int q_offset, int Hq, int Hkv, int dqk, int dv,
                                             int blk, int W, float scale, void* workspace, size_t workspace_bytes,
                                             hcadsa_stream stream) {
  using namespace hcadsa;
  Geometry G;
  if ((dqk != 576 || dv != 512) && Q && Kw && O && (n_c == 0 || Kc) && B >= 0 && Lq >= 0 && Hq > 0 && Hkv > 0 &&
      Hq % Hkv == 0)
    return HCADSA_ERR_UNSUPPORTED;  // before anything that needs the device, like hca_attn_fwd
  const hcadsa_status st = check_call(Q, Kc, Kc, n_c, Kw, Kw, win_start, n_w, O, lse, B, Lq, q_offset, Hq, Hkv, blk,
                                      W, workspace, workspace_bytes, &G);
  if (st == HCADSA_OK && (dqk != 576 || dv != 512)) return HCADSA_ERR_UNSUPPORTED;
  if (st != HCADSA_OK || B == 0 || Lq == 0) return st;
  return launch_hca<576>(Q, Kc, Kc, n_c, Kw, Kw, 576, win_start, n_w, O, lse, B, Lq, q_offset, Hq, Hkv, blk, W,
                         scale, workspace, G, as_stream(stream));
}
