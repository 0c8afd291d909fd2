// hca_attn_bwd.cu -- HCA attention backward on sm_100a (tcgen05 + TMEM + TMA).
//
// Method: the backward of the HCA attention of the mirrorspeed page, section "Hybrid sparse
// attention, 1/7 full context access" (a query attends to the compressed entries and to a short
// window of the latest raw tokens; 512-wide heads).  For a loss with output gradient dO, per query
// row (token t, head h) and visible key s (entries and window positions, one softmax over both):
//     p[s]   = exp(scale <q, k_s> - lse)           (lse from the forward)
//     D      = <dO, O>
//     dS[s]  = p[s] (<dO, v_s> - D)
//     dQ     = scale sum_s dS[s] k_s,   dK[s] += scale dS[s] q,   dV[s] += p[s] dO
//
// Kernel design.  With d = 512 neither a 128-row Q tile and its dO (256 KB) fit in shared memory
// together, nor the dK and dV accumulators of a 128-key tile (1024 fp32 columns) in TMEM, so the
// backward is four launches over (row tile, key tile) blocks:
//   1. prep: D per query row (a warp per row; HBM stream of O and dO).
//   2. scores: one CTA per row tile (128 rows = 128/g tokens x the g query heads of one K/V
//      head, as in the forward); for each of its key tiles S = Q K^T and dP = dO V^T are
//      accumulated over eight 64-column chunks of d (SS MMAs, N = 128, K-major operands streamed
//      through a three-stage TMA ring), two TMEM buffers of (S, dP) so that the epilogue of one
//      block overlaps the MMAs of the next.  The epilogue warps (thread = row = TMEM lane) form
//      P and dS with the visibility mask of the block and write both as bf16 128 x 128 blocks to
//      a workspace.
//   3./4. blocked GEMMs D[128 x 512] = sum over blocks of A_b[128 x 128] B_b[128 x 512], the
//      whole 512-column fp32 accumulator in TMEM, operands through a two-stage TMA ring
//      (N = 256 MMAs, B MN-major):
//        dQ of a row tile:   A = dS blocks (K-major), B = the key tiles' K rows;
//        dK / dV of a key tile: A = dS^T / P^T blocks (MN-major), B = the row tiles' Q / dO,
//      the key-tile units split into chunks of row tiles.  Epilogue: rows staged in shared
//      memory and written with bulk copies (dQ) or bulk fp32 reductions (dK, dV, which several
//      chunks add to).
// Key tiles are aligned 128-wide tiles of the entry index (entries) and of the raw position
// (window), so a key tile is the same for every row tile that sees it; a row tile has
// ceil(n_c(t_last)/128) entry tiles and the window tiles that its band
// [max(0, t_first - W + 1), t_last] touches.  Every wait is bounded (the library's 2 s limit);
// on expiry the error word records a timeout and every role leaves its loop.
#include <cuda_bf16.h>

#include "host_common.h"
#include "ptx.cuh"

namespace hcadsa {
namespace {

constexpr int kD = 512;
constexpr int kTile = 128;
constexpr int kChunk = 64;                  // d columns per scores stage
constexpr int kChunkBytes = kTile * 128;    // 128 rows x 64 bf16
constexpr int kThreads = 192;               // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue
constexpr int kScoreStages = 3;
constexpr int kScoreStageBytes = 4 * kChunkBytes;  // Q, dO, K, V chunks
constexpr int kGemmStages = 2;
constexpr int kGemmABytes = kTile * 64 * 2;        // 16 KB
constexpr int kGemmBHalfBytes = 64 * (kD / 2) * 2;  // 32 KB: 64 K-rows x 256 columns
constexpr int kGemmStageBytes = kGemmABytes + 2 * kGemmBHalfBytes;  // whole 512 columns
constexpr int kStageCols = 128;                    // epilogue: fp32 columns per bulk operation
constexpr int kStageRow = kStageCols * 4 + 16;     // staging row: 128 fp32 + pad (conflict free)
constexpr int kChunkRows = 16;                     // row tiles per dK / dV unit
constexpr uint32_t kBlockElems = kTile * kTile;

static_assert(kTile * kStageRow <= kGemmStages * (kGemmABytes + kGemmBHalfBytes), "staging fits in the ring");

// Geometry of one call (same for every (b, kv)).
struct Geo {
  int B, Lq, q_offset, Hq, Hkv, g, tpt, n_rt, n_c, win_start, n_w, blk, W;
  int E_max, Wt_max, J;     // entry tiles, window tiles per row tile (bounds), slots per row tile
  int m_first, n_wt;        // window tiles of the whole call
  int n_ch_e, n_ch_w;       // row-tile chunks per entry / window key tile (dK, dV units)
  float scale, scale_log2;
};

__host__ __device__ inline int win_start_of(int t, int W) { return t - W + 1 > 0 ? t - W + 1 : 0; }
__host__ __device__ inline int n_c_of(int t, int W, int blk) {
  const int a = t - W + 1;
  return a > 0 ? a / blk : 0;
}

struct RowTile {
  int t_first, t_last;  // token range (t_last inclusive, clipped to the call)
  int E;                // entry tiles
  int mlo, mhi;         // window tiles [mlo, mhi]
  __device__ void init(const Geo& G, int i) {
    t_first = G.q_offset + i * G.tpt;
    t_last = min(t_first + G.tpt, G.q_offset + G.Lq) - 1;
    E = (n_c_of(t_last, G.W, G.blk) + kTile - 1) / kTile;
    mlo = win_start_of(t_first, G.W) / kTile;
    mhi = t_last / kTile;
  }
  __device__ int count() const { return E + (mhi - mlo + 1); }
};

__device__ __forceinline__ size_t block_index(const Geo& G, int bkv, int i, int slot) {
  return ((size_t)bkv * G.n_rt + i) * G.J + slot;
}

__device__ __forceinline__ void bulk_store(float* dst, uint32_t src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(src), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_reduce_add_f32(float* dst, uint32_t src, uint32_t bytes) {
  asm volatile("cp.reduce.async.bulk.global.shared::cta.bulk_group.add.f32 [%0], [%1], %2;" ::"l"(dst), "r"(src),
               "r"(bytes)
               : "memory");
}

// ------------------------------------------------------------------------------------ 1. prep

__global__ void __launch_bounds__(256) hca_bwd_prep_kernel(const uint16_t* __restrict__ O,
                                                           const uint16_t* __restrict__ dO,
                                                           float* __restrict__ Dout, long long rows) {
  const long long r = (long long)blockIdx.x * 8 + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  if (r >= rows) return;
  const uint4* o4 = reinterpret_cast<const uint4*>(O + r * kD);
  const uint4* g4 = reinterpret_cast<const uint4*>(dO + r * kD);
  float acc = 0.0f;
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const uint4 a = o4[lane + 32 * i], b = g4[lane + 32 * i];
    const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      acc = fmaf(__uint_as_float(aw[q] << 16), __uint_as_float(bw[q] << 16), acc);
      acc = fmaf(__uint_as_float(aw[q] & 0xFFFF0000u), __uint_as_float(bw[q] & 0xFFFF0000u), acc);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) Dout[r] = acc;
}

// ---------------------------------------------------------------------------------- 2. scores

struct ScoreMaps {
  CUtensorMap q, dO, kc, vc, kw, vw;  // Q / dO box {64, g, tpt, 1}; K/V box {64, 1, 128, 1}
};

struct ScoreParams {
  Geo G;
  const float* lse;  // [B, Lq, Hq]
  const float* Dv;   // [B, Lq, Hq]
  uint16_t* P;       // blocks of 128 x 128 bf16
  uint16_t* dS;
  int* err;
};

struct __align__(8) ScoreBars {
  uint64_t full[kScoreStages], empty[kScoreStages];
  uint64_t tfull[2], tempty[2];
  uint32_t tmem_base;
  int abort_flag;
};

__global__ void __launch_bounds__(kThreads, 1)
    hca_bwd_scores_kernel(const __grid_constant__ ScoreMaps maps, const __grid_constant__ ScoreParams p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) raise_device_error(p.err, kErrDeviceBounds);
    return;
  }
  ScoreBars& bar = *reinterpret_cast<ScoreBars*>(smem + kScoreStages * kScoreStageBytes);
  const Geo& G = p.G;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int i = blockIdx.x % G.n_rt;
  const int bkv = blockIdx.x / G.n_rt;
  const int b = bkv / G.Hkv, kv = bkv % G.Hkv;
  RowTile rt;
  rt.init(G, i);
  const int nblk = rt.count();
  if (threadIdx.x == 0) {
    for (int s = 0; s < kScoreStages; ++s) {
      mbar_init(&bar.full[s], 1);
      mbar_init(&bar.empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar.tfull[s], 1);
      mbar_init(&bar.tempty[s], 128);
    }
    bar.abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&bar.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar.tmem_base;

  if (warp == 0) {
    if (lane == 0) {
      uint32_t cnt = 0;
      bool ok = true;
      for (int jb = 0; jb < nblk && ok; ++jb) {
        const bool entry = jb < rt.E;
        const int key0 = entry ? jb * kTile : (rt.mlo + jb - rt.E) * kTile - G.win_start;
        const CUtensorMap* mk = entry ? &maps.kc : &maps.kw;
        const CUtensorMap* mv = entry ? &maps.vc : &maps.vw;
        for (int c = 0; c < kD / kChunk && ok; ++c, ++cnt) {
          const int s = cnt % kScoreStages;
          ok = mbar_wait(&bar.empty[s], ((cnt / kScoreStages) & 1) ^ 1, &bar.abort_flag, p.err);
          if (!ok) break;
          uint8_t* st = smem + s * kScoreStageBytes;
          mbar_arrive_expect_tx(&bar.full[s], kScoreStageBytes);
          tma_load_4d(st, &maps.q, &bar.full[s], c * kChunk, kv * G.g, rt.t_first - G.q_offset, b);
          tma_load_4d(st + kChunkBytes, &maps.dO, &bar.full[s], c * kChunk, kv * G.g, rt.t_first - G.q_offset, b);
          tma_load_4d(st + 2 * kChunkBytes, mk, &bar.full[s], c * kChunk, kv, key0, b);
          tma_load_4d(st + 3 * kChunkBytes, mv, &bar.full[s], c * kChunk, kv, key0, b);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kTile, kTile, false, false);
      uint32_t cnt = 0;
      bool ok = true;
      for (int jb = 0; jb < nblk && ok; ++jb) {
        const int ab = jb & 1;
        if (jb >= 2) {
          ok = mbar_wait(&bar.tempty[ab], ((jb >> 1) - 1) & 1, &bar.abort_flag, p.err);
          if (!ok) break;
          tc_fence_after();
        }
        const uint32_t tS = tmem + ab * 256, tP = tS + kTile;
        for (int c = 0; c < kD / kChunk && ok; ++c, ++cnt) {
          const int s = cnt % kScoreStages;
          ok = mbar_wait(&bar.full[s], (cnt / kScoreStages) & 1, &bar.abort_flag, p.err);
          if (!ok) break;
          tc_fence_after();
          const uint32_t st = smem_u32(smem + s * kScoreStageBytes);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint32_t acc = (c | kk) != 0;
            mma_ss(tS, smem_desc_sw128(st + kk * 32, 16, 1024), smem_desc_sw128(st + 2 * kChunkBytes + kk * 32, 16, 1024),
                   idesc, acc);
            mma_ss(tP, smem_desc_sw128(st + kChunkBytes + kk * 32, 16, 1024),
                   smem_desc_sw128(st + 3 * kChunkBytes + kk * 32, 16, 1024), idesc, acc);
          }
          mma_commit(&bar.empty[s]);
        }
        if (ok) mma_commit(&bar.tfull[ab]);
      }
    }
  } else {
    // epilogue: thread = row of the tile = TMEM lane
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const int t = rt.t_first + r / G.g;
    const int h = kv * G.g + r % G.g;
    const bool row_ok = t <= rt.t_last;
    float lse2 = 0.0f, Dr = 0.0f;
    if (row_ok) {
      const size_t qi = ((size_t)b * G.Lq + (t - G.q_offset)) * G.Hq + h;
      lse2 = p.lse[qi] * 1.4426950408889634f;
      Dr = p.Dv[qi];
    }
    const int nc_t = n_c_of(t, G.W, G.blk), ws_t = win_start_of(t, G.W);
    bool ok = true;
    for (int jb = 0; jb < nblk; ++jb) {
      const int ab = jb & 1;
      ok = mbar_wait(&bar.tfull[ab], (jb >> 1) & 1, &bar.abort_flag, p.err) && ok;
      tc_fence_after();
      const bool entry = jb < rt.E;
      // visible key columns [lo, hi) of this block for this row
      int lo, hi;
      if (entry) {
        lo = 0;
        hi = min(kTile, nc_t - jb * kTile);
      } else {
        const int m0 = (rt.mlo + jb - rt.E) * kTile;
        lo = max(0, ws_t - m0);
        hi = min(kTile, t - m0 + 1);
      }
      if (!row_ok) hi = lo;  // rows past the end of the call: P = dS = 0
      const size_t blk_i = block_index(G, bkv, i, entry ? jb : G.E_max + (jb - rt.E));
      uint4* prow = reinterpret_cast<uint4*>(p.P + blk_i * kBlockElems + (size_t)r * kTile);
      uint4* drow = reinterpret_cast<uint4*>(p.dS + blk_i * kBlockElems + (size_t)r * kTile);
      const uint32_t tS = tmem + lane_off + ab * 256, tP = tS + kTile;
#pragma unroll 1
      for (int c0 = 0; c0 < kTile; c0 += 32) {
        uint32_t sv[32], dv[32];
        tmem_ld32_nowait(tS + c0, sv);
        tmem_ld32_nowait(tP + c0, dv);
        tmem_wait_ld_regs2(sv, dv);
        uint32_t pw[16], qw[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int k0 = c0 + 2 * e;
          float p0 = 0.0f, p1 = 0.0f;
          if (k0 >= lo && k0 < hi) p0 = fast_exp2(fmaf(__uint_as_float(sv[2 * e]), G.scale_log2, -lse2));
          if (k0 + 1 >= lo && k0 + 1 < hi) p1 = fast_exp2(fmaf(__uint_as_float(sv[2 * e + 1]), G.scale_log2, -lse2));
          pw[e] = pack_bf16x2(p0, p1);
          qw[e] = pack_bf16x2(p0 * (__uint_as_float(dv[2 * e]) - Dr), p1 * (__uint_as_float(dv[2 * e + 1]) - Dr));
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          prow[c0 / 8 + q] = make_uint4(pw[4 * q], pw[4 * q + 1], pw[4 * q + 2], pw[4 * q + 3]);
          drow[c0 / 8 + q] = make_uint4(qw[4 * q], qw[4 * q + 1], qw[4 * q + 2], qw[4 * q + 3]);
        }
      }
      tc_fence_before();
      mbar_arrive(&bar.tempty[ab]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------------------- 3./4. blocked GEMM

struct GemmMaps {
  CUtensorMap dsK;   // dS blocks as [rows x 128 keys], box {64 keys, 128 rows}   (dQ: K-major A)
  CUtensorMap dsM;   // dS blocks, box {64 keys, 64 rows}                        (dK: MN-major A)
  CUtensorMap pM;    // P blocks, box {64 keys, 64 rows}                         (dV: MN-major A)
  CUtensorMap kc, kw;  // K rows, box {64, 1, 64, 1}                             (dQ: B)
  CUtensorMap q, dO;   // Q / dO rows, box {64, bh, bt, 1}                        (dK / dV: B)
};

struct GemmParams {
  Geo G;
  int mode;  // 0: dQ units (one per row tile and 256-column half); 1: dK / dV units (key tile x
             // row-tile chunk, all 512 columns)
  int bh, bt;
  float* dQ;   // [B, Lq, Hq, 512] fp32 (written)
  float* dKc;  // [B, n_c, Hkv, 512] fp32 (added to)
  float* dVc;
  float* dKw;  // [B, n_w, Hkv, 512] fp32 (added to)
  float* dVw;
  int* err;
};

struct __align__(8) GemmBars {
  uint64_t full[kGemmStages], empty[kGemmStages];
  uint64_t tfull;
  uint32_t tmem_base;
  int abort_flag;
};

// One unit's sequence of blocks.  dQ: the key tiles of row tile i.  dK / dV: the row tiles of a
// chunk that see key tile kt (entries: kt < E_i; window: mlo <= m <= mhi).
struct Unit {
  int bkv, b, kv;
  int grad;     // dK / dV units: 0 = dK, 1 = dV; dQ units: the 256-column half
  bool entry;   // dK / dV units: entry key tile (else a window key tile)
  int tile;     // dQ: row tile; dK / dV: entry tile e or window tile m
  int i0, i1;   // dK / dV: row-tile range of the chunk
  __device__ bool decode(const Geo& G, int mode, int u) {
    grad = 0;
    entry = false;
    i0 = i1 = 0;
    if (mode == 0) {
      grad = u & 1;
      u >>= 1;
      tile = u % G.n_rt;
      bkv = u / G.n_rt;
    } else {
      grad = u & 1;
      u >>= 1;
      const int per = G.E_max * G.n_ch_e + G.n_wt * G.n_ch_w;
      bkv = u / per;
      int v = u % per;
      if (v < G.E_max * G.n_ch_e) {
        entry = true;
        tile = v / G.n_ch_e;
        const int ch = v % G.n_ch_e;
        i0 = ch * kChunkRows;
        i1 = min(G.n_rt, i0 + kChunkRows);
      } else {
        v -= G.E_max * G.n_ch_e;
        entry = false;
        tile = G.m_first + v / G.n_ch_w;
        const int ch = v % G.n_ch_w;
        // row tiles whose band can touch window tile m: tokens [128 m, 128 m + 126 + W]
        const int tlo = max(tile * kTile, G.q_offset);
        const int thi = min(tile * kTile + kTile - 2 + G.W, G.q_offset + G.Lq - 1);
        if (thi < tlo) {
          i0 = i1 = 0;
        } else {
          const int ilo = (tlo - G.q_offset) / G.tpt, ihi = (thi - G.q_offset) / G.tpt + 1;
          i0 = min(ihi, ilo + ch * kChunkRows);
          i1 = min(ihi, i0 + kChunkRows);
        }
      }
    }
    b = bkv / G.Hkv;
    kv = bkv % G.Hkv;
    return bkv < G.B * G.Hkv;
  }
  // dK / dV: does row tile i take part, and with which slot
  __device__ bool member(const Geo& G, int i, int* slot) const {
    RowTile rt;
    rt.init(G, i);
    if (entry) {
      *slot = tile;
      return tile < rt.E;
    }
    *slot = G.E_max + (tile - rt.mlo);
    return tile >= rt.mlo && tile <= rt.mhi;
  }
};

__global__ void __launch_bounds__(kThreads, 1)
    hca_bwd_gemm_kernel(const __grid_constant__ GemmMaps maps, const __grid_constant__ GemmParams p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) raise_device_error(p.err, kErrDeviceBounds);
    return;
  }
  // dQ: one 256-column half per CTA (two CTAs per SM); dK / dV: both halves
  const int nh = p.mode == 0 ? 1 : 2;
  const int stage_bytes = kGemmABytes + nh * kGemmBHalfBytes;
  GemmBars& bar = *reinterpret_cast<GemmBars*>(smem + kGemmStages * stage_bytes);
  const Geo& G = p.G;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  Unit U;
  if (!U.decode(G, p.mode, blockIdx.x)) return;
  // number of blocks of this unit (uniform across the CTA)
  RowTile rtq;
  int nblk = 0;
  if (p.mode == 0) {
    rtq.init(G, U.tile);
    nblk = rtq.count();
  } else {
    for (int i = U.i0; i < U.i1; ++i) {
      int slot;
      nblk += U.member(G, i, &slot) ? 1 : 0;
    }
  }
  if (nblk == 0) return;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kGemmStages; ++s) {
      mbar_init(&bar.full[s], 1);
      mbar_init(&bar.empty[s], 1);
    }
    mbar_init(&bar.tfull, 1);
    bar.abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&bar.tmem_base, nh * 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar.tmem_base;
  const int c_first = p.mode == 0 ? U.grad * 4 : 0;  // first 64-column box of B

  if (warp == 0) {
    if (lane == 0) {
      uint32_t cnt = 0;
      bool ok = true;
      int i = U.i0;
      for (int jb = 0; jb < nblk && ok; ++jb) {
        size_t blk_i;
        int key0 = 0, t_first = 0;
        const CUtensorMap* mb;
        if (p.mode == 0) {
          const bool entry = jb < rtq.E;
          blk_i = block_index(G, U.bkv, U.tile, entry ? jb : G.E_max + (jb - rtq.E));
          key0 = entry ? jb * kTile : (rtq.mlo + jb - rtq.E) * kTile - G.win_start;
          mb = entry ? &maps.kc : &maps.kw;
        } else {
          int slot;
          while (!U.member(G, i, &slot)) ++i;
          blk_i = block_index(G, U.bkv, i, slot);
          t_first = G.q_offset + i * G.tpt;
          mb = U.grad == 0 ? &maps.q : &maps.dO;
          ++i;
        }
        const int row0 = (int)(blk_i * kTile);
        for (int hf = 0; hf < 2 && ok; ++hf, ++cnt) {
          const int s = cnt % kGemmStages;
          ok = mbar_wait(&bar.empty[s], ((cnt / kGemmStages) & 1) ^ 1, &bar.abort_flag, p.err);
          if (!ok) break;
          uint8_t* sa = smem + s * stage_bytes;
          uint8_t* sb = sa + kGemmABytes;
          mbar_arrive_expect_tx(&bar.full[s], stage_bytes);
          if (p.mode == 0) {
            tma_load_2d(sa, &maps.dsK, &bar.full[s], hf * 64, row0);
            for (int c = 0; c < 4; ++c)
              tma_load_4d(sb + c * 8192, mb, &bar.full[s], (c_first + c) * 64, U.kv, key0 + hf * 64, U.b);
          } else {
            const CUtensorMap* ma = U.grad == 0 ? &maps.dsM : &maps.pM;
            tma_load_2d(sa, ma, &bar.full[s], 0, row0 + hf * 64);
            tma_load_2d(sa + 8192, ma, &bar.full[s], 64, row0 + hf * 64);
            const int r0 = hf * 64;  // rows [r0, r0 + 64) of the row tile
            const int tok = t_first - G.q_offset + r0 / G.g;
            const int head = U.kv * G.g + (G.g > 64 ? r0 % G.g : 0);
            for (int c = 0; c < kD / 64; ++c) tma_load_4d(sb + c * 8192, mb, &bar.full[s], c * 64, head, tok, U.b);
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kTile, kD / 2, p.mode != 0, true);
      uint32_t cnt = 0;
      bool ok = true;
      for (int jb = 0; jb < nblk && ok; ++jb) {
        for (int hf = 0; hf < 2 && ok; ++hf, ++cnt) {
          const int s = cnt % kGemmStages;
          ok = mbar_wait(&bar.full[s], (cnt / kGemmStages) & 1, &bar.abort_flag, p.err);
          if (!ok) break;
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + s * stage_bytes), sb = sa + kGemmABytes;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t da = p.mode == 0 ? smem_desc_sw128(sa + kk * 32, 16, 1024)
                                            : smem_desc_sw128(sa + kk * 2048, 8192, 1024);
            for (int n = 0; n < nh; ++n)
              mma_ss(tmem + n * 256, da, smem_desc_sw128(sb + n * 4 * 8192 + kk * 2048, 8192, 1024), idesc,
                     (jb | hf | kk) != 0 ? 1u : 0u);
          }
          mma_commit(&bar.empty[s]);
        }
      }
      if (ok) mma_commit(&bar.tfull);
    }
  } else {
    // epilogue: thread = output row (TMEM lane); 128 columns at a time staged and handed to the
    // bulk-copy unit as one 512-byte row
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    bool ok = mbar_wait(&bar.tfull, 0, &bar.abort_flag, p.err);
    tc_fence_after();
    float* dst = nullptr;
    float f = 1.0f;
    if (p.mode == 0) {
      const int t = rtq.t_first + r / G.g;
      if (t <= rtq.t_last)
        dst = p.dQ + (((size_t)U.b * G.Lq + (t - G.q_offset)) * G.Hq + U.kv * G.g + r % G.g) * kD;
      f = G.scale;
    } else if (U.entry) {
      const int j = U.tile * kTile + r;
      if (j < G.n_c) dst = (U.grad == 0 ? p.dKc : p.dVc) + (((size_t)U.b * G.n_c + j) * G.Hkv + U.kv) * kD;
      f = U.grad == 0 ? G.scale : 1.0f;
    } else {
      const int row = U.tile * kTile + r - G.win_start;
      if (row >= 0 && row < G.n_w)
        dst = (U.grad == 0 ? p.dKw : p.dVw) + (((size_t)U.b * G.n_w + row) * G.Hkv + U.kv) * kD;
      f = U.grad == 0 ? G.scale : 1.0f;
    }
    uint8_t* srow = smem + r * kStageRow;
    const int col0 = p.mode == 0 ? U.grad * 256 : 0;  // output column of TMEM column 0
    if (ok) {
#pragma unroll 1
      for (int n = 0; n < nh * 256; n += kStageCols) {
        if (n > 0) bulk_wait_group_read0();
#pragma unroll 1
        for (int c0 = 0; c0 < kStageCols; c0 += 32) {
          uint32_t v[32];
          tmem_ld32_nowait(tmem + lane_off + n + c0, v);
          tmem_wait_ld_regs(v);
#pragma unroll
          for (int q = 0; q < 8; ++q)
            *reinterpret_cast<float4*>(srow + c0 * 4 + q * 16) =
                make_float4(f * __uint_as_float(v[4 * q]), f * __uint_as_float(v[4 * q + 1]),
                            f * __uint_as_float(v[4 * q + 2]), f * __uint_as_float(v[4 * q + 3]));
        }
        if (dst) {
          fence_proxy_async_smem();
          if (p.mode == 0)
            bulk_store(dst + col0 + n, smem_u32(srow), kStageCols * 4);
          else
            bulk_reduce_add_f32(dst + col0 + n, smem_u32(srow), kStageCols * 4);
          bulk_commit_group();
        }
      }
      bulk_wait_group0();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, nh * 256);
}

// ------------------------------------------------------------------------------------ host side

bool make_geo(Geo& G, int B, int Lq, int q_offset, int Hq, int Hkv, int n_c, int win_start, int n_w, int blk, int W,
              float scale) {
  if (Hkv <= 0 || Hq % Hkv) return false;
  G.B = B;
  G.Lq = Lq;
  G.q_offset = q_offset;
  G.Hq = Hq;
  G.Hkv = Hkv;
  G.g = Hq / Hkv;
  if (G.g > kTile || kTile % G.g) return false;
  G.tpt = kTile / G.g;
  G.n_rt = (Lq + G.tpt - 1) / G.tpt;
  G.n_c = n_c;
  G.win_start = win_start;
  G.n_w = n_w;
  G.blk = blk;
  G.W = W;
  const int t_end = q_offset + Lq - 1;
  G.E_max = (n_c_of(t_end, W, blk) + kTile - 1) / kTile;
  G.Wt_max = (G.tpt + W - 1 + kTile - 1) / kTile + 1;
  G.J = G.E_max + G.Wt_max;
  G.m_first = win_start_of(q_offset, W) / kTile;
  G.n_wt = t_end / kTile - G.m_first + 1;
  G.n_ch_e = (G.n_rt + kChunkRows - 1) / kChunkRows;
  const int rw = (kTile - 1 + W) / G.tpt + 2;  // row tiles whose band can touch one window tile
  G.n_ch_w = (rw + kChunkRows - 1) / kChunkRows;
  G.scale = scale;
  G.scale_log2 = scale * 1.4426950408889634f;
  return true;
}

size_t scratch_blocks(const Geo& G) { return (size_t)G.B * G.Hkv * G.n_rt * G.J; }

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace
}  // namespace hcadsa

extern "C" size_t hca_attn_bwd_workspace_size(int B, int Lq, int q_offset, int Hq, int Hkv, int d, int n_c, int blk,
                                             int W) {
  using namespace hcadsa;
  if (B <= 0 || Lq <= 0 || q_offset < 0 || d != kD || blk <= 0 || W <= 0 || n_c < 0) return 0;
  Geo G;
  if (!make_geo(G, B, Lq, q_offset, Hq, Hkv, n_c, 0, 1, blk, W, 1.0f)) return 0;
  return align256((size_t)B * Lq * Hq * 4) + 2 * scratch_blocks(G) * kBlockElems * 2;
}

extern "C" hcadsa_status hca_attn_bwd(const hcadsa_bf16* Q, const hcadsa_bf16* Kc, const hcadsa_bf16* Vc, int n_c,
                                      const hcadsa_bf16* Kw, const hcadsa_bf16* Vw, int win_start, int n_w,
                                      const hcadsa_bf16* O, const hcadsa_bf16* dO, const float* lse, float* dQ,
                                      float* dKc, float* dVc, float* dKw, float* dVw, int B, int Lq, int q_offset,
                                      int Hq, int Hkv, int d, int blk, int W, float scale, void* workspace,
                                      size_t workspace_bytes, hcadsa_stream stream) {
  using namespace hcadsa;
  if (!Q || !Kw || !Vw || !O || !dO || !lse || !dQ || !dKw || !dVw) return HCADSA_ERR_NULL;
  if (n_c > 0 && (!Kc || !Vc || !dKc || !dVc)) return HCADSA_ERR_NULL;
  if (B < 0 || Lq < 0 || q_offset < 0 || n_c < 0 || n_w < 0 || win_start < 0 || Hq <= 0 || Hkv <= 0 || blk <= 0 ||
      W <= 0)
    return HCADSA_ERR_SHAPE;
  if (Hq % Hkv) return HCADSA_ERR_SHAPE;
  if (d != kD || kTile % (Hq / Hkv)) return HCADSA_ERR_UNSUPPORTED;
  if (B == 0 || Lq == 0) return HCADSA_OK;
  // every query's window inside the raw buffer, every visible entry inside Kc
  const int t_end = q_offset + Lq - 1;
  if (win_start_of(q_offset, W) < win_start || t_end >= win_start + n_w || n_c_of(t_end, W, blk) > n_c)
    return HCADSA_ERR_SHAPE;
  if (!aligned16(Q) || !aligned16(Kw) || !aligned16(Vw) || !aligned16(O) || !aligned16(dO) || !aligned16(dQ) ||
      !aligned16(dKw) || !aligned16(dVw) || (n_c > 0 && (!aligned16(Kc) || !aligned16(Vc) || !aligned16(dKc) ||
                                                          !aligned16(dVc))) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u))
    return HCADSA_ERR_ALIGN;
  if ((long long)B * Lq * Hq > (1LL << 31) || (long long)B * n_w > (1LL << 31)) return HCADSA_ERR_UNSUPPORTED;
  Geo G;
  if (!make_geo(G, B, Lq, q_offset, Hq, Hkv, n_c, win_start, n_w, blk, W, scale)) return HCADSA_ERR_UNSUPPORTED;
  const size_t nblocks = scratch_blocks(G);
  if (nblocks * kTile > 0x7fffffffULL) return HCADSA_ERR_UNSUPPORTED;
  const size_t need = hca_attn_bwd_workspace_size(B, Lq, q_offset, Hq, Hkv, d, n_c, blk, W);
  if (!workspace || workspace_bytes < need) return HCADSA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return HCADSA_ERR_ALIGN;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* Dbuf = reinterpret_cast<float*>(ws);
  uint16_t* Pbuf = reinterpret_cast<uint16_t*>(ws + align256((size_t)B * Lq * Hq * 4));
  uint16_t* dSbuf = Pbuf + nblocks * kBlockElems;
  int* err = device_error_ptr();
  if (!err) return HCADSA_ERR_CUDA;
  cudaStream_t s = as_stream(stream);

  // ---- tensor maps
  const uint64_t qdims[4] = {(uint64_t)kD, (uint64_t)Hq, (uint64_t)Lq, (uint64_t)B};
  const uint64_t qstr[3] = {(uint64_t)kD * 2, (uint64_t)Hq * kD * 2, (uint64_t)Lq * Hq * kD * 2};
  const int bh = G.g > 64 ? 64 : G.g, bt = 64 / bh;
  ScoreMaps sm;
  GemmMaps gm;
  {
    const uint32_t qbox[4] = {64, (uint32_t)G.g, (uint32_t)G.tpt, 1};
    const uint32_t qbox64[4] = {64, (uint32_t)bh, (uint32_t)bt, 1};
    if (!encode_tmap_bf16(&sm.q, 4, const_cast<hcadsa_bf16*>(Q), qdims, qstr, qbox, true) ||
        !encode_tmap_bf16(&sm.dO, 4, const_cast<hcadsa_bf16*>(dO), qdims, qstr, qbox, true) ||
        !encode_tmap_bf16(&gm.q, 4, const_cast<hcadsa_bf16*>(Q), qdims, qstr, qbox64, true) ||
        !encode_tmap_bf16(&gm.dO, 4, const_cast<hcadsa_bf16*>(dO), qdims, qstr, qbox64, true))
      return HCADSA_ERR_CUDA;
    const uint32_t kbox[4] = {64, 1, (uint32_t)kTile, 1};
    const uint32_t kbox64[4] = {64, 1, 64, 1};
    const uint64_t wdims[4] = {(uint64_t)kD, (uint64_t)Hkv, (uint64_t)n_w, (uint64_t)B};
    const uint64_t wstr[3] = {(uint64_t)kD * 2, (uint64_t)Hkv * kD * 2, (uint64_t)n_w * Hkv * kD * 2};
    if (!encode_tmap_bf16(&sm.kw, 4, const_cast<hcadsa_bf16*>(Kw), wdims, wstr, kbox, true) ||
        !encode_tmap_bf16(&sm.vw, 4, const_cast<hcadsa_bf16*>(Vw), wdims, wstr, kbox, true) ||
        !encode_tmap_bf16(&gm.kw, 4, const_cast<hcadsa_bf16*>(Kw), wdims, wstr, kbox64, true))
      return HCADSA_ERR_CUDA;
    if (n_c > 0) {
      const uint64_t cdims[4] = {(uint64_t)kD, (uint64_t)Hkv, (uint64_t)n_c, (uint64_t)B};
      const uint64_t cstr[3] = {(uint64_t)kD * 2, (uint64_t)Hkv * kD * 2, (uint64_t)n_c * Hkv * kD * 2};
      if (!encode_tmap_bf16(&sm.kc, 4, const_cast<hcadsa_bf16*>(Kc), cdims, cstr, kbox, true) ||
          !encode_tmap_bf16(&sm.vc, 4, const_cast<hcadsa_bf16*>(Vc), cdims, cstr, kbox, true) ||
          !encode_tmap_bf16(&gm.kc, 4, const_cast<hcadsa_bf16*>(Kc), cdims, cstr, kbox64, true))
        return HCADSA_ERR_CUDA;
    } else {  // never read: no entry tiles
      sm.kc = sm.kw;
      sm.vc = sm.vw;
      gm.kc = gm.kw;
    }
    const uint64_t sdims[2] = {(uint64_t)kTile, (uint64_t)(nblocks * kTile)};
    const uint64_t sstr[1] = {(uint64_t)kTile * 2};
    const uint32_t box128[2] = {64, (uint32_t)kTile};
    const uint32_t box64[2] = {64, 64};
    if (!encode_tmap_bf16(&gm.dsK, 2, dSbuf, sdims, sstr, box128, true) ||
        !encode_tmap_bf16(&gm.dsM, 2, dSbuf, sdims, sstr, box64, true) ||
        !encode_tmap_bf16(&gm.pM, 2, Pbuf, sdims, sstr, box64, true))
      return HCADSA_ERR_CUDA;
  }

  // ---- 1. D per row
  const long long rows = (long long)B * Lq * Hq;
  hca_bwd_prep_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, s>>>(reinterpret_cast<const uint16_t*>(O),
                                                                  reinterpret_cast<const uint16_t*>(dO), Dbuf, rows);
  hcadsa_status st = launch_status();
  if (st != HCADSA_OK) return st;

  // ---- 2. P and dS blocks
  ScoreParams sp;
  sp.G = G;
  sp.lse = lse;
  sp.Dv = Dbuf;
  sp.P = Pbuf;
  sp.dS = dSbuf;
  sp.err = err;
  const int score_smem = kScoreStages * kScoreStageBytes + (int)sizeof(ScoreBars);
  if (cudaFuncSetAttribute(hca_bwd_scores_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, score_smem) !=
      cudaSuccess)
    return launch_status();
  const long long n_score = (long long)B * Hkv * G.n_rt;
  hca_bwd_scores_kernel<<<(unsigned)n_score, kThreads, score_smem, s>>>(sm, sp);
  st = launch_status();
  if (st != HCADSA_OK) return st;

  // ---- 3./4. dQ, then dK and dV
  GemmParams gp;
  gp.G = G;
  gp.bh = bh;
  gp.bt = bt;
  gp.dQ = dQ;
  gp.dKc = dKc;
  gp.dVc = dVc;
  gp.dKw = dKw;
  gp.dVw = dVw;
  gp.err = err;
  const int gemm_smem = kGemmStages * kGemmStageBytes + (int)sizeof(GemmBars);
  const int gemm_smem_half = kGemmStages * (kGemmABytes + kGemmBHalfBytes) + (int)sizeof(GemmBars);
  if (cudaFuncSetAttribute(hca_bwd_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, gemm_smem) !=
      cudaSuccess)
    return launch_status();
  gp.mode = 0;  // two units per row tile (column halves), two CTAs per SM
  hca_bwd_gemm_kernel<<<(unsigned)(2 * n_score), kThreads, gemm_smem_half, s>>>(gm, gp);
  st = launch_status();
  if (st != HCADSA_OK) return st;
  gp.mode = 1;
  const long long n_kv = 2LL * B * Hkv * ((long long)G.E_max * G.n_ch_e + (long long)G.n_wt * G.n_ch_w);
  if (n_kv > 0x7fffffffLL) return HCADSA_ERR_UNSUPPORTED;
  hca_bwd_gemm_kernel<<<(unsigned)n_kv, kThreads, gemm_smem, s>>>(gm, gp);
  return launch_status();
}
