// hca_attn.cu -- HCA attention forward on sm_100a (tcgen05 + TMEM + TMA).
//
// Method: the mirrorspeed page, section "Hybrid sparse attention, 1/7 full context
// access" (and the besthub page, "Core Architectural Innovations", item 1): every 128
// tokens are compressed into one cache entry and a query attends over the compressed
// entries plus a recent uncompressed window; HCA heads are 512 wide (ai-club.cn page,
// section "混合注意力（MLA + HCA）").  Visible set of a query at t (this library's
// reading): raw positions [max(0,t-W+1), t] and entries j < n_c(t) = max(0,(t-W+1)/blk).
//
// Kernel design (persistent: a CTA walks row tiles T = blockIdx.x + i*gridDim.x and runs the
// two 256-wide halves of d_v of each tile back to back as two work items):
//   * A row tile = 128 rows = (128/g) consecutive tokens x the g query heads sharing one K/V
//     head, so every K/V tile is shared by the whole tile and the window band of 128/g
//     tokens spans only 128/g + W - 1 keys.
//   * d = 512 makes a 128 x 512 fp32 O accumulator fill all of TMEM, so a work item keeps O
//     for one half of d_v: TMEM = O half [0,256) + two S buffers [256,384), [384,512).  Each
//     item recomputes S = Q K^T (1.5x the algorithmic MMA work); Q is loaded once per tile.
//   * warp 0: TMA producer (Q per tile, then K chunks and V chunks through a 5-slot ring of
//     16 KB stages, in exactly the order the MMA warp consumes them; key tiles of at most
//     32 keys use 32-row boxes); warp 1: TMEM allocation and the single MMA-issuing thread;
//     warps 2-5: softmax, one thread per row (TMEM lane), then the item's epilogue.  The next
//     item's S MMAs run while the epilogue drains O.
//   * S_j = Q K_j^T accumulates over eight 64-wide d chunks (SS MMA, K-major operands,
//     128B swizzle).  Softmax converts S_j to P_j (bf16) in place in TMEM and PV runs as
//     a TS MMA (A = P from TMEM, B = V chunk, MN-major).  Online softmax with a lazy
//     rescale: the reference max only moves when the tile max exceeds it by 2^8.
//   * Key tiles: compressed entries [0, n_c(t_last)) in tiles of 128, then the window
//     band [max(0, t_first-W+1), t_last] in tiles of 128; per-row visibility is one
//     column interval per tile.
//   * Barrier phases run on across work items: s_full / p_ready / pv_done are per S buffer
//     and follow a key-tile counter that never resets, o_full / o_empty follow the item
//     counter, q_full / q_empty the row-tile counter.  MMAs on different accumulators are
//     not ordered, so an S buffer is rewritten only after the PV that read its P completed.
#include <cuda_bf16.h>

#include <mutex>

#include "host_common.h"
#include "ptx.cuh"

namespace hcadsa {
namespace {

constexpr int kD = 512;
constexpr int kDHalf = 256;
constexpr int kKeyTile = 128;
constexpr int kSmallRows = 32;  // TMA box height for key tiles of at most 32 keys
constexpr int kStages = 5;
constexpr int kChunkBytes = 128 * 128;  // 128 rows x 64 bf16
constexpr int kSmallChunkBytes = kSmallRows * 128;
constexpr int kQChunks = kD / 64;      // 8
constexpr int kVChunks = kDHalf / 64;  // 4
constexpr int kQBytes = kQChunks * kChunkBytes;
constexpr int kSmemBytes = kQBytes + kStages * kChunkBytes + 1024;
constexpr int kThreads = 192;
constexpr float kLazyRescale = 8.0f;  // log2 units

struct Params {
  int Lq, q_offset, Hq, Hkv, g, TT, n_c, win_start, W, blk;
  int n_tiles;      // token tiles per (b, kv head)
  int total_tiles;  // B * Hkv * n_tiles
  float scale_log2;
  uint16_t* O;
  float* lse;
  int* err;
};

// Q, then K and V over {compressed entries, window} x {128-row box, 32-row box}.
struct Maps {
  CUtensorMap q;
  CUtensorMap kv[2][2][2];  // [0 = K, 1 = V][0 = compressed, 1 = window][0 = 128 rows, 1 = 32 rows]
};

__device__ __forceinline__ int n_compressed(int t, int W, int blk) {
  const int s = t - W + 1;
  return s > 0 ? s / blk : 0;
}
__device__ __forceinline__ int window_start(int t, int W) {
  const int s = t - W + 1;
  return s > 0 ? s : 0;
}

struct KeyTile {
  int window;  // 0: compressed entries, 1: raw window positions
  int start;   // first entry / position
  int n;       // MMA N (multiple of 16, <= 128)
};

// The key tiles of one row tile.
struct TileSet {
  int b, hk, tok0;  // batch, kv head, first token (relative to q_offset)
  int J_c, J;       // number of compressed tiles, total tiles
  int nc_hi;        // entries needed by the last token
  int ws_lo;        // window start of the first token
  int t_hi;         // last valid token position
  __device__ void init(int T, const Params& p) {
    const int bh = T / p.n_tiles, tile = T % p.n_tiles;
    b = bh / p.Hkv;
    hk = bh % p.Hkv;
    tok0 = tile * p.TT;
    t_hi = p.q_offset + min(tok0 + p.TT, p.Lq) - 1;
    nc_hi = n_compressed(t_hi, p.W, p.blk);
    ws_lo = window_start(p.q_offset + tok0, p.W);
    J_c = (nc_hi + kKeyTile - 1) / kKeyTile;
    J = J_c + (t_hi - ws_lo + kKeyTile) / kKeyTile;
  }
  __device__ KeyTile get(int j) const {
    KeyTile kt;
    if (j < J_c) {
      kt.window = 0;
      kt.start = j * kKeyTile;
      const int rem = min(kKeyTile, nc_hi - kt.start);
      kt.n = (rem + 15) & ~15;
    } else {
      kt.window = 1;
      kt.start = ws_lo + (j - J_c) * kKeyTile;
      const int rem = min(kKeyTile, t_hi + 1 - kt.start);
      kt.n = (rem + 15) & ~15;
    }
    return kt;
  }
};

struct __align__(8) Barriers {
  uint64_t q_full, q_empty;
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t s_full[2];
  uint64_t p_ready[2];
  uint64_t pv_done[2];  // the PV that read P from S buffer i has completed
  uint64_t o_full;      // every PV of the work item has completed
  uint64_t o_empty;     // the epilogue has read O
};

__global__ void __launch_bounds__(kThreads, 1) hca_attn_kernel(const __grid_constant__ Maps maps, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sRing = smem + kQBytes;
  __shared__ Barriers bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    mbar_init(&bar.q_full, 1);
    mbar_init(&bar.q_empty, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bar.full[s], 1);
      mbar_init(&bar.empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar.s_full[s], 1);
      mbar_init(&bar.p_ready[s], 128);
      mbar_init(&bar.pv_done[s], 1);
    }
    mbar_init(&bar.o_full, 1);
    mbar_init(&bar.o_empty, 128);
    abort_flag = 0;
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
      uint32_t q = 0;       // ring chunks issued: slot q % kStages, phase (q / kStages) & 1
      uint32_t tcount = 0;  // row tiles started
      bool ok = true;
      for (int T = blockIdx.x; ok && T < p.total_tiles; T += gridDim.x, ++tcount) {
        TileSet ts;
        ts.init(T, p);
        // Q of this tile, once the previous tile's last S MMA has read the buffer
        ok = mbar_wait(&bar.q_empty, (tcount & 1) ^ 1, &abort_flag, p.err);
        if (!ok) break;
        mbar_arrive_expect_tx(&bar.q_full, kQBytes);
        for (int c = 0; c < kQChunks; ++c)
          tma_load_4d(sQ + c * kChunkBytes, &maps.q, &bar.q_full, c * 64, ts.hk * p.g, ts.tok0, ts.b);
        for (int half = 0; ok && half < 2; ++half) {
          for (int step = 0; ok && step <= ts.J; ++step) {
            // step s: the K chunks of key tile s, then the V chunks (this half) of key tile s-1
            for (int part = 0; ok && part < 2; ++part) {
              const int is_v = part;
              const int j = step - is_v;
              if (j < 0 || j >= ts.J) continue;
              const KeyTile kt = ts.get(j);
              const int small = kt.n <= kSmallRows ? 1 : 0;
              const CUtensorMap* m = &maps.kv[is_v][kt.window][small];
              const int row0 = kt.window ? kt.start - p.win_start : kt.start;
              const int n_ch = is_v ? kVChunks : kQChunks;
              const int col0 = is_v ? half * kDHalf : 0;
              for (int c = 0; c < n_ch; ++c, ++q) {
                const uint32_t slot = q % kStages;
                ok = mbar_wait(&bar.empty[slot], ((q / kStages) & 1) ^ 1, &abort_flag, p.err);
                if (!ok) break;
                mbar_arrive_expect_tx(&bar.full[slot], small ? kSmallChunkBytes : kChunkBytes);
                tma_load_4d(sRing + slot * kChunkBytes, m, &bar.full[slot], col0 + c * 64, ts.hk, row0, ts.b);
              }
            }
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t sQa = smem_u32(sQ), sRa = smem_u32(sRing);
      uint32_t q = 0;       // ring chunks consumed
      uint32_t tcount = 0;  // row tiles
      uint32_t g = 0;       // key tiles of all earlier work items
      uint32_t it = 0;      // work items
      bool ok = true;
      for (int T = blockIdx.x; ok && T < p.total_tiles; T += gridDim.x, ++tcount) {
        TileSet ts;
        ts.init(T, p);
        ok = mbar_wait(&bar.q_full, tcount & 1, &abort_flag, p.err);
        if (!ok) break;
        tc_fence_after();
        for (int half = 0; ok && half < 2; ++half, ++it) {
          for (int step = 0; ok && step <= ts.J; ++step) {
            if (step < ts.J) {
              const uint32_t gs = g + step;
              const KeyTile kt = ts.get(step);
              const uint32_t tS = tmem + kDHalf + (gs & 1) * kKeyTile;
              const uint32_t idesc = idesc_bf16_f32(128, kt.n, false, false);
              // S buffer gs&1 holds P_{gs-2}, the TMEM operand of PV_{gs-2}
              if (gs >= 2) {
                ok = mbar_wait(&bar.pv_done[gs & 1], ((gs >> 1) - 1) & 1, &abort_flag, p.err);
                if (!ok) break;
                tc_fence_after();
              }
              for (int c = 0; ok && c < kQChunks; ++c, ++q) {
                const uint32_t slot = q % kStages;
                ok = mbar_wait(&bar.full[slot], (q / kStages) & 1, &abort_flag, p.err);
                if (!ok) break;
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                  const uint64_t da = smem_desc_sw128(sQa + c * kChunkBytes + k * 32, 16, 1024);
                  const uint64_t db = smem_desc_sw128(sRa + slot * kChunkBytes + k * 32, 16, 1024);
                  mma_ss(tS, da, db, idesc, (c | k) != 0);
                }
                mma_commit(&bar.empty[slot]);
              }
              if (!ok) break;
              mma_commit(&bar.s_full[gs & 1]);
              if (half == 1 && step == ts.J - 1) mma_commit(&bar.q_empty);
            }
            if (step >= 1) {
              const int j = step - 1;
              const uint32_t gj = g + j;
              const KeyTile kt = ts.get(j);
              if (j == 0) {  // the previous item's epilogue must have read O
                ok = mbar_wait(&bar.o_empty, (it & 1) ^ 1, &abort_flag, p.err);
                if (!ok) break;
              }
              ok = mbar_wait(&bar.p_ready[gj & 1], (gj >> 1) & 1, &abort_flag, p.err);
              if (!ok) break;
              tc_fence_after();
              const uint32_t tP = tmem + kDHalf + (gj & 1) * kKeyTile;
              const uint32_t idesc = idesc_bf16_f32(128, 64, false, true);
              for (int c = 0; ok && c < kVChunks; ++c, ++q) {
                const uint32_t slot = q % kStages;
                ok = mbar_wait(&bar.full[slot], (q / kStages) & 1, &abort_flag, p.err);
                if (!ok) break;
                tc_fence_after();
                for (int kk = 0; kk < kt.n / 16; ++kk) {
                  const uint64_t db = smem_desc_sw128(sRa + slot * kChunkBytes + kk * 2048, kChunkBytes, 1024);
                  mma_ts(tmem + c * 64, tP + kk * 8, db, idesc, (j > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(&bar.empty[slot]);
              }
              if (!ok) break;
              mma_commit(&bar.pv_done[gj & 1]);
              if (j == ts.J - 1) mma_commit(&bar.o_full);
            }
          }
          g += ts.J;
        }
      }
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // row of the tile == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    uint32_t g = 0, it = 0;
    bool ok = true;
    for (int T = blockIdx.x; ok && T < p.total_tiles; T += gridDim.x) {
      TileSet ts;
      ts.init(T, p);
      const int tok = ts.tok0 + r / p.g;  // relative token index
      const int h = ts.hk * p.g + r % p.g;
      const bool row_valid = tok < p.Lq;
      const int t = p.q_offset + min(tok, p.Lq - 1);
      const int nc_t = n_compressed(t, p.W, p.blk);
      const int ws_t = window_start(t, p.W);
      for (int half = 0; ok && half < 2; ++half, ++it) {
        float m_ref = -INFINITY, l_run = 0.0f;
        for (int j = 0; ok && j < ts.J; ++j) {
          const uint32_t gs = g + j;
          const KeyTile kt = ts.get(j);
          int lo, hi;
          if (kt.window) {
            lo = max(ws_t, kt.start) - kt.start;
            hi = min(t + 1, kt.start + kt.n) - kt.start;
          } else {
            lo = 0;
            hi = min(nc_t, kt.start + kt.n) - kt.start;
          }
          if (!row_valid) hi = lo;  // padding rows see nothing
          const uint32_t tS = tmem + lane_off + kDHalf + (gs & 1) * kKeyTile;
          ok = mbar_wait(&bar.s_full[gs & 1], (gs >> 1) & 1, &abort_flag, p.err);
          if (!ok) break;
          tc_fence_after();
          // pass 1: tile max over this row's visible columns
          float mx = -INFINITY;
          for (int c0 = 0; c0 < kt.n; c0 += 32) {
            uint32_t v[32];
            tmem_ld32_nowait(tS + c0, v);
            tmem_wait_ld_regs(v);
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int col = c0 + i;
              if (col >= lo && col < hi) mx = fmaxf(mx, __uint_as_float(v[i]));
            }
          }
          const float m_tile = mx * p.scale_log2;  // -inf stays -inf
          bool need = false;
          if (m_ref == -INFINITY) {
            m_ref = m_tile;
          } else if (m_tile > m_ref + kLazyRescale) {
            need = true;
          }
          if (__any_sync(0xffffffffu, need)) {
            // O must hold every PV of this item up to key tile j-1 (j >= 1 here) before the rescale
            const uint32_t gp = gs - 1;
            ok = mbar_wait(&bar.pv_done[gp & 1], (gp >> 1) & 1, &abort_flag, p.err);
            if (!ok) break;
            tc_fence_after();
            const float alpha = need ? fast_exp2(m_ref - m_tile) : 1.0f;
            if (need) m_ref = m_tile;
            l_run *= alpha;
            for (int oc = 0; oc < kDHalf; oc += 32) {
              uint32_t v[32];
              tmem_ld32_nowait(tmem + lane_off + oc, v);
              tmem_wait_ld_regs(v);
#pragma unroll
              for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * alpha);
              tmem_st32(tmem + lane_off + oc, v);
            }
            tmem_wait_st();
          }
          // pass 2: P = exp2(s*scale*log2e - m_ref) as bf16, in place over S
          const bool any_visible = m_ref != -INFINITY;
          for (int c0 = 0; c0 < kt.n; c0 += 32) {
            uint32_t v[32];
            tmem_ld32_nowait(tS + c0, v);
            tmem_wait_ld_regs(v);
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const int c = c0 + 2 * i;
              float p0 = 0.0f, p1 = 0.0f;
              if (any_visible && c >= lo && c < hi) p0 = fast_exp2(__uint_as_float(v[2 * i]) * p.scale_log2 - m_ref);
              if (any_visible && c + 1 >= lo && c + 1 < hi)
                p1 = fast_exp2(__uint_as_float(v[2 * i + 1]) * p.scale_log2 - m_ref);
              l_run += p0 + p1;
              pk[i] = pack_bf16x2(p0, p1);
            }
            tmem_st16(tS + c0 / 2, pk);
          }
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(&bar.p_ready[gs & 1]);
        }
        if (!ok) break;
        // ---- epilogue of the item: O half -> bf16 -> global, then hand O back to the MMA warp
        ok = mbar_wait(&bar.o_full, it & 1, &abort_flag, p.err);
        if (!ok) break;
        tc_fence_after();
        const float inv_l = l_run > 0.0f ? 1.0f / l_run : 0.0f;
        uint16_t* orow = p.O + ((size_t)((size_t)ts.b * p.Lq + tok) * p.Hq + h) * kD + half * kDHalf;
        for (int oc = 0; oc < kDHalf; oc += 32) {
          uint32_t v[32];
          tmem_ld32_nowait(tmem + lane_off + oc, v);
          tmem_wait_ld_regs(v);
          if (row_valid) {
            uint4 packed[4];
            uint32_t* pw = reinterpret_cast<uint32_t*>(packed);
#pragma unroll
            for (int i = 0; i < 16; ++i)
              pw[i] = pack_bf16x2(__uint_as_float(v[2 * i]) * inv_l, __uint_as_float(v[2 * i + 1]) * inv_l);
            uint4* dst = reinterpret_cast<uint4*>(orow + oc);
#pragma unroll
            for (int i = 0; i < 4; ++i) dst[i] = packed[i];
          }
        }
        tc_fence_before();
        mbar_arrive(&bar.o_empty);
        if (half == 0 && p.lse && row_valid)
          p.lse[((size_t)ts.b * p.Lq + tok) * p.Hq + h] = (m_ref + __log2f(l_run)) * 0.69314718055994531f;
        g += ts.J;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

bool make_map_4d(CUtensorMap* m, const void* base, int d, int heads, int rows, int B, int box_heads, int box_rows) {
  const uint64_t dims[4] = {(uint64_t)d, (uint64_t)heads, (uint64_t)rows, (uint64_t)B};
  const uint64_t strides[3] = {(uint64_t)d * 2, (uint64_t)heads * d * 2, (uint64_t)rows * heads * d * 2};
  const uint32_t box[4] = {64, (uint32_t)box_heads, (uint32_t)box_rows, 1};
  return encode_tmap_bf16(m, 4, const_cast<void*>(base), dims, strides, box, true);
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

}  // namespace
}  // namespace hcadsa

extern "C" size_t hca_attn_fwd_workspace_size(int B, int Lq, int q_offset, int Hq, int Hkv, int d, int n_c, int blk,
                                              int W) {
  (void)B; (void)Lq; (void)q_offset; (void)Hq; (void)Hkv; (void)d; (void)n_c; (void)blk; (void)W;
  return 0;
}

extern "C" hcadsa_status hca_attn_fwd(const hcadsa_bf16* Q, const hcadsa_bf16* Kc, const hcadsa_bf16* Vc, int n_c,
                                      const hcadsa_bf16* Kw, const hcadsa_bf16* Vw, int win_start, int n_w,
                                      hcadsa_bf16* O, float* lse, int B, int Lq, int q_offset, int Hq, int Hkv,
                                      int d, int blk, int W, float scale, void* workspace, size_t workspace_bytes,
                                      hcadsa_stream stream) {
  using namespace hcadsa;
  (void)workspace; (void)workspace_bytes;
  if (!Q || !Kw || !Vw || !O) return HCADSA_ERR_NULL;
  if (n_c > 0 && (!Kc || !Vc)) return HCADSA_ERR_NULL;
  if (B < 0 || Lq < 0 || q_offset < 0 || Hq <= 0 || Hkv <= 0 || n_c < 0 || n_w < 0 || win_start < 0 || blk <= 0 ||
      W <= 0)
    return HCADSA_ERR_SHAPE;
  if (Hq % Hkv != 0) return HCADSA_ERR_SHAPE;
  const int g = Hq / Hkv;
  if (d != kD || g > 128 || 128 % g != 0) return HCADSA_ERR_UNSUPPORTED;
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
  const int TT = 128 / g;
  const long long n_tiles = (Lq + TT - 1) / TT;
  if ((long long)B * Hkv * n_tiles > 2147483647LL) return HCADSA_ERR_UNSUPPORTED;

  Maps maps;
  if (!make_map_4d(&maps.q, Q, kD, Hq, Lq, B, g, TT)) return HCADSA_ERR_CUDA;
  for (int small = 0; small < 2; ++small) {
    const int rows = small ? kSmallRows : 128;
    if (!make_map_4d(&maps.kv[0][1][small], Kw, kD, Hkv, n_w, B, 1, rows)) return HCADSA_ERR_CUDA;
    if (!make_map_4d(&maps.kv[1][1][small], Vw, kD, Hkv, n_w, B, 1, rows)) return HCADSA_ERR_CUDA;
    if (n_c > 0) {
      if (!make_map_4d(&maps.kv[0][0][small], Kc, kD, Hkv, n_c, B, 1, rows)) return HCADSA_ERR_CUDA;
      if (!make_map_4d(&maps.kv[1][0][small], Vc, kD, Hkv, n_c, B, 1, rows)) return HCADSA_ERR_CUDA;
    } else {  // no query sees an entry: these maps are never read
      maps.kv[0][0][small] = maps.kv[0][1][small];
      maps.kv[1][0][small] = maps.kv[1][1][small];
    }
  }
  Params p;
  p.Lq = Lq;
  p.q_offset = q_offset;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.g = g;
  p.TT = TT;
  p.n_c = n_c;
  p.win_start = win_start;
  p.W = W;
  p.blk = blk;
  p.n_tiles = (int)n_tiles;
  p.total_tiles = (int)((long long)B * Hkv * n_tiles);
  p.scale_log2 = scale * 1.4426950408889634f;
  p.O = O;
  p.lse = lse;
  p.err = device_error_ptr();
  if (cudaFuncSetAttribute(hca_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) != cudaSuccess)
    return HCADSA_ERR_CUDA;
  const int sms = num_sms();
  if (sms <= 0) return HCADSA_ERR_CUDA;
  const int grid = p.total_tiles < sms ? p.total_tiles : sms;
  hca_attn_kernel<<<grid, kThreads, kSmemBytes, as_stream(stream)>>>(maps, p);
  return launch_status();
}
