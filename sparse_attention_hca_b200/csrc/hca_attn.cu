// hca_attn.cu -- HCA attention forward on sm_100a (tcgen05 + TMEM + TMA).
//
// Method: the mirrorspeed page, section "Hybrid sparse attention, 1/7 full context
// access" (and the besthub page, "Core Architectural Innovations", item 1): every 128
// tokens are compressed into one cache entry and a query attends over the compressed
// entries plus a recent uncompressed window; HCA heads are 512 wide (ai-club.cn page,
// section "混合注意力（MLA + HCA）").  Visible set of a query at t (this library's
// reading): raw positions [max(0,t-W+1), t] and entries j < n_c(t) = max(0,(t-W+1)/blk).
//
// Kernel design (one CTA per work item = 128 query rows x one 256-wide half of d_v):
//   * 128 rows = (128/g) consecutive tokens x the g query heads sharing one K/V head,
//     so every K/V tile is shared by the whole tile and the window band of 128/g
//     tokens spans only 128/g + W - 1 keys.
//   * d = 512 makes the fp32 O accumulator 128 x 512 = all of TMEM, so each CTA owns
//     one half of d_v: TMEM = O half [0,256) + two S buffers [256,384), [384,512).
//     The pair of CTAs of a row tile recomputes S = Q K^T (1.5x the algorithmic MMA
//     work) but reads each Q tile from HBM once (the pair runs back to back).
//   * warp 0: TMA producer (Q once, then K chunks and V chunks through a 5-slot ring of
//     16 KB stages, in exactly the order the MMA warp consumes them);
//     warp 1: TMEM allocation and the single MMA-issuing thread;
//     warps 2-5: softmax, one thread per row (TMEM lane), then the epilogue.
//   * S_j = Q K_j^T accumulates over eight 64-wide d chunks (SS MMA, K-major operands,
//     128B swizzle).  Softmax converts S_j to P_j (bf16) in place in TMEM and PV runs as
//     a TS MMA (A = P from TMEM, B = V chunk, MN-major).  Online softmax with a lazy
//     rescale: the reference max only moves when the tile max exceeds it by 2^8.
//   * Key tiles: compressed entries [0, n_c(t_last)) in tiles of 128, then the window
//     band [max(0, t_first-W+1), t_last] in tiles of 128; per-row visibility is one
//     column interval per tile.
#include <cuda_bf16.h>

#include "host_common.h"
#include "ptx.cuh"

namespace hcadsa {
namespace {

constexpr int kD = 512;
constexpr int kDHalf = 256;
constexpr int kKeyTile = 128;
constexpr int kStages = 5;
constexpr int kChunkBytes = 128 * 128;       // 128 rows x 64 bf16
constexpr int kQChunks = kD / 64;            // 8
constexpr int kVChunks = kDHalf / 64;        // 4
constexpr int kQBytes = kQChunks * kChunkBytes;
constexpr int kSmemBytes = kQBytes + kStages * kChunkBytes + 1024;
constexpr int kThreads = 192;
constexpr float kLazyRescale = 8.0f;  // log2 units

struct Params {
  int Lq, q_offset, Hq, Hkv, g, TT, n_c, win_start, W, blk;
  int n_tiles;  // token tiles per (b, kv head)
  float scale_log2;
  uint16_t* O;
  float* lse;
  int* err;
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

struct TileSet {
  int J_c, J;      // number of compressed tiles, total tiles
  int nc_hi;       // entries needed by the last token
  int ws_lo;       // window start of the first token
  int t_hi;        // last valid token position
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
  uint64_t q_full;
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t s_full[2];
  uint64_t p_ready[2];
  uint64_t pv_done;
  uint64_t o_full;  // one-shot: every PV of the work item has completed
};

__global__ void __launch_bounds__(kThreads, 1)
    hca_attn_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_kc,
                    const __grid_constant__ CUtensorMap map_vc, const __grid_constant__ CUtensorMap map_kw,
                    const __grid_constant__ CUtensorMap map_vw, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sRing = smem + kQBytes;
  __shared__ Barriers bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int half = blockIdx.x & 1;
  const int tile = blockIdx.x >> 1;
  const int b = blockIdx.y / p.Hkv, hk = blockIdx.y % p.Hkv;

  // token range of this tile
  const int tok0 = tile * p.TT;                           // relative to q_offset
  const int tok_hi = min(tok0 + p.TT, p.Lq) - 1;
  TileSet ts;
  ts.t_hi = p.q_offset + tok_hi;
  ts.nc_hi = n_compressed(ts.t_hi, p.W, p.blk);
  ts.ws_lo = window_start(p.q_offset + tok0, p.W);
  ts.J_c = (ts.nc_hi + kKeyTile - 1) / kKeyTile;
  ts.J = ts.J_c + (ts.t_hi - ts.ws_lo + kKeyTile) / kKeyTile;

  if (threadIdx.x == 0) {
    mbar_init(&bar.q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bar.full[s], 1);
      mbar_init(&bar.empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar.s_full[s], 1);
      mbar_init(&bar.p_ready[s], 128);
    }
    mbar_init(&bar.pv_done, 1);
    mbar_init(&bar.o_full, 1);
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
      tma_prefetch_desc(&map_q);
      mbar_arrive_expect_tx(&bar.q_full, kQBytes);
      for (int c = 0; c < kQChunks; ++c)
        tma_load_4d(sQ + c * kChunkBytes, &map_q, &bar.q_full, c * 64, hk * p.g, tok0, b);
      int slot = 0;
      uint32_t phase = 0;
      auto next_slot = [&](bool& ok) {
        ok = mbar_wait(&bar.empty[slot], phase ^ 1, &abort_flag, p.err);
        return slot;
      };
      for (int step = 0; step <= ts.J && !abort_flag; ++step) {
        if (step < ts.J) {
          const KeyTile kt = ts.get(step);
          const CUtensorMap* mk = kt.window ? &map_kw : &map_kc;
          const int row0 = kt.window ? kt.start - p.win_start : kt.start;
          for (int c = 0; c < kQChunks; ++c) {
            bool ok;
            next_slot(ok);
            if (!ok) break;
            mbar_arrive_expect_tx(&bar.full[slot], kChunkBytes);
            tma_load_4d(sRing + slot * kChunkBytes, mk, &bar.full[slot], c * 64, hk, row0, b);
            if (++slot == kStages) { slot = 0; phase ^= 1; }
          }
        }
        if (step >= 1) {
          const KeyTile kt = ts.get(step - 1);
          const CUtensorMap* mv = kt.window ? &map_vw : &map_vc;
          const int row0 = kt.window ? kt.start - p.win_start : kt.start;
          for (int c = 0; c < kVChunks; ++c) {
            bool ok;
            next_slot(ok);
            if (!ok) break;
            mbar_arrive_expect_tx(&bar.full[slot], kChunkBytes);
            tma_load_4d(sRing + slot * kChunkBytes, mv, &bar.full[slot], half * kDHalf + c * 64, hk, row0, b);
            if (++slot == kStages) { slot = 0; phase ^= 1; }
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait(&bar.q_full, 0, &abort_flag, p.err);
      tc_fence_after();
      int slot = 0;
      uint32_t phase = 0;
      const uint32_t sQa = smem_u32(sQ), sRa = smem_u32(sRing);
      for (int step = 0; ok && step <= ts.J; ++step) {
        if (step < ts.J) {
          const KeyTile kt = ts.get(step);
          const uint32_t tS = tmem + kDHalf + (step & 1) * kKeyTile;
          const uint32_t idesc = idesc_bf16_f32(128, kt.n, false, false);
          // S buffer (step & 1) still holds P_{step-2}, the TMEM A operand of PV_{step-2}.
          // MMAs on different accumulators are not ordered, so wait for that PV to finish.
          if (step >= 2) {
            ok = mbar_wait(&bar.pv_done, (step - 2) & 1, &abort_flag, p.err);
            if (!ok) break;
            tc_fence_after();
          }
          for (int c = 0; c < kQChunks && ok; ++c) {
            ok = mbar_wait(&bar.full[slot], phase, &abort_flag, p.err);
            if (!ok) break;
            tc_fence_after();
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const uint64_t da = smem_desc_sw128(sQa + c * kChunkBytes + k * 32, 16, 1024);
              const uint64_t db = smem_desc_sw128(sRa + slot * kChunkBytes + k * 32, 16, 1024);
              mma_ss(tS, da, db, idesc, (c | k) != 0);
            }
            mma_commit(&bar.empty[slot]);
            if (++slot == kStages) { slot = 0; phase ^= 1; }
          }
          if (!ok) break;
          mma_commit(&bar.s_full[step & 1]);
        }
        if (step >= 1) {
          const int j = step - 1;
          const KeyTile kt = ts.get(j);
          ok = mbar_wait(&bar.p_ready[j & 1], (j >> 1) & 1, &abort_flag, p.err);
          if (!ok) break;
          tc_fence_after();
          const uint32_t tP = tmem + kDHalf + (j & 1) * kKeyTile;
          const uint32_t idesc = idesc_bf16_f32(128, 64, false, true);
          for (int c = 0; c < kVChunks && ok; ++c) {
            ok = mbar_wait(&bar.full[slot], phase, &abort_flag, p.err);
            if (!ok) break;
            tc_fence_after();
            for (int kk = 0; kk < kt.n / 16; ++kk) {
              const uint64_t db = smem_desc_sw128(sRa + slot * kChunkBytes + kk * 2048, kChunkBytes, 1024);
              mma_ts(tmem + c * 64, tP + kk * 8, db, idesc, (j > 0 || kk > 0) ? 1u : 0u);
            }
            mma_commit(&bar.empty[slot]);
            if (++slot == kStages) { slot = 0; phase ^= 1; }
          }
          if (!ok) break;
          mma_commit(&bar.pv_done);
          if (j == ts.J - 1) mma_commit(&bar.o_full);
        }
      }
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // row of the tile == TMEM lane
    const int tok = tok0 + r / p.g;     // relative token index
    const int h = hk * p.g + r % p.g;
    const bool row_valid = tok < p.Lq;
    const int t = p.q_offset + min(tok, p.Lq - 1);
    const int nc_t = n_compressed(t, p.W, p.blk);
    const int ws_t = window_start(t, p.W);
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    float m_ref = -INFINITY, l_run = 0.0f;
    bool ok = true;
    for (int j = 0; j < ts.J && ok; ++j) {
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
      const uint32_t tS = tmem + lane_off + kDHalf + (j & 1) * kKeyTile;
      ok = mbar_wait(&bar.s_full[j & 1], (j >> 1) & 1, &abort_flag, p.err);
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
        // O (this half) must hold every PV up to tile j-1 before it is rescaled
        ok = mbar_wait(&bar.pv_done, (j - 1) & 1, &abort_flag, p.err);
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
      mbar_arrive(&bar.p_ready[j & 1]);
    }
    // pv_done may be two phases behind here, so its parity cannot be trusted: use o_full
    if (ok) ok = mbar_wait(&bar.o_full, 0, &abort_flag, p.err);
    if (ok) {
      tc_fence_after();
      const float inv_l = l_run > 0.0f ? 1.0f / l_run : 0.0f;
      uint16_t* orow = p.O + ((size_t)((size_t)b * p.Lq + tok) * p.Hq + h) * kD + half * kDHalf;
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
      if (half == 0 && p.lse && row_valid)
        p.lse[((size_t)b * p.Lq + tok) * p.Hq + h] = (m_ref + __log2f(l_run)) * 0.69314718055994531f;
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
  if (!aligned16(Q) || !aligned16(Kw) || !aligned16(Vw) || !aligned16(O) || (n_c > 0 && (!aligned16(Kc) || !aligned16(Vc))) ||
      (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)))
    return HCADSA_ERR_ALIGN;
  if (B == 0 || Lq == 0) return HCADSA_OK;
  // every query's visible set must be stored
  const long long t_first = q_offset, t_last = (long long)q_offset + Lq - 1;
  if (t_last > 2147483647LL - 256) return HCADSA_ERR_UNSUPPORTED;
  const long long ws_first = t_first - W + 1 > 0 ? t_first - W + 1 : 0;
  const long long nc_last = t_last - W + 1 > 0 ? (t_last - W + 1) / blk : 0;
  if (ws_first < win_start || t_last - win_start >= n_w || nc_last > n_c) return HCADSA_ERR_SHAPE;
  if (B * Hkv > 65535) return HCADSA_ERR_UNSUPPORTED;

  const int TT = 128 / g;
  CUtensorMap mq, mkc, mvc, mkw, mvw;
  if (!make_map_4d(&mq, Q, kD, Hq, Lq, B, g, TT)) return HCADSA_ERR_CUDA;
  if (!make_map_4d(&mkw, Kw, kD, Hkv, n_w, B, 1, 128)) return HCADSA_ERR_CUDA;
  if (!make_map_4d(&mvw, Vw, kD, Hkv, n_w, B, 1, 128)) return HCADSA_ERR_CUDA;
  if (n_c > 0) {
    if (!make_map_4d(&mkc, Kc, kD, Hkv, n_c, B, 1, 128)) return HCADSA_ERR_CUDA;
    if (!make_map_4d(&mvc, Vc, kD, Hkv, n_c, B, 1, 128)) return HCADSA_ERR_CUDA;
  } else {
    mkc = mkw;
    mvc = mvw;
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
  p.n_tiles = (Lq + TT - 1) / TT;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.O = O;
  p.lse = lse;
  p.err = device_error_ptr();
  if (cudaFuncSetAttribute(hca_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) != cudaSuccess)
    return HCADSA_ERR_CUDA;
  dim3 grid((unsigned)(p.n_tiles * 2), (unsigned)(B * Hkv));
  hca_attn_kernel<<<grid, kThreads, kSmemBytes, as_stream(stream)>>>(mq, mkc, mvc, mkw, mvw, p);
  return launch_status();
}
