// dsa_attn_bwd.cu -- DSA sparse attention backward on sm_100a (tcgen05 + TMEM; K/V rows gathered
// with cp.async, Q and dO loaded by TMA).
//
// Method: the forward of the mirrorspeed page's section "Hybrid sparse attention, 1/7 full
// context access" (each query attends only to its k selected positions; 64 heads of 256 share
// one K/V head and the index row).  For a loss with gradient dO on the output, per token t,
// head h and selected key s (p = softmax probabilities, reproduced from the forward's lse):
//     dV[s]  += sum_h p[h,s] dO[h]
//     dP[h,s] = <dO[h], V[s]>,   dS[h,s] = p[h,s] (dP[h,s] - D[h]),  D[h] = <dO[h], O[h]>
//     dQ[h]   = scale sum_s dS[h,s] K[s]
//     dK[s]  += scale sum_h dS[h,s] Q[h]
//
// Kernel design (one CTA per token; the token's 128-key tiles in order):
//   * Transposed like the forward, keys as M (128 per tile):
//       S^T  = K_g Q^T,   dP^T = V_g dO^T        (SS, K-major, N = 64 heads, fp32 in TMEM)
//     the four softmax warps (thread = key = TMEM lane) form P^T and dS^T (bf16) and write them,
//     128B-swizzled, over the V tile (whose last reader was the dP^T MMA), then
//       dV_g = P^T dO,    dK_g = dS^T Q          (A = P^T / dS^T K-major, B = dO / Q MN-major,
//                                                 N = 256, one 256-column TMEM region in turn)
//       dQ^T += K_g^T dS^T                       (A = K_g MN-major, B = dS^T MN-major, over all
//                                                 tiles of the token, 2 x 64 TMEM columns)
//     TMEM: S^T 64 + dP^T 64 + dK_g/dV_g 256 + dQ^T 128 = 512 columns.
//   * MMA order per tile: S^T, dP^T | dV_g, dQ^T (the K tile is free) | dK_g (the V tile's space
//     is free), so the next tile's K rows are gathered while dK_g waits for the read-out of dV_g.
//   * dK_g / dV_g rows go to dK[s] / dV[s] as bulk asynchronous reductions (cp.reduce.async.bulk
//     add.f32, 256 bytes = 64 columns of one key per operation): four reduction warps (thread =
//     key) stage a key's 64 columns in their own padded shared-memory row (272-byte stride:
//     conflict-free 16-byte stores) and hand the row to the bulk-copy unit, which adds whole
//     lines in L2; the softmax warps meanwhile work on the next tile.  Several tokens select the
//     same key, in any order, so dK and dV are summed in fp32 in an order that is not fixed.
//     dQ is written once per token (fp32) by the softmax warps.
//   * Warps 0-2 gather the K and V rows of a tile with cp.async (one 512-byte row per warp
//     instruction, 128B-swizzled), warp 3 allocates TMEM and issues every MMA, warps 4-7 are the
//     softmax warps, warps 8-11 the reduction warps.  One K and one V tile are resident.
//   * D[h] = <dO[h], O[h]> is computed at the token's start by the softmax warps.
// Every wait is bounded (the library's 2 s limit); on expiry the error word records a timeout
// and every role leaves its loop.
#include <cuda_bf16.h>

#include <mutex>

#include "host_common.h"
#include "ptx.cuh"

namespace hcadsa {
namespace {

constexpr int kD = 256;
constexpr int kH = 64;
constexpr int kKeyTile = 128;
constexpr int kChunkBytes = 128 * 128;     // 128 rows x 64 bf16
constexpr int kTileBytes = 4 * kChunkBytes;  // 64 KB: 128 rows x 256 bf16
constexpr int kQChunkBytes = kH * 128;     // 64 heads x 64 bf16
constexpr int kQBytes = 4 * kQChunkBytes;  // 32 KB
constexpr int kPBytes = kKeyTile * 128;    // 128 keys x 64 heads bf16 (16 KB)
constexpr int kMaxK = 4096;
constexpr int kProducerWarps = 3;
constexpr int kMmaWarp = kProducerWarps;
constexpr int kSoftWarp0 = kProducerWarps + 1;  // 4 warps: P^T, dS^T, D, the dQ epilogue
constexpr int kRedWarp0 = kSoftWarp0 + 4;       // 4 warps: dV_g / dK_g read-out and reductions
constexpr int kThreads = 32 * (kRedWarp0 + 4);
constexpr int kStageCols = 64;                     // fp32 columns per bulk reduction
constexpr int kStageStride = kStageCols * 4 + 16;  // padded row: 16-byte stores conflict-free
// layout (no static shared memory, so the dynamic window starts 1024-byte aligned):
// Q | dO | K tile | V tile (later P^T, dS^T) | reduction staging | barriers and small arrays
constexpr int kOffQ = 0, kOffDO = kQBytes, kOffK = 2 * kQBytes, kOffV = kOffK + kTileBytes;
constexpr int kOffStage = kOffV + kTileBytes;
constexpr int kOffMisc = kOffStage + kKeyTile * kStageStride;
constexpr uint32_t kTmemS = 0, kTmemDP = 64, kTmemKV = 128, kTmemDQ = 384;

struct Params {
  const uint16_t* K;
  const uint16_t* V;
  const uint16_t* O;
  const uint16_t* dO;
  const float* lse;
  const int32_t* idx;
  float* dQ;
  float* dK;
  float* dV;
  int* err;
  int Lq, Lk, k;
  float scale, scale_log2;
};

struct __align__(8) Misc {
  uint64_t q_full;    // Q and dO of the token landed (TMA)
  uint64_t k_full, v_full;  // the tile's K / V rows landed (192 producer-thread arrivals)
  uint64_t k_free;    // the tile's MMAs are done with the K tile (after dQ^T)
  uint64_t v_free;    // ... and with the V tile's space (P^T, dS^T: after dK_g)
  uint64_t s_ready;   // S^T and dP^T are in TMEM
  uint64_t p_ready;   // P^T and dS^T are in shared memory (128 row threads)
  uint64_t dv_ready, dk_ready;  // dV_g / dK_g in TMEM
  uint64_t kv_read;   // the reduction warps have read the dK_g / dV_g region (twice per tile)
  uint64_t dq_full;   // dQ^T of the token is complete
  uint32_t tmem_base;
  int abort_flag;
  uint32_t mask;      // bit j: tile j holds a valid entry
  float lse2[kH], D[kH];
};
constexpr int kSmemBytes = kOffMisc + (int)sizeof(Misc);
static_assert(kSmemBytes <= 232448, "shared memory");

__device__ __forceinline__ bool idx_ok(int s, int Lk) { return s >= 0 && s < Lk; }

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
__device__ __forceinline__ void bulk_reduce_add_f32(float* dst, uint32_t src, uint32_t bytes) {
  asm volatile("cp.reduce.async.bulk.global.shared::cta.bulk_group.add.f32 [%0], [%1], %2;" ::"l"(dst), "r"(src),
               "r"(bytes)
               : "memory");
}

__global__ void __launch_bounds__(kThreads, 1)
    dsa_attn_bwd_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_do,
                        const Params p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  if (smem_u32(smem) & 1023u) {  // the swizzled tiles need 1024-byte alignment (uniform branch)
    if (threadIdx.x == 0) raise_device_error(p.err, kErrDeviceBounds);
    return;
  }
  Misc& bar = *reinterpret_cast<Misc*>(smem + kOffMisc);
  uint32_t& tmem_base_sh = bar.tmem_base;
  int& abort_flag = bar.abort_flag;
  uint32_t& s_mask = bar.mask;
  float* s_lse2 = bar.lse2;
  float* s_D = bar.D;
  const int32_t* row = p.idx + (size_t)blockIdx.x * p.k;  // the token's index row (global)

  const int tok = blockIdx.x;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int k = p.k, Lk = p.Lk;
  if (threadIdx.x == 0) {
    mbar_init(&bar.q_full, 1);
    mbar_init(&bar.k_full, kProducerWarps * 32);
    mbar_init(&bar.v_full, kProducerWarps * 32);
    mbar_init(&bar.k_free, 1);
    mbar_init(&bar.v_free, 1);
    mbar_init(&bar.s_ready, 1);
    mbar_init(&bar.p_ready, 128);
    mbar_init(&bar.dv_ready, 1);
    mbar_init(&bar.dk_ready, 1);
    mbar_init(&bar.kv_read, 128);
    mbar_init(&bar.dq_full, 1);
    abort_flag = 0;
    s_mask = 0;
    fence_mbarrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&tmem_base_sh, 512);
    tmem_relinquish();
  }
  // which 128-entry tiles of the index row hold a valid entry
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  for (int j = warp; j < (k + kKeyTile - 1) / kKeyTile; j += kThreads / 32) {  // k <= 4096: at most 32 tiles
    bool any = false;
    for (int e = j * kKeyTile + lane; e < min(k, (j + 1) * kKeyTile); e += 32) any |= idx_ok(row[e], Lk);
    if (__any_sync(0xffffffffu, any) && lane == 0) atomicOr(&s_mask, 1u << j);
  }
  __syncthreads();
  const uint32_t mask = s_mask;
  const int J = __popc(mask);
  const uint32_t tmem = tmem_base_sh;
  const size_t kv_row0 = (size_t)(tok / p.Lq) * Lk;

  if (warp < kProducerWarps) {
    // ------------------------------------------------------------ producers (cp.async rows)
    const uint32_t sK = smem_u32(smem + kOffK), sV = smem_u32(smem + kOffV);
    const int chunk = lane >> 3, piece = lane & 7;
    const int n_rows_w = (kKeyTile - warp + kProducerWarps - 1) / kProducerWarps;  // 43 or 42
    bool ok = true;
    uint32_t m = mask;
    for (int t = 0; t < J && ok; ++t) {
      const int j = __ffs(m) - 1;
      m &= m - 1;
      // lane l holds the K/V row of the warp's l-th and (32 + l)-th rows
      const int ea = j * kKeyTile + warp + kProducerWarps * lane;
      const int eb = j * kKeyTile + warp + kProducerWarps * (32 + lane);
      const int sa = (lane < n_rows_w && ea < k) ? row[ea] : -1;
      const int sb = (32 + lane < n_rows_w && eb < k) ? row[eb] : -1;
      const int ra = idx_ok(sa, Lk) ? sa : 0, rb = idx_ok(sb, Lk) ? sb : 0;
      for (int part = 0; part < 2 && ok; ++part) {
        if (t > 0) {  // the previous tile's K (after dQ^T) / V space (after dK_g) is free
          ok = __all_sync(0xffffffffu, mbar_wait(part == 0 ? &bar.k_free : &bar.v_free, (t - 1) & 1, &abort_flag,
                                                 p.err));
          if (!ok) break;
        }
        const uint16_t* base = (part == 0 ? p.K : p.V) + kv_row0 * kD + lane * 8;
        const uint32_t dst0 = (part == 0 ? sK : sV) + chunk * kChunkBytes;
#pragma unroll 4
        for (int i = 0; i < n_rows_w; ++i) {
          const int trow = warp + kProducerWarps * i;
          const int src_row = __shfl_sync(0xffffffffu, i < 32 ? ra : rb, i & 31);
          cp_async16(dst0 + trow * 128 + ((piece ^ (trow & 7)) << 4), base + (size_t)src_row * kD);
        }
        cp_async_arrive_noinc(part == 0 ? &bar.k_full : &bar.v_full);
      }
    }
    cp_async_wait_all();
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && J > 0) {
      const uint32_t sQ = smem_u32(smem + kOffQ), sDO = smem_u32(smem + kOffDO);
      const uint32_t sK = smem_u32(smem + kOffK), sV = smem_u32(smem + kOffV);
      const uint32_t sP = sV, sDS = sV + kPBytes;
      mbar_arrive_expect_tx(&bar.q_full, 2 * kQBytes);
      for (int c = 0; c < 4; ++c) {
        tma_load_3d(smem + kOffQ + c * kQChunkBytes, &map_q, &bar.q_full, c * 64, 0, tok);
        tma_load_3d(smem + kOffDO + c * kQChunkBytes, &map_do, &bar.q_full, c * 64, 0, tok);
      }
      const uint32_t idesc_t = idesc_bf16_f32(128, kH, false, false);   // S^T, dP^T
      const uint32_t idesc_kv = idesc_bf16_f32(128, kD, false, true);   // dV_g, dK_g
      const uint32_t idesc_q = idesc_bf16_f32(128, kH, true, true);     // dQ^T
      bool ok = mbar_wait(&bar.q_full, 0, &abort_flag, p.err);
      for (int t = 0; t < J && ok; ++t) {
        ok = mbar_wait(&bar.k_full, t & 1, &abort_flag, p.err) && mbar_wait(&bar.v_full, t & 1, &abort_flag, p.err);
        if (!ok) break;
        fence_proxy_async_smem();  // cp.async (generic proxy) writes -> tensor core reads
        tc_fence_after();
        // S^T = K_g Q^T and dP^T = V_g dO^T over four 64-wide chunks of d
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint32_t acc = (c | kk) != 0;
            mma_ss(tmem + kTmemS, smem_desc_sw128(sK + c * kChunkBytes + kk * 32, 16, 1024),
                   smem_desc_sw128(sQ + c * kQChunkBytes + kk * 32, 16, 1024), idesc_t, acc);
            mma_ss(tmem + kTmemDP, smem_desc_sw128(sV + c * kChunkBytes + kk * 32, 16, 1024),
                   smem_desc_sw128(sDO + c * kQChunkBytes + kk * 32, 16, 1024), idesc_t, acc);
          }
        mma_commit(&bar.s_ready);
        ok = mbar_wait(&bar.p_ready, t & 1, &abort_flag, p.err);
        if (!ok) break;
        tc_fence_after();
        // dV_g = P^T dO (K = 64 heads): A = P^T rows of 64 heads; B = dO as [heads x d], d in
        // four 64-wide groups 8 KB apart.  The region must have been read out (dK_g of t - 1).
        if (t > 0) {
          ok = mbar_wait(&bar.kv_read, 1, &abort_flag, p.err);
          if (!ok) break;
          tc_fence_after();
        }
#pragma unroll
        for (int kk = 0; kk < kH / 16; ++kk)
          mma_ss(tmem + kTmemKV, smem_desc_sw128(sP + kk * 32, 16, 1024),
                 smem_desc_sw128(sDO + kk * 2048, kQChunkBytes, 1024), idesc_kv, kk > 0);
        mma_commit(&bar.dv_ready);
        // dQ^T += K_g^T dS^T: d in two halves of 128 rows (K chunks 2hv, 2hv+1), keys as K; the
        // K tile is free once these are done
#pragma unroll
        for (int hv = 0; hv < 2; ++hv)
#pragma unroll
          for (int kk = 0; kk < kKeyTile / 16; ++kk)
            mma_ss(tmem + kTmemDQ + hv * kH, smem_desc_sw128(sK + hv * 2 * kChunkBytes + kk * 2048, kChunkBytes, 1024),
                   smem_desc_sw128(sDS + kk * 2048, kPBytes, 1024), idesc_q, (t > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&bar.k_free);
        ok = mbar_wait(&bar.kv_read, 0, &abort_flag, p.err);  // dV_g read out
        if (!ok) break;
        tc_fence_after();
        // dK_g = dS^T Q (the scale is applied when it is added to dK); then the V space is free
#pragma unroll
        for (int kk = 0; kk < kH / 16; ++kk)
          mma_ss(tmem + kTmemKV, smem_desc_sw128(sDS + kk * 32, 16, 1024),
                 smem_desc_sw128(sQ + kk * 2048, kQChunkBytes, 1024), idesc_kv, kk > 0);
        mma_commit(&bar.dk_ready);
        mma_commit(&bar.v_free);
        if (t == J - 1) mma_commit(&bar.dq_full);
      }
    }
  } else if (warp < kRedWarp0) {
    // ------------------------------------------------------------ softmax warps (thread = key)
    const int quarter = warp & 3;
    const int kl = quarter * 32 + lane;  // key of a tile == TMEM lane; d row of dQ^T
    const int tid = (warp - kSoftWarp0) * 32 + lane;  // 0..127
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    // D[h] = <dO[h], O[h]> and lse in log2 units; two threads per head, 128 columns each
    {
      const int h = tid >> 1, half = tid & 1;
      const uint4* o4 = reinterpret_cast<const uint4*>(p.O + ((size_t)tok * kH + h) * kD + half * 128);
      const uint4* g4 = reinterpret_cast<const uint4*>(p.dO + ((size_t)tok * kH + h) * kD + half * 128);
      float acc = 0.0f;
#pragma unroll 4
      for (int i = 0; i < 16; ++i) {
        const uint4 a = o4[i], b = g4[i];
        const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          acc = fmaf(__uint_as_float(aw[q] << 16), __uint_as_float(bw[q] << 16), acc);
          acc = fmaf(__uint_as_float(aw[q] & 0xFFFF0000u), __uint_as_float(bw[q] & 0xFFFF0000u), acc);
        }
      }
      acc += __shfl_xor_sync(0xffffffffu, acc, 1);
      if (half == 0) {
        s_D[h] = acc;
        s_lse2[h] = p.lse[(size_t)tok * kH + h] * 1.4426950408889634f;
      }
    }
    asm volatile("bar.sync 1, 128;" ::: "memory");
    bool ok = true;
    uint8_t* sP = smem + kOffV;
    uint8_t* sDS = smem + kOffV + kPBytes;
    uint32_t m = mask;
    for (int t = 0; t < J; ++t) {
      const int j = __ffs(m) - 1;
      m &= m - 1;
      const int e = j * kKeyTile + kl;
      const int s_idx = e < k ? row[e] : -1;
      const bool valid = idx_ok(s_idx, Lk);
      if (s_idx >= Lk) raise_device_error(p.err, kErrDeviceBounds);
      ok = mbar_wait(&bar.s_ready, t & 1, &abort_flag, p.err) && ok;
      tc_fence_after();
      uint32_t sv[64], dv[64];
      {
        uint32_t (&s0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sv[0]);
        uint32_t (&s1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sv[32]);
        uint32_t (&d0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&dv[0]);
        uint32_t (&d1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&dv[32]);
        tmem_ld32_nowait(tmem + lane_off + kTmemS, s0);
        tmem_ld32_nowait(tmem + lane_off + kTmemS + 32, s1);
        tmem_ld32_nowait(tmem + lane_off + kTmemDP, d0);
        tmem_ld32_nowait(tmem + lane_off + kTmemDP + 32, d1);
        tmem_wait_ld_regs2(s0, s1);
        tmem_wait_ld_regs2(d0, d1);
      }
      // P^T and dS^T rows of this key (64 heads, bf16), 128B-swizzled like a K-major tile row
      uint8_t* prow = sP + kl * 128;
      uint8_t* drow = sDS + kl * 128;
#pragma unroll
      for (int c8 = 0; c8 < 8; ++c8) {
        uint32_t pw[4], dw[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int h = c8 * 8 + 2 * q;
          float p0 = 0.0f, p1 = 0.0f;
          if (valid) {
            p0 = fast_exp2(fmaf(__uint_as_float(sv[h]), p.scale_log2, -s_lse2[h]));
            p1 = fast_exp2(fmaf(__uint_as_float(sv[h + 1]), p.scale_log2, -s_lse2[h + 1]));
          }
          pw[q] = pack_bf16x2(p0, p1);
          dw[q] = pack_bf16x2(p0 * (__uint_as_float(dv[h]) - s_D[h]), p1 * (__uint_as_float(dv[h + 1]) - s_D[h + 1]));
        }
        const int off = (c8 ^ (kl & 7)) << 4;
        *reinterpret_cast<uint4*>(prow + off) = make_uint4(pw[0], pw[1], pw[2], pw[3]);
        *reinterpret_cast<uint4*>(drow + off) = make_uint4(dw[0], dw[1], dw[2], dw[3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&bar.p_ready);
    }
    // dQ[h, d] = scale * dQ^T[d, h]: this thread's d rows kl and 128 + kl
    float* dq = p.dQ + (size_t)tok * kH * kD;
    if (J > 0) {
      ok = mbar_wait(&bar.dq_full, 0, &abort_flag, p.err) && ok;
      tc_fence_after();
    }
#pragma unroll 1
    for (int hv = 0; hv < 2; ++hv) {
      uint32_t v0[32], v1[32];
      if (J > 0) {
        tmem_ld32_nowait(tmem + lane_off + kTmemDQ + hv * kH, v0);
        tmem_ld32_nowait(tmem + lane_off + kTmemDQ + hv * kH + 32, v1);
        tmem_wait_ld_regs2(v0, v1);
      }
#pragma unroll
      for (int h = 0; h < kH; ++h) {
        const float x = J > 0 ? __uint_as_float(h < 32 ? v0[h] : v1[h - 32]) * p.scale : 0.0f;
        dq[(size_t)h * kD + hv * 128 + kl] = x;
      }
    }
  } else {
    // ------------------------------------------------------------ reduction warps (thread = key)
    // dV_g, then dK_g: this key's 256 values added to dV[s] / dK[s], 64 columns per bulk
    // reduction through the thread's staging row, while the softmax warps and the tensor cores
    // go on with the next tile
    const int quarter = warp & 3;
    const int kl = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    uint8_t* stage_row = smem + kOffStage + kl * kStageStride;
    bool ok = true;
    uint32_t m = mask;
    for (int t = 0; t < J; ++t) {
      const int j = __ffs(m) - 1;
      m &= m - 1;
      const int e = j * kKeyTile + kl;
      const int s_idx = e < k ? row[e] : -1;
      const bool valid = idx_ok(s_idx, Lk);
      for (int which = 0; which < 2; ++which) {
        ok = mbar_wait(which == 0 ? &bar.dv_ready : &bar.dk_ready, t & 1, &abort_flag, p.err) && ok;
        tc_fence_after();
        float* dst = (which == 0 ? p.dV : p.dK) + (kv_row0 + (size_t)(valid ? s_idx : 0)) * kD;
        const float f = which == 0 ? 1.0f : p.scale;
#pragma unroll 1
        for (int c0 = 0; c0 < kD; c0 += kStageCols) {
          uint32_t v0[32], v1[32];
          tmem_ld32_nowait(tmem + lane_off + kTmemKV + c0, v0);
          tmem_ld32_nowait(tmem + lane_off + kTmemKV + c0 + 32, v1);
          tmem_wait_ld_regs2(v0, v1);
          if (c0 + kStageCols == kD) {  // the region may be rewritten once every thread has read it
            tc_fence_before();
            mbar_arrive(&bar.kv_read);
          }
          if (valid) {
            bulk_wait_group_read0();  // this thread's previous reduction has read the row
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              *reinterpret_cast<float4*>(stage_row + 16 * i) =
                  make_float4(f * __uint_as_float(v0[4 * i]), f * __uint_as_float(v0[4 * i + 1]),
                              f * __uint_as_float(v0[4 * i + 2]), f * __uint_as_float(v0[4 * i + 3]));
              *reinterpret_cast<float4*>(stage_row + 128 + 16 * i) =
                  make_float4(f * __uint_as_float(v1[4 * i]), f * __uint_as_float(v1[4 * i + 1]),
                              f * __uint_as_float(v1[4 * i + 2]), f * __uint_as_float(v1[4 * i + 3]));
            }
            fence_proxy_async_smem();
            bulk_reduce_add_f32(dst + c0, smem_u32(stage_row), kStageCols * 4);
            bulk_commit_group();
          }
        }
      }
    }
    bulk_wait_group0();  // every reduction of this thread has completed
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) tmem_dealloc(tmem, 512);
}

}  // namespace
}  // namespace hcadsa

extern "C" hcadsa_status dsa_sparse_attn_bwd(const hcadsa_bf16* Q, const hcadsa_bf16* K, const hcadsa_bf16* V,
                                             const int32_t* idx, const hcadsa_bf16* O, const hcadsa_bf16* dO,
                                             const float* lse, float* dQ, float* dK, float* dV, int B, int Lq, int Lk,
                                             int Hq, int d, int k, float scale, hcadsa_stream stream) {
  using namespace hcadsa;
  if (!Q || !K || !V || !idx || !O || !dO || !lse || !dQ || !dK || !dV) return HCADSA_ERR_NULL;
  if (B < 0 || Lq < 0 || Lk < 0 || k <= 0) return HCADSA_ERR_SHAPE;
  if (d != kD || Hq != kH || k > kMaxK) return HCADSA_ERR_UNSUPPORTED;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(idx) || !aligned16(O) || !aligned16(dO) ||
      !aligned16(dQ) || !aligned16(dK) || !aligned16(dV) || (reinterpret_cast<uintptr_t>(lse) & 3u))
    return HCADSA_ERR_ALIGN;
  if (B == 0 || Lq == 0) return HCADSA_OK;
  if ((long long)B * Lq > 2147483647LL || (long long)B * Lk > 2147483647LL) return HCADSA_ERR_UNSUPPORTED;
  CUtensorMap mq, mdo;
  {
    const uint64_t dims[3] = {(uint64_t)kD, (uint64_t)kH, (uint64_t)B * Lq};
    const uint64_t strides[2] = {(uint64_t)kD * 2, (uint64_t)kH * kD * 2};
    const uint32_t box[3] = {64, (uint32_t)kH, 1};
    if (!encode_tmap_bf16(&mq, 3, const_cast<hcadsa_bf16*>(Q), dims, strides, box, true) ||
        !encode_tmap_bf16(&mdo, 3, const_cast<hcadsa_bf16*>(dO), dims, strides, box, true))
      return HCADSA_ERR_CUDA;
  }
  Params p;
  p.K = K;
  p.V = V;
  p.O = O;
  p.dO = dO;
  p.lse = lse;
  p.idx = idx;
  p.dQ = dQ;
  p.dK = dK;
  p.dV = dV;
  p.err = device_error_ptr();
  p.Lq = Lq;
  p.Lk = Lk;
  p.k = k;
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  if (cudaFuncSetAttribute(dsa_attn_bwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) !=
      cudaSuccess)
    return launch_status();
  dsa_attn_bwd_kernel<<<(unsigned)(B * Lq), kThreads, kSmemBytes, as_stream(stream)>>>(mq, mdo, p);
  return launch_status();
}
