// dsa_attn.cu -- DSA sparse attention forward on sm_100a (tcgen05 + TMEM).
//
// Method: the mirrorspeed page, section "Hybrid sparse attention, 1/7 full context
// access": in the MLA layers "the core attention is computed only on the top-k
// positions with the highest scores"; MLA heads are 256 wide (ai-club.cn page,
// section "混合注意力（MLA + HCA）").  All 64 query heads of a token share one K/V
// head (the MLA latent reading) and the token's index row.
//
// Kernel design (one CTA per query token):
//   * The 64 heads of a token are too few rows for a full-rate M=128 tcgen05 tile, so
//     the contraction is transposed: the 128 gathered keys of a tile are M.
//       S^T[key, head]  = K_g (A, K-major, 128 x 256)  *  Q^T (B, K-major, 64 heads)
//       O^T[dv, head]  += V_g^T (A, MN-major, 2 x 128 dv) * P^T (B, MN-major, 64 heads)
//     TMEM: O^T halves [0,64), [64,128); S^T double buffer [128,192), [192,256).
//   * Producer warps (one thread per key row) gather K and V rows with cp.async into
//     128B-swizzled 16 KB chunks of an 8-slot ring; the MMA warp consumes K_0, K_1, V_0,
//     K_2, V_1, ... in exactly the order they were loaded.
//   * Softmax warps: one thread per key (TMEM lane) holding its 64 head scores; per-head
//     maxima come from a warp reduce-scatter (62 shuffles) plus a 4-warp combine in shared
//     memory; lazy rescale (reference max moves only when exceeded by 2^8); P^T rows are
//     written to shared memory as bf16 and handed to the tensor core after a proxy fence.
//     Row sums are kept per thread and reduced once at the end.
#include <cuda_bf16.h>

#include "host_common.h"
#include "ptx.cuh"

namespace hcadsa {
namespace {

constexpr int kD = 256;
constexpr int kH = 64;
constexpr int kKeyTile = 128;
constexpr int kChunkBytes = 128 * 128;     // 128 rows x 64 bf16
constexpr int kRingSlots = 8;
constexpr int kQChunkBytes = kH * 128;     // 64 heads x 64 bf16
constexpr int kQBytes = 4 * kQChunkBytes;  // 32 KB
constexpr int kPBytes = kKeyTile * 128;    // 128 keys x 64 heads bf16
constexpr int kMaxK = 4096;
constexpr int kSmemBytes = kQBytes + kRingSlots * kChunkBytes + 2 * kPBytes + 1024;
constexpr int kProducerWarps = 4;
constexpr int kSoftmaxWarps = 4;
constexpr int kThreads = 32 * (kProducerWarps + 1 + kSoftmaxWarps);  // 288
constexpr int kMmaWarp = kProducerWarps;                            // warp 4
constexpr int kSoftmaxWarp0 = kProducerWarps + 1;                   // warps 5..8
constexpr float kLazyRescale = 8.0f;
constexpr int kInFlight = 3;  // cp.async groups a producer thread keeps in flight

struct Params {
  const uint16_t* K;
  const uint16_t* V;
  const int32_t* idx;
  uint16_t* O;
  float* lse;
  int* err;
  int Lq, Lk, k;
  float scale_log2;
};

struct __align__(8) Barriers {
  uint64_t q_full;
  uint64_t full[kRingSlots];
  uint64_t empty[kRingSlots];
  uint64_t s_full[2];
  uint64_t p_ready[2];
  uint64_t pv_done;
  uint64_t o_full;  // one-shot: every PV of the work item has completed
};

struct SoftShared {
  float wred[kSoftmaxWarps][kH];
  float m_ref[kH];
  float alpha[kH];
  float l_tot[kH];
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void softmax_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// Warp reduce-scatter of 64 per-lane values: afterwards lane l holds, in v[0] and v[1],
// the reduction over all 32 lanes of heads 2l and 2l+1.
template <bool kMax, int W>
__device__ __forceinline__ void reduce_scatter_stage(float (&v)[64], int lane) {
  constexpr int o = W / 4;  // lane offset: 16, 8, 4, 2, 1 for W = 64 .. 4
  const bool upper = (lane & o) != 0;
#pragma unroll
  for (int i = 0; i < W / 2; ++i) {
    const float send = upper ? v[i] : v[i + W / 2];
    const float keep = upper ? v[i + W / 2] : v[i];
    const float recv = __shfl_xor_sync(0xffffffffu, send, o);
    v[i] = kMax ? fmaxf(keep, recv) : keep + recv;
  }
}
template <bool kMax>
__device__ __forceinline__ void warp_reduce_scatter64(float (&v)[64], int lane) {
  reduce_scatter_stage<kMax, 64>(v, lane);
  reduce_scatter_stage<kMax, 32>(v, lane);
  reduce_scatter_stage<kMax, 16>(v, lane);
  reduce_scatter_stage<kMax, 8>(v, lane);
  reduce_scatter_stage<kMax, 4>(v, lane);
}

__global__ void __launch_bounds__(kThreads, 1)
    dsa_attn_kernel(const __grid_constant__ CUtensorMap map_q, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sRing = smem + kQBytes;
  uint8_t* sP = sRing + kRingSlots * kChunkBytes;
  __shared__ Barriers bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;
  __shared__ int s_idx[kMaxK];
  __shared__ int s_nvalid;
  __shared__ int s_wcount[kThreads / 32];
  __shared__ SoftShared ss;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int row = blockIdx.x;  // flat b * Lq + r
  const int b = row / p.Lq;

  // ---- stable compaction of the valid index entries (all threads)
  {
    const int32_t* irow = p.idx + (size_t)row * p.k;
    const int per = (p.k + kThreads - 1) / kThreads;
    const int i0 = threadIdx.x * per;
    int cnt = 0;
    for (int i = i0; i < min(i0 + per, p.k); ++i) {
      const int s = irow[i];
      if (s >= p.Lk) raise_device_error(p.err, kErrDeviceBounds);
      cnt += (s >= 0 && s < p.Lk);
    }
    int x = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) s_wcount[warp] = x;
    __syncthreads();
    int before = 0;
    for (int w = 0; w < warp; ++w) before += s_wcount[w];
    int pos = before + x - cnt;
    for (int i = i0; i < min(i0 + per, p.k); ++i) {
      const int s = irow[i];
      if (s >= 0 && s < p.Lk) s_idx[pos++] = s;
    }
    if (threadIdx.x == kThreads - 1) s_nvalid = before + x;
  }
  if (threadIdx.x == 0) {
    mbar_init(&bar.q_full, 1);
    for (int s = 0; s < kRingSlots; ++s) {
      mbar_init(&bar.full[s], kProducerWarps * 32);
      mbar_init(&bar.empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar.s_full[s], 1);
      mbar_init(&bar.p_ready[s], kSoftmaxWarps * 32);
    }
    mbar_init(&bar.pv_done, 1);
    mbar_init(&bar.o_full, 1);
    abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&tmem_base_sh, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  const int n_valid = s_nvalid;
  const int J = (n_valid + kKeyTile - 1) / kKeyTile;

  if (warp < kProducerWarps) {
    // ------------------------------------------------------------ gather producers
    const int i = threadIdx.x;  // key row within a tile
    if (i == 0 && J > 0) {
      mbar_arrive_expect_tx(&bar.q_full, kQBytes);
      for (int c = 0; c < 4; ++c) tma_load_3d(sQ + c * kQChunkBytes, &map_q, &bar.q_full, c * 64, 0, row);
    }
    const uint16_t* Kb = p.K + (size_t)b * p.Lk * kD;
    const uint16_t* Vb = p.V + (size_t)b * p.Lk * kD;
    const uint32_t ring = smem_u32(sRing);
    int slot = 0;
    int pending_slot[kInFlight + 1] = {};  // FIFO of slots whose copies are not yet signalled
    uint32_t phase = 0;
    int n_pending = 0, pending_head = 0;
    bool ok = true;
    auto issue_chunk = [&](const uint16_t* base, int tile, int c) {
      const int key = tile * kKeyTile + i;
      const bool valid = key < n_valid;
      const uint16_t* src = base + (size_t)(valid ? s_idx[key] : 0) * kD + c * 64;
      const uint32_t dst = ring + slot * kChunkBytes + i * 128;
#pragma unroll
      for (int piece = 0; piece < 8; ++piece)
        cp_async16(dst + ((piece ^ (i & 7)) << 4), src + piece * 8, valid);
      cp_async_commit();
    };
    auto retire_oldest = [&]() {
      fence_proxy_async_smem();
      mbar_arrive(&bar.full[pending_slot[pending_head]]);
      pending_head = (pending_head + 1) % (kInFlight + 1);
      --n_pending;
    };
    for (int step = 0; step <= J && ok; ++step) {
      for (int part = 0; part < 2 && ok; ++part) {
        // part 0: K chunks of tile `step`; part 1: V chunks of tile `step - 1`
        const int tile = part == 0 ? step : step - 1;
        if (tile < 0 || tile >= J) continue;
        for (int c = 0; c < 4; ++c) {
          ok = mbar_wait(&bar.empty[slot], phase ^ 1, &abort_flag, p.err);
          if (!ok) break;
          issue_chunk(part == 0 ? Kb : Vb, tile, c);
          pending_slot[(pending_head + n_pending) % (kInFlight + 1)] = slot;
          ++n_pending;
          if (n_pending > kInFlight) {
            cp_async_wait<kInFlight>();
            retire_oldest();
          }
          if (++slot == kRingSlots) { slot = 0; phase ^= 1; }
        }
      }
    }
    cp_async_wait<0>();
    while (n_pending > 0) retire_oldest();
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && J > 0) {
      bool ok = mbar_wait(&bar.q_full, 0, &abort_flag, p.err);
      tc_fence_after();
      int slot = 0;
      uint32_t phase = 0;
      const uint32_t sQa = smem_u32(sQ), sRa = smem_u32(sRing), sPa = smem_u32(sP);
      const uint32_t idesc_s = idesc_bf16_f32(128, kH, false, false);
      const uint32_t idesc_o = idesc_bf16_f32(128, kH, true, true);
      for (int step = 0; ok && step <= J; ++step) {
        if (step < J) {
          const uint32_t tS = tmem + 128 + (step & 1) * kH;
          for (int c = 0; c < 4 && ok; ++c) {
            ok = mbar_wait(&bar.full[slot], phase, &abort_flag, p.err);
            if (!ok) break;
            tc_fence_after();
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const uint64_t da = smem_desc_sw128(sRa + slot * kChunkBytes + k * 32, 16, 1024);
              const uint64_t db = smem_desc_sw128(sQa + c * kQChunkBytes + k * 32, 16, 1024);
              mma_ss(tS, da, db, idesc_s, (c | k) != 0);
            }
            mma_commit(&bar.empty[slot]);
            if (++slot == kRingSlots) { slot = 0; phase ^= 1; }
          }
          if (!ok) break;
          mma_commit(&bar.s_full[step & 1]);
        }
        if (step >= 1) {
          const int j = step - 1;
          ok = mbar_wait(&bar.p_ready[j & 1], (j >> 1) & 1, &abort_flag, p.err);
          if (!ok) break;
          tc_fence_after();
          const uint32_t pbase = sPa + (j & 1) * kPBytes;
          for (int hv = 0; hv < 2 && ok; ++hv) {
            // V chunks 2hv, 2hv+1 sit in consecutive slots (slot is even here)
            ok = mbar_wait(&bar.full[slot], phase, &abort_flag, p.err) &&
                 mbar_wait(&bar.full[slot + 1], phase, &abort_flag, p.err);
            if (!ok) break;
            tc_fence_after();
            for (int kk = 0; kk < kKeyTile / 16; ++kk) {
              const uint64_t da = smem_desc_sw128(sRa + slot * kChunkBytes + kk * 2048, kChunkBytes, 1024);
              const uint64_t db = smem_desc_sw128(pbase + kk * 2048, kPBytes, 1024);
              mma_ss(tmem + hv * kH, da, db, idesc_o, (j > 0 || kk > 0) ? 1u : 0u);
            }
            mma_commit(&bar.empty[slot]);
            mma_commit(&bar.empty[slot + 1]);
            slot += 2;
            if (slot == kRingSlots) { slot = 0; phase ^= 1; }
          }
          if (!ok) break;
          mma_commit(&bar.pv_done);
          if (j == J - 1) mma_commit(&bar.o_full);
        }
      }
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int sw = warp - kSoftmaxWarp0;  // 0..3
    const int quarter = warp & 3;         // TMEM lane quarter this warp may access
    const int key_lane = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const int tid = sw * 32 + lane;       // 0..127
    float lpart[kH];
#pragma unroll
    for (int h = 0; h < kH; ++h) lpart[h] = 0.0f;
    if (tid < kH) ss.m_ref[tid] = -INFINITY;
    softmax_bar();
    bool ok = true;
    // No early exit in this loop: the four softmax warps meet at named barriers, so after an
    // abort every thread keeps walking the same barrier sequence (waits then fail fast).
    for (int j = 0; j < J; ++j) {
      ok = mbar_wait(&bar.s_full[j & 1], (j >> 1) & 1, &abort_flag, p.err) && ok;
      tc_fence_after();
      const bool valid = j * kKeyTile + key_lane < n_valid;
      const uint32_t tS = tmem + lane_off + 128 + (j & 1) * kH;
      float red[kH];
      {
        uint32_t u[32];
        tmem_ld32(tS, u);
        tmem_wait_ld();
#pragma unroll
        for (int h = 0; h < 32; ++h) red[h] = valid ? __uint_as_float(u[h]) * p.scale_log2 : -INFINITY;
        tmem_ld32(tS + 32, u);
        tmem_wait_ld();
#pragma unroll
        for (int h = 0; h < 32; ++h) red[32 + h] = valid ? __uint_as_float(u[h]) * p.scale_log2 : -INFINITY;
      }
      warp_reduce_scatter64<true>(red, lane);
      ss.wred[sw][2 * lane] = red[0];
      ss.wred[sw][2 * lane + 1] = red[1];
      softmax_bar();
      if (tid < kH) {
        const float mt = fmaxf(fmaxf(ss.wred[0][tid], ss.wred[1][tid]), fmaxf(ss.wred[2][tid], ss.wred[3][tid]));
        const float mo = ss.m_ref[tid];
        float alpha = 1.0f, mn = mo;
        if (mo == -INFINITY) {
          mn = mt;
        } else if (mt > mo + kLazyRescale) {
          mn = mt;
          alpha = fast_exp2(mo - mt);
        }
        ss.m_ref[tid] = mn;
        ss.alpha[tid] = alpha;
      }
      softmax_bar();
      bool rescale = false;
#pragma unroll 8
      for (int h = 0; h < kH; ++h) rescale |= ss.alpha[h] != 1.0f;
      if (rescale) {
        // O^T must hold every PV up to tile j-1 before it is rescaled
        ok = mbar_wait(&bar.pv_done, (j - 1) & 1, &abort_flag, p.err) && ok;
        tc_fence_after();
#pragma unroll
        for (int hv = 0; hv < 2; ++hv) {
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            uint32_t u[32];
            const uint32_t tO = tmem + lane_off + hv * kH + c * 32;
            tmem_ld32(tO, u);
            tmem_wait_ld();
#pragma unroll
            for (int h = 0; h < 32; ++h) u[h] = __float_as_uint(__uint_as_float(u[h]) * ss.alpha[c * 32 + h]);
            tmem_st32(tO, u);
          }
        }
        tmem_wait_st();
#pragma unroll
        for (int h = 0; h < kH; ++h) lpart[h] *= ss.alpha[h];
      }
      // P^T row of this key: 64 heads, bf16, 128B-swizzled (scores re-read from TMEM)
      uint8_t* prow = sP + (j & 1) * kPBytes + key_lane * 128;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t u[32];
        tmem_ld32(tS + hh * 32, u);
        tmem_wait_ld();
#pragma unroll
        for (int c8 = 0; c8 < 4; ++c8) {
          uint32_t w4[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int hl = c8 * 8 + 2 * q, h = hh * 32 + hl;
            float p0 = 0.0f, p1 = 0.0f;
            if (valid) {
              p0 = fast_exp2(__uint_as_float(u[hl]) * p.scale_log2 - ss.m_ref[h]);
              p1 = fast_exp2(__uint_as_float(u[hl + 1]) * p.scale_log2 - ss.m_ref[h + 1]);
            }
            lpart[h] += p0;
            lpart[h + 1] += p1;
            w4[q] = pack_bf16x2(p0, p1);
          }
          const int chunk = hh * 4 + c8;
          *reinterpret_cast<uint4*>(prow + ((chunk ^ (key_lane & 7)) << 4)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&bar.p_ready[j & 1]);
    }
    // ---- final: row sums, normalisation, store
    // pv_done may be two phases behind here, so its parity cannot be trusted: use o_full
    if (ok && J > 0) ok = mbar_wait(&bar.o_full, 0, &abort_flag, p.err);
    warp_reduce_scatter64<false>(lpart, lane);
    ss.wred[sw][2 * lane] = lpart[0];
    ss.wred[sw][2 * lane + 1] = lpart[1];
    softmax_bar();
    if (tid < kH) ss.l_tot[tid] = ss.wred[0][tid] + ss.wred[1][tid] + ss.wred[2][tid] + ss.wred[3][tid];
    softmax_bar();
    if (ok) {
      tc_fence_after();
      uint16_t* obase = p.O + (size_t)row * kH * kD;
#pragma unroll
      for (int hv = 0; hv < 2; ++hv) {
        const int dv = hv * 128 + key_lane;  // this lane's d_v row of O^T
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t u[32];
          if (J > 0) {
            tmem_ld32(tmem + lane_off + hv * kH + c * 32, u);
            tmem_wait_ld();
          }
#pragma unroll
          for (int h = 0; h < 32; ++h) {
            const float l = ss.l_tot[c * 32 + h];
            const float o = (J > 0 && l > 0.0f) ? __uint_as_float(u[h]) / l : 0.0f;
            reinterpret_cast<__nv_bfloat16*>(obase)[(size_t)(c * 32 + h) * kD + dv] = __float2bfloat16_rn(o);
          }
        }
      }
      if (p.lse && tid < kH) {
        const float l = ss.l_tot[tid];
        p.lse[(size_t)row * kH + tid] = l > 0.0f ? (ss.m_ref[tid] + __log2f(l)) * 0.69314718055994531f : -INFINITY;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) tmem_dealloc(tmem, 256);
}

}  // namespace
}  // namespace hcadsa

extern "C" hcadsa_status dsa_sparse_attn_fwd(const hcadsa_bf16* Q, const hcadsa_bf16* K, const hcadsa_bf16* V,
                                             const int32_t* idx, hcadsa_bf16* O, float* lse, int B, int Lq, int Lk,
                                             int Hq, int d, int k, float scale, hcadsa_stream stream) {
  using namespace hcadsa;
  if (!Q || !K || !V || !idx || !O) return HCADSA_ERR_NULL;
  if (B < 0 || Lq < 0 || Lk < 0 || k <= 0) return HCADSA_ERR_SHAPE;
  if (d != kD || Hq != kH || k > kMaxK) return HCADSA_ERR_UNSUPPORTED;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(idx) ||
      (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)))
    return HCADSA_ERR_ALIGN;
  if (B == 0 || Lq == 0) return HCADSA_OK;
  if ((long long)B * Lq > 2147483647LL) return HCADSA_ERR_UNSUPPORTED;
  CUtensorMap mq;
  const uint64_t dims[3] = {(uint64_t)kD, (uint64_t)kH, (uint64_t)B * Lq};
  const uint64_t strides[2] = {(uint64_t)kD * 2, (uint64_t)kH * kD * 2};
  const uint32_t box[3] = {64, (uint32_t)kH, 1};
  if (!encode_tmap_bf16(&mq, 3, const_cast<hcadsa_bf16*>(Q), dims, strides, box, true)) return HCADSA_ERR_CUDA;
  Params p;
  p.K = K;
  p.V = V;
  p.idx = idx;
  p.O = O;
  p.lse = lse;
  p.err = device_error_ptr();
  p.Lq = Lq;
  p.Lk = Lk;
  p.k = k;
  p.scale_log2 = scale * 1.4426950408889634f;
  if (cudaFuncSetAttribute(dsa_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) != cudaSuccess)
    return HCADSA_ERR_CUDA;
  dsa_attn_kernel<<<(unsigned)(B * Lq), kThreads, kSmemBytes, as_stream(stream)>>>(mq, p);
  return launch_status();
}
