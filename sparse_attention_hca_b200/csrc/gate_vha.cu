// gate_vha.cu -- the attention output's low-rank gate and virtual-head mix, fused into one
// tcgen05 GEMM with its epilogue (sm_100a: TMA, tcgen05.mma kind::f16, TMEM).
//
// Method: the mirrorspeed page, section "Hybrid sparse attention, 1/7 full context access"
// (last paragraph), and the besthub page, "Core Architectural Innovations": the output gate is
// computed from the layer's own low-rank query latent (a quarter of the hidden width), and
// virtual head attention (VHA) mixes the heads with a light low-rank term beside an identity
// path, folded into the attention operator at inference.  This library's reading:
//     Ohat[t,h,c] = O[t,h,c] + sum_m U[h,m] sum_h' V[h',m] O[t,h',c]     (per token and channel)
//     Y[t,h,c]    = sigmoid(sum_i cq[t,i] Wg[h*dv + c, i]) * Ohat[t,h,c]
//
// Design: the gate logits are a GEMM (M = tokens, N = H * dv, K = rq), so the kernel is a
// tcgen05 GEMM whose epilogue does the rest.  Its N tile is chosen so that the epilogue needs
// no data from other threads: 256 columns = all H heads x cw = 256 / H channels of one channel
// block, so the thread that owns token t (TMEM lane t) holds every head of those channels and
// mixes them in registers.
//   * A = cq tile (128 tokens x 64 of K per stage, TMA, SW128); B = the 256 rows (h, c) of Wg
//     for the channel block (a 3D TMA box {64, cw, H} over Wg viewed as [H][dv][rq], SW128).
//   * Warp 0: TMA producer (4 stages of 48 KB); warp 1: TMEM allocation + the MMA thread
//     (4 MMAs of M = 128, N = 256, K = 16 per stage, fp32 accumulator of 256 TMEM columns,
//     double-buffered across tiles); warps 2-9: epilogue, two threads per token (each half of the
//     channel block, every head; its O values loaded at once and kept in registers): the rank-r
//     projections sum_h V[h,m] O[t,h,c] of its channels, then per head the mix, the sigmoid of
//     the logit from TMEM and the bf16 store of Y.
//   * Persistent CTAs walk the tiles (token tile, channel block); consecutive CTAs share the
//     token tile, so the cq tile and Wg stay in L2.
#include <cuda_bf16.h>

#include <mutex>

#include "host_common.h"
#include "ptx.cuh"

namespace hcadsa {
namespace {

constexpr int kM = 128;      // tokens per tile
constexpr int kN = 256;      // gate columns per tile (H heads x cw channels)
constexpr int kKStep = 64;   // K per stage (one 128-byte swizzle row of bf16)
constexpr int kStages = 4;
constexpr int kABytes = kM * kKStep * 2;  // 16 KB
constexpr int kBBytes = kN * kKStep * 2;  // 32 KB
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kMaxR = 4;     // rank of the head mix
constexpr int kMaxH = 64;
constexpr int kSmemBytes = kStages * kStageBytes + 1024;
constexpr int kEpiWarps = 8;  // two per TMEM lane quarter: each takes half of the tile's channels
constexpr int kThreads = 64 + 32 * kEpiWarps;

struct Params {
  const uint16_t* O;
  const float* U;
  const float* V;
  uint16_t* Y;
  int* err;
  int rows, H, dv, rq, r, cw, n_blocks, n_tiles;
};

struct __align__(8) Barriers {
  uint64_t full[kStages], empty[kStages];
  uint64_t tfull[2], tempty[2];
};

// sigmoid(z) = (1 + tanh(z / 2)) / 2: one hardware tanh (tanh.approx.f32, relative error about
// 2^-11) instead of an exponential and a reciprocal; the absolute error, below 2.5e-4, is under
// the bf16 rounding of the output
__device__ __forceinline__ float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float sigmoidf(float z) { return fmaf(0.5f, tanh_approx(0.5f * z), 0.5f); }

// n bf16 (n = 8, 4 or 2) <-> packed words
template <int N>
__device__ __forceinline__ void load_packed(const uint16_t* p, uint32_t (&w)[N / 2]) {
  if constexpr (N == 8) {
    const uint4 a = *reinterpret_cast<const uint4*>(p);
    w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
  } else if constexpr (N == 4) {
    const uint2 a = *reinterpret_cast<const uint2*>(p);
    w[0] = a.x; w[1] = a.y;
  } else {
    w[0] = *reinterpret_cast<const uint32_t*>(p);
  }
}
template <int N>
__device__ __forceinline__ void store_packed(uint16_t* p, const uint32_t (&w)[N / 2]) {
  if constexpr (N == 8) {
    *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
  } else if constexpr (N == 4) {
    *reinterpret_cast<uint2*>(p) = make_uint2(w[0], w[1]);
  } else {
    *reinterpret_cast<uint32_t*>(p) = w[0];
  }
}
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

template <int CW>
// 10 warps put three on two of the four SM sub-partitions (16K registers each): at most 168
// registers per thread, which __launch_bounds__ makes the compiler respect
__global__ void __launch_bounds__(kThreads, 1)
    gate_vha_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                    const Params p) {
  constexpr int H = kN / CW;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ Barriers bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;
  __shared__ float sU[kMaxH * kMaxR], sV[kMaxH * kMaxR];

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  for (int i = threadIdx.x; i < H * p.r; i += kThreads) {
    sU[i] = p.U[i];
    sV[i] = p.V[i];
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bar.full[s], 1);
      mbar_init(&bar.empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar.tfull[s], 1);
      mbar_init(&bar.tempty[s], 32 * kEpiWarps);
    }
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
  const int k_steps = p.rq / kKStep;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&map_a);
      tma_prefetch_desc(&map_b);
      uint32_t g = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < p.n_tiles; t += gridDim.x) {
        const int m = t / p.n_blocks, nb = t % p.n_blocks;
        for (int ks = 0; ok && ks < k_steps; ++ks, ++g) {
          const uint32_t st = g % kStages;
          ok = mbar_wait(&bar.empty[st], ((g / kStages) & 1) ^ 1, &abort_flag, p.err);
          if (!ok) break;
          uint8_t* sa = smem + st * kStageBytes;
          mbar_arrive_expect_tx(&bar.full[st], kStageBytes);
          tma_load_2d(sa, &map_a, &bar.full[st], ks * kKStep, m * kM);
          tma_load_3d(sa + kABytes, &map_b, &bar.full[st], ks * kKStep, nb * CW, 0);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kM, kN, false, false);
      uint32_t g = 0, tl = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < p.n_tiles; t += gridDim.x, ++tl) {
        const uint32_t buf = tl & 1;
        ok = mbar_wait(&bar.tempty[buf], ((tl >> 1) & 1) ^ 1, &abort_flag, p.err);
        if (!ok) break;
        tc_fence_after();
        for (int ks = 0; ok && ks < k_steps; ++ks, ++g) {
          const uint32_t st = g % kStages;
          ok = mbar_wait(&bar.full[st], (g / kStages) & 1, &abort_flag, p.err);
          if (!ok) break;
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + st * kStageBytes);
          const uint64_t da = smem_desc_sw128(sa, 16, 1024), db = smem_desc_sw128(sa + kABytes, 16, 1024);
#pragma unroll
          for (int kk = 0; kk < kKStep / 16; ++kk)  // start address in 16-byte units: 32 bytes per K = 16
            mma_ss(tmem + buf * kN, da + (uint64_t)(kk * 2), db + (uint64_t)(kk * 2), idesc, (ks | kk) != 0);
          mma_commit(&bar.empty[st]);
        }
        if (!ok) break;
        mma_commit(&bar.tfull[buf]);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue: two threads per token
    // Thread (token, half) owns channels half * CH .. + CH - 1 of the channel block, all heads.
    constexpr int CH = CW / 2;
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const int R = p.r;
    uint32_t tl = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < p.n_tiles; t += gridDim.x, ++tl) {
      const int m = t / p.n_blocks, nb = t % p.n_blocks;
      const int token = m * kM + r;
      const bool valid = token < p.rows;
      const uint32_t buf = tl & 1;
      const size_t base = ((size_t)(valid ? token : 0) * H) * p.dv + (size_t)nb * CW + half * CH;
      // this thread's O values, every head at once (loads in flight together), kept for the mix
      uint32_t ow[H][CH / 2];
      if (valid) {
#pragma unroll
        for (int h = 0; h < H; ++h) load_packed<CH>(p.O + base + (size_t)h * p.dv, ow[h]);
      }
      // rank-r projections sum_h V[h,m] O[t,h,c] of this thread's channels
      float proj[kMaxR][CH];
#pragma unroll
      for (int q = 0; q < kMaxR; ++q)
#pragma unroll
        for (int c = 0; c < CH; ++c) proj[q][c] = 0.0f;
      if (valid) {
#pragma unroll
        for (int h = 0; h < H; ++h)
#pragma unroll
          for (int q = 0; q < kMaxR; ++q)
            if (q < R) {
              const float vv = sV[h * R + q];
#pragma unroll
              for (int c = 0; c < CH; c += 2) {
                proj[q][c] = fmaf(vv, bf16_lo(ow[h][c / 2]), proj[q][c]);
                proj[q][c + 1] = fmaf(vv, bf16_hi(ow[h][c / 2]), proj[q][c + 1]);
              }
            }
      }
      ok = mbar_wait(&bar.tfull[buf], (tl >> 1) & 1, &abort_flag, p.err) && ok;
      tc_fence_after();
      // 32 TMEM columns = 32 / CW heads at a time: logits, mix, gate, store
#pragma unroll
      for (int c0 = 0; c0 < kN; c0 += 32) {
        uint32_t zr[32];
        tmem_ld32_nowait(tmem + lane_off + buf * kN + c0, zr);
        tmem_wait_ld_regs(zr);
        if (c0 + 32 == kN) {  // every logit of the tile is in registers: the buffer may be reused
          tc_fence_before();
          mbar_arrive(&bar.tempty[buf]);
        }
        if (!valid) continue;
#pragma unroll
        for (int hh = 0; hh < 32 / CW; ++hh) {
          const int h = c0 / CW + hh;
          uint32_t yw[CH / 2];
#pragma unroll
          for (int c = 0; c < CH; c += 2) {
            float o0 = bf16_lo(ow[h][c / 2]), o1 = bf16_hi(ow[h][c / 2]);
#pragma unroll
            for (int q = 0; q < kMaxR; ++q)
              if (q < R) {
                const float uu = sU[h * R + q];
                o0 = fmaf(uu, proj[q][c], o0);
                o1 = fmaf(uu, proj[q][c + 1], o1);
              }
            // this thread's logits: channel c of its half (both indices compile-time constants)
            const float z0 = __uint_as_float(half ? zr[hh * CW + CH + c] : zr[hh * CW + c]);
            const float z1 = __uint_as_float(half ? zr[hh * CW + CH + c + 1] : zr[hh * CW + c + 1]);
            yw[c / 2] = pack_bf16x2(sigmoidf(z0) * o0, sigmoidf(z1) * o1);
          }
          store_packed<CH>(p.Y + base + (size_t)h * p.dv, yw);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

int sm_count() {
  static std::mutex mu;
  static int cache[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  std::lock_guard<std::mutex> lock(mu);
  if (!cache[dev] && cudaDeviceGetAttribute(&cache[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return 0;
  return cache[dev];
}

template <int CW>
hcadsa_status launch(const CUtensorMap& ma, const CUtensorMap& mb, const Params& p, cudaStream_t s) {
  if (cudaFuncSetAttribute(gate_vha_kernel<CW>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) !=
      cudaSuccess)
    return launch_status();
  const int sms = sm_count();
  if (sms <= 0) return HCADSA_ERR_CUDA;
  const int grid = p.n_tiles < sms ? p.n_tiles : sms;
  gate_vha_kernel<CW><<<grid, kThreads, kSmemBytes, s>>>(ma, mb, p);
  return launch_status();
}

}  // namespace
}  // namespace hcadsa

extern "C" hcadsa_status attn_gate_vha_fwd(const hcadsa_bf16* O, const hcadsa_bf16* cq, const hcadsa_bf16* Wg,
                                           const float* U, const float* V, hcadsa_bf16* Y, int B, int L, int H,
                                           int dv, int rq, int r, hcadsa_stream stream) {
  using namespace hcadsa;
  if (!O || !cq || !Wg || !Y || (r > 0 && (!U || !V))) return HCADSA_ERR_NULL;
  if (B < 0 || L < 0 || H <= 0 || dv <= 0 || rq <= 0 || r < 0) return HCADSA_ERR_SHAPE;
  if ((H != 16 && H != 32 && H != 64) || dv % (kN / H) != 0 || dv % 8 != 0 || rq % kKStep != 0 || r > kMaxR)
    return HCADSA_ERR_UNSUPPORTED;
  if (!aligned16(O) || !aligned16(cq) || !aligned16(Wg) || !aligned16(Y) ||
      (r > 0 && ((reinterpret_cast<uintptr_t>(U) & 3u) || (reinterpret_cast<uintptr_t>(V) & 3u))))
    return HCADSA_ERR_ALIGN;
  const long long rows = (long long)B * L;
  if (rows == 0) return HCADSA_OK;
  const int cw = kN / H;
  const long long n_blocks = dv / cw;
  const long long n_tiles = (rows + kM - 1) / kM * n_blocks;
  if (rows > 2147483647LL || n_tiles > 2147483647LL || (long long)H * dv * rq > (1LL << 40))
    return HCADSA_ERR_UNSUPPORTED;
  CUtensorMap ma, mb;
  {
    const uint64_t dims[2] = {(uint64_t)rq, (uint64_t)rows};
    const uint64_t strides[1] = {(uint64_t)rq * 2};
    const uint32_t box[2] = {(uint32_t)kKStep, (uint32_t)kM};
    if (!encode_tmap_bf16(&ma, 2, const_cast<hcadsa_bf16*>(cq), dims, strides, box, true)) return HCADSA_ERR_CUDA;
  }
  {
    const uint64_t dims[3] = {(uint64_t)rq, (uint64_t)dv, (uint64_t)H};
    const uint64_t strides[2] = {(uint64_t)rq * 2, (uint64_t)dv * rq * 2};
    const uint32_t box[3] = {(uint32_t)kKStep, (uint32_t)cw, (uint32_t)H};
    if (!encode_tmap_bf16(&mb, 3, const_cast<hcadsa_bf16*>(Wg), dims, strides, box, true)) return HCADSA_ERR_CUDA;
  }
  Params p;
  p.O = O;
  p.U = U;
  p.V = V;
  p.Y = Y;
  p.err = device_error_ptr();
  p.rows = (int)rows;
  p.H = H;
  p.dv = dv;
  p.rq = rq;
  p.r = r;
  p.cw = cw;
  p.n_blocks = (int)n_blocks;
  p.n_tiles = (int)n_tiles;
  cudaStream_t s = as_stream(stream);
  switch (cw) {
    case 16: return launch<16>(ma, mb, p, s);
    case 8: return launch<8>(ma, mb, p, s);
    default: return launch<4>(ma, mb, p, s);
  }
}
