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
//   * CTA pairs (clusters of 2, tcgen05 cta_group::2): a pair computes 256 tokens x the 256 gate
//     columns of a channel block with M = 256 MMAs.  Each CTA loads its own 128-token cq tile
//     (A) and HALF of the Wg rows (B: heads [r H/2, (r+1) H/2) of the block, a 3D TMA box
//     {64, cw, H/2} over Wg viewed as [H][dv][rq], SW128), so a stage is 32 KB instead of 48 KB
//     and the operand traffic from L2 per output drops by a third -- with single-CTA 128 x 256
//     tiles every tile re-read 768 KB of operands, and that stream from L2 was the bound.
//     Both CTAs' TMA loads complete on the leader's (rank 0) barrier; the leader's thread
//     issues every MMA and its commits reach the barriers of both CTAs (.multicast::cluster).
//     Each CTA's TMEM holds its 128 tokens x 256 columns, so the epilogue is per CTA.
//   * Warp 0: TMA producer (6 stages of 32 KB); warp 1: TMEM allocation (both CTAs) + the MMA
//     thread (leader only: 4 MMAs of M = 256, N = 256, K = 16 per stage, fp32 accumulator of
//     256 TMEM columns, double-buffered across tiles); warps 2-9: epilogue, two threads per
//     token (each half of the channel block, every head; its O values loaded at once and kept in
//     registers): the rank-r projections sum_h V[h,m] O[t,h,c] of its channels, then per head
//     the mix, the sigmoid of the logit from TMEM and the bf16 store of Y.  An epilogue warp
//     frees a TMEM buffer with one arrival on the leader's barrier.
//   * Persistent pairs walk the pair tiles (token-tile pair, channel block); consecutive pairs
//     share the token tiles, so the cq tiles and Wg stay in L2.
#include <cuda_bf16.h>

#include <mutex>

#include "host_common.h"
#include "ptx.cuh"

namespace hcadsa {
namespace {

constexpr int kM = 128;      // tokens per tile
constexpr int kN = 256;      // gate columns per tile (H heads x cw channels)
constexpr int kKStep = 64;   // K per stage (one 128-byte swizzle row of bf16)
constexpr int kStages = 6;
constexpr int kABytes = kM * kKStep * 2;        // 16 KB
constexpr int kBBytes = (kN / 2) * kKStep * 2;  // 16 KB: this CTA's half of the 256 Wg rows
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kMaxR = 4;     // rank of the head mix
static_assert(kMaxR == 4, "the mix reads the per-head U / V slots as one float4");
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
  int rows, H, dv, rq, r, cw, n_blocks, n_tiles;  // n_tiles: pair tiles (token-tile pair, block)
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

// 16 TMEM lanes, N columns, twice (.16x32bx2): threads 0-15 of the warp read lanes base + t at
// columns [c, c + N), threads 16-31 the same lanes at columns [c + kOff, c + kOff + N).
template <int N, int kOff>
__device__ __forceinline__ void tmem_ld_16x2(uint32_t taddr, uint32_t (&r)[N]) {
  if constexpr (N == 8) {
    asm volatile("tcgen05.ld.sync.aligned.16x32bx2.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8], %9;"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr), "n"(kOff)
                 : "memory");
  } else if constexpr (N == 4) {
    asm volatile("tcgen05.ld.sync.aligned.16x32bx2.x4.b32 {%0,%1,%2,%3}, [%4], %5;"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(taddr), "n"(kOff)
                 : "memory");
  } else {
    static_assert(N == 2, "x2, x4 or x8");
    asm volatile("tcgen05.ld.sync.aligned.16x32bx2.x2.b32 {%0,%1}, [%2], %3;"
                 : "=r"(r[0]), "=r"(r[1])
                 : "r"(taddr), "n"(kOff)
                 : "memory");
  }
}

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// The address of the same shared variable in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t cluster_addr(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
  return r;
}
__device__ __forceinline__ void arrive_cluster(uint32_t addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(addr) : "memory");
}
// TMA loads of a CTA pair: the data lands in this CTA's shared memory, the transaction bytes
// complete on `bar` (a shared::cluster address, here the leader's barrier).
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* map, uint32_t bar, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1)
      : "memory");
}
__device__ __forceinline__ void tma_load_3d_pair(void* dst, const CUtensorMap* map, uint32_t bar, int c0, int c1,
                                                 int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
// D[tmem] (+)= A * B over the pair (M = 256: each CTA's A rows and half of B's rows).
__device__ __forceinline__ void mma_ss_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive once on `bar` in both CTAs of the pair when every earlier MMA of this thread is done.
__device__ __forceinline__ void mma_commit_pair(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;"
               ::"r"(smem_u32(bar)), "h"((uint16_t)3)
               : "memory");
}

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
  // U and V with kMaxR slots per head (zero past the rank), so the mix reads one float4 per head
  __shared__ __align__(16) float sU[kMaxH * kMaxR];
  __shared__ __align__(16) float sV[kMaxH * kMaxR];

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t rank = cluster_rank();          // 0: the leader, which issues the MMAs
  const int pair = (int)blockIdx.x >> 1, n_pairs = (int)gridDim.x >> 1;
  for (int i = threadIdx.x; i < H * kMaxR; i += kThreads) {
    const int hq = i / kMaxR, q = i % kMaxR;
    sU[i] = q < p.r ? p.U[hq * p.r + q] : 0.0f;
    sV[i] = q < p.r ? p.V[hq * p.r + q] : 0.0f;
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bar.full[s], 1);
      mbar_init(&bar.empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar.tfull[s], 1);
      mbar_init(&bar.tempty[s], 2 * kEpiWarps);  // the leader's copy: one arrival per epilogue warp of the pair
    }
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {  // the same warp in both CTAs, the same shared slot
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_base_sh)),
                 "r"(512));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::);
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // barriers and TMEM of both CTAs exist before any cross-CTA operation
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
      for (int t = pair; ok && t < p.n_tiles; t += n_pairs) {
        const int m = 2 * (t / p.n_blocks) + (int)rank, nb = t % p.n_blocks;  // this CTA's token tile
        for (int ks = 0; ok && ks < k_steps; ++ks, ++g) {
          const uint32_t st = g % kStages;
          // the slot is free in this CTA once the pair's MMAs that read it are done (multicast)
          ok = mbar_wait(&bar.empty[st], ((g / kStages) & 1) ^ 1, &abort_flag, p.err);
          if (!ok) break;
          uint8_t* sa = smem + st * kStageBytes;
          const uint32_t full_leader = cluster_addr(&bar.full[st], 0);
          if (rank == 0) mbar_arrive_expect_tx(&bar.full[st], 2 * kStageBytes);  // both CTAs' bytes
          tma_load_2d_pair(sa, &map_a, full_leader, ks * kKStep, m * kM);
          tma_load_3d_pair(sa + kABytes, &map_b, full_leader, ks * kKStep, nb * CW, (int)rank * (H / 2));
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && rank == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(2 * kM, kN, false, false);
      uint32_t g = 0, tl = 0;
      bool ok = true;
      for (int t = pair; ok && t < p.n_tiles; t += n_pairs, ++tl) {
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
            mma_ss_pair(tmem + buf * kN, da + (uint64_t)(kk * 2), db + (uint64_t)(kk * 2), idesc, (ks | kk) != 0);
          mma_commit_pair(&bar.empty[st]);
        }
        if (!ok) break;
        mma_commit_pair(&bar.tfull[buf]);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue: two threads per token
    // Thread (token, half) owns channels half * CH .. + CH - 1 of the channel block, all heads.
    // A token's two threads are lanes t and t + 16 of one warp (the warp covers 16 TMEM lanes
    // of its quarter), so their O loads and Y stores fill whole 32-byte sectors per instruction.
    constexpr int CH = CW / 2;
    const int quarter = warp & 3;
    const int wq = (warp - 2) >> 2;  // which 16 lanes of the quarter
    const int half = lane >> 4;
    const int r = quarter * 32 + wq * 16 + (lane & 15);
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32 + wq * 16) << 16;
    uint32_t tl = 0;
    bool ok = true;
    // this thread's row of a tile: whether it is a token, and where its O / Y values start
    auto row_of = [&](int t, bool& v, size_t& b) {
      const int m = 2 * (t / p.n_blocks) + (int)rank, nb = t % p.n_blocks;
      const int token = m * kM + r;
      v = t < p.n_tiles && token < p.rows;
      b = ((size_t)(v ? token : 0) * H) * p.dv + (size_t)nb * CW + half * CH;
    };
    // this thread's O values, every head; the next tile's are loaded head by head as soon as a
    // head's mix has used them, so their latency overlaps the rest of the tile
    uint32_t ow[H][CH / 2];
    bool valid;
    size_t base;
    row_of(pair, valid, base);
    if (valid) {
#pragma unroll
      for (int h = 0; h < H; ++h) load_packed<CH>(p.O + base + (size_t)h * p.dv, ow[h]);
    }
    for (int t = pair; t < p.n_tiles; t += n_pairs, ++tl) {
      const uint32_t buf = tl & 1;
      bool valid_n;
      size_t base_n;
      row_of(t + n_pairs, valid_n, base_n);
      // rank-r projections sum_h V[h,m] O[t,h,c] of this thread's channels
      float proj[kMaxR][CH];
#pragma unroll
      for (int q = 0; q < kMaxR; ++q)
#pragma unroll
        for (int c = 0; c < CH; ++c) proj[q][c] = 0.0f;
      if (valid) {
#pragma unroll
        for (int h = 0; h < H; ++h) {
          const float4 v4 = *reinterpret_cast<const float4*>(&sV[h * kMaxR]);
          const float vq[kMaxR] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
          for (int c = 0; c < CH; c += 2) {
            const float x0 = bf16_lo(ow[h][c / 2]), x1 = bf16_hi(ow[h][c / 2]);
#pragma unroll
            for (int q = 0; q < kMaxR; ++q) {  // slots past the rank hold 0: they add nothing
              proj[q][c] = fmaf(vq[q], x0, proj[q][c]);
              proj[q][c + 1] = fmaf(vq[q], x1, proj[q][c + 1]);
            }
          }
        }
      }
      ok = mbar_wait(&bar.tfull[buf], (tl >> 1) & 1, &abort_flag, p.err) && ok;
      tc_fence_after();
      // kHB heads at a time (32 logit registers): this thread's CH logits of each head, then the
      // mix, the gate and the store
      constexpr int kHB = 32 / CH;
      static_assert(H % kHB == 0, "whole head batches");
#pragma unroll
      for (int h0 = 0; h0 < H; h0 += kHB) {
        uint32_t zr[kHB][CH];
#pragma unroll
        for (int hh = 0; hh < kHB; ++hh) tmem_ld_16x2<CH, CH>(tmem + lane_off + buf * kN + (h0 + hh) * CW, zr[hh]);
        tmem_wait_ld_regs(reinterpret_cast<uint32_t(&)[32]>(zr));
        if (h0 + kHB == H) {  // every logit of the tile is in registers: the buffer may be reused
          tc_fence_before();
          __syncwarp();
          if (lane == 0) arrive_cluster(cluster_addr(&bar.tempty[buf], 0));
        }
        if (!valid) {
#pragma unroll
          for (int hh = 0; hh < kHB; ++hh)
            if (valid_n) load_packed<CH>(p.O + base_n + (size_t)(h0 + hh) * p.dv, ow[h0 + hh]);
          continue;
        }
#pragma unroll
        for (int hh = 0; hh < kHB; ++hh) {
          const int h = h0 + hh;
          const float4 u4 = *reinterpret_cast<const float4*>(&sU[h * kMaxR]);
          const float uq[kMaxR] = {u4.x, u4.y, u4.z, u4.w};
          uint32_t yw[CH / 2];
#pragma unroll
          for (int c = 0; c < CH; c += 2) {
            float o0 = bf16_lo(ow[h][c / 2]), o1 = bf16_hi(ow[h][c / 2]);
#pragma unroll
            for (int q = 0; q < kMaxR; ++q) {
              o0 = fmaf(uq[q], proj[q][c], o0);
              o1 = fmaf(uq[q], proj[q][c + 1], o1);
            }
            const float z0 = __uint_as_float(zr[hh][c]), z1 = __uint_as_float(zr[hh][c + 1]);
            yw[c / 2] = pack_bf16x2(sigmoidf(z0) * o0, sigmoidf(z1) * o1);
          }
          store_packed<CH>(p.Y + base + (size_t)h * p.dv, yw);
          if (valid_n) load_packed<CH>(p.O + base_n + (size_t)h * p.dv, ow[h]);  // head h is done
        }
      }
      valid = valid_n;
      base = base_n;
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // no MMA of the pair and no cross-CTA arrival is pending any more
  tc_fence_after();
  if (warp == 1) asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
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
  if (sms < 2) return HCADSA_ERR_CUDA;
  const int pairs = p.n_tiles < sms / 2 ? p.n_tiles : sms / 2;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, gate_vha_kernel<CW>, ma, mb, p) != cudaSuccess) return launch_status();
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
  const long long n_tiles = ((rows + kM - 1) / kM + 1) / 2 * n_blocks;  // pair tiles
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
    const uint32_t box[3] = {(uint32_t)kKStep, (uint32_t)cw, (uint32_t)(H / 2)};  // a CTA's half of the rows
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
