// dsa_attn.cu -- DSA sparse attention forward on sm_100a (tcgen05 + TMEM; K/V rows gathered
// with cp.async, Q loaded by TMA).
//
// Method: the mirrorspeed page, section "Hybrid sparse attention, 1/7 full context
// access": in the MLA layers each query attends only to the k positions its indexer
// scored highest; MLA heads are 256 wide (ai-club.cn page,
// section "混合注意力（MLA + HCA）").  All 64 query heads of a token share one K/V
// head (the MLA latent reading) and the token's index row.
//
// Kernel design (persistent: one CTA per SM walks query tokens tok = blockIdx.x + i*gridDim.x):
//   * The 64 heads of a token are too few rows for a full-rate M=128 tcgen05 tile, so the
//     contraction is transposed: the 128 gathered keys of a tile are M.
//       S^T[key, head]  = K_g (A, K-major, 128 x 256)  *  Q^T (B, K-major, 64 heads)
//       O^T[dv, head]  += V_g^T (A, MN-major, 2 x 128 dv) * P^T (B, MN-major, 64 heads)
//     TMEM: O^T double-buffered per token [0,128) / [128,256) so one token's epilogue
//     overlaps the next token's MMAs; S^T double-buffered per tile [256,320) / [320,384).
//   * Warps 0-5 gather K and V rows with cp.async: one warp instruction moves one whole
//     512-byte row (lane l -> 16 bytes of 64-column chunk l/8), written 128B-swizzled into a
//     ring of two 64 KB groups (4 chunk slots each); a group holds one K or one V tile, loaded
//     in exactly the order warp 6 consumes them: K_0, K_1, V_0, K_2, V_1, ...  Completion is
//     tracked with cp.async.mbarrier.arrive.noinc, one arrival per producer thread per tile, so
//     the MMA thread waits once per tile (a wait costs the issuing thread a few hundred cycles,
//     which only a whole tile of MMAs hides) and issues a proxy fence after it so the tensor
//     core sees the generic-proxy writes.  (Measured on B200: this reaches ~105 GB/s per SM
//     from L2, TMA tile::gather4 of 4 x 128 B rows ~16 GB/s.)
//     Q (32 KB, TMA) is reloaded per token once the previous token's last S^T MMA is done.
//   * Warp 6, lane 0 issues every MMA.  Warps 7-10: softmax (one thread per key = TMEM lane,
//     64 head scores each; per-head row sums reduced across the warp every tile).  The first tile of a token sets the per-head reference max by a
//     warp reduce-scatter + 4-warp combine; later tiles only check their scores against it and
//     redo the reduction (and rescale O^T) when some score exceeds it by 2^8.  P^T rows go to
//     shared memory; then the token's epilogue (normalise O^T, store O).
//   * Index rows may hold padding (< 0) anywhere; a 128-entry tile without any valid entry
//     is skipped, other invalid entries read row 0 and are masked.  Index rows are staged in
//     shared memory (double buffer): the softmax warps prefetch token i+2's row with cp.async
//     as soon as the producer and MMA warps have released the buffer token i used, so no
//     role waits on the index tensor in HBM.
//   * Barrier phases continue across tokens: s_full/p_ready/pv_done are indexed by a global
//     tile counter, q_full/q_empty/o_full/o_empty by a counter of tokens with work.
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
constexpr int kRingSlots = 8;  // two groups of 4 slots: one K tile or one V tile per group
constexpr int kQChunkBytes = kH * 128;     // 64 heads x 64 bf16
constexpr int kQBytes = 4 * kQChunkBytes;  // 32 KB
constexpr int kPBytes = kKeyTile * 128;    // 128 keys x 64 heads bf16
constexpr int kMaxK = 4096;                // 32 tiles: one bit per tile in a 32-bit mask
constexpr int kIdxBytes = kMaxK * 4;  // one index row
constexpr int kSmemBytes = kQBytes + kRingSlots * kChunkBytes + 2 * kPBytes + 2 * kIdxBytes + 1024;
// Gather throughput scales with the number of producer warps.  11 warps put 3 on some SM
// sub-partitions (16K-entry register file each), which caps a thread at 168 registers; the
// softmax keeps its per-head row sums reduced across the warp (2 per lane) to fit.
constexpr int kProducerWarps = 6;
constexpr int kMmaWarp = kProducerWarps;
constexpr int kSoftmaxWarp0 = kProducerWarps + 1;
constexpr int kThreads = 32 * (kProducerWarps + 1 + 4);
constexpr uint32_t kTmemS = 256;  // S^T buffers at columns 256 and 320
constexpr float kLazyRescale = 8.0f;

struct Params {
  const uint16_t* K;
  const uint16_t* V;
  const int32_t* idx;
  uint16_t* O;
  float* lse;
  int* err;
  int n_tok, Lq, Lk, k;
  float scale_log2;
};

struct __align__(8) Barriers {
  uint64_t q_full, q_empty;
  uint64_t full[2];   // ring group g holds a whole K or V tile (192 producer-thread arrivals)
  uint64_t empty[2];  // the MMAs that read group g have completed
  uint64_t s_full[2];
  uint64_t p_ready[2];
  uint64_t pv_done;
  uint64_t o_full[2];
  uint64_t o_empty[2];
  uint64_t idx_full[2];   // index row of a token landed (128 softmax-thread cp.async arrivals)
  uint64_t idx_empty[2];  // producers (3 warps) and MMA warp are done with the row
};

struct SoftShared {
  float wred[4][kH];
  __align__(16) float m_ref[kH];
  __align__(16) float alpha[kH];  // rescale factors; 1/l in the epilogue
};

__device__ __forceinline__ bool idx_ok(int s, int Lk) { return s >= 0 && s < Lk; }

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
// Arrives on bar once every cp.async this thread issued so far has landed (no pending-count bump).
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// Bit j set iff tile j (entries [128j, 128j+128) of the row) holds a valid entry.  Whole warp;
// `row` is the shared-memory copy of the index row.
__device__ __forceinline__ uint32_t tile_mask_of_row(const int32_t* row, int k, int Lk, int lane) {
  uint32_t mask = 0;
  const int n_tiles = (k + kKeyTile - 1) / kKeyTile;
  for (int j = 0; j < n_tiles; ++j) {
    bool any = false;
#pragma unroll
    for (int q = 0; q < 4; ++q) {  // consecutive lanes read consecutive words: no bank conflicts
      const int e = j * kKeyTile + q * 32 + lane;
      if (e < k) any |= idx_ok(row[e], Lk);
    }
    if (__any_sync(0xffffffffu, any)) mask |= 1u << j;
  }
  return mask;
}

__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}

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

__device__ __forceinline__ void softmax_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
// Named barrier over the 128 softmax threads that also ORs a predicate across them.
__device__ __forceinline__ bool softmax_bar_or(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 1, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred)
      : "memory");
  return r != 0;
}

// Softmax threads: once the producers and the MMA warp released buffer `buf` (used by local
// token i), fetch the index row of token `next` into it with cp.async.
__device__ __forceinline__ void refill_idx_row(const Params& p, Barriers& bar, uint32_t sIdx_a, int buf, int i,
                                               int next, int tid, volatile int& abort_flag, bool& ok) {
  if (next >= p.n_tok) return;
  ok = mbar_wait(&bar.idx_empty[buf], (i >> 1) & 1, &abort_flag, p.err) && ok;
  for (int e = tid; e < p.k; e += 128) cp_async4(sIdx_a + (buf * kMaxK + e) * 4, p.idx + (size_t)next * p.k + e);
  cp_async_arrive_noinc(&bar.idx_full[buf]);
}

__global__ void __launch_bounds__(kThreads, 1)
    dsa_attn_kernel(const __grid_constant__ CUtensorMap map_q, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sRing = smem + kQBytes;
  uint8_t* sP = sRing + kRingSlots * kChunkBytes;
  int32_t* sIdx = reinterpret_cast<int32_t*>(sP + 2 * kPBytes);  // [2][kMaxK]
  __shared__ Barriers bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;
  __shared__ SoftShared ss;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    mbar_init(&bar.q_full, 1);
    mbar_init(&bar.q_empty, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar.full[s], kProducerWarps * 32);
      mbar_init(&bar.empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar.s_full[s], 1);
      mbar_init(&bar.p_ready[s], 128);
      mbar_init(&bar.o_full[s], 1);
      mbar_init(&bar.o_empty[s], 128);
    }
    mbar_init(&bar.pv_done, 1);
    for (int s2 = 0; s2 < 2; ++s2) {
      mbar_init(&bar.idx_full[s2], 128);
      mbar_init(&bar.idx_empty[s2], kProducerWarps + 1);
    }
    abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&tmem_base_sh, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  const int Lk = p.Lk, k = p.k;

  if (warp < kProducerWarps) {
    // ------------------------------------------------------------ producers (cp.async rows)
    const uint32_t ring = smem_u32(sRing);
    const uint16_t* Kg = p.K;
    const uint16_t* Vg = p.V;
    uint32_t u = 0;  // K/V tiles issued so far: ring group u & 1, phase (u >> 1) & 1
    int it = 0;  // tokens with work so far
    bool ok = true;
    const int chunk = lane >> 3, piece = lane & 7;
    int i = 0;   // tokens of this CTA so far (index-row buffer i & 1)
    for (int tok = blockIdx.x; tok < p.n_tok && ok; tok += gridDim.x, ++i) {
      const int buf = i & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(&bar.idx_full[buf], (i >> 1) & 1, &abort_flag, p.err));
      if (!ok) break;
      const int32_t* row = sIdx + buf * kMaxK;
      const uint32_t mask = tile_mask_of_row(row, k, Lk, lane);
      if (!mask) {
        if (lane == 0) mbar_arrive(&bar.idx_empty[buf]);
        continue;
      }
      const int J = __popc(mask);
      const size_t kv_row0 = (size_t)(tok / p.Lq) * Lk;  // first K/V row of this token's batch
      // warp w gathers tile rows w, w+3, w+6, ...: lane l holds the K/V row of the warp's
      // l-th row (ra) and (32+l)-th row (rb)
      const int n_rows_w = (kKeyTile - warp + kProducerWarps - 1) / kProducerWarps;  // 43, 43, 42
      int ra_prev = 0, rb_prev = 0, ra_cur = 0, rb_cur = 0;
      uint32_t m = mask;
      for (int step = 0; step <= J && ok; ++step) {
        if (step < J) {
          const int j = __ffs(m) - 1;
          m &= m - 1;
          const int ea = j * kKeyTile + warp + kProducerWarps * lane;
          const int eb = j * kKeyTile + warp + kProducerWarps * (32 + lane);
          const int sa = ea < k ? row[ea] : -1;
          const int sb = (32 + lane < n_rows_w && eb < k) ? row[eb] : -1;
          ra_cur = idx_ok(sa, Lk) ? sa : 0;
          rb_cur = idx_ok(sb, Lk) ? sb : 0;
        }
        for (int part = 0; part < 2 && ok; ++part) {
          const bool is_k = part == 0;
          if (is_k ? step >= J : step < 1) continue;
          const int ra = is_k ? ra_cur : ra_prev, rb = is_k ? rb_cur : rb_prev;
          const uint16_t* base = (is_k ? Kg : Vg) + kv_row0 * kD + lane * 8;
          ok = __all_sync(0xffffffffu, mbar_wait(&bar.empty[u & 1], ((u >> 1) & 1) ^ 1, &abort_flag, p.err));
          if (!ok) break;
          const uint32_t dst0 = ring + ((u & 1) * 4 + chunk) * kChunkBytes;
#pragma unroll 4
          for (int i = 0; i < n_rows_w; ++i) {
            const int trow = warp + kProducerWarps * i;  // row of the tile
            const int src_row = __shfl_sync(0xffffffffu, i < 32 ? ra : rb, i & 31);
            cp_async16(dst0 + trow * 128 + ((piece ^ (trow & 7)) << 4), base + (size_t)src_row * kD);
          }
          cp_async_arrive_noinc(&bar.full[u & 1]);
          ++u;
          if (is_k && step == 0 && warp == 0) {
            // Q of this token (after its first K tile is in flight), once the previous token's
            // last S^T MMA no longer reads the buffer
            ok = __all_sync(0xffffffffu, mbar_wait(&bar.q_empty, (it & 1) ^ 1, &abort_flag, p.err));
            if (ok && lane == 0) {
              mbar_arrive_expect_tx(&bar.q_full, kQBytes);
              for (int c = 0; c < 4; ++c) tma_load_3d(sQ + c * kQChunkBytes, &map_q, &bar.q_full, c * 64, 0, tok);
            }
          }
        }
        ra_prev = ra_cur;
        rb_prev = rb_cur;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar.idx_empty[buf]);  // this warp read its last row index
      ++it;
    }
    cp_async_wait_all();
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    uint32_t u = 0;  // K/V tiles consumed so far (same sequence as the producers)
    int it = 0;
    uint32_t g = 0;  // global tile counter
    bool ok = true;
    const uint32_t sQa = smem_u32(sQ), sRa = smem_u32(sRing), sPa = smem_u32(sP);
    const uint32_t idesc_s = idesc_bf16_f32(128, kH, false, false);
    const uint32_t idesc_o = idesc_bf16_f32(128, kH, true, true);
    int i = 0;
    for (int tok = blockIdx.x; tok < p.n_tok && ok; tok += gridDim.x, ++i) {
      const int buf = i & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(&bar.idx_full[buf], (i >> 1) & 1, &abort_flag, p.err));
      if (!ok) break;
      const uint32_t mask = tile_mask_of_row(sIdx + buf * kMaxK, k, Lk, lane);
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar.idx_empty[buf]);  // only the mask was needed
      if (!mask) continue;
      const int J = __popc(mask);
      const int ob = it & 1;
      if (lane == 0) {
        ok = mbar_wait(&bar.q_full, it & 1, &abort_flag, p.err);
        tc_fence_after();
        for (int step = 0; step <= J && ok; ++step) {
          if (step < J) {
            const uint32_t gs = g + step;
            const uint32_t tS = tmem + kTmemS + (gs & 1) * kH;
            // one wait per K tile: every producer thread arrives once all of its row copies of
            // the tile (all 4 chunks) have landed
            ok = mbar_wait(&bar.full[u & 1], (u >> 1) & 1, &abort_flag, p.err);
            if (!ok) break;
            fence_proxy_async_smem();  // cp.async (generic proxy) writes -> tensor core reads
            tc_fence_after();
            {
              const uint64_t da0 = smem_desc_sw128(sRa + (u & 1) * 4 * kChunkBytes, 16, 1024);
              const uint64_t db0 = smem_desc_sw128(sQa, 16, 1024);
#pragma unroll
              for (int c = 0; c < 4; ++c)
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)  // descriptor start address field is in 16-byte units
                  mma_ss(tS, da0 + (uint64_t)((c * kChunkBytes + kk * 32) >> 4),
                         db0 + (uint64_t)((c * kQChunkBytes + kk * 32) >> 4), idesc_s, (c | kk) != 0);
            }
            mma_commit(&bar.empty[u & 1]);
            ++u;
            mma_commit(&bar.s_full[gs & 1]);
            if (step == J - 1) mma_commit(&bar.q_empty);
          }
          if (step >= 1) {
            const int j = step - 1;
            const uint32_t gj = g + j;
            if (j == 0) {  // O^T buffer ob must have been drained by the epilogue of token it-2
              ok = mbar_wait(&bar.o_empty[ob], ((it >> 1) & 1) ^ 1, &abort_flag, p.err);
              if (!ok) break;
            }
            ok = mbar_wait(&bar.p_ready[gj & 1], (gj >> 1) & 1, &abort_flag, p.err);
            if (!ok) break;
            tc_fence_after();
            const uint32_t pbase = sPa + (gj & 1) * kPBytes;
            ok = mbar_wait(&bar.full[u & 1], (u >> 1) & 1, &abort_flag, p.err);  // the whole V tile
            if (!ok) break;
            fence_proxy_async_smem();
            tc_fence_after();
            {
              // V^T chunk pair (2hv, 2hv+1): M = 128 d_v rows, the pair's slots are LBO apart
              const uint64_t da0 = smem_desc_sw128(sRa + (u & 1) * 4 * kChunkBytes, kChunkBytes, 1024);
              const uint64_t db0 = smem_desc_sw128(pbase, kPBytes, 1024);
              const uint32_t acc0 = j > 0 ? 1u : 0u;
#pragma unroll
              for (int hv = 0; hv < 2; ++hv)
#pragma unroll
                for (int kk = 0; kk < kKeyTile / 16; ++kk)
                  mma_ss(tmem + ob * 128 + hv * kH, da0 + (uint64_t)((hv * 2 * kChunkBytes + kk * 2048) >> 4),
                         db0 + (uint64_t)((kk * 2048) >> 4), idesc_o, kk > 0 ? 1u : acc0);
            }
            mma_commit(&bar.empty[u & 1]);
            ++u;
            mma_commit(&bar.pv_done);
            if (j == J - 1) mma_commit(&bar.o_full[ob]);
          }
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      u = __shfl_sync(0xffffffffu, u, 0);
      g += J;
      ++it;
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int sw = warp - kSoftmaxWarp0;  // 0..3
    const int quarter = warp & 3;         // TMEM lane quarter this warp may access
    const int kl = quarter * 32 + lane;   // key lane of a tile / d_v row of O^T
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const int tid = sw * 32 + lane;       // 0..127
    int it = 0;
    uint32_t g = 0;
    bool ok = true;
    // No early exit in this loop: the four softmax warps meet at named barriers, so after an
    // abort every thread keeps walking the same barrier sequence (waits then fail fast).
    const uint32_t sIdx_a = smem_u32(sIdx);
    // index rows of this CTA's first two tokens
    for (int i0 = 0; i0 < 2; ++i0) {
      const int t0 = blockIdx.x + i0 * gridDim.x;
      if (t0 < p.n_tok) {
        for (int e = tid; e < k; e += 128) cp_async4(sIdx_a + (i0 * kMaxK + e) * 4, p.idx + (size_t)t0 * k + e);
        cp_async_arrive_noinc(&bar.idx_full[i0]);
      }
    }
    int i = 0;
    for (int tok = blockIdx.x; tok < p.n_tok; tok += gridDim.x, ++i) {
      const int buf = i & 1;
      ok = mbar_wait(&bar.idx_full[buf], (i >> 1) & 1, &abort_flag, p.err) && ok;
      const int32_t* row = sIdx + buf * kMaxK;
      const uint32_t mask = tile_mask_of_row(row, k, Lk, lane);
      uint16_t* obase = p.O + (size_t)tok * kH * kD;
      if (!mask) {  // no valid entry: O = 0, lse = -inf
        for (int e = tid; e < kH * kD / 8; e += 128) reinterpret_cast<uint4*>(obase)[e] = make_uint4(0, 0, 0, 0);
        if (p.lse && tid < kH) p.lse[(size_t)tok * kH + tid] = -INFINITY;
        softmax_bar();  // every softmax thread has read the row before it is refilled
        refill_idx_row(p, bar, sIdx_a, buf, i, tok + 2 * gridDim.x, tid, abort_flag, ok);
        continue;
      }
      const int J = __popc(mask);
      const int ob = it & 1;
      if (tid < kH) ss.m_ref[tid] = -INFINITY;
      float lsum0 = 0.0f, lsum1 = 0.0f;  // row sums of heads 2*lane, 2*lane+1 over this warp's keys
      uint32_t m = mask;
      for (int jj = 0; jj < J; ++jj) {
        const int j = __ffs(m) - 1;
        m &= m - 1;
        const uint32_t gs = g + jj;
        const int e = j * kKeyTile + kl;
        const int s_idx = e < k ? row[e] : -1;
        const bool valid = idx_ok(s_idx, Lk);
        if (s_idx >= Lk) raise_device_error(p.err, kErrDeviceBounds);
        ok = mbar_wait(&bar.s_full[gs & 1], (gs >> 1) & 1, &abort_flag, p.err) && ok;
        tc_fence_after();
        const uint32_t tS = tmem + lane_off + kTmemS + (gs & 1) * kH;
        uint8_t* prow = sP + (gs & 1) * kPBytes + kl * 128;
        uint32_t u0[32], u1[32];  // scores, then p (fp32 bits)
        tmem_ld32_nowait(tS, u0);
        tmem_ld32_nowait(tS + 32, u1);
        tmem_wait_ld_regs2(u0, u1);
        // Speculative pass: P against the current per-head reference max, and whether any score
        // exceeds it by more than 2^8 (then the tile is redone after a reduction).  The first
        // tile of a token always takes the reduction path (its reference is still -inf).
        bool over = jj == 0;
        if (!over) {
#pragma unroll
          for (int c8 = 0; c8 < 8; ++c8) {
            const float4 ma = *reinterpret_cast<const float4*>(&ss.m_ref[c8 * 8]);
            const float4 mb = *reinterpret_cast<const float4*>(&ss.m_ref[c8 * 8 + 4]);
            const float mr[8] = {ma.x, ma.y, ma.z, ma.w, mb.x, mb.y, mb.z, mb.w};
            uint32_t w4[4];
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) {
              const int h = c8 * 8 + 2 * qq;
              uint32_t& r0 = h < 32 ? u0[h] : u1[h - 32];
              uint32_t& r1 = h + 1 < 32 ? u0[h + 1] : u1[h + 1 - 32];
              const float x0 = fmaf(__uint_as_float(r0), p.scale_log2, -mr[2 * qq]);
              const float x1 = fmaf(__uint_as_float(r1), p.scale_log2, -mr[2 * qq + 1]);
              over |= valid && (x0 > kLazyRescale || x1 > kLazyRescale);
              const float p0 = valid ? fast_exp2(x0) : 0.0f;
              const float p1 = valid ? fast_exp2(x1) : 0.0f;
              r0 = __float_as_uint(p0);
              r1 = __float_as_uint(p1);
              w4[qq] = pack_bf16x2(p0, p1);
            }
            *reinterpret_cast<uint4*>(prow + ((c8 ^ (kl & 7)) << 4)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
          }
        }
        if (!softmax_bar_or(over)) {
          float pv[kH];
#pragma unroll
          for (int h = 0; h < 32; ++h) {
            pv[h] = __uint_as_float(u0[h]);
            pv[32 + h] = __uint_as_float(u1[h]);
          }
          warp_reduce_scatter64<false>(pv, lane);
          lsum0 += pv[0];
          lsum1 += pv[1];
        } else {
          // reduction path: new per-head reference, rescale O^T if it moved, P from scratch
          float red[kH];
          {
            uint32_t t0[32], t1[32];
            tmem_ld32_nowait(tS, t0);
            tmem_ld32_nowait(tS + 32, t1);
            tmem_wait_ld_regs2(t0, t1);
#pragma unroll
            for (int h = 0; h < 32; ++h) {
              red[h] = valid ? __uint_as_float(t0[h]) * p.scale_log2 : -INFINITY;
              red[32 + h] = valid ? __uint_as_float(t1[h]) * p.scale_log2 : -INFINITY;
            }
          }
          warp_reduce_scatter64<true>(red, lane);
          ss.wred[sw][2 * lane] = red[0];
          ss.wred[sw][2 * lane + 1] = red[1];
          softmax_bar();
          bool resc = false;
          if (tid < kH) {
            const float mt = fmaxf(fmaxf(ss.wred[0][tid], ss.wred[1][tid]), fmaxf(ss.wred[2][tid], ss.wred[3][tid]));
            const float mo = ss.m_ref[tid];
            float alpha = 1.0f, mn = mo;
            if (mo == -INFINITY) {
              mn = mt;
            } else if (mt > mo + kLazyRescale) {
              mn = mt;
              alpha = fast_exp2(mo - mt);
              resc = true;
            }
            ss.m_ref[tid] = mn;
            ss.alpha[tid] = alpha;
          }
          if (softmax_bar_or(resc)) {
            // O^T must hold every PV of this token up to tile jj-1 before it is rescaled
            ok = mbar_wait(&bar.pv_done, (gs - 1) & 1, &abort_flag, p.err) && ok;
            tc_fence_after();
#pragma unroll
            for (int hv = 0; hv < 2; ++hv) {
#pragma unroll
              for (int c = 0; c < 2; ++c) {
                uint32_t u[32];
                const uint32_t tO = tmem + lane_off + ob * 128 + hv * kH + c * 32;
                tmem_ld32_nowait(tO, u);
                tmem_wait_ld_regs(u);
#pragma unroll
                for (int h = 0; h < 32; ++h) u[h] = __float_as_uint(__uint_as_float(u[h]) * ss.alpha[c * 32 + h]);
                tmem_st32(tO, u);
              }
            }
            tmem_wait_st();
            lsum0 *= ss.alpha[2 * lane];
            lsum1 *= ss.alpha[2 * lane + 1];
          }
          tmem_ld32_nowait(tS, u0);
          tmem_ld32_nowait(tS + 32, u1);
          tmem_wait_ld_regs2(u0, u1);
#pragma unroll
          for (int c8 = 0; c8 < 8; ++c8) {
            const float4 ma = *reinterpret_cast<const float4*>(&ss.m_ref[c8 * 8]);
            const float4 mb = *reinterpret_cast<const float4*>(&ss.m_ref[c8 * 8 + 4]);
            const float mr[8] = {ma.x, ma.y, ma.z, ma.w, mb.x, mb.y, mb.z, mb.w};
            uint32_t w4[4];
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) {
              const int h = c8 * 8 + 2 * qq;
              const uint32_t s0 = h < 32 ? u0[h] : u1[h - 32];
              const uint32_t s1 = h + 1 < 32 ? u0[h + 1] : u1[h + 1 - 32];
              float p0 = 0.0f, p1 = 0.0f;
              if (valid) {
                p0 = fast_exp2(fmaf(__uint_as_float(s0), p.scale_log2, -mr[2 * qq]));
                p1 = fast_exp2(fmaf(__uint_as_float(s1), p.scale_log2, -mr[2 * qq + 1]));
              }
              (h < 32 ? u0[h] : u1[h - 32]) = __float_as_uint(p0);
              (h + 1 < 32 ? u0[h + 1] : u1[h + 1 - 32]) = __float_as_uint(p1);
              w4[qq] = pack_bf16x2(p0, p1);
            }
            *reinterpret_cast<uint4*>(prow + ((c8 ^ (kl & 7)) << 4)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
          }
          float pv[kH];
#pragma unroll
          for (int h = 0; h < 32; ++h) {
            pv[h] = __uint_as_float(u0[h]);
            pv[32 + h] = __uint_as_float(u1[h]);
          }
          warp_reduce_scatter64<false>(pv, lane);
          lsum0 += pv[0];
          lsum1 += pv[1];
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&bar.p_ready[gs & 1]);
      }
      // ---- epilogue of this token
      ss.wred[sw][2 * lane] = lsum0;
      ss.wred[sw][2 * lane + 1] = lsum1;
      softmax_bar();
      if (tid < kH) {  // per-head row sum -> 1/l (kept in ss.alpha) and log-sum-exp
        const float l = ss.wred[0][tid] + ss.wred[1][tid] + ss.wred[2][tid] + ss.wred[3][tid];
        ss.alpha[tid] = 1.0f / l;
        if (p.lse) p.lse[(size_t)tok * kH + tid] = (ss.m_ref[tid] + __log2f(l)) * 0.69314718055994531f;
      }
      softmax_bar();
      ok = mbar_wait(&bar.o_full[ob], (it >> 1) & 1, &abort_flag, p.err) && ok;
      tc_fence_after();
      {
        __nv_bfloat16* ob16 = reinterpret_cast<__nv_bfloat16*>(obase);
#pragma unroll
        for (int hv = 0; hv < 2; ++hv) {
          const int dv = hv * 128 + kl;  // this lane's d_v row of O^T
          uint32_t u0[32], u1[32];
          tmem_ld32_nowait(tmem + lane_off + ob * 128 + hv * kH, u0);
          tmem_ld32_nowait(tmem + lane_off + ob * 128 + hv * kH + 32, u1);
          tmem_wait_ld_regs2(u0, u1);
#pragma unroll
          for (int h4 = 0; h4 < 16; ++h4) {
            const float4 il = *reinterpret_cast<const float4*>(&ss.alpha[h4 * 4]);
            const float inv[4] = {il.x, il.y, il.z, il.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int h = h4 * 4 + q;
              const float o = __uint_as_float(h < 32 ? u0[h] : u1[h - 32]) * inv[q];
              ob16[(size_t)h * kD + dv] = __float2bfloat16_rn(o);
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&bar.o_empty[ob]);
      softmax_bar();  // wred / m_ref are rewritten by the next token; the row has been read
      refill_idx_row(p, bar, sIdx_a, buf, i, tok + 2 * gridDim.x, tid, abort_flag, ok);
      g += J;
      ++it;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) tmem_dealloc(tmem, 512);
}

int num_sms_current_device() {
  static std::mutex mu;
  static int cache[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  std::lock_guard<std::mutex> lock(mu);
  if (!cache[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    cache[dev] = n;
  }
  return cache[dev];
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
  if ((long long)B * Lq > 2147483647LL || (long long)B * Lk > 2147483647LL) return HCADSA_ERR_UNSUPPORTED;
  CUtensorMap mq;
  {
    const uint64_t dims[3] = {(uint64_t)kD, (uint64_t)kH, (uint64_t)B * Lq};
    const uint64_t strides[2] = {(uint64_t)kD * 2, (uint64_t)kH * kD * 2};
    const uint32_t box[3] = {64, (uint32_t)kH, 1};
    if (!encode_tmap_bf16(&mq, 3, const_cast<hcadsa_bf16*>(Q), dims, strides, box, true)) return HCADSA_ERR_CUDA;
  }
  Params p;
  p.K = K;
  p.V = V;
  p.idx = idx;
  p.O = O;
  p.lse = lse;
  p.err = device_error_ptr();
  p.n_tok = B * Lq;
  p.Lq = Lq;
  p.Lk = Lk;
  p.k = k;
  p.scale_log2 = scale * 1.4426950408889634f;
  if (cudaFuncSetAttribute(dsa_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) != cudaSuccess)
    return HCADSA_ERR_CUDA;
  const int sms = num_sms_current_device();
  if (sms <= 0) return HCADSA_ERR_CUDA;
  const int grid = p.n_tok < sms ? p.n_tok : sms;
  dsa_attn_kernel<<<grid, kThreads, kSmemBytes, as_stream(stream)>>>(mq, p);
  return launch_status();
}
