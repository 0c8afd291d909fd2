// dsa_indexer.cu -- DSA lightning indexer and per-query top-k selection.
//
// The pages ("Hybrid sparse attention, 1/7 full context access", mirrorspeed and
// besthub pages) describe "a lightweight indexer to score historical positions for
// each query" whose top-k positions receive attention.  The indexer form this library
// fixes: score[t,s] = sum_j w_idx[j] * <q_idx[t,j,:], k_idx[s,:]>, exact int32, over
// candidates s <= t; top-k by (score desc, position asc), written ascending, -1 padded.
//
// Three kernels:
//   * score_tiled_kernel   -- prefill: 128 queries x 128 keys per tile on the int8 tensor
//                             path (mma.sync m16n8k32 s8), one accumulator per indexer head,
//                             weighted in int32; writes int32 score rows to the workspace.
//   * score_stream_kernel  -- decode / few queries: one thread per key, dp4a, reading k_idx
//                             exactly once (HBM stream).
//   * select_kernel        -- one thread block per query row: exact radix select of the
//                             k-th largest score over the row (staged in shared memory when it
//                             fits), then an ordered compaction so ties go to lower positions
//                             and the output is ascending.
#include <cuda_bf16.h>

#include <mutex>

#include "host_common.h"
#include "ptx.cuh"

namespace hcadsa {
namespace {

constexpr int kDIdx = 64;   // indexer head dim
constexpr int kHIdx = 4;    // indexer heads
constexpr int kQTile = 128;
constexpr int kKTile = 128;
constexpr int kKeyTilesPerCta = 8;
constexpr int kARow = kHIdx * kDIdx + 16;  // padded bytes per query row in smem (bank-conflict free)
constexpr int kBRow = kDIdx + 16;          // padded bytes per key row in smem

__host__ __device__ inline long long round_up(long long x, long long m) { return (x + m - 1) / m * m; }

// Row stride (in int32 scores) of the workspace score matrix.
__host__ __device__ inline long long score_row_stride(int Lq, int q_offset, int Lk) {
  long long n_max = (long long)q_offset + Lq;  // candidates of the last query
  if (n_max > Lk) n_max = Lk;
  if (n_max < 1) n_max = 1;
  return round_up(n_max, kKTile);
}

__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool valid) {
  const uint32_t d = smem_u32(dst);
  const int n = valid ? 16 : 0;  // src-size 0 -> zero fill
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

__device__ __forceinline__ void mma_s8_16832(int (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// ------------------------------------------------------------------ tiled scorer (prefill)
//
// grid.x = key chunks of kKeyTilesPerCta*128 keys, grid.y = query tiles, grid.z = B.
// 8 warps; warp w owns query rows [16w, 16w+16) of the tile and all 128 keys.
__global__ void __launch_bounds__(256) score_tiled_kernel(const int8_t* __restrict__ q_idx,
                                                          const int8_t* __restrict__ k_idx,
                                                          const int32_t* __restrict__ w_idx,
                                                          int32_t* __restrict__ scores, int Lq, int q_offset,
                                                          int Lk, long long row_stride) {
  const int b = blockIdx.z;
  const int r0 = blockIdx.y * kQTile;
  const int t_last = q_offset + min(r0 + kQTile, Lq) - 1;  // largest query position in the tile
  const int n_hi = min(t_last + 1, Lk);                     // keys needed by the tile: [0, n_hi)
  const int s_begin = blockIdx.x * kKeyTilesPerCta * kKTile;
  if (s_begin >= n_hi) return;
  const int s_end = min(s_begin + kKeyTilesPerCta * kKTile, n_hi);

  extern __shared__ __align__(16) int8_t score_smem[];
  int8_t* sA = score_smem;                                   // [kQTile][kARow]
  int8_t (*sB)[kKTile * kBRow] = reinterpret_cast<int8_t (*)[kKTile * kBRow]>(score_smem + kQTile * kARow);
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int g = lane / 4, c4 = lane % 4;

  int w[kHIdx];
#pragma unroll
  for (int j = 0; j < kHIdx; ++j) w[j] = w_idx[j];

  // query tile: 128 rows x 256 bytes = 2048 chunks of 16 B
  const int8_t* qbase = q_idx + ((size_t)b * Lq + r0) * (kHIdx * kDIdx);
  for (int ch = tid; ch < kQTile * 16; ch += 256) {
    const int row = ch / 16, part = ch % 16;
    const bool ok = r0 + row < Lq;
    cp_async16(sA + row * kARow + part * 16, ok ? qbase + (size_t)row * 256 + part * 16 : qbase, ok);
  }
  auto load_keys = [&](int buf, int s0) {
    const int8_t* kb = k_idx + (size_t)b * Lk * kDIdx;
    for (int ch = tid; ch < kKTile * 4; ch += 256) {
      const int row = ch / 4, part = ch % 4;
      const bool ok = s0 + row < Lk;
      cp_async16(sB[buf] + row * kBRow + part * 16, ok ? kb + (size_t)(s0 + row) * kDIdx + part * 16 : kb, ok);
    }
  };
  load_keys(0, s_begin);
  cp_async_commit();

  int buf = 0;
  for (int s0 = s_begin; s0 < s_end; s0 += kKTile, buf ^= 1) {
    if (s0 + kKTile < s_end) load_keys(buf ^ 1, s0 + kKTile);
    cp_async_commit();
    cp_async_wait_1();
    __syncthreads();

    int total[16][4];
#pragma unroll
    for (int n = 0; n < 16; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) total[n][e] = 0;

    const int8_t* arow0 = sA + (warp * 16 + g) * kARow;
    const int8_t* arow8 = arow0 + 8 * kARow;
#pragma unroll
    for (int j = 0; j < kHIdx; ++j) {
      int acc[16][4];
#pragma unroll
      for (int n = 0; n < 16; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[n][e] = 0;
#pragma unroll
      for (int kk = 0; kk < 2; ++kk) {
        const int ka = j * kDIdx + kk * 32 + c4 * 4;
        uint32_t a[4];
        a[0] = *reinterpret_cast<const uint32_t*>(arow0 + ka);
        a[1] = *reinterpret_cast<const uint32_t*>(arow8 + ka);
        a[2] = *reinterpret_cast<const uint32_t*>(arow0 + ka + 16);
        a[3] = *reinterpret_cast<const uint32_t*>(arow8 + ka + 16);
#pragma unroll
        for (int n = 0; n < 16; ++n) {
          const int8_t* brow = sB[buf] + (n * 8 + g) * kBRow + kk * 32 + c4 * 4;
          uint32_t bb[2];
          bb[0] = *reinterpret_cast<const uint32_t*>(brow);
          bb[1] = *reinterpret_cast<const uint32_t*>(brow + 16);
          mma_s8_16832(acc[n], a, bb);
        }
      }
#pragma unroll
      for (int n = 0; n < 16; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) total[n][e] += w[j] * acc[n][e];
    }

    // write: rows (warp*16 + g) and (+8), columns s0 + n*8 + 2*c4 (+1)
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int r = r0 + warp * 16 + g + half * 8;
      if (r < Lq) {
        int32_t* dst = scores + ((size_t)b * Lq + r) * row_stride + s0 + 2 * c4;
#pragma unroll
        for (int n = 0; n < 16; ++n)
          *reinterpret_cast<int2*>(dst + n * 8) = make_int2(total[n][2 * half], total[n][2 * half + 1]);
      }
    }
    __syncthreads();
  }
}

// ------------------------------------------------------------------ streaming scorer (decode)
//
// grid.x = key blocks, grid.y = B * Lq query rows.  Each thread scores kKeysPerThread keys.
constexpr int kStreamThreads = 256;
constexpr int kKeysPerThread = 4;

__global__ void __launch_bounds__(kStreamThreads) score_stream_kernel(const int8_t* __restrict__ q_idx,
                                                                     const int8_t* __restrict__ k_idx,
                                                                     const int32_t* __restrict__ w_idx,
                                                                     int32_t* __restrict__ scores, int Lq,
                                                                     int q_offset, int Lk, long long row_stride) {
  const int row = blockIdx.y;
  const int b = row / Lq, r = row % Lq;
  const int n = min(q_offset + r + 1, Lk);
  __shared__ int sq[kHIdx * kDIdx / 4];
  __shared__ int sw[kHIdx];
  if (threadIdx.x < kHIdx * kDIdx / 4)
    sq[threadIdx.x] = reinterpret_cast<const int*>(q_idx + (size_t)row * kHIdx * kDIdx)[threadIdx.x];
  if (threadIdx.x < kHIdx) sw[threadIdx.x] = w_idx[threadIdx.x];
  __syncthreads();
  int q[kHIdx * kDIdx / 4];
#pragma unroll
  for (int i = 0; i < kHIdx * kDIdx / 4; ++i) q[i] = sq[i];
  const int s_base = blockIdx.x * kStreamThreads * kKeysPerThread + threadIdx.x;
  const int8_t* kb = k_idx + (size_t)b * Lk * kDIdx;
  int32_t* out = scores + (size_t)row * row_stride;
  uint4 kv[kKeysPerThread][4];
#pragma unroll
  for (int u = 0; u < kKeysPerThread; ++u) {
    const int s = s_base + u * kStreamThreads;
    if (s < n) {
      const uint4* kp = reinterpret_cast<const uint4*>(kb + (size_t)s * kDIdx);
#pragma unroll
      for (int v = 0; v < 4; ++v) kv[u][v] = kp[v];
    }
  }
#pragma unroll
  for (int u = 0; u < kKeysPerThread; ++u) {
    const int s = s_base + u * kStreamThreads;
    if (s < n) {
      const int* kw = reinterpret_cast<const int*>(&kv[u][0]);
      int total = 0;
#pragma unroll
      for (int j = 0; j < kHIdx; ++j) {
        int dot = 0;
#pragma unroll
        for (int i = 0; i < kDIdx / 4; ++i) dot = __dp4a(q[j * (kDIdx / 4) + i], kw[i], dot);
        total += sw[j] * dot;
      }
      out[s] = total;
    }
  }
}

// ------------------------------------------------------------------ selection
constexpr int kSelThreads = 512;
constexpr int kSelItems = 4;                 // consecutive elements per thread per chunk
constexpr int kSelChunk = kSelThreads * kSelItems;
constexpr int kRadixBits = 11;
constexpr int kRadixBins = 1 << kRadixBits;  // 2048
constexpr int kSelSmemCap = 40960;           // row entries staged in shared memory (160 KB)

struct SelShared {
  unsigned int hist[kRadixBins];
  int warp_tot[kSelThreads / 32];
  int warp_tot2[kSelThreads / 32];
  int bcast[4];
};

// Block-wide exclusive prefix sum of one int per thread; returns the exclusive prefix
// and writes the block total to *total.
__device__ __forceinline__ int block_exclusive_scan(int v, int* warp_tot, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tot[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int t = lane < kSelThreads / 32 ? warp_tot[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    if (lane < kSelThreads / 32) warp_tot[lane] = t;  // inclusive
  }
  __syncthreads();
  const int warp_excl = warp == 0 ? 0 : warp_tot[warp - 1];
  *total = warp_tot[kSelThreads / 32 - 1];
  __syncthreads();
  return warp_excl + x - v;
}

template <bool kInSmem>
__device__ __forceinline__ int load_score(const int* row_smem, const int* row_gmem, int i) {
  return kInSmem ? row_smem[i] : __ldcg(row_gmem + i);
}

template <bool kInSmem>
__device__ void select_row(const int* __restrict__ row_g, int* row_s, int n, int k, int32_t* __restrict__ out,
                           SelShared& sh) {
  const int tid = threadIdx.x;
  // ---- stage + min/max
  int mn = INT_MAX, mx = INT_MIN;
  for (int i = tid; i < n; i += kSelThreads) {
    const int v = __ldcg(row_g + i);
    if (kInSmem) row_s[i] = v;
    mn = min(mn, v);
    mx = max(mx, v);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  if ((tid & 31) == 0) {
    sh.warp_tot[tid >> 5] = mn;
    sh.warp_tot2[tid >> 5] = mx;
  }
  __syncthreads();
  if (tid == 0) {
    int a = INT_MAX, c = INT_MIN;
    for (int i = 0; i < kSelThreads / 32; ++i) {
      a = min(a, sh.warp_tot[i]);
      c = max(c, sh.warp_tot2[i]);
    }
    sh.bcast[0] = a;
    sh.bcast[1] = c;
  }
  __syncthreads();
  const int vmin = sh.bcast[0];
  const unsigned range = (unsigned)sh.bcast[1] - (unsigned)vmin;
  __syncthreads();

  // ---- radix select on u = score - vmin (unsigned, order preserving)
  int nbits = range == 0 ? 0 : 32 - __clz((int)range);
  unsigned prefix = 0, pmask = 0;
  int remaining = k;  // rank (1-based from the top) still to locate among prefix matches
  while (nbits > 0) {
    const int dbits = nbits < kRadixBits ? nbits : kRadixBits;
    const int lo = nbits - dbits;
    const unsigned dmask = (1u << dbits) - 1u;
    for (int i = tid; i < (1 << dbits); i += kSelThreads) sh.hist[i] = 0;
    __syncthreads();
    for (int i = tid; i < n; i += kSelThreads) {
      const unsigned u = (unsigned)load_score<kInSmem>(row_s, row_g, i) - (unsigned)vmin;
      if ((u & pmask) == prefix) atomicAdd(&sh.hist[(u >> lo) & dmask], 1u);
    }
    __syncthreads();
    // find the bin holding the remaining-th largest: scan bins from the top
    const int nb = 1 << dbits;
    const int per = (nb + kSelThreads - 1) / kSelThreads;  // bins per thread (<= 4)
    const int top = nb - 1 - tid * per;                   // this thread covers bins top, top-1, ...
    int cnt = 0;
    for (int q = 0; q < per; ++q)
      if (top - q >= 0) cnt += (int)sh.hist[top - q];
    int tot;
    const int above = block_exclusive_scan(cnt, sh.warp_tot, &tot);  // elements in higher bins
    if (above < remaining && above + cnt >= remaining) {
      int acc = above;
      for (int q = 0; q < per; ++q) {
        const int bin = top - q;
        const int c = (int)sh.hist[bin];
        if (acc + c >= remaining) {
          sh.bcast[2] = bin;
          sh.bcast[3] = remaining - acc;
          break;
        }
        acc += c;
      }
    }
    __syncthreads();
    prefix |= (unsigned)sh.bcast[2] << lo;
    pmask |= dmask << lo;
    remaining = sh.bcast[3];
    nbits = lo;
    __syncthreads();
  }
  const unsigned thr = prefix;   // u of the k-th largest
  const int need_eq = remaining; // how many elements equal to thr are taken (lowest positions)

  // ---- ordered compaction
  int written = 0, eq_seen = 0;
  for (int base = 0; base < n && written < k; base += kSelChunk) {
    const int i0 = base + tid * kSelItems;
    unsigned u[kSelItems];
    int n_eq = 0;
#pragma unroll
    for (int q = 0; q < kSelItems; ++q) {
      const int i = i0 + q;
      u[q] = i < n ? (unsigned)load_score<kInSmem>(row_s, row_g, i) - (unsigned)vmin : 0u;
      if (i < n && u[q] == thr) ++n_eq;
    }
    int eq_tot;
    const int eq_before = eq_seen + block_exclusive_scan(n_eq, sh.warp_tot, &eq_tot);
    bool take[kSelItems];
    int n_take = 0, eq_rank = eq_before;
#pragma unroll
    for (int q = 0; q < kSelItems; ++q) {
      const int i = i0 + q;
      bool t = false;
      if (i < n) {
        if (u[q] > thr) t = true;
        else if (u[q] == thr) t = (eq_rank++ < need_eq);
      }
      take[q] = t;
      n_take += t;
    }
    int take_tot;
    int pos = written + block_exclusive_scan(n_take, sh.warp_tot, &take_tot);
#pragma unroll
    for (int q = 0; q < kSelItems; ++q)
      if (take[q] && pos < k) out[pos++] = i0 + q;
    written += take_tot;
    eq_seen += eq_tot;
  }
  for (int i = written + tid; i < k; i += kSelThreads) out[i] = -1;
}

__global__ void __launch_bounds__(kSelThreads) select_kernel(const int32_t* __restrict__ scores,
                                                              int32_t* __restrict__ idx, int Lq, int q_offset,
                                                              int Lk, int k, long long row_stride) {
  extern __shared__ __align__(16) int sel_row[];
  __shared__ SelShared sh;
  const int row = blockIdx.x;
  const int r = row % Lq;
  const int n = max(0, min(q_offset + r + 1, Lk));
  int32_t* out = idx + (size_t)row * k;
  if (n <= k) {
    for (int i = threadIdx.x; i < k; i += kSelThreads) out[i] = i < n ? i : -1;
    return;
  }
  const int* row_g = scores + (size_t)row * row_stride;
  if (n <= kSelSmemCap)
    select_row<true>(row_g, sel_row, n, k, out, sh);
  else
    select_row<false>(row_g, nullptr, n, k, out, sh);
}

}  // namespace
}  // namespace hcadsa

extern "C" size_t dsa_index_topk_workspace_size(int B, int Lq, int q_offset, int Lk, int k) {
  using namespace hcadsa;
  (void)k;
  if (B <= 0 || Lq <= 0 || Lk <= 0 || q_offset < 0) return 0;
  return (size_t)B * (size_t)Lq * (size_t)score_row_stride(Lq, q_offset, Lk) * sizeof(int32_t);
}

extern "C" hcadsa_status dsa_index_topk(const int8_t* q_idx, const int8_t* k_idx, const int32_t* w_idx,
                                        int32_t* idx, void* ws, size_t ws_bytes, int B, int Lq, int q_offset,
                                        int Lk, int H_idx, int d_idx, int k, hcadsa_stream stream) {
  using namespace hcadsa;
  if (!q_idx || !k_idx || !w_idx || !idx) return HCADSA_ERR_NULL;
  if (B < 0 || Lq < 0 || Lk < 0 || q_offset < 0 || k <= 0) return HCADSA_ERR_SHAPE;
  if (H_idx != kHIdx || d_idx != kDIdx || k > 4096) return HCADSA_ERR_UNSUPPORTED;
  if ((long long)q_offset + Lq > 2147483647LL - 1 || (long long)B * Lq > 2147483647LL) return HCADSA_ERR_UNSUPPORTED;
  if (!aligned16(q_idx) || !aligned16(k_idx) || !aligned16(w_idx) || !aligned16(idx)) return HCADSA_ERR_ALIGN;
  if (B == 0 || Lq == 0) return HCADSA_OK;
  cudaStream_t s = as_stream(stream);
  const bool need_scores = (long long)q_offset + Lq > k && Lk > k;  // some row has more than k candidates
  const long long stride = score_row_stride(Lq, q_offset, Lk);
  if (need_scores) {
    if (!ws) return HCADSA_ERR_WORKSPACE;
    if (!aligned16(ws)) return HCADSA_ERR_ALIGN;
    if (ws_bytes < dsa_index_topk_workspace_size(B, Lq, q_offset, Lk, k)) return HCADSA_ERR_WORKSPACE;
    int32_t* scores = static_cast<int32_t*>(ws);
    if (Lq >= 64) {
      const long long n_max = stride;
      dim3 grid((unsigned)((n_max + kKeyTilesPerCta * kKTile - 1) / (kKeyTilesPerCta * kKTile)),
                (unsigned)((Lq + kQTile - 1) / kQTile), (unsigned)B);
      if (grid.y > 65535u || grid.z > 65535u) return HCADSA_ERR_UNSUPPORTED;
      const int smem_tiled = kQTile * kARow + 2 * kKTile * kBRow;
      if (cudaFuncSetAttribute(score_tiled_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_tiled) !=
          cudaSuccess)
        return HCADSA_ERR_CUDA;
      score_tiled_kernel<<<grid, 256, smem_tiled, s>>>(q_idx, k_idx, w_idx, scores, Lq, q_offset, Lk, stride);
    } else {
      const long long n_max = stride;
      dim3 grid((unsigned)((n_max + kStreamThreads * kKeysPerThread - 1) / (kStreamThreads * kKeysPerThread)),
                (unsigned)(B * Lq));
      if (grid.y > 65535u) return HCADSA_ERR_UNSUPPORTED;
      score_stream_kernel<<<grid, kStreamThreads, 0, s>>>(q_idx, k_idx, w_idx, scores, Lq, q_offset, Lk, stride);
    }
    if (cudaGetLastError() != cudaSuccess) return HCADSA_ERR_CUDA;
  }
  const int smem = kSelSmemCap * (int)sizeof(int);
  if (cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return HCADSA_ERR_CUDA;
  select_kernel<<<(unsigned)(B * Lq), kSelThreads, smem, s>>>(need_scores ? static_cast<int32_t*>(ws) : nullptr,
                                                              idx, Lq, q_offset, Lk, k, stride);
  return launch_status();
}

// ---------------------------------------------------------------------------------------------
// dsa_index_topk_noalloc: the same indexer + top-k for callers that cannot allocate device
// memory.  The score rows live in a fixed array compiled into this library instead of a
// caller-provided workspace.
// ---------------------------------------------------------------------------------------------
namespace hcadsa {
namespace {

// Built-in score scratch: 16,777,216 int32 scores = 64 MiB per device, resident from the
// moment the library's device code is loaded on a GPU until the process exits.
constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;
static __device__ __align__(256) int32_t g_noalloc_scores[kNoAllocScratchBytes / sizeof(int32_t)];

// Device address of g_noalloc_scores for the current device, looked up once per device.
// The name g_noalloc_scores is only a host-side stand-in in host code; kernels must be given
// the address that cudaGetSymbolAddress returns for the device they run on.
int32_t* noalloc_scratch_for_current_device() {
  static std::mutex mu;
  static int32_t* ptr_by_device[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!ptr_by_device[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scores) != cudaSuccess || !p) return nullptr;
    ptr_by_device[dev] = static_cast<int32_t*>(p);
  }
  return ptr_by_device[dev];
}

}  // namespace
}  // namespace hcadsa

extern "C" size_t dsa_index_topk_noalloc_max_scratch_bytes(void) { return hcadsa::kNoAllocScratchBytes; }

extern "C" hcadsa_status dsa_index_topk_noalloc(const int8_t* q_idx, const int8_t* k_idx, const int32_t* w_idx,
                                                int32_t* idx, int B, int Lq, int q_offset, int Lk, int H_idx,
                                                int d_idx, int k, hcadsa_stream stream) {
  using namespace hcadsa;
  if (!q_idx || !k_idx || !w_idx || !idx) return HCADSA_ERR_NULL;
  if (B < 0 || Lq < 0 || Lk < 0 || q_offset < 0 || k <= 0) return HCADSA_ERR_SHAPE;
  if (H_idx != kHIdx || d_idx != kDIdx || k > 4096) return HCADSA_ERR_UNSUPPORTED;
  if ((long long)q_offset + Lq > 2147483647LL - 1 || (long long)B * Lq > 2147483647LL) return HCADSA_ERR_UNSUPPORTED;
  if (!aligned16(q_idx) || !aligned16(k_idx) || !aligned16(w_idx) || !aligned16(idx)) return HCADSA_ERR_ALIGN;
  if (B == 0 || Lq == 0) return HCADSA_OK;
  const bool need_scores = (long long)q_offset + Lq > k && Lk > k;
  const long long stride = score_row_stride(Lq, q_offset, Lk);
  // size check first: a call that does not fit is refused before any CUDA call
  if (need_scores && dsa_index_topk_workspace_size(B, Lq, q_offset, Lk, k) > kNoAllocScratchBytes)
    return HCADSA_ERR_WORKSPACE;
  cudaStream_t s = as_stream(stream);
  int32_t* scores = nullptr;
  if (need_scores) {
    scores = noalloc_scratch_for_current_device();
    if (!scores) return HCADSA_ERR_CUDA;
    if (Lq >= 64) {
      dim3 grid((unsigned)((stride + kKeyTilesPerCta * kKTile - 1) / (kKeyTilesPerCta * kKTile)),
                (unsigned)((Lq + kQTile - 1) / kQTile), (unsigned)B);
      if (grid.y > 65535u || grid.z > 65535u) return HCADSA_ERR_UNSUPPORTED;
      const int smem_tiled = kQTile * kARow + 2 * kKTile * kBRow;
      if (cudaFuncSetAttribute(score_tiled_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_tiled) !=
          cudaSuccess)
        return HCADSA_ERR_CUDA;
      score_tiled_kernel<<<grid, 256, smem_tiled, s>>>(q_idx, k_idx, w_idx, scores, Lq, q_offset, Lk, stride);
    } else {
      dim3 grid((unsigned)((stride + kStreamThreads * kKeysPerThread - 1) / (kStreamThreads * kKeysPerThread)),
                (unsigned)(B * Lq));
      if (grid.y > 65535u) return HCADSA_ERR_UNSUPPORTED;
      score_stream_kernel<<<grid, kStreamThreads, 0, s>>>(q_idx, k_idx, w_idx, scores, Lq, q_offset, Lk, stride);
    }
    if (cudaGetLastError() != cudaSuccess) return HCADSA_ERR_CUDA;
  }
  const int smem = kSelSmemCap * (int)sizeof(int);
  if (cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return HCADSA_ERR_CUDA;
  select_kernel<<<(unsigned)(B * Lq), kSelThreads, smem, s>>>(scores, idx, Lq, q_offset, Lk, k, stride);
  return launch_status();
}
