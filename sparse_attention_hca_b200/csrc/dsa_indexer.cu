// dsa_indexer.cu -- DSA lightning indexer and per-query top-k selection.
//
// The pages (section "Hybrid sparse attention, 1/7 full context access" of the mirrorspeed
// page, and the besthub page) describe a small scoring network that rates every earlier
// position for each query; attention then covers only the best-rated k.  The indexer form this library
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
// Few query rows over very many keys (decode) would leave all but a handful of SMs idle in
// select_kernel, so those calls select with every SM instead:
//   * the streaming scorer also records each row's score range,
//   * hist_kernel          -- many CTAs per row: 2048-bin histogram of the row over that range,
//   * candidates_kernel    -- many CTAs per row: the bin b* holding the k-th largest score is
//                             found from the histogram; every key in a bin >= b* (a superset of
//                             the top k, at most kCandCap of them) is appended to a candidate
//                             list,
//   * finalize_kernel      -- one CTA per row: bitonic sort of the candidates by (score desc,
//                             position asc), the first k positions sorted ascending.  A row
//                             whose candidates overflow (e.g. massive ties) falls back to the
//                             exact single-CTA select of that row.
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

// Candidates of the query at position t: keys s < min((t + 1) / ratio, Lk).  ratio = 1 is DSA
// (every position up to and including t); ratio = blk is CSA over compressed entries (an entry
// is a candidate once its block of blk tokens is complete).
__host__ __device__ inline int n_cand(long long t, int ratio, int Lk) {
  long long n = (t + 1) / ratio;
  if (n > Lk) n = Lk;
  return n < 0 ? 0 : (int)n;
}

// Row stride (in int32 scores) of the workspace score matrix.
__host__ __device__ inline long long score_row_stride(int Lq, int q_offset, int Lk, int ratio) {
  long long n_max = n_cand((long long)q_offset + Lq - 1, ratio, Lk);  // candidates of the last query
  if (n_max < 1) n_max = 1;
  return round_up(n_max, kKTile);
}

// Multi-CTA selection for few rows over many keys: per-row state after the score rows.
constexpr int kHistBins = 2048;
constexpr int kCandCap = 8192;
constexpr int kSplitRowsMax = 64;       // at most this many query rows (B * Lq) ...
constexpr long long kSplitMinKeys = 32768;  // ... each over at least this many keys (row stride)
struct RowSel {
  int vmin, vmax;   // score range of the row (streaming scorer)
  int n_cand, pad;  // candidates appended (may exceed kCandCap: overflow)
  unsigned int hist[kHistBins];
};
__host__ __device__ inline bool use_split_select(int B, int Lq, int q_offset, int Lk, int ratio) {
  return (long long)B * Lq <= kSplitRowsMax && Lq < 64 && score_row_stride(Lq, q_offset, Lk, ratio) >= kSplitMinKeys;
}
// bytes after the score rows: RowSel per row, then kCandCap (u, position) pairs per row
__host__ __device__ inline long long split_select_bytes(int rows) {
  return (long long)rows * ((long long)sizeof(RowSel) + (long long)kCandCap * 8);
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
// grid.x = key blocks of kStreamKeysPerCta, grid.y = B * Lq query rows.
constexpr int kStreamThreads = 256;
constexpr int kStreamLoads = 8;                                          // 16-byte loads in flight per lane
constexpr int kStreamKeysPerIter = kStreamThreads / 4 * kStreamLoads;    // 512 keys per CTA iteration
constexpr int kStreamIters = 8;                                          // iterations per CTA
constexpr int kStreamKeysPerCta = kStreamKeysPerIter * kStreamIters;     // 4096

// Four lanes share one 64-byte key: lane l reads bytes 16*(l%4) .. +15 of key l/4 of its group
// of 8 keys, so each warp load instruction moves 512 contiguous bytes.  A lane dots its slice
// with the matching 16 bytes of each indexer head's query (dp4a), weights the 4 partial dots,
// and the 4 lanes of a key add their partial totals (all int32, exact).
__global__ void __launch_bounds__(kStreamThreads) score_stream_kernel(const int8_t* __restrict__ q_idx,
                                                                     const int8_t* __restrict__ k_idx,
                                                                     const int32_t* __restrict__ w_idx,
                                                                     int32_t* __restrict__ scores, int Lq,
                                                                     int q_offset, int Lk, int ratio,
                                                                     long long row_stride,
                                                                     RowSel* __restrict__ rowsel) {
  const int row = blockIdx.y;
  const int b = row / Lq, r = row % Lq;
  const int n = n_cand((long long)q_offset + r, ratio, Lk);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int part = lane & 3;  // 16-byte slice of the key
  int q[kHIdx][4];
  int w[kHIdx];
  {
    const int4* qrow = reinterpret_cast<const int4*>(q_idx + (size_t)row * kHIdx * kDIdx);
#pragma unroll
    for (int j = 0; j < kHIdx; ++j) {
      const int4 v = qrow[j * (kDIdx / 16) + part];
      q[j][0] = v.x;
      q[j][1] = v.y;
      q[j][2] = v.z;
      q[j][3] = v.w;
      w[j] = w_idx[j];
    }
  }
  const uint4* kb = reinterpret_cast<const uint4*>(k_idx + (size_t)b * Lk * kDIdx);
  int32_t* out = scores + (size_t)row * row_stride;
  int vmn = INT_MAX, vmx = INT_MIN;
  const int warp_s0 = blockIdx.x * kStreamKeysPerCta + warp * (8 * kStreamLoads);
  // key of load u in iteration it: warp_s0 + it*kStreamKeysPerIter + u*8 + lane/4
  auto load_iter = [&](uint4 (&kv)[kStreamLoads], int it) {
#pragma unroll
    for (int u = 0; u < kStreamLoads; ++u) {
      const int s = warp_s0 + it * kStreamKeysPerIter + u * 8 + (lane >> 2);
      kv[u] = s < n ? __ldcs(kb + (size_t)s * 4 + part) : make_uint4(0u, 0u, 0u, 0u);
    }
  };
  uint4 kv[2][kStreamLoads];
  load_iter(kv[0], 0);
#pragma unroll
  for (int it = 0; it < kStreamIters; ++it) {
    if (warp_s0 + it * kStreamKeysPerIter >= n) break;  // warp-uniform
    if (it + 1 < kStreamIters) load_iter(kv[(it + 1) & 1], it + 1);  // next iteration's keys in flight
#pragma unroll
    for (int u = 0; u < kStreamLoads; ++u) {
      const uint4 x = kv[it & 1][u];
      const int s = warp_s0 + it * kStreamKeysPerIter + u * 8 + (lane >> 2);
      int total = 0;
#pragma unroll
      for (int j = 0; j < kHIdx; ++j) {
        int dot = __dp4a(q[j][0], (int)x.x, 0);
        dot = __dp4a(q[j][1], (int)x.y, dot);
        dot = __dp4a(q[j][2], (int)x.z, dot);
        dot = __dp4a(q[j][3], (int)x.w, dot);
        total += w[j] * dot;
      }
      total += __shfl_xor_sync(0xffffffffu, total, 1);
      total += __shfl_xor_sync(0xffffffffu, total, 2);
      if (part == 0 && s < n) {
        out[s] = total;
        vmn = min(vmn, total);
        vmx = max(vmx, total);
      }
    }
  }
  if (rowsel) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      vmn = min(vmn, __shfl_xor_sync(0xffffffffu, vmn, o));
      vmx = max(vmx, __shfl_xor_sync(0xffffffffu, vmx, o));
    }
    if (lane == 0 && vmn <= vmx) {
      atomicMin(&rowsel[row].vmin, vmn);
      atomicMax(&rowsel[row].vmax, vmx);
    }
  }
}

// ------------------------------------------------------------------ selection
//
// One thread block per query row.  The row is staged in shared memory (when it fits) with
// coalesced 16-byte loads; then thread t owns the contiguous segment [t*E, t*E + E) of it,
// E odd so the 32 lanes of a warp read 32 different banks.  Radix select on u = score - min:
// 8-bit digits from the top, each counted into a per-warp histogram (contention only within a
// warp), summed, and the bin holding the k-th largest found by one warp.  The compaction then
// needs a single block scan of packed (count > threshold, count == threshold) pairs: a thread's
// output position is (greater elements before it) + min(equal elements before it, equal
// elements to take), so ties go to the lowest positions and the output is ascending.
constexpr int kSelThreads = 512;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kDigitBits = 8;
constexpr int kDigitBins = 1 << kDigitBits;
constexpr int kSelSmemCap = 40960;  // row entries staged in shared memory (160 KB)

struct SelShared {
  unsigned int hist[kSelWarps][kDigitBins];
  unsigned long long scan_warp[kSelWarps];
  int red_a[kSelWarps], red_b[kSelWarps];
  int bcast[4];
};

// Block-wide exclusive prefix sum of a 64-bit value per thread; returns the exclusive prefix
// and writes the block total to *total.
__device__ __forceinline__ unsigned long long block_exclusive_scan64(unsigned long long v, SelShared& sh,
                                                                     unsigned long long* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  unsigned long long x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sh.scan_warp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    unsigned long long t = lane < kSelWarps ? sh.scan_warp[lane] : 0ull;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned long long y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    if (lane < kSelWarps) sh.scan_warp[lane] = t;  // inclusive
  }
  __syncthreads();
  const unsigned long long before = warp == 0 ? 0ull : sh.scan_warp[warp - 1];
  *total = sh.scan_warp[kSelWarps - 1];
  return before + x - v;
}

// Stages row_g[c0, c0 + len) into row_s[0, len) with coalesced 16-byte loads (c0 % 4 == 0).
__device__ __forceinline__ void stage_chunk(const int* __restrict__ row_g, int* row_s, int c0, int len) {
  const int tid = threadIdx.x;
  const int n4 = len >> 2;
  const int4* src4 = reinterpret_cast<const int4*>(row_g + c0);  // 16-byte aligned: c0 % 4 == 0
  constexpr int kUnroll = 8;
  for (int base = tid; base < n4; base += kSelThreads * kUnroll) {
    int4 v[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int i4 = base + u * kSelThreads;
      v[u] = i4 < n4 ? __ldcg(src4 + i4) : make_int4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int i4 = base + u * kSelThreads;
      if (i4 < n4) reinterpret_cast<int4*>(row_s)[i4] = v[u];
    }
  }
  for (int i = (n4 << 2) + tid; i < len; i += kSelThreads) row_s[i] = __ldcg(row_g + c0 + i);
}

// kInSmem: the whole row is staged in row_s; otherwise the passes read global memory (strided,
// coalesced) and the ordered compaction walks the row in chunks staged through row_s.
template <bool kInSmem>
__device__ void select_row(const int* __restrict__ row_g, int* row_s, int n, int k, int32_t* __restrict__ out,
                           SelShared& sh) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (kInSmem) {
    stage_chunk(row_g, row_s, 0, n);
    __syncthreads();
  }
  auto at = [&](int i) { return kInSmem ? row_s[i] : __ldcg(row_g + i); };

  // ---- min / max (strided: coalesced in global memory, conflict-free in shared memory)
  int mn = INT_MAX, mx = INT_MIN;
  for (int i = tid; i < n; i += kSelThreads) {
    const int v = at(i);
    mn = min(mn, v);
    mx = max(mx, v);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  if (lane == 0) {
    sh.red_a[warp] = mn;
    sh.red_b[warp] = mx;
  }
  __syncthreads();
  if (warp == 0) {
    int a = lane < kSelWarps ? sh.red_a[lane] : INT_MAX, c = lane < kSelWarps ? sh.red_b[lane] : INT_MIN;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      a = min(a, __shfl_xor_sync(0xffffffffu, a, o));
      c = max(c, __shfl_xor_sync(0xffffffffu, c, o));
    }
    if (lane == 0) {
      sh.bcast[0] = a;
      sh.bcast[1] = c;
    }
  }
  __syncthreads();
  const int vmin = sh.bcast[0];
  const unsigned range = (unsigned)sh.bcast[1] - (unsigned)vmin;

  // ---- radix select on u = score - vmin (unsigned, order preserving)
  int nbits = range == 0 ? 0 : 32 - __clz((int)range);
  unsigned prefix = 0, pmask = 0;
  int remaining = k;  // rank (1 = largest) still to locate among the prefix matches
  if (kInSmem) {
    // 11-bit digits counted into one block-wide 2048-bin histogram (the per-warp histograms'
    // storage): two passes cover the 18-bit score range of the indexer's usual inputs
    constexpr int kBins = 2048, kPer = kBins / kSelThreads;
    unsigned int* hb = &sh.hist[0][0];
    while (nbits > 0) {
      const int dbits = nbits < 11 ? nbits : 11;
      const int lo = nbits - dbits;
      const unsigned dmask = (1u << dbits) - 1u;
      for (int b = tid; b < kBins; b += kSelThreads) hb[b] = 0;
      __syncthreads();
      for (int i = tid; i < n; i += kSelThreads) {
        const unsigned u = (unsigned)row_s[i] - (unsigned)vmin;
        if ((u & pmask) == prefix) atomicAdd(&hb[(u >> lo) & dmask], 1u);
      }
      __syncthreads();
      // thread t owns bins kBins-1-(t*kPer+q), q < kPer: counts from the top down
      int cnt[kPer], tot = 0;
#pragma unroll
      for (int q = 0; q < kPer; ++q) {
        cnt[q] = (int)hb[kBins - 1 - (tid * kPer + q)];
        tot += cnt[q];
      }
      int incl = tot;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      if (lane == 31) sh.red_a[warp] = incl;
      __syncthreads();
      for (int w = 0; w < warp; ++w) incl += sh.red_a[w];
      const int above = incl - tot;
      if (above < remaining && incl >= remaining) {
        int acc = above;
#pragma unroll
        for (int q = 0; q < kPer; ++q) {
          if (acc + cnt[q] >= remaining) {
            sh.bcast[2] = kBins - 1 - (tid * kPer + q);
            sh.bcast[3] = remaining - acc;
            break;
          }
          acc += cnt[q];
        }
      }
      __syncthreads();
      prefix |= (unsigned)sh.bcast[2] << lo;
      pmask |= dmask << lo;
      remaining = sh.bcast[3];
      nbits = lo;
      __syncthreads();  // red_a and the histogram are rewritten by the next pass
    }
  } else {
    while (nbits > 0) {
      const int dbits = nbits < kDigitBits ? nbits : kDigitBits;
      const int lo = nbits - dbits;
      const unsigned dmask = (1u << dbits) - 1u;
      unsigned int* hw = sh.hist[warp];
      for (int b = lane; b < kDigitBins; b += 32) hw[b] = 0;
      __syncwarp();
      for (int i = tid; i < n; i += kSelThreads) {
        const unsigned u = (unsigned)at(i) - (unsigned)vmin;
        if ((u & pmask) == prefix) atomicAdd(&hw[(u >> lo) & dmask], 1u);
      }
      __syncthreads();
      if (warp == 0) {
        // lane l owns bins 255 - 8l - q, q = 0..7: counts from the top down
        int cnt[8];
        int lane_tot = 0;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int bin = kDigitBins - 1 - (lane * 8 + q);
          int c = 0;
          for (int w = 0; w < kSelWarps; ++w) c += (int)sh.hist[w][bin];
          cnt[q] = c;
          lane_tot += c;
        }
        int incl = lane_tot;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        const int above = incl - lane_tot;  // elements in higher bins than this lane's
        if (above < remaining && incl >= remaining) {
          int acc = above;
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            if (acc + cnt[q] >= remaining) {
              sh.bcast[2] = kDigitBins - 1 - (lane * 8 + q);
              sh.bcast[3] = remaining - acc;
              break;
            }
            acc += cnt[q];
          }
        }
      }
      __syncthreads();
      prefix |= (unsigned)sh.bcast[2] << lo;
      pmask |= dmask << lo;
      remaining = sh.bcast[3];
      nbits = lo;
      __syncthreads();  // histograms are cleared again by the next pass
    }
  }
  const unsigned thr = prefix;    // u of the k-th largest
  const int need_eq = remaining;  // elements equal to thr that are kept (lowest positions first)

  // ---- ordered compaction: per chunk, one scan of packed (greater, equal) counts; thread t owns
  // the contiguous segment [t*E, t*E + E) of the chunk, E odd so a warp hits 32 banks
  const int chunk = kInSmem ? n : kSelSmemCap;
  int written_gt = 0, eq_seen = 0;
  for (int c0 = 0; c0 < n; c0 += chunk) {
    const int len = min(chunk, n - c0);
    if (!kInSmem) {
      __syncthreads();  // previous chunk fully consumed
      stage_chunk(row_g, row_s, c0, len);
      __syncthreads();
    }
    const int E = ((len + kSelThreads - 1) / kSelThreads) | 1;
    const int s0 = min(tid * E, len), s1 = min(s0 + E, len);
    int gt = 0, eq = 0;
    for (int i = s0; i < s1; ++i) {
      const unsigned u = (unsigned)row_s[i] - (unsigned)vmin;
      gt += u > thr;
      eq += u == thr;
    }
    unsigned long long tot;
    const unsigned long long before =
        block_exclusive_scan64(((unsigned long long)gt << 32) | (unsigned)eq, sh, &tot);
    const int gt_before = written_gt + (int)(before >> 32);
    const int eq_before = eq_seen + (int)(before & 0xffffffffu);
    int pos = gt_before + min(eq_before, need_eq);
    int eq_rank = eq_before;
    for (int i = s0; i < s1; ++i) {
      const unsigned u = (unsigned)row_s[i] - (unsigned)vmin;
      if (u > thr) {
        out[pos++] = c0 + i;
      } else if (u == thr) {
        if (eq_rank < need_eq) out[pos++] = c0 + i;
        ++eq_rank;
      }
    }
    written_gt += (int)(tot >> 32);
    eq_seen += (int)(tot & 0xffffffffu);
  }
}

__global__ void __launch_bounds__(kSelThreads) select_kernel(const int32_t* __restrict__ scores,
                                                              int32_t* __restrict__ idx, int Lq, int q_offset,
                                                              int Lk, int ratio, int k, long long row_stride) {
  extern __shared__ __align__(16) int sel_row[];
  __shared__ SelShared sh;
  const int row = blockIdx.x;
  const int r = row % Lq;
  const int n = n_cand((long long)q_offset + r, ratio, Lk);
  int32_t* out = idx + (size_t)row * k;
  if (n <= k) {
    for (int i = threadIdx.x; i < k; i += kSelThreads) out[i] = i < n ? i : -1;
    return;
  }
  const int* row_g = scores + (size_t)row * row_stride;
  if (n <= kSelSmemCap)
    select_row<true>(row_g, sel_row, n, k, out, sh);
  else
    select_row<false>(row_g, sel_row, n, k, out, sh);  // sel_row stages compaction chunks
}


// ------------------------------------------------------------------ multi-CTA selection (few rows)

constexpr int kSplitChunk = 16384;  // scores per CTA in hist_kernel / candidates_kernel

__global__ void __launch_bounds__(256) rowsel_init_kernel(RowSel* __restrict__ rs) {
  RowSel& r = rs[blockIdx.x];
  if (threadIdx.x == 0) {
    r.vmin = INT_MAX;
    r.vmax = INT_MIN;
    r.n_cand = 0;
    r.pad = 0;
  }
  for (int i = threadIdx.x; i < kHistBins; i += 256) r.hist[i] = 0;
}

// bins of u = score - vmin: u >> shift, shift such that the whole range fits in kHistBins bins
__device__ __forceinline__ int hist_shift(unsigned range) {
  const int bits = range == 0u ? 0 : 32 - __clz(range);
  return bits > 11 ? bits - 11 : 0;
}

__global__ void __launch_bounds__(256) hist_kernel(const int32_t* __restrict__ scores, RowSel* __restrict__ rs,
                                                   int Lq, int q_offset, int Lk, int ratio, int k,
                                                   long long row_stride) {
  const int row = blockIdx.y, r = row % Lq;
  const int n = n_cand((long long)q_offset + r, ratio, Lk);
  const int c0 = blockIdx.x * kSplitChunk;
  if (n <= k || c0 >= n) return;
  __shared__ unsigned int h[kHistBins];
  for (int i = threadIdx.x; i < kHistBins; i += 256) h[i] = 0;
  __syncthreads();
  const int vmin = rs[row].vmin;
  const int sh = hist_shift((unsigned)rs[row].vmax - (unsigned)vmin);
  const int* rowp = scores + (size_t)row * row_stride;
  const int c1 = min(c0 + kSplitChunk, n);
  // 4 scores per thread per load (rows are 16-byte aligned: c0 and the row stride are multiples of 128)
  for (int base = c0; base < c1; base += 256 * 4 * 4) {
    int4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = base + (u * 256 + threadIdx.x) * 4;
      v[u] = i < c1 ? __ldcg(reinterpret_cast<const int4*>(rowp + i)) : make_int4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = base + (u * 256 + threadIdx.x) * 4;
      const int e[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (i + q < c1) atomicAdd(&h[((unsigned)e[q] - (unsigned)vmin) >> sh], 1u);
    }
  }
  __syncthreads();
  for (int b = threadIdx.x; b < kHistBins; b += 256)
    if (h[b]) atomicAdd(&rs[row].hist[b], h[b]);
}

// The bin holding the k-th largest score of a row (bins counted from the top) and the number of
// keys in the bins above it.  Whole block of kThreads threads; results in *bin_sh / *above_sh.
template <int kThreads>
__device__ __forceinline__ void threshold_bin(const unsigned int* __restrict__ hist, int k, int* wsum_sh, int* bin_sh,
                                              int* above_sh) {
  constexpr int kPer = kHistBins / kThreads;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int cnt[kPer], tot = 0;
#pragma unroll
  for (int q = 0; q < kPer; ++q) {
    cnt[q] = (int)hist[kHistBins - 1 - (tid * kPer + q)];
    tot += cnt[q];
  }
  int incl = tot;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) wsum_sh[warp] = incl;
  __syncthreads();
  int before_warp = 0;
  for (int w = 0; w < warp; ++w) before_warp += wsum_sh[w];
  incl += before_warp;
  const int above = incl - tot;
  if (above < k && incl >= k) {
    int acc = above;
#pragma unroll
    for (int q = 0; q < kPer; ++q) {
      if (acc + cnt[q] >= k) {
        *bin_sh = kHistBins - 1 - (tid * kPer + q);
        *above_sh = acc;
        break;
      }
      acc += cnt[q];
    }
  }
  __syncthreads();
}

__global__ void __launch_bounds__(256) candidates_kernel(const int32_t* __restrict__ scores, RowSel* __restrict__ rs,
                                                         int2* __restrict__ cand, int Lq, int q_offset, int Lk,
                                                         int ratio, int k, long long row_stride) {
  const int row = blockIdx.y, r = row % Lq;
  const int n = n_cand((long long)q_offset + r, ratio, Lk);
  const int c0 = blockIdx.x * kSplitChunk;
  if (n <= k || c0 >= n) return;
  const int tid = threadIdx.x, lane = tid & 31;
  __shared__ int wsum[8];
  __shared__ int bstar, above_b;
  threshold_bin<256>(rs[row].hist, k, wsum, &bstar, &above_b);
  const unsigned b_lo = (unsigned)bstar;
  const int vmin = rs[row].vmin;
  const int sh = hist_shift((unsigned)rs[row].vmax - (unsigned)vmin);
  const int* rowp = scores + (size_t)row * row_stride;
  int2* cr = cand + (size_t)row * kCandCap;
  const int c1 = min(c0 + kSplitChunk, n);
  for (int base = c0; base < c1; base += 256 * 4 * 4) {  // warp-uniform trip count
    int4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = base + (u * 256 + tid) * 4;
      v[u] = i < c1 ? __ldcg(reinterpret_cast<const int4*>(rowp + i)) : make_int4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = base + (u * 256 + tid) * 4;
      const int e[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
      unsigned takes = 0;  // bit q: score i+q is a candidate
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (i + q < c1 && (((unsigned)e[q] - (unsigned)vmin) >> sh) >= b_lo) takes |= 1u << q;
      if (!__any_sync(0xffffffffu, takes != 0)) continue;
      // warp-aggregated append: exclusive prefix of the lanes' candidate counts
      const int cnt = __popc(takes);
      int incl = cnt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      int slot0 = 0;
      if (lane == 31) slot0 = atomicAdd(&rs[row].n_cand, incl);
      int slot = __shfl_sync(0xffffffffu, slot0, 31) + incl - cnt;
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (takes & (1u << q)) {
          if (slot < kCandCap) cr[slot] = make_int2((int)((unsigned)e[q] - (unsigned)vmin), i + q);
          ++slot;
        }
    }
  }
}

// Ascending bitonic sort of P (a power of two) keys in shared memory by the whole block.
template <typename T>
__device__ void block_bitonic_sort(T* keys, int P) {
  for (int size = 2; size <= P; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = threadIdx.x; i < P / 2; i += kSelThreads) {
        const int lo = 2 * i - (i & (stride - 1));
        const int hi = lo + stride;
        const bool up = (lo & size) == 0;
        const T a = keys[lo], b = keys[hi];
        if ((a > b) == up) {
          keys[lo] = b;
          keys[hi] = a;
        }
      }
      __syncthreads();
    }
  }
}

__global__ void __launch_bounds__(kSelThreads) finalize_kernel(const int32_t* __restrict__ scores,
                                                               const RowSel* __restrict__ rs,
                                                               const int2* __restrict__ cand,
                                                               int32_t* __restrict__ idx, int Lq, int q_offset,
                                                               int Lk, int ratio, int k, long long row_stride) {
  extern __shared__ __align__(16) int sel_row[];
  __shared__ SelShared sh;
  const int row = blockIdx.x, r = row % Lq;
  const int n = n_cand((long long)q_offset + r, ratio, Lk);
  int32_t* out = idx + (size_t)row * k;
  if (n <= k) {
    for (int i = threadIdx.x; i < k; i += kSelThreads) out[i] = i < n ? i : -1;
    return;
  }
  const int nc = rs[row].n_cand;
  if (nc > kCandCap) {  // too many keys tie at the threshold bin: exact select over the whole row
    const int* row_g = scores + (size_t)row * row_stride;
    if (n <= kSelSmemCap)
      select_row<true>(row_g, sel_row, n, k, out, sh);
    else
      select_row<false>(row_g, sel_row, n, k, out, sh);
    return;
  }
  // Keys in bins above b* are all selected; of the keys in bin b*, the (k - above) largest by
  // (u desc, position asc).  Sort those few, then the k positions ascending.
  __shared__ int wsum[kSelWarps];
  __shared__ int bstar, above_b, n_tie, n_sure;
  threshold_bin<kSelThreads>(rs[row].hist, k, wsum, &bstar, &above_b);
  if (threadIdx.x == 0) {
    n_tie = 0;
    n_sure = 0;
  }
  __syncthreads();
  const int sh_bits = hist_shift((unsigned)rs[row].vmax - (unsigned)rs[row].vmin);
  int* pos = sel_row;                                                               // k positions (<= 4096)
  unsigned long long* keys = reinterpret_cast<unsigned long long*>(sel_row + 4096);  // bin b*, <= kCandCap
  const int2* cr = cand + (size_t)row * kCandCap;
  for (int i = threadIdx.x; i < nc; i += kSelThreads) {
    const int2 c = cr[i];
    const int bin = (int)((unsigned)c.x >> sh_bits);
    if (bin > bstar) {
      pos[atomicAdd(&n_sure, 1)] = c.y;
    } else {  // bin == bstar: every candidate is in a bin >= b*
      keys[atomicAdd(&n_tie, 1)] = ((unsigned long long)(0xFFFFFFFFu - (unsigned)c.x) << 32) | (unsigned)c.y;
    }
  }
  __syncthreads();
  const int nt = n_tie, need = k - above_b;  // n_sure == above_b
  int P = 2;
  while (P < nt) P <<= 1;
  for (int i = nt + threadIdx.x; i < P; i += kSelThreads) keys[i] = ~0ull;
  __syncthreads();
  block_bitonic_sort(keys, P);
  for (int i = threadIdx.x; i < need; i += kSelThreads) pos[above_b + i] = (int)(keys[i] & 0xFFFFFFFFull);
  int Pk = 2;
  while (Pk < k) Pk <<= 1;
  for (int i = k + threadIdx.x; i < Pk; i += kSelThreads) pos[i] = INT_MAX;
  __syncthreads();
  block_bitonic_sort(pos, Pk);
  for (int i = threadIdx.x; i < k; i += kSelThreads) out[i] = pos[i];
}

// Calls with at least this many query rows per sequence take the fused path (one CTA per 128
// query rows); fewer rows (decode) use the streaming scorer and the score rows.
constexpr int kFusedMinRows = 64;

// int32 score rows of a call (the workspace part both entry points need)
size_t score_rows_bytes(int B, int Lq, int q_offset, int Lk, int ratio) {
  return (size_t)B * (size_t)Lq * (size_t)score_row_stride(Lq, q_offset, Lk, ratio) * sizeof(int32_t);
}

// Workspace of an indexer + top-k call (both the DSA and the CSA entry points).
size_t index_topk_workspace(int B, int Lq, int q_offset, int Lk, int ratio) {
  if (B <= 0 || Lq <= 0 || Lk <= 0 || q_offset < 0 || ratio <= 0) return 0;
  if (Lq >= kFusedMinRows) return topk_fused_workspace_bytes(B);  // no score rows at all
  size_t bytes = score_rows_bytes(B, Lq, q_offset, Lk, ratio);
  if (use_split_select(B, Lq, q_offset, Lk, ratio)) bytes += (size_t)split_select_bytes(B * Lq);
  return bytes;
}

// Indexer + top-k with candidates s < min((t + 1) / ratio, Lk) for the query at t.
hcadsa_status index_topk(const int8_t* q_idx, const int8_t* k_idx, const int32_t* w_idx, int32_t* idx, void* ws,
                         size_t ws_bytes, int B, int Lq, int q_offset, int Lk, int H_idx, int d_idx, int k,
                         int ratio, hcadsa_stream stream) {
  if (!q_idx || !k_idx || !w_idx || !idx) return HCADSA_ERR_NULL;
  if (B < 0 || Lq < 0 || Lk < 0 || q_offset < 0 || k <= 0 || ratio <= 0) return HCADSA_ERR_SHAPE;
  if (H_idx != kHIdx || d_idx != kDIdx || k > 4096) return HCADSA_ERR_UNSUPPORTED;
  if ((long long)q_offset + Lq > 2147483647LL - 1 || (long long)B * Lq > 2147483647LL) return HCADSA_ERR_UNSUPPORTED;
  if (!aligned16(q_idx) || !aligned16(k_idx) || !aligned16(w_idx) || !aligned16(idx)) return HCADSA_ERR_ALIGN;
  if (B == 0 || Lq == 0) return HCADSA_OK;
  cudaStream_t s = as_stream(stream);
  // some row has more than k candidates
  const bool need_scores = Lk > 0 && n_cand((long long)q_offset + Lq - 1, ratio, Lk) > k;
  if (need_scores) {
    if (!ws) return HCADSA_ERR_WORKSPACE;
    if (!aligned16(ws)) return HCADSA_ERR_ALIGN;
    if (ws_bytes < index_topk_workspace(B, Lq, q_offset, Lk, ratio)) return HCADSA_ERR_WORKSPACE;
  }
  if (need_scores && Lq >= kFusedMinRows)  // many query rows: the fused tensor-core path (dsa_topk_tc.cu)
    return launch_topk_fused(q_idx, k_idx, w_idx, idx, ws, B, Lq, q_offset, Lk, k, ratio, s);
  const long long stride = score_row_stride(Lq, q_offset, Lk, ratio);
  const bool split = need_scores && use_split_select(B, Lq, q_offset, Lk, ratio);
  const int rows = B * Lq;
  RowSel* rowsel =
      split ? reinterpret_cast<RowSel*>(static_cast<char*>(ws) + score_rows_bytes(B, Lq, q_offset, Lk, ratio))
            : nullptr;
  int2* cand = split ? reinterpret_cast<int2*>(rowsel + rows) : nullptr;
  if (need_scores) {
    int32_t* scores = static_cast<int32_t*>(ws);
    if (split) rowsel_init_kernel<<<(unsigned)(B * Lq), 256, 0, s>>>(rowsel);
    dim3 grid((unsigned)((stride + kStreamKeysPerCta - 1) / kStreamKeysPerCta), (unsigned)(B * Lq));
    if (grid.y > 65535u) return HCADSA_ERR_UNSUPPORTED;
    score_stream_kernel<<<grid, kStreamThreads, 0, s>>>(q_idx, k_idx, w_idx, scores, Lq, q_offset, Lk, ratio, stride,
                                                         rowsel);
    if (cudaGetLastError() != cudaSuccess) return HCADSA_ERR_CUDA;
  }
  const int smem = kSelSmemCap * (int)sizeof(int);
  if (split) {
    int32_t* scores = static_cast<int32_t*>(ws);
    const dim3 grid((unsigned)((stride + kSplitChunk - 1) / kSplitChunk), (unsigned)rows);
    hist_kernel<<<grid, 256, 0, s>>>(scores, rowsel, Lq, q_offset, Lk, ratio, k, stride);
    candidates_kernel<<<grid, 256, 0, s>>>(scores, rowsel, cand, Lq, q_offset, Lk, ratio, k, stride);
    if (cudaFuncSetAttribute(finalize_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
      return HCADSA_ERR_CUDA;
    finalize_kernel<<<(unsigned)rows, kSelThreads, smem, s>>>(scores, rowsel, cand, idx, Lq, q_offset, Lk, ratio, k,
                                                              stride);
    return launch_status();
  }
  if (cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return HCADSA_ERR_CUDA;
  select_kernel<<<(unsigned)(B * Lq), kSelThreads, smem, s>>>(need_scores ? static_cast<int32_t*>(ws) : nullptr,
                                                              idx, Lq, q_offset, Lk, ratio, k, stride);
  return launch_status();
}

}  // namespace
}  // namespace hcadsa

extern "C" size_t dsa_index_topk_workspace_size(int B, int Lq, int q_offset, int Lk, int k) {
  (void)k;
  return hcadsa::index_topk_workspace(B, Lq, q_offset, Lk, 1);
}

extern "C" hcadsa_status dsa_index_topk(const int8_t* q_idx, const int8_t* k_idx, const int32_t* w_idx,
                                        int32_t* idx, void* ws, size_t ws_bytes, int B, int Lq, int q_offset,
                                        int Lk, int H_idx, int d_idx, int k, hcadsa_stream stream) {
  return hcadsa::index_topk(q_idx, k_idx, w_idx, idx, ws, ws_bytes, B, Lq, q_offset, Lk, H_idx, d_idx, k, 1, stream);
}

extern "C" size_t csa_index_topk_workspace_size(int B, int Lq, int q_offset, int n_c, int k, int blk) {
  (void)k;
  if (blk <= 0) return 0;
  return hcadsa::index_topk_workspace(B, Lq, q_offset, n_c, blk);
}

extern "C" hcadsa_status csa_index_topk(const int8_t* q_idx, const int8_t* kc_idx, const int32_t* w_idx,
                                        int32_t* idx, void* ws, size_t ws_bytes, int B, int Lq, int q_offset,
                                        int n_c, int H_idx, int d_idx, int k, int blk, hcadsa_stream stream) {
  if (blk <= 0) return HCADSA_ERR_SHAPE;
  return hcadsa::index_topk(q_idx, kc_idx, w_idx, idx, ws, ws_bytes, B, Lq, q_offset, n_c, H_idx, d_idx, k, blk,
                            stream);
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
  const long long stride = score_row_stride(Lq, q_offset, Lk, 1);
  // size check first: a call that does not fit is refused before any CUDA call
  if (need_scores && score_rows_bytes(B, Lq, q_offset, Lk, 1) > kNoAllocScratchBytes) return HCADSA_ERR_WORKSPACE;
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
      dim3 grid((unsigned)((stride + kStreamKeysPerCta - 1) / kStreamKeysPerCta), (unsigned)(B * Lq));
      if (grid.y > 65535u) return HCADSA_ERR_UNSUPPORTED;
      score_stream_kernel<<<grid, kStreamThreads, 0, s>>>(q_idx, k_idx, w_idx, scores, Lq, q_offset, Lk, 1, stride,
                                                           nullptr);
    }
    if (cudaGetLastError() != cudaSuccess) return HCADSA_ERR_CUDA;
  }
  const int smem = kSelSmemCap * (int)sizeof(int);
  if (cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return HCADSA_ERR_CUDA;
  select_kernel<<<(unsigned)(B * Lq), kSelThreads, smem, s>>>(scores, idx, Lq, q_offset, Lk, 1, k, stride);
  return launch_status();
}
