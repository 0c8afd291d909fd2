// dsa_topk_tc.cu -- DSA indexer + exact per-query top-k for many query rows, fused, on sm_100a
// (tcgen05 kind::i8 MMA, TMEM, TMA).
//
// Method: the mirrorspeed page, section "Hybrid sparse attention, 1/7 full context access"
// (and the besthub page, "Core Architectural Innovations", item 1): in the MLA layers a small
// scoring network rates every earlier position for each query, and attention then covers only
// the k best-rated positions.  The indexer form this library fixes:
//     score[t, s] = sum_j w_idx[j] * <q_idx[t, j, :], k_idx[s, :]>      (exact int32)
// over the candidates s < n(t) = min((t + 1) / ratio, Lk) (ratio 1: every position up to and
// including t); the k candidates with the largest (score, -s) are written in ascending order.
//
// Design: one CTA per 128-query tile, no score matrix anywhere.  The CTA streams its keys
// through the tensor cores several times ("passes"); every pass recomputes the same exact
// int32 scores, so nothing but the selection state survives between passes:
//   * Scores on the int8 tensor cores (tcgen05.mma kind::i8, M = 128 queries, K = 64 int8 per
//     head in two K = 32 steps; A = the tile's q_idx (two 128-byte SW128 boxes, two heads
//     each), B = a 192-key k_idx stage (SW64)).  When every w_j * q_j of the tile fits
//     int8 (the usual inputs: |w| <= 4, |q| <= 8), the row threads rewrite the tile in place as
//     w_j * q_j and the four heads accumulate into ONE int32 accumulator, which is the score
//     itself: eight N = 192 MMAs per 192-key stage (TMEM: two buffers of 256 columns).
//     Otherwise each head keeps its own accumulator (four N = 64 accumulators per 64 keys, the
//     same two 256-column buffers) and the thread of query row r (= TMEM lane r) weights them:
//     score = sum_j w_j D_j[r, :].  Both are exact.  (One thread issues every MMA, and its
//     cost is per instruction and per barrier round trip, so wide MMAs matter.)
//   * Selection by narrowing an interval that holds the k-th largest score of the row:
//       level 1: [lo, hi] = exact bounds of the row's scores from its weighted query q' =
//                sum_j w_j q_j and the per-channel min / max of k_idx (a small pre-pass), cut
//                into 256 bins of 2^s values; a histogram of the row's scores is counted in
//                shared memory (layout [bin][row], so a warp's 32 rows hit 32 banks);
//       the bin holding the k-th largest becomes the next interval, the rank inside it is
//       rem = k - (scores in higher bins); further levels histogram only the scores inside it,
//       until the interval is a single value thr, with need_eq = rem of the scores equal to
//       thr to take (the lowest positions first).
//     levels = 1 + ceil(s_1 / 8) for the widest row of the tile (s_1 = bits(hi - lo) - 8):
//     two for the usual indexer inputs (scores within about +-2^14).
//   * Last pass (emit): the positions with score > thr and the first need_eq with score == thr
//     -- exactly the k positions, ascending.  Each of a row's three threads forms the bit masks
//     of its 64-key group of a stage and posts its (above, equal) counts; after the three warps
//     of the lane quarter meet, each knows how many positions the earlier groups take (and how
//     many equal keys are left) and writes its own at that offset.
// Rows with at most k candidates write 0 .. n-1 and -1 padding without scores.  Tiles are
// issued longest first (causal rows near the end of the sequence have the most keys).
//
// Warps: 0 = TMA producer (Q once, then the k_idx stages of 192 keys of every pass through a
// 4-stage ring), 1 = TMEM allocation + the MMA-issuing thread, 2-13 = three threads per query
// row (warp w reaches TMEM lanes 32 (w % 4) ..; each takes one 64-key group of every stage).
// 14 warps keep 128 registers a thread (16 warps, four groups of a 256-key stage, capped them at
// 96 and spilled: 1.19 against 1.14 ms at L = 32768).
#include <climits>

#include "host_common.h"
#include "ptx.cuh"

namespace hcadsa {
namespace {

constexpr int kRows = 128;                    // query rows per CTA (MMA M, TMEM lanes)
constexpr int kStageKeys = 192;               // keys per k_idx stage (one N = 192 MMA per head and K step)
constexpr int kSub = 64;                      // keys per MMA when each head has its own accumulator
constexpr int kDIdx = 64;                     // indexer dim (int8 per head and key)
constexpr int kHIdx = 4;                      // indexer heads
constexpr int kStages = 4;                    // k_idx stage ring
constexpr int kBins = 256;                    // histogram bins per level (8 bits)
constexpr int kQBoxBytes = kRows * 128;       // one SW128 box: 128 rows x (2 heads x 64 int8)
constexpr int kQBytes = 2 * kQBoxBytes;       // 32 KB
constexpr int kKStageBytes = kStageKeys * kDIdx;  // 12 KB
constexpr int kHistBytes = (kBins + 1) * kRows * 4;  // 128.5 KB: 256 bins + a discard bin per row
constexpr int kSmemBytes = kQBytes + kStages * kKStageBytes + kHistBytes + 1024;
constexpr int kRowWarps = 12;                 // three warps per TMEM lane quarter (32 rows)
constexpr int kSubs = kRowWarps / 4;          // threads per query row
constexpr int kRowThreads = kRowWarps * 32;
constexpr int kThreads = 64 + kRowThreads;
constexpr uint32_t kTmemCols = 512;           // two buffers of 256 columns: 256 keys, or 4 heads x 64 keys
constexpr int kBufs = 2;

struct Params {
  const int32_t* w_idx;
  const int32_t* kstat;  // [B][2][64]: per channel min, then max, of k_idx over the batch's keys
  int32_t* idx;
  int* err;
  int B, Lq, q_offset, Lk, k, ratio, n_qt;
};

struct __align__(8) Barriers {
  uint64_t q_full;
  uint64_t plan;               // the row threads have set s_passes and s_single and made the Q tile final
  uint64_t full[kStages];      // k_idx chunk landed
  uint64_t empty[kStages];     // the MMAs that read the chunk completed
  uint64_t tfull[kBufs];       // the scores of a TMEM chunk are in TMEM
  uint64_t tempty[kBufs];      // the row threads have read them
};

__device__ __forceinline__ int n_candidates(long long t, int ratio, int Lk) {
  const long long n = (t + 1) / ratio;
  return (int)(n < Lk ? n : Lk);
}

__device__ __forceinline__ int bit_width(uint32_t x) { return x ? 32 - __clz((int)x) : 0; }

// Shift of a level over an interval of `width` (hi - lo): bins of 2^shift values, at most 256.
__device__ __forceinline__ int level_shift(uint32_t width) {
  const int b = bit_width(width);
  return b > 8 ? b - 8 : 0;
}

// Levels needed to narrow an interval of `width` to a single value (the worst case: the k-th
// largest always in a full bin).
__device__ __forceinline__ int levels_for(uint32_t width) {
  int lv = 0;
  while (width) {
    const int s = level_shift(width);
    ++lv;
    width = s ? (1u << s) - 1u : 0u;
  }
  return lv;
}

__device__ __forceinline__ void rows_bar() { asm volatile("bar.sync 1, %0;" ::"n"(kRowThreads) : "memory"); }
// Named barrier of the row warps that share TMEM lane quarter q (ids 2..5).
__device__ __forceinline__ void quad_bar(int q) { asm volatile("bar.sync %0, %1;" ::"r"(2 + q), "n"(kSubs * 32) : "memory"); }
// Named barrier over the 256 row threads that also ANDs a predicate across them.
__device__ __forceinline__ bool rows_bar_and(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 1, %2, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "n"(kRowThreads)
      : "memory");
  return r != 0;
}

// Output of one row: positions appended in ascending order, four at a time when the row is
// 16-byte aligned (k % 4 == 0).  The last four values sit in b0..b3 (b3 newest), shifted along
// on every append, so no register array is indexed dynamically.
struct RowWriter {
  int32_t* out;
  int pos;  // values written to memory
  int nb;   // values held (0..3)
  int b0, b1, b2, b3;
  bool vec;
  __device__ __forceinline__ void init(int32_t* o, bool v) {
    out = o;
    pos = 0;
    nb = 0;
    b0 = b1 = b2 = b3 = 0;
    vec = v;
  }
  __device__ __forceinline__ void put(int x) {
    if (!vec) {
      out[pos++] = x;
      return;
    }
    b0 = b1;
    b1 = b2;
    b2 = b3;
    b3 = x;
    if (++nb == 4) {
      *reinterpret_cast<int4*>(out + pos) = make_int4(b0, b1, b2, b3);
      pos += 4;
      nb = 0;
    }
  }
  __device__ __forceinline__ void flush() {  // the nb newest values, oldest first
    if (nb >= 3) out[pos++] = b1;
    if (nb >= 2) out[pos++] = b2;
    if (nb >= 1) out[pos++] = b3;
    nb = 0;
  }
};

__global__ void __launch_bounds__(kThreads, 1)
    topk_fused_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                      const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = smem + kQBytes;
  uint32_t* hist = reinterpret_cast<uint32_t*>(sK + kStages * kKStageBytes);  // [kBins][kRows]
  __shared__ Barriers bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;
  __shared__ int s_passes;
  __shared__ int s_single;  // 1: the tile holds w_j * q_j (int8), one score accumulator per chunk
  __shared__ int s_lv[kRowWarps];
  __shared__ int32_t s_kstat[2 * kDIdx];

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  // tile: longest first (blockIdx.x / B counts down the query tiles), batches interleaved
  const int b = blockIdx.x % p.B;
  const int qt = p.n_qt - 1 - (int)(blockIdx.x / p.B);
  const int r0 = qt * kRows;
  const int r_last = min(r0 + kRows, p.Lq) - 1;
  const int n_hi = n_candidates((long long)p.q_offset + r_last, p.ratio, p.Lk);  // keys of the tile
  const bool any_long = n_hi > p.k;  // some row needs scores (positions alone decide)
  const int n_stages = (n_hi + kStageKeys - 1) / kStageKeys;  // k_idx stages per pass

  if (threadIdx.x == 0) {
    mbar_init(&bar.q_full, 1);
    mbar_init(&bar.plan, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bar.full[s], 1);
      mbar_init(&bar.empty[s], 1);
    }
    for (int s = 0; s < kBufs; ++s) {
      mbar_init(&bar.tfull[s], 1);
      mbar_init(&bar.tempty[s], kRowThreads);
    }
    abort_flag = 0;
    s_passes = 0;
    fence_mbarrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_sh, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && any_long) {
      tma_prefetch_desc(&map_q);
      tma_prefetch_desc(&map_k);
      mbar_arrive_expect_tx(&bar.q_full, kQBytes);
      const int qrow = b * p.Lq + r0;
      tma_load_2d(sQ, &map_q, &bar.q_full, 0, qrow);
      tma_load_2d(sQ + kQBoxBytes, &map_q, &bar.q_full, 128, qrow);
      bool ok = true;
      int passes = 1;  // at least the emit pass; the rest is known once the row threads planned
      uint32_t g = 0;
      for (int pass = 0; ok; ++pass) {
        if (pass == 1) {  // planned by now: one pass per narrowing level, then the emit pass
          ok = mbar_wait(&bar.plan, 0, &abort_flag, p.err);
          passes = *reinterpret_cast<volatile int*>(&s_passes);
        }
        if (!ok || pass >= passes) break;
        for (int c = 0; ok && c < n_stages; ++c, ++g) {
          const uint32_t st = g % kStages, ph = (g / kStages) & 1;
          ok = mbar_wait(&bar.empty[st], ph ^ 1, &abort_flag, p.err);
          if (!ok) break;
          mbar_arrive_expect_tx(&bar.full[st], kKStageBytes);
          tma_load_2d(sK + st * kKStageBytes, &map_k, &bar.full[st], 0, b * p.Lk + c * kStageKeys);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && any_long) {
      // the row threads finish the Q tile (possibly rewritten as w_j * q_j) before any MMA
      bool ok = mbar_wait(&bar.plan, 0, &abort_flag, p.err);
      tc_fence_after();
      const bool single = *reinterpret_cast<volatile int*>(&s_single) != 0;
      const int passes = *reinterpret_cast<volatile int*>(&s_passes);
      const uint32_t sQa = smem_u32(sQ), sKa = smem_u32(sK);
      constexpr uint32_t idesc_all = idesc_s8_s32(kRows, kStageKeys);
      constexpr uint32_t idesc_sub = idesc_s8_s32(kRows, kSub);
      uint32_t g = 0, tc = 0;  // k_idx stages, TMEM chunks
      // one TMEM chunk: buffer tc % 2 once the row threads have read its previous contents
      auto take_buffer = [&](uint32_t& buf) {
        buf = tc % kBufs;
        ok = mbar_wait(&bar.tempty[buf], ((tc / kBufs) & 1) ^ 1, &abort_flag, p.err);
        return ok;
      };
      for (int pass = 0; ok && pass < passes; ++pass) {
        for (int c = 0; ok && c < n_stages; ++c, ++g) {
          const uint32_t st = g % kStages, ph = (g / kStages) & 1;
          ok = mbar_wait(&bar.full[st], ph, &abort_flag, p.err);
          if (!ok) break;
          tc_fence_after();
          const uint32_t kst = sKa + st * kKStageBytes;
          if (single) {  // all heads into one accumulator, 256 keys per MMA: sum_j (w_j q_j) . k
            uint32_t buf;
            if (!take_buffer(buf)) break;
            tc_fence_after();
#pragma unroll
            for (int j = 0; j < kHIdx; ++j)
#pragma unroll
              for (int kk = 0; kk < 2; ++kk)  // head j: bytes (j & 1) * 64 + kk * 32 of box j / 2
                mma_i8_ss(tmem + buf * 256, smem_desc_sw128(sQa + (j >> 1) * kQBoxBytes + (j & 1) * 64 + kk * 32, 16, 1024),
                          smem_desc_sw64(kst + kk * 32, 512), idesc_all, (j | kk) != 0);
            mma_commit(&bar.tfull[buf]);
            ++tc;
          } else {  // one accumulator per head, weighted by the row threads: four chunks of 64 keys
            for (int sc = 0; ok && sc < kStageKeys / kSub; ++sc) {
              uint32_t buf;
              if (!take_buffer(buf)) break;
              tc_fence_after();
#pragma unroll
              for (int j = 0; j < kHIdx; ++j)
#pragma unroll
                for (int kk = 0; kk < 2; ++kk)
                  mma_i8_ss(tmem + buf * 256 + j * kSub,
                            smem_desc_sw128(sQa + (j >> 1) * kQBoxBytes + (j & 1) * 64 + kk * 32, 16, 1024),
                            smem_desc_sw64(kst + sc * kSub * kDIdx + kk * 32, 512), idesc_sub, kk);
              mma_commit(&bar.tfull[buf]);
              ++tc;
            }
          }
          mma_commit(&bar.empty[st]);
        }
      }
    }
  } else {
    // ------------------------------------------------------------ four threads per query row
    // Warps 2-5 (sub 0), 6-9, 10-13 and 14-17 (subs 1-3) each cover the tile's 128 rows (warp w
    // reaches TMEM lanes 32 (w % 4) ..); in the histogram passes the four threads of a row take
    // one 64-key group of every 256-key chunk each; in the emit pass sub 0 takes the keys in
    // order, the other subs hand it bit masks of their groups.  All four keep the same row state
    // (computed from the same inputs); only sub 0 writes.
    const int quarter = warp & 3;
    const int sub = (warp - 2) >> 2;
    const int r = quarter * 32 + lane;  // row of the tile == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const int tid = sub * kRows + r;    // 0 .. 511
    const int gr = r0 + r;
    const bool valid = gr < p.Lq;
    const int n = valid ? n_candidates((long long)p.q_offset + gr, p.ratio, p.Lk) : 0;
    const int k = p.k;
    int32_t* out = p.idx + ((size_t)b * p.Lq + (valid ? gr : 0)) * k;
    const bool vec = (k & 3) == 0;
    int w[kHIdx];
#pragma unroll
    for (int j = 0; j < kHIdx; ++j) w[j] = p.w_idx[j];

    // mode: 0 = nothing to do (padding row), 1 = fewer candidates than k (all, -1 padded),
    //       2 = narrowing levels then emit, 3 = all scores equal (emit the first k)
    int mode = !valid ? 0 : (n <= k ? 1 : 2);
    int lo = 0, shift = 0, rem = k, thr = 0, need_eq = 0;
    uint32_t width = 0;
    bool done = mode != 2;
    int lv = 0;
    bool ok = true;
    if (any_long) {
      for (int i = tid; i < 2 * kDIdx; i += kRowThreads) s_kstat[i] = p.kstat[(size_t)b * 2 * kDIdx + i];
      ok = mbar_wait(&bar.q_full, 0, &abort_flag, p.err);
      rows_bar();  // s_kstat complete
      // This row of the tile: 16-byte unit u of box pb, row r, holds bytes 16u .. 16u+15 of that
      // box's 128-byte row (heads 2 pb + (u >> 2), channels 16 (u & 3) ..) at unit u ^ (r & 7).
      // The weighted query q' = sum_j w_j q_j (exact int32) is formed 16 channels at a time (the
      // four heads' units of a channel group) and folded straight into the score bounds, so
      // few registers are live; also: whether every w_j q_j fits int8.
      auto q_unit = [&](int j, int cg) -> uint8_t* {
        return sQ + (j >> 1) * kQBoxBytes + r * 128 + (((((j & 1) << 2) | cg) ^ (r & 7)) << 4);
      };
      bool fits = true;
      long long lo64 = 0, hi64 = 0;
#pragma unroll 1
      for (int cg = 0; cg < 4; ++cg) {
        int qp[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) qp[e] = 0;
#pragma unroll
        for (int j = 0; j < kHIdx; ++j) {
          const uint4 a = *reinterpret_cast<const uint4*>(q_unit(j, cg));
          const uint32_t wd[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int x = w[j] * (int)(int8_t)(wd[e >> 2] >> (8 * (e & 3)));
            qp[e] += x;
            fits = fits && x >= -128 && x <= 127;
          }
        }
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int c = cg * 16 + e;
          const long long a = (long long)qp[e] * s_kstat[c], z = (long long)qp[e] * s_kstat[kDIdx + c];
          lo64 += a < z ? a : z;
          hi64 += a < z ? z : a;
        }
      }
      if (mode == 2) {
        // the true scores fit int32 (caller contract), so clamping keeps them inside [lo, hi]
        lo64 = lo64 < INT_MIN ? INT_MIN : lo64;
        hi64 = hi64 > INT_MAX ? INT_MAX : hi64;
        lo = (int)lo64;
        width = (uint32_t)((long long)hi64 - lo64);
        if (width == 0) {
          mode = 3;
          done = true;
          thr = lo;
          need_eq = k;
        } else {
          shift = level_shift(width);
          lv = levels_for(width);
        }
      }
      // When every row's w_j q_j fits int8, the tile is rewritten in place as w_j q_j, so that
      // summing the four heads' products in one accumulator gives the score directly (exact:
      // the int32 sum is order free).  Otherwise the MMA keeps one accumulator per head.
      const bool single = rows_bar_and(fits);  // every sub has read the tile by now
      if (single && sub == 0) {
#pragma unroll
        for (int j = 0; j < kHIdx; ++j)
#pragma unroll 1
          for (int cg = 0; cg < 4; ++cg) {
            uint4* up = reinterpret_cast<uint4*>(q_unit(j, cg));
            const uint4 a = *up;
            uint32_t wd[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
            for (int e4 = 0; e4 < 4; ++e4) {
              uint32_t o = 0;
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int x = w[j] * (int)(int8_t)(wd[e4] >> (8 * e));
                o |= (uint32_t)(x & 0xFF) << (8 * e);
              }
              wd[e4] = o;
            }
            *up = make_uint4(wd[0], wd[1], wd[2], wd[3]);
          }
        fence_proxy_async_smem();  // generic-proxy writes -> tensor-core operand reads
      }
      // passes of the tile = the widest row's levels + the emit pass
      int lvmax = __reduce_max_sync(0xffffffffu, lv);
      if (lane == 0) s_lv[warp - 2] = lvmax;
      rows_bar();  // also: every row of the tile is final
      if (tid == 0) {
        for (int i = 1; i < kRowWarps; ++i) lvmax = max(lvmax, s_lv[i]);
        s_passes = lvmax + 1;
        s_single = single ? 1 : 0;
        mbar_arrive(&bar.plan);
      }
      if (!done && sub == 0)
        for (int bb = 0; bb <= kBins; ++bb) hist[bb * kRows + r] = 0;
    }

    // rows with at most k candidates: every candidate, then -1
    if (mode == 1 && sub == 0) {
      RowWriter wr;
      wr.init(out, vec);
      for (int s = 0; s < n; ++s) wr.put(s);
      for (int s = n; s < k; ++s) wr.put(-1);
      wr.flush();
    }

    if (any_long) {
      rows_bar();  // s_passes / s_single written
      const int passes = s_passes;
      const bool single = s_single != 0;
      uint32_t g = 0;
      for (int pass = 0; pass < passes; ++pass) {
        const bool emit = pass == passes - 1;
        const bool done_before = done;  // the row counted nothing in this level
        RowWriter wr;
        wr.init(out, vec);
        int eq_seen = 0, taken = 0;
        // emit: bit i of gt / eq = key s0 + i is a candidate above / equal to the threshold
        auto masks = [&](const int (&sc)[32], int s0, uint32_t& gt, uint32_t& eq) {
          const int lim = n - s0;
          gt = eq = 0u;
          if (mode < 2 || lim <= 0) return;
          uint32_t gt4[4] = {0u, 0u, 0u, 0u}, eq4[4] = {0u, 0u, 0u, 0u};  // four independent chains
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            gt4[i & 3] |= (uint32_t)(sc[i] > thr) << i;
            eq4[i & 3] |= (uint32_t)(sc[i] == thr) << i;
          }
          const uint32_t inr = lim >= 32 ? 0xffffffffu : ((1u << lim) - 1u);
          gt = (gt4[0] | gt4[1] | gt4[2] | gt4[3]) & inr;
          eq = (eq4[0] | eq4[1] | eq4[2] | eq4[3]) & inr;
        };
        // emit, in key order: the keys above the threshold and the lowest-positioned equal ones
        // until need_eq of them are in
        auto take = [&](uint32_t gt, uint32_t eq, int s0) {
          const int ne = __popc(eq);
          if (eq_seen + ne > need_eq) {
            uint32_t keep = 0, e = eq;
            for (int q = eq_seen; q < need_eq; ++q) {
              keep |= e & (0u - e);  // lowest remaining set bit
              e &= e - 1;
            }
            eq = keep;
          }
          eq_seen += ne;
          uint32_t sel = gt | eq;
          while (sel && taken < k) {  // ascending positions
            wr.put(s0 + __ffs(sel) - 1);
            sel &= sel - 1;
            ++taken;
          }
        };
        // the pass's work on 32 consecutive scores of this row, keys s0 .. s0 + 31
        auto consume = [&](const int (&sc)[32], int s0) {
          const int lim = n - s0;  // keys s0 + i with i < lim are candidates of the row
          if (!emit) {
            if (!done) {
              if (pass == 0 && lim >= 32) {
                // every score lies in the exact bounds [lo, hi] and every key is a candidate:
                // count it in its bin, nothing to check
                uint32_t* hr = hist + r;
#pragma unroll
                for (int i = 0; i < 32; ++i) atomicAdd(hr + (((uint32_t)sc[i] - (uint32_t)lo) >> shift) * kRows, 1u);
              } else if (pass == 0) {
                // the row's last keys: those past its candidates go to the discard bin kBins
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                  const uint32_t u = (uint32_t)sc[i] - (uint32_t)lo;
                  const uint32_t bin = ((i < lim) & (u <= width)) ? (u >> shift) : (uint32_t)kBins;
                  atomicAdd(&hist[bin * kRows + r], 1u);
                }
              } else {  // later levels count only the few scores inside the narrowed interval
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                  const uint32_t u = (uint32_t)sc[i] - (uint32_t)lo;
                  if ((i < lim) & (u <= width)) atomicAdd(&hist[(u >> shift) * kRows + r], 1u);
                }
              }
            }
          } else {
            uint32_t gt, eq;
            masks(sc, s0, gt, eq);
            take(gt, eq, s0);
          }
        };
        // TMEM chunks of this pass: one per 256-key stage (single accumulator), or four of 64 keys
        const int chunks = single ? n_stages : n_stages * (kStageKeys / kSub);
        // the emit pass of per-head accumulators is sub 0's alone (key order); with one
        // accumulator subs 1-3 form the bit masks of the chunk's later 64-key groups for sub 0.
        // Per-head accumulators (64 keys a chunk) split over subs 0 and 1 in the counting passes.
        const bool active = single || (emit ? sub == 0 : sub < 2);
        for (int c = 0; c < chunks; ++c, ++g) {
          const uint32_t buf = g % kBufs;
          ok = mbar_wait(&bar.tfull[buf], (g / kBufs) & 1, &abort_flag, p.err) && ok;
          tc_fence_after();
          if (!active) {  // nothing to read: release the buffer for this thread
            tc_fence_before();
            mbar_arrive(&bar.tempty[buf]);
            continue;
          }
          if (single && emit) {
            // 256 scores of keys c*256 .. c*256+255: every sub forms the bit masks of its 64-key
            // group and posts its (above, equal) counts (shared memory, two buffers by chunk
            // parity); after the four warps of a lane quarter meet, each sub knows how many
            // keys the earlier groups take and writes its own positions at that offset
            uint32_t* cn = hist + (c & 1) * 4 * kRows + r;  // [buffer][sub][row]: gt | eq << 16
            const uint32_t ta = tmem + lane_off + buf * 256 + sub * 64;
            const int s0 = c * kStageKeys + sub * 64;
            uint32_t gt0, eq0, gt1, eq1;
            {
              uint32_t v[32];
              tmem_ld32_nowait(ta, v);
              tmem_wait_ld_regs(v);
              masks(reinterpret_cast<const int(&)[32]>(v), s0, gt0, eq0);
            }
            {
              uint32_t v[32];
              tmem_ld32_nowait(ta + 32, v);
              tmem_wait_ld_regs(v);
              tc_fence_before();
              mbar_arrive(&bar.tempty[buf]);
              masks(reinterpret_cast<const int(&)[32]>(v), s0 + 32, gt1, eq1);
            }
            cn[sub * kRows] = (uint32_t)(__popc(gt0) + __popc(gt1)) | ((uint32_t)(__popc(eq0) + __popc(eq1)) << 16);
            quad_bar(quarter);
            int gt_before = 0, eq_before = 0, gt_tot = 0, eq_tot = 0;
#pragma unroll
            for (int s2 = 0; s2 < kSubs; ++s2) {
              const uint32_t w2 = cn[s2 * kRows];
              const int g2 = (int)(w2 & 0xFFFFu), e2 = (int)(w2 >> 16);
              if (s2 < sub) {
                gt_before += g2;
                eq_before += e2;
              }
              gt_tot += g2;
              eq_tot += e2;
            }
            // equal keys are taken in position order until need_eq of them are in
            const int eq_room = max(0, need_eq - eq_seen);
            const int eq_taken_before = min(eq_before, eq_room);
            int eq_take = min(__popc(eq0) + __popc(eq1), eq_room - eq_taken_before);
            int pos = taken + gt_before + eq_taken_before;
            if (mode >= 2) {
              // this group's selected keys, ascending: all above, the first eq_take equal ones
              uint32_t sel0 = gt0, e = eq0;
              while (e && eq_take > 0) {
                sel0 |= e & (0u - e);
                e &= e - 1;
                --eq_take;
              }
              uint32_t sel1 = gt1;
              e = eq1;
              while (e && eq_take > 0) {
                sel1 |= e & (0u - e);
                e &= e - 1;
                --eq_take;
              }
              while (sel0) {
                out[pos++] = s0 + __ffs(sel0) - 1;
                sel0 &= sel0 - 1;
              }
              while (sel1) {
                out[pos++] = s0 + 32 + __ffs(sel1) - 1;
                sel1 &= sel1 - 1;
              }
            }
            taken += gt_tot + min(eq_tot, eq_room);
            eq_seen += eq_tot;
          } else if (single) {
            // 256 scores of keys c*256 .. c*256+255: this sub's 64-key group
            {
              const uint32_t ta = tmem + lane_off + buf * 256 + sub * 64;
              {
                uint32_t v[32];
                tmem_ld32_nowait(ta, v);
                tmem_wait_ld_regs(v);
                consume(reinterpret_cast<const int(&)[32]>(v), c * kStageKeys + sub * 64);
              }
              {
                uint32_t v[32];
                tmem_ld32_nowait(ta + 32, v);
                tmem_wait_ld_regs(v);
                tc_fence_before();
                mbar_arrive(&bar.tempty[buf]);
                consume(reinterpret_cast<const int(&)[32]>(v), c * kStageKeys + sub * 64 + 32);
              }
            }
          } else {
            const int h0 = emit ? 0 : sub, h1 = emit ? 2 : sub + 1;
#pragma unroll 1
            for (int h = h0; h < h1; ++h) {
              const uint32_t ta = tmem + lane_off + buf * 256 + h * 32;
              int sc[32];
#pragma unroll
              for (int i = 0; i < 32; ++i) sc[i] = 0;
#pragma unroll
              for (int hd = 0; hd < kHIdx; ++hd) {  // one head's accumulator at a time
                uint32_t v[32];
                tmem_ld32_nowait(ta + hd * kSub, v);
                tmem_wait_ld_regs(v);
#pragma unroll
                for (int i = 0; i < 32; ++i) sc[i] += w[hd] * (int)v[i];
              }
              if (h == h1 - 1) {
                tc_fence_before();
                mbar_arrive(&bar.tempty[buf]);
              }
              consume(sc, c * kSub + h * 32);
            }
          }
        }
        if (!emit) rows_bar();  // every sub's counts of this level are in
        if (!emit && !done) {
          // the bin holding the rank-rem score of the interval, counted from the top (both
          // threads of the row read the same counts and reach the same state)
          uint32_t above = 0;
          int bstar = -1;
          for (int bb = kBins - 1; bb >= 0; --bb) {
            const uint32_t cnt = hist[bb * kRows + r];
            if (bstar < 0) {
              if (above + cnt >= (uint32_t)rem)
                bstar = bb;
              else
                above += cnt;
            }
          }
          if (bstar < 0) {  // cannot happen for consistent scores; keep the row well defined
            raise_device_error(p.err, kErrDeviceBounds);
            bstar = 0;
          }
          const uint32_t off = (uint32_t)bstar << shift;
          lo = (int)((uint32_t)lo + off);
          rem -= (int)above;
          const uint32_t cap = shift ? (1u << shift) - 1u : 0u;
          width = min(width - off, cap);
          if (width == 0) {
            done = true;
            thr = lo;
            need_eq = rem;
          } else {
            shift = level_shift(width);
          }
        }
        if (!emit) {
          rows_bar();  // every sub has read the counts
          if (sub == 0 && !done_before)
            for (int bb = 0; bb <= kBins; ++bb) hist[bb * kRows + r] = 0;
          rows_bar();  // cleared before the next level counts
        }
        if (emit && mode >= 2 && sub == 0 && !single) wr.flush();
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

// Per-channel min and max of k_idx over every key of each batch: kstat[b] = {min[64], max[64]}.
// kstat must hold INT_MAX-like / INT_MIN-like start values (memset 0x7f / 0x80 bytes).
constexpr int kStatKeysPerCta = 4096;
__global__ void __launch_bounds__(256) kstat_kernel(const int8_t* __restrict__ k_idx, int Lk,
                                                    int32_t* __restrict__ kstat) {
  const int b = blockIdx.y;
  const int part = threadIdx.x & 3;  // 16-byte slice of the 64-byte key: channels 16*part ..
  const int s_begin = blockIdx.x * kStatKeysPerCta;
  const int s_end = min(s_begin + kStatKeysPerCta, Lk);
  int mn[16], mx[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    mn[e] = 127;
    mx[e] = -128;
  }
  const uint4* kb = reinterpret_cast<const uint4*>(k_idx + (size_t)b * Lk * kDIdx);
  for (int s = s_begin + (threadIdx.x >> 2); s < s_end; s += 64) {
    const uint4 v = __ldg(kb + (size_t)s * 4 + part);
    const uint32_t wd[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const int x = (int)(int8_t)(wd[e >> 2] >> (8 * (e & 3)));
      mn[e] = min(mn[e], x);
      mx[e] = max(mx[e], x);
    }
  }
  // lanes l and l ^ 4, l ^ 8, ... hold the same channels
#pragma unroll
  for (int o = 4; o < 32; o <<= 1)
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      mn[e] = min(mn[e], __shfl_xor_sync(0xffffffffu, mn[e], o));
      mx[e] = max(mx[e], __shfl_xor_sync(0xffffffffu, mx[e], o));
    }
  if ((threadIdx.x & 31) < 4) {
    int32_t* ks = kstat + (size_t)b * 2 * kDIdx;
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      atomicMin(&ks[part * 16 + e], mn[e]);
      atomicMax(&ks[kDIdx + part * 16 + e], mx[e]);
    }
  }
}

}  // namespace

size_t topk_fused_workspace_bytes(int B) { return (size_t)B * 2 * kDIdx * sizeof(int32_t); }

hcadsa_status launch_topk_fused(const int8_t* q_idx, const int8_t* k_idx, const int32_t* w_idx, int32_t* idx,
                                void* kstat, int B, int Lq, int q_offset, int Lk, int k, int ratio,
                                cudaStream_t s) {
  if (B <= 0 || Lq <= 0 || Lk <= 0 || ratio <= 0 || k <= 0) return HCADSA_ERR_SHAPE;
  const long long n_qt = (Lq + kRows - 1) / kRows;
  if (n_qt * B > 2147483647LL || (long long)B * Lq > 2147483647LL || (long long)B * Lk > 2147483647LL)
    return HCADSA_ERR_UNSUPPORTED;
  CUtensorMap mq, mk;
  {
    const uint64_t dims[2] = {(uint64_t)(kHIdx * kDIdx), (uint64_t)B * Lq};
    const uint64_t strides[1] = {(uint64_t)(kHIdx * kDIdx)};
    const uint32_t box[2] = {128, (uint32_t)kRows};
    if (!encode_tmap_u8_swizzle(&mq, 2, const_cast<int8_t*>(q_idx), dims, strides, box, 128)) return HCADSA_ERR_CUDA;
  }
  {
    const uint64_t dims[2] = {(uint64_t)kDIdx, (uint64_t)B * Lk};
    const uint64_t strides[1] = {(uint64_t)kDIdx};
    const uint32_t box[2] = {(uint32_t)kDIdx, (uint32_t)kStageKeys};
    if (!encode_tmap_u8_swizzle(&mk, 2, const_cast<int8_t*>(k_idx), dims, strides, box, 64)) return HCADSA_ERR_CUDA;
  }
  int32_t* ks = static_cast<int32_t*>(kstat);
  for (int bb = 0; bb < B; ++bb) {
    // start values: 0x7f7f7f7f for the minima, 0x80808080 (negative) for the maxima
    if (cudaMemsetAsync(ks + (size_t)bb * 2 * kDIdx, 0x7f, kDIdx * sizeof(int32_t), s) != cudaSuccess ||
        cudaMemsetAsync(ks + (size_t)bb * 2 * kDIdx + kDIdx, 0x80, kDIdx * sizeof(int32_t), s) != cudaSuccess)
      return launch_status();
  }
  const dim3 sgrid((unsigned)((Lk + kStatKeysPerCta - 1) / kStatKeysPerCta), (unsigned)B);
  if (sgrid.y > 65535u) return HCADSA_ERR_UNSUPPORTED;
  kstat_kernel<<<sgrid, 256, 0, s>>>(k_idx, Lk, ks);
  Params p;
  p.w_idx = w_idx;
  p.kstat = ks;
  p.idx = idx;
  p.err = device_error_ptr();
  p.B = B;
  p.Lq = Lq;
  p.q_offset = q_offset;
  p.Lk = Lk;
  p.k = k;
  p.ratio = ratio;
  p.n_qt = (int)n_qt;
  if (cudaFuncSetAttribute(topk_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) !=
      cudaSuccess)
    return launch_status();
  topk_fused_kernel<<<(unsigned)(n_qt * B), kThreads, kSmemBytes, s>>>(mq, mk, p);
  return launch_status();
}

}  // namespace hcadsa
