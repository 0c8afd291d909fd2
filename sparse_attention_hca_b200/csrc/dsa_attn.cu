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
//   * The 64 heads of a token are the M of every MMA (M = 64: half of the datapath, so an
//     instruction takes as long as its M = 128 twin, measured on B200):
//       S  = Q (A, smem, K-major, 64 x 256) * K_g^T (B, smem, K-major, 128 gathered keys)
//       O += P (A, TMEM, bf16)               * V_g (B, smem, MN-major, 256 d_v)
//     P never touches shared memory: the softmax writes it as bf16 pairs over the first 64
//     columns of its S tile, where the PV MMA reads it as the TMEM A operand.  Against the
//     keys-as-M form (S^T = K_g Q^T, P^T staged in shared memory) this saves 48 KB of
//     shared-memory traffic per 128-key tile and every per-head cross-thread reduction:
//     a head is a TMEM lane, so its max and sum are two threads' business.
//   * An M = 64 accumulator fills 16 of the 32 lanes of each lane quarter; the other 16 lanes
//     hold a second one (lane offset 16).  Token i uses half i & 1 for everything: O at
//     columns [0, 256) and two S tiles at [256, 384) / [384, 512).  A TS MMA needs A and D in
//     the same half, which this keeps, and one token's epilogue overlaps the next token's MMAs
//     in the other half.
//   * Warps 0-5 gather K and V rows with cp.async: one warp instruction moves one whole
//     512-byte row (lane l -> 16 bytes of 64-column chunk l/8), written 128B-swizzled into a
//     ring of two 64 KB groups (4 chunk slots each); a group holds one K or one V tile, loaded
//     in exactly the order warp 6 consumes them: K_0, K_1, V_0, K_2, V_1, ...  Completion is
//     tracked with cp.async.mbarrier.arrive.noinc, one arrival per producer thread per tile, so
//     the MMA thread waits once per tile and issues a proxy fence after it so the tensor core
//     sees the generic-proxy writes.  (Measured on B200: this reaches ~105 GB/s per SM from L2,
//     TMA tile::gather4 of 4 x 128 B rows ~16 GB/s.)
//     Q (32 KB, TMA, double-buffered) is loaded as soon as the producers start a token.
//   * Warp 6, lane 0 issues every MMA.  Warps 7-10: softmax.  Warp 7+q owns heads 16q..16q+15
//     (TMEM lane quarter q); thread t of it holds head 16q + t%16 and keys 64(t/16)..+63 of a
//     tile.  Online softmax per head with a lazy reference max: the first tile sets it, a later
//     tile moves it (and rescales that head's O in TMEM) only when a score exceeds it by 2^8.
//     Then the token's epilogue: O / l to bf16, and the log-sum-exp.
//   * Index rows may hold padding (< 0) anywhere; a 128-entry tile without any valid entry
//     is skipped, other invalid entries read row 0 and are masked.  Index rows are staged in
//     shared memory (double buffer): the softmax warps prefetch token i+2's row with cp.async
//     as soon as the producer and MMA warps have released the buffer token i used, so no
//     role waits on the index tensor in HBM.
//   * Barrier phases continue across tokens: s_full/p_ready/pv_done are indexed by a global
//     tile counter, q_full/q_empty/o_full/o_empty by a counter of tokens with work.
//   * Few tokens (at most half as many as SMs: decode batches) split: the CTAs walk units
//     (token, part), part p of S taking ranks [p J / S, (p+1) J / S) of the token's J tiles,
//     write unnormalised fp32 O rows and per-head (max, sum) to a workspace, and
//     dsa_combine_kernel merges a token's parts (the online-softmax merge) into O and lse.
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
constexpr int kMaxK = 4096;                // 32 tiles: one bit per tile in a 32-bit mask
constexpr int kIdxBytes = kMaxK * 4;  // one index row
constexpr int kSmemBytes = 2 * kQBytes + kRingSlots * kChunkBytes + 2 * kIdxBytes + 1024;  // 225 KB
// Gather throughput scales with the number of producer warps; 11 warps cap a thread at 168
// registers, which the softmax (64 scores per thread) stays well inside.
constexpr int kProducerWarps = 6;
constexpr int kMmaWarp = kProducerWarps;
constexpr int kSoftmaxWarp0 = kProducerWarps + 1;
constexpr int kThreads = 32 * (kProducerWarps + 1 + 4);
constexpr uint32_t kTmemS = 256;  // S tiles at columns 256 and 384 of a token's half; O at 0
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
  // Split mode (few tokens, split > 1): unit u = token u / split, part u % split of its key
  // tiles; the unit's unnormalised O (fp32) and per-head (max, sum) go to ws_O / ws_ml and a
  // combine pass writes O and lse.  split == 1: units are tokens and O is written directly.
  int split, n_units;
  float* ws_O;   // [n_units][64][256]
  float* ws_ml;  // [n_units][2][64]: reference max (log2 units), then sum of p
};

struct __align__(8) Barriers {
  uint64_t q_full[2], q_empty[2];  // Q double buffer, by the count of tokens with work
  uint64_t full[2];   // ring group g holds a whole K or V tile (192 producer-thread arrivals)
  uint64_t empty[2];  // the MMAs that read group g have completed
  uint64_t s_full[2];
  uint64_t p_ready[2];
  uint64_t pv_done;
  uint64_t o_full[2];
  uint64_t o_empty[2];
  uint64_t idx_full[2];   // index row of a token landed (128 softmax-thread cp.async arrivals)
  uint64_t idx_empty[2];  // the producer warps and the MMA warp are done with the row
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

// Bit j set iff tile j (entries [128j, 128j+128) of the row) holds a valid entry; with
// kAll, `all_valid` gets bit j iff all 128 entries of tile j are valid.  Whole warp; `row` is
// the 16-byte aligned shared-memory copy of the index row.  Each lane reads its four entries of
// a whole tile as one 16-byte word (a warp reads 512 contiguous bytes: no bank conflicts), eight
// tiles' words in flight at a time, and sets one bit per tile; one reduction over the warp then
// gives the mask.  This runs between the tokens of the MMA warp, while the tensor pipe only
// has its queue left, so it has to be short.
template <bool kAll>
__device__ __forceinline__ uint32_t tile_mask_of_row(const int32_t* row, int k, int Lk, int lane,
                                                     uint32_t* all_valid = nullptr) {
  const int full = k / kKeyTile;
  uint32_t bits = 0, all_bits = 0;
  for (int j0 = 0; j0 < full; j0 += 8) {
    int4 v[8];
#pragma unroll
    for (int q = 0; q < 8; ++q)
      v[q] = j0 + q < full ? *reinterpret_cast<const int4*>(row + (j0 + q) * kKeyTile + 4 * lane)
                           : make_int4(-1, -1, -1, -1);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const bool a = idx_ok(v[q].x, Lk), b = idx_ok(v[q].y, Lk), c = idx_ok(v[q].z, Lk), d = idx_ok(v[q].w, Lk);
      if (a | b | c | d) bits |= 1u << (j0 + q);
      if (kAll && (a & b & c & d)) all_bits |= 1u << (j0 + q);
    }
  }
  if (full * kKeyTile < k) {  // the ragged last tile (never all-valid: it has fewer than 128 entries)
    bool any = false;
    for (int e = full * kKeyTile + lane; e < k; e += 32) any |= idx_ok(row[e], Lk);
    if (any) bits |= 1u << full;
  }
  if (kAll) *all_valid = __reduce_and_sync(0xffffffffu, all_bits);
  return __reduce_or_sync(0xffffffffu, bits);
}

// The tiles of `mask` that part `part` of `split` takes: ranks [part J / split, (part+1) J / split)
// of its J set bits, in ascending order.  Every role derives the same subset.
__device__ __forceinline__ uint32_t part_of_mask(uint32_t mask, int part, int split) {
  if (split == 1) return mask;
  const int J = __popc(mask);
  const int lo = part * J / split, hi = (part + 1) * J / split;
  uint32_t out = 0;
  int r = 0;
  for (uint32_t m = mask; m; m &= m - 1, ++r)
    if (r >= lo && r < hi) out |= m & (0u - m);
  return out;
}

__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}

// Half-quarter TMEM access (.16x32bx2): threads 0-15 of the warp address lanes base + t at
// columns [c, c + 32), threads 16-31 the same 16 lanes at columns [c + kOff, c + kOff + 32).
template <int kOff>
__device__ __forceinline__ void tmem_ld_half32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.16x32bx2.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32], %33;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]),
        "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]),
        "=r"(r[30]), "=r"(r[31])
      : "r"(taddr), "n"(kOff)
      : "memory");
}
template <int kOff>
__device__ __forceinline__ void tmem_st_half32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.16x32bx2.x32.b32 [%0], %1, "
      "{%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,"
      "%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,%33};" ::"r"(taddr),
      "n"(kOff), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]),
      "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]),
      "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

template <int kOff>
__device__ __forceinline__ void tmem_st_half16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.16x32bx2.x16.b32 [%0], %1, "
      "{%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17};" ::"r"(taddr),
      "n"(kOff), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

__device__ __forceinline__ void softmax_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// Softmax threads: once the producers and the MMA warp released buffer `buf` (used by local
// unit i), fetch the index row of unit `next`'s token into it with cp.async.
__device__ __forceinline__ void refill_idx_row(const Params& p, Barriers& bar, uint32_t sIdx_a, int buf, int i,
                                               int next, int tid, volatile int& abort_flag, bool& ok) {
  if (next >= p.n_units) return;
  ok = mbar_wait(&bar.idx_empty[buf], (i >> 1) & 1, &abort_flag, p.err) && ok;
  const int32_t* src = p.idx + (size_t)(next / p.split) * p.k;
  for (int e = tid; e < p.k; e += 128) cp_async4(sIdx_a + (buf * kMaxK + e) * 4, src + e);
  cp_async_arrive_noinc(&bar.idx_full[buf]);
}

__global__ void __launch_bounds__(kThreads, 1)
    dsa_attn_kernel(const __grid_constant__ CUtensorMap map_q, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;  // [2][kQBytes]
  uint8_t* sRing = smem + 2 * kQBytes;
  int32_t* sIdx = reinterpret_cast<int32_t*>(sRing + kRingSlots * kChunkBytes);  // [2][kMaxK]
  __shared__ Barriers bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar.q_full[s], 1);
      mbar_init(&bar.q_empty[s], 1);
    }
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
    int i = 0;  // units of this CTA so far (index-row buffer i & 1)
    for (int unit = blockIdx.x; unit < p.n_units && ok; unit += gridDim.x, ++i) {
      const int tok = unit / p.split;
      const int buf = i & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(&bar.idx_full[buf], (i >> 1) & 1, &abort_flag, p.err));
      if (!ok) break;
      const int32_t* row = sIdx + buf * kMaxK;
      const uint32_t mask = part_of_mask(tile_mask_of_row<false>(row, k, Lk, lane), unit % p.split, p.split);
      if (!mask) {
        if (lane == 0) mbar_arrive(&bar.idx_empty[buf]);
        continue;
      }
      const int J = __popc(mask);
      if (warp == 0) {
        // Q of this token into its buffer, ahead of the token's first K tile: the buffer was last
        // read by the S MMAs of token it-2
        const int qb = it & 1;
        ok = __all_sync(0xffffffffu, mbar_wait(&bar.q_empty[qb], ((it >> 1) & 1) ^ 1, &abort_flag, p.err));
        if (ok && lane == 0) {
          mbar_arrive_expect_tx(&bar.q_full[qb], kQBytes);
          for (int c = 0; c < 4; ++c)
            tma_load_3d(sQ + qb * kQBytes + c * kQChunkBytes, &map_q, &bar.q_full[qb], c * 64, 0, tok);
        }
      }
      const size_t kv_row0 = (size_t)(tok / p.Lq) * Lk;  // first K/V row of this token's batch
      // warp w gathers tile rows w, w+6, w+12, ...: lane l holds the K/V row of the warp's
      // l-th row (ra) and (32+l)-th row (rb)
      const int n_rows_w = (kKeyTile - warp + kProducerWarps - 1) / kProducerWarps;  // 22 or 21
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
    const uint32_t sQa = smem_u32(sQ), sRa = smem_u32(sRing);
    const uint32_t idesc_s = idesc_bf16_f32(kH, kKeyTile, false, false);  // S: M = 64 heads, N = 128 keys
    const uint32_t idesc_o = idesc_bf16_f32(kH, kD, false, true);         // O: N = 256 d_v, V MN-major
    int i = 0;
    for (int unit = blockIdx.x; unit < p.n_units && ok; unit += gridDim.x, ++i) {
      const int buf = i & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(&bar.idx_full[buf], (i >> 1) & 1, &abort_flag, p.err));
      if (!ok) break;
      const uint32_t mask =
          part_of_mask(tile_mask_of_row<false>(sIdx + buf * kMaxK, k, Lk, lane), unit % p.split, p.split);
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar.idx_empty[buf]);  // only the mask was needed
      if (!mask) continue;
      const int J = __popc(mask);
      const int hf = it & 1;  // this token's TMEM half (lane offset 16 * hf)
      if (lane == 0) {
        const uint32_t t_half = tmem + (static_cast<uint32_t>(16 * hf) << 16);
        const int qb = it & 1;
        ok = mbar_wait(&bar.q_full[qb], (it >> 1) & 1, &abort_flag, p.err);
        tc_fence_after();
        for (int step = 0; step <= J && ok; ++step) {
          if (step < J) {
            const uint32_t gs = g + step;
            const uint32_t tS = t_half + kTmemS + (gs & 1) * kKeyTile;
            // one wait per K tile: every producer thread arrives once all of its row copies of
            // the tile (all 4 chunks) have landed
            ok = mbar_wait(&bar.full[u & 1], (u >> 1) & 1, &abort_flag, p.err);
            if (!ok) break;
            fence_proxy_async_smem();  // cp.async (generic proxy) writes -> tensor core reads
            tc_fence_after();
            {
              const uint64_t da0 = smem_desc_sw128(sQa + qb * kQBytes, 16, 1024);
              const uint64_t db0 = smem_desc_sw128(sRa + (u & 1) * 4 * kChunkBytes, 16, 1024);
#pragma unroll
              for (int c = 0; c < 4; ++c)
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)  // descriptor start address field is in 16-byte units
                  mma_ss(tS, da0 + (uint64_t)((c * kQChunkBytes + kk * 32) >> 4),
                         db0 + (uint64_t)((c * kChunkBytes + kk * 32) >> 4), idesc_s, (c | kk) != 0);
            }
            mma_commit(&bar.empty[u & 1]);
            ++u;
            mma_commit(&bar.s_full[gs & 1]);
            if (step == J - 1) mma_commit(&bar.q_empty[qb]);
          }
          if (step >= 1) {
            const int j = step - 1;
            const uint32_t gj = g + j;
            if (j == 0) {  // O in this half must have been drained by the epilogue of token it-2
              ok = mbar_wait(&bar.o_empty[hf], ((it >> 1) & 1) ^ 1, &abort_flag, p.err);
              if (!ok) break;
            }
            ok = mbar_wait(&bar.p_ready[gj & 1], (gj >> 1) & 1, &abort_flag, p.err);
            if (!ok) break;
            tc_fence_after();
            const uint32_t tP = t_half + kTmemS + (gj & 1) * kKeyTile;  // P: bf16 pairs, 64 columns
            ok = mbar_wait(&bar.full[u & 1], (u >> 1) & 1, &abort_flag, p.err);  // the whole V tile
            if (!ok) break;
            fence_proxy_async_smem();
            tc_fence_after();
            {
              // V as MN-major B: 64-d_v chunks one slot (LBO) apart, 8-key groups 1024 B apart;
              // 16 keys (one MMA) are 2048 B of the slot, 16 keys of P are 8 TMEM columns
              const uint64_t db0 = smem_desc_sw128(sRa + (u & 1) * 4 * kChunkBytes, kChunkBytes, 1024);
#pragma unroll
              for (int kk = 0; kk < kKeyTile / 16; ++kk)
                mma_ts(t_half, tP + kk * 8, db0 + (uint64_t)((kk * 2048) >> 4), idesc_o, (j > 0 || kk > 0) ? 1u : 0u);
            }
            mma_commit(&bar.empty[u & 1]);
            ++u;
            mma_commit(&bar.pv_done);
            if (j == J - 1) mma_commit(&bar.o_full[hf]);
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
    const int quarter = warp & 3;  // TMEM lane quarter this warp may access: heads 16q..16q+15
    const int kh = lane >> 4;      // keys 64kh..64kh+63 of a tile, d_v 128kh..128kh+127 of O
    const int h = quarter * 16 + (lane & 15);
    const int tid = (warp - kSoftmaxWarp0) * 32 + lane;  // 0..127
    int it = 0;
    uint32_t g = 0;
    bool ok = true;
    // No early exit in this loop: the four softmax warps meet at a named barrier, so after an
    // abort every thread keeps walking the same barrier sequence (waits then fail fast).
    const uint32_t sIdx_a = smem_u32(sIdx);
    // index rows of this CTA's first two units
    for (int i0 = 0; i0 < 2; ++i0) {
      const int u0 = blockIdx.x + i0 * gridDim.x;
      if (u0 < p.n_units) {
        const int32_t* src = p.idx + (size_t)(u0 / p.split) * k;
        for (int e = tid; e < k; e += 128) cp_async4(sIdx_a + (i0 * kMaxK + e) * 4, src + e);
        cp_async_arrive_noinc(&bar.idx_full[i0]);
      }
    }
    int i = 0;
    for (int unit = blockIdx.x; unit < p.n_units; unit += gridDim.x, ++i) {
      const int tok = unit / p.split;
      const int buf = i & 1;
      ok = mbar_wait(&bar.idx_full[buf], (i >> 1) & 1, &abort_flag, p.err) && ok;
      const int32_t* row = sIdx + buf * kMaxK;
      uint32_t all_valid = 0;
      const uint32_t mask = part_of_mask(tile_mask_of_row<true>(row, k, Lk, lane, &all_valid), unit % p.split, p.split);
      uint16_t* obase = p.O + (size_t)tok * kH * kD;
      if (!mask) {
        if (p.split > 1) {  // no tile in this part: an empty record for the combine pass
          if (tid < kH) {
            p.ws_ml[(size_t)unit * 2 * kH + tid] = -INFINITY;
            p.ws_ml[(size_t)unit * 2 * kH + kH + tid] = 0.0f;
          }
        } else {  // no valid entry: O = 0, lse = -inf
          for (int e = tid; e < kH * kD / 8; e += 128) reinterpret_cast<uint4*>(obase)[e] = make_uint4(0, 0, 0, 0);
          if (p.lse && tid < kH) p.lse[(size_t)tok * kH + tid] = -INFINITY;
        }
        softmax_bar();  // every softmax thread has read the row before it is refilled
        refill_idx_row(p, bar, sIdx_a, buf, i, unit + 2 * gridDim.x, tid, abort_flag, ok);
        continue;
      }
      const int J = __popc(mask);
      const int hf = it & 1;
      const uint32_t t_lanes = tmem + (static_cast<uint32_t>(quarter * 32 + hf * 16) << 16);
      float m_run = -INFINITY;  // reference max of head h (log2 units), same in both threads of the head
      float l_run = 0.0f;       // sum of p over this thread's keys
      uint32_t m = mask;
      for (int jj = 0; jj < J; ++jj) {
        const int j = __ffs(m) - 1;
        m &= m - 1;
        const uint32_t gs = g + jj;
        // validity of this thread's 64 keys (bit i: entry j*128 + 64kh + i); whole valid tiles skip it
        uint32_t v_lo = 0xffffffffu, v_hi = 0xffffffffu;
        if (!((all_valid >> j) & 1u)) {
          v_lo = v_hi = 0;
          bool oob = false;
          const int e0 = j * kKeyTile + kh * 64;
#pragma unroll 4
          for (int q4 = 0; q4 < 16; ++q4) {
            const int4 w = *reinterpret_cast<const int4*>(row + e0 + 4 * q4);  // inside the row buffer
            const int e = e0 + 4 * q4;
            const int s0 = e < k ? w.x : -1, s1 = e + 1 < k ? w.y : -1;
            const int s2 = e + 2 < k ? w.z : -1, s3 = e + 3 < k ? w.w : -1;
            oob |= (s0 >= Lk) | (s1 >= Lk) | (s2 >= Lk) | (s3 >= Lk);
            const uint32_t nib = (idx_ok(s0, Lk) ? 1u : 0u) | (idx_ok(s1, Lk) ? 2u : 0u) | (idx_ok(s2, Lk) ? 4u : 0u) |
                                 (idx_ok(s3, Lk) ? 8u : 0u);
            if (q4 < 8) v_lo |= nib << (4 * q4);
            else v_hi |= nib << (4 * q4 - 32);
          }
          if (oob) raise_device_error(p.err, kErrDeviceBounds);
        }
        ok = mbar_wait(&bar.s_full[gs & 1], (gs >> 1) & 1, &abort_flag, p.err) && ok;
        tc_fence_after();
        const uint32_t tS = t_lanes + kTmemS + (gs & 1) * kKeyTile;
        uint32_t sa[32], sb[32];  // scores of keys 64kh + [0, 32) and 64kh + [32, 64)
        tmem_ld_half32<64>(tS, sa);
        tmem_ld_half32<64>(tS + 32, sb);
        tmem_wait_ld_regs2(sa, sb);
        if (!((all_valid >> j) & 1u)) {  // partial tile: invalid keys score -inf, so their p is 0
#pragma unroll
          for (int x = 0; x < 32; ++x) {
            if (!((v_lo >> x) & 1u)) sa[x] = 0xff800000u;
            if (!((v_hi >> x) & 1u)) sb[x] = 0xff800000u;
          }
        }
        float mt;
        {
          float m0 = -INFINITY, m1 = -INFINITY, m2 = -INFINITY, m3 = -INFINITY;
#pragma unroll
          for (int x = 0; x < 32; x += 2) {
            m0 = fmaxf(m0, __uint_as_float(sa[x]));
            m1 = fmaxf(m1, __uint_as_float(sa[x + 1]));
            m2 = fmaxf(m2, __uint_as_float(sb[x]));
            m3 = fmaxf(m3, __uint_as_float(sb[x + 1]));
          }
          mt = fmaxf(fmaxf(m0, m1), fmaxf(m2, m3));
        }
        mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 16));  // the tile's max of head h (finite:
                                                                // a tile in the mask has a valid key)
        const float xt = mt * p.scale_log2;
        bool resc = false;
        float alpha = 1.0f;
        if (m_run == -INFINITY) {
          m_run = xt;  // first tile of the token: its PV starts O from zero
        } else if (xt > m_run + kLazyRescale) {
          alpha = fast_exp2(m_run - xt);
          m_run = xt;
          resc = true;
        }
        l_run *= alpha;
        // P = 2^(x - m_run) (0 for invalid keys) as bf16 pairs over the tile's first 64 columns:
        // keys 64kh + [0, 64) -> columns 32kh + [0, 32), the A operand of this tile's PV MMA
        // (the S values were all read above, by both halves of the warp)
        {
          uint32_t pw[16];
          float la = 0.0f, lb = 0.0f;
#pragma unroll
          for (int x2 = 0; x2 < 16; ++x2) {
            const float p0 = fast_exp2(fmaf(__uint_as_float(sa[2 * x2]), p.scale_log2, -m_run));
            const float p1 = fast_exp2(fmaf(__uint_as_float(sa[2 * x2 + 1]), p.scale_log2, -m_run));
            la += p0;
            lb += p1;
            pw[x2] = pack_bf16x2(p0, p1);
          }
          tmem_st_half16<32>(tS, pw);  // columns 32kh + [0, 16)
#pragma unroll
          for (int x2 = 0; x2 < 16; ++x2) {
            const float p0 = fast_exp2(fmaf(__uint_as_float(sb[2 * x2]), p.scale_log2, -m_run));
            const float p1 = fast_exp2(fmaf(__uint_as_float(sb[2 * x2 + 1]), p.scale_log2, -m_run));
            la += p0;
            lb += p1;
            pw[x2] = pack_bf16x2(p0, p1);
          }
          tmem_st_half16<32>(tS + 16, pw);  // columns 32kh + [16, 32)
          l_run += la + lb;
        }
        if (__any_sync(0xffffffffu, resc)) {
          // O must hold every PV of this token up to tile jj-1 before it is rescaled (and this
          // tile's PV, which waits for p_ready, comes after)
          ok = mbar_wait(&bar.pv_done, (gs - 1) & 1, &abort_flag, p.err) && ok;
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t o[32];
            tmem_ld_half32<128>(t_lanes + c * 32, o);
            tmem_wait_ld_regs(o);
#pragma unroll
            for (int x = 0; x < 32; ++x) o[x] = __float_as_uint(__uint_as_float(o[x]) * alpha);
            tmem_st_half32<128>(t_lanes + c * 32, o);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bar.p_ready[gs & 1]);
      }
      // ---- epilogue of this token: head h, d_v 128kh..128kh+127
      const float l = l_run + __shfl_xor_sync(0xffffffffu, l_run, 16);
      const float inv = 1.0f / l;
      if (p.split == 1 && p.lse && kh == 0) p.lse[(size_t)tok * kH + h] = (m_run + __log2f(l)) * 0.69314718055994531f;
      ok = mbar_wait(&bar.o_full[hf], (it >> 1) & 1, &abort_flag, p.err) && ok;
      tc_fence_after();
      if (p.split > 1) {  // unnormalised fp32 O rows and (max, sum) of this part
        if (kh == 0) {
          p.ws_ml[(size_t)unit * 2 * kH + h] = m_run;
          p.ws_ml[(size_t)unit * 2 * kH + kH + h] = l;
        }
        float4* orow = reinterpret_cast<float4*>(p.ws_O + ((size_t)unit * kH + h) * kD + kh * 128);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t o[32];
          tmem_ld_half32<128>(t_lanes + c * 32, o);
          tmem_wait_ld_regs(o);
#pragma unroll
          for (int q = 0; q < 8; ++q)
            orow[c * 8 + q] = make_float4(__uint_as_float(o[4 * q]), __uint_as_float(o[4 * q + 1]),
                                          __uint_as_float(o[4 * q + 2]), __uint_as_float(o[4 * q + 3]));
        }
      } else {
        uint4* orow = reinterpret_cast<uint4*>(obase + (size_t)h * kD + kh * 128);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t o[32];
          tmem_ld_half32<128>(t_lanes + c * 32, o);
          tmem_wait_ld_regs(o);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(o[8 * q + 0]) * inv, __uint_as_float(o[8 * q + 1]) * inv);
            w.y = pack_bf16x2(__uint_as_float(o[8 * q + 2]) * inv, __uint_as_float(o[8 * q + 3]) * inv);
            w.z = pack_bf16x2(__uint_as_float(o[8 * q + 4]) * inv, __uint_as_float(o[8 * q + 5]) * inv);
            w.w = pack_bf16x2(__uint_as_float(o[8 * q + 6]) * inv, __uint_as_float(o[8 * q + 7]) * inv);
            orow[c * 4 + q] = w;
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&bar.o_empty[hf]);
      softmax_bar();  // every softmax thread has read the row before it is refilled
      refill_idx_row(p, bar, sIdx_a, buf, i, unit + 2 * gridDim.x, tid, abort_flag, ok);
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

// Split mode: O of a token = sum over its parts of 2^(m_p - M) O_p / sum of 2^(m_p - M) l_p,
// M = max m_p over the parts with l_p > 0 (the same online-softmax merge the kernel does per
// tile); lse = (M + log2 of the denominator) ln 2.  A token with no valid entry in any part
// gets O = 0 and lse = -inf.  One CTA per token; thread t: head t / 4, d_v 64 (t % 4) .. +63.
constexpr int kMaxSplit = 8;

__global__ void __launch_bounds__(256) dsa_combine_kernel(const float* __restrict__ ws_O,
                                                          const float* __restrict__ ws_ml, uint16_t* __restrict__ O,
                                                          float* __restrict__ lse, int split) {
  const int tok = blockIdx.x;
  const int h = threadIdx.x >> 2, q4 = threadIdx.x & 3;
  const size_t u0 = (size_t)tok * split;
  float M = -INFINITY;
  for (int s = 0; s < split; ++s) {
    const float* ml = ws_ml + (u0 + s) * 2 * kH;
    if (ml[kH + h] > 0.0f) M = fmaxf(M, ml[h]);
  }
  float acc[64];
#pragma unroll
  for (int x = 0; x < 64; ++x) acc[x] = 0.0f;
  float den = 0.0f;
  for (int s = 0; s < split; ++s) {
    const float* ml = ws_ml + (u0 + s) * 2 * kH;
    const float l = ml[kH + h];
    if (!(l > 0.0f)) continue;  // a part without tiles left its O rows unwritten
    const float w = exp2f(ml[h] - M);
    den += w * l;
    const float4* src = reinterpret_cast<const float4*>(ws_O + ((u0 + s) * kH + h) * kD + q4 * 64);
#pragma unroll
    for (int x = 0; x < 16; ++x) {
      const float4 v = src[x];
      acc[4 * x] = fmaf(w, v.x, acc[4 * x]);
      acc[4 * x + 1] = fmaf(w, v.y, acc[4 * x + 1]);
      acc[4 * x + 2] = fmaf(w, v.z, acc[4 * x + 2]);
      acc[4 * x + 3] = fmaf(w, v.w, acc[4 * x + 3]);
    }
  }
  const float inv = den > 0.0f ? 1.0f / den : 0.0f;
  uint4* dst = reinterpret_cast<uint4*>(O + ((size_t)tok * kH + h) * kD + q4 * 64);
#pragma unroll
  for (int x = 0; x < 8; ++x) {
    uint4 w;
    w.x = pack_bf16x2(acc[8 * x] * inv, acc[8 * x + 1] * inv);
    w.y = pack_bf16x2(acc[8 * x + 2] * inv, acc[8 * x + 3] * inv);
    w.z = pack_bf16x2(acc[8 * x + 4] * inv, acc[8 * x + 5] * inv);
    w.w = pack_bf16x2(acc[8 * x + 6] * inv, acc[8 * x + 7] * inv);
    dst[x] = w;
  }
  if (lse && q4 == 0) lse[(size_t)tok * kH + h] = den > 0.0f ? (M + __log2f(den)) * 0.69314718055994531f : -INFINITY;
}

// Parts per token: only calls with at most half as many tokens as SMs split (decode batches),
// into as many parts as fill the SMs, at most kMaxSplit and at most one per key tile.
int split_of(int n_tok, int k, int sms) {
  if (n_tok <= 0 || sms <= 0 || 2 * n_tok > sms) return 1;
  const int n_tiles = (k + kKeyTile - 1) / kKeyTile;
  int s = sms / n_tok;
  if (s > kMaxSplit) s = kMaxSplit;
  if (s > n_tiles) s = n_tiles;
  return s < 1 ? 1 : s;
}

constexpr size_t kUnitWsBytes = (size_t)kH * kD * 4 + 2 * kH * 4;  // O rows + (max, sum) per unit

hcadsa_status check_args(const hcadsa_bf16* Q, const hcadsa_bf16* K, const hcadsa_bf16* V, const int32_t* idx,
                         hcadsa_bf16* O, float* lse, int B, int Lq, int Lk, int Hq, int d, int k, float scale) {
  if (!Q || !K || !V || !idx || !O) return HCADSA_ERR_NULL;
  if (B < 0 || Lq < 0 || Lk < 0 || k <= 0 || !(scale > 0.0f)) return HCADSA_ERR_SHAPE;
  if (d != kD || Hq != kH || k > kMaxK) return HCADSA_ERR_UNSUPPORTED;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(idx) ||
      (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)))
    return HCADSA_ERR_ALIGN;
  if ((long long)B * Lq > 2147483647LL || (long long)B * Lk > 2147483647LL) return HCADSA_ERR_UNSUPPORTED;
  return HCADSA_OK;
}

hcadsa_status launch(const hcadsa_bf16* Q, const hcadsa_bf16* K, const hcadsa_bf16* V, const int32_t* idx,
                     hcadsa_bf16* O, float* lse, int B, int Lq, int Lk, int k, float scale, int split, float* ws,
                     int sms, hcadsa_stream stream) {
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
  p.split = split;
  p.n_units = p.n_tok * split;
  p.ws_O = split > 1 ? ws : nullptr;
  p.ws_ml = split > 1 ? ws + (size_t)p.n_units * kH * kD : nullptr;
  if (cudaFuncSetAttribute(dsa_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) != cudaSuccess)
    return HCADSA_ERR_CUDA;
  const int grid = p.n_units < sms ? p.n_units : sms;
  dsa_attn_kernel<<<grid, kThreads, kSmemBytes, as_stream(stream)>>>(mq, p);
  if (split > 1) {
    const hcadsa_status st = launch_status();
    if (st != HCADSA_OK) return st;
    dsa_combine_kernel<<<p.n_tok, 256, 0, as_stream(stream)>>>(p.ws_O, p.ws_ml, reinterpret_cast<uint16_t*>(O), lse,
                                                               split);
  }
  return launch_status();
}

}  // namespace
}  // namespace hcadsa

extern "C" hcadsa_status dsa_sparse_attn_fwd(const hcadsa_bf16* Q, const hcadsa_bf16* K, const hcadsa_bf16* V,
                                             const int32_t* idx, hcadsa_bf16* O, float* lse, int B, int Lq, int Lk,
                                             int Hq, int d, int k, float scale, hcadsa_stream stream) {
  using namespace hcadsa;
  const hcadsa_status st = check_args(Q, K, V, idx, O, lse, B, Lq, Lk, Hq, d, k, scale);
  if (st != HCADSA_OK) return st;
  if (B == 0 || Lq == 0) return HCADSA_OK;
  const int sms = num_sms_current_device();
  if (sms <= 0) return HCADSA_ERR_CUDA;
  return launch(Q, K, V, idx, O, lse, B, Lq, Lk, k, scale, 1, nullptr, sms, stream);
}

extern "C" size_t dsa_sparse_attn_fwd_workspace_size(int B, int Lq, int k) {
  using namespace hcadsa;
  if (B <= 0 || Lq <= 0 || k <= 0 || k > kMaxK || (long long)B * Lq > 2147483647LL) return 0;
  const int sms = num_sms_current_device();
  const int split = split_of(B * Lq, k, sms);
  return split > 1 ? (size_t)B * Lq * split * kUnitWsBytes : 0;
}

extern "C" hcadsa_status dsa_sparse_attn_fwd_ws(const hcadsa_bf16* Q, const hcadsa_bf16* K, const hcadsa_bf16* V,
                                                const int32_t* idx, hcadsa_bf16* O, float* lse, int B, int Lq,
                                                int Lk, int Hq, int d, int k, float scale, void* workspace,
                                                size_t workspace_bytes, hcadsa_stream stream) {
  using namespace hcadsa;
  const hcadsa_status st = check_args(Q, K, V, idx, O, lse, B, Lq, Lk, Hq, d, k, scale);
  if (st != HCADSA_OK) return st;
  if (B == 0 || Lq == 0) return HCADSA_OK;
  const int sms = num_sms_current_device();
  if (sms <= 0) return HCADSA_ERR_CUDA;
  const int split = split_of(B * Lq, k, sms);
  if (split > 1) {
    if (!workspace || workspace_bytes < (size_t)B * Lq * split * kUnitWsBytes) return HCADSA_ERR_WORKSPACE;
    if (!aligned16(workspace)) return HCADSA_ERR_ALIGN;
  }
  return launch(Q, K, V, idx, O, lse, B, Lq, Lk, k, scale, split, static_cast<float*>(workspace), sms, stream);
}
