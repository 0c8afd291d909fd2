/*
 * hcadsa.h -- C ABI of the hybrid sparse attention forward (HCA + MLA-DSA) on
 * NVIDIA B200 (sm_100a).  Library: sparse_attention_hca_b200/libhcadsa.so.
 *
 * The method, as the pages state it:
 *   "Baidu open-sourced a brand-new pretraining model, still focusing on
 *   efficiency with Flash" (blog.mirrorspeed.com), section "Hybrid sparse
 *   attention, 1/7 full context access"; the same section of "Baidu
 *   Open-Sources ERNIE 5.5 Flash Base: Efficient 280B MoE for Agents"
 *   (besthub.dev, "Core Architectural Innovations", item 1); and the ai-club.cn
 *   article, section "混合注意力（MLA + HCA）" (512-wide HCA heads, 256-wide
 *   MLA heads).  HCA layers compress every 128 tokens into one cache entry and
 *   attend over the compressed entries plus a short recent raw window; MLA
 *   layers use DSA: an indexer scores earlier positions per query and
 *   attention runs over the top-k positions only.
 *
 * Conventions for every call:
 *   - All tensor pointers are DEVICE pointers owned by the caller; the library
 *     never allocates, frees or retains them.  Tensors are dense, row-major,
 *     last dimension contiguous.  bf16 tensors hold raw bfloat16 bit patterns.
 *   - Every tensor pointer must be 16-byte aligned (HCADSA_ERR_ALIGN otherwise).
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream) and only enqueue kernels; they are thread-safe.
 *   - Errors the host can see (null pointers, shapes, alignment, unsupported
 *     sizes, short workspace, launch failures) are returned before anything is
 *     enqueued.  Errors only the device can see (a bounded wait that expired,
 *     an index out of range) are recorded in a per-device error word that
 *     hcadsa_check_device_error() reads and clears.
 *   - Query row r of batch b sits at absolute position t = q_offset + r.
 *     Prefill: q_offset = 0, Lq = L.  Decode: Lq = 1, q_offset = t.
 */
#ifndef HCADSA_H_
#define HCADSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t hcadsa_bf16; /* bfloat16 bit pattern */
typedef void* hcadsa_stream;  /* cudaStream_t */

typedef enum {
  HCADSA_OK = 0,
  HCADSA_ERR_NULL = -1,          /* a required pointer is NULL */
  HCADSA_ERR_SHAPE = -2,         /* sizes inconsistent with each other */
  HCADSA_ERR_ALIGN = -3,         /* a pointer is not 16-byte aligned */
  HCADSA_ERR_UNSUPPORTED = -4,   /* valid but not implemented (e.g. head dim) */
  HCADSA_ERR_WORKSPACE = -5,     /* workspace missing or too small */
  HCADSA_ERR_CUDA = -6,          /* a CUDA runtime/driver call failed */
  HCADSA_ERR_TIMEOUT = -7,       /* device: a bounded wait expired */
  HCADSA_ERR_DEVICE_BOUNDS = -8  /* device: an index input was out of range */
} hcadsa_status;

/* Library version (major*10000 + minor*100 + patch). */
int hcadsa_version(void);

/* Human-readable name of a status code (static string, never NULL). */
const char* hcadsa_status_string(hcadsa_status status);

/*
 * Message of the last CUDA runtime error this thread saw inside the library (after a call
 * returned HCADSA_ERR_CUDA); "" if none.  Static thread-local storage, never NULL.
 */
const char* hcadsa_last_error_string(void);

/*
 * Synchronises `stream`, then returns and clears the device error word of the
 * current device (HCADSA_OK if no kernel recorded an error).  Returns
 * HCADSA_ERR_CUDA if the synchronisation itself failed.
 */
hcadsa_status hcadsa_check_device_error(hcadsa_stream stream);

/*
 * Self-test of the device-side failure path (no counterpart on the pages): launches one
 * block that waits on a barrier nothing arrives on, with a limit of `timeout_us`
 * microseconds (1 .. 10^7).  The wait gives up, records HCADSA_ERR_TIMEOUT in the device
 * error word and the kernel returns normally; a following hcadsa_check_device_error()
 * reports it.  Every wait inside the library's kernels uses the same bounded mechanism
 * (limit 2 s), so a lost arrival turns into an error status instead of a hung GPU.
 */
hcadsa_status hcadsa_selftest_bounded_wait(unsigned timeout_us, hcadsa_stream stream);

/*
 * HCA block compression.  Source: mirrorspeed / besthub sections cited above
 * (the cache keeps one entry per 128 tokens).  Compressor form
 * (the pages leave it open): entry j of head h, channel c is
 *     acc = 0; for i in 0..blk-1: acc = fma(w[i], X[b, blk*j + i, h, c], acc)
 *     Xc[b, j, h, c] = bf16_round_nearest_even(acc)
 * with fp32 accumulation in ascending i, applied to K and V with the same w.
 * Only complete blocks are compressed: n_c = floor(L / blk) entries.
 *
 *   K, V   : [B, L, Hkv, d] bf16              (read)
 *   w      : [blk] fp32                        (read)
 *   Kc, Vc : [B, L/blk, Hkv, d] bf16           (written)
 *   d must be a multiple of 8; 1 <= blk <= 1024.
 */
hcadsa_status hca_compress_kv(const hcadsa_bf16* K, const hcadsa_bf16* V, const float* w, hcadsa_bf16* Kc,
                              hcadsa_bf16* Vc, int B, int L, int Hkv, int d, int blk, hcadsa_stream stream);

/*
 * Size in bytes of the workspace hca_attn_fwd needs for these sizes on the current
 * device (0 if the sizes are invalid or unsupported; the call then reports why).
 * The kernel computes each probability tile P once, for the first half of the
 * 512-wide value dimension, and keeps it in this workspace (bf16, plus one fp32
 * rescale factor per row and key tile) for the second half:
 *     min(#units, #SMs) * J_max * (128*128*2 + 128*4) bytes,
 * where #tiles = B * Hkv * ceil(Lq / (128 / (Hq/Hkv))) row tiles and J_max =
 * ceil(n_c(t_last)/128) + floor((128/(Hq/Hkv) + W + 126) / 128) key tiles.  #units =
 * #tiles, except when #tiles <= #SMs/2: then every row tile's key tiles are split over
 * several CTAs (#units <= #SMs, at most 64 per row tile, each with at least one key tile;
 * when all row tiles have the same number of key tiles, as in decode, each of #SMs CTAs
 * takes an equal share of all of them and #units = #SMs + #tiles record slots), and the
 * workspace also holds each unit's partial result, 128 * (512*4 + 8) bytes per unit, for
 * the combine pass.  The workspace holds no state between calls; concurrent calls need
 * separate workspaces.
 */
size_t hca_attn_fwd_workspace_size(int B, int Lq, int q_offset, int Hq, int Hkv, int d, int n_c, int blk,
                                   int W);

/*
 * HCA attention forward.  Source: the sections cited above (a query attends to
 * the compressed entries and to a short window of the latest raw tokens, and to
 * nothing else; 512-wide heads).  Visible set of a query at position t (reading of
 * the pages, which do not say how the two parts meet):
 *     raw window  s in [max(0, t-W+1), t]
 *     entries     j in [0, n_c(t)),  n_c(t) = max(0, floor((t-W+1)/blk))
 * i.e. an entry is visible once every token it summarises lies before the
 * window.  One softmax over the union, scores = scale * <q, k>:
 *     O[b,r,h,:] = sum_k softmax_k(score) * v_k,   lse = log sum_k exp(score)
 * Query head h reads K/V head h / (Hq/Hkv).
 *
 *   Q        : [B, Lq, Hq, d] bf16
 *   Kc, Vc   : [B, n_c, Hkv, d] bf16   compressed entries (may be NULL iff n_c == 0)
 *   Kw, Vw   : [B, n_w, Hkv, d] bf16   raw tokens; row i holds position win_start + i
 *              (prefill: Kw = K, win_start = 0, n_w = L)
 *   O        : [B, Lq, Hq, d] bf16     (written)
 *   lse      : [B, Lq, Hq] fp32 natural-log log-sum-exp, or NULL
 *   workspace: at least hca_attn_fwd_workspace_size(...) bytes of device memory, 16-byte
 *              aligned (HCADSA_ERR_WORKSPACE if NULL or smaller, HCADSA_ERR_ALIGN if misaligned)
 * Requirements: d == 512; Hq % Hkv == 0 and (Hq/Hkv) divides 128; every query
 * must have its window inside [win_start, win_start + n_w) and n_c(t) <= n_c.
 */
hcadsa_status hca_attn_fwd(const hcadsa_bf16* Q, const hcadsa_bf16* Kc, const hcadsa_bf16* Vc, int n_c,
                           const hcadsa_bf16* Kw, const hcadsa_bf16* Vw, int win_start, int n_w, hcadsa_bf16* O,
                           float* lse, int B, int Lq, int q_offset, int Hq, int Hkv, int d, int blk, int W,
                           float scale, void* workspace, size_t workspace_bytes, hcadsa_stream stream);

/*
 * HCA attention with FlashMask-4's head shape: 576-wide scores, 512-wide values.  Source: the
 * mirrorspeed page, section "More structural improvements, data, and infrastructure", and the
 * ai-club.cn article, section "训练：Muon 优化器 + 自研注意力算子" (an attention operator for
 * qk_head_dim 576 / v_head_dim 512, meant for HCA's 512-wide heads).  Reading taken (MLA-style
 * shared latent): a key row is 576 wide -- the 512-wide latent and a 64-wide positional slice --
 * and the value of a key is the first 512 columns of the same row, so the caches hold one
 * tensor per part (entries Kc, raw window Kw) and no separate V.  Visible set, softmax, lse,
 * layouts of Q/O/lse, workspace rules and errors as hca_attn_fwd, with
 *   Q      : [B, Lq, Hq, 576] bf16         scores use all 576 columns
 *   Kc, Kw : [B, n_c | n_w, Hkv, 576] bf16 (Kc may be NULL iff n_c == 0)
 *   O      : [B, Lq, Hq, 512] bf16
 * Requirements: dqk == 576, dv == 512 (HCADSA_ERR_UNSUPPORTED otherwise).  scale is usually
 * 1/sqrt(576).  The workspace size is that of hca_attn_fwd with d = 512.
 */
size_t hca_attn_fwd_latent_workspace_size(int B, int Lq, int q_offset, int Hq, int Hkv, int dqk, int dv, int n_c,
                                          int blk, int W);
hcadsa_status hca_attn_fwd_latent(const hcadsa_bf16* Q, const hcadsa_bf16* Kc, int n_c, const hcadsa_bf16* Kw,
                                  int win_start, int n_w, hcadsa_bf16* O, float* lse, int B, int Lq, int q_offset,
                                  int Hq, int Hkv, int dqk, int dv, int blk, int W, float scale, void* workspace,
                                  size_t workspace_bytes, hcadsa_stream stream);

/*
 * Size in bytes of the workspace dsa_index_topk needs.
 *   - Lq >= 64 query rows per sequence (prefill, chunked prefill): B * 512 bytes -- the
 *     per-channel min and max of k_idx.  Scoring and selection run fused on the tensor cores
 *     and keep no score matrix, so the workspace does not grow with the sequence.
 *   - Lq < 64 (decode shapes): the int32 indexer score rows,
 *         B * Lq * round_up(min(q_offset + Lq, Lk), 128) * 4 bytes
 *     (4 MiB per row at 1M keys), plus, for few query rows over many keys (B*Lq <= 64 and at
 *     least 32768 keys, where the selection is spread over all SMs), per row 16 + 2048*4 +
 *     8192*8 bytes of selection state (score range, histogram, candidate list).
 */
size_t dsa_index_topk_workspace_size(int B, int Lq, int q_offset, int Lk, int k);

/*
 * DSA indexer + per-query top-k.  Source: mirrorspeed / besthub sections cited
 * above (a small scoring network rates every earlier position for each query,
 * and attention then covers only the k best-rated positions).  Indexer form
 * (left open by the pages):
 *     score[t, s] = sum_j w_idx[j] * sum_c q_idx[b, r, j, c] * k_idx[b, s, c]
 * exact in int32.  Candidates of a query at t are the positions s <= t with
 * s < Lk (its own position included).  The k candidates with the largest
 * (score, -s) are kept -- equal scores go to the lower position -- and written
 * in ascending position order, padded with -1 when fewer than k exist.
 *
 *   q_idx : [B, Lq, H_idx, d_idx] int8
 *   k_idx : [B, Lk, d_idx] int8          (one key shared by the indexer heads)
 *   w_idx : [H_idx] int32  (device)
 *   idx   : [B, Lq, k] int32             (written)
 *   ws    : workspace of dsa_index_topk_workspace_size(...) bytes
 * Requirements: H_idx == 4, d_idx == 64, 1 <= k <= 4096.  The caller keeps
 * sum_j |w_idx[j]| <= 2047, so that no score (|q . k| <= 64 * 128 * 128 = 2^20 per head)
 * overflows int32; this is not checked.
 */
hcadsa_status dsa_index_topk(const int8_t* q_idx, const int8_t* k_idx, const int32_t* w_idx, int32_t* idx,
                             void* ws, size_t ws_bytes, int B, int Lq, int q_offset, int Lk, int H_idx, int d_idx,
                             int k, hcadsa_stream stream);

/*
 * CSA selection: indexer + per-query top-k over compressed entries.  Source: the mirrorspeed
 * page, section "Hybrid sparse attention, 1/7 full context access" (and the besthub page,
 * "Core Architectural Innovations"): the alternative the pages compare HCA + MLA against,
 * compressed sparse attention, compresses the history 4:1 and then selects sparsely.  Reading
 * taken (the pages give no more): entry j summarises tokens blk*j .. blk*j + blk - 1 (made by
 * hca_compress_kv with block size blk), carries its own indexer key kc_idx[j], and becomes a
 * candidate of the query at t once its block is complete:
 *     candidates of t = entries j < min(floor((t + 1) / blk), n_c)      (no raw window)
 * Scores, tie rule and output as in dsa_index_topk (entry numbers instead of positions).  The
 * CSA layer is then hca_compress_kv(blk) -> csa_index_topk -> dsa_sparse_attn_fwd over the
 * compressed K/V (a query with no complete block gets O = 0, lse = -inf).
 *
 *   q_idx  : [B, Lq, H_idx, d_idx] int8
 *   kc_idx : [B, n_c, d_idx] int8      (one indexer key per compressed entry)
 *   w_idx  : [H_idx] int32 (device)
 *   idx    : [B, Lq, k] int32          (written: ascending entry numbers, -1 padded)
 *   ws     : workspace of csa_index_topk_workspace_size(...) bytes
 * Requirements and errors as dsa_index_topk; blk >= 1 (HCADSA_ERR_SHAPE otherwise).  With
 * blk = 1 it is dsa_index_topk over n_c positions.
 */
size_t csa_index_topk_workspace_size(int B, int Lq, int q_offset, int n_c, int k, int blk);
hcadsa_status csa_index_topk(const int8_t* q_idx, const int8_t* kc_idx, const int32_t* w_idx, int32_t* idx,
                             void* ws, size_t ws_bytes, int B, int Lq, int q_offset, int n_c, int H_idx, int d_idx,
                             int k, int blk, hcadsa_stream stream);

/*
 * DSA indexer + top-k without any device allocation by anyone.  The pages have no
 * counterpart: this is a library convenience for callers that cannot allocate device
 * memory -- code that must not call cudaMalloc/cudaFree on its hot path (those calls can
 * stall the device), plugins hosted by a framework that owns all device memory, or callers
 * with no workspace allocator at all.  Same arguments, computation and result as
 * dsa_index_topk, minus the workspace: the int32 score rows go to a fixed scratch array of
 * dsa_index_topk_noalloc_max_scratch_bytes() bytes (64 MiB) compiled into the library.
 * Every GPU that loads the library holds that array until the process exits.
 *   - Calls whose int32 score rows (B * Lq * round_up(min(q_offset + Lq, Lk), 128) * 4
 *     bytes) exceed the maximum return HCADSA_ERR_WORKSPACE before anything is enqueued.  This
 *     entry always selects with one thread block per query row.  Example limits:
 *     prefill up to 4096 x 4096, or decode (Lq = 1) of 16 sequences at 1M keys.
 *   - The first call on each device looks up the array's device address (one
 *     cudaGetSymbolAddress, no allocation); make that first call before any stream capture.
 *   - All calls share the one array and it keeps the last call's scores.  Nothing in it needs
 *     clearing (every score a call reads is written earlier in the same call), but calls whose
 *     kernels overlap on the GPU (different streams, or several host threads) race on it:
 *     serialise them.
 */
size_t dsa_index_topk_noalloc_max_scratch_bytes(void);
hcadsa_status dsa_index_topk_noalloc(const int8_t* q_idx, const int8_t* k_idx, const int32_t* w_idx, int32_t* idx,
                                     int B, int Lq, int q_offset, int Lk, int H_idx, int d_idx, int k,
                                     hcadsa_stream stream);

/*
 * DSA sparse attention forward.  Source: mirrorspeed / besthub sections cited
 * above, and the ai-club.cn section for the 256-wide MLA heads.  All Hq query
 * heads read one shared K/V head (the MLA latent reading) and share the index
 * row of their query:
 *     O[b,r,h,:] = sum_{s in idx[b,r]} softmax_s(scale * <Q[b,r,h], K[b,s]>) V[b,s]
 * Entries < 0 in idx are padding; the order of entries does not matter.
 *
 *   Q   : [B, Lq, Hq, d] bf16
 *   K, V: [B, Lk, d] bf16
 *   idx : [B, Lq, k] int32, entries in [0, Lk) or < 0
 *   O   : [B, Lq, Hq, d] bf16 (written); lse: [B, Lq, Hq] fp32 or NULL
 * Requirements: d == 256, Hq == 64, 1 <= k <= 4096 (HCADSA_ERR_UNSUPPORTED
 * otherwise), scale > 0 (HCADSA_ERR_SHAPE otherwise: the kernel takes each tile's maximum
 * over the unscaled scores).  An entry >= Lk is skipped and recorded as
 * HCADSA_ERR_DEVICE_BOUNDS.
 */
hcadsa_status dsa_sparse_attn_fwd(const hcadsa_bf16* Q, const hcadsa_bf16* K, const hcadsa_bf16* V,
                                  const int32_t* idx, hcadsa_bf16* O, float* lse, int B, int Lq, int Lk, int Hq,
                                  int d, int k, float scale, hcadsa_stream stream);

/*
 * The same computation with a caller-provided workspace, for calls with few query rows
 * (decode batches): when B*Lq is at most half the number of SMs of the current device, each
 * row's key tiles (128 entries of its index row each) are divided among up to 8 CTAs, which
 * write unnormalised fp32 partial outputs and per-head (max, sum) pairs to the workspace; a
 * second kernel on the same stream merges them (the online-softmax merge) and writes O and
 * lse.  Same arguments, requirements and result as dsa_sparse_attn_fwd (up to the rounding of
 * the merge), plus:
 *   workspace      : device memory of at least dsa_sparse_attn_fwd_workspace_size(B, Lq, k)
 *                    bytes, 16-byte aligned; caller-owned, contents need no initialisation and
 *                    are scratch after the call.  Calls that share a workspace must be
 *                    serialised on one stream.
 *   workspace_bytes: its size.  HCADSA_ERR_WORKSPACE if the call splits and the workspace is
 *                    NULL or smaller, HCADSA_ERR_ALIGN if it is misaligned.
 * dsa_sparse_attn_fwd_workspace_size returns 0 when the call does not split (then workspace
 * may be NULL and the call runs exactly as dsa_sparse_attn_fwd), and for invalid shapes; it
 * depends on the current device's SM count.
 */
size_t dsa_sparse_attn_fwd_workspace_size(int B, int Lq, int k);
hcadsa_status dsa_sparse_attn_fwd_ws(const hcadsa_bf16* Q, const hcadsa_bf16* K, const hcadsa_bf16* V,
                                     const int32_t* idx, hcadsa_bf16* O, float* lse, int B, int Lq, int Lk, int Hq,
                                     int d, int k, float scale, void* workspace, size_t workspace_bytes,
                                     hcadsa_stream stream);

/*
 * Attention output gate + virtual-head mix, fused (tensor-core GEMM + epilogue).  Source: the
 * mirrorspeed page, section "Hybrid sparse attention, 1/7 full context access" (last
 * paragraph), and the besthub page, "Core Architectural Innovations": low-rank gated attention
 * computes the output gate from the layer's low-rank query latent (a quarter of the hidden
 * width); virtual head attention (VHA) mixes the heads with a light low-rank term beside an
 * identity path and can be folded into the attention operator at inference.  Reading taken
 * (the pages give no formulas): elementwise gate, mix applied per token and channel before it:
 *     Ohat[t,h,c] = O[t,h,c] + sum_{m<r} U[h,m] * sum_h' V[h',m] * O[t,h',c]
 *     Y[t,h,c]    = sigmoid(sum_i cq[t,i] * Wg[h*dv + c, i]) * Ohat[t,h,c]
 *
 *   O  : [B, L, H, dv] bf16   attention output (hca_attn_fwd / dsa_sparse_attn_fwd)
 *   cq : [B, L, rq] bf16      low-rank query latent
 *   Wg : [H*dv, rq] bf16      gate projection (row h*dv + c: head h, channel c)
 *   U, V: [H, r] fp32 (device; may be NULL iff r == 0)
 *   Y  : [B, L, H, dv] bf16   (written; must not alias O)
 * Requirements: H in {16, 32, 64} (HCA: 16 heads of 512, DSA: 64 heads of 256); dv a multiple of
 * 256 / H and of 8; rq a multiple of 64; 0 <= r <= 4.  HCADSA_ERR_UNSUPPORTED otherwise.
 */
hcadsa_status attn_gate_vha_fwd(const hcadsa_bf16* O, const hcadsa_bf16* cq, const hcadsa_bf16* Wg, const float* U,
                                const float* V, hcadsa_bf16* Y, int B, int L, int H, int dv, int rq, int r,
                                hcadsa_stream stream);

/* ------------------------------------------------------------------ backward pass */

/*
 * Backward of the HCA compressor.  Source: the sections cited for hca_compress_kv (one cache
 * entry per block of tokens); with the compressor form fixed there the map is linear,
 *     Xc[b, j, h, c] = sum_i w[i] * X[b, blk*j + i, h, c],
 * and its adjoint, for a gradient dXc of the entries, is
 *     dX[b, blk*j + i, h, c] += w[i] * dXc[b, j, h, c]       (tail tokens past the last
 *                                                              complete block get nothing)
 *     dw[i]                  += sum_{b, j, h, c} dXc[b, j, h, c] * X[b, blk*j + i, h, c]
 * (the bf16 rounding of the forward is not differentiated).  Both outputs are ADDED to, so the
 * compressor's share of a key or value gradient can be added to the share of the raw window;
 * zero them first for the compressor's share alone.  dw is summed with fp32 atomics (order not
 * fixed: results can differ in the last bits between runs).
 *
 *   X   : [B, L, H, d] bf16       (the forward input, K or V)
 *   w   : [blk] fp32
 *   dXc : [B, L/blk, H, d] fp32
 *   dX  : [B, L, H, d] fp32       (accumulated)
 *   dw  : [blk] fp32              (accumulated)
 * Requirements: d a multiple of 8, 1 <= blk <= 1024; X, dXc, dX 16-byte aligned.
 */
hcadsa_status hca_compress_bwd(const hcadsa_bf16* X, const float* w, const float* dXc, float* dX, float* dw, int B,
                               int L, int H, int d, int blk, hcadsa_stream stream);

/*
 * Backward of DSA sparse attention.  Source: the forward above (the mirrorspeed page, section
 * "Hybrid sparse attention, 1/7 full context access": attention over the k selected positions;
 * 64 heads of 256 on one shared K/V head).  For a loss with output gradient dO, with the
 * forward's probabilities p[h, s] = exp(scale <Q[h], K[s]> - lse[h]) over the selected s:
 *     D[h]    = <dO[h], O[h]>
 *     dS[h,s] = p[h,s] (<dO[h], V[s]> - D[h])
 *     dQ[h]   = scale sum_s dS[h,s] K[s]                      (written)
 *     dK[s]  += scale sum_h dS[h,s] Q[h],  dV[s] += sum_h p[h,s] dO[h]   (ADDED to)
 * P and dS enter the tensor cores as bf16; accumulation is fp32.  dK and dV are summed over
 * tokens with fp32 atomics (order not fixed: results can differ in the last bits between
 * runs); zero them first.  Padding entries (< 0) contribute nothing; an entry >= Lk is skipped
 * and recorded as HCADSA_ERR_DEVICE_BOUNDS.
 *
 *   Q, O, dO : [B, Lq, Hq, d] bf16 (O and lse from dsa_sparse_attn_fwd)
 *   K, V     : [B, Lk, d] bf16
 *   idx      : [B, Lq, k] int32 (as for the forward)
 *   lse      : [B, Lq, Hq] fp32, natural log
 *   dQ       : [B, Lq, Hq, d] fp32 (written)
 *   dK, dV   : [B, Lk, d] fp32 (accumulated)
 * Requirements: d == 256, Hq == 64, 1 <= k <= 4096.
 */
hcadsa_status dsa_sparse_attn_bwd(const hcadsa_bf16* Q, const hcadsa_bf16* K, const hcadsa_bf16* V,
                                  const int32_t* idx, const hcadsa_bf16* O, const hcadsa_bf16* dO, const float* lse,
                                  float* dQ, float* dK, float* dV, int B, int Lq, int Lk, int Hq, int d, int k,
                                  float scale, hcadsa_stream stream);

/*
 * Size in bytes of the workspace hca_attn_bwd needs: one fp32 per query row (D = <dO, O>) and
 * the bf16 probability and score-gradient blocks of every (row tile, key tile) pair,
 *     B*Lq*Hq*4 (rounded up to 256) + 2 * B*Hkv*n_rt*J * 128*128*2 bytes,
 * n_rt = ceil(Lq / (128/(Hq/Hkv))) row tiles, J = ceil(n_c(t_last)/128) +
 * ceil((128/(Hq/Hkv) + W - 1)/128) + 1 key tiles per row tile.  0 for unsupported sizes.
 */
size_t hca_attn_bwd_workspace_size(int B, int Lq, int q_offset, int Hq, int Hkv, int d, int n_c, int blk, int W);

/*
 * Backward of HCA attention.  Source: the forward above (the mirrorspeed page, section "Hybrid
 * sparse attention, 1/7 full context access": one softmax over a query's visible compressed
 * entries and raw window positions; 512-wide heads).  For output gradient dO, with the
 * forward's probabilities p_s = exp(scale <q, k_s> - lse) over the visible set (same reading
 * of the visible set as hca_attn_fwd):
 *     D = <dO, O>,  dS_s = p_s (<dO, v_s> - D)
 *     dQ  = scale sum_s dS_s k_s                                    (written)
 *     dK_s += scale sum_rows dS_s q,  dV_s += sum_rows p_s dO       (ADDED to; entries s go to
 *                                                                    dKc/dVc, window rows to dKw/dVw)
 * P and dS enter the tensor cores as bf16; accumulation is fp32.  Several units add to the same
 * dK / dV rows with fp32 reductions in no fixed order (last-bit differences between runs).
 * The entry gradients dKc / dVc feed hca_compress_bwd to reach the raw keys and the weights.
 *
 *   Q, O, dO : [B, Lq, Hq, d] bf16 (O and lse from hca_attn_fwd)
 *   Kc, Vc   : [B, n_c, Hkv, d] bf16 (NULL allowed iff n_c == 0), Kw, Vw: [B, n_w, Hkv, d] bf16
 *   lse      : [B, Lq, Hq] fp32
 *   dQ       : [B, Lq, Hq, d] fp32 (written)
 *   dKc, dVc : [B, n_c, Hkv, d] fp32, dKw, dVw: [B, n_w, Hkv, d] fp32 (accumulated)
 *   workspace: hca_attn_bwd_workspace_size(...) bytes, 16-byte aligned
 * Requirements as hca_attn_fwd (d == 512, (Hq/Hkv) divides 128, windows inside the raw buffer,
 * n_c(t) <= n_c): HCADSA_ERR_SHAPE / _UNSUPPORTED / _WORKSPACE / _ALIGN otherwise.
 */
hcadsa_status hca_attn_bwd(const hcadsa_bf16* Q, const hcadsa_bf16* Kc, const hcadsa_bf16* Vc, int n_c,
                           const hcadsa_bf16* Kw, const hcadsa_bf16* Vw, int win_start, int n_w,
                           const hcadsa_bf16* O, const hcadsa_bf16* dO, const float* lse, float* dQ, float* dKc,
                           float* dVc, float* dKw, float* dVw, int B, int Lq, int q_offset, int Hq, int Hkv, int d,
                           int blk, int W, float scale, void* workspace, size_t workspace_bytes,
                           hcadsa_stream stream);

#ifdef __cplusplus
}
#endif

#endif /* HCADSA_H_ */
