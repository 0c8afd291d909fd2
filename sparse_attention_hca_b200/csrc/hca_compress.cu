// hca_compress.cu -- HCA block compression: every blk consecutive tokens of K and V
// become one cache entry, entry = bf16(sum_i w[i] * x[blk*j + i]) with an fp32
// fused-multiply-add chain in ascending i (the compressor form this library fixes;
// the pages -- "Hybrid sparse attention, 1/7 full context access" on the mirrorspeed
// page -- only say that 128 tokens become one entry).
//
// The work is a pure HBM stream.  Persistent CTAs walk work units (tensor, batch, block,
// 256-channel column group; for blocks shorter than 128 tokens a unit takes 128 / blk
// consecutive blocks, so a box is never mostly unused).  One thread streams each unit's rows into a 3-stage ring of
// shared-memory boxes (TMA, up to 128 rows x 256 channels = 64 KB per box) so plenty of
// bytes are in flight per SM; four warps then run the sequential FMA chains from shared
// memory, two channels per thread, rows in ascending order -- exactly the fixed
// accumulation order, so results are bit-identical to a plain loop.
#include <cuda_bf16.h>

#include <mutex>

#include "host_common.h"
#include "ptx.cuh"

namespace hcadsa {
namespace {

constexpr int kCols = 256;            // channels per work unit (TMA box width)
constexpr int kBoxRows = 128;         // rows per TMA box
constexpr int kStages = 3;
constexpr int kBoxBytes = kCols * kBoxRows * 2;  // 64 KB
constexpr int kConsumerWarps = 4;     // 128 threads x 2 channels = 256 channels
constexpr int kThreads = 32 * (kConsumerWarps + 1);
constexpr int kSmemBytes = kStages * kBoxBytes + 128;

struct Params {
  const float* w;
  uint16_t* Kc;
  uint16_t* Vc;
  int* err;
  int B, L, row_elems, n_c, blk, col_groups, n_units;
  int bpu;       // blocks per unit: 128 / blk consecutive blocks share one 128-row box when blk < 128
  int n_groups;  // block groups per batch: ceil(n_c / bpu)
};

__global__ void __launch_bounds__(kThreads, 1)
    hca_compress_kernel(const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v,
                        const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  __shared__ uint64_t full[kStages], empty[kStages];
  __shared__ float sw[1024];
  __shared__ int abort_flag;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  for (int i = threadIdx.x; i < p.blk; i += kThreads) sw[i] = p.w[i];
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumerWarps * 32);
    }
    abort_flag = 0;
    fence_mbarrier_init();
  }
  __syncthreads();
  const int boxes_per_unit = (p.blk + kBoxRows - 1) / kBoxRows;

  if (warp == kConsumerWarps) {
    // ------------------------------------------------------------ producer (one thread)
    if (lane == 0) {
      uint32_t q = 0;  // boxes issued: stage q % kStages, phase (q / kStages) & 1
      for (int u = blockIdx.x; u < p.n_units; u += gridDim.x) {
        const int cg = u % p.col_groups;
        const int rest = u / p.col_groups;
        const int tensor = rest & 1;
        const int bg = rest >> 1;  // b * n_groups + block group
        const int b = bg / p.n_groups, j = (bg % p.n_groups) * p.bpu;  // first block of the unit
        const int row0 = b * p.L + j * p.blk;
        for (int bx = 0; bx < boxes_per_unit; ++bx, ++q) {
          const uint32_t st = q % kStages;
          if (!mbar_wait(&empty[st], ((q / kStages) & 1) ^ 1, &abort_flag, p.err)) return;
          mbar_arrive_expect_tx(&full[st], kBoxBytes);
          tma_load_2d(ring + st * kBoxBytes, tensor ? &map_v : &map_k, &full[st], cg * kCols, row0 + bx * kBoxRows);
        }
      }
    }
    return;
  }

  // -------------------------------------------------------------- consumers: FMA chains
  const int col = threadIdx.x * 2;  // 2 channels of the unit's 256
  uint32_t q = 0;
  for (int u = blockIdx.x; u < p.n_units; u += gridDim.x) {
    const int cg = u % p.col_groups;
    const int rest = u / p.col_groups;
    const int tensor = rest & 1;
    const int bg = rest >> 1;
    const int b = bg / p.n_groups, j0 = (bg % p.n_groups) * p.bpu;
    const int gcol = cg * kCols + col;
    uint16_t* dst_base = (tensor ? p.Vc : p.Kc) + (size_t)b * p.n_c * p.row_elems + gcol;
    if (p.bpu > 1) {
      // one box holds bpu whole blocks: each block's chain over its blk rows, in order
      const uint32_t st = q % kStages;
      if (!mbar_wait(&full[st], (q / kStages) & 1, &abort_flag, p.err)) return;
      const uint32_t* box = reinterpret_cast<const uint32_t*>(ring + st * kBoxBytes) + threadIdx.x;
      const int nb = min(p.bpu, p.n_c - j0);
      for (int jj = 0; jj < nb; ++jj) {
        float a0 = 0.0f, a1 = 0.0f;
        const uint32_t* rows = box + jj * p.blk * (kCols / 2);
        for (int i = 0; i < p.blk; ++i) {
          const uint32_t x = rows[i * (kCols / 2)];
          a0 = fmaf(sw[i], __uint_as_float(x << 16), a0);
          a1 = fmaf(sw[i], __uint_as_float(x & 0xFFFF0000u), a1);
        }
        if (gcol < p.row_elems)
          *reinterpret_cast<uint32_t*>(dst_base + (size_t)(j0 + jj) * p.row_elems) = pack_bf16x2(a0, a1);
      }
      mbar_arrive(&empty[st]);
      ++q;
      continue;
    }
    float a0 = 0.0f, a1 = 0.0f;
    for (int bx = 0; bx < boxes_per_unit; ++bx, ++q) {
      const uint32_t st = q % kStages;
      if (!mbar_wait(&full[st], (q / kStages) & 1, &abort_flag, p.err)) return;
      const uint32_t* box = reinterpret_cast<const uint32_t*>(ring + st * kBoxBytes) + threadIdx.x;
      const int rows = min(kBoxRows, p.blk - bx * kBoxRows);
      const float* wr = sw + bx * kBoxRows;
#pragma unroll 8
      for (int i = 0; i < rows; ++i) {
        const uint32_t x = box[i * (kCols / 2)];
        a0 = fmaf(wr[i], __uint_as_float(x << 16), a0);
        a1 = fmaf(wr[i], __uint_as_float(x & 0xFFFF0000u), a1);
      }
      mbar_arrive(&empty[st]);
    }
    if (gcol < p.row_elems) *reinterpret_cast<uint32_t*>(dst_base + (size_t)j0 * p.row_elems) = pack_bf16x2(a0, a1);
  }
}

int num_sms() {
  static std::mutex mu;
  static int cache[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  std::lock_guard<std::mutex> lock(mu);
  if (!cache[dev] && cudaDeviceGetAttribute(&cache[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return 0;
  return cache[dev];
}

}  // namespace
}  // namespace hcadsa

extern "C" hcadsa_status hca_compress_kv(const hcadsa_bf16* K, const hcadsa_bf16* V, const float* w,
                                         hcadsa_bf16* Kc, hcadsa_bf16* Vc, int B, int L, int Hkv, int d, int blk,
                                         hcadsa_stream stream) {
  using namespace hcadsa;
  if (!K || !V || !w || !Kc || !Vc) return HCADSA_ERR_NULL;
  if (B < 0 || L < 0 || Hkv <= 0 || d <= 0 || blk <= 0) return HCADSA_ERR_SHAPE;
  if (blk > 1024 || d % 8 != 0) return HCADSA_ERR_UNSUPPORTED;
  if (!aligned16(K) || !aligned16(V) || !aligned16(Kc) || !aligned16(Vc) || !aligned16(w))
    return HCADSA_ERR_ALIGN;
  const int n_c = L / blk;
  if (B == 0 || n_c == 0) return HCADSA_OK;
  const long long row_elems = (long long)Hkv * d;
  const long long rows = (long long)B * L;
  if (row_elems > (1LL << 24) || rows > 2147483647LL) return HCADSA_ERR_UNSUPPORTED;
  const long long col_groups = (row_elems + kCols - 1) / kCols;
  // short blocks (blk < 128) are batched: 128 / blk consecutive blocks per 128-row box
  const int bpu = blk < kBoxRows ? kBoxRows / blk : 1;
  const long long n_groups = (n_c + bpu - 1) / bpu;
  const long long n_units = 2LL * B * n_groups * col_groups;
  if (n_units > 2147483647LL) return HCADSA_ERR_UNSUPPORTED;
  // [rows, row_elems] bf16, box = 128 rows x 256 channels, no swizzle; box parts past the last
  // row or the last channel are zero-filled and never stored
  CUtensorMap mk, mv;
  const uint64_t dims[2] = {(uint64_t)row_elems, (uint64_t)rows};
  const uint64_t strides[1] = {(uint64_t)row_elems * 2};
  const uint32_t box[2] = {(uint32_t)kCols, (uint32_t)kBoxRows};
  if (!encode_tmap_bf16(&mk, 2, const_cast<hcadsa_bf16*>(K), dims, strides, box, false)) return HCADSA_ERR_CUDA;
  if (!encode_tmap_bf16(&mv, 2, const_cast<hcadsa_bf16*>(V), dims, strides, box, false)) return HCADSA_ERR_CUDA;
  Params p;
  p.w = w;
  p.Kc = Kc;
  p.Vc = Vc;
  p.err = device_error_ptr();
  p.B = B;
  p.L = L;
  p.row_elems = (int)row_elems;
  p.n_c = n_c;
  p.blk = blk;
  p.col_groups = (int)col_groups;
  p.n_units = (int)n_units;
  p.bpu = bpu;
  p.n_groups = (int)n_groups;
  if (cudaFuncSetAttribute(hca_compress_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) !=
      cudaSuccess)
    return HCADSA_ERR_CUDA;
  const int sms = num_sms();
  if (sms <= 0) return HCADSA_ERR_CUDA;
  const int grid = (int)(n_units < sms ? n_units : sms);
  hca_compress_kernel<<<grid, kThreads, kSmemBytes, as_stream(stream)>>>(mk, mv, p);
  return launch_status();
}
