// hca_compress.cu -- HCA block compression: every blk consecutive tokens of K and V
// become one cache entry, entry = bf16(sum_i w[i] * x[blk*j + i]) with an fp32
// fused-multiply-add chain in ascending i (the compressor form this library fixes;
// the pages -- "Hybrid sparse attention, 1/7 full context access" on the mirrorspeed
// page -- only say that 128 tokens become one entry).
//
// The work is a pure HBM stream: each thread owns 8 adjacent channels of one block
// and walks its blk rows in order, so one warp reads 512 contiguous bytes per row
// and the FMA order per channel is exactly the sequential chain.  Loads for 16 rows
// are issued before their FMAs to keep enough bytes in flight per SM.
#include <cuda_bf16.h>

#include "host_common.h"
#include "ptx.cuh"

namespace hcadsa {
namespace {

constexpr int kMaxThreads = 128;
constexpr int kRowsInFlight = 16;

__device__ __forceinline__ float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }

__device__ __forceinline__ uint4 ld_stream(const uint4* p) { return __ldg(p); }

// grid: x = B * n_c blocks, y = column groups of blockDim.x*8 channels, z = 2 (K, V)
__global__ void __launch_bounds__(kMaxThreads) hca_compress_kernel(const uint16_t* __restrict__ K,
                                                                const uint16_t* __restrict__ V,
                                                                const float* __restrict__ w,
                                                                uint16_t* __restrict__ Kc,
                                                                uint16_t* __restrict__ Vc, int L, int row_elems,
                                                                int n_c, int blk) {
  __shared__ float sw[1024];
  for (int i = threadIdx.x; i < blk; i += blockDim.x) sw[i] = w[i];
  __syncthreads();

  const int col = (blockIdx.y * blockDim.x + threadIdx.x) * 8;
  if (col >= row_elems) return;
  const int b = blockIdx.x / n_c, j = blockIdx.x % n_c;
  const uint16_t* src = (blockIdx.z == 0 ? K : V) + ((size_t)b * L + (size_t)blk * j) * row_elems + col;
  uint16_t* dst = (blockIdx.z == 0 ? Kc : Vc) + ((size_t)b * n_c + j) * row_elems + col;

  float acc[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) acc[c] = 0.0f;

  int i = 0;
  for (; i + kRowsInFlight <= blk; i += kRowsInFlight) {
    uint4 x[kRowsInFlight];
#pragma unroll
    for (int u = 0; u < kRowsInFlight; ++u)
      x[u] = ld_stream(reinterpret_cast<const uint4*>(src + (size_t)(i + u) * row_elems));
#pragma unroll
    for (int u = 0; u < kRowsInFlight; ++u) {
      const float wi = sw[i + u];
      acc[0] = fmaf(wi, bf16_lo(x[u].x), acc[0]);
      acc[1] = fmaf(wi, bf16_hi(x[u].x), acc[1]);
      acc[2] = fmaf(wi, bf16_lo(x[u].y), acc[2]);
      acc[3] = fmaf(wi, bf16_hi(x[u].y), acc[3]);
      acc[4] = fmaf(wi, bf16_lo(x[u].z), acc[4]);
      acc[5] = fmaf(wi, bf16_hi(x[u].z), acc[5]);
      acc[6] = fmaf(wi, bf16_lo(x[u].w), acc[6]);
      acc[7] = fmaf(wi, bf16_hi(x[u].w), acc[7]);
    }
  }
  for (; i < blk; ++i) {
    const uint4 x = ld_stream(reinterpret_cast<const uint4*>(src + (size_t)i * row_elems));
    const float wi = sw[i];
    acc[0] = fmaf(wi, bf16_lo(x.x), acc[0]);
    acc[1] = fmaf(wi, bf16_hi(x.x), acc[1]);
    acc[2] = fmaf(wi, bf16_lo(x.y), acc[2]);
    acc[3] = fmaf(wi, bf16_hi(x.y), acc[3]);
    acc[4] = fmaf(wi, bf16_lo(x.z), acc[4]);
    acc[5] = fmaf(wi, bf16_hi(x.z), acc[5]);
    acc[6] = fmaf(wi, bf16_lo(x.w), acc[6]);
    acc[7] = fmaf(wi, bf16_hi(x.w), acc[7]);
  }
  uint4 out;
  out.x = pack_bf16x2(acc[0], acc[1]);
  out.y = pack_bf16x2(acc[2], acc[3]);
  out.z = pack_bf16x2(acc[4], acc[5]);
  out.w = pack_bf16x2(acc[6], acc[7]);
  *reinterpret_cast<uint4*>(dst) = out;
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
  if ((long long)B * n_c > 2147483647LL || row_elems > (1LL << 30)) return HCADSA_ERR_UNSUPPORTED;
  const long long groups8 = row_elems / 8;
  const int threads = (int)(groups8 >= kMaxThreads ? kMaxThreads : ((groups8 + 31) / 32) * 32);
  const long long col_blocks = (groups8 + threads - 1) / threads;
  if (col_blocks > 65535) return HCADSA_ERR_UNSUPPORTED;
  dim3 grid((unsigned)(B * n_c), (unsigned)col_blocks, 2);
  hca_compress_kernel<<<grid, threads, 0, as_stream(stream)>>>(K, V, w, Kc, Vc, L, (int)row_elems, n_c, blk);
  return launch_status();
}
