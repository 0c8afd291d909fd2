// compress_bwd.cu -- backward of the HCA block compressor (the adjoint of a linear map).
//
// The compressor of the mirrorspeed page's section "Hybrid sparse attention, 1/7 full context
// access" (every 128 tokens become one cache entry) is, in this library's form, the linear map
//     Xc[b, j, h, c] = sum_i w[i] * X[b, blk*j + i, h, c]          (i < blk, complete blocks)
// so a loss with gradient dXc on the entries has
//     dX[b, blk*j + i, h, c] = w[i] * dXc[b, j, h, c]              (tail tokens get nothing)
//     dw[i]                  = sum_{b,j,h,c} dXc[b, j, h, c] * X[b, blk*j + i, h, c]
// (the bf16 rounding of the forward is not differentiated).  Both outputs are accumulated into
// (dX += ..., dw += ...), so a caller can add the compressor's share of a key/value gradient to
// the share the attention already wrote for the raw window.
//
// The work is an HBM stream: per raw element one bf16 read of X, one fp32 read-modify-write of
// dX, per entry element one fp32 read of dXc.  A CTA takes kRows consecutive rows of one block
// (grid = blocks x row groups x batches, thousands of CTAs); thread t owns channel pairs of the
// H*d row, reads dXc of its channels once and walks the CTA's rows; the dw partial sums of each
// row are reduced across the CTA in shared memory and added to dw once per CTA and row.
#include <cuda_runtime.h>

#include "host_common.h"
#include "ptx.cuh"

namespace hcadsa {
namespace {

constexpr int kThreads = 256;
constexpr int kRows = 8;

__global__ void __launch_bounds__(kThreads) compress_bwd_kernel(const uint16_t* __restrict__ X,
                                                                const float* __restrict__ w,
                                                                const float* __restrict__ dXc,
                                                                float* __restrict__ dX, float* __restrict__ dw,
                                                                int L, int row_elems, int n_c, int blk,
                                                                int groups) {
  __shared__ float s_part[kThreads / 32][kRows];
  const int b = blockIdx.y;
  const int j = blockIdx.x / groups;
  const int i0 = (blockIdx.x % groups) * kRows;
  const int nr = min(kRows, blk - i0);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const float* g = dXc + ((size_t)b * n_c + j) * row_elems;
  float wi[kRows], part[kRows];
#pragma unroll
  for (int i = 0; i < kRows; ++i) {
    wi[i] = i < nr ? w[i0 + i] : 0.0f;
    part[i] = 0.0f;
  }
  const size_t row0 = (size_t)b * L + (size_t)j * blk + i0;
  for (int c2 = threadIdx.x; c2 < row_elems / 2; c2 += kThreads) {
    const float2 gc = reinterpret_cast<const float2*>(g)[c2];
#pragma unroll
    for (int i = 0; i < kRows; ++i) {
      if (i < nr) {
        const uint32_t xv = reinterpret_cast<const uint32_t*>(X + (row0 + i) * row_elems)[c2];
        float2* d2 = reinterpret_cast<float2*>(dX + (row0 + i) * row_elems) + c2;
        float2 dv = *d2;
        dv.x = fmaf(wi[i], gc.x, dv.x);
        dv.y = fmaf(wi[i], gc.y, dv.y);
        *d2 = dv;
        part[i] = fmaf(gc.x, __uint_as_float(xv << 16), part[i]);
        part[i] = fmaf(gc.y, __uint_as_float(xv & 0xFFFF0000u), part[i]);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < kRows; ++i) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) part[i] += __shfl_xor_sync(0xffffffffu, part[i], o);
    if (lane == 0) s_part[warp][i] = part[i];
  }
  __syncthreads();
  if (threadIdx.x < nr) {
    float acc = 0.0f;
    for (int q = 0; q < kThreads / 32; ++q) acc += s_part[q][threadIdx.x];
    atomicAdd(&dw[i0 + threadIdx.x], acc);
  }
}

}  // namespace
}  // namespace hcadsa

extern "C" hcadsa_status hca_compress_bwd(const hcadsa_bf16* X, const float* w, const float* dXc, float* dX,
                                          float* dw, int B, int L, int H, int d, int blk, hcadsa_stream stream) {
  using namespace hcadsa;
  if (!X || !w || !dXc || !dX || !dw) return HCADSA_ERR_NULL;
  if (B < 0 || L < 0 || H <= 0 || d <= 0 || blk <= 0) return HCADSA_ERR_SHAPE;
  if (blk > 1024 || d % 8 != 0) return HCADSA_ERR_UNSUPPORTED;
  if (!aligned16(X) || !aligned16(dXc) || !aligned16(dX) || (reinterpret_cast<uintptr_t>(w) & 3u) ||
      (reinterpret_cast<uintptr_t>(dw) & 3u))
    return HCADSA_ERR_ALIGN;
  const int n_c = L / blk;
  if (B == 0 || n_c == 0) return HCADSA_OK;
  const long long row_elems = (long long)H * d;
  if (row_elems > (1LL << 24) || (long long)B * L * row_elems > (1LL << 40) || B > 65535)
    return HCADSA_ERR_UNSUPPORTED;
  const int groups = (blk + kRows - 1) / kRows;
  if ((long long)n_c * groups > 0x7fffffffLL) return HCADSA_ERR_UNSUPPORTED;
  const dim3 grid((unsigned)(n_c * groups), (unsigned)B);
  compress_bwd_kernel<<<grid, kThreads, 0, as_stream(stream)>>>(reinterpret_cast<const uint16_t*>(X), w, dXc, dX,
                                                                 dw, L, (int)row_elems, n_c, blk, groups);
  return launch_status();
}
