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
// dX, per entry element one fp32 read of dXc.  A CTA takes a run of consecutive blocks of one
// batch; thread t owns channel pairs of the H*d row, walks the block's rows in order and keeps
// dXc of its channels in registers; the dw partial sums of a row are reduced across the CTA in
// shared memory (one float per block position) and added to dw once per CTA.
#include <cuda_runtime.h>

#include <mutex>

#include "host_common.h"
#include "ptx.cuh"

namespace hcadsa {
namespace {

constexpr int kThreads = 256;
constexpr int kBlocksPerCta = 4;

__global__ void __launch_bounds__(kThreads) compress_bwd_kernel(const uint16_t* __restrict__ X,
                                                                const float* __restrict__ w,
                                                                const float* __restrict__ dXc,
                                                                float* __restrict__ dX, float* __restrict__ dw,
                                                                int L, int row_elems, int n_c, int blk) {
  extern __shared__ float s_dw[];  // [blk] partial sums of this CTA
  for (int i = threadIdx.x; i < blk; i += kThreads) s_dw[i] = 0.0f;
  __syncthreads();
  const int b = blockIdx.y;
  const int j0 = blockIdx.x * kBlocksPerCta;
  const int lane = threadIdx.x & 31;
  for (int j = j0; j < min(j0 + kBlocksPerCta, n_c); ++j) {
    const float* g = dXc + ((size_t)b * n_c + j) * row_elems;
    for (int i = 0; i < blk; ++i) {
      const size_t row = (size_t)b * L + (size_t)j * blk + i;
      const uint32_t* x2 = reinterpret_cast<const uint32_t*>(X + row * row_elems);
      float2* d2 = reinterpret_cast<float2*>(dX + row * row_elems);
      const float wi = w[i];
      float part = 0.0f;
      for (int c2 = threadIdx.x; c2 < row_elems / 2; c2 += kThreads) {
        const float2 gc = reinterpret_cast<const float2*>(g)[c2];
        const uint32_t xv = x2[c2];
        float2 dv = d2[c2];
        dv.x = fmaf(wi, gc.x, dv.x);
        dv.y = fmaf(wi, gc.y, dv.y);
        d2[c2] = dv;
        part = fmaf(gc.x, __uint_as_float(xv << 16), part);
        part = fmaf(gc.y, __uint_as_float(xv & 0xFFFF0000u), part);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
      if (lane == 0) atomicAdd(&s_dw[i], part);
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < blk; i += kThreads) atomicAdd(&dw[i], s_dw[i]);
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
  const dim3 grid((unsigned)((n_c + kBlocksPerCta - 1) / kBlocksPerCta), (unsigned)B);
  compress_bwd_kernel<<<grid, kThreads, (size_t)blk * sizeof(float), as_stream(stream)>>>(
      reinterpret_cast<const uint16_t*>(X), w, dXc, dX, dw, L, (int)row_elems, n_c, blk);
  return launch_status();
}
