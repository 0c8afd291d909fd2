// capi.cu -- library-wide C entry points (version, status strings, device error word)
// and the host helpers the launchers share (TMA tensor-map encoding).
#include <cudaTypedefs.h>

#include <cstdio>
#include <mutex>

#include "host_common.h"
#include "ptx.cuh"

namespace hcadsa {
namespace {

// One error word per device, in the module's global memory.  Kernels receive its
// address; the host reads and clears it in hcadsa_check_device_error.
__device__ int g_error_word = 0;

constexpr int kMaxDevices = 64;
int* g_error_ptr[kMaxDevices] = {};
std::mutex g_mu;

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

}  // namespace

int* device_error_ptr() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_error_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_error_word) != cudaSuccess) return nullptr;
    g_error_ptr[dev] = static_cast<int*>(p);
  }
  return g_error_ptr[dev];
}

bool encode_tmap_bf16_swizzle(CUtensorMap* map, int rank, void* base, const uint64_t* dims,
                              const uint64_t* strides_bytes, const uint32_t* box, int swizzle_bytes) {
  return encode_tmap_typed(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, base, dims, strides_bytes, box,
                           swizzle_bytes);
}

bool encode_tmap_u8_swizzle(CUtensorMap* map, int rank, void* base, const uint64_t* dims,
                            const uint64_t* strides_bytes, const uint32_t* box, int swizzle_bytes) {
  return encode_tmap_typed(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, rank, base, dims, strides_bytes, box,
                           swizzle_bytes);
}

bool encode_tmap_typed(CUtensorMap* map, CUtensorMapDataType dtype, int rank, void* base, const uint64_t* dims,
                       const uint64_t* strides_bytes, const uint32_t* box, int swizzle_bytes) {
  CUtensorMapSwizzle sw;
  switch (swizzle_bytes) {
    case 0: sw = CU_TENSOR_MAP_SWIZZLE_NONE; break;
    case 32: sw = CU_TENSOR_MAP_SWIZZLE_32B; break;
    case 64: sw = CU_TENSOR_MAP_SWIZZLE_64B; break;
    case 128: sw = CU_TENSOR_MAP_SWIZZLE_128B; break;
    default: return false;
  }
  if (rank < 1 || rank > 5) return false;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_encode) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
          q != cudaDriverEntryPointSuccess || !fn)
        return false;
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
  }
  cuuint64_t d[5];
  cuuint64_t st[4];
  cuuint32_t bx[5], es[5];
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    bx[i] = box[i];
    es[i] = 1;
    if (i + 1 < rank) st[i] = strides_bytes[i];
  }
  const CUresult r = g_encode(map, dtype, (cuuint32_t)rank, base, d, st, bx, es,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool encode_tmap_bf16(CUtensorMap* map, int rank, void* base, const uint64_t* dims, const uint64_t* strides_bytes,
                      const uint32_t* box, bool swizzle128) {
  return encode_tmap_bf16_swizzle(map, rank, base, dims, strides_bytes, box, swizzle128 ? 128 : 0);
}

thread_local char t_last_error[256] = "";

// Waits on an mbarrier that nothing ever arrives on, with a short limit: exercises the bounded
// wait every kernel uses, which must give up, record HCADSA_ERR_TIMEOUT and return.
__global__ void bounded_wait_selftest_kernel(int* err, unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbarrier_init();
  }
  __syncthreads();
  mbar_wait_for(&bar, 0, &abort_flag, err, limit_ns);
}

void record_cuda_error(cudaError_t e) {
  snprintf(t_last_error, sizeof(t_last_error), "%s: %s", cudaGetErrorName(e), cudaGetErrorString(e));
}

}  // namespace hcadsa

extern "C" const char* hcadsa_last_error_string(void) { return hcadsa::t_last_error; }

extern "C" hcadsa_status hcadsa_selftest_bounded_wait(unsigned timeout_us, hcadsa_stream stream) {
  using namespace hcadsa;
  if (timeout_us == 0 || timeout_us > 10000000u) return HCADSA_ERR_SHAPE;
  int* err = device_error_ptr();
  if (!err) return HCADSA_ERR_CUDA;
  bounded_wait_selftest_kernel<<<1, 32, 0, as_stream(stream)>>>(err, 1000ull * timeout_us);
  return launch_status();
}

extern "C" int hcadsa_version(void) { return 100; }

extern "C" const char* hcadsa_status_string(hcadsa_status status) {
  switch (status) {
    case HCADSA_OK: return "HCADSA_OK";
    case HCADSA_ERR_NULL: return "HCADSA_ERR_NULL: a required pointer is NULL";
    case HCADSA_ERR_SHAPE: return "HCADSA_ERR_SHAPE: inconsistent sizes";
    case HCADSA_ERR_ALIGN: return "HCADSA_ERR_ALIGN: pointer not 16-byte aligned";
    case HCADSA_ERR_UNSUPPORTED: return "HCADSA_ERR_UNSUPPORTED: sizes not supported by this build";
    case HCADSA_ERR_WORKSPACE: return "HCADSA_ERR_WORKSPACE: workspace missing or too small";
    case HCADSA_ERR_CUDA: return "HCADSA_ERR_CUDA: a CUDA call failed";
    case HCADSA_ERR_TIMEOUT: return "HCADSA_ERR_TIMEOUT: a device-side bounded wait expired";
    case HCADSA_ERR_DEVICE_BOUNDS: return "HCADSA_ERR_DEVICE_BOUNDS: an index input was out of range";
  }
  return "HCADSA: unknown status";
}

extern "C" hcadsa_status hcadsa_check_device_error(hcadsa_stream stream) {
  using namespace hcadsa;
  const cudaError_t se = cudaStreamSynchronize(as_stream(stream));
  if (se != cudaSuccess) {
    record_cuda_error(se);
    return HCADSA_ERR_CUDA;
  }
  int* p = device_error_ptr();
  if (!p) return HCADSA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, p, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return HCADSA_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpy(p, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return HCADSA_ERR_CUDA;
  }
  return static_cast<hcadsa_status>(v);
}
