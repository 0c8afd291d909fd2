// host_common.h -- host-side helpers shared by the launchers: status mapping,
// argument checks, TMA tensor-map encoding, the per-device error word.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/hcadsa.h"

namespace hcadsa {

// Address of the device error word for the current device (set up on first use).
// Returns nullptr if the CUDA runtime call failed.
int* device_error_ptr();

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline cudaStream_t as_stream(hcadsa_stream s) { return reinterpret_cast<cudaStream_t>(s); }

// Encodes a tiled bf16 tensor map with 128-byte swizzle over a tensor of rank `rank`
// (dims[0] innermost, element counts; strides_bytes[i] = byte stride of dim i+1).
// Returns false if the driver rejects it.
bool encode_tmap_bf16(CUtensorMap* map, int rank, void* base, const uint64_t* dims,
                      const uint64_t* strides_bytes, const uint32_t* box, bool swizzle128);

// Same, with the swizzle span given in bytes: 0 (none), 32, 64 or 128.
bool encode_tmap_bf16_swizzle(CUtensorMap* map, int rank, void* base, const uint64_t* dims,
                              const uint64_t* strides_bytes, const uint32_t* box, int swizzle_bytes);

// Same for 8-bit integer tensors (element = 1 byte), and for any driver data type.
bool encode_tmap_u8_swizzle(CUtensorMap* map, int rank, void* base, const uint64_t* dims,
                            const uint64_t* strides_bytes, const uint32_t* box, int swizzle_bytes);
bool encode_tmap_typed(CUtensorMap* map, CUtensorMapDataType dtype, int rank, void* base, const uint64_t* dims,
                       const uint64_t* strides_bytes, const uint32_t* box, int swizzle_bytes);

// Indexer + exact top-k of many query rows in one fused kernel (dsa_topk_tc.cu): scores on the
// int8 tensor cores, selection by per-row histograms, no score matrix.  Candidates of the query
// at position t are the keys s < min((t + 1) / ratio, Lk).  `kstat` is workspace for
// topk_fused_workspace_bytes(B) bytes.  Enqueues on `s`; returns a status before launch.
size_t topk_fused_workspace_bytes(int B);
hcadsa_status launch_topk_fused(const int8_t* q_idx, const int8_t* k_idx, const int32_t* w_idx, int32_t* idx,
                                void* kstat, int B, int Lq, int q_offset, int Lk, int k, int ratio,
                                cudaStream_t s);

// Records the message of a failed CUDA call for hcadsa_last_error_string().
void record_cuda_error(cudaError_t e);

inline hcadsa_status launch_status() {
  const cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) return HCADSA_OK;
  record_cuda_error(e);
  return HCADSA_ERR_CUDA;
}

}  // namespace hcadsa
