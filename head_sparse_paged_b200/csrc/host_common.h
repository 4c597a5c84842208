// host_common.h -- host-side helpers shared by the library's entry points: device attributes, TMA
// tensor-map encoding and the argument checks every call makes.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cstdint>
#include <mutex>

#include "../../include/segpaged.h"

namespace segpaged {
namespace host {

constexpr int kMaxDevices = 64;

// SM count of a device, looked up once per device (atomics: entry points may be called from several host
// threads; a race only repeats the lookup).
inline int device_sm_count(int dev) {
  static std::atomic<int> cache[kMaxDevices];
  if (dev < 0 || dev >= kMaxDevices) return 0;
  int n = cache[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    cache[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

inline PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

// 3-D bf16 tensor map, innermost dimension first, 128-byte swizzle.
inline bool encode_3d(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t b0, uint32_t b1,
               uint32_t b2) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};
  cuuint32_t box[3] = {b0, b1, b2};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline int check_dims(const segpaged_dims* d) {
  if (!d) return SEGPAGED_ERR_NULL;
  if (d->num_seqs < 0 || d->num_kv_heads < 1 || d->num_q_heads < 1 || d->num_q_heads % d->num_kv_heads != 0)
    return SEGPAGED_ERR_DIMS;
  const int G = d->num_q_heads / d->num_kv_heads;
  if (G > 128 || (G & (G - 1)) != 0) return SEGPAGED_ERR_DIMS;
  if (d->head_dim != 64 && d->head_dim != 128) return SEGPAGED_ERR_DIMS;
  if (d->page_size != 16 && d->page_size != 32 && d->page_size != 64 && d->page_size != 128) return SEGPAGED_ERR_DIMS;
  if (d->num_pages < 0) return SEGPAGED_ERR_DIMS;
  return SEGPAGED_OK;
}

inline int check_class(const segpaged_head_class& c) {
  if (c.is_global) return SEGPAGED_OK;
  if (c.sink < 0 || c.window < 1) return SEGPAGED_ERR_CLASS;
  return SEGPAGED_OK;
}

inline int log2_int(int x) {
  int r = 0;
  while ((1 << r) < x) ++r;
  return r;
}

}  // namespace host
}  // namespace segpaged
