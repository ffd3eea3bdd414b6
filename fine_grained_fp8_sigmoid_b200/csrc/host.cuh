// Host-side helpers: status mapping, device properties, TMA descriptors.
#pragma once

#include <cudaTypedefs.h>
#include <cstdio>
#include <mutex>

#include "common.cuh"

namespace moe {

#define MOE_CHECK_ARG(cond)                 \
  do {                                      \
    if (!(cond)) return MOE_ERR_INVALID_ARG; \
  } while (0)

#define MOE_CHECK_SUPPORTED(cond)           \
  do {                                      \
    if (!(cond)) return MOE_ERR_UNSUPPORTED; \
  } while (0)

// Text of the last host-side failure in this thread (moe_last_error_detail).
inline char* last_error_buf() {
  static thread_local char buf[256] = {0};
  return buf;
}

inline int record_failure(int status, const char* where, const char* what) {
  snprintf(last_error_buf(), 256, "%s: %s", where, what);
  return status;
}

inline int cuda_status(cudaError_t e, const char* where) {
  if (e == cudaSuccess) return MOE_OK;
  return record_failure(MOE_ERR_CUDA, where, cudaGetErrorString(e));
}

inline int launch_status(const char* where = "kernel launch") {
  return cuda_status(cudaGetLastError(), where);
}

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

struct DeviceInfo {
  int sm_count = 0;
  int major = 0;
};

// SM count and compute capability of the current device (cached per device).
inline int device_info(DeviceInfo* out) {
  static std::mutex mu;
  static DeviceInfo cache[64];
  static bool have[64] = {false};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MOE_ERR_NO_DEVICE;
  std::lock_guard<std::mutex> lock(mu);
  if (!have[dev]) {
    cudaDeviceProp p;
    if (cudaGetDeviceProperties(&p, dev) != cudaSuccess) return MOE_ERR_NO_DEVICE;
    cache[dev].sm_count = p.multiProcessorCount;
    cache[dev].major = p.major;
    have[dev] = true;
  }
  *out = cache[dev];
  return cache[dev].major == 10 ? MOE_OK : MOE_ERR_NO_DEVICE;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point, so the
// library does not link libcuda directly.
inline PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D row-major tensor [rows][cols] of `elem_bytes`-byte elements, copied in
// boxes of box_rows x box_cols with the 128-byte swizzle (box_cols *
// elem_bytes must be 128). Out-of-range boxes are zero-filled.
inline int make_tmap_2d(CUtensorMap* m, const void* base, CUtensorMapDataType dtype,
                        int elem_bytes, uint64_t rows, uint64_t cols, uint32_t box_rows,
                        uint32_t box_cols) {
  auto enc = tensor_map_encoder();
  if (!enc) return record_failure(MOE_ERR_CUDA, "cuTensorMapEncodeTiled", "entry point not found");
  if (reinterpret_cast<uintptr_t>(base) % 16 != 0) return MOE_ERR_INVALID_ARG;
  if ((cols * elem_bytes) % 16 != 0) return MOE_ERR_UNSUPPORTED;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * static_cast<cuuint64_t>(elem_bytes)};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    char what[96];
    snprintf(what, sizeof what, "CUresult %d (rows %llu, cols %llu, box %ux%u)", static_cast<int>(r),
             static_cast<unsigned long long>(rows), static_cast<unsigned long long>(cols), box_rows,
             box_cols);
    return record_failure(MOE_ERR_CUDA, "cuTensorMapEncodeTiled", what);
  }
  return MOE_OK;
}

}  // namespace moe
