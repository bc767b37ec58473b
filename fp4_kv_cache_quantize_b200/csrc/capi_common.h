// capi_common.h -- host-side helpers shared by the C ABI translation units:
// thread-local error text, argument checks, device properties.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <cstdarg>
#include <cstdio>
#include <string>

#include "../../include/csa2.h"

namespace csa2 {

csa2_status fail(csa2_status s, const char* fmt, ...);
csa2_status cuda_fail(cudaError_t e, const char* what);
int num_sms();
// Records the next trace event (see csa2_trace_set) before a launch.
void trace_mark(const char* stage, cudaStream_t st);

// Host-side checks of csa2_index_full's view and sizes (capi_index.cu).
csa2_status check_index_args(const csa2_kv_view* kv, int top_k, int pool_blocks);

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

#define CSA2_REQUIRE(cond, status, ...) \
  do {                                  \
    if (!(cond)) return ::csa2::fail(status, __VA_ARGS__); \
  } while (0)

#define CSA2_REQUIRE_PTR(p)                                                       \
  do {                                                                           \
    if ((p) == nullptr) return ::csa2::fail(CSA2_ERR_INVALID_ARG, "%s is NULL", #p); \
    if (!::csa2::aligned16(p))                                                   \
      return ::csa2::fail(CSA2_ERR_ALIGNMENT, "%s is not 16-byte aligned", #p);   \
  } while (0)

#define CSA2_CUDA(call)                                   \
  do {                                                    \
    cudaError_t e_ = (call);                              \
    if (e_ != cudaSuccess) return ::csa2::cuda_fail(e_, #call); \
  } while (0)

// kernels (defined in the .cu files)
cudaError_t launch_pack(const uint16_t* x, int64_t rows, int32_t ch, uint8_t* codes,
                        uint8_t* scales, cudaStream_t st, int num_sms);
cudaError_t launch_unpack(const uint8_t* codes, const uint8_t* scales, int64_t rows, int32_t ch,
                          uint16_t* y, cudaStream_t st, int num_sms);

}  // namespace csa2
