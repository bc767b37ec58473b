// capi.cu -- the extern "C" entry points of libcsa2.so: argument checks,
// status plumbing, and launches.  No allocation, no synchronisation (except
// csa2_sync_status), no exceptions across the ABI.
#include <cuda_runtime.h>

#include <cstring>
#include <mutex>
#include <string>

#include "capi_common.h"
#include "csa2_internal.cuh"

namespace csa2 {

static thread_local std::string t_last_error;
static thread_local csa2_trace* t_trace = nullptr;

void trace_mark(const char* stage, cudaStream_t st) {
  csa2_trace* t = t_trace;
  if (!t || t->count < 0 || t->count >= t->capacity || t->count >= 64) return;
  if (cudaEventRecord(static_cast<cudaEvent_t>(t->events[t->count]), st) != cudaSuccess) return;
  t->names[t->count++] = stage;
}

csa2_status fail(csa2_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  t_last_error = buf;
  return s;
}

csa2_status cuda_fail(cudaError_t e, const char* what) {
  return fail(CSA2_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// A wait on an mbarrier that nothing completes, through the same bounded
// wait every pipeline uses: it gives up after `budget` cycles and records
// ST_TIMEOUT, then the kernel returns normally.
__global__ void bounded_wait_selftest_kernel(uint32_t* status, long long budget) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
    if (!mbar_wait(&bar, 0, nullptr, budget)) set_status(status, ST_TIMEOUT);
    mbar_arrive(&bar);  // complete the phase so that nothing is left pending
  }
}

int num_sms() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    return 148;
  return n;
}

}  // namespace csa2

using namespace csa2;

extern "C" {

const char* csa2_status_string(csa2_status s) {
  switch (s) {
    case CSA2_OK: return "CSA2_OK";
    case CSA2_ERR_INVALID_ARG: return "CSA2_ERR_INVALID_ARG";
    case CSA2_ERR_SHAPE: return "CSA2_ERR_SHAPE";
    case CSA2_ERR_ALIGNMENT: return "CSA2_ERR_ALIGNMENT";
    case CSA2_ERR_WORKSPACE: return "CSA2_ERR_WORKSPACE";
    case CSA2_ERR_CUDA: return "CSA2_ERR_CUDA";
    case CSA2_ERR_TIMEOUT: return "CSA2_ERR_TIMEOUT";
    case CSA2_ERR_DEVICE_CHECK: return "CSA2_ERR_DEVICE_CHECK";
  }
  return "CSA2_UNKNOWN_STATUS";
}

const char* csa2_last_error(void) { return t_last_error.c_str(); }

void csa2_trace_set(csa2_trace* trace) { t_trace = trace; }

csa2_status csa2_workspace_init(void* ws, size_t ws_bytes, csa2_stream_t stream) {
  CSA2_REQUIRE_PTR(ws);
  CSA2_REQUIRE(ws_bytes >= CSA2_WS_HEADER, CSA2_ERR_WORKSPACE,
               "workspace of %zu bytes is smaller than its %d-byte header", ws_bytes,
               CSA2_WS_HEADER);
  CSA2_CUDA(cudaMemsetAsync(ws, 0, CSA2_WS_HEADER, (cudaStream_t)stream));
  return CSA2_OK;
}

csa2_status csa2_selftest_bounded_wait(void* ws, size_t ws_bytes, int64_t cycles,
                                       csa2_stream_t stream) {
  CSA2_REQUIRE_PTR(ws);
  CSA2_REQUIRE(ws_bytes >= CSA2_WS_HEADER, CSA2_ERR_WORKSPACE,
               "workspace of %zu bytes is smaller than its %d-byte header", ws_bytes,
               CSA2_WS_HEADER);
  CSA2_REQUIRE(cycles >= 1000 && cycles <= kWaitCycles, CSA2_ERR_INVALID_ARG,
               "cycles = %lld outside [1000, %lld]", (long long)cycles, (long long)kWaitCycles);
  bounded_wait_selftest_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(static_cast<uint32_t*>(ws),
                                                                  (long long)cycles);
  CSA2_CUDA(cudaGetLastError());
  return CSA2_OK;
}

csa2_status csa2_sync_status(void* ws, csa2_stream_t stream) {
  CSA2_REQUIRE_PTR(ws);
  uint32_t word = 0;
  CSA2_CUDA(cudaMemcpyAsync(&word, ws, sizeof word, cudaMemcpyDeviceToHost, (cudaStream_t)stream));
  CSA2_CUDA(cudaStreamSynchronize((cudaStream_t)stream));
  CSA2_CUDA(cudaGetLastError());
  if (word) {
    CSA2_CUDA(cudaMemsetAsync(ws, 0, sizeof word, (cudaStream_t)stream));
    if (word & ST_TIMEOUT)
      return fail(CSA2_ERR_TIMEOUT, "a device-side bounded wait expired (status 0x%x)", word);
    return fail(CSA2_ERR_DEVICE_CHECK,
                "a device-side bounds check clamped an out-of-range row (status 0x%x)", word);
  }
  return CSA2_OK;
}

csa2_status csa2_quantize_fp4(const uint16_t* x_bf16, int64_t rows, int32_t ch, uint8_t* codes,
                              uint8_t* scales, csa2_stream_t stream) {
  CSA2_REQUIRE(rows >= 0, CSA2_ERR_SHAPE, "rows = %lld is negative", (long long)rows);
  CSA2_REQUIRE(ch > 0 && ch % 16 == 0, CSA2_ERR_SHAPE, "ch = %d is not a positive multiple of 16",
               ch);
  if (rows == 0) return CSA2_OK;
  CSA2_REQUIRE_PTR(x_bf16);
  CSA2_REQUIRE_PTR(codes);
  CSA2_REQUIRE_PTR(scales);
  trace_mark("pack", (cudaStream_t)stream);
  CSA2_CUDA(launch_pack(x_bf16, rows, ch, codes, scales, (cudaStream_t)stream, num_sms()));
  trace_mark("end", (cudaStream_t)stream);
  return CSA2_OK;
}

csa2_status csa2_dequantize_fp4(const uint8_t* codes, const uint8_t* scales, int64_t rows,
                                int32_t ch, uint16_t* y_bf16, csa2_stream_t stream) {
  CSA2_REQUIRE(rows >= 0, CSA2_ERR_SHAPE, "rows = %lld is negative", (long long)rows);
  CSA2_REQUIRE(ch > 0 && ch % 16 == 0, CSA2_ERR_SHAPE, "ch = %d is not a positive multiple of 16",
               ch);
  if (rows == 0) return CSA2_OK;
  CSA2_REQUIRE_PTR(codes);
  CSA2_REQUIRE_PTR(scales);
  CSA2_REQUIRE_PTR(y_bf16);
  trace_mark("unpack", (cudaStream_t)stream);
  CSA2_CUDA(launch_unpack(codes, scales, rows, ch, y_bf16, (cudaStream_t)stream, num_sms()));
  trace_mark("end", (cudaStream_t)stream);
  return CSA2_OK;
}

}  // extern "C"
