// noalloc.cu -- csa2_index_full_noalloc: the Full-mode indexer for callers
// that cannot allocate device memory.
//
// Its scratch (status word, block maxima, candidate blocks) is a file-scope
// static __device__ array of CSA2_NOALLOC_SCRATCH_BYTES that every GPU which
// loads this library holds until the process exits.  Host code must not pass
// the array's name to a kernel: on the host that name is a stand-in, not a
// device address.  The device address is looked up once per device with
// cudaGetSymbolAddress (on that device's first call) and handed to the same
// code path as csa2_index_full with a caller workspace.  The address is
// cached with the context it belongs to and looked up again when the
// device's current context is a different one (after cudaDeviceReset the
// library's module is loaded again, at another address).
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "capi_common.h"

namespace csa2 {

static __device__ __align__(256) uint8_t g_noalloc_scratch[CSA2_NOALLOC_SCRATCH_BYTES];

static std::mutex g_noalloc_mu;
static void* g_noalloc_ptr[256];      // per device ordinal
static CUcontext g_noalloc_ctx[256];  // the context each address belongs to

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

// The current context of the calling thread (nullptr if it cannot be read).
static CUcontext current_context() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  CUcontext ctx = nullptr;
  if (fn == nullptr || fn(&ctx) != CUDA_SUCCESS) return nullptr;
  return ctx;
}

// Device address of the static scratch on the current device.
static csa2_status noalloc_scratch(void** out) {
  int dev = 0;
  CSA2_CUDA(cudaGetDevice(&dev));
  CSA2_REQUIRE(dev >= 0 && dev < 256, CSA2_ERR_INVALID_ARG, "device ordinal %d", dev);
  // (no context is current before the runtime's first use of the device: the
  // look-up below then runs again on the next call, with the context known)
  const CUcontext ctx = current_context();
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr || ctx == nullptr || ctx != g_noalloc_ctx[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(g_noalloc_scratch)");
    g_noalloc_ptr[dev] = p;
    g_noalloc_ctx[dev] = ctx;
  }
  *out = g_noalloc_ptr[dev];
  return CSA2_OK;
}

}  // namespace csa2

extern "C" csa2_status csa2_index_full_noalloc(const csa2_kv_view* kv, const uint16_t* q_idx,
                                               const float* w, int32_t top_k,
                                               int32_t pool_blocks, int32_t* idx,
                                               int32_t* idx_count, int32_t* pool,
                                               int32_t* pool_count, csa2_stream_t stream) {
  using namespace csa2;
  // the same argument checks as csa2_index_full, before the size check and
  // before anything is enqueued
  csa2_status r = check_index_args(kv, top_k, pool_blocks);
  if (r) return r;
  CSA2_REQUIRE_PTR(q_idx);
  CSA2_REQUIRE_PTR(w);
  CSA2_REQUIRE_PTR(idx);
  CSA2_REQUIRE_PTR(idx_count);
  if (pool_blocks > 0) {
    CSA2_REQUIRE_PTR(pool);
    CSA2_REQUIRE_PTR(pool_count);
  }
  const size_t need = csa2_index_workspace_size(kv, top_k, pool_blocks);
  CSA2_REQUIRE(need <= (size_t)CSA2_NOALLOC_SCRATCH_BYTES, CSA2_ERR_WORKSPACE,
               "this batch and context need %zu bytes of scratch but the static scratch holds "
               "%u; use csa2_index_full with a caller workspace",
               need, (unsigned)CSA2_NOALLOC_SCRATCH_BYTES);
  void* scratch = nullptr;
  r = noalloc_scratch(&scratch);
  if (r) return r;
  // The status word must start at zero; everything else in the scratch is
  // written before it is read.
  CSA2_CUDA(cudaMemsetAsync(scratch, 0, CSA2_WS_HEADER, (cudaStream_t)stream));
  return csa2_index_full(kv, q_idx, w, top_k, pool_blocks, idx, idx_count, pool, pool_count,
                         scratch, (size_t)CSA2_NOALLOC_SCRATCH_BYTES, stream);
}
