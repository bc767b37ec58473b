// quant.cu -- FP4 main-KV pack (quantise) and unpack (dequantise) kernels.
//
// Format: see fp4_codec.cuh.
//
// Both kernels are pure HBM streams: 16-byte coalesced loads and stores, a
// grid of a few CTAs per SM looping over the data, no shared memory.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp4.h>
#include <cuda_fp8.h>

#include "csa2_internal.cuh"
#include "fp4_codec.cuh"

namespace csa2 {

__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// One thread packs one 16-byte chunk (8 channels); lanes 2j and 2j+1 share a
// 16-channel scale group.  n_chunks = rows * ch / 8 (even).
__global__ void __launch_bounds__(256) fp4_pack_kernel(const uint4* __restrict__ x,
                                                       int64_t n_chunks,
                                                       uint32_t* __restrict__ codes,
                                                       uint8_t* __restrict__ scales) {
  constexpr int U = 4;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  for (int64_t base = tid;; base += U * stride) {
    if (__all_sync(0xffffffffu, base >= n_chunks)) break;
    uint4 v[U];
#pragma unroll
    for (int u = 0; u < U; u++) {
      const int64_t i = base + u * stride;
      v[u] = (i < n_chunks) ? ld_stream(x + i) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < U; u++) {
      const int64_t i = base + u * stride;
      float f[8];
      unpack_bf16x8(v[u], f);
      float amax = amax8(f);
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
      uint8_t sb;
      const uint32_t packed = fp4_encode8(f, amax, &sb);
      if (i < n_chunks) {
        codes[i] = packed;
        if ((i & 1) == 0) scales[i >> 1] = sb;
      }
    }
  }
}

// One thread unpacks one 4-byte code word (8 channels) into 16 bytes of bf16.
__global__ void __launch_bounds__(256) fp4_unpack_kernel(const uint32_t* __restrict__ codes,
                                                         const uint8_t* __restrict__ scales,
                                                         int64_t n_chunks,
                                                         uint4* __restrict__ y) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n_chunks; i += stride) {
    const uint32_t c = __ldg(codes + i);
    const __half s = __half(__nv_cvt_fp8_to_halfraw(__ldg(scales + (i >> 1)), __NV_E4M3));
    const __half2 s2 = __half2(s, s);
    uint32_t out[4];
#pragma unroll
    for (int k = 0; k < 4; k++) {
      const __half2 v = __half2(__nv_cvt_fp4x2_to_halfraw2(
          (__nv_fp4x2_storage_t)((c >> (8 * k)) & 0xFFu), __NV_E2M1));
      // e2m1 * e4m3 has at most 5 significant bits and lies in [2^-10, 2688]:
      // exact in fp16, and exact again in bf16.
      const float2 f = __half22float2(__hmul2(v, s2));
      const __nv_bfloat162 b = __float22bfloat162_rn(f);
      out[k] = *reinterpret_cast<const uint32_t*>(&b);
    }
    y[i] = make_uint4(out[0], out[1], out[2], out[3]);
  }
}

int grid_for_stream(int64_t n_items, int threads, int num_sms) {
  const int64_t want = (n_items + threads - 1) / threads;
  const int64_t cap = (int64_t)num_sms * 8;
  return (int)(want < 1 ? 1 : (want < cap ? want : cap));
}

cudaError_t launch_pack(const uint16_t* x, int64_t rows, int32_t ch, uint8_t* codes,
                        uint8_t* scales, cudaStream_t st, int num_sms) {
  const int64_t n = rows * (int64_t)ch / 8;
  if (n == 0) return cudaSuccess;
  fp4_pack_kernel<<<grid_for_stream(n / 4, 256, num_sms), 256, 0, st>>>(
      reinterpret_cast<const uint4*>(x), n, reinterpret_cast<uint32_t*>(codes), scales);
  return cudaGetLastError();
}

cudaError_t launch_unpack(const uint8_t* codes, const uint8_t* scales, int64_t rows, int32_t ch,
                          uint16_t* y, cudaStream_t st, int num_sms) {
  const int64_t n = rows * (int64_t)ch / 8;
  if (n == 0) return cudaSuccess;
  fp4_unpack_kernel<<<grid_for_stream(n / 2, 256, num_sms), 256, 0, st>>>(
      reinterpret_cast<const uint32_t*>(codes), scales, n, reinterpret_cast<uint4*>(y));
  return cudaGetLastError();
}

}  // namespace csa2
