// quant.cu -- FP4 main-KV pack (quantise) and unpack (dequantise) kernels.
//
// Format: E2M1 codes with one E4M3 scale per 16 channels and no global
// scale, i.e. NVFP4 without its second-level scale (release note
// "DeepSeek-V4.1-Flash 发布：100 万上下文 + FP4 KV Cache + 跨层注意力复用",
// section "FP4 KV、Bounded Replay 及其他扩展"; yomxxx.com CSA2 paper notes,
// section 三 "FP4 与部署侧的两个数字池").
//
// Both kernels are pure HBM streams: 16-byte coalesced loads and stores, a
// grid of a few CTAs per SM looping over the data, no shared memory.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp4.h>
#include <cuda_fp8.h>

#include "csa2_internal.cuh"

namespace csa2 {

__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// x / s for an E4M3 scale s, exact enough for E2M1 rounding: q0 = x * (1/s)
// is refined with one fused residual step.  When x/s is exactly an E2M1
// rounding midpoint (x = T*s, T in {.25,.75,1.25,1.75,2.5,3.5,5}) the result
// is exactly T, so ties round as they would from the true quotient; every
// other quotient of a bf16 by an E4M3 value lies at least ~2^-9 (relative)
// away from every midpoint, far beyond the few-ulp error of q0.  The sign is
// copied from x because the residual step turns x = -0 into +0.
__device__ __forceinline__ float div_by_scale(float x, float s, float r) {
  const float q0 = __fmul_rn(x, r);
  const float res = __fmaf_rn(-q0, s, x);
  return copysignf(__fmaf_rn(res, r, q0), x);
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
      float f[8] = {bf16_lo(v[u].x), bf16_hi(v[u].x), bf16_lo(v[u].y), bf16_hi(v[u].y),
                    bf16_lo(v[u].z), bf16_hi(v[u].z), bf16_lo(v[u].w), bf16_hi(v[u].w)};
      float amax = 0.0f;
#pragma unroll
      for (int k = 0; k < 8; k++) amax = fmaxf(amax, fabsf(f[k]));
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
      // scale = E4M3(amax / 6): one correctly rounded fp32 division, then
      // the hardware's round-to-nearest-even, saturate-to-finite conversion.
      const float t = __fdiv_rn(amax, 6.0f);
      const __nv_fp8_storage_t sb = __nv_cvt_float_to_fp8(t, __NV_SATFINITE, __NV_E4M3);
      const float s = __half2float(__half(__nv_cvt_fp8_to_halfraw(sb, __NV_E4M3)));
      uint32_t packed = 0;
      if (s != 0.0f) {
        const float r = __frcp_rn(s);
#pragma unroll
        for (int k = 0; k < 4; k++) {
          const float2 qq = make_float2(div_by_scale(f[2 * k], s, r),
                                        div_by_scale(f[2 * k + 1], s, r));
          const uint32_t byte =
              (uint32_t)__nv_cvt_float2_to_fp4x2(qq, __NV_E2M1, cudaRoundNearest);
          packed |= (byte & 0xFFu) << (8 * k);
        }
      }
      if (i < n_chunks) {
        codes[i] = packed;
        if ((i & 1) == 0) scales[i >> 1] = (uint8_t)sb;
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
