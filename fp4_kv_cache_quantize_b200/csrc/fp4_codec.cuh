// fp4_codec.cuh -- the FP4 main-KV encoding of eight channels, shared by the
// bulk pack kernel and the cache-append kernel so that both produce the same
// bits.  Format: E2M1 codes with one E4M3 scale per 16 channels and no global
// scale (release note "DeepSeek-V4.1-Flash 发布：100 万上下文 + FP4 KV Cache +
// 跨层注意力复用", section "FP4 KV、Bounded Replay 及其他扩展"; yomxxx.com CSA2
// paper notes, section 三 "FP4 与部署侧的两个数字池").
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp4.h>
#include <cuda_fp8.h>
#include <stdint.h>

namespace csa2 {

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ void unpack_bf16x8(const uint4& v, float (&f)[8]) {
  f[0] = bf16_lo(v.x); f[1] = bf16_hi(v.x); f[2] = bf16_lo(v.y); f[3] = bf16_hi(v.y);
  f[4] = bf16_lo(v.z); f[5] = bf16_hi(v.z); f[6] = bf16_lo(v.w); f[7] = bf16_hi(v.w);
}

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

// Largest magnitude of eight channels.
__device__ __forceinline__ float amax8(const float (&f)[8]) {
  float a = 0.0f;
#pragma unroll
  for (int k = 0; k < 8; k++) a = fmaxf(a, fabsf(f[k]));
  return a;
}

// Encode eight channels of a 16-channel group whose magnitude maximum is
// group_amax: returns the four code bytes (even channel in the low nibble of
// each) and writes the group's E4M3 scale bits to *scale_bits.
//   scale = E4M3_RNE_satfinite(fp32(amax) / 6), one correctly rounded division;
//   scale == 0 -> codes 0; else code = E2M1_RNE_satfinite(x / scale).
__device__ __forceinline__ uint32_t fp4_encode8(const float (&f)[8], float group_amax,
                                                uint8_t* scale_bits) {
  const float t = __fdiv_rn(group_amax, 6.0f);
  const __nv_fp8_storage_t sb = __nv_cvt_float_to_fp8(t, __NV_SATFINITE, __NV_E4M3);
  const float s = __half2float(__half(__nv_cvt_fp8_to_halfraw(sb, __NV_E4M3)));
  *scale_bits = (uint8_t)sb;
  uint32_t packed = 0;
  if (s != 0.0f) {
    const float r = __frcp_rn(s);
#pragma unroll
    for (int k = 0; k < 4; k++) {
      const float2 qq = make_float2(div_by_scale(f[2 * k], s, r), div_by_scale(f[2 * k + 1], s, r));
      const uint32_t byte = (uint32_t)__nv_cvt_float2_to_fp4x2(qq, __NV_E2M1, cudaRoundNearest);
      packed |= (byte & 0xFFu) << (8 * k);
    }
  }
  return packed;
}

}  // namespace csa2
