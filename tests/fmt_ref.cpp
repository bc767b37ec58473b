// Independent format reference for the oracle pins: thin extern "C" wrappers
// that only CALL the host conversion routines of CUDA's cuda_fp8.h and
// cuda_fp4.h (round-to-nearest-even with saturation to the largest finite
// value).  Compiled by the tests with the host C++ compiler; no GPU involved.
#include <cuda_fp4.h>
#include <cuda_fp8.h>
#include <cstring>

extern "C" {
unsigned char ref_e4m3_satfinite(float x) {
  return (unsigned char)__nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3);
}
unsigned char ref_e2m1_rn(float x) {
  return (unsigned char)__nv_cvt_float_to_fp4(x, __NV_E2M1, cudaRoundNearest);
}
float ref_e2m1_value(unsigned char code) {
  __half_raw h = __nv_cvt_fp4_to_halfraw((__nv_fp4_storage_t)code, __NV_E2M1);
  __half hh(h);
  return __half2float(hh);
}
float ref_e4m3_value(unsigned char bits) {
  __half_raw h = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)bits, __NV_E4M3);
  __half hh(h);
  return __half2float(hh);
}
}
