// Host-side calls of the FP4 / FP8 conversion functions that CUDA's public
// headers (cuda_fp4.h, cuda_fp8.h) provide.  Test-only: the oracle's own
// encoders are checked against these, element by element.  Nothing here is a
// copy of the headers' implementation; the functions are called.
#include <cuda_fp4.h>
#include <cuda_fp8.h>
#include <cuda_fp16.h>
#include <stdint.h>

extern "C" void cu_e2m1_encode_n(const float* v, int64_t n, uint8_t* out) {
  for (int64_t i = 0; i < n; i++)
    out[i] = (uint8_t)__nv_cvt_float_to_fp4(v[i], __NV_E2M1, cudaRoundNearest);
}

extern "C" void cu_e4m3_encode_n(const float* v, int64_t n, uint8_t* out) {
  for (int64_t i = 0; i < n; i++)
    out[i] = (uint8_t)__nv_cvt_float_to_fp8(v[i], __NV_SATFINITE, __NV_E4M3);
}

extern "C" void cu_e4m3_decode_n(const uint8_t* c, int64_t n, float* out) {
  for (int64_t i = 0; i < n; i++) {
    __half_raw hr = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)c[i], __NV_E4M3);
    out[i] = __half2float(__half(hr));
  }
}

extern "C" void cu_e2m1_decode_n(const uint8_t* c, int64_t n, float* out) {
  for (int64_t i = 0; i < n; i++) {
    __half_raw hr = __nv_cvt_fp4_to_halfraw((__nv_fp4_storage_t)c[i], __NV_E2M1);
    out[i] = __half2float(__half(hr));
  }
}
