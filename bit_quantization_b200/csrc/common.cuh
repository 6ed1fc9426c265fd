// Shared definitions of the CUDA path: status word, 16-bit loads, E2M1 and
// UE4M3 conversions through the hardware cvt instructions.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "thrift_nvfp4.h"

namespace thrift {

// Device status word of this library (THRIFT_OK or THRIFT_ERR_TIMEOUT); one
// per device, read and reset by thrift_device_status().  The library is one
// translation unit, so the definition lives here.
__device__ int g_device_status = 0;

__device__ __forceinline__ void set_device_status(int code) {
  atomicCAS(&g_device_status, 0, code);
}

// 16-bit storage -> fp32 (exact).  DT: 0 = fp16, 1 = bf16.
template <int DT>
__device__ __forceinline__ float h2f(uint16_t h) {
  if constexpr (DT == 1) {
    return __uint_as_float(((uint32_t)h) << 16);
  } else {
    return __half2float(__ushort_as_half(h));
  }
}

// fp32 -> 16-bit storage, round to nearest even.
template <int DT>
__device__ __forceinline__ uint16_t f2h(float f) {
  if constexpr (DT == 1) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(f));
  } else {
    return __half_as_ushort(__float2half_rn(f));
  }
}

// Two fp32 values -> one byte of E2M1 codes (lo in bits 0..3, hi in 4..7),
// round to nearest even, saturating.
__device__ __forceinline__ uint32_t e2m1x2(float lo, float hi) {
  uint32_t out;
  asm("{\n\t.reg .b8 b0;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.u32.u8 %0, b0;\n\t}"
      : "=r"(out)
      : "f"(lo), "f"(hi));
  return out & 0xFF;
}

// Non-negative fp32 -> UE4M3 byte, round to nearest even, saturating at 448.
__device__ __forceinline__ uint32_t ue4m3(float v) {
  uint16_t out;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %2, %1;" : "=h"(out) : "f"(v), "f"(0.0f));
  return out & 0x7F;
}

// UE4M3 byte -> fp32 (exact), bytes 0..126.
__device__ __forceinline__ float ue4m3_decode(uint32_t b) {
  const uint32_t e = (b >> 3) & 15u, m = b & 7u;
  if (e == 0) return (float)m * 0.001953125f;  // m * 2^-9
  return __uint_as_float(((e + 120u) << 23) | (m << 20));
}

__host__ __device__ __forceinline__ int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

}  // namespace thrift
