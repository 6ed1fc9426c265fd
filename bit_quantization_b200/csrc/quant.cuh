// NVFP4 quantiser: per-tensor absmax, optional Hadamard rotation, per-block
// UE4M3 scale (max scaling or ScaleSearch), E2M1 codes.
//
// Sources: "Busca tus Escalas de Punto Flotante por Bloques" -- ScaleSearch,
// Mecanismo (max scaling maps the block absmax to FP4 6; candidate scales
// are integer offsets f on the UE4M3 bit pattern), Estrategia de Busqueda
// (f in [-2, 6], least block MSE); ScaleSearchAttention (Hadamard rotation of
// Q and K).  "Attn-QAT", Resumo tecnico 1 (E2M1 grid).
//
// Arithmetic (every step an IEEE-754 correctly rounded fp32/fp64 op, so the
// result is reproducible bit for bit):
//   g       = amax / 2688 (g = 1 when amax = 0)
//   S0      = ue4m3(amax_b / (6 g))
//   dec(S)  = ue4m3_value(S) * g,  r = 1 / dec
//   code_e  = e2m1(x_e * r)
//   err(S)  = (sequential fmaf sum of (t_e - q_e)^2) * ue4m3_value(S)^2 in fp64
//   ScaleSearch visits f = 0,-2,-1,1,...,6 (bytes 1..126 only) and keeps the
//   first strict minimum; S0 = 0 keeps 0 (all codes 0).
#pragma once
#include "common.cuh"

namespace thrift {

constexpr float kTensorScaleDiv = 2688.0f;  // 6 * 448: FP4 max times UE4M3 max

__device__ __forceinline__ float tensor_scale_from_amax(uint32_t amax_bits) {
  const float amax = __uint_as_float(amax_bits);
  return amax == 0.0f ? 1.0f : __fdiv_rn(amax, kTensorScaleDiv);
}

// E2M1 round trip of two values: q = decode(E2M1(t)) (round to nearest
// even, saturating), through the hardware converts to E2M1 and back to f16
// (every E2M1 value, signed zeros included, is exact in f16 and in fp32).
__device__ __forceinline__ void e2m1x2_roundtrip(float t0, float t1, float& q0, float& q1) {
  asm("{\n\t.reg .b8 c;\n\t.reg .b32 h;\n\t.reg .b16 lo, hi;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 c, %3, %2;\n\t"
      "cvt.rn.f16x2.e2m1x2 h, c;\n\t"
      "mov.b32 {lo, hi}, h;\n\t"
      "cvt.f32.f16 %0, lo;\n\t"
      "cvt.f32.f16 %1, hi;\n\t}"
      : "=f"(q0), "=f"(q1)
      : "f"(t0), "f"(t1));
}

// A byte of two E2M1 codes (element 2i in the low nibble) -> their values.
__device__ __forceinline__ void e2m1x2_values(uint32_t byte, float& v0, float& v1) {
  asm("{\n\t.reg .b8 c;\n\t.reg .b32 h;\n\t.reg .b16 lo, hi;\n\t"
      "cvt.u8.u32 c, %2;\n\t"
      "cvt.rn.f16x2.e2m1x2 h, c;\n\t"
      "mov.b32 {lo, hi}, h;\n\t"
      "cvt.f32.f16 %0, lo;\n\t"
      "cvt.f32.f16 %1, hi;\n\t}"
      : "=f"(v0), "=f"(v1)
      : "r"(byte));
}

// Block error of candidate byte S (see header comment).
__device__ __forceinline__ double block_err(const float (&x)[16], float g, uint32_t S) {
  const float sv = ue4m3_decode(S);
  const float r = __frcp_rn(__fmul_rn(sv, g));
  float acc = 0.0f;
#pragma unroll
  for (int e = 0; e < 16; e += 2) {
    const float t0 = __fmul_rn(x[e], r), t1 = __fmul_rn(x[e + 1], r);
    float q0, q1;
    e2m1x2_roundtrip(t0, t1, q0, q1);
    const float d0 = __fsub_rn(t0, q0), d1 = __fsub_rn(t1, q1);
    acc = __fmaf_rn(d0, d0, acc);
    acc = __fmaf_rn(d1, d1, acc);
  }
  const double s = (double)sv;
  return __dmul_rn((double)acc, __dmul_rn(s, s));
}

// Quantises one 16-element block.  Returns the scale byte; codes in
// lo (elements 0..7) and hi (elements 8..15), element 2c in the low nibble.
__device__ __forceinline__ uint32_t quant_block16(const float (&x)[16], float g, bool ss,
                                                  uint32_t& lo, uint32_t& hi) {
  float amax = 0.0f;
#pragma unroll
  for (int e = 0; e < 16; ++e) amax = fmaxf(amax, fabsf(x[e]));
  uint32_t S = ue4m3(__fdiv_rn(amax, __fmul_rn(6.0f, g)));
  if (S == 0) {
    lo = hi = 0;
    return 0;
  }
  if (ss) {
    double best = 0.0;
    int best_f = 0;
    bool have = false;
    // candidates in the order 0, -2, -1, 1, 2, ..., 6 (a rolled loop keeps
    // the code small enough for the instruction cache)
#pragma unroll 1
    for (int oi = 0; oi < 9; ++oi) {
      const int f = oi == 0 ? 0 : (oi <= 2 ? oi - 3 : oi - 2);
      const int b = (int)S + f;
      if (b >= 1 && b <= 126) {
        const double err = block_err(x, g, (uint32_t)b);
        if (!have || err < best) {
          best = err;
          best_f = f;
          have = true;
        }
      }
    }
    S = (uint32_t)((int)S + best_f);
  }
  const float r = __frcp_rn(__fmul_rn(ue4m3_decode(S), g));
  uint32_t c[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) c[i] = e2m1x2(__fmul_rn(x[2 * i], r), __fmul_rn(x[2 * i + 1], r));
  lo = c[0] | (c[1] << 8) | (c[2] << 16) | (c[3] << 24);
  hi = c[4] | (c[5] << 8) | (c[6] << 16) | (c[7] << 24);
  return S;
}

// Loads 16 consecutive 16-bit values (32-byte aligned) as fp32.
template <int DT>
__device__ __forceinline__ void load16(const uint16_t* p, float (&x)[16]) {
  const uint4 a = __ldg(reinterpret_cast<const uint4*>(p));
  const uint4 b = __ldg(reinterpret_cast<const uint4*>(p) + 1);
  const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    x[2 * i] = h2f<DT>((uint16_t)(w[i] & 0xFFFF));
    x[2 * i + 1] = h2f<DT>((uint16_t)(w[i] >> 16));
  }
}

// Unnormalised Sylvester-Hadamard transform of rows of D = 16 * G elements
// spread over G consecutive lanes (16 elements each, lane-group aligned).
// Butterfly strides 1, 2, 4, 8 inside a lane, then 16, 32, 64 across lanes;
// (a, b) -> (a + b, a - b) with a at the lower index, the same DAG as a
// sequential in-place transform with ascending strides.
template <int G>
__device__ __forceinline__ void fwht_rows16(float (&x)[16]) {
#pragma unroll
  for (int h = 1; h < 16; h *= 2) {
#pragma unroll
    for (int i = 0; i < 16; i += 2 * h) {
#pragma unroll
      for (int j = i; j < i + h; ++j) {
        const float a = x[j], b = x[j + h];
        x[j] = __fadd_rn(a, b);
        x[j + h] = __fsub_rn(a, b);
      }
    }
  }
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int m = 1; m < G; m *= 2) {
    const bool upper = (lane & m) != 0;
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const float other = __shfl_xor_sync(0xffffffffu, x[e], m);
      x[e] = upper ? __fsub_rn(other, x[e]) : __fadd_rn(x[e], other);
    }
  }
}

__device__ __forceinline__ float block_absmax(const float (&x)[16]) {
  float a = 0.0f;
#pragma unroll
  for (int e = 0; e < 16; ++e) a = fmaxf(a, fabsf(x[e]));
  return a;
}

// Warp max followed by one atomicMax per warp on the bit pattern of a
// non-negative float (the ordering of such patterns is the float ordering).
__device__ __forceinline__ void warp_atomic_amax(float a, uint32_t* dst) {
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, m));
  if ((threadIdx.x & 31) == 0 && a > 0.0f) atomicMax(dst, __float_as_uint(a));
}

}  // namespace thrift
