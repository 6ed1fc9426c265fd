// Quantiser kernels: tensor absmax, row-blocked and column-blocked NVFP4
// quantisation (the C-ABI layouts), and the tile images the attention kernel
// streams with bulk copies (codes swizzled for the tensor-core operand
// layout, scale factors in the tensor-memory copy layout, 16-bit tiles for
// the FP16 path).
#pragma once
#include "quant.cuh"
#include "tc.cuh"

namespace thrift {

// Sequence bounds of packed sequence `s`: cu_seqlens when given, else
// uniform sequences of `uniform_len` tokens.
struct SeqInfo {
  const int32_t* cu;
  int uniform_len;
  __device__ __forceinline__ void get(int s, int64_t& start, int& len) const {
    if (cu) {
      const int32_t a = __ldg(cu + s), b = __ldg(cu + s + 1);
      start = a;
      len = b - a;
    } else {
      start = (int64_t)s * uniform_len;
      len = uniform_len;
    }
  }
};

// ---------------------------------------------------------------- absmax --

// CTA-wide max of one value per thread; thread 0 then does one atomicMax on
// the bit pattern of the (non-negative) result.
__device__ __forceinline__ void cta_atomic_amax(float a, uint32_t* dst) {
  __shared__ float red[32];
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, m));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = a;
  __syncthreads();
  if (threadIdx.x < 32) {
    a = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.0f;
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, m));
    if (threadIdx.x == 0 && a > 0.0f) atomicMax(dst, __float_as_uint(a));
  }
}

// Loads the 32-byte block b (or zeros past the end) as raw 16-bit pairs.
__device__ __forceinline__ void load_raw(const uint16_t* x, int64_t b, int64_t n_blocks,
                                         uint4& r0, uint4& r1) {
  if (b < n_blocks) {
    r0 = __ldg(reinterpret_cast<const uint4*>(x + b * 16));
    r1 = __ldg(reinterpret_cast<const uint4*>(x + b * 16) + 1);
  } else {
    r0 = r1 = make_uint4(0, 0, 0, 0);
  }
}

template <int DT>
__device__ __forceinline__ void unpack16(const uint4& r0, const uint4& r1, float (&v)[16]) {
  const uint32_t w[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    v[2 * i] = h2f<DT>((uint16_t)(w[i] & 0xFFFF));
    v[2 * i + 1] = h2f<DT>((uint16_t)(w[i] >> 16));
  }
}

// Grid-stride absmax over 16-element blocks of x, KPT blocks in flight per
// thread.  G lanes hold one row when rows are rotated (G = d/16), G = 0 for
// no rotation.
constexpr int kKPT = 4;

template <int DT, int G>
__global__ void __launch_bounds__(256) amax_kernel(const uint16_t* __restrict__ x,
                                                   int64_t n_blocks, uint32_t* amax_out) {
  const int64_t nthreads = (int64_t)gridDim.x * blockDim.x;
  const int lane = threadIdx.x & 31;
  float a = 0.0f;
  for (int64_t base = (int64_t)blockIdx.x * blockDim.x + (threadIdx.x & ~31); base < n_blocks;
       base += nthreads * kKPT) {
    uint4 r[kKPT][2];
#pragma unroll
    for (int k = 0; k < kKPT; ++k) load_raw(x, base + lane + k * nthreads, n_blocks, r[k][0], r[k][1]);
#pragma unroll
    for (int k = 0; k < kKPT; ++k) {
      float v[16];
      unpack16<DT>(r[k][0], r[k][1], v);
      if constexpr (G > 0) fwht_rows16<G>(v);
      a = fmaxf(a, block_absmax(v));
    }
  }
  cta_atomic_amax(a, amax_out);
}

// ------------------------------------------------- row-blocked quantiser --
// codes [rows, cols/2], scales [rows, cols/16] as flat arrays of blocks.
template <int DT, int G, bool SS>
__global__ void __launch_bounds__(256) quant_rows_kernel(
    const uint16_t* __restrict__ x, int64_t n_blocks, const uint32_t* amax_in,
    float* tensor_scale, int scale_given, uint8_t* __restrict__ codes,
    uint8_t* __restrict__ scales) {
  const float g = scale_given ? *tensor_scale : tensor_scale_from_amax(*amax_in);
  if (!scale_given && blockIdx.x == 0 && threadIdx.x == 0) *tensor_scale = g;
  const int64_t nthreads = (int64_t)gridDim.x * blockDim.x;
  const int64_t wbase0 = (int64_t)blockIdx.x * blockDim.x + (threadIdx.x & ~31);
  const int lane = threadIdx.x & 31;
  for (int64_t base = wbase0; base < n_blocks; base += nthreads * kKPT) {
    uint4 r[kKPT][2];
#pragma unroll
    for (int k = 0; k < kKPT; ++k) load_raw(x, base + lane + k * nthreads, n_blocks, r[k][0], r[k][1]);
#pragma unroll
    for (int k = 0; k < kKPT; ++k) {
      const int64_t b = base + lane + k * nthreads;
      float v[16];
      unpack16<DT>(r[k][0], r[k][1], v);
      if constexpr (G > 0) fwht_rows16<G>(v);
      if (b < n_blocks) {
        uint32_t lo, hi;
        const uint32_t S = quant_block16(v, g, SS, lo, hi);
        *reinterpret_cast<uint2*>(codes + b * 8) = make_uint2(lo, hi);
        scales[b] = (uint8_t)S;
      }
    }
  }
}

// ---------------------------------------------- column-blocked quantiser --
// x [rows, cols]; 16-blocks along rows.  codes [cols, rows/2], scales
// [cols, rows/16].  One thread per (row block, column); columns fastest.
template <int DT, bool SS>
__global__ void __launch_bounds__(256) quant_cols_kernel(
    const uint16_t* __restrict__ x, int64_t rows, int64_t cols, const uint32_t* amax_in,
    float* tensor_scale, int scale_given, uint8_t* __restrict__ codes,
    uint8_t* __restrict__ scales) {
  const float g = scale_given ? *tensor_scale : tensor_scale_from_amax(*amax_in);
  if (!scale_given && blockIdx.x == 0 && threadIdx.x == 0) *tensor_scale = g;
  const int64_t n = (rows / 16) * cols;
  for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < n;
       idx += (int64_t)gridDim.x * blockDim.x) {
    const int64_t rb = idx / cols, c = idx % cols;
    float v[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) v[e] = h2f<DT>(__ldg(x + (rb * 16 + e) * cols + c));
    uint32_t lo, hi;
    const uint32_t S = quant_block16(v, g, SS, lo, hi);
    *reinterpret_cast<uint2*>(codes + c * (rows / 2) + rb * 8) = make_uint2(lo, hi);
    scales[c * (rows / 16) + rb] = (uint8_t)S;
  }
}

// ------------------------------------------------- attention tile images --

// Byte sizes of one tile image.
__host__ __device__ constexpr uint32_t fp4_tile_bytes(uint32_t rows, uint32_t kdim) {
  // codes rows x kdim/2, then one 512-byte scale-factor block per 64 of K
  return rows * kdim / 2 + (kdim / 64) * 512;
}
__host__ __device__ constexpr uint32_t f16_tile_bytes(uint32_t rows, uint32_t kdim) {
  return rows * kdim * 2;
}

// Q or K ([total, nh, d] 16-bit) -> per (sequence, head, tile) images:
//   img4:  codes [tile_rows, d/2] swizzled (pitch d/2), then scale factors;
//   img16: the unrotated 16-bit rows, d/64 regions of [tile_rows, 128 B]
//          with 128-byte swizzle.
// Rows past the sequence end are written as zeros.  G = d/16.
template <int DT, int G, bool HAD, bool SS>
__global__ void __launch_bounds__(256) qk_image_kernel(
    const uint16_t* __restrict__ x, SeqInfo seqs, int nseq, int nh, int tile_rows, int ntiles,
    const uint32_t* amax_in, uint8_t* __restrict__ img4, uint8_t* __restrict__ img16) {
  constexpr int D = G * 16;
  const float g = tensor_scale_from_amax(*amax_in);
  const uint32_t t4 = fp4_tile_bytes(tile_rows, D), t16 = f16_tile_bytes(tile_rows, D);
  const int64_t rows_per_seq = (int64_t)ntiles * tile_rows * nh;
  const int64_t n_blocks = (int64_t)nseq * rows_per_seq * G;
  const int64_t nthreads = (int64_t)gridDim.x * blockDim.x;
  for (int64_t base = (int64_t)blockIdx.x * blockDim.x + (threadIdx.x & ~31);
       base < n_blocks; base += nthreads) {
    const int64_t b = base + (threadIdx.x & 31);
    const int kb = (int)(b % G);
    const int64_t rho = b / G;
    const int head = (int)(rho % nh);
    const int64_t tp = (rho / nh) % ((int64_t)ntiles * tile_rows);
    const int seq = (int)(rho / rows_per_seq);
    bool write = false, real = false;
    int64_t start = 0;
    int len = 0;
    if (b < n_blocks) {
      seqs.get(seq, start, len);
      write = tp < ceil_div(len, tile_rows) * tile_rows;
      real = tp < len;
    }
    float v[16];
    uint4 raw0 = make_uint4(0, 0, 0, 0), raw1 = raw0;
    if (real) {
      const uint16_t* p = x + ((start + tp) * nh + head) * D + kb * 16;
      raw0 = __ldg(reinterpret_cast<const uint4*>(p));
      raw1 = __ldg(reinterpret_cast<const uint4*>(p) + 1);
    }
    {
      const uint32_t w[8] = {raw0.x, raw0.y, raw0.z, raw0.w, raw1.x, raw1.y, raw1.z, raw1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        v[2 * i] = h2f<DT>((uint16_t)(w[i] & 0xFFFF));
        v[2 * i + 1] = h2f<DT>((uint16_t)(w[i] >> 16));
      }
    }
    if constexpr (HAD) fwht_rows16<G>(v);
    if (write) {
      const int tile = (int)(tp / tile_rows), r = (int)(tp % tile_rows);
      const int64_t tidx = ((int64_t)seq * nh + head) * ntiles + tile;
      uint8_t* t4p = img4 + tidx * t4;
      uint32_t lo, hi;
      const uint32_t S = quant_block16(v, g, SS, lo, hi);
      *reinterpret_cast<uint2*>(t4p + swz_offset(r, kb * 8, D / 2)) = make_uint2(lo, hi);
      uint8_t* sf = t4p + (uint32_t)tile_rows * (D / 2);
      sf[sf_offset(r, kb)] = (uint8_t)S;
      if (tile_rows == 64) sf[sf_offset(r + 64, kb)] = 0;
      uint8_t* t16p = img16 + tidx * t16;
      const uint32_t e0 = kb * 16;
      uint8_t* reg = t16p + (e0 / 64) * ((uint32_t)tile_rows * 128);
      *reinterpret_cast<uint4*>(reg + swz_offset(r, (e0 % 64) * 2, 128)) = raw0;
      *reinterpret_cast<uint4*>(reg + swz_offset(r, (e0 % 64) * 2 + 16, 128)) = raw1;
    }
  }
}

// V ([total, Hkv, d] 16-bit) -> per (sequence, kv head, key tile) images with
// 16-blocks along tokens: img4 codes [d, blk/2] swizzled (pitch blk/2) then
// scale factors (rows = channels); img16 = V^T tile [d, blk] in blk/64
// regions of [d, 128 B] with 128-byte swizzle.  Keys past the sequence end
// are zeros.  One thread per (sequence, head, 16-token block, channel).
template <int DT, bool SS>
__global__ void __launch_bounds__(256) v_image_kernel(
    const uint16_t* __restrict__ v, SeqInfo seqs, int nseq, int Hkv, int d, int blk, int ntiles,
    const uint32_t* amax_in, uint8_t* __restrict__ img4, uint8_t* __restrict__ img16) {
  const float g = tensor_scale_from_amax(*amax_in);
  const uint32_t t4 = fp4_tile_bytes(d, blk), t16 = f16_tile_bytes(d, blk);
  const int ntb = ntiles * blk / 16;
  const int64_t n = (int64_t)nseq * Hkv * ntb * d;
  for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < n;
       idx += (int64_t)gridDim.x * blockDim.x) {
    const int c = (int)(idx % d);
    const int tb = (int)((idx / d) % ntb);
    const int hk = (int)((idx / ((int64_t)d * ntb)) % Hkv);
    const int seq = (int)(idx / ((int64_t)d * ntb * Hkv));
    int64_t start;
    int len;
    seqs.get(seq, start, len);
    const int t0 = tb * 16;
    if (t0 >= ceil_div(len, blk) * blk) continue;
    float val[16];
    uint16_t raw[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      raw[e] = (t0 + e < len) ? __ldg(v + ((start + t0 + e) * Hkv + hk) * d + c) : (uint16_t)0;
      val[e] = h2f<DT>(raw[e]);
    }
    const int j = t0 / blk, kb = t0 % blk;
    const int64_t tidx = ((int64_t)seq * Hkv + hk) * ntiles + j;
    uint8_t* t4p = img4 + tidx * t4;
    uint32_t lo, hi;
    const uint32_t S = quant_block16(val, g, SS, lo, hi);
    *reinterpret_cast<uint2*>(t4p + swz_offset(c, kb / 2, blk / 2)) = make_uint2(lo, hi);
    uint8_t* sf = t4p + (uint32_t)d * (blk / 2);
    sf[sf_offset(c, kb / 16)] = (uint8_t)S;
    if (d == 64) sf[sf_offset(c + 64, kb / 16)] = 0;
    uint8_t* reg = img16 + tidx * t16 + (kb / 64) * ((uint32_t)d * 128);
    uint4 h0, h1;
    h0.x = raw[0] | ((uint32_t)raw[1] << 16);
    h0.y = raw[2] | ((uint32_t)raw[3] << 16);
    h0.z = raw[4] | ((uint32_t)raw[5] << 16);
    h0.w = raw[6] | ((uint32_t)raw[7] << 16);
    h1.x = raw[8] | ((uint32_t)raw[9] << 16);
    h1.y = raw[10] | ((uint32_t)raw[11] << 16);
    h1.z = raw[12] | ((uint32_t)raw[13] << 16);
    h1.w = raw[14] | ((uint32_t)raw[15] << 16);
    *reinterpret_cast<uint4*>(reg + swz_offset(c, (kb % 64) * 2, 128)) = h0;
    *reinterpret_cast<uint4*>(reg + swz_offset(c, (kb % 64) * 2 + 16, 128)) = h1;
  }
}

}  // namespace thrift
