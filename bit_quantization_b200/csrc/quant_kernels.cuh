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

// ------------------------------------------- quantiser: partial maxima --
// First kernel of the quantiser when the tensor scale is computed: CTA c
// writes the absmax of its share of x (blocks c*KPT*256 + ..., grid-stride)
// to partial[c].  Launched with programmatic dependent launch: the loads
// and the maximum run while the previous kernel of the stream may still be
// finishing (a quantise kernel of an earlier call reading these same
// partial slots), and only the store waits for it.
template <int DT, int G>
__global__ void __launch_bounds__(256) amax_partial_kernel(const uint16_t* __restrict__ x,
                                                           int64_t n_blocks, float* partial) {
  __shared__ float red[8];
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
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, m));
  if (lane == 0) red[threadIdx.x >> 5] = a;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < (int)(blockDim.x >> 5); ++w) a = fmaxf(a, red[w]);
    pdl_wait();
    partial[blockIdx.x] = a;
  }
  pdl_trigger();
}

// The tensor scale of a quantise kernel: given (read once the previous
// kernel of the stream, which may have written it, is done), or g of the
// largest of the n_partial maxima of amax_partial_kernel.
__device__ __forceinline__ float quant_tensor_scale(const float* partial, int n_partial,
                                                    const float* tensor_scale, int given) {
  __shared__ float red[8];
  pdl_wait();
  if (given) return *tensor_scale;
  float m = 0.0f;
  for (int c = threadIdx.x; c < n_partial; c += blockDim.x) m = fmaxf(m, partial[c]);
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  m = red[0];
  for (int w = 1; w < (int)(blockDim.x >> 5); ++w) m = fmaxf(m, red[w]);
  return tensor_scale_from_amax(__float_as_uint(m));
}

// ------------------------------------------------- row-blocked quantiser --
// codes [rows, cols/2], scales [rows, cols/16] as flat arrays of blocks.
// Programmatic dependent launch: the first blocks' loads are issued before
// the wait for the previous kernel of the stream; everything it may have
// written (the partial maxima, a given tensor scale, the outputs) is touched
// after it.
// Blocks in flight per thread in the quantise kernel: two, so that four
// CTAs of 256 threads fit an SM (64 registers a thread).
constexpr int kQuantKPT = 2;

template <int DT, int G, bool SS>
__global__ void __launch_bounds__(256, 4) quant_rows_kernel(
    const uint16_t* __restrict__ x, int64_t n_blocks, const float* partial, int n_partial,
    float* tensor_scale, int scale_given, uint8_t* __restrict__ codes,
    uint8_t* __restrict__ scales) {
  const int64_t nthreads = (int64_t)gridDim.x * blockDim.x;
  const int64_t wbase0 = (int64_t)blockIdx.x * blockDim.x + (threadIdx.x & ~31);
  const int lane = threadIdx.x & 31;
  uint4 r[kQuantKPT][2];
#pragma unroll
  for (int k = 0; k < kQuantKPT; ++k) load_raw(x, wbase0 + lane + k * nthreads, n_blocks, r[k][0], r[k][1]);
  pdl_trigger();
  const float g = quant_tensor_scale(partial, n_partial, tensor_scale, scale_given);
  if (!scale_given && blockIdx.x == 0 && threadIdx.x == 0) *tensor_scale = g;
  for (int64_t base = wbase0; base < n_blocks; base += nthreads * kQuantKPT) {
    if (base != wbase0) {
#pragma unroll
      for (int k = 0; k < kQuantKPT; ++k)
        load_raw(x, base + lane + k * nthreads, n_blocks, r[k][0], r[k][1]);
    }
#pragma unroll
    for (int k = 0; k < kQuantKPT; ++k) {
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
    const uint16_t* __restrict__ x, int64_t rows, int64_t cols, const float* partial,
    int n_partial, float* tensor_scale, int scale_given, uint8_t* __restrict__ codes,
    uint8_t* __restrict__ scales) {
  pdl_trigger();
  const float g = quant_tensor_scale(partial, n_partial, tensor_scale, scale_given);
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

// Stages rows [0, nrows) of a tile into shared memory (row r from
// src + r * src_stride elements, row_bytes each, 16-byte aligned), one bulk
// copy per row spread over all threads, and zero-fills rows [nvalid, nrows).
// Every thread returns once the copies have landed; false if the wait timed
// out (device status set, the copies given a last bounded wait).
__device__ __forceinline__ bool stage_tile_rows(uint4* dst, const uint16_t* src,
                                                int64_t src_stride, int nvalid, int nrows,
                                                int row_bytes, uint64_t* bar) {
  const int row16 = row_bytes / 16;
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
    mbar_arrive_expect_tx(bar, (uint32_t)(nvalid * row_bytes));
  }
  for (int i = nvalid * row16 + threadIdx.x; i < nrows * row16; i += blockDim.x)
    dst[i] = make_uint4(0, 0, 0, 0);
  __syncthreads();
  for (int r = threadIdx.x; r < nvalid; r += blockDim.x)
    bulk_g2s(dst + r * row16, src + r * src_stride, (uint32_t)row_bytes, bar);
  int never = 0;
  if (mbar_wait(bar, 0, &never)) return true;
  int again = 0;
  mbar_wait(bar, 0, &again, 200000000ull);
  return false;
}

// Q or K ([total, nh, d] 16-bit) -> per (sequence, head, tile) images, one
// CTA per tile of tile_rows rows:
//   img4:  codes [tile_rows, d/2] swizzled (pitch d/2), then scale factors;
//   img16: the unrotated 16-bit rows, d/64 regions of [tile_rows, 128 B]
//          with 128-byte swizzle.
// Rows past the sequence end are written as zeros.  When means is given, the
// CTA also writes the fp64 means [nseq, nh, nB, d] of the blk-row blocks in
// its tile (ThriftAttention, Metodologia step 1): the unrotated values summed
// in row order from the block start, divided by the row count.  The tile is
// read from HBM once, one bulk copy per row, into shared memory.  G = d/16.
//
// K smoothing (optional): with mu and without corr (K) the row's channel
// means mu [nseq, nh, D] are subtracted (fp32) before the NVFP4 quantisation;
// the 16-bit image and the block means keep the raw values.  With mu and
// corr (Q) the rows are quantised as usual and corr [nseq, nh, ntiles *
// tile_rows] receives q^ . mu of the row's kv head (head / mu_group), the
// dequantised NVFP4 row against the means (fp32).
template <int DT, int G, bool HAD, bool SS>
__global__ void __launch_bounds__(256) qk_tile_kernel(
    const uint16_t* __restrict__ x, SeqInfo seqs, int nh, int tile_rows, int ntiles, int blk,
    int nB, const uint32_t* amax_in, uint8_t* __restrict__ img4, uint8_t* __restrict__ img16,
    double* __restrict__ means, const float* __restrict__ mu, int mu_group,
    float* __restrict__ corr) {
  constexpr int D = G * 16;
  extern __shared__ uint4 tsm[];  // [tile_rows][D] 16-bit values
  __shared__ __align__(8) uint64_t s_bar;
  const int tile = blockIdx.x, head = blockIdx.y, seq = blockIdx.z;
  int64_t start;
  int len;
  seqs.get(seq, start, len);
  const int t0 = tile * tile_rows;
  if (t0 >= len) return;
  if (!stage_tile_rows(tsm, x + ((start + t0) * nh + head) * D, (int64_t)nh * D,
                       min(tile_rows, len - t0), tile_rows, D * 2, &s_bar))
    return;
  const float g = tensor_scale_from_amax(*amax_in);
  const uint32_t t4 = fp4_tile_bytes(tile_rows, D), t16 = f16_tile_bytes(tile_rows, D);
  const int64_t tidx = ((int64_t)seq * nh + head) * ntiles + tile;
  uint8_t* t4p = img4 + tidx * t4;
  uint8_t* t16p = img16 + tidx * t16;
  uint8_t* sf = t4p + (uint32_t)tile_rows * (D / 2);
  // one 16-element block per thread and step; the G blocks of a row sit in
  // G consecutive lanes (the Hadamard exchanges between them)
  for (int i = threadIdx.x; i < tile_rows * G; i += blockDim.x) {
    const int r = i / G, kb = i % G;
    const uint4 raw0 = tsm[(r * D + kb * 16) / 8], raw1 = tsm[(r * D + kb * 16) / 8 + 1];
    float v[16];
    const uint32_t w[8] = {raw0.x, raw0.y, raw0.z, raw0.w, raw1.x, raw1.y, raw1.z, raw1.w};
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      v[2 * e] = h2f<DT>((uint16_t)(w[e] & 0xFFFF));
      v[2 * e + 1] = h2f<DT>((uint16_t)(w[e] >> 16));
    }
    const float* mrow = mu ? mu + ((int64_t)seq * (nh / mu_group) + head / mu_group) * D + kb * 16
                           : nullptr;
    if (mrow && !corr) {
#pragma unroll
      for (int e = 0; e < 16; ++e) v[e] = __fsub_rn(v[e], __ldg(mrow + e));
    }
    if constexpr (HAD) fwht_rows16<G>(v);
    uint32_t lo, hi;
    const uint32_t S = quant_block16(v, g, SS, lo, hi);
    if (mrow && corr) {
      // q^ . mu over the row: this block's part, then the G lanes of the row
      float part = 0.0f;
      const uint32_t cw[2] = {lo, hi};
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        float c0, c1;
        e2m1x2_values((cw[e / 4] >> (8 * (e % 4))) & 0xFFu, c0, c1);
        part = fmaf(c0, __ldg(mrow + 2 * e), part);
        part = fmaf(c1, __ldg(mrow + 2 * e + 1), part);
      }
      part *= ue4m3_decode(S) * g;
#pragma unroll
      for (int o = 1; o < G; o <<= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
      if (kb == 0) corr[((int64_t)seq * nh + head) * ((int64_t)ntiles * tile_rows) + t0 + r] = part;
    }
    *reinterpret_cast<uint2*>(t4p + swz_offset(r, kb * 8, D / 2)) = make_uint2(lo, hi);
    sf[sf_offset(r, kb)] = (uint8_t)S;
    if (tile_rows == 64) sf[sf_offset(r + 64, kb)] = 0;
    const uint32_t e0 = kb * 16;
    uint8_t* reg = t16p + (e0 / 64) * ((uint32_t)tile_rows * 128);
    *reinterpret_cast<uint4*>(reg + swz_offset(r, (e0 % 64) * 2, 128)) = raw0;
    *reinterpret_cast<uint4*>(reg + swz_offset(r, (e0 % 64) * 2 + 16, 128)) = raw1;
  }
  if (means != nullptr) {
    const uint16_t* tv = reinterpret_cast<const uint16_t*>(tsm);
    const int nbt = tile_rows / blk;  // selection blocks in this tile
    for (int e = threadIdx.x; e < nbt * D; e += blockDim.x) {
      const int c = e % D, bi = e / D;
      const int b0 = t0 + bi * blk;
      if (b0 >= len) continue;
      const int b1 = min(len, b0 + blk);
      double sum = 0.0;
      for (int t = b0; t < b1; ++t) sum = __dadd_rn(sum, (double)h2f<DT>(tv[(t - t0) * D + c]));
      means[(((int64_t)seq * nh + head) * nB + tile * nbt + bi) * D + c] =
          __ddiv_rn(sum, (double)(b1 - b0));
    }
  }
}

// K smoothing statistics: per (sequence, kv head, 128-token block, channel)
// the fp64 sum of the block's values in token order, their fp32 minimum and
// maximum.  One CTA per (block, kv head, sequence), one thread per channel.
template <int DT>
__global__ void __launch_bounds__(128) k_stats_kernel(const uint16_t* __restrict__ k,
                                                      SeqInfo seqs, int Hkv, int d, int nb128,
                                                      double* __restrict__ sums,
                                                      float* __restrict__ mins,
                                                      float* __restrict__ maxs) {
  const int b = blockIdx.x, hk = blockIdx.y, seq = blockIdx.z;
  int64_t start;
  int len;
  seqs.get(seq, start, len);
  const int t0 = b * 128, t1 = min(len, t0 + 128);
  const int64_t o = (((int64_t)seq * Hkv + hk) * nb128 + b) * d;
  for (int c = threadIdx.x; c < d; c += blockDim.x) {
    double sum = 0.0;
    float mn = INFINITY, mx = -INFINITY;
#pragma unroll 8
    for (int t = t0; t < t1; ++t) {
      const float xv = h2f<DT>(__ldg(k + ((start + t) * Hkv + hk) * d + c));
      sum = __dadd_rn(sum, (double)xv);
      mn = fminf(mn, xv);
      mx = fmaxf(mx, xv);
    }
    sums[o + c] = sum;
    mins[o + c] = mn;
    maxs[o + c] = mx;
  }
}

// mu [nseq, Hkv, d] = the block sums added in block order / length, rounded
// to fp32; and the absmax of K - mu folded into *amax_k: over the blocks,
// max(fl(max - mu), fl(mu - min)) (fp32 subtraction is monotone, so this is
// the largest |fl(k - mu)| of the block).  One CTA per (kv head, sequence).
__global__ void __launch_bounds__(128) k_mean_kernel(const double* __restrict__ sums,
                                                     const float* __restrict__ mins,
                                                     const float* __restrict__ maxs,
                                                     SeqInfo seqs, int Hkv, int d, int nb128,
                                                     float* __restrict__ mu,
                                                     uint32_t* __restrict__ amax_k) {
  const int hk = blockIdx.x, seq = blockIdx.y;
  int64_t start;
  int len;
  seqs.get(seq, start, len);
  const int nb = (int)ceil_div(len, 128);
  float a = 0.0f;
  for (int c = threadIdx.x; c < d; c += blockDim.x) {
    const int64_t o = ((int64_t)seq * Hkv + hk) * nb128 * d + c;
    double tot = 0.0;
    for (int b = 0; b < nb; ++b) tot = __dadd_rn(tot, sums[o + (int64_t)b * d]);
    const float m = len > 0 ? (float)__ddiv_rn(tot, (double)len) : 0.0f;
    mu[((int64_t)seq * Hkv + hk) * d + c] = m;
    for (int b = 0; b < nb; ++b)
      a = fmaxf(a, fmaxf(__fsub_rn(maxs[o + (int64_t)b * d], m), __fsub_rn(m, mins[o + (int64_t)b * d])));
  }
  cta_atomic_amax(a, amax_k);
}

// V ([total, Hkv, d] 16-bit) -> per (sequence, kv head, key tile) images with
// 16-blocks along tokens, one CTA per key tile: img4 codes [d, blk/2]
// swizzled (pitch blk/2) then scale factors (rows = channels); img16 = V^T
// tile [d, blk] in blk/64 regions of [d, 128 B] with 128-byte swizzle.  Keys
// past the sequence end are zeros.  The tile is read once, one bulk copy per
// row, into shared memory; each thread then takes one (channel, 16-key)
// column block from there.
template <int DT, bool SS>
__global__ void __launch_bounds__(256) v_tile_kernel(
    const uint16_t* __restrict__ v, SeqInfo seqs, int Hkv, int d, int blk, int ntiles,
    const uint32_t* amax_in, uint8_t* __restrict__ img4, uint8_t* __restrict__ img16) {
  extern __shared__ uint4 tsm[];  // [blk][d] 16-bit values
  __shared__ __align__(8) uint64_t s_bar;
  const int j = blockIdx.x, hk = blockIdx.y, seq = blockIdx.z;
  int64_t start;
  int len;
  seqs.get(seq, start, len);
  const int t0 = j * blk;
  if (t0 >= len) return;
  if (!stage_tile_rows(tsm, v + ((start + t0) * Hkv + hk) * d, (int64_t)Hkv * d,
                       min(blk, len - t0), blk, d * 2, &s_bar))
    return;
  const float g = tensor_scale_from_amax(*amax_in);
  const uint32_t t4 = fp4_tile_bytes(d, blk), t16 = f16_tile_bytes(d, blk);
  const int64_t tidx = ((int64_t)seq * Hkv + hk) * ntiles + j;
  // the two output images are assembled in shared memory (transposed rows
  // would make scattered global stores) and leave by two bulk copies
  uint8_t* o4 = reinterpret_cast<uint8_t*>(tsm) + (size_t)blk * d * 2;
  uint8_t* o16 = o4 + ((t4 + 127) & ~127u);
  uint8_t* sf = o4 + (uint32_t)d * (blk / 2);
  const uint16_t* tv = reinterpret_cast<const uint16_t*>(tsm);
  for (int i = threadIdx.x; i < d * (blk / 16); i += blockDim.x) {
    const int c = i % d, kb = (i / d) * 16;
    float val[16];
    uint16_t raw[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      raw[e] = tv[(kb + e) * d + c];
      val[e] = h2f<DT>(raw[e]);
    }
    uint32_t lo, hi;
    const uint32_t S = quant_block16(val, g, SS, lo, hi);
    *reinterpret_cast<uint2*>(o4 + swz_offset(c, kb / 2, blk / 2)) = make_uint2(lo, hi);
    sf[sf_offset(c, kb / 16)] = (uint8_t)S;
    if (d == 64) sf[sf_offset(c + 64, kb / 16)] = 0;
    uint8_t* reg = o16 + (kb / 64) * ((uint32_t)d * 128);
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
  fence_proxy_async_smem();
  __syncthreads();
  if (threadIdx.x == 0) {
    bulk_s2g(img4 + tidx * t4, o4, t4);
    bulk_s2g(img16 + tidx * t16, o16, t16);
    bulk_commit_and_wait_read();
  }
}

}  // namespace thrift
