// Block selection (ThriftAttention, Metodologia step 1): block means of Q
// and K, block-pair scores S^_ij = qbar_i . kbar_j, and the top-k pairs per
// (sequence, head) that run on the FP16 path.
//
// Arithmetic, reproducible bit for bit: block sums in fp64 in token order
// from 0, divided by the token count; scores by a sequential fp64 fma over
// the channels; k = ceil(frac * n_valid - 1e-9) clamped to [0, n_valid] over
// the valid pairs (causal: j <= i); ties between equal scores go to the lower
// linear index i * nB + j.
#pragma once
#include "quant_kernels.cuh"

namespace thrift {

// means [nseq, nh, nB, d] fp64 of x [total, nh, d]; one thread per
// (sequence, head, block, channel), channels fastest.  The sum runs in token
// order; loads are issued eight tokens ahead of the additions.
template <int DT>
__global__ void __launch_bounds__(256) block_means_kernel(const uint16_t* __restrict__ x,
                                                          SeqInfo seqs, int nseq, int nh, int d,
                                                          int blk, int nB,
                                                          double* __restrict__ means) {
  const int64_t n = (int64_t)nseq * nh * nB * d;
  for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < n;
       idx += (int64_t)gridDim.x * blockDim.x) {
    const int c = (int)(idx % d);
    const int i = (int)((idx / d) % nB);
    const int head = (int)((idx / ((int64_t)d * nB)) % nh);
    const int seq = (int)(idx / ((int64_t)d * nB * nh));
    int64_t start;
    int len;
    seqs.get(seq, start, len);
    const int t0 = i * blk;
    if (t0 >= len) continue;
    const int t1 = min(len, t0 + blk);
    const uint16_t* px = x + ((start + t0) * nh + head) * d + c;
    const int64_t stride = (int64_t)nh * d;
    double sum = 0.0;
    int t = t0;
    for (; t + 8 <= t1; t += 8) {
      uint16_t v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = __ldg(px + (int64_t)(t - t0 + u) * stride);
#pragma unroll
      for (int u = 0; u < 8; ++u) sum = __dadd_rn(sum, (double)h2f<DT>(v[u]));
    }
    for (; t < t1; ++t) sum = __dadd_rn(sum, (double)h2f<DT>(__ldg(px + (int64_t)(t - t0) * stride)));
    means[idx] = __ddiv_rn(sum, (double)(t1 - t0));
  }
}

// scores [nseq, H, nB, nB] fp64 (valid i, j < nb of the sequence only).
// One CTA per (sequence, head, 16 query blocks); the key means pass through
// shared memory transposed, 8 channels at a time, and every score keeps its
// sequential fma order over the channels.  nB <= 512.
constexpr int kScoreRows = 16, kScoreChunk = 8;

__global__ void __launch_bounds__(256) pair_scores_kernel(const double* __restrict__ qm,
                                                          const double* __restrict__ km,
                                                          SeqInfo seqs, int nseq, int H,
                                                          int Hkv, int d, int blk, int nB,
                                                          double* __restrict__ scores) {
  extern __shared__ double ssm[];
  double* qs = ssm;                                   // [kScoreRows][kScoreChunk]
  double* ks = ssm + kScoreRows * kScoreChunk;        // [kScoreChunk][nB]
  const int groups = (nB + kScoreRows - 1) / kScoreRows;
  const int ig = blockIdx.x % groups;
  const int h = (blockIdx.x / groups) % H;
  const int seq = blockIdx.x / (groups * H);
  int64_t start;
  int len;
  seqs.get(seq, start, len);
  const int nb = (int)ceil_div(len, blk);
  const int i0 = ig * kScoreRows;
  if (i0 >= nb) return;
  const int hk = h / (H / Hkv);
  const double* qrow = qm + (((int64_t)seq * H + h) * nB + i0) * d;
  const double* krow = km + ((int64_t)seq * Hkv + hk) * nB * d;
  double acc[kScoreRows][2];
#pragma unroll
  for (int a = 0; a < kScoreRows; ++a) acc[a][0] = acc[a][1] = 0.0;
  const int j0 = threadIdx.x, j1 = threadIdx.x + 256;
  for (int c0 = 0; c0 < d; c0 += kScoreChunk) {
    __syncthreads();
    for (int e = threadIdx.x; e < kScoreRows * kScoreChunk; e += blockDim.x) {
      const int a = e / kScoreChunk, cc = e % kScoreChunk;
      qs[e] = (i0 + a < nb) ? __ldg(qrow + (int64_t)a * d + c0 + cc) : 0.0;
    }
    for (int e = threadIdx.x; e < nb * kScoreChunk; e += blockDim.x) {
      const int j = e / kScoreChunk, cc = e % kScoreChunk;
      ks[cc * nB + j] = __ldg(krow + (int64_t)j * d + c0 + cc);
    }
    __syncthreads();
#pragma unroll
    for (int cc = 0; cc < kScoreChunk; ++cc) {
      const double k0 = j0 < nb ? ks[cc * nB + j0] : 0.0;
      const double k1 = j1 < nb ? ks[cc * nB + j1] : 0.0;
#pragma unroll
      for (int a = 0; a < kScoreRows; ++a) {
        const double q = qs[a * kScoreChunk + cc];
        acc[a][0] = __fma_rn(q, k0, acc[a][0]);
        acc[a][1] = __fma_rn(q, k1, acc[a][1]);
      }
    }
  }
  double* out = scores + (((int64_t)seq * H + h) * nB + i0) * nB;
#pragma unroll
  for (int a = 0; a < kScoreRows; ++a) {
    if (i0 + a >= nb) break;
    if (j0 < nb) out[(int64_t)a * nB + j0] = acc[a][0];
    if (j1 < nb) out[(int64_t)a * nB + j1] = acc[a][1];
  }
}

inline size_t pair_scores_smem(int nB) {
  return sizeof(double) * (kScoreRows * kScoreChunk + kScoreChunk * (size_t)nB);
}

inline int pair_scores_grid(int nseq, int H, int nB) {
  return nseq * H * ((nB + kScoreRows - 1) / kScoreRows);
}

// Order-preserving map of a double to an unsigned 64-bit key.
__device__ __forceinline__ uint64_t order_key(double s) {
  const uint64_t u = (uint64_t)__double_as_longlong(s);
  return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}

__device__ __forceinline__ int64_t topk_count_dev(float frac, int64_t n_valid) {
  double kk = ceil(__dsub_rn(__dmul_rn((double)frac, (double)n_valid), 1e-9));
  if (kk < 0.0) kk = 0.0;
  if (kk > (double)n_valid) kk = (double)n_valid;
  return (int64_t)kk;
}

constexpr int kTopkThreads = 1024;

// Block-wide exclusive prefix sum of one int per thread; returns the
// exclusive prefix and writes the total to *total.
__device__ __forceinline__ int block_exclusive_scan(int v, int* warp_sums, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = lane < (int)(blockDim.x >> 5) ? warp_sums[lane] : 0;
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += y;
    }
    warp_sums[lane] = wi - w;  // exclusive
    if (lane == 31) *total = wi;
  }
  __syncthreads();
  const int r = warp_sums[warp] + incl - v;
  __syncthreads();
  return r;
}

// One CTA per (sequence, head): exact top-k by an 8-pass radix select on the
// 64-bit keys, then ties at the threshold taken in ascending linear index.
// mask [nseq, H, nB, nB] uint8 (1 = FP16 pair); every entry is written.
__global__ void __launch_bounds__(kTopkThreads) topk_kernel(const double* __restrict__ scores,
                                                            SeqInfo seqs, int H, int blk, int nB,
                                                            int causal, float frac,
                                                            uint8_t* __restrict__ mask) {
  __shared__ int hist[256];
  __shared__ int warp_sums[32];
  __shared__ int s_total;
  __shared__ uint64_t s_prefix;
  __shared__ int64_t s_remaining;
  const int seq = blockIdx.x / H, h = blockIdx.x % H;
  int64_t start;
  int len;
  seqs.get(seq, start, len);
  const int nb = (int)ceil_div(len, blk);
  const int64_t npairs = (int64_t)nB * nB;
  const double* sc = scores + ((int64_t)seq * H + h) * npairs;
  uint8_t* mk = mask + ((int64_t)seq * H + h) * npairs;
  const int64_t n_valid = causal ? (int64_t)nb * (nb + 1) / 2 : (int64_t)nb * nb;
  const int64_t k = topk_count_dev(frac, n_valid);
  auto valid = [&](int64_t lin) {
    const int i = (int)(lin / nB), j = (int)(lin % nB);
    return i < nb && j < nb && (!causal || j <= i);
  };
  if (k == 0 || k == n_valid) {
    for (int64_t lin = threadIdx.x; lin < npairs; lin += blockDim.x)
      mk[lin] = (k != 0 && valid(lin)) ? 1 : 0;
    return;
  }
  uint64_t prefix = 0, pmask = 0;
  if (threadIdx.x == 0) s_remaining = k;
  for (int pass = 0; pass < 8; ++pass) {
    const int shift = 56 - 8 * pass;
    for (int i = threadIdx.x; i < 256; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    for (int64_t lin = threadIdx.x; lin < npairs; lin += blockDim.x) {
      if (!valid(lin)) continue;
      const uint64_t key = order_key(sc[lin]);
      if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & 255], 1);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      int64_t rem = s_remaining, cum = 0;
      int sel = 0;
      for (int dgt = 255; dgt >= 0; --dgt) {
        if (cum + hist[dgt] >= rem) {
          sel = dgt;
          break;
        }
        cum += hist[dgt];
      }
      s_remaining = rem - cum;
      s_prefix = prefix | ((uint64_t)sel << shift);
    }
    __syncthreads();
    prefix = s_prefix;
    pmask |= (uint64_t)255 << shift;
    __syncthreads();
  }
  const uint64_t T = prefix;
  const int64_t take_eq = s_remaining;
  int64_t taken = 0;
  for (int64_t base = 0; base < npairs; base += blockDim.x) {
    const int64_t lin = base + threadIdx.x;
    uint64_t key = 0;
    bool ok = false;
    if (lin < npairs && valid(lin)) {
      key = order_key(sc[lin]);
      ok = true;
    }
    const int eq = (ok && key == T) ? 1 : 0;
    const int before = block_exclusive_scan(eq, warp_sums, &s_total);
    if (lin < npairs) mk[lin] = (ok && (key > T || (eq && taken + before < take_eq))) ? 1 : 0;
    taken += s_total;
    __syncthreads();
  }
}

}  // namespace thrift
