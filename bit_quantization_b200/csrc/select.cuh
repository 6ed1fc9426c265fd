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
#include <cooperative_groups.h>

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

// scores [nseq, H, nB, nB] fp64 (valid i, j < nb of the sequence only;
// causal: j <= i).  One CTA per (sequence, head, 32 x 32 tile of pairs);
// each thread holds a 2 x 2 block of scores in registers, every score a
// sequential fma over the channels in order.  The means pass through shared
// memory 32 channels at a time, channel-major.  nB <= 512.
constexpr int kPairTile = 32, kPairChunk = 32, kPairSub = kPairTile / 16;

__global__ void __launch_bounds__(256) pair_scores_kernel(const double* __restrict__ qm,
                                                          const double* __restrict__ km,
                                                          SeqInfo seqs, int nseq, int H,
                                                          int Hkv, int d, int blk, int nB,
                                                          int causal,
                                                          double* __restrict__ scores) {
  __shared__ double qs[kPairChunk][kPairTile + 1];
  __shared__ double ks[kPairChunk][kPairTile + 1];
  const int T = (nB + kPairTile - 1) / kPairTile;
  const int tile = blockIdx.x % (T * T);
  const int h = (blockIdx.x / (T * T)) % H;
  const int seq = blockIdx.x / (T * T * H);
  const int i0 = (tile / T) * kPairTile, j0 = (tile % T) * kPairTile;
  int64_t start;
  int len;
  seqs.get(seq, start, len);
  const int nb = (int)ceil_div(len, blk);
  if (i0 >= nb || j0 >= nb || (causal && j0 > i0 + kPairTile - 1)) return;
  const int hk = h / (H / Hkv);
  const double* qrow = qm + ((int64_t)seq * H + h) * nB * d;
  const double* krow = km + ((int64_t)seq * Hkv + hk) * nB * d;
  const int ti = threadIdx.x >> 4, tj = threadIdx.x & 15;
  double acc[kPairSub][kPairSub];
#pragma unroll
  for (int a = 0; a < kPairSub; ++a)
#pragma unroll
    for (int b = 0; b < kPairSub; ++b) acc[a][b] = 0.0;
  for (int c0 = 0; c0 < d; c0 += kPairChunk) {
    __syncthreads();
    // rows i0.. / j0.. of the means, 32 channels each, transposed into
    // shared memory (consecutive threads read consecutive channels)
    for (int e = threadIdx.x; e < kPairTile * kPairChunk; e += blockDim.x) {
      const int r = e / kPairChunk, c = e % kPairChunk;
      qs[c][r] = (i0 + r < nb) ? __ldg(qrow + (int64_t)(i0 + r) * d + c0 + c) : 0.0;
      ks[c][r] = (j0 + r < nb) ? __ldg(krow + (int64_t)(j0 + r) * d + c0 + c) : 0.0;
    }
    __syncthreads();
#pragma unroll 8
    for (int c = 0; c < kPairChunk; ++c) {
      double qv[kPairSub], kv[kPairSub];
#pragma unroll
      for (int a = 0; a < kPairSub; ++a) qv[a] = qs[c][kPairSub * ti + a];
#pragma unroll
      for (int b = 0; b < kPairSub; ++b) kv[b] = ks[c][tj + 16 * b];
#pragma unroll
      for (int a = 0; a < kPairSub; ++a)
#pragma unroll
        for (int b = 0; b < kPairSub; ++b) acc[a][b] = __fma_rn(qv[a], kv[b], acc[a][b]);
    }
  }
  double* out = scores + ((int64_t)seq * H + h) * nB * nB;
#pragma unroll
  for (int a = 0; a < kPairSub; ++a) {
    const int i = i0 + kPairSub * ti + a;
    if (i >= nb) continue;
#pragma unroll
    for (int b = 0; b < kPairSub; ++b) {
      const int j = j0 + tj + 16 * b;
      if (j < nb) out[(int64_t)i * nB + j] = acc[a][b];
    }
  }
}

inline size_t pair_scores_smem(int) { return 0; }

inline int pair_scores_grid(int nseq, int H, int nB) {
  const int T = (nB + kPairTile - 1) / kPairTile;
  return nseq * H * T * T;
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

// Largest digit whose count, accumulated from digit 255 downwards, reaches
// rem; returns it and the count strictly above it.  Warp 0 only: lane l takes
// digits 255 - 8l ... 248 - 8l.
__device__ __forceinline__ int select_digit(const int* hist, int64_t rem, int64_t* above) {
  const int lane = threadIdx.x & 31;
  int c[8];
  int sum = 0;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    c[e] = hist[255 - 8 * lane - e];
    sum += c[e];
  }
  int incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  const unsigned hit = __ballot_sync(0xffffffffu, (int64_t)incl >= rem);
  const int src = hit ? __ffs(hit) - 1 : 31;
  int64_t cum = (int64_t)(incl - sum);  // count above this lane's digits
  int sel = 0;
  if (lane == src) {
    sel = 255 - 8 * lane - 7;
    for (int e = 0; e < 8; ++e) {
      if (cum + c[e] >= rem) {
        sel = 255 - 8 * lane - e;
        break;
      }
      cum += c[e];
    }
  }
  sel = __shfl_sync(0xffffffffu, sel, src);
  cum = __shfl_sync(0xffffffffu, cum, src);
  *above = cum;
  return sel;
}

// Exact top-k of one CTA over n entries by a radix select on the 64-bit
// order keys (up to 8 passes of 8 bits, most significant first), then ties
// at the threshold taken in ascending index.  The select stops early once
// the threshold digit's bucket holds exactly the entries still wanted: all
// of them are taken, so the lower bits cannot change the result.
// out[i] = 1 for the k largest valid entries and for every valid entry that
// `fixed` names, else 0 (every out[i], i < n, is written).  The keys are read
// once into `kcache` when it is given (n entries).  All threads of the CTA
// call it.
struct TopkShared {
  int hist[256];
  int warp_sums[32];
  int total;
  int done;
  uint64_t prefix;
  int64_t remaining;
};

template <class Valid, class Fixed, class Score>
__device__ void radix_topk(int64_t n, int64_t k, int64_t n_valid, Valid valid, Fixed fixed,
                           Score score, uint64_t* kcache, TopkShared& sh,
                           uint8_t* __restrict__ out) {
  if (k == 0 || k == n_valid) {
    for (int64_t i = threadIdx.x; i < n; i += blockDim.x)
      out[i] = (valid(i) && (k != 0 || fixed(i))) ? 1 : 0;
    return;
  }
  if (kcache) {
    for (int64_t i = threadIdx.x; i < n; i += blockDim.x)
      kcache[i] = valid(i) ? order_key(score(i)) : 0ull;
  }
  auto key_of = [&](int64_t i) { return kcache ? kcache[i] : order_key(score(i)); };
  // keys of kU consecutive strides per thread, loaded before any is used (an
  // invalid or out-of-range entry reads as 0 with ok = false)
  constexpr int kU = 4;
  auto load_keys = [&](int64_t base, uint64_t (&key)[kU], bool (&ok)[kU]) {
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int64_t i = base + (int64_t)u * blockDim.x + threadIdx.x;
      ok[u] = i < n && valid(i);
      key[u] = ok[u] ? key_of(i) : 0ull;
    }
  };
  uint64_t prefix = 0, pmask = 0;
  int64_t rem = k;
  bool whole_bucket = false;  // the threshold bucket is taken whole
  for (int pass = 0; pass < 8; ++pass) {
    const int shift = 56 - 8 * pass;
    for (int i = threadIdx.x; i < 256; i += blockDim.x) sh.hist[i] = 0;
    __syncthreads();
    // keys sharing a digit in a warp add to its bin once (the leading
    // digits of nearby scores coincide, and same-address shared atomics
    // serialise)
    for (int64_t base = 0; base < n; base += (int64_t)kU * blockDim.x) {
      uint64_t key[kU];
      bool ok[kU];
      load_keys(base, key, ok);
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int digit =
            (ok[u] && (key[u] & pmask) == prefix) ? (int)((key[u] >> shift) & 255) : -1;
        const unsigned same = __match_any_sync(0xffffffffu, digit);
        if (digit >= 0 && (threadIdx.x & 31) == __ffs(same) - 1)
          atomicAdd(&sh.hist[digit], __popc(same));
      }
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      int64_t above;
      const int sel = select_digit(sh.hist, rem, &above);
      if (threadIdx.x == 0) {
        sh.remaining = rem - above;
        sh.prefix = prefix | ((uint64_t)sel << shift);
        sh.done = (int64_t)sh.hist[sel] == rem - above;
      }
    }
    __syncthreads();
    prefix = sh.prefix;
    rem = sh.remaining;
    pmask |= (uint64_t)255 << shift;
    whole_bucket = sh.done != 0;
    __syncthreads();  // sh.done is rewritten by the next pass
    if (whole_bucket) break;  // uniform: every thread read the same word
  }
  // compare on the decided bits only (all of them unless the select stopped
  // early, when every key of the threshold bucket is taken)
  const uint64_t T = prefix;
  if (whole_bucket) {
    // every key at the threshold is taken: no order among them to keep
    for (int64_t base = 0; base < n; base += (int64_t)kU * blockDim.x) {
      uint64_t key[kU];
      bool ok[kU];
      load_keys(base, key, ok);
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int64_t i = base + (int64_t)u * blockDim.x + threadIdx.x;
        if (i < n) out[i] = (ok[u] && ((key[u] & pmask) >= T || fixed(i))) ? 1 : 0;
      }
    }
    return;
  }
  const int64_t take_eq = rem;
  int64_t taken = 0;
  for (int64_t base = 0; base < n; base += blockDim.x) {
    const int64_t i = base + threadIdx.x;
    uint64_t key = 0;
    bool ok = false;
    if (i < n && valid(i)) {
      key = key_of(i) & pmask;
      ok = true;
    }
    const int eq = (ok && key == T) ? 1 : 0;
    const int before = block_exclusive_scan(eq, sh.warp_sums, &sh.total);
    if (i < n) out[i] = (ok && (key > T || (eq && taken + before < take_eq) || fixed(i))) ? 1 : 0;
    taken += sh.total;
    __syncthreads();
  }
}

// One CTA per (sequence, head) of the pair selection.  mask [nseq, H, nB, nB]
// uint8 (1 = FP16 pair); every entry is written.  The keys are cached in
// shared memory when they fit (kTopkCache).
constexpr int kTopkCache = 4096;  // 32 KB of keys: within the default shared-memory limit

__global__ void __launch_bounds__(kTopkThreads) topk_kernel(const double* __restrict__ scores,
                                                            SeqInfo seqs, int H, int blk, int nB,
                                                            int causal, float frac, int sink,
                                                            int recent,
                                                            uint8_t* __restrict__ mask) {
  __shared__ TopkShared sh;
  extern __shared__ uint64_t kcache[];
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
  // pair indices fit 32 bits (nB <= 512): a 32-bit division, not the
  // software-emulated 64-bit one
  auto valid = [&](int64_t lin) {
    const int l = (int)lin, i = l / nB, j = l - i * nB;
    return i < nb && j < nb && (!causal || j <= i);
  };
  // ScaleSearchAttention's sink-aware pairs, added to the top-k ones: the
  // first `sink` key blocks and the `recent` newest ones query block i sees
  auto fixed = [&](int64_t lin) {
    const int l = (int)lin, i = l / nB, j = l - i * nB;
    return j < sink || (causal ? (j > i - recent) : (j >= nb - recent));
  };
  auto score = [&](int64_t lin) { return sc[lin]; };
  radix_topk(npairs, k, n_valid, valid, fixed, score, npairs <= kTopkCache ? kcache : nullptr,
             sh, mk);
}

inline size_t topk_smem(int nB) {
  const int64_t np = (int64_t)nB * nB;
  return np <= kTopkCache ? (size_t)np * 8 : 0;
}

// ---------------------------------------------- top-k over a CTA cluster --
// The same exact selection as radix_topk with the n entries split into
// kTopkCluster contiguous index ranges, one per CTA of a cluster; each CTA
// caches its range's keys in shared memory when they fit.  Per pass every
// CTA counts its range, rank 0 adds the histograms (distributed shared
// memory) and decides the digit, and every CTA reads the decision back.
// Ties at the threshold keep ascending index order across the ranges: each
// CTA's count of threshold keys, summed over the lower ranks, starts its
// scan.  All CTAs of the cluster call it with the same n, k, n_valid.
constexpr int kTopkCluster = 4;
constexpr int kTopkClusterCacheBytes = 192 * 1024;

struct TopkClusterShared {
  int hist[256];
  int warp_sums[32];
  int total;
  int done;
  uint64_t prefix;
  int64_t remaining;
  unsigned long long eq_count;  // this CTA's keys at the threshold
};

template <class Valid, class Fixed, class Score>
__device__ void radix_topk_cluster(int64_t n, int64_t k, int64_t n_valid, Valid valid,
                                   Fixed fixed, Score score, uint64_t* kcache,
                                   TopkClusterShared& sh, uint8_t* __restrict__ out) {
  namespace cgx = cooperative_groups;
  cgx::cluster_group cl = cgx::this_cluster();
  const int rank = (int)cl.block_rank();
  const int64_t per = (n + kTopkCluster - 1) / kTopkCluster;
  const int64_t lo = min(n, (int64_t)rank * per), hi = min(n, lo + per);
  if (k == 0 || k == n_valid) {
    for (int64_t i = lo + threadIdx.x; i < hi; i += blockDim.x)
      out[i] = (valid(i) && (k != 0 || fixed(i))) ? 1 : 0;
    return;
  }
  if (kcache) {
    for (int64_t i = lo + threadIdx.x; i < hi; i += blockDim.x)
      kcache[i - lo] = valid(i) ? order_key(score(i)) : 0ull;
    __syncthreads();
  }
  auto key_of = [&](int64_t i) { return kcache ? kcache[i - lo] : order_key(score(i)); };
  constexpr int kU = 4;
  auto load_keys = [&](int64_t base, uint64_t (&key)[kU], bool (&ok)[kU]) {
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int64_t i = base + (int64_t)u * blockDim.x + threadIdx.x;
      ok[u] = i < hi && valid(i);
      key[u] = ok[u] ? key_of(i) : 0ull;
    }
  };
  TopkClusterShared* s0 = cl.map_shared_rank(&sh, 0);
  uint64_t prefix = 0, pmask = 0;
  int64_t rem = k;
  bool whole_bucket = false;
  for (int pass = 0; pass < 8; ++pass) {
    const int shift = 56 - 8 * pass;
    for (int i = threadIdx.x; i < 256; i += blockDim.x) sh.hist[i] = 0;
    __syncthreads();
    for (int64_t base = lo; base < hi; base += (int64_t)kU * blockDim.x) {
      uint64_t key[kU];
      bool ok[kU];
      load_keys(base, key, ok);
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int digit =
            (ok[u] && (key[u] & pmask) == prefix) ? (int)((key[u] >> shift) & 255) : -1;
        const unsigned same = __match_any_sync(0xffffffffu, digit);
        if (digit >= 0 && (threadIdx.x & 31) == __ffs(same) - 1)
          atomicAdd(&sh.hist[digit], __popc(same));
      }
    }
    cl.sync();  // every range counted
    if (rank == 0) {
      for (int b = threadIdx.x; b < 256; b += blockDim.x) {
        int t = sh.hist[b];
#pragma unroll
        for (int r = 1; r < kTopkCluster; ++r) t += cl.map_shared_rank(sh.hist, r)[b];
        sh.hist[b] = t;
      }
      __syncthreads();
      if (threadIdx.x < 32) {
        int64_t above;
        const int sel = select_digit(sh.hist, rem, &above);
        if (threadIdx.x == 0) {
          sh.remaining = rem - above;
          sh.prefix = prefix | ((uint64_t)sel << shift);
          sh.done = (int64_t)sh.hist[sel] == rem - above;
        }
      }
    }
    cl.sync();  // the decision is published
    prefix = s0->prefix;
    rem = s0->remaining;
    whole_bucket = s0->done != 0;
    pmask |= (uint64_t)255 << shift;
    cl.sync();  // read before rank 0 decides again (or leaves)
    if (whole_bucket) break;  // uniform across the cluster
  }
  const uint64_t T = prefix;
  if (whole_bucket) {
    for (int64_t base = lo; base < hi; base += (int64_t)kU * blockDim.x) {
      uint64_t key[kU];
      bool ok[kU];
      load_keys(base, key, ok);
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int64_t i = base + (int64_t)u * blockDim.x + threadIdx.x;
        if (i < hi) out[i] = (ok[u] && ((key[u] & pmask) >= T || fixed(i))) ? 1 : 0;
      }
    }
    return;
  }
  // ties: this range's threshold keys, then the lower ranks' counts
  if (threadIdx.x == 0) sh.eq_count = 0;
  __syncthreads();
  {
    unsigned long long cnt = 0;
    for (int64_t i = lo + threadIdx.x; i < hi; i += blockDim.x)
      if (valid(i) && (key_of(i) & pmask) == T) ++cnt;
    if (cnt) atomicAdd(&sh.eq_count, cnt);
  }
  cl.sync();
  int64_t taken = 0;
  for (int r = 0; r < rank; ++r) taken += (int64_t)cl.map_shared_rank(&sh, r)->eq_count;
  const int64_t take_eq = rem;
  for (int64_t base = lo; base < hi; base += blockDim.x) {
    const int64_t i = base + threadIdx.x;
    uint64_t key = 0;
    bool ok = false;
    if (i < hi && valid(i)) {
      key = key_of(i) & pmask;
      ok = true;
    }
    const int eq = (ok && key == T) ? 1 : 0;
    const int before = block_exclusive_scan(eq, sh.warp_sums, &sh.total);
    if (i < hi) out[i] = (ok && (key > T || (eq && taken + before < take_eq) || fixed(i))) ? 1 : 0;
    taken += sh.total;
    __syncthreads();
  }
  cl.sync();  // no CTA leaves while another may still read its counts
}

// topk_kernel's work over a cluster of kTopkCluster CTAs per (sequence,
// head): grid nseq * H * kTopkCluster; dynamic shared memory holds a range's
// keys when topk_cluster_smem(nB) is nonzero.
__global__ void __cluster_dims__(kTopkCluster, 1, 1) __launch_bounds__(kTopkThreads)
    topk_cluster_kernel(const double* __restrict__ scores, SeqInfo seqs, int H, int blk, int nB,
                        int causal, float frac, int sink, int recent,
                        uint8_t* __restrict__ mask, int use_cache) {
  __shared__ TopkClusterShared sh;
  extern __shared__ uint64_t kcache[];
  const int head = blockIdx.x / kTopkCluster;
  const int seq = head / H, h = head % H;
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
    const int l = (int)lin, i = l / nB, j = l - i * nB;
    return i < nb && j < nb && (!causal || j <= i);
  };
  auto fixed = [&](int64_t lin) {
    const int l = (int)lin, i = l / nB, j = l - i * nB;
    return j < sink || (causal ? (j > i - recent) : (j >= nb - recent));
  };
  auto score = [&](int64_t lin) { return sc[lin]; };
  radix_topk_cluster(npairs, k, n_valid, valid, fixed, score, use_cache ? kcache : nullptr, sh,
                     mk);
}

// Shared memory of a range's key cache (0: the keys are read from global
// memory in every pass).
inline size_t topk_cluster_smem(int nB) {
  const int64_t per = ((int64_t)nB * nB + kTopkCluster - 1) / kTopkCluster;
  return per * 8 <= kTopkClusterCacheBytes ? (size_t)per * 8 : 0;
}

}  // namespace thrift
