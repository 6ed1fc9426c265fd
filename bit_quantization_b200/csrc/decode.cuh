// Decode over the double KV cache (ThriftAttention, Resultados: decode on the
// FP4 + FP16 cache; Significado: the cache grows by 28% because every token
// is kept in both formats).  One new query token per sequence attends to the
// tokens cached for it.
//
// The cache is caller-owned memory whose content this library defines: for
// every (sequence, kv head, key tile of 128 tokens) the K and V tiles in
// NVFP4 and in 16 bits, already in the operand layouts the tensor cores read
// (the same tile images the prefill path builds per call), and the fp64 means
// of the K tiles for the selection.  Appending tokens writes their rows and
// columns into those images, re-quantises the 16-token V blocks they touch
// (from the 16-bit V kept in the cache) and recomputes the touched K means.
//
// A decode step: the query tensor's absmax, the query images (NVFP4 and
// 16-bit) per kv head group, the block scores q . kbar_j and a top-k per
// (sequence, head), then the attention kernel (split over the key tiles,
// tensor cores with the key tile as the 128-row operand and the query group
// as the 16-column one), and a merge of the splits.
#pragma once

#include "attn.cuh"
#include "select.cuh"

namespace thrift {

// ------------------------------------------------------------ cache format --

constexpr int kDecTile = 128;  // tokens per key tile (= selection block)
constexpr int kDecD = 128;     // head dimension
constexpr int kDecMaxG = 16;   // query heads per kv head
constexpr int kDecN = 16;      // MMA N: query columns of the S and O buffers (>= kDecMaxG)

struct CacheGeom {
  int B, Hkv, ntc;  // key tiles per (sequence, kv head)
  static constexpr uint32_t K4 = fp4_tile_bytes(kDecTile, kDecD);   // codes + scale factors
  static constexpr uint32_t V4 = fp4_tile_bytes(kDecD, kDecTile);   // V^T: rows = channels
  static constexpr uint32_t K16 = f16_tile_bytes(kDecTile, kDecD);  // two 64-column regions
  static constexpr uint32_t V16 = f16_tile_bytes(kDecD, kDecTile);  // V^T, two 64-key regions
  static constexpr uint32_t MEANS = kDecD * 8;                      // fp64 means of the tile
  __host__ __device__ int64_t tiles() const { return (int64_t)B * Hkv * ntc; }
  __host__ __device__ int64_t off_v4() const { return tiles() * K4; }
  __host__ __device__ int64_t off_k16() const { return off_v4() + tiles() * V4; }
  __host__ __device__ int64_t off_v16() const { return off_k16() + tiles() * K16; }
  __host__ __device__ int64_t off_means() const { return off_v16() + tiles() * V16; }
  __host__ __device__ int64_t bytes() const { return off_means() + tiles() * MEANS; }
  __host__ __device__ int64_t tile(int b, int hk, int j) const {
    return ((int64_t)b * Hkv + hk) * ntc + j;
  }
};

// Byte offset of element (row, col) of a 16-bit tile image with 128 rows:
// 64-column regions of [128 rows, 128 B] with the 128-byte swizzle.
__device__ __forceinline__ uint32_t f16_img_off(uint32_t row, uint32_t col) {
  return (col >> 6) * (128u * 128u) + swz_offset(row, (col & 63u) * 2u, 128);
}

// ---------------------------------------------------------------- append --

// One CTA per appended token and kv head: the K row goes into the 16-bit and
// the NVFP4 K images (eight 16-blocks along d under g_K), the V row into the
// 16-bit V^T image as one column.  k_new, v_new [B, max_new, Hkv, 128].
template <int DT, bool SS>
__global__ void __launch_bounds__(kDecD) kv_append_kernel(
    const uint16_t* __restrict__ kn, const uint16_t* __restrict__ vn, CacheGeom cg, int max_new,
    int capacity, const int32_t* __restrict__ cache_len, const int32_t* __restrict__ n_new,
    const float* __restrict__ kv_scale, uint8_t* __restrict__ cache) {
  __shared__ __align__(16) uint16_t krow[kDecD];
  const int i = blockIdx.x, hk = blockIdx.y, b = blockIdx.z, c = threadIdx.x;
  const int n = min(__ldg(n_new + b), max_new);
  if (i >= n) return;
  const int t = __ldg(cache_len + b) + i;
  if (t < 0 || t >= capacity) return;
  const int j = t / kDecTile, kr = t % kDecTile;
  const int64_t src = (((int64_t)b * max_new + i) * cg.Hkv + hk) * kDecD;
  const uint16_t kval = __ldg(kn + src + c), vval = __ldg(vn + src + c);
  krow[c] = kval;
  const int64_t tl = cg.tile(b, hk, j);
  *reinterpret_cast<uint16_t*>(cache + cg.off_k16() + tl * CacheGeom::K16 + f16_img_off(kr, c)) =
      kval;
  *reinterpret_cast<uint16_t*>(cache + cg.off_v16() + tl * CacheGeom::V16 + f16_img_off(c, kr)) =
      vval;
  __syncthreads();
  if (c < kDecD / 16) {
    float v[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) v[e] = h2f<DT>(krow[16 * c + e]);
    uint32_t lo, hi;
    const uint32_t S = quant_block16(v, __ldg(kv_scale), SS, lo, hi);
    uint8_t* k4 = cache + tl * CacheGeom::K4;
    *reinterpret_cast<uint2*>(k4 + swz_offset(kr, c * 8, kDecD / 2)) = make_uint2(lo, hi);
    k4[kDecTile * (kDecD / 2) + sf_offset(kr, c)] = (uint8_t)S;
  }
}

// After the rows are in: CTAs [0, nv16) re-quantise the 16-token V blocks the
// appended tokens touch (one thread per channel, from the 16-bit V^T image,
// tokens not yet cached read as the zeros of the initial cache), CTAs from
// nv16 on recompute the fp64 means of the touched K tiles (the cached rows
// summed in order from the tile start, divided by their count).
template <int DT, bool SS>
__global__ void __launch_bounds__(kDecD) kv_requant_kernel(
    CacheGeom cg, int max_new, int capacity, const int32_t* __restrict__ cache_len,
    const int32_t* __restrict__ n_new, const float* __restrict__ kv_scale, int nv16,
    uint8_t* __restrict__ cache) {
  const int hk = blockIdx.y, b = blockIdx.z, c = threadIdx.x;
  const int from = __ldg(cache_len + b);
  const int to = min(capacity, from + min(__ldg(n_new + b), max_new));
  if (from < 0 || to <= from) return;
  if ((int)blockIdx.x < nv16) {
    const int vb = from / 16 + (int)blockIdx.x;  // 16-token block
    if (vb * 16 >= to) return;
    const int j = vb / (kDecTile / 16), kb = vb % (kDecTile / 16);
    const int64_t tl = cg.tile(b, hk, j);
    const uint8_t* v16 = cache + cg.off_v16() + tl * CacheGeom::V16;
    const uint32_t o0 = f16_img_off(c, 16 * kb), o1 = f16_img_off(c, 16 * kb + 8);
    const uint4 r0 = *reinterpret_cast<const uint4*>(v16 + o0);
    const uint4 r1 = *reinterpret_cast<const uint4*>(v16 + o1);
    float v[16];
    unpack16<DT>(r0, r1, v);
    uint32_t lo, hi;
    const uint32_t S = quant_block16(v, __ldg(kv_scale + 1), SS, lo, hi);
    uint8_t* v4 = cache + cg.off_v4() + tl * CacheGeom::V4;
    *reinterpret_cast<uint2*>(v4 + swz_offset(c, kb * 8, kDecTile / 2)) = make_uint2(lo, hi);
    v4[kDecD * (kDecTile / 2) + sf_offset(c, kb)] = (uint8_t)S;
  } else {
    const int j = from / kDecTile + ((int)blockIdx.x - nv16);
    if (j * kDecTile >= to) return;
    const int rows = min(kDecTile, to - j * kDecTile);
    const int64_t tl = cg.tile(b, hk, j);
    const uint8_t* k16 = cache + cg.off_k16() + tl * CacheGeom::K16;
    double sum = 0.0;
    for (int r = 0; r < rows; ++r)
      sum = __dadd_rn(sum, (double)h2f<DT>(*reinterpret_cast<const uint16_t*>(k16 + f16_img_off(r, c))));
    reinterpret_cast<double*>(cache + cg.off_means())[tl * kDecD + c] =
        __ddiv_rn(sum, (double)rows);
  }
}

// ---------------------------------------------------------- query images --

// Per (sequence, kv head): the G query rows of the group as B operands of
// 64 rows (rows >= G zero): NVFP4 codes [64, 64 B] with the 64-byte swizzle
// then the 128-row scale-factor image (1 KB), and the 16-bit rows in two
// 64-column regions of [64, 128 B] with the 128-byte swizzle.
constexpr uint32_t kDecQ4Bytes = 64 * (kDecD / 2) + (kDecD / 64) * 512;  // 5120
constexpr uint32_t kDecQ16Bytes = 64 * kDecD * 2;                        // 16384

// amax: the query tensor's absmax (bits of a non-negative float), read when
// self_amax == 0.  With self_amax != 0 every CTA reduces the whole query
// tensor itself (q_elems values; for small tensors, read from L2, which saves
// a launch) and CTA (0, 0) stores the result in *amax for the later kernels.
constexpr int64_t kDecQSelfAmaxMax = 32768;

template <int DT, bool SS>
__global__ void __launch_bounds__(128) dec_q_image_kernel(const uint16_t* __restrict__ q, int H,
                                                          int G, uint32_t* amax, int self_amax,
                                                          int64_t q_elems,
                                                          uint8_t* __restrict__ q4img,
                                                          uint8_t* __restrict__ q16img) {
  const int hk = blockIdx.x, b = blockIdx.y, Hkv = gridDim.x;
  float g;
  if (!self_amax) {
    g = tensor_scale_from_amax(*amax);
  } else {
    __shared__ float red[4];
    float a = 0.0f;
    const uint4* q8 = reinterpret_cast<const uint4*>(q);
    for (int64_t e = threadIdx.x; e < q_elems / 8; e += blockDim.x) {
      const uint4 r = __ldg(q8 + e);
      const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
      for (int k = 0; k < 4; ++k)
        a = fmaxf(a, fmaxf(fabsf(h2f<DT>((uint16_t)(w[k] & 0xFFFF))),
                           fabsf(h2f<DT>((uint16_t)(w[k] >> 16)))));
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = a;
    __syncthreads();
    a = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
    g = tensor_scale_from_amax(__float_as_uint(a));
    if (hk == 0 && b == 0 && threadIdx.x == 0) *amax = __float_as_uint(a);
  }
  const int64_t img = (int64_t)b * Hkv + hk;
  uint8_t* q4 = q4img + img * kDecQ4Bytes;
  uint8_t* q16 = q16img + img * kDecQ16Bytes;
  for (int it = threadIdx.x; it < 128 * (kDecD / 16); it += blockDim.x) {
    const int r = it / (kDecD / 16), kb = it % (kDecD / 16);
    uint32_t S = 0, lo = 0, hi = 0;
    uint4 raw0 = make_uint4(0, 0, 0, 0), raw1 = raw0;
    if (r < G) {
      const uint16_t* src = q + ((int64_t)b * H + hk * G + r) * kDecD + kb * 16;
      raw0 = __ldg(reinterpret_cast<const uint4*>(src));
      raw1 = __ldg(reinterpret_cast<const uint4*>(src) + 1);
      float v[16];
      unpack16<DT>(raw0, raw1, v);
      S = quant_block16(v, g, SS, lo, hi);
    }
    q4[64 * (kDecD / 2) + sf_offset(r, kb)] = (uint8_t)S;
    if (r < 64) {
      *reinterpret_cast<uint2*>(q4 + swz_offset(r, kb * 8, kDecD / 2)) = make_uint2(lo, hi);
      uint8_t* reg = q16 + (kb / 4) * (64 * 128);
      *reinterpret_cast<uint4*>(reg + swz_offset(r, (kb % 4) * 32, 128)) = raw0;
      *reinterpret_cast<uint4*>(reg + swz_offset(r, (kb % 4) * 32 + 16, 128)) = raw1;
    }
  }
}

// ------------------------------------------------------------- selection --

// scores [B, H, nbcap] fp64: q . kbar_j by a sequential fp64 fma over d, the
// query taken as its own block mean.  One CTA per (32 key tiles, kv head,
// sequence), 32 G threads: thread (tile, head of the group).  Shared memory
// (dynamic, dec_scores_smem bytes): the tiles' means, rows padded to 129
// doubles, then the G query rows.
constexpr int kDecScoreTiles = 32;

__host__ __device__ constexpr size_t dec_scores_smem(int G) {
  return (size_t)kDecScoreTiles * (kDecD + 1) * 8 + (size_t)G * kDecD * 8;
}

template <int DT>
__global__ void __launch_bounds__(512) dec_scores_kernel(const uint16_t* __restrict__ q, int H,
                                                         int G, CacheGeom cg,
                                                         const uint8_t* __restrict__ cache,
                                                         const int32_t* __restrict__ seq_len,
                                                         int capacity, int nbcap,
                                                         double* __restrict__ scores) {
  extern __shared__ double dsm_scores[];
  double* km = dsm_scores;                                 // [32][129]
  double* qm = dsm_scores + kDecScoreTiles * (kDecD + 1);  // [G][128]
  const int j0 = blockIdx.x * kDecScoreTiles, hk = blockIdx.y, b = blockIdx.z;
  const int len = min(capacity, max(0, __ldg(seq_len + b)));
  const int nb = (int)ceil_div(len, kDecTile);
  if (j0 >= nb) return;
  const int nj = min(kDecScoreTiles, nb - j0);
  const double* means =
      reinterpret_cast<const double*>(cache + cg.off_means()) + cg.tile(b, hk, j0) * kDecD;
  // the means arrive as 16-byte pairs, eight loads in flight per thread
  // before any is stored (the rows' padding breaks a single bulk copy)
  const double2* m2 = reinterpret_cast<const double2*>(means);
  const int npair = nj * kDecD / 2;
  for (int e0 = threadIdx.x; e0 < npair; e0 += 8 * blockDim.x) {
    double2 r[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int e = e0 + k * blockDim.x;
      r[k] = e < npair ? __ldg(m2 + e) : make_double2(0.0, 0.0);
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int e = 2 * (e0 + k * blockDim.x);
      if (e < 2 * npair) {
        double* dst = km + (e / kDecD) * (kDecD + 1) + e % kDecD;
        dst[0] = r[k].x;
        dst[1] = r[k].y;
      }
    }
  }
  for (int e = threadIdx.x; e < G * kDecD; e += blockDim.x)
    qm[e] = (double)h2f<DT>(__ldg(q + ((int64_t)b * H + hk * G + e / kDecD) * kDecD + e % kDecD));
  __syncthreads();
  for (int w = threadIdx.x; w < kDecScoreTiles * G; w += blockDim.x) {
    const int jj = w % kDecScoreTiles, gq = w / kDecScoreTiles;
    if (jj >= nj) continue;
    const double* kr = km + jj * (kDecD + 1);
    const double* qr = qm + gq * kDecD;
    double acc = 0.0;
#pragma unroll 8
    for (int c = 0; c < kDecD; ++c) acc = __fma_rn(qr[c], kr[c], acc);
    scores[((int64_t)b * H + hk * G + gq) * nbcap + j0 + jj] = acc;
  }
}

// mask [B, H, nbcap] uint8 (1 = FP16 key tile): the k = ceil(frac * nb)
// best tiles of each (sequence, head), ties to the lower tile, plus the
// first `sink` and the last `recent` tiles.  One CTA per (sequence, head).
constexpr int kDecTopkThreads = 1024;

__global__ void __launch_bounds__(kDecTopkThreads) dec_topk_kernel(
    const double* __restrict__ scores, const int32_t* __restrict__ seq_len, int capacity, int H,
    int nbcap, float frac, int sink, int recent, uint8_t* __restrict__ mask) {
  __shared__ TopkShared sh;
  extern __shared__ uint64_t kcache[];
  const int b = blockIdx.x / H;
  const int len = min(capacity, max(0, __ldg(seq_len + b)));
  const int nb = (int)ceil_div(len, kDecTile);
  const double* sc = scores + (int64_t)blockIdx.x * nbcap;
  uint8_t* mk = mask + (int64_t)blockIdx.x * nbcap;
  const int64_t k = topk_count_dev(frac, nb);
  auto valid = [&](int64_t j) { return j < nb; };
  auto fixed = [&](int64_t j) { return j < sink || j >= nb - recent; };
  auto score = [&](int64_t j) { return sc[j]; };
  radix_topk(nbcap, k, nb, valid, fixed, score, nbcap <= kTopkCache ? kcache : nullptr, sh, mk);
}

// ----------------------------------------------------------------- merge --

// Splits of one (sequence, head) merged (at most 128 splits, one per
// thread for the weights): each split s left its output O_s
// relative to its own running max m_s (log2 units) and its sum l_s.
//   M = max m_s,  out = sum 2^(m_s - M) O_s / sum 2^(m_s - M) l_s,
//   lse = M ln 2 + ln(sum 2^(m_s - M) l_s).
// An empty sequence gives a zero row and lse = -inf.
template <int DT>
__global__ void __launch_bounds__(kDecD) dec_combine_kernel(const float* __restrict__ part_o,
                                                            const float* __restrict__ part_ml,
                                                            int nsplit, uint16_t* __restrict__ out,
                                                            float* __restrict__ lse) {
  __shared__ float s_w[128];  // weight 2^(m_s - M) of each split (0: empty)
  __shared__ float s_part[4];
  __shared__ float s_ML[2];
  const int64_t bh = blockIdx.x;
  const float* ml = part_ml + bh * nsplit * 2;
  const int tid = threadIdx.x;
  // splits spread over the threads: the maximum, then the weights and L
  const float ms = tid < nsplit ? __ldg(ml + 2 * tid) : -INFINITY;
  const float ls = tid < nsplit ? __ldg(ml + 2 * tid + 1) : 0.0f;
  float M = ms;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  if ((tid & 31) == 0) s_part[tid >> 5] = M;
  __syncthreads();
  M = fmaxf(fmaxf(s_part[0], s_part[1]), fmaxf(s_part[2], s_part[3]));
  const float wgt = (ms == -INFINITY || M == -INFINITY) ? 0.0f : exp2f(ms - M);
  s_w[tid] = wgt;
  float L = wgt * ls;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
  __syncthreads();
  if ((tid & 31) == 0) s_part[tid >> 5] = L;
  __syncthreads();
  if (tid == 0) {
    s_ML[0] = M;
    s_ML[1] = s_part[0] + s_part[1] + s_part[2] + s_part[3];
  }
  __syncthreads();
  L = s_ML[1];
  // channel tid: the weighted sum over the splits, four loads in flight
  const float* po = part_o + bh * nsplit * kDecD + tid;
  float o0 = 0.0f, o1 = 0.0f, o2 = 0.0f, o3 = 0.0f;
  int s2 = 0;
  for (; s2 + 4 <= nsplit; s2 += 4) {
    o0 = fmaf(s_w[s2], __ldg(po + (int64_t)s2 * kDecD), o0);
    o1 = fmaf(s_w[s2 + 1], __ldg(po + (int64_t)(s2 + 1) * kDecD), o1);
    o2 = fmaf(s_w[s2 + 2], __ldg(po + (int64_t)(s2 + 2) * kDecD), o2);
    o3 = fmaf(s_w[s2 + 3], __ldg(po + (int64_t)(s2 + 3) * kDecD), o3);
  }
  for (; s2 < nsplit; ++s2) o0 = fmaf(s_w[s2], __ldg(po + (int64_t)s2 * kDecD), o0);
  const float o = (o0 + o1) + (o2 + o3);
  const float r = L > 0.0f ? o / L : 0.0f;
  if constexpr (DT == 1) {
    out[bh * kDecD + tid] = __bfloat16_as_ushort(__float2bfloat16_rn(r));
  } else {
    out[bh * kDecD + tid] = __half_as_ushort(__float2half_rn(r));
  }
  if (tid == 0) lse[bh] = L > 0.0f ? M * 0.6931471805599453f + logf(L) : -INFINITY;
}

// ------------------------------------------------------ attention kernel --
//
// One CTA per (split of the key tiles, kv head, sequence).  Tensor cores
// compute S^T = K Q^T with the key tile as the 128-row A operand and the G
// query heads of the group as the B operand (N = 16 rows of a 64-row image,
// G used), and
// O^T += V^T P^T with the 128 channels as A and the probability rows as B.
// The key tiles whose heads all run on one path are read once per CTA in
// that format; a tile some heads take in NVFP4 and others in FP16 is read in
// both, each pass with the other heads' probability rows zero.  All NVFP4
// tiles come first, then the FP16 ones (the order of the online softmax).
//
// Two softmax groups of four warps take alternate tiles (group g the tiles
// t = g, g + 2, ...), each with its own S, P and O buffers and its own running
// state: every group is an independent split of the online softmax, merged
// with the others by dec_combine_kernel.  Thread i of a group reads TMEM lane
// i, which is key i of the score tile and channel i of the output tile.  The
// scores of the G heads leave TMEM into a transposed shared-memory tile, so
// that the probability work runs per (head, 16-key block): thread 8c + b
// takes block b of head c, with the eight blocks of a head in eight
// consecutive lanes.  Each PV lands in an output buffer of its own; the
// group folds it into its running output, held in registers (channel i,
// G heads), out of the critical path:
//   O <- alpha O + sigma PV(t),
// alpha = 2^(m - m_new), sigma = 2^(mt - m_new) / 2688 * g_V for an NVFP4
// tile (probabilities taken relative to the tile's own max mt, as in the
// prefill kernel) and 1 for an FP16 one.

__host__ __device__ constexpr uint32_t dec_align(uint32_t x) { return (x + 1023u) & ~1023u; }

// Maximum of a float over the warp (one redux instruction).
__device__ __forceinline__ float redux_max_f32(float v) {
  float r;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}

// Sum of N values by a pairwise tree.
template <int N>
__device__ __forceinline__ float tree_sum(const float* x) {
  float y[N];
#pragma unroll
  for (int e = 0; e < N; ++e) y[e] = x[e];
#pragma unroll
  for (int w = N / 2; w >= 1; w >>= 1) {
#pragma unroll
    for (int e = 0; e < w; ++e) y[e] += y[e + w];
  }
  return y[0];
}

// Four fp32 values -> four E2M1 codes in the low 16 bits (value 2i in the
// low nibble of byte i), round to nearest even, saturating.
__device__ __forceinline__ uint32_t e2m1x4(const float* x) {
  uint32_t out;
  asm("{\n\t.reg .b8 b0, b1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "mov.b32 %0, {b0, b1, 0, 0};\n\t}"
      : "=r"(out)
      : "f"(x[0]), "f"(x[1]), "f"(x[2]), "f"(x[3]));
  return out;
}

struct DecLayout {
  static constexpr uint32_t P4B = fp4_tile_bytes(64, kDecTile);       // 5120
  static constexpr uint32_t P16B = 64 * kDecTile * 2;                 // 16384
  static constexpr uint32_t STG4 = CacheGeom::K4 + CacheGeom::V4;     // 18432
  static constexpr uint32_t STG16 = CacheGeom::K16 + CacheGeom::V16;  // 65536
  //   NVFP4 view: Q4 | P4 x4 (two per group) | NS4 stages (K4 + V4)
  //   FP16 view:  Q16 | P16 x2 (one per group) | NS16 stages (K16 + V16)
  static constexpr uint32_t OFF4_Q = 0;
  static constexpr uint32_t OFF4_P = dec_align(kDecQ4Bytes);
  static constexpr uint32_t OFF4_STG = OFF4_P + 4 * dec_align(P4B);  // two slots per group
  static constexpr uint32_t OFF16_Q = 0;
  static constexpr uint32_t OFF16_P = dec_align(kDecQ16Bytes);
  static constexpr uint32_t OFF16_STG = OFF16_P + 2 * P16B;
  static constexpr uint32_t NS16 = 2;
  static constexpr uint32_t REGION = OFF16_STG + NS16 * STG16;
  static constexpr uint32_t NS4 = (REGION - OFF4_STG) / STG4;
  static constexpr uint32_t MAX_TILES = 1024;  // tile-list entries (a tile may appear twice)
  static constexpr uint32_t OFF_LIST = REGION;
  static constexpr uint32_t ST_PITCH = kDecTile + 4;  // floats per transposed score row
  static constexpr uint32_t ST_BYTES = kDecMaxG * ST_PITCH * 4;
  static constexpr uint32_t OFF_ST = OFF_LIST + 4 * MAX_TILES;       // [group][2][16][132]
  static constexpr uint32_t OFF_COEF = OFF_ST + 2 * 2 * ST_BYTES;    // [group][4][16][2]
  static constexpr uint32_t OFF_BAR = OFF_COEF + 2 * 4 * kDecMaxG * 2 * 4;
  static constexpr uint32_t BYTES = OFF_BAR + 512;
  static constexpr uint32_t SMEM_ALLOC = BYTES + 1024;
  // tensor-memory columns (N = kDecN query columns per S or O buffer)
  static constexpr uint32_t T_S = 0;      // + kDecN (2 g + slot)
  static constexpr uint32_t T_O = 64;     // + kDecN (2 g + slot)
  static constexpr uint32_t T_QSF = 128;  // + 8 g (two K-steps of 4 columns)
  static constexpr uint32_t T_KSF = 144;  // + 8 g
  static constexpr uint32_t T_PSF = 160;  // + 8 g
  static constexpr uint32_t T_VSF = 176;  // + 8 g
  static constexpr uint32_t T_COLS = 256;  // allocation
  static_assert(NS4 == 8, "barrier plan assumes eight NVFP4 stages");
  static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
};

// Barriers.  GB: per group g, the group's own barrier (one phase per tile).
// Per group g and slot s (tile t of the group uses slot (t >> 1) & 1): SF /
// SE S buffer s full (QK commit) / read, PF its P tile written, OD its PV
// retired into O buffer s, OE O buffer s folded (free again).  A
// barrier of a slot only completes its next phase after its waiter has
// passed the previous one: the slot's next PV waits OE, whose fold waited
// OD; the slot's next P waits for that fold (or for OD, FP16).
enum : int {
  D_Q4 = 0, D_Q16 = 1, D_SF = 2 /* 2..5 */, D_SE = 6 /* 6..9 */, D_PF = 10 /* 10..13 */,
  D_OD = 14 /* 14..17 */, D_OE = 18 /* 18..21 */, D_GB = 22 /* 22,23 */, D_P4DONE = 24,
  D_DONE = 25, D_KVF16 = 26 /* 26,27 */, D_KVE16 = 28 /* 28,29 */, D_KVF4 = 30 /* 30..37 */,
  D_KVE4 = 38 /* 38..45 */, D_N = 46
};

// warps 0..7 softmax (two groups), 8 producer, 9 + g the QK^T issuer of
// group g (warp 9 also owns tensor memory), 11 + g its PV issuer
constexpr int kDecProducerWarp = 8, kDecQkWarp = 9, kDecPvWarp = 11;
constexpr int kDecThreads = 32 * 13;

struct DecParams {
  const uint8_t* cache;
  CacheGeom cg;
  const uint8_t* q4img;
  const uint8_t* q16img;
  const uint8_t* mask;  // [B, H, nbcap]
  const int32_t* seq_len;
  const uint32_t* amax_q;
  const float* kv_scale;  // g_K, g_V
  float* part_o;          // [B * H, 2 * nsplit, d]
  float* part_ml;         // [B * H, 2 * nsplit, 2]
  int nbcap, capacity, H, G, nsplit;
  float scale;  // log2(e) / sqrt(d)
};

template <int DT, int GC>
__global__ void __launch_bounds__(kDecThreads, 1) attn_decode_kernel(const DecParams p) {
  using L = DecLayout;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~(uintptr_t)1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::OFF_BAR);
  uint32_t* s_list = reinterpret_cast<uint32_t*>(sm + L::OFF_LIST);
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + L::OFF_BAR + 8 * D_N);
  int* s_n = reinterpret_cast<int*>(s_tmem + 1);
  int* s_n4 = s_n + 1;
  volatile int* s_abort = s_n + 2;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
  const int G = p.G;
  const int len = min(p.capacity, max(0, __ldg(p.seq_len + b)));
  const int nb = (int)ceil_div(len, kDecTile);
  const int j0 = (int)((int64_t)nb * split / p.nsplit);
  const int j1 = (int)((int64_t)nb * (split + 1) / p.nsplit);

  if (tid == 0) {
    for (int i = 0; i < D_N; ++i) {
      uint32_t cnt = 1;
      if ((i >= D_SE && i < D_SE + 4) || (i >= D_PF && i < D_PF + 4) ||
          (i >= D_OE && i < D_OE + 4) || (i >= D_GB && i < D_GB + 2))
        cnt = 128;
      if (i == D_DONE) cnt = 4;     // one commit per MMA issuer
      if (i == D_P4DONE) cnt = 2;   // one commit per PV issuer
      mbar_init(&bars[i], cnt);
    }
    *s_abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    // Tile list: tiles some head takes in NVFP4 (ascending), then tiles some
    // head takes in FP16 (ascending).  Entry: tile j (bits 0..14), the FP16
    // heads of the group (bits 16..31).  The mask bytes of up to 128 tiles
    // are requested before any is used (one memory round trip per 128).
    const uint32_t all = (1u << G) - 1u;
    const uint8_t* mk = p.mask + ((int64_t)b * p.H + hk * G) * p.nbcap;
    int n = 0, nf = 0;
    uint32_t* l16 = s_list + L::MAX_TILES / 2;  // FP16 entries, moved after the NVFP4 ones
    for (int jb = j0; jb < j1; jb += 128) {
      uint32_t bits[4] = {0, 0, 0, 0};
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int j = jb + 32 * r + lane;
        if (j < j1)
          for (int c = 0; c < G; ++c)
            bits[r] |= (uint32_t)(__ldg(mk + (int64_t)c * p.nbcap + j) != 0) << c;
      }
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int j = jb + 32 * r + lane;
        const bool in = j < j1;
        const bool t4 = in && bits[r] != all, t16 = in && bits[r] != 0;
        const unsigned v4 = __ballot_sync(0xffffffffu, t4), v16 = __ballot_sync(0xffffffffu, t16);
        const uint32_t e = (uint32_t)j | (bits[r] << 16);
        if (t4) s_list[n + __popc(v4 & ((1u << lane) - 1u))] = e;
        if (t16) l16[nf + __popc(v16 & ((1u << lane) - 1u))] = e;
        n += __popc(v4);
        nf += __popc(v16);
      }
    }
    __syncwarp();
    for (int e = lane; e < nf; e += 32) s_list[n + e] = l16[e];
    if (lane == 0) {
      *s_n4 = n;
      *s_n = n + nf;
    }
  }
  __syncthreads();
  if (warp == kDecQkWarp) {
    tmem_alloc(s_tmem, L::T_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;
  const int n = *s_n, n4 = *s_n4;
  const int64_t img = (int64_t)b * p.cg.Hkv + hk;

  if (warp == kDecProducerWarp) {
    // ------------------------------------------------------- producer --
    if (lane == 0) {
      bool q4_issued = false, q16_issued = false;
      int last4[L::NS4], last16[L::NS16];
      for (int i = 0; i < (int)L::NS4; ++i) last4[i] = -1;
      for (int i = 0; i < (int)L::NS16; ++i) last16[i] = -1;
      if (n4 > 0) {
        mbar_arrive_expect_tx(&bars[D_Q4], kDecQ4Bytes);
        bulk_g2s(sm + L::OFF4_Q, p.q4img + img * kDecQ4Bytes, kDecQ4Bytes, &bars[D_Q4]);
        q4_issued = true;
      }
      for (int t = 0; t < n && !*s_abort; ++t) {
        const int j = (int)(s_list[t] & 0x7FFFu);
        const int64_t tl = p.cg.tile(b, hk, j);
        if (t < n4) {
          const int i = t, sl = i % L::NS4;
          if (i >= (int)L::NS4 &&
              !mbar_wait(&bars[D_KVE4 + sl], ((i / L::NS4) - 1) & 1, s_abort))
            break;
          uint8_t* stg = sm + L::OFF4_STG + sl * L::STG4;
          mbar_arrive_expect_tx(&bars[D_KVF4 + sl], L::STG4);
          bulk_g2s(stg, p.cache + tl * CacheGeom::K4, CacheGeom::K4, &bars[D_KVF4 + sl]);
          bulk_g2s(stg + CacheGeom::K4, p.cache + p.cg.off_v4() + tl * CacheGeom::V4,
                   CacheGeom::V4, &bars[D_KVF4 + sl]);
          last4[sl] = i;
        } else {
          if (t == n4) {
            // the FP16 view overlays the NVFP4 one: every NVFP4 PV has retired
            if (n4 > 0 && !mbar_wait(&bars[D_P4DONE], 0, s_abort)) break;
            mbar_arrive_expect_tx(&bars[D_Q16], kDecQ16Bytes);
            bulk_g2s(sm + L::OFF16_Q, p.q16img + img * kDecQ16Bytes, kDecQ16Bytes, &bars[D_Q16]);
            q16_issued = true;
          }
          const int i = t - n4, sl = i % L::NS16;
          if (i >= (int)L::NS16 &&
              !mbar_wait(&bars[D_KVE16 + sl], ((i / L::NS16) - 1) & 1, s_abort))
            break;
          uint8_t* stg = sm + L::OFF16_STG + sl * L::STG16;
          mbar_arrive_expect_tx(&bars[D_KVF16 + sl], L::STG16);
          bulk_g2s(stg, p.cache + p.cg.off_k16() + tl * CacheGeom::K16, CacheGeom::K16,
                   &bars[D_KVF16 + sl]);
          bulk_g2s(stg + CacheGeom::K16, p.cache + p.cg.off_v16() + tl * CacheGeom::V16,
                   CacheGeom::V16, &bars[D_KVF16 + sl]);
          last16[sl] = i;
        }
      }
      // Drain: every copy this thread issued has landed before the CTA ends.
      int dummy = 0;
      volatile int* never = &dummy;
      if (q4_issued) mbar_wait(&bars[D_Q4], 0, never, 200000000ull);
      if (q16_issued) mbar_wait(&bars[D_Q16], 0, never, 200000000ull);
      for (int sl = 0; sl < (int)L::NS4; ++sl)
        if (last4[sl] >= 0)
          mbar_wait(&bars[D_KVF4 + sl], (last4[sl] / L::NS4) & 1, never, 200000000ull);
      for (int sl = 0; sl < (int)L::NS16; ++sl)
        if (last16[sl] >= 0)
          mbar_wait(&bars[D_KVF16 + sl], (last16[sl] / L::NS16) & 1, never, 200000000ull);
    }
  } else if (warp >= kDecQkWarp) {
    // ---------------------------------------------------- MMA issuers --
    // Group g's tiles t = g, g + 2, ...: QK^T by warp kDecQkWarp + g, PV by
    // warp kDecPvWarp + g, each with its own scale-factor columns.  Stage of
    // tile t: the NVFP4 ring for t < n4, then the FP16 ring from t = n4.
    if (lane == 0) {
      const bool is_qk = warp < kDecPvWarp;
      const int g = is_qk ? warp - kDecQkWarp : warp - kDecPvWarp;
      constexpr uint32_t id4 = idesc_nvf4(128, kDecN), id16 = idesc_f16(DT, 128, kDecN);
      const uint32_t base = smem_u32(sm);
      const uint64_t d_sf = make_sdesc(base, 512, 128, SW_NONE);  // + (byte offset >> 4)
      // operands of 64-byte rows (NVFP4, K = 128 elements) and of 128-byte
      // rows (16-bit, one 64-column region)
      const uint64_t d4 = make_sdesc(base, 16, 8 * 64, SW_64B);
      const uint64_t d16 = make_sdesc(base, 16, 1024, SW_128B);
      auto stage_of = [&](int t, int& sl, int& par) {
        if (t < n4) {
          sl = t % (int)L::NS4;
          par = (t / (int)L::NS4) & 1;
        } else {
          sl = (t - n4) % (int)L::NS16;
          par = ((t - n4) / (int)L::NS16) & 1;
        }
      };
      bool ok = true;
      if (is_qk) {
        bool q4_ready = false, q16_ready = false;
        const uint32_t qsf = tmem + L::T_QSF + 8 * g, ksf = tmem + L::T_KSF + 8 * g;
        for (int t = g; t < n && ok; t += 2) {
          const int u = t >> 1;
          const bool f16 = t >= n4;
          int sl, par;
          stage_of(t, sl, par);
          uint64_t* full = f16 ? &bars[D_KVF16 + sl] : &bars[D_KVF4 + sl];
          if (!mbar_wait(full, par, s_abort)) { ok = false; break; }
          if (!f16 && !q4_ready) {
            if (!mbar_wait(&bars[D_Q4], 0, s_abort)) { ok = false; break; }
          }
          if (f16 && !q16_ready) {
            if (!mbar_wait(&bars[D_Q16], 0, s_abort)) { ok = false; break; }
            q16_ready = true;
          }
          const uint32_t dS = tmem + L::T_S + kDecN * (2 * g + (u & 1));
          if (!f16) {
            // scale factors first: they wait only for the stage (the slot's
            // previous reader, QK(t - 2), was issued earlier by this thread)
            tc_fence_after();
            const uint32_t stg = L::OFF4_STG + sl * L::STG4;
            if (!q4_ready) {
#pragma unroll
              for (int s2 = 0; s2 < 2; ++s2)
                tc_cp_32x128b_x4(qsf + 4 * s2,
                                 d_sf + ((L::OFF4_Q + 64 * (kDecD / 2) + 512 * s2) >> 4));
              q4_ready = true;
            }
#pragma unroll
            for (int s2 = 0; s2 < 2; ++s2)
              tc_cp_32x128b_x4(ksf + 4 * s2, d_sf + ((stg + kDecTile * (kDecD / 2) + 512 * s2) >> 4));
            if (u >= 2 && !mbar_wait(&bars[D_SE + 2 * g + (u & 1)], ((u >> 1) - 1) & 1, s_abort)) {
              ok = false;
              break;
            }
            tc_fence_after();
#pragma unroll
            for (int s2 = 0; s2 < 2; ++s2)
              mma_nvf4(dS, d4 + (stg >> 4) + 2 * s2, d4 + (L::OFF4_Q >> 4) + 2 * s2, id4,
                       ksf + 4 * s2, qsf + 4 * s2, s2 > 0);
          } else {
            if (u >= 2 && !mbar_wait(&bars[D_SE + 2 * g + (u & 1)], ((u >> 1) - 1) & 1, s_abort)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t stg = L::OFF16_STG + sl * L::STG16;
#pragma unroll
            for (int kk = 0; kk < kDecD / 16; ++kk)
              mma_f16(dS, d16 + ((stg + (kk / 4) * 128 * 128) >> 4) + 2 * (kk % 4),
                      d16 + ((L::OFF16_Q + (kk / 4) * 64 * 128) >> 4) + 2 * (kk % 4), id16, kk > 0);
          }
          tc_commit(&bars[D_SF + 2 * g + (u & 1)]);
        }
      } else {
        const uint32_t vsf = tmem + L::T_VSF + 8 * g, psf = tmem + L::T_PSF + 8 * g;
        // this issuer's share of "every NVFP4 PV retired": after its last
        // NVFP4 tile, or at once when it has none
        bool p4_signalled = false;
        if (g >= n4) {
          tc_commit(&bars[D_P4DONE]);
          p4_signalled = true;
        }
        for (int t = g; t < n && ok; t += 2) {
          const int u = t >> 1;
          const bool f16 = t >= n4;
          int sl, par;
          stage_of(t, sl, par);
          uint64_t* empty = f16 ? &bars[D_KVE16 + sl] : &bars[D_KVE4 + sl];
          const int sl2 = u & 1, use = u >> 1;  // P / O slot and its use count
          if (!f16) {
            // V's scale factors as soon as the stage has landed (the slot's
            // previous reader, PV(t - 2), was issued earlier by this thread)
            if (!mbar_wait(&bars[D_KVF4 + sl], par, s_abort)) { ok = false; break; }
            tc_fence_after();
            const uint32_t stg = L::OFF4_STG + sl * L::STG4 + CacheGeom::K4;
#pragma unroll
            for (int s2 = 0; s2 < 2; ++s2)
              tc_cp_32x128b_x4(vsf + 4 * s2, d_sf + ((stg + kDecD * (kDecTile / 2) + 512 * s2) >> 4));
          }
          if (!mbar_wait(&bars[D_PF + 2 * g + sl2], use & 1, s_abort)) { ok = false; break; }
          if (use >= 1 && !mbar_wait(&bars[D_OE + 2 * g + sl2], (use - 1) & 1, s_abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t dO = tmem + L::T_O + kDecN * (2 * g + sl2);
          if (!f16) {
            const uint32_t stg = L::OFF4_STG + sl * L::STG4 + CacheGeom::K4;
            const uint32_t pp = L::OFF4_P + (2 * g + sl2) * dec_align(L::P4B);
#pragma unroll
            for (int s2 = 0; s2 < 2; ++s2)
              tc_cp_32x128b_x4(psf + 4 * s2, d_sf + ((pp + 64 * (kDecTile / 2) + 512 * s2) >> 4));
#pragma unroll
            for (int s2 = 0; s2 < 2; ++s2)
              mma_nvf4(dO, d4 + (stg >> 4) + 2 * s2, d4 + (pp >> 4) + 2 * s2, id4, vsf + 4 * s2,
                       psf + 4 * s2, s2 > 0);
          } else {
            const uint32_t stg = L::OFF16_STG + sl * L::STG16 + CacheGeom::K16;
            const uint32_t pp = L::OFF16_P + g * L::P16B;
#pragma unroll
            for (int kk = 0; kk < kDecTile / 16; ++kk)
              mma_f16(dO, d16 + ((stg + (kk / 4) * 128 * 128) >> 4) + 2 * (kk % 4),
                      d16 + ((pp + (kk / 4) * 64 * 128) >> 4) + 2 * (kk % 4), id16, kk > 0);
          }
          tc_commit(&bars[D_OD + 2 * g + sl2]);
          tc_commit(empty);
          if (!p4_signalled && t + 2 >= n4) {
            tc_commit(&bars[D_P4DONE]);
            p4_signalled = true;
          }
        }
      }
      // every MMA of the four issuers has completed before the CTA ends
      tc_commit(&bars[D_DONE]);
      int dummy = 0;
      volatile int* never = &dummy;
      mbar_wait(&bars[D_DONE], 0, never, 200000000ull);
    }
  } else if (warp < 8) {
    // -------------------------------------------------------- softmax --
    const int g = warp >> 2, wq = warp & 3, i = tid & 127;
    const float gq = tensor_scale_from_amax(*p.amax_q);
    const float gk = __ldg(p.kv_scale), gv = __ldg(p.kv_scale + 1);
    const float cs4 = __fmul_rn(__fmul_rn(gq, gk), p.scale), cs16 = p.scale;
    float* sT0 = reinterpret_cast<float*>(sm + L::OFF_ST) + g * 2 * (L::ST_BYTES / 4);
    float* coef = reinterpret_cast<float*>(sm + L::OFF_COEF) + g * (4 * kDecMaxG * 2);
    const uint32_t lane_base = tmem + ((uint32_t)(wq * 32) << 16);
    const uint32_t s_addr = lane_base + L::T_S + kDecN * (2 * g);  // + kDecN slot
    const uint32_t o_addr = lane_base + L::T_O + kDecN * (2 * g);  // + kDecN slot
    uint8_t* p4g = sm + L::OFF4_P + 2 * g * dec_align(L::P4B);   // + slot * P4 slot
    uint8_t* p16 = sm + L::OFF16_P + g * L::P16B;
    // work item of this thread: keys [16 bb + KPL hb, + KPL) of head c, the
    // LPB lanes of a 16-key block and the eight blocks of a head adjacent
    constexpr int LPB = GC >= 16 ? 1 : (GC >= 8 ? 2 : 4);  // lanes per 16-key block
    constexpr int KPL = 16 / LPB;                          // keys per lane
    const int c = i / (8 * LPB), bb = (i / LPB) % 8, hb = i % LPB;
    const bool has_item = i < 8 * LPB * GC;  // uniform over each warp
    const bool is_owner = (i % (8 * LPB)) == 0;
    // running state of head c, kept by each of its 8 LPB lanes: the same
    // max m on all of them, and each lane's share of the sum l (its keys'
    // probabilities; the shares are added once, at the end)
    float m = -INFINITY, l = 0.0f;
    float orun[GC];
#pragma unroll
    for (int k = 0; k < GC; ++k) orun[k] = 0.0f;
    // probability rows past the group stay zero (NVFP4 slot now, FP16 slot
    // when its phase begins).  The NVFP4 view overlays the FP16 one, whose
    // query image the producer loads at once when there is no NVFP4 tile:
    // the NVFP4 slot is only touched when that phase exists.
    if (n4 > 0) {
      for (int sl2 = 0; sl2 < 2; ++sl2) {
        uint8_t* p4 = p4g + sl2 * dec_align(L::P4B);
        for (int e = i; e < (64 - GC) * 4; e += 128)
          *reinterpret_cast<uint4*>(p4 + (GC + e / 4) * 64 + (e % 4) * 16) = make_uint4(0, 0, 0, 0);
        for (int e = i; e < (64 - GC) * 8; e += 128)
          p4[64 * (kDecTile / 2) + sf_offset(GC + e / 8, e % 8)] = 0;
      }
    }
    // fold of the group's tile with use count v (slot v & 1): wait for its
    // PV and start the load (fold_issue), then add it to the running output
    // with the coefficients its owners wrote (slot v & 3) and free the O
    // buffer (fold_finish, after tcgen05.wait::ld)
    float o[GC];
    auto fold_issue = [&](int v) -> bool {
      if (!warp_wait(&bars[D_OD + 2 * g + (v & 1)], (v >> 1) & 1, s_abort)) return false;
      tc_fence_after();
      tmem_ld_cols<GC>(o_addr + kDecN * (v & 1), o);
      return true;
    };
    auto fold_finish = [&](int v) {
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(&bars[D_OE + 2 * g + (v & 1)]);
      const float* cf = coef + (v & 3) * (kDecMaxG * 2);
#pragma unroll
      for (int k = 0; k < GC; ++k) orun[k] = fmaf(cf[2 * k], orun[k], cf[2 * k + 1] * o[k]);
    };
    bool p16_ready = false;
    bool ok = true;
    int u_last = -1;
    for (int t = g; t < n && ok; t += 2) {
      const int u = t >> 1;
      const uint32_t ent = s_list[t];
      const int j = (int)(ent & 0x7FFFu);
      const uint32_t bits = ent >> 16;
      const bool f16 = t >= n4;
      if (f16 && !p16_ready) {
        if (n4 > 0 && !warp_wait(&bars[D_P4DONE], 0, s_abort)) { ok = false; break; }
        for (int e = i; e < (64 - GC) * 16; e += 128) {
          const int r = GC + e / 16, ch = e % 16;  // 16-byte chunks of a 256-byte row
          *reinterpret_cast<uint4*>(p16 + (ch / 8) * (64 * 128) + r * 128 + (ch % 8) * 16) =
              make_uint4(0, 0, 0, 0);
        }
        p16_ready = true;
      }
      float* sT = sT0 + (u & 1) * (L::ST_BYTES / 4);
      // A: scores of key i for the group's heads -> transposed tile
      if (!warp_wait(&bars[D_SF + 2 * g + (u & 1)], (u >> 1) & 1, s_abort)) { ok = false; break; }
      tc_fence_after();
      {
        float a[GC];
        tmem_ld_cols<GC>(s_addr + kDecN * (u & 1), a);
        tmem_ld_wait();
        const bool valid = j * kDecTile + i < len;
#pragma unroll
        for (int k = 0; k < GC; ++k) sT[k * L::ST_PITCH + i] = valid ? a[k] : -INFINITY;
      }
      tc_fence_before();
      mbar_arrive(&bars[D_SE + 2 * g + (u & 1)]);
      mbar_arrive(&bars[D_GB + g]);
      if (!warp_wait(&bars[D_GB + g], u & 1, s_abort)) { ok = false; break; }
      // E (first half): PV(t - 2) retired (the single FP16 P buffer is then
      // free too); its load runs while the probabilities are computed
      if (u >= 1 && !fold_issue(u - 1)) { ok = false; break; }
      uint8_t* p4 = p4g + (u & 1) * dec_align(L::P4B);
      // C: probabilities of keys [16 bb + KPL hb, + KPL) of head c
      if (has_item) {
        float x[KPL];
        const float4* src =
            reinterpret_cast<const float4*>(sT + c * L::ST_PITCH + 16 * bb + KPL * hb);
#pragma unroll
        for (int q = 0; q < KPL / 4; ++q) {
          const float4 v4 = src[q];
          x[4 * q] = v4.x;
          x[4 * q + 1] = v4.y;
          x[4 * q + 2] = v4.z;
          x[4 * q + 3] = v4.w;
        }
        float bm = x[0];
#pragma unroll
        for (int e = 1; e < KPL; ++e) bm = fmaxf(bm, x[e]);
#pragma unroll
        for (int o2 = 1; o2 < LPB; o2 <<= 1) bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, o2));
        float mt_raw;
        if constexpr (8 * LPB == 32) {
          mt_raw = redux_max_f32(bm);  // the head is the whole warp
        } else {
          mt_raw = bm;
#pragma unroll
          for (int o2 = LPB; o2 < 8 * LPB; o2 <<= 1)
            mt_raw = fmaxf(mt_raw, __shfl_xor_sync(0xffffffffu, mt_raw, o2));
        }
        const bool active = c < G && (((bits >> c) & 1u) != 0) == f16;
        float alpha = 1.0f, sigma = 0.0f;
        if (!f16) {
          uint32_t S = 0;
          uint32_t code[KPL / 8 > 0 ? KPL / 8 : 1] = {};
          uint32_t code4 = 0;  // KPL == 4: two bytes
          bool drop = false;
          if (active) {
            const float mt = mt_raw * cs4;
            const float m_new = fmaxf(m, mt);
            const float e = ex2_ftz(fmaf(bm, cs4, -mt));  // block max / tile max
            S = ue4m3(448.0f * e);
            const float dec = ue4m3_decode_fast(S);
            const float cc = S ? 11.392317422778760f - mt - lg2_ftz(dec) : -INFINITY;  // log2(2688)
#pragma unroll
            for (int e2 = 0; e2 < KPL; e2 += 2) fma2(x[e2], x[e2 + 1], x[e2], x[e2 + 1], cs4, cs4, cc, cc);
#pragma unroll
            for (int e2 = 0; e2 < KPL; ++e2) x[e2] = ex2_ftz(x[e2]);  // masked (-inf) -> 0
            const float ls = tree_sum<KPL>(x) * dec;
            if constexpr (KPL >= 8) {
#pragma unroll
              for (int q = 0; q < KPL / 8; ++q) code[q] = e2m1x8(x + 8 * q);
            } else {
              code4 = e2m1x4(x);
            }
            const float rowmax = ex2_ftz(mt - m_new);
            float sigma_raw = rowmax >= 8.6736174e-19f ? rowmax * (1.0f / 2688.0f) : 0.0f;  // 2^-60
            sigma = sigma_raw * gv;
            if (!(sigma >= 1.17549435e-38f)) sigma = sigma_raw = 0.0f;
            drop = sigma == 0.0f;
            alpha = m == -INFINITY ? 0.0f : ex2_ftz(m - m_new);
            l = fmaf(ls, sigma_raw, alpha * l);
            m = m_new;
          }
          uint8_t* dst = p4 + swz_offset(c, 8 * bb + (KPL / 2) * hb, kDecTile / 2);
          if constexpr (KPL == 16) {
            *reinterpret_cast<uint2*>(dst) = make_uint2(code[0], code[1]);
          } else if constexpr (KPL == 8) {
            *reinterpret_cast<uint32_t*>(dst) = code[0];
          } else {
            *reinterpret_cast<uint16_t*>(dst) = (uint16_t)code4;
          }
          if (hb == 0) p4[64 * (kDecTile / 2) + sf_offset(c, bb)] = drop ? 0 : (uint8_t)S;
        } else {
          uint32_t w[KPL / 2] = {};
          if (active) {
            const float mt = mt_raw * cs16;
            const float m_new = fmaxf(m, mt);
            const float negm = -m_new;
#pragma unroll
            for (int e2 = 0; e2 < KPL; e2 += 2)
              fma2(x[e2], x[e2 + 1], x[e2], x[e2 + 1], cs16, cs16, negm, negm);
#pragma unroll
            for (int e2 = 0; e2 < KPL; ++e2) x[e2] = ex2_ftz(x[e2]);
            const float ls = tree_sum<KPL>(x);
#pragma unroll
            for (int e2 = 0; e2 < KPL / 2; ++e2) w[e2] = pack2<DT>(x[2 * e2], x[2 * e2 + 1]);
            alpha = m == -INFINITY ? 0.0f : ex2_ftz(m - m_new);
            sigma = 1.0f;
            l = fmaf(alpha, l, ls);
            m = m_new;
          }
          const uint32_t k0 = 16 * bb + KPL * hb;
          uint8_t* reg = p16 + (k0 / 64) * (64 * 128);
#pragma unroll
          for (int q = 0; q < KPL / 8; ++q)
            *reinterpret_cast<uint4*>(reg + swz_offset(c, (k0 % 64) * 2 + 16 * q, 128)) =
                make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
          if constexpr (KPL == 4)
            *reinterpret_cast<uint2*>(reg + swz_offset(c, (k0 % 64) * 2, 128)) = make_uint2(w[0], w[1]);
        }
        if (is_owner) {
          float* cf = coef + (u & 3) * (kDecMaxG * 2);
          cf[2 * c] = alpha;
          cf[2 * c + 1] = sigma;
        }
      }
      // D: P(t) is in shared memory
      fence_proxy_async_smem();
      mbar_arrive(&bars[D_PF + 2 * g + (u & 1)]);
      // E (second half): fold PV(t - 2) (its coefficients were written
      // before this tile's barrier)
      if (u >= 1) fold_finish(u - 1);
      u_last = u;
    }
    // the group's last PV, folded once every owner lane has written the
    // coefficients of its tile (one more phase of the group barrier)
    if (ok && u_last >= 0) {
      mbar_arrive(&bars[D_GB + g]);
      ok = warp_wait(&bars[D_GB + g], (u_last + 1) & 1, s_abort);
      if (ok) ok = fold_issue(u_last);
      if (ok) fold_finish(u_last);
    }
    if (ok) {
      // this group's split: output relative to its running max, m and l
      const int ns = 2 * p.nsplit, sidx = 2 * split + g;
      const int64_t row0 = (int64_t)b * p.H + hk * G;
#pragma unroll
      for (int k = 0; k < GC; ++k)
        if (k < G) p.part_o[((row0 + k) * ns + sidx) * kDecD + i] = orun[k];
      if (has_item) {
#pragma unroll
        for (int o2 = 1; o2 < 8 * LPB; o2 <<= 1) l += __shfl_xor_sync(0xffffffffu, l, o2);
        if (is_owner && c < G) {
          p.part_ml[((row0 + c) * ns + sidx) * 2] = m;
          p.part_ml[((row0 + c) * ns + sidx) * 2 + 1] = l;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kDecQkWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, L::T_COLS);
  }
}

}  // namespace thrift
