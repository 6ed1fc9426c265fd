// Attn-QAT attention: forward on fake-quantised NVFP4 operands and the
// backward with FP4 recomputation of the probabilities.
//
// Source: "Attn-QAT: 4-Bit Attention With Quantization-Aware Training",
// Metodologia (1: the backward recomputes the probabilities at the forward's
// FP4 precision; 2: the scalar term of the softmax gradient is taken from a
// high-precision output O' kept beside the FP4 output).
//
// What is computed (every quantiser passes gradients straight through):
//   Q^, K^  NVFP4 blocks of 16 along d; V^ blocks of 16 along the tokens of
//           each sequence (zero padded); per-tensor scales g = amax / 2688
//   S = Q^ K^T / sqrt(d),  lse = log sum_j exp S,  P = exp(S - lse)
//   P^  two-level FP4 image of P per (row, key tile of blk keys):
//       sigma = rowmax / 2688; the 16-key blocks of P / sigma are quantised
//       with block scale E4M3(amax / 6) and no tensor scale
//   O = P^ V^ (the FP4 output),  O' = P V^,  D = rowsum(dO o O')
//   dV = (P^)^T dO,  dP = dO V^T,  dS = P o (dP - D),
//   dQ = dS K^ / sqrt(d),  dK = dS^T Q^ / sqrt(d)
//   (dK, dV summed over the query heads of a kv head)
//
// Design.  Memory-bound kernels write the fake-quantised images once: each
// element is E2M1 value x UE4M3 block scale, exact in the 16-bit input type,
// with the tensor scales applied to the fp32 accumulators instead.  The
// three attention kernels run warp-level m16n8k16 MMAs (fp32 accumulate) on
// those images; P^ enters the MMAs rounded to the 16-bit type, dS and the P
// of O' as sums of two 16-bit parts.  Operand tiles are staged by cp.async
// with the next tile in flight; B operands that run along the rows of a
// staged tile are transposed by ldmatrix.
//   qat_fwd_kernel     per 128-query tile, one pass over the key tiles:
//                      running max, P, its FP4 image, O, O', lse
//   qat_rowdot_kernel  D = rowsum(dO o O')
//   qat_bwd_kv_kernel  per key tile of blk keys, over every 64-query chunk
//                      of the kv head's query heads: S^T, P^T, its FP4
//                      image, dP^T, dS^T; dV += (P^)^T dO, dK += dS^T Q^
//   qat_bwd_q_kernel   per 64-query tile: S, P, dP, dS; dQ += dS K^
#pragma once
#include "quant_kernels.cuh"

namespace thrift {

constexpr int kQatFwdRows = 128;  // query rows of a forward CTA (8 warps x 16)
constexpr int kQatRows = 64;   // query rows of a dQ CTA (4 warps x 16)
constexpr int kQatChunk = 64;  // query chunk of the key-tile kernel, key chunk of the dQ kernel
constexpr float kQatLog2e = 1.4426950408889634f;
constexpr float kQatLn2 = 0.6931471805599453f;

struct QatParams {
  const uint16_t* qi;  // fake-quantised images [total, H|Hkv, D] in the input type
  const uint16_t* ki;
  const uint16_t* vi;
  const uint16_t* dout;  // [total, H, D] (backward)
  const float* g;        // tensor scales of Q, K, V
  SeqInfo si;
  int H, Hkv;
  int64_t total;
  int causal;
  float sc;          // 1 / sqrt(d)
  uint16_t* out;     // forward: O [total, H, D] in the input type
  float* out_hp;     // forward: O' [total, H, D]; backward: read
  float* lse;        // [H, total], natural log
  const float* dsum; // D [H, total]
  float* dq;         // [total, H, D]
  float* dk;         // [total, Hkv, D]
  float* dv;
};

// ------------------------------------------------------- fake quantisers --

// One 16-element value of a code byte (element 2i in the low nibble) times
// the block scale, exact in either 16-bit type.
template <int DT>
__device__ __forceinline__ uint32_t fq_pair(uint32_t byte, float sv) {
  float v0, v1;
  e2m1x2_values(byte, v0, v1);
  return (uint32_t)f2h<DT>(__fmul_rn(v0, sv)) | ((uint32_t)f2h<DT>(__fmul_rn(v1, sv)) << 16);
}

// Rows blocked along the contiguous axis (Q, K): n_blocks blocks of 16.
template <int DT, bool SS>
__global__ void __launch_bounds__(256) qat_fq_rows_kernel(const uint16_t* __restrict__ x,
                                                          int64_t n_blocks, const uint32_t* amax,
                                                          float* g_out,
                                                          uint16_t* __restrict__ img) {
  const float g = tensor_scale_from_amax(*amax);
  if (blockIdx.x == 0 && threadIdx.x == 0) *g_out = g;
  for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < n_blocks;
       b += (int64_t)gridDim.x * blockDim.x) {
    float v[16];
    load16<DT>(x + b * 16, v);
    uint32_t lo, hi;
    const float sv = ue4m3_decode(quant_block16(v, g, SS, lo, hi));
    uint4 w0, w1;
    w0.x = fq_pair<DT>(lo & 0xFF, sv);
    w0.y = fq_pair<DT>((lo >> 8) & 0xFF, sv);
    w0.z = fq_pair<DT>((lo >> 16) & 0xFF, sv);
    w0.w = fq_pair<DT>(lo >> 24, sv);
    w1.x = fq_pair<DT>(hi & 0xFF, sv);
    w1.y = fq_pair<DT>((hi >> 8) & 0xFF, sv);
    w1.z = fq_pair<DT>((hi >> 16) & 0xFF, sv);
    w1.w = fq_pair<DT>(hi >> 24, sv);
    uint4* o = reinterpret_cast<uint4*>(img + b * 16);
    o[0] = w0;
    o[1] = w1;
  }
}

// V: blocks of 16 tokens of one channel from each sequence's start, the last
// block zero-padded.  grid (ceil(maxlen / 16), nseq); ncols = Hkv * d.
template <int DT, bool SS>
__global__ void __launch_bounds__(256) qat_fq_v_kernel(const uint16_t* __restrict__ v, SeqInfo si,
                                                       int ncols, const uint32_t* amax,
                                                       float* g_out, uint16_t* __restrict__ img) {
  int64_t st;
  int len;
  si.get(blockIdx.y, st, len);
  const float g = tensor_scale_from_amax(*amax);
  if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) *g_out = g;
  const int t0 = blockIdx.x * 16;
  if (t0 >= len) return;
  const int n = min(16, len - t0);
  for (int c = threadIdx.x; c < ncols; c += blockDim.x) {
    float x[16];
#pragma unroll
    for (int e = 0; e < 16; ++e)
      x[e] = e < n ? h2f<DT>(v[(st + t0 + e) * ncols + c]) : 0.0f;
    uint32_t lo, hi;
    const float sv = ue4m3_decode(quant_block16(x, g, SS, lo, hi));
#pragma unroll
    for (int e = 0; e < 16; e += 2) {
      const uint32_t byte = ((e < 8 ? lo : hi) >> (8 * ((e & 7) >> 1))) & 0xFF;
      const uint32_t pr = fq_pair<DT>(byte, sv);
      if (e < n) img[(st + t0 + e) * ncols + c] = (uint16_t)(pr & 0xFFFF);
      if (e + 1 < n) img[(st + t0 + e + 1) * ncols + c] = (uint16_t)(pr >> 16);
    }
  }
}

// ------------------------------------------------------------ warp MMAs --

template <int DT>
__device__ __forceinline__ uint32_t qpack2(float lo, float hi) {
  return (uint32_t)f2h<DT>(lo) | ((uint32_t)f2h<DT>(hi) << 16);
}

// c += a (16 x 16, row) * b (16 x 8, col), fp32 accumulate.  Fragments:
// a[0] (row g, k 2t..2t+1), a[1] (row g+8, same k), a[2] (row g, k 2t+8..),
// a[3] (row g+8, k 2t+8..); b0 (k 2t..2t+1, col g), b1 (k 2t+8.., col g);
// c[0..1] (row g, cols 2t, 2t+1), c[2..3] (row g+8, same cols); g = lane/4,
// t = lane%4.
template <int DT>
__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  if constexpr (DT == 1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  } else {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
}

// Shared-memory tiles are row-major 16-bit with LD = cols + 8 elements per
// row: a warp's fragment loads then touch 32 distinct banks, and every row
// starts on a 16-byte boundary.
template <int LD>
__device__ __forceinline__ void frag_a(uint32_t (&a)[4], const uint16_t* t, int row0, int k0,
                                       int g, int tq) {
  const uint16_t* p = t + (row0 + g) * LD + k0 + 2 * tq;
  a[0] = *reinterpret_cast<const uint32_t*>(p);
  a[1] = *reinterpret_cast<const uint32_t*>(p + 8 * LD);
  a[2] = *reinterpret_cast<const uint32_t*>(p + 8);
  a[3] = *reinterpret_cast<const uint32_t*>(p + 8 * LD + 8);
}

template <int LD>
__device__ __forceinline__ void frag_b(uint32_t& b0, uint32_t& b1, const uint16_t* t, int n0, int k0,
                                       int g, int tq) {
  const uint16_t* p = t + (n0 + g) * LD + k0 + 2 * tq;
  b0 = *reinterpret_cast<const uint32_t*>(p);
  b1 = *reinterpret_cast<const uint32_t*>(p + 8);
}

// B fragments of n-tiles n0 and n0 + 8 for the k-step at row k0 of a
// row-major tile whose rows run along the contraction (k) axis, transposed
// on the way in by ldmatrix: b[0], b[1] for n-tile n0, b[2], b[3] for n0 + 8.
// Lane l addresses row k0 + (l & 15), column n0 + 8 (l >> 4); rows are
// 16-byte aligned and 8 consecutive rows hit distinct banks (LD = cols + 8).
template <int LD>
__device__ __forceinline__ void frag_b_t2(uint32_t (&b)[4], const uint16_t* t, int k0, int n0,
                                          int lane) {
  const uint32_t a = smem_u32(t + (k0 + (lane & 15)) * LD + n0 + 8 * (lane >> 4));
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(b[0]), "=r"(b[1]), "=r"(b[2]), "=r"(b[3])
               : "r"(a));
}

// The A fragment of k-step s from accumulator tiles c[2s], c[2s+1] (the C
// layout of two n-tiles is the A layout of one 16-wide k-step).
template <int DT>
__device__ __forceinline__ void c_to_a(uint32_t (&a)[4], const float (&c0)[4],
                                       const float (&c1)[4]) {
  a[0] = qpack2<DT>(c0[0], c0[1]);
  a[1] = qpack2<DT>(c0[2], c0[3]);
  a[2] = qpack2<DT>(c1[0], c1[1]);
  a[3] = qpack2<DT>(c1[2], c1[3]);
}

// dS as the sum of two 16-bit parts, hi = round(dS) and lo = round(dS - hi),
// for two MMAs into one accumulator: rows of dS sum to zero, and rounding
// dS once would leave a residue that the products with K^ (whose channel
// means can be large) or Q^ magnify; the split carries about 16 bits.
template <int DT>
__device__ __forceinline__ void c_to_a_split(uint32_t (&hi)[4], uint32_t (&lo)[4],
                                             const float (&c0)[4], const float (&c1)[4]) {
  const float* src[2] = {c0, c1};
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const float* c = src[r >> 1] + 2 * (r & 1);
    const uint32_t h = qpack2<DT>(c[0], c[1]);
    hi[r] = h;
    lo[r] = qpack2<DT>(c[0] - h2f<DT>((uint16_t)(h & 0xFFFF)), c[1] - h2f<DT>((uint16_t)(h >> 16)));
  }
}

// Rows [r0, r0 + R) of a [tokens, nh, D] image (head h) -> tile [R][LD]
// through cp.async, 16 bytes a copy; rows at or past len are zero-filled.
// The caller commits the group and waits for it.
template <int D, int R, int LD>
__device__ __forceinline__ void stage_rows_async(uint16_t* t, const uint16_t* x, int64_t st,
                                                 int len, int r0, int nh, int h) {
  constexpr int CH = D / 8;
  for (int i = threadIdx.x; i < R * CH; i += blockDim.x) {
    const int r = i / CH, c = i % CH;
    const bool ok = r0 + r < len;
    const uint16_t* src = ok ? x + ((st + r0 + r) * nh + h) * D + 8 * c : x;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(t + r * LD + 8 * c)),
                 "l"(src), "r"(ok ? 16 : 0)
                 : "memory");
  }
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }

template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ float quad_max(float v) {
  v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 1));
  return fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 2));
}

// FP4 value of a probability already divided by sigma: the 16-key block's
// scale byte from amax (the block's largest scaled value), then the E2M1 code
// of x / scale; returns code value x scale (0 when the byte is 0).
// rcp: the correctly rounded reciprocals of the UE4M3 values by byte
// (qat_rcp_table), read instead of recomputed.
struct PBlock {
  float dec, rr;
  bool zero;
  __device__ __forceinline__ PBlock(float amax, const float* rcp) {
    const uint32_t sp = ue4m3(__fdiv_rn(amax, 6.0f));
    zero = sp == 0;
    dec = ue4m3_decode(sp);
    rr = rcp[sp];
  }
  __device__ __forceinline__ void apply(float x0, float x1, float& q0, float& q1) const {
    e2m1x2_roundtrip(__fmul_rn(x0, rr), __fmul_rn(x1, rr), q0, q1);
    q0 = zero ? 0.0f : __fmul_rn(q0, dec);
    q1 = zero ? 0.0f : __fmul_rn(q1, dec);
  }
};

// Fills rcp[b] = 1 / ue4m3_value(b) for the bytes 1..126 (rcp[0] = 0) in
// shared memory; the caller synchronises before use.
__device__ __forceinline__ void qat_rcp_table(float* rcp) {
  for (int b = threadIdx.x; b < 128; b += blockDim.x)
    rcp[b] = (b == 0 || b == 127) ? 0.0f : __frcp_rn(ue4m3_decode((uint32_t)b));
}

template <int D, int BLK>
struct QatFwdSmem {
  static constexpr int LD = D + 8;
  static constexpr int Q = 0;
  static constexpr int K = Q + kQatFwdRows * LD;  // two buffers of K and V each: the
  static constexpr int V = K + 2 * BLK * LD;   // key tile in use and the next one
  static constexpr int RCP = V + 2 * BLK * LD;  // 128 floats follow the 16-bit tiles
  static constexpr size_t BYTES = (size_t)RCP * 2 + 128 * 4;
};

// ------------------------------------------------------------- forward --
// grid (ceil(maxlen / 128) * H, nseq), 256 threads, the tile index the
// slowest: causal grids start the longest rows of every head first.  Warp w
// owns query rows 16w..16w+15 of the tile; the eight warps share the
// double-buffered K and V tiles.
//
// One pass over the key tiles with a running maximum m (log2 units): the
// FP4 image of P on a key tile does not depend on lse, because
// P / sigma = 2688 exp(S - max_tile S); the tile's sigma =
// exp(max_tile S - lse) / 2688 enters as exp2(mt - m) / 2688 x (the rescale
// of the running sums to the final m and the division by l), the same
// bookkeeping as O' = sum exp2(s - m) V / l.
template <int DT, int D, int BLK>
__global__ void __launch_bounds__(256) qat_fwd_kernel(QatParams p) {
  using L = QatFwdSmem<D, BLK>;
  constexpr int LD = L::LD, NT = BLK / 8, ND = D / 8, ROWS = kQatFwdRows;
  extern __shared__ __align__(16) uint16_t qsm[];
  uint16_t* sQ = qsm + L::Q;
  int64_t st;
  int len;
  p.si.get(blockIdx.y, st, len);
  const int tiles = (len + ROWS - 1) / ROWS;
  const int ti = (int)blockIdx.x / p.H, h = (int)blockIdx.x % p.H, hk = h / (p.H / p.Hkv);
  if (ti >= tiles) return;
  const int q0 = (p.causal ? tiles - 1 - ti : ti) * ROWS;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, tq = lane & 3;
  const float c2 = p.g[0] * p.g[1] * p.sc * kQatLog2e;
  const int row[2] = {q0 + 16 * warp + g, q0 + 16 * warp + g + 8};
  const int kend = p.causal ? min(len, q0 + ROWS) : len;
  const int ntiles = (kend + BLK - 1) / BLK;

  auto issue = [&](int kt) {
    const int buf = kt & 1;
    stage_rows_async<D, BLK, LD>(qsm + L::K + buf * BLK * LD, p.ki, st, len, kt * BLK, p.Hkv, hk);
    stage_rows_async<D, BLK, LD>(qsm + L::V + buf * BLK * LD, p.vi, st, len, kt * BLK, p.Hkv, hk);
  };
  float* s_rcp = reinterpret_cast<float*>(qsm + L::RCP);
  qat_rcp_table(s_rcp);  // visible after the first barrier of the loop
  stage_rows_async<D, ROWS, LD>(sQ, p.qi, st, len, q0, p.H, h);
  issue(0);
  cp_async_commit();

  float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.0f, 0.0f};
  float o[ND][4], oh[ND][4];
#pragma unroll
  for (int n = 0; n < ND; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) o[n][e] = oh[n][e] = 0.0f;
  for (int kt = 0; kt < ntiles; ++kt) {
    const uint16_t* sK = qsm + L::K + (kt & 1) * BLK * LD;
    const uint16_t* sV = qsm + L::V + (kt & 1) * BLK * LD;
    if (kt + 1 < ntiles) {
      issue(kt + 1);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const int j0 = kt * BLK;
    float s[NT][4];
#pragma unroll
    for (int n = 0; n < NT; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.0f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      uint32_t a[4];
      frag_a<LD>(a, sQ, 16 * warp, 16 * kk, g, tq);
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        uint32_t b0, b1;
        frag_b<LD>(b0, b1, sK, 8 * n, 16 * kk, g, tq);
        mma16816<DT>(s[n], a, b0, b1);
      }
    }
    // scores in log2 units, masked; tile row maxima; running maxima
    float mt[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int j = j0 + 8 * n + 2 * tq + (e & 1), i = row[e >> 1];
        const bool ok = j < len && (!p.causal || j <= i);
        s[n][e] = ok ? s[n][e] * c2 : -INFINITY;
        mt[e >> 1] = fmaxf(mt[e >> 1], s[n][e]);
      }
    float fct[2], inv2688 = 1.0f / kTensorScaleDiv;
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      mt[r] = quad_max(mt[r]);
      const float mn = fmaxf(m[r], mt[r]);
      const float alpha = (m[r] == -INFINITY || mn == -INFINITY) ? 0.0f : exp2f(m[r] - mn);
      m[r] = mn;
      l[r] *= alpha;
#pragma unroll
      for (int n = 0; n < ND; ++n) {
        o[n][2 * r] *= alpha;
        o[n][2 * r + 1] *= alpha;
        oh[n][2 * r] *= alpha;
        oh[n][2 * r + 1] *= alpha;
      }
      // sigma of this tile relative to the running maximum
      fct[r] = mt[r] == -INFINITY ? 0.0f : exp2f(mt[r] - mn) * inv2688;
    }
    // a row without a visible key in the tile has s = -inf throughout:
    // finite references keep its exponentials at 0
    const float mr[2] = {m[0] == -INFINITY ? 0.0f : m[0], m[1] == -INFINITY ? 0.0f : m[1]};
    const float mtr[2] = {mt[0] == -INFINITY ? 0.0f : mt[0], mt[1] == -INFINITY ? 0.0f : mt[1]};
#pragma unroll
    for (int b = 0; b < NT / 2; ++b) {
      float qv[2][4], pe[2][4];  // P^ / (tile factor) and exp2(s - m), C layout
#pragma unroll
      for (int u = 0; u < 2; ++u)
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const float s0 = s[2 * b + u][2 * r], s1 = s[2 * b + u][2 * r + 1];
          pe[u][2 * r] = exp2f(s0 - mr[r]);
          pe[u][2 * r + 1] = exp2f(s1 - mr[r]);
          l[r] += pe[u][2 * r] + pe[u][2 * r + 1];
          // P / sigma of the oracle's reading: 2688 exp(S - max_tile S)
          qv[u][2 * r] = kTensorScaleDiv * exp2f(s0 - mtr[r]);
          qv[u][2 * r + 1] = kTensorScaleDiv * exp2f(s1 - mtr[r]);
        }
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const PBlock pb(quad_max(fmaxf(fmaxf(qv[0][2 * r], qv[0][2 * r + 1]),
                                       fmaxf(qv[1][2 * r], qv[1][2 * r + 1]))),
                        s_rcp);
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          float y0, y1;
          pb.apply(qv[u][2 * r], qv[u][2 * r + 1], y0, y1);
          qv[u][2 * r] = __fmul_rn(y0, fct[r]);
          qv[u][2 * r + 1] = __fmul_rn(y1, fct[r]);
        }
      }
      // O' carries P in two parts: it sets D = rowsum(dO o O') of the
      // backward, whose error reaches dQ multiplied by the keys' means
      uint32_t aq[4], ph[4], pl[4];
      c_to_a<DT>(aq, qv[0], qv[1]);
      c_to_a_split<DT>(ph, pl, pe[0], pe[1]);
#pragma unroll
      for (int n = 0; n < ND; n += 2) {
        uint32_t bb[4];
        frag_b_t2<LD>(bb, sV, 16 * b, 8 * n, lane);
        mma16816<DT>(oh[n], ph, bb[0], bb[1]);
        mma16816<DT>(oh[n + 1], ph, bb[2], bb[3]);
        mma16816<DT>(o[n], aq, bb[0], bb[1]);
        mma16816<DT>(o[n + 1], aq, bb[2], bb[3]);
        mma16816<DT>(oh[n], pl, bb[0], bb[1]);
        mma16816<DT>(oh[n + 1], pl, bb[2], bb[3]);
      }
    }
    __syncthreads();  // every read of this buffer done before it is refilled
  }
  const float gv = p.g[2];
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    float t = l[r];
    t += __shfl_xor_sync(0xffffffffu, t, 1);
    t += __shfl_xor_sync(0xffffffffu, t, 2);
    if (row[r] >= len) continue;
    if (tq == 0) p.lse[(int64_t)h * p.total + st + row[r]] = (m[r] + log2f(t)) * kQatLn2;
    const float sc_out = gv / t;
    const int64_t base = ((st + row[r]) * p.H + h) * D;
#pragma unroll
    for (int n = 0; n < ND; ++n) {
      const int c = 8 * n + 2 * tq;
      *reinterpret_cast<uint32_t*>(p.out + base + c) =
          qpack2<DT>(o[n][2 * r] * sc_out, o[n][2 * r + 1] * sc_out);
      *reinterpret_cast<float2*>(p.out_hp + base + c) =
          make_float2(oh[n][2 * r] * sc_out, oh[n][2 * r + 1] * sc_out);
    }
  }
}

// D = rowsum(dO o O') per (token, head); one warp per row.
template <int DT, int D>
__global__ void __launch_bounds__(256) qat_rowdot_kernel(const uint16_t* __restrict__ dout,
                                                         const float* __restrict__ out_hp,
                                                         int64_t total, int H,
                                                         float* __restrict__ dsum) {
  const int lane = threadIdx.x & 31;
  const int64_t nrows = total * H;
  for (int64_t rr = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; rr < nrows;
       rr += ((int64_t)gridDim.x * blockDim.x) >> 5) {
    float acc = 0.0f;
#pragma unroll
    for (int c = lane; c < D; c += 32) acc = fmaf(h2f<DT>(dout[rr * D + c]), out_hp[rr * D + c], acc);
#pragma unroll
    for (int m2 = 16; m2 >= 1; m2 >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, m2);
    if (lane == 0) dsum[(rr % H) * total + rr / H] = acc;
  }
}

template <int D, int BLK>
struct QatKvSmem {
  static constexpr int LD = D + 8, NW = BLK / 16;
  static constexpr int K = 0;
  static constexpr int V = K + BLK * LD;
  static constexpr int Q = V + BLK * LD;             // two buffers of [64][LD] each:
  static constexpr int DO = Q + 2 * kQatChunk * LD;  // the chunk in use and the next one
  static constexpr int END16 = DO + 2 * kQatChunk * LD;  // 16-bit elements; fp32 arrays follow
  // fp32: lse (log2 units) [2][64], D [2][64], column maxima [NW][64], the
  // columns' 2688 / max and max / 2688 [2][64], UE4M3 reciprocals [128]
  static constexpr size_t BYTES =
      (size_t)END16 * 2 + (size_t)(6 + NW) * kQatChunk * 4 + 128 * 4;
};

// ------------------------------------------------- backward: dK and dV --
// grid (ceil(maxlen / BLK) * Hkv, nseq), BLK / 16 warps, the key tile the
// slowest (causal grids start the tiles with the most queries first); warp w
// owns keys 16w..16w+15 of the tile (one 16-key block of the P
// quantisation).
template <int DT, int D, int BLK>
__global__ void __launch_bounds__(BLK * 2) qat_bwd_kv_kernel(QatParams p) {
  using L = QatKvSmem<D, BLK>;
  constexpr int LD = L::LD, NW = L::NW, QC = kQatChunk, NQ = QC / 8, ND = D / 8;
  extern __shared__ __align__(16) uint16_t qsm[];
  uint16_t* sK = qsm + L::K;
  uint16_t* sV = qsm + L::V;
  float* s_lse2b = reinterpret_cast<float*>(qsm + L::END16);  // [2][QC]
  float* s_Db = s_lse2b + 2 * QC;                               // [2][QC]
  float* s_cmax = s_Db + 2 * QC;                                // [NW][QC]
  float* s_cinv = s_cmax + NW * QC;                             // [QC]
  float* s_csig = s_cinv + QC;                                  // [QC]
  float* s_rcp = s_csig + QC;                                   // [128]
  int64_t st;
  int len;
  p.si.get(blockIdx.y, st, len);
  const int j0 = (int)blockIdx.x / p.Hkv * BLK, hk = (int)blockIdx.x % p.Hkv, grp = p.H / p.Hkv;
  if (j0 >= len) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, tq = lane & 3;
  const float c2 = p.g[0] * p.g[1] * p.sc * kQatLog2e, gv = p.g[2];
  const int key[2] = {j0 + 16 * warp + g, j0 + 16 * warp + g + 8};
  // query chunks: every head of the group, from the first chunk that sees a
  // key of this tile; chunk it + 1 is fetched while chunk it is computed
  const int qstart = p.causal ? j0 / QC * QC : 0;
  const int nch = (len - qstart + QC - 1) / QC;
  const int n_it = grp * nch;
  auto issue = [&](int it) {
    const int buf = it & 1, h = hk * grp + it / nch, qc0 = qstart + (it % nch) * QC;
    stage_rows_async<D, QC, LD>(qsm + L::Q + buf * QC * LD, p.qi, st, len, qc0, p.H, h);
    stage_rows_async<D, QC, LD>(qsm + L::DO + buf * QC * LD, p.dout, st, len, qc0, p.H, h);
    for (int i = threadIdx.x; i < QC; i += blockDim.x) {
      const bool ok = qc0 + i < len;
      s_lse2b[buf * QC + i] = ok ? p.lse[(int64_t)h * p.total + st + qc0 + i] * kQatLog2e : 0.0f;
      s_Db[buf * QC + i] = ok ? p.dsum[(int64_t)h * p.total + st + qc0 + i] : 0.0f;
    }
  };

  qat_rcp_table(s_rcp);  // visible after the first barrier of the loop
  stage_rows_async<D, BLK, LD>(sK, p.ki, st, len, j0, p.Hkv, hk);
  stage_rows_async<D, BLK, LD>(sV, p.vi, st, len, j0, p.Hkv, hk);
  issue(0);
  cp_async_commit();
  float dk[ND][4], dv[ND][4];
#pragma unroll
  for (int n = 0; n < ND; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) dk[n][e] = dv[n][e] = 0.0f;

  for (int it = 0; it < n_it; ++it) {
    if (it + 1 < n_it) {
      issue(it + 1);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    {
      const int buf = it & 1, qc0 = qstart + (it % nch) * QC;
      const uint16_t* sQ = qsm + L::Q + buf * QC * LD;
      const uint16_t* sdO = qsm + L::DO + buf * QC * LD;
      const float* s_lse2 = s_lse2b + buf * QC;
      const float* s_D = s_Db + buf * QC;
      // S^T (keys x queries) and P^T
      float s[NQ][4];
#pragma unroll
      for (int n = 0; n < NQ; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.0f;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        uint32_t a[4];
        frag_a<LD>(a, sK, 16 * warp, 16 * kk, g, tq);
#pragma unroll
        for (int n = 0; n < NQ; ++n) {
          uint32_t b0, b1;
          frag_b<LD>(b0, b1, sQ, 8 * n, 16 * kk, g, tq);
          mma16816<DT>(s[n], a, b0, b1);
        }
      }
#pragma unroll
      for (int n = 0; n < NQ; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int il = 8 * n + 2 * tq + (e & 1), i = qc0 + il, j = key[e >> 1];
          const bool ok = j < len && i < len && (!p.causal || j <= i);
          s[n][e] = ok ? exp2f(s[n][e] * c2 - s_lse2[il]) : 0.0f;
        }
      // per query: max of P over the key tile (all warps)
#pragma unroll
      for (int n = 0; n < NQ; ++n)
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          float v = fmaxf(s[n][c], s[n][c + 2]);
          v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
          v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
          v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 16));
          if (g == 0) s_cmax[warp * QC + 8 * n + 2 * tq + c] = v;
        }
      __syncthreads();
      // per query column, once: the max over the key tile and its factors
      for (int c = threadIdx.x; c < QC; c += blockDim.x) {
        float cm = 0.0f;
#pragma unroll
        for (int w = 0; w < NW; ++w) cm = fmaxf(cm, s_cmax[w * QC + c]);
        s_cinv[c] = cm > 0.0f ? __fdiv_rn(kTensorScaleDiv, cm) : 0.0f;
        s_csig[c] = __fdiv_rn(cm, kTensorScaleDiv);
      }
      __syncthreads();
      // dV += (P^)^T dO, one 16-query k-step at a time
#pragma unroll
      for (int b = 0; b < NQ / 2; ++b) {
        float qv[2][4];
#pragma unroll
        for (int u = 0; u < 2; ++u)
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            const int il = 8 * (2 * b + u) + 2 * tq + c;
            const float inv = s_cinv[il], sig = s_csig[il];
            const float x0 = __fmul_rn(s[2 * b + u][c], inv), x1 = __fmul_rn(s[2 * b + u][c + 2], inv);
            float am = fmaxf(x0, x1);
            am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 4));
            am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 8));
            am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 16));
            const PBlock pb(am, s_rcp);
            float y0, y1;
            pb.apply(x0, x1, y0, y1);
            qv[u][c] = __fmul_rn(y0, sig);
            qv[u][c + 2] = __fmul_rn(y1, sig);
          }
        uint32_t a[4];
        c_to_a<DT>(a, qv[0], qv[1]);
#pragma unroll
        for (int n = 0; n < ND; n += 2) {
          uint32_t bb[4];
          frag_b_t2<LD>(bb, sdO, 16 * b, 8 * n, lane);
          mma16816<DT>(dv[n], a, bb[0], bb[1]);
          mma16816<DT>(dv[n + 1], a, bb[2], bb[3]);
        }
      }
      // dP^T = V^ dO^T, dS^T = P^T o (dP^T - D)
      float dp[NQ][4];
#pragma unroll
      for (int n = 0; n < NQ; ++n) dp[n][0] = dp[n][1] = dp[n][2] = dp[n][3] = 0.0f;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        uint32_t a[4];
        frag_a<LD>(a, sV, 16 * warp, 16 * kk, g, tq);
#pragma unroll
        for (int n = 0; n < NQ; ++n) {
          uint32_t b0, b1;
          frag_b<LD>(b0, b1, sdO, 8 * n, 16 * kk, g, tq);
          mma16816<DT>(dp[n], a, b0, b1);
        }
      }
#pragma unroll
      for (int n = 0; n < NQ; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int il = 8 * n + 2 * tq + (e & 1);
          dp[n][e] = s[n][e] * (dp[n][e] * gv - s_D[il]);
        }
      // dK += dS^T Q^
#pragma unroll
      for (int b = 0; b < NQ / 2; ++b) {
        uint32_t ah[4], al[4];
        c_to_a_split<DT>(ah, al, dp[2 * b], dp[2 * b + 1]);
#pragma unroll
        for (int n = 0; n < ND; n += 2) {
          uint32_t bb[4];
          frag_b_t2<LD>(bb, sQ, 16 * b, 8 * n, lane);
          mma16816<DT>(dk[n], ah, bb[0], bb[1]);
          mma16816<DT>(dk[n + 1], ah, bb[2], bb[3]);
          mma16816<DT>(dk[n], al, bb[0], bb[1]);
          mma16816<DT>(dk[n + 1], al, bb[2], bb[3]);
        }
      }
    }
    __syncthreads();  // every read of this buffer done before it is refilled
  }
  const float kscale = p.g[0] * p.sc;
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    if (key[r] >= len) continue;
    const int64_t base = ((st + key[r]) * p.Hkv + hk) * D;
#pragma unroll
    for (int n = 0; n < ND; ++n) {
      const int c = 8 * n + 2 * tq;
      *reinterpret_cast<float2*>(p.dk + base + c) =
          make_float2(dk[n][2 * r] * kscale, dk[n][2 * r + 1] * kscale);
      *reinterpret_cast<float2*>(p.dv + base + c) = make_float2(dv[n][2 * r], dv[n][2 * r + 1]);
    }
  }
}

template <int D>
struct QatQSmem {
  static constexpr int LD = D + 8;
  static constexpr int Q = 0;
  static constexpr int DO = Q + kQatRows * LD;
  static constexpr int K = DO + kQatRows * LD;  // two buffers each: the key chunk
  static constexpr int V = K + 2 * kQatChunk * LD;  // in use and the next one
  static constexpr size_t BYTES = (size_t)(V + 2 * kQatChunk * LD) * 2;
};

// ------------------------------------------------------ backward: dQ --
// grid (ceil(maxlen / 64) * H, nseq), 128 threads, the tile index the
// slowest (causal grids start the longest rows first); warp w owns query
// rows 16w..16w+15; keys in chunks of 64.
template <int DT, int D>
__global__ void __launch_bounds__(128) qat_bwd_q_kernel(QatParams p) {
  using L = QatQSmem<D>;
  constexpr int LD = L::LD, KC = kQatChunk, NK = KC / 8, ND = D / 8;
  extern __shared__ __align__(16) uint16_t qsm[];
  uint16_t* sQ = qsm + L::Q;
  uint16_t* sdO = qsm + L::DO;
  int64_t st;
  int len;
  p.si.get(blockIdx.y, st, len);
  const int tiles = (len + kQatRows - 1) / kQatRows;
  const int ti = (int)blockIdx.x / p.H, h = (int)blockIdx.x % p.H, hk = h / (p.H / p.Hkv);
  if (ti >= tiles) return;
  const int q0 = (p.causal ? tiles - 1 - ti : ti) * kQatRows;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, tq = lane & 3;
  const float c2 = p.g[0] * p.g[1] * p.sc * kQatLog2e, gv = p.g[2];
  const int row[2] = {q0 + 16 * warp + g, q0 + 16 * warp + g + 8};
  float lse2[2], dsum[2];
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const bool ok = row[r] < len;
    lse2[r] = ok ? p.lse[(int64_t)h * p.total + st + row[r]] * kQatLog2e : 0.0f;
    dsum[r] = ok ? p.dsum[(int64_t)h * p.total + st + row[r]] : 0.0f;
  }
  float dq[ND][4];
#pragma unroll
  for (int n = 0; n < ND; ++n) dq[n][0] = dq[n][1] = dq[n][2] = dq[n][3] = 0.0f;
  const int kend = p.causal ? min(len, q0 + kQatRows) : len;
  const int n_it = (kend + KC - 1) / KC;
  // key chunk it + 1 is fetched while chunk it is computed
  auto issue = [&](int it) {
    const int buf = it & 1;
    stage_rows_async<D, KC, LD>(qsm + L::K + buf * KC * LD, p.ki, st, len, it * KC, p.Hkv, hk);
    stage_rows_async<D, KC, LD>(qsm + L::V + buf * KC * LD, p.vi, st, len, it * KC, p.Hkv, hk);
  };
  stage_rows_async<D, kQatRows, LD>(sQ, p.qi, st, len, q0, p.H, h);
  stage_rows_async<D, kQatRows, LD>(sdO, p.dout, st, len, q0, p.H, h);
  issue(0);
  cp_async_commit();
  for (int it = 0; it < n_it; ++it) {
    const int k0 = it * KC;
    const uint16_t* sK = qsm + L::K + (it & 1) * KC * LD;
    const uint16_t* sV = qsm + L::V + (it & 1) * KC * LD;
    if (it + 1 < n_it) {
      issue(it + 1);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    float s[NK][4], dp[NK][4];
#pragma unroll
    for (int n = 0; n < NK; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) s[n][e] = dp[n][e] = 0.0f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      uint32_t aq[4], ad[4];
      frag_a<LD>(aq, sQ, 16 * warp, 16 * kk, g, tq);
      frag_a<LD>(ad, sdO, 16 * warp, 16 * kk, g, tq);
#pragma unroll
      for (int n = 0; n < NK; ++n) {
        uint32_t b0, b1;
        frag_b<LD>(b0, b1, sK, 8 * n, 16 * kk, g, tq);
        mma16816<DT>(s[n], aq, b0, b1);
        frag_b<LD>(b0, b1, sV, 8 * n, 16 * kk, g, tq);
        mma16816<DT>(dp[n], ad, b0, b1);
      }
    }
#pragma unroll
    for (int n = 0; n < NK; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int j = k0 + 8 * n + 2 * tq + (e & 1), r = e >> 1, i = row[r];
        const bool ok = j < len && i < len && (!p.causal || j <= i);
        const float pr = ok ? exp2f(s[n][e] * c2 - lse2[r]) : 0.0f;
        dp[n][e] = pr * (dp[n][e] * gv - dsum[r]);
      }
#pragma unroll
    for (int b = 0; b < NK / 2; ++b) {
      uint32_t ah[4], al[4];
      c_to_a_split<DT>(ah, al, dp[2 * b], dp[2 * b + 1]);
#pragma unroll
      for (int n = 0; n < ND; n += 2) {
        uint32_t bb[4];
        frag_b_t2<LD>(bb, sK, 16 * b, 8 * n, lane);
        mma16816<DT>(dq[n], ah, bb[0], bb[1]);
        mma16816<DT>(dq[n + 1], ah, bb[2], bb[3]);
        mma16816<DT>(dq[n], al, bb[0], bb[1]);
        mma16816<DT>(dq[n + 1], al, bb[2], bb[3]);
      }
    }
    __syncthreads();  // every read of this buffer done before it is refilled
  }
  const float qscale = p.g[1] * p.sc;
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    if (row[r] >= len) continue;
    const int64_t base = ((st + row[r]) * p.H + h) * D;
#pragma unroll
    for (int n = 0; n < ND; ++n)
      *reinterpret_cast<float2*>(p.dq + base + 8 * n + 2 * tq) =
          make_float2(dq[n][2 * r] * qscale, dq[n][2 * r + 1] * qscale);
  }
}

}  // namespace thrift
