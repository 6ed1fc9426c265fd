// Attn-QAT attention: forward on fake-quantised NVFP4 operands and the
// backward with FP4 recomputation of the probabilities, on the Blackwell
// tensor cores (tcgen05 kind::f16, fp32 accumulators in tensor memory).
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
// Operand tiles.  Every 16-bit operand lives in HBM as tiles of 128 rows:
// D / 64 regions of [128 rows][128 B] with the 128-byte swizzle, element
// (r, c) at (c / 64) * 16384 + swizzle(r, 2 (c % 64)).  A tile is a K-major
// operand when its rows are the M or N dimension of a product and an
// MN-major one when its rows run along the contraction, so no transposed
// copy is ever made: O = P^ V^ and dQ = dS K^ read V^ and K^ MN-major,
// dV = P^T dO and dK = dS^T Q^ read both operands MN-major.  The tiles of a
// sequence s that starts at token st are slots st / 128 + s + t
// (t < ceil(len / 128)) of its head; nslot = total / 128 + nseq bounds them.
// The fake-quantised elements (E2M1 value x UE4M3 block scale) are exact in
// the 16-bit input type; the tensor scales multiply the fp32 accumulators.
// P^ enters the products rounded to the 16-bit type, P (of O') and the dS
// of dQ as two 16-bit parts, hi = round(x) and lo = round(x - hi).  Rows of
// dS sum to zero, so in dQ = dS K^ (a contraction over the keys) K^'s
// channel means cancel in exact arithmetic and would multiply the residue of
// a single rounding; dK = dS^T Q^ contracts over the queries, where dS has no
// such structure, and takes dS rounded once.
//
// Kernels.
//   qat_fq_tile_kernel      Q, K (blocks along d) or V (blocks along the
//                           tokens) -> fake-quantised tiles, one 128-row
//                           tile per CTA staged in shared memory
//   qat_rowdot_tile_kernel  D = rowsum(dO o O') and the dO tiles
//   qat_fwd_kernel          per 128 query rows, one pass over the key
//                           tiles: S, P and P^, O += P^ V^ and O' += P V^
//                           against a per-row reference maximum that moves
//                           (rescaling O and O') only when a tile passes it
//                           by more than 2^8, lse
//   qat_bwd_q_kernel        per 128 query rows: S, dP, dS; dQ += dS K^
//   qat_bwd_kv_kernel       per 128-key tile over the 128-row query chunks
//                           of its query heads: S, dP, P, P^, dS;
//                           dV += P^T dO, dK += dS^T Q^
// The three attention kernels have ten warps: warps 0-7 own the rows (two
// per tensor-memory lane quarter, each taking half of the 128 columns of
// a score tile), warp 8 moves tiles with bulk copies, warp 9 issues the MMAs
// (the whole warp runs the loop and its waits, one elected lane issues).
// Every wait is bounded.  Where the A operand of a product has the query
// rows on its M side (P of O' in the forward, dS of dQ), the
// rows write it to tensor memory and the MMA reads it from there: no
// shared-memory round trip.
#pragma once
#include "attn.cuh"

namespace thrift {

constexpr float kQatLog2e = 1.4426950408889634f;
constexpr float kQatLn2 = 0.6931471805599453f;
constexpr float kLog2TensorScaleDiv = 11.392317422778761f;  // log2(2688)

constexpr int kQtWarps = 8;             // row-owning warps, two per lane quarter
constexpr int kQtProducer = kQtWarps;   // warp 8
constexpr int kQtMma = kQtWarps + 1;    // warp 9
constexpr int kQtThreads = 32 * (kQtWarps + 2);
constexpr uint32_t kQtPTile = 128u * 128u * 2u;  // [128][128] 16-bit
constexpr uint32_t kQtShBytes = 2048;            // barriers, flags, tables
constexpr int kQtRing = 4;                       // K/V tile slots of the forward

__host__ __device__ constexpr uint32_t qt_tile_bytes(int d) { return 128u * (uint32_t)d * 2u; }
__host__ __device__ constexpr int64_t qat_nslot(int64_t total, int nseq) {
  return total / 128 + nseq;
}

struct QatParams {
  const uint8_t* qt;   // fake-quantised tiles: Q [H][nslot], K, V [Hkv][nslot]
  const uint8_t* kt;
  const uint8_t* vt;
  const uint8_t* dot;  // dO tiles [H][nslot] (backward)
  int64_t nslot;
  const float* g;      // tensor scales of Q, K, V
  SeqInfo si;
  int H, Hkv;
  int64_t total;
  int causal;
  float sc;            // 1 / sqrt(d)
  uint16_t* out;       // forward: O [total, H, D] in the input type
  float* out_hp;       // forward: O' [total, H, D]
  float* lse;          // [H, total], natural log
  const float* dsum;   // D [H, total]
  float* dq;           // [total, H, D]
  float* dk;           // [total, Hkv, D]
  float* dv;
};

__device__ __forceinline__ int64_t qat_slot(int hd, int64_t nslot, int64_t st, int seq, int t) {
  return (int64_t)hd * nslot + st / 128 + seq + t;
}

// Byte offset of element (r, c) of a 128-row tile.
__device__ __forceinline__ uint32_t qt_elem(int r, int c) {
  return (uint32_t)(c >> 6) * 16384u + swz_offset((uint32_t)r, (uint32_t)(c & 63) * 2u, 128);
}

// K-major operand of a 128-row tile, K-step s (16 elements along the row):
// 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t qt_desc_k(uint32_t tile, int s) {
  return make_sdesc(tile + (uint32_t)(s >> 2) * 16384u + 32u * (uint32_t)(s & 3), 16, 1024,
                    SW_128B);
}

// MN-major operand of a 128-row tile whose rows run along the contraction:
// K-step s takes rows 16s..16s+15; the 64-element groups along M or N are
// 16384 bytes apart (leading offset), the 8-row groups along K 1024
// (stride offset).
__device__ __forceinline__ uint64_t qt_desc_mn(uint32_t tile, int s) {
  return make_sdesc(tile + (uint32_t)s * 2048u, 16384, 1024, SW_128B);
}

constexpr uint32_t kIdescAmn = 1u << 15, kIdescBmn = 1u << 16;

// ------------------------------------------------------- fake quantisers --

// One 16-element value of a code byte (element 2i in the low nibble) times
// the block scale, exact in either 16-bit type.
template <int DT>
__device__ __forceinline__ uint32_t fq_pair(uint32_t byte, float sv) {
  float v0, v1;
  e2m1x2_values(byte, v0, v1);
  return (uint32_t)f2h<DT>(__fmul_rn(v0, sv)) | ((uint32_t)f2h<DT>(__fmul_rn(v1, sv)) << 16);
}

// x [total, nh, D] -> fake-quantised tiles.  COLS = false: blocks of 16
// along d (Q, K); COLS = true: blocks of 16 tokens of one channel from the
// sequence's start (V; the 128-row tiles hold whole blocks).  Rows past the
// sequence end are zero.  grid (ceil(maxlen / 128), nh, nseq), 256 threads.
template <int DT, bool SS, int D, bool COLS>
__global__ void __launch_bounds__(256) qat_fq_tile_kernel(const uint16_t* __restrict__ x,
                                                          SeqInfo si, int nh, int64_t nslot,
                                                          const uint32_t* amax, float* g_out,
                                                          uint8_t* __restrict__ tiles) {
  __shared__ __align__(128) uint8_t img[128 * D * 2];
  const int t = blockIdx.x, hd = blockIdx.y, seq = blockIdx.z;
  const float g = tensor_scale_from_amax(*amax);
  if ((t | hd | seq) == 0 && threadIdx.x == 0) *g_out = g;
  int64_t st;
  int len;
  si.get(seq, st, len);
  const int r0 = t * 128;
  if (r0 >= len) return;
  const int n = min(128, len - r0);
  constexpr int NB = 128 * D / 16;
  for (int b = threadIdx.x; b < NB; b += blockDim.x) {
    float v[16];
    int r, c;
    if constexpr (!COLS) {
      r = b / (D / 16);
      c = (b % (D / 16)) * 16;
      if (r < n) {
        load16<DT>(x + ((st + r0 + r) * nh + hd) * D + c, v);
      } else {
#pragma unroll
        for (int e = 0; e < 16; ++e) v[e] = 0.0f;
      }
    } else {
      c = b % D;
      r = (b / D) * 16;
#pragma unroll
      for (int e = 0; e < 16; ++e)
        v[e] = r + e < n ? h2f<DT>(x[((st + r0 + r + e) * nh + hd) * D + c]) : 0.0f;
    }
    uint32_t lo, hi;
    const float sv = ue4m3_decode(quant_block16(v, g, SS, lo, hi));
    uint32_t w[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) w[i] = fq_pair<DT>(((i < 4 ? lo : hi) >> (8 * (i & 3))) & 0xFF, sv);
    if constexpr (!COLS) {
      *reinterpret_cast<uint4*>(img + qt_elem(r, c)) = make_uint4(w[0], w[1], w[2], w[3]);
      *reinterpret_cast<uint4*>(img + qt_elem(r, c + 8)) = make_uint4(w[4], w[5], w[6], w[7]);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        *reinterpret_cast<uint16_t*>(img + qt_elem(r + 2 * i, c)) = (uint16_t)(w[i] & 0xFFFF);
        *reinterpret_cast<uint16_t*>(img + qt_elem(r + 2 * i + 1, c)) = (uint16_t)(w[i] >> 16);
      }
    }
  }
  __syncthreads();
  uint4* dst = reinterpret_cast<uint4*>(tiles + qat_slot(hd, nslot, st, seq, t) * qt_tile_bytes(D));
  const uint4* src = reinterpret_cast<const uint4*>(img);
  for (int i = threadIdx.x; i < 128 * D / 8; i += blockDim.x) dst[i] = src[i];
}

// D = rowsum(dO o O') per (token, head), and the dO tiles.  One thread per
// 16-byte chunk of dO; the D / 8 chunks of a row are consecutive lanes.
// grid (ceil(maxlen / 128), H, nseq), 256 threads.
template <int DT, int D>
__global__ void __launch_bounds__(256) qat_rowdot_tile_kernel(
    const uint16_t* __restrict__ dout, const float* __restrict__ out_hp, SeqInfo si, int H,
    int64_t total, int64_t nslot, float* __restrict__ dsum, uint8_t* __restrict__ tiles) {
  constexpr int CH = D / 8;
  const int t = blockIdx.x, h = blockIdx.y, seq = blockIdx.z;
  int64_t st;
  int len;
  si.get(seq, st, len);
  const int r0 = t * 128;
  if (r0 >= len) return;
  uint8_t* tile = tiles + qat_slot(h, nslot, st, seq, t) * qt_tile_bytes(D);
  for (int i = threadIdx.x; i < 128 * CH; i += blockDim.x) {  // 128 * CH: a multiple of 256
    const int r = i / CH, c = i % CH;
    const bool ok = r0 + r < len;
    uint4 v = make_uint4(0, 0, 0, 0);
    float acc = 0.0f;
    if (ok) {
      const int64_t e = ((st + r0 + r) * H + h) * D + 8 * c;
      v = __ldg(reinterpret_cast<const uint4*>(dout + e));
      const float4 o0 = __ldg(reinterpret_cast<const float4*>(out_hp + e));
      const float4 o1 = __ldg(reinterpret_cast<const float4*>(out_hp + e) + 1);
      const float o[8] = {o0.x, o0.y, o0.z, o0.w, o1.x, o1.y, o1.z, o1.w};
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        acc = fmaf(h2f<DT>((uint16_t)(w[k] & 0xFFFF)), o[2 * k], acc);
        acc = fmaf(h2f<DT>((uint16_t)(w[k] >> 16)), o[2 * k + 1], acc);
      }
    }
#pragma unroll
    for (int m = CH / 2; m >= 1; m >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, m);
    if (ok && c == 0) dsum[(int64_t)h * total + st + r0 + r] = acc;
    *reinterpret_cast<uint4*>(tile + qt_elem(r, 8 * c)) = v;
  }
}

// ------------------------------------------------------ shared helpers --

// FP4 value of a probability already divided by sigma: the 16-key block's
// scale byte from amax (the block's largest scaled value), then the E2M1 code
// of x / scale; returns code value x scale (0 when the byte is 0).
// rcp: the correctly rounded reciprocals of the UE4M3 values by byte
// (qat_rcp_table), read instead of recomputed.
struct PBlock {
  float dec, rr;
  bool zero;
  // by_mul: amax / 6 as amax times the fp32 value of 1/6 (a multiply
  // instead of a division; it can differ from the quotient by one fp32 ulp,
  // which moves the UE4M3 byte only when amax / 6 lies that close to a
  // rounding boundary of the byte)
  __device__ __forceinline__ PBlock(float amax, const float* rcp, bool by_mul = false) {
    const uint32_t sp = ue4m3(by_mul ? amax * (1.0f / 6.0f) : __fdiv_rn(amax, 6.0f));
    zero = sp == 0;
    dec = ue4m3_decode(sp);
    rr = rcp[sp];
  }
  // The 16-bit pair of the FP4 values of x0, x1 times t (t = sigma): the
  // code values times (block scale x t), 0 for a zero block.
  template <int DT>
  __device__ __forceinline__ uint32_t scaled(float x0, float x1, float t) const {
    float q0, q1;
    e2m1x2_roundtrip(__fmul_rn(x0, rr), __fmul_rn(x1, rr), q0, q1);
    const float f = zero ? 0.0f : dec * t;
    return pack2<DT>(q0 * f, q1 * f);
  }
};

// Fills rcp[b] = 1 / ue4m3_value(b) for the bytes 1..126 (rcp[0] = 0) in
// shared memory; the caller synchronises before use.
__device__ __forceinline__ void qat_rcp_table(float* rcp) {
  for (int b = threadIdx.x; b < 128; b += blockDim.x)
    rcp[b] = (b == 0 || b == 127) ? 0.0f : __frcp_rn(ue4m3_decode((uint32_t)b));
}

// 16-bit pair of two fp32 values, and the pair of the residuals (x - hi).
template <int DT>
__device__ __forceinline__ void qt_split2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  hi = pack2<DT>(x0, x1);
  lo = pack2<DT>(x0 - h2f<DT>((uint16_t)(hi & 0xFFFF)), x1 - h2f<DT>((uint16_t)(hi >> 16)));
}

// Stores 32 consecutive 16-bit values (columns c0..c0+31, c0 % 32 == 0) of
// row r of a tile.
__device__ __forceinline__ void qt_store32(uint8_t* tile, int r, int c0, const uint32_t (&w)[16]) {
#pragma unroll
  for (int q = 0; q < 4; ++q)
    *reinterpret_cast<uint4*>(tile + qt_elem(r, c0 + 8 * q)) =
        make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
}

// Stores 16 consecutive 16-bit values (columns c0..c0+15, c0 % 16 == 0).
__device__ __forceinline__ void qt_store16(uint8_t* tile, int r, int c0, const uint32_t (&w)[8]) {
  *reinterpret_cast<uint4*>(tile + qt_elem(r, c0)) = make_uint4(w[0], w[1], w[2], w[3]);
  *reinterpret_cast<uint4*>(tile + qt_elem(r, c0 + 8)) = make_uint4(w[4], w[5], w[6], w[7]);
}

// Shared-memory control block of the attention kernels (kQtShBytes):
// barriers [0, 192), the lane quarters' pair barriers [192, 224), the
// tensor-memory base and the abort flag, the UE4M3 reciprocals [256, 768),
// the pair exchange [1024, 2048).
struct QtShared {
  uint64_t* bars;
  uint64_t* xbar;
  uint32_t* tmem;
  volatile int* abort;
  float* rcp;
  float* xch;
};

// m256: the barriers every row-owning thread arrives on (count 256); m128:
// those one half of them (four warps) arrives on; the others complete on one
// arrival or an MMA commit.
__device__ __forceinline__ QtShared qt_setup(uint8_t* sh, int nbar, uint32_t m256,
                                             uint32_t m128) {
  QtShared s;
  s.bars = reinterpret_cast<uint64_t*>(sh);
  s.xbar = reinterpret_cast<uint64_t*>(sh + 192);
  s.tmem = reinterpret_cast<uint32_t*>(sh + 224);
  s.abort = reinterpret_cast<volatile int*>(sh + 228);
  s.rcp = reinterpret_cast<float*>(sh + 256);
  s.xch = reinterpret_cast<float*>(sh + 1024);
  if (threadIdx.x == 0) {
    for (int i = 0; i < nbar; ++i)
      mbar_init(&s.bars[i], ((m256 >> i) & 1u) ? 256 : (((m128 >> i) & 1u) ? 128 : 1));
    for (int i = 0; i < 4; ++i) mbar_init(&s.xbar[i], 64);
    *s.abort = 0;
    fence_mbar_init();
  }
  qat_rcp_table(s.rcp);
  __syncthreads();
  if ((threadIdx.x >> 5) == kQtMma) {
    tmem_alloc(s.tmem, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  return s;
}

__device__ __forceinline__ void qt_teardown(const QtShared& s) {
  tc_fence_before();
  __syncthreads();
  if ((threadIdx.x >> 5) == kQtMma) {
    tc_fence_after();
    tmem_dealloc(*s.tmem, 512);
  }
}

// Bounded wait a copy or MMA role makes at its end for the last phase it
// armed: no copy or MMA outlives the CTA.
__device__ __forceinline__ void qt_drain(uint64_t* bar, uint32_t parity) {
  int flag = 0;
  volatile int* never = &flag;
  mbar_wait(bar, parity, never, 200000000ull);
}

// One value per row exchanged between the two warps of a lane quarter
// (phase `phase` of the quarter's pair barrier): returns the partner's.
__device__ __forceinline__ bool qt_pair_swap(const QtShared& s, int quarter, int half, int r,
                                             uint32_t phase, float mine, float& other) {
  s.xch[half * 128 + r] = mine;
  mbar_arrive(&s.xbar[quarter]);
  const bool ok = warp_wait(&s.xbar[quarter], phase & 1, s.abort);
  other = s.xch[(half ^ 1) * 128 + r];
  return ok;
}

// Raw scores of keys key0..key0+31 with the invisible ones (key >= klim)
// set to -inf; the compare runs only where a lane of the warp needs it.
__device__ __forceinline__ void qt_mask32(float (&a)[32], int key0, int klim) {
  if (!__all_sync(0xffffffffu, key0 + 32 <= klim)) {
#pragma unroll
    for (int i = 0; i < 32; ++i) a[i] = key0 + i < klim ? a[i] : -INFINITY;
  }
}

// Largest raw score of 32 columns over the visible keys; -inf when none is
// visible.  tcgen05.ld is warp-wide: called by all lanes.
__device__ __forceinline__ float qt_chunk_max(uint32_t taddr, int key0, int klim) {
  float a[32];
  tmem_ld32(taddr, a);
  tmem_ld_wait();
  qt_mask32(a, key0, klim);
  float mx = a[0];
#pragma unroll
  for (int i = 1; i < 32; ++i) mx = fmaxf(mx, a[i]);
  return mx;
}

// Largest raw score of 64 columns (two loads, one wait).
__device__ __forceinline__ float qt_max64(uint32_t taddr, int key0, int klim) {
  float a[32], b[32];
  tmem_ld32(taddr, a);
  tmem_ld32(taddr + 32, b);
  tmem_ld_wait();
  qt_mask32(a, key0, klim);
  qt_mask32(b, key0 + 32, klim);
  float mx = fmaxf(a[0], b[0]);
#pragma unroll
  for (int i = 1; i < 32; ++i) mx = fmaxf(mx, fmaxf(a[i], b[i]));
  return mx;
}

__device__ __forceinline__ uint8_t* qt_smem_base() {
  extern __shared__ uint8_t qt_raw[];
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(qt_raw) + 1023) &
                                    ~(uintptr_t)1023);
}

// ============================================================ forward ==
template <int D>
struct QtFwdLayout {
  static constexpr uint32_t T = qt_tile_bytes(D);
  static constexpr uint32_t Q = 0, RING = T, P = (1 + kQtRing) * T;  // RING: K or V tiles
  static constexpr uint32_t SH = P + kQtPTile;
  static constexpr uint32_t SMEM_ALLOC = SH + kQtShBytes + 1024;
  // S; O and O'; P hi and lo (the A operand of O' += P V^, two 16-bit
  // values a column)
  static constexpr uint32_t T_S = 0, T_O = 128, T_OH = 128 + D, T_PH = 384, T_PL = 448;
  static_assert(T_OH + D <= T_PH, "tensor memory budget");
  static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
};

// The K and V tiles of a forward CTA pass through one ring of kQtRing slots
// in the order the MMAs read them: K(0), then for each key tile j: K(j+1)
// (when j+1 < nt), V(j).  Item i sits in slot i % kQtRing.
__device__ __forceinline__ int qt_ring_item(int i, int nt, bool& is_v) {
  is_v = false;
  if (i == 0) return 0;
  const int q = i - 1;
  if (q == 2 * (nt - 1)) {
    is_v = true;
    return nt - 1;
  }
  is_v = (q & 1) != 0;
  return is_v ? (q >> 1) : (q >> 1) + 1;
}
// Ring index of K(j) and of V(j).
__device__ __forceinline__ int qt_ring_k(int j) { return j == 0 ? 0 : 2 * j - 1; }
__device__ __forceinline__ int qt_ring_v(int j, int nt) {
  return j == nt - 1 ? 2 * nt - 1 : 2 * j + 2;
}

// RF + s / RE + s: ring slot s loaded / free; FSF / FSE: S written / read;
// FPF: P^ (shared memory) and P's two parts (tensor memory) written, with O
// and O' rescaled; FPE: the products of a key tile done.
enum : int {
  FQ = 0, RF = 1 /* 1..4 */, RE = 5 /* 5..8 */, FSF = 9, FSE = 10, FPF = 11, FPE = 12,
  FDONE = 13, FN = 14
};
constexpr uint32_t kFwd256 = (1u << FSE) | (1u << FPF);
// A row's reference maximum (log2 units) moves only when a key tile's
// maximum exceeds it by more than this: P and l stay below 2^8 times their
// values against the exact running maximum, and O, O' are rescaled rarely.
constexpr float kQtRescale = 8.0f;

// grid (ceil(maxlen / 128) * H, nseq), kQtThreads threads; causal grids
// start the query tiles with the most keys.  One pass over the key tiles:
// S(j+1) is computed while the rows turn S(j) into P^ and P, then O += P^ V^
// and O' += P V^ against each row's reference maximum.
template <int DT, int D, int BLK>
__global__ void __launch_bounds__(kQtThreads, 1) qat_fwd_kernel(const QatParams p) {
  using L = QtFwdLayout<D>;
  uint8_t* sm = qt_smem_base();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int seq = blockIdx.y;
  int64_t st;
  int len;
  p.si.get(seq, st, len);
  const int ntq = (len + 127) / 128;
  const int ti = (int)blockIdx.x / p.H, h = (int)blockIdx.x % p.H, hk = h / (p.H / p.Hkv);
  if (ti >= ntq) return;
  const int qt = p.causal ? ntq - 1 - ti : ti;
  const int q0 = qt * 128;
  const int kend = p.causal ? min(len, q0 + 128) : len;
  const int nt = (kend + 127) / 128;
  const QtShared S = qt_setup(sm + L::SH, FN, kFwd256, 0);
  uint64_t* bars = S.bars;
  const uint32_t tmem = *S.tmem;

  if (warp == kQtProducer) {
    if (lane == 0) {
      const uint8_t* kbase = p.kt + qat_slot(hk, p.nslot, st, seq, 0) * L::T;
      const uint8_t* vbase = p.vt + qat_slot(hk, p.nslot, st, seq, 0) * L::T;
      mbar_arrive_expect_tx(&bars[FQ], L::T);
      bulk_g2s(sm + L::Q, p.qt + qat_slot(h, p.nslot, st, seq, qt) * L::T, L::T, &bars[FQ]);
      const int nitems = 2 * nt;
      int last[kQtRing];
#pragma unroll
      for (int sl = 0; sl < kQtRing; ++sl) last[sl] = -1;
      for (int i = 0; i < nitems && !*S.abort; ++i) {
        const int sl = i % kQtRing;
        if (i >= kQtRing && !mbar_wait(&bars[RE + sl], (i / kQtRing - 1) & 1, S.abort)) break;
        bool is_v;
        const int t = qt_ring_item(i, nt, is_v);
        mbar_arrive_expect_tx(&bars[RF + sl], L::T);
        bulk_g2s(sm + L::RING + sl * L::T, (is_v ? vbase : kbase) + (int64_t)t * L::T, L::T,
                 &bars[RF + sl]);
        last[sl] = i;
      }
      qt_drain(&bars[FQ], 0);
      for (int sl = 0; sl < kQtRing; ++sl)
        if (last[sl] >= 0) qt_drain(&bars[RF + sl], (last[sl] / kQtRing) & 1);
    }
  } else if (warp == kQtMma) {
    // The whole warp runs the issuer's loop and waits (uniform operand
    // descriptors); the elected lane issues every MMA and commit.
    {
      const bool leader = elect_one();
      constexpr uint32_t idS = idesc_f16(DT, 128, 128);
      constexpr uint32_t idPV = idesc_f16(DT, 128, D) | kIdescBmn;
      const uint32_t base = smem_u32(sm);
      auto issue_s = [&](int j) -> bool {
        const int i = qt_ring_k(j), rs = i % kQtRing;
        if (!warp_wait(&bars[RF + rs], (i / kQtRing) & 1, S.abort)) return false;
        // the rows have read the previous scores
        if (j >= 1 && !warp_wait(&bars[FSE], (j - 1) & 1, S.abort)) return false;
        tc_fence_after();
        if (leader) {
#pragma unroll
          for (int s = 0; s < D / 16; ++s)
            mma_f16(tmem + L::T_S, qt_desc_k(base + L::Q, s),
                    qt_desc_k(base + L::RING + rs * L::T, s), idS, s > 0);
          tc_commit(&bars[FSF]);
          tc_commit(&bars[RE + rs]);
        }
        __syncwarp();
        return true;
      };
      bool ok = warp_wait(&bars[FQ], 0, S.abort) && issue_s(0);
      for (int j = 0; j < nt && ok; ++j) {
        // the next tile's scores go ahead of this tile's products
        if (j + 1 < nt && !issue_s(j + 1)) break;
        const int i = qt_ring_v(j, nt), rs = i % kQtRing;
        if (!warp_wait(&bars[RF + rs], (i / kQtRing) & 1, S.abort)) break;
        if (!warp_wait(&bars[FPF], j & 1, S.abort)) break;
        tc_fence_after();
        const uint32_t vt = base + L::RING + rs * L::T;
        if (leader) {
#pragma unroll
          for (int s = 0; s < 8; ++s) {
            const uint64_t bv = qt_desc_mn(vt, s);
            mma_f16(tmem + L::T_O, qt_desc_k(base + L::P, s), bv, idPV, j > 0 || s > 0);
            mma_f16_ta(tmem + L::T_OH, tmem + L::T_PH + 8 * s, bv, idPV, j > 0 || s > 0);
            mma_f16_ta(tmem + L::T_OH, tmem + L::T_PL + 8 * s, bv, idPV, 1);
          }
          tc_commit(&bars[FPE]);
          tc_commit(&bars[RE + rs]);
        }
        __syncwarp();
      }
      if (leader) {
        tc_commit(&bars[FDONE]);
      }
      __syncwarp();
      qt_drain(&bars[FDONE], 0);
    }
  } else {
    // row r of the tile; this warp's columns 64 half .. 64 half + 63
    const int quarter = warp & 3, half = warp >> 2;
    const int r = quarter * 32 + lane, row = q0 + r;
    const bool row_ok = row < len;
    const int klim = row_ok ? (p.causal ? row + 1 : len) : 0;  // visible keys: key < klim
    const uint32_t tl = tmem + ((uint32_t)(quarter * 32) << 16);
    const float c2 = p.g[0] * p.g[1] * p.sc * kQatLog2e;  // raw score -> log2 units
    const int c0 = 64 * half;
    uint8_t* tP = sm + L::P;
    bool ok = true;
    // mref: the row's reference maximum (log2 units, -inf before the first
    // visible key); lsum: this warp's share of l = sum 2^(s - mref)
    float mref = -INFINITY, lsum = 0.0f;
    for (int j = 0; j < nt && ok; ++j) {
      const int kb = j * 128;
      const uint32_t ts = tl + L::T_S;
      if (!warp_wait(&bars[FSF], j & 1, S.abort)) { ok = false; break; }
      tc_fence_after();
      // the tile's row maximum from both halves' columns (the two warps of a
      // row compute the same value), this half's maximum for a 64-key sigma
      const float mpart = qt_max64(ts + (c0 ^ 64), kb + (c0 ^ 64), klim);
      float a[2][32];
      tmem_ld32(ts + c0, a[0]);
      tmem_ld32(ts + c0 + 32, a[1]);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(&bars[FSE]);
      qt_mask32(a[0], kb + c0, klim);
      qt_mask32(a[1], kb + c0 + 32, klim);
      float mown = -INFINITY;
#pragma unroll
      for (int i = 0; i < 32; ++i) mown = fmaxf(mown, fmaxf(a[0][i], a[1][i]));
      const float mtile = half == 0 ? fmaxf(mown, mpart) : fmaxf(mpart, mown);
      const float msig_raw = BLK == 128 ? mtile : mown;
      // a new reference when the tile's maximum passes the old one by more
      // than kQtRescale: O, O' and l are multiplied by alpha = 2^(old - new)
      float alpha = 1.0f;
      if (mtile != -INFINITY && mtile * c2 > mref + kQtRescale) {
        alpha = mref == -INFINITY ? 0.0f : ex2_ftz(mref - mtile * c2);
        mref = mtile * c2;
      }
      lsum *= alpha;
      const bool live = msig_raw != -INFINITY;
      // P / sigma of the sub-tile = 2688 exp(S - max_sub S) = 2^(s c2 + off);
      // P = that times fct = 2^(max_sub - mref) / 2688
      const float off = live ? kLog2TensorScaleDiv - msig_raw * c2 : 0.0f;
      const float fct = live ? ex2_ftz(msig_raw * c2 - mref) * (1.0f / kTensorScaleDiv) : 0.0f;
      // P^ and the two parts of P in registers first; they are written (P^
      // to shared memory, P to tensor memory) once the products of the
      // previous tile are done
      uint32_t wq[2][16], wh[2][16], wl[2][16];
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
#pragma unroll
        for (int b = 0; b < 2; ++b) {
          float qv[16];
          float am = 0.0f;
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            qv[i] = ex2_ftz(fmaf(a[cc][16 * b + i], c2, off));
            am = fmaxf(am, qv[i]);
          }
          const PBlock pb(am, S.rcp);
#pragma unroll
          for (int i = 0; i < 16; i += 2) {
            wq[cc][8 * b + i / 2] = pb.scaled<DT>(qv[i], qv[i + 1], fct);
            const float p0 = qv[i] * fct, p1 = qv[i + 1] * fct;
            lsum += p0 + p1;
            qt_split2<DT>(p0, p1, wh[cc][8 * b + i / 2], wl[cc][8 * b + i / 2]);
          }
        }
      }
      if (j >= 1 && !warp_wait(&bars[FPE], (j - 1) & 1, S.abort)) { ok = false; break; }
      tc_fence_after();
      if (j >= 1 && __any_sync(0xffffffffu, alpha != 1.0f)) {
        // this warp's columns of O and O' against the new reference
#pragma unroll 1
        for (int c = half * (D / 2); c < (half + 1) * (D / 2); c += 16) {
          float o[16], oh[16];
          tmem_ld16(tl + L::T_O + c, o);
          tmem_ld16(tl + L::T_OH + c, oh);
          tmem_ld_wait();
          uint32_t uo[16], uh[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            uo[i] = __float_as_uint(o[i] * alpha);
            uh[i] = __float_as_uint(oh[i] * alpha);
          }
          tmem_st16u(tl + L::T_O + c, uo);
          tmem_st16u(tl + L::T_OH + c, uh);
        }
      }
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        qt_store32(tP, r, c0 + 32 * cc, wq[cc]);
        tmem_st16u(tl + L::T_PH + 32 * half + 16 * cc, wh[cc]);
        tmem_st16u(tl + L::T_PL + 32 * half + 16 * cc, wl[cc]);
      }
      fence_proxy_async_smem();
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&bars[FPF]);
    }
    const float m = mref;
    // epilogue: O = P^ V^ g_V / l, O' = P V^ g_V / l, lse; the row sum l
    // from both halves
    if (ok) ok = warp_wait(&bars[FDONE], 0, S.abort);
    float lo = 0.0f;
    if (ok) ok = qt_pair_swap(S, quarter, half, r, 0, lsum, lo);
    if (ok) {
      tc_fence_after();
      const float l = half == 0 ? lsum + lo : lo + lsum;
      const float sc_out = l > 0.0f ? p.g[2] / l : 0.0f;
      const int64_t base = ((st + (row_ok ? row : 0)) * p.H + h) * D;
#pragma unroll 1
      for (int c = half * (D / 2); c < (half + 1) * (D / 2); c += 32) {
        float o[32], oh[32];
        tmem_ld32(tl + L::T_O + c, o);
        tmem_ld32(tl + L::T_OH + c, oh);
        tmem_ld_wait();
        if (row_ok) {
#pragma unroll
          for (int i = 0; i < 32; i += 8) {
            uint4 w;
            w.x = pack2<DT>(o[i] * sc_out, o[i + 1] * sc_out);
            w.y = pack2<DT>(o[i + 2] * sc_out, o[i + 3] * sc_out);
            w.z = pack2<DT>(o[i + 4] * sc_out, o[i + 5] * sc_out);
            w.w = pack2<DT>(o[i + 6] * sc_out, o[i + 7] * sc_out);
            *reinterpret_cast<uint4*>(p.out + base + c + i) = w;
            *reinterpret_cast<float4*>(p.out_hp + base + c + i) =
                make_float4(oh[i] * sc_out, oh[i + 1] * sc_out, oh[i + 2] * sc_out,
                            oh[i + 3] * sc_out);
            *reinterpret_cast<float4*>(p.out_hp + base + c + i + 4) =
                make_float4(oh[i + 4] * sc_out, oh[i + 5] * sc_out, oh[i + 6] * sc_out,
                            oh[i + 7] * sc_out);
          }
        }
      }
      if (row_ok && half == 0)
        p.lse[(int64_t)h * p.total + st + row] = l > 0.0f ? (m + log2f(l)) * kQatLn2 : -INFINITY;
    }
  }
  qt_teardown(S);
}

// ======================================================= backward: dQ ==
template <int D>
struct QtQLayout {
  static constexpr uint32_t T = qt_tile_bytes(D);
  static constexpr uint32_t Q = 0, DO = T, K = 2 * T, V = 5 * T;  // K: 3 slots, V: 2
  static constexpr uint32_t SH = 7 * T;
  static constexpr uint32_t SMEM_ALLOC = SH + kQtShBytes + 1024;
  // dS hi and lo: the A operand of dQ += dS K^ in tensor memory (64 columns
  // each, two 16-bit values a column)
  static constexpr uint32_t T_S = 0, T_DP = 128, T_DQ = 256, T_DSH = 384, T_DSL = 448;
  static_assert(T_DQ + D <= T_DSH, "tensor memory budget");
  static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
};

// QSF / QSR: S computed / read by the rows; QDF / QDR: dP computed / read;
// QPF + h / QPE + h: key half h of dS written / consumed.
enum : int {
  QQ = 0, QKF = 1 /* 1..3 */, QKE = 4 /* 4..6 */, QVF = 7 /* 7,8 */, QVE = 9 /* 9,10 */,
  QSF = 11, QSR = 12, QDF = 13, QDR = 14, QPF = 15 /* 15,16 */, QPE = 17 /* 17,18 */,
  QDONE = 19, QN = 20
};
constexpr uint32_t kQ256 = (1u << QSR) | (1u << QDR);
constexpr uint32_t kQ128 = (1u << QPF) | (1u << (QPF + 1));

// grid (ceil(maxlen / 128) * H, nseq), kQtThreads threads.
template <int DT, int D>
__global__ void __launch_bounds__(kQtThreads, 1) qat_bwd_q_kernel(const QatParams p) {
  using L = QtQLayout<D>;
  uint8_t* sm = qt_smem_base();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int seq = blockIdx.y;
  int64_t st;
  int len;
  p.si.get(seq, st, len);
  const int ntq = (len + 127) / 128;
  const int ti = (int)blockIdx.x / p.H, h = (int)blockIdx.x % p.H, hk = h / (p.H / p.Hkv);
  if (ti >= ntq) return;
  const int qt = p.causal ? ntq - 1 - ti : ti;
  const int q0 = qt * 128;
  const int kend = p.causal ? min(len, q0 + 128) : len;
  const int nt = (kend + 127) / 128;
  const QtShared S = qt_setup(sm + L::SH, QN, kQ256, kQ128);
  uint64_t* bars = S.bars;
  const uint32_t tmem = *S.tmem;

  if (warp == kQtProducer) {
    if (lane == 0) {
      const int64_t qs = qat_slot(h, p.nslot, st, seq, qt);
      const uint8_t* kbase = p.kt + qat_slot(hk, p.nslot, st, seq, 0) * L::T;
      const uint8_t* vbase = p.vt + qat_slot(hk, p.nslot, st, seq, 0) * L::T;
      mbar_arrive_expect_tx(&bars[QQ], 2 * L::T);
      bulk_g2s(sm + L::Q, p.qt + qs * L::T, L::T, &bars[QQ]);
      bulk_g2s(sm + L::DO, p.dot + qs * L::T, L::T, &bars[QQ]);
      int lastk[3] = {-1, -1, -1}, lastv[2] = {-1, -1};
      for (int j = 0; j < nt && !*S.abort; ++j) {
        const int ks = j % 3, vs = j & 1;
        if (j >= 3 && !mbar_wait(&bars[QKE + ks], (j / 3 - 1) & 1, S.abort)) break;
        mbar_arrive_expect_tx(&bars[QKF + ks], L::T);
        bulk_g2s(sm + L::K + ks * L::T, kbase + (int64_t)j * L::T, L::T, &bars[QKF + ks]);
        lastk[ks] = j;
        if (j >= 2 && !mbar_wait(&bars[QVE + vs], ((j >> 1) - 1) & 1, S.abort)) break;
        mbar_arrive_expect_tx(&bars[QVF + vs], L::T);
        bulk_g2s(sm + L::V + vs * L::T, vbase + (int64_t)j * L::T, L::T, &bars[QVF + vs]);
        lastv[vs] = j;
      }
      qt_drain(&bars[QQ], 0);
      for (int sl = 0; sl < 3; ++sl)
        if (lastk[sl] >= 0) qt_drain(&bars[QKF + sl], (lastk[sl] / 3) & 1);
      for (int sl = 0; sl < 2; ++sl)
        if (lastv[sl] >= 0) qt_drain(&bars[QVF + sl], (lastv[sl] >> 1) & 1);
    }
  } else if (warp == kQtMma) {
    // The whole warp runs the issuer's loop and waits (uniform operand
    // descriptors); the elected lane issues every MMA and commit.
    {
      const bool leader = elect_one();
      constexpr uint32_t idS = idesc_f16(DT, 128, 128);
      constexpr uint32_t idDQ = idesc_f16(DT, 128, D) | kIdescBmn;
      const uint32_t base = smem_u32(sm);
      // S = Q^ K^T of key tile j once the rows have read S(j - 1)
      auto issue_s = [&](int j) -> bool {
        const int ks = j % 3;
        if (!warp_wait(&bars[QKF + ks], (j / 3) & 1, S.abort)) return false;
        if (j >= 1 && !warp_wait(&bars[QSR], (j - 1) & 1, S.abort)) return false;
        tc_fence_after();
        if (leader) {
#pragma unroll
          for (int s = 0; s < D / 16; ++s)
            mma_f16(tmem + L::T_S, qt_desc_k(base + L::Q, s), qt_desc_k(base + L::K + ks * L::T, s),
                    idS, s > 0);
          tc_commit(&bars[QSF]);
        }
        __syncwarp();
        return true;
      };
      // dP = dO V^T of key tile j once the rows have read dP(j - 1)
      auto issue_dp = [&](int j) -> bool {
        const int vs = j & 1;
        if (!warp_wait(&bars[QVF + vs], (j >> 1) & 1, S.abort)) return false;
        if (j >= 1 && !warp_wait(&bars[QDR], (j - 1) & 1, S.abort)) return false;
        tc_fence_after();
        if (leader) {
#pragma unroll
          for (int s = 0; s < D / 16; ++s)
            mma_f16(tmem + L::T_DP, qt_desc_k(base + L::DO, s), qt_desc_k(base + L::V + vs * L::T, s),
                    idS, s > 0);
          tc_commit(&bars[QDF]);
          tc_commit(&bars[QVE + vs]);
        }
        __syncwarp();
        return true;
      };
      bool ok = warp_wait(&bars[QQ], 0, S.abort) && issue_s(0) && issue_dp(0);
      for (int j = 0; j < nt && ok; ++j) {
        if (j + 1 < nt && !(issue_s(j + 1) && issue_dp(j + 1))) break;
        const uint32_t kt = base + L::K + (j % 3) * L::T;
        bool fine = true;
#pragma unroll
        for (int hf = 0; hf < 2 && fine; ++hf) {
          if (!warp_wait(&bars[QPF + hf], j & 1, S.abort)) { fine = false; break; }
          tc_fence_after();
          if (leader) {
#pragma unroll
            for (int s = 4 * hf; s < 4 * hf + 4; ++s) {
              const uint64_t bk = qt_desc_mn(kt, s);
              mma_f16_ta(tmem + L::T_DQ, tmem + L::T_DSH + 8 * s, bk, idDQ, j > 0 || s > 0);
              mma_f16_ta(tmem + L::T_DQ, tmem + L::T_DSL + 8 * s, bk, idDQ, 1);
            }
            tc_commit(&bars[QPE + hf]);
          }
          __syncwarp();
        }
        if (!fine) break;
        if (leader) {
          tc_commit(&bars[QKE + j % 3]);
        }
        __syncwarp();
      }
      if (leader) {
        tc_commit(&bars[QDONE]);
      }
      __syncwarp();
      qt_drain(&bars[QDONE], 0);
    }
  } else {
    const int quarter = warp & 3, half = warp >> 2;
    const int r = quarter * 32 + lane, row = q0 + r;
    const bool row_ok = row < len;
    const int klim = row_ok ? (p.causal ? row + 1 : len) : 0;
    const uint32_t tl = tmem + ((uint32_t)(quarter * 32) << 16);
    const float c2 = p.g[0] * p.g[1] * p.sc * kQatLog2e, gv = p.g[2];
    const float nlse2 = row_ok ? -p.lse[(int64_t)h * p.total + st + row] * kQatLog2e : 0.0f;
    const float dsum = row_ok ? p.dsum[(int64_t)h * p.total + st + row] : 0.0f;
    bool ok = true;
    for (int j = 0; j < nt && ok; ++j) {
      if (!warp_wait(&bars[QSF], j & 1, S.abort)) { ok = false; break; }
      tc_fence_after();
      // this warp's 64 scores into registers, released at once (S of the
      // next tile may overwrite them); then dP chunk by chunk
      float a[2][32];
      tmem_ld32(tl + L::T_S + 64 * half, a[0]);
      tmem_ld32(tl + L::T_S + 64 * half + 32, a[1]);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(&bars[QSR]);
      qt_mask32(a[0], j * 128 + 64 * half, klim);
      qt_mask32(a[1], j * 128 + 64 * half + 32, klim);
      if (!warp_wait(&bars[QDF], j & 1, S.abort)) { ok = false; break; }
      // this half's dS columns are free once the products of the previous
      // tile have read them
      if (j >= 1 && !warp_wait(&bars[QPE + half], (j - 1) & 1, S.abort)) { ok = false; break; }
      tc_fence_after();
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        float dp[32];
        tmem_ld32(tl + L::T_DP + 64 * half + 32 * cc, dp);
        tmem_ld_wait();
        if (cc == 1) {
          tc_fence_before();
          mbar_arrive(&bars[QDR]);
        }
        uint32_t wh[16], wl[16];
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          const float d0 = ex2_ftz(fmaf(a[cc][i], c2, nlse2)) * fmaf(dp[i], gv, -dsum);
          const float d1 = ex2_ftz(fmaf(a[cc][i + 1], c2, nlse2)) * fmaf(dp[i + 1], gv, -dsum);
          qt_split2<DT>(d0, d1, wh[i / 2], wl[i / 2]);
        }
        tmem_st16u(tl + L::T_DSH + 32 * half + 16 * cc, wh);
        tmem_st16u(tl + L::T_DSL + 32 * half + 16 * cc, wl);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&bars[QPF + half]);
    }
    if (ok && warp_wait(&bars[QDONE], 0, S.abort)) {
      tc_fence_after();
      const float qscale = p.g[1] * p.sc;
      const int64_t base = ((st + (row_ok ? row : 0)) * p.H + h) * D;
#pragma unroll 1
      for (int c = half * (D / 2); c < (half + 1) * (D / 2); c += 32) {
        float gq[32];
        tmem_ld32(tl + L::T_DQ + c, gq);
        tmem_ld_wait();
        if (row_ok) {
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            *reinterpret_cast<float4*>(p.dq + base + c + i) =
                make_float4(gq[i] * qscale, gq[i + 1] * qscale, gq[i + 2] * qscale,
                            gq[i + 3] * qscale);
        }
      }
    }
  }
  qt_teardown(S);
}

// =================================================== backward: dK, dV ==
template <int D>
struct QtKvLayout {
  static constexpr uint32_t T = qt_tile_bytes(D);
  static constexpr uint32_t K = 0, V = T, Q = 2 * T, DO = 4 * T;  // Q: 2 slots
  static constexpr uint32_t P = 5 * T, DS = P + kQtPTile;
  static constexpr uint32_t SH = DS + kQtPTile;
  static constexpr uint32_t SMEM_ALLOC = SH + kQtShBytes + 1024;
  static constexpr uint32_t T_S = 0, T_DP = 128, T_DV = 256, T_DK = 256 + D;
  static_assert(T_DK + D <= 512, "tensor memory budget");
  static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
};

// KQF + s / KQE + s: Q slot s loaded / free (its chunk's dK done); KOF /
// KOE: the dO chunk and the P^ tile loaded / free (the chunk's dV done);
// KSF / KSR: S computed / read by the rows; KDF / KDR: dP computed / read;
// KPPF: P^ written; KDSF: dS written; KPE: the chunk's dK done.
enum : int {
  KKV = 0, KQF = 1 /* 1,2 */, KQE = 3 /* 3,4 */, KOF = 5, KOE = 6, KSF = 7, KSR = 8, KDF = 9,
  KDR = 10, KPPF = 11, KDSF = 12, KPE = 13, KDONE = 14, KN = 15
};
constexpr uint32_t kKv256 = (1u << KSR) | (1u << KDR) | (1u << KPPF) | (1u << KDSF);

// grid (ceil(maxlen / 128) * Hkv, nseq), kQtThreads threads: key tile
// blockIdx.x / Hkv (causal grids: the tiles with the most queries first).
// Iteration it takes query chunk c0 + it % nch of query head
// hk * grp + it / nch.  The rows read S(it) into registers first, so S of
// the next chunk (its Q in the second slot) runs while they work; they form
// P and P^ from S alone and publish P^, so dV (P^T dO) runs while they wait
// for dP and form dS; dK (dS^T Q^) follows, and the next dO chunk loads from
// the end of dV on.
template <int DT, int D, int BLK>
__global__ void __launch_bounds__(kQtThreads, 1) qat_bwd_kv_kernel(const QatParams p) {
  using L = QtKvLayout<D>;
  uint8_t* sm = qt_smem_base();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int seq = blockIdx.y;
  int64_t st;
  int len;
  p.si.get(seq, st, len);
  const int kt = (int)blockIdx.x / p.Hkv, hk = (int)blockIdx.x % p.Hkv, grp = p.H / p.Hkv;
  const int j0 = kt * 128;
  if (j0 >= len) return;
  const int c0 = p.causal ? kt : 0;  // first query chunk that sees a key of the tile
  const int nch = (len + 127) / 128 - c0;
  const int n_it = grp * nch;
  const QtShared S = qt_setup(sm + L::SH, KN, kKv256, 0);
  uint64_t* bars = S.bars;
  const uint32_t tmem = *S.tmem;

  if (warp == kQtProducer) {
    if (lane == 0) {
      const int64_t ks = qat_slot(hk, p.nslot, st, seq, kt);
      mbar_arrive_expect_tx(&bars[KKV], 2 * L::T);
      bulk_g2s(sm + L::K, p.kt + ks * L::T, L::T, &bars[KKV]);
      bulk_g2s(sm + L::V, p.vt + ks * L::T, L::T, &bars[KKV]);
      int lastq[2] = {-1, -1}, lasto = -1;
      for (int it = 0; it < n_it && !*S.abort; ++it) {
        const int64_t qs = qat_slot(hk * grp + it / nch, p.nslot, st, seq, c0 + it % nch);
        const int sl = it & 1;
        if (it >= 2 && !mbar_wait(&bars[KQE + sl], ((it >> 1) - 1) & 1, S.abort)) break;
        mbar_arrive_expect_tx(&bars[KQF + sl], L::T);
        bulk_g2s(sm + L::Q + sl * L::T, p.qt + qs * L::T, L::T, &bars[KQF + sl]);
        lastq[sl] = it;
        if (it >= 1 && !mbar_wait(&bars[KOE], (it - 1) & 1, S.abort)) break;
        mbar_arrive_expect_tx(&bars[KOF], L::T);
        bulk_g2s(sm + L::DO, p.dot + qs * L::T, L::T, &bars[KOF]);
        lasto = it;
      }
      qt_drain(&bars[KKV], 0);
      for (int sl = 0; sl < 2; ++sl)
        if (lastq[sl] >= 0) qt_drain(&bars[KQF + sl], (lastq[sl] >> 1) & 1);
      if (lasto >= 0) qt_drain(&bars[KOF], lasto & 1);
    }
  } else if (warp == kQtMma) {
    // The whole warp runs the issuer's loop and waits (uniform operand
    // descriptors); the elected lane issues every MMA and commit.
    {
      const bool leader = elect_one();
      constexpr uint32_t idS = idesc_f16(DT, 128, 128);
      constexpr uint32_t idG = idesc_f16(DT, 128, D) | kIdescAmn | kIdescBmn;
      const uint32_t base = smem_u32(sm);
      // S(it) = Q^ K^T into the S columns (the rows have read S(it - 1))
      auto issue_s = [&](int it) -> bool {
        const int sl = it & 1;
        if (!warp_wait(&bars[KQF + sl], (it >> 1) & 1, S.abort)) return false;
        if (it >= 1 && !warp_wait(&bars[KSR], (it - 1) & 1, S.abort)) return false;
        tc_fence_after();
        if (leader) {
#pragma unroll
          for (int s = 0; s < D / 16; ++s)
            mma_f16(tmem + L::T_S, qt_desc_k(base + L::Q + sl * L::T, s),
                    qt_desc_k(base + L::K, s), idS, s > 0);
          tc_commit(&bars[KSF]);
        }
        __syncwarp();
        return true;
      };
      bool ok = warp_wait(&bars[KKV], 0, S.abort) && issue_s(0);
      for (int it = 0; it < n_it && ok; ++it) {
        // dP(it) = dO V^T (the rows have read dP(it - 1))
        if (!warp_wait(&bars[KOF], it & 1, S.abort)) break;
        if (it >= 1 && !warp_wait(&bars[KDR], (it - 1) & 1, S.abort)) break;
        tc_fence_after();
        if (leader) {
#pragma unroll
          for (int s = 0; s < D / 16; ++s)
            mma_f16(tmem + L::T_DP, qt_desc_k(base + L::DO, s), qt_desc_k(base + L::V, s), idS,
                    s > 0);
          tc_commit(&bars[KDF]);
        }
        __syncwarp();
        // the next chunk's scores while the rows work on this one
        if (it + 1 < n_it && !issue_s(it + 1)) break;
        // dV += P^T dO, dK += dS^T Q^: M = the 128 keys, K = the 128 queries
        if (!warp_wait(&bars[KPPF], it & 1, S.abort)) break;
        tc_fence_after();
        const uint32_t qt = base + L::Q + (it & 1) * L::T;
        if (leader) {
#pragma unroll
          for (int s = 0; s < 8; ++s)
            mma_f16(tmem + L::T_DV, qt_desc_mn(base + L::P, s), qt_desc_mn(base + L::DO, s), idG,
                    it > 0 || s > 0);
          tc_commit(&bars[KOE]);
        }
        __syncwarp();
        if (!warp_wait(&bars[KDSF], it & 1, S.abort)) break;
        tc_fence_after();
        if (leader) {
#pragma unroll
          for (int s = 0; s < 8; ++s)
            mma_f16(tmem + L::T_DK, qt_desc_mn(base + L::DS, s), qt_desc_mn(qt, s), idG,
                    it > 0 || s > 0);
          tc_commit(&bars[KQE + (it & 1)]);
          tc_commit(&bars[KPE]);
        }
        __syncwarp();
      }
      if (leader) {
        tc_commit(&bars[KDONE]);
      }
      __syncwarp();
      qt_drain(&bars[KDONE], 0);
    }
  } else {
    const int quarter = warp & 3, half = warp >> 2;
    const int r = quarter * 32 + lane, cb = 64 * half;
    const uint32_t tl = tmem + ((uint32_t)(quarter * 32) << 16);
    const float c2 = p.g[0] * p.g[1] * p.sc * kQatLog2e, gv = p.g[2];
    uint8_t* tP = sm + L::P;
    uint8_t* tD = sm + L::DS;
    // -lse (log2 units) and D of this thread's query row in iteration it
    auto row_stats = [&](int it, float& nl, float& dsv) {
      const int hq = hk * grp + it / nch, row = (c0 + it % nch) * 128 + r;
      const bool ok_row = row < len;
      nl = ok_row ? -p.lse[(int64_t)hq * p.total + st + row] * kQatLog2e : 0.0f;
      dsv = ok_row ? p.dsum[(int64_t)hq * p.total + st + row] : 0.0f;
    };
    float nl_next, ds_next;
    row_stats(0, nl_next, ds_next);
    bool ok = true;
    for (int it = 0; it < n_it && ok; ++it) {
      const int row = (c0 + it % nch) * 128 + r;
      const int klim = row < len ? (p.causal ? row + 1 : len) : 0;
      const float nlse2 = nl_next, dsum = ds_next;
      if (it + 1 < n_it) row_stats(it + 1, nl_next, ds_next);  // in flight meanwhile
      if (!warp_wait(&bars[KSF], it & 1, S.abort)) { ok = false; break; }
      tc_fence_after();
      // this warp's 64 scores into registers, and with them (and, for a
      // 128-key sigma, the partner's columns) the largest visible one
      float a[2][32];
      tmem_ld32(tl + L::T_S + cb, a[0]);
      tmem_ld32(tl + L::T_S + cb + 32, a[1]);
      tmem_ld_wait();
      qt_mask32(a[0], j0 + cb, klim);
      qt_mask32(a[1], j0 + cb + 32, klim);
      float cm_raw = -INFINITY;
#pragma unroll
      for (int i = 0; i < 32; ++i) cm_raw = fmaxf(cm_raw, fmaxf(a[0][i], a[1][i]));
      if constexpr (BLK == 128) {
#pragma unroll 1
        for (int c = 0; c < 2; ++c)
          cm_raw = fmaxf(cm_raw, qt_chunk_max(tl + L::T_S + (cb ^ 64) + 32 * c,
                                              j0 + (cb ^ 64) + 32 * c, klim));
      }
      tc_fence_before();
      mbar_arrive(&bars[KSR]);  // the next chunk's S may overwrite these columns
      // sigma of this warp's BLK-key sub-tile: the largest P there / 2688
      const float cm = cm_raw == -INFINITY ? 0.0f : ex2_ftz(fmaf(cm_raw, c2, nlse2));
      const float inv = cm > 0.0f ? __fdiv_rn(kTensorScaleDiv, cm) : 0.0f;
      const float sig = __fdiv_rn(cm, kTensorScaleDiv);
      // P (kept in place of S) and P^, written once dV of the previous chunk
      // has read the P^ tile
      if (it >= 1 && !warp_wait(&bars[KOE], (it - 1) & 1, S.abort)) { ok = false; break; }
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        const int col = cb + 32 * cc;
#pragma unroll
        for (int b = 0; b < 2; ++b) {
          float x[16];
          float am = 0.0f;
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float pr = ex2_ftz(fmaf(a[cc][16 * b + i], c2, nlse2));
            a[cc][16 * b + i] = pr;
            x[i] = pr * inv;
            am = fmaxf(am, x[i]);
          }
          const PBlock pb(am, S.rcp, true);
          uint32_t wq[8];
#pragma unroll
          for (int i = 0; i < 16; i += 2) wq[i / 2] = pb.scaled<DT>(x[i], x[i + 1], sig);
          qt_store16(tP, r, col + 16 * b, wq);
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(&bars[KPPF]);
      // dS = P o (dP g_V - D), written once dK of the previous chunk has read
      // the dS tile
      if (!warp_wait(&bars[KDF], it & 1, S.abort)) { ok = false; break; }
      if (it >= 1 && !warp_wait(&bars[KPE], (it - 1) & 1, S.abort)) { ok = false; break; }
      tc_fence_after();
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        const int col = cb + 32 * cc;
        float dp[32];
        tmem_ld32(tl + L::T_DP + col, dp);
        tmem_ld_wait();
        if (cc == 1) {
          tc_fence_before();
          mbar_arrive(&bars[KDR]);
        }
#pragma unroll
        for (int b = 0; b < 2; ++b) {
          uint32_t wd[8];
#pragma unroll
          for (int i = 0; i < 16; i += 2) {
            const int e = 16 * b + i;
            wd[i / 2] = pack2<DT>(a[cc][e] * fmaf(dp[e], gv, -dsum),
                                  a[cc][e + 1] * fmaf(dp[e + 1], gv, -dsum));
          }
          qt_store16(tD, r, col + 16 * b, wd);
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(&bars[KDSF]);
    }
    // epilogue: lane r of the dV and dK accumulators is key j0 + r
    if (ok && warp_wait(&bars[KDONE], 0, S.abort)) {
      tc_fence_after();
      const int key = j0 + r;
      const bool key_ok = key < len;
      const float kscale = p.g[0] * p.sc;
      const int64_t base = ((st + (key_ok ? key : 0)) * p.Hkv + hk) * D;
#pragma unroll 1
      for (int c = half * (D / 2); c < (half + 1) * (D / 2); c += 32) {
        float gdv[32], gdk[32];
        tmem_ld32(tl + L::T_DV + c, gdv);
        tmem_ld32(tl + L::T_DK + c, gdk);
        tmem_ld_wait();
        if (key_ok) {
#pragma unroll
          for (int i = 0; i < 32; i += 4) {
            *reinterpret_cast<float4*>(p.dv + base + c + i) =
                make_float4(gdv[i], gdv[i + 1], gdv[i + 2], gdv[i + 3]);
            *reinterpret_cast<float4*>(p.dk + base + c + i) =
                make_float4(gdk[i] * kscale, gdk[i + 1] * kscale, gdk[i + 2] * kscale,
                            gdk[i + 3] * kscale);
          }
        }
      }
    }
  }
  qt_teardown(S);
}

}  // namespace thrift
