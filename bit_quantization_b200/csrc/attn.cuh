// Mixed NVFP4 / FP16 attention forward (one CTA per 128 query rows of one
// head of one sequence).
//
// ThriftAttention, Metodologia step 2 and the kernel paragraph after it:
// the key tiles whose block pair was not selected are visited first on the
// NVFP4 path, then the selected ones on the FP16 path; a CTA with no selected
// pair never loads its 16-bit Q tile.  Both paths feed one online softmax
// (FlashAttention-2 style, base-2, running max m and sum l).  The NVFP4 path
// follows ScaleSearchAttention's native execution: QK^T and PV as
// block-scaled E2M1 MMAs with UE4M3 scales and fp32 accumulation; P is
// quantised in two levels (per row and key tile an fp32 factor rowmax/2688,
// then NVFP4 16-key blocks).
//
// Roles (23 warps, 736 threads):
//   warps 0-15  softmax, two groups of eight taking alternate key tiles;
//               in a group, query row r (TMEM lane r) is shared by two
//               warps, each owning half of the key columns; the groups take
//               turns at the exponentials;
//   warps 16-19 correction + output: one thread per row keeps the running
//               max and sum, rescales the output accumulator O (in tensor
//               memory) between PV(t-1) and PV(t), then divides by the row
//               sum and writes the output and LSE;
//   warp 20     producer: bulk copies of the pre-quantised tile images;
//   warp 21     tensor-memory owner and QK^T issuer;
//   warp 22     PV issuer (each issuer warp runs its loop and waits with
//               all lanes, one elected lane issuing the tensor
//               instructions and commits).
// The MMA accumulates every PV straight into O, so the softmax warps never
// wait on a PV product.
// Tensor memory (512 columns): S double buffer [2][BLK], O [D], then the
// scale factors of Q, K (x2), P (x2) and V (x2).
// Every wait is bounded; a wait that gives up sets the device status word
// and the CTA drains and exits.
#pragma once
#include "quant_kernels.cuh"

namespace thrift {

struct AttnParams {
  const uint8_t* q4;
  const uint8_t* k4;
  const uint8_t* v4;
  const uint8_t* q16;
  const uint8_t* k16;
  const uint8_t* v16;
  const uint8_t* mask;     // [nseq, H, nB, nB], 1 = FP16 pair
  const uint32_t* amax;    // absmax bit patterns of (rotated) Q, K and of V
  uint16_t* out;           // [total, H, D]
  float* lse;
  SeqInfo seqs;
  int nseq, H, Hkv, nB, nTq, causal, lse_varlen;
  int64_t total;
  float scale4;            // log2(e)/sqrt(d), divided by d with the rotation
  float scale16;           // log2(e)/sqrt(d)
  const float* corr;       // K smoothing: q^ . mu per query row [nseq, H, nTq * 128], or null
};

template <int D, int BLK>
struct AttnLayout {
  static constexpr uint32_t align(uint32_t x) { return (x + 1023u) & ~1023u; }
  static constexpr uint32_t QT4 = fp4_tile_bytes(128, D);
  static constexpr uint32_t Q16B = f16_tile_bytes(128, D);
  static constexpr uint32_t KT4 = fp4_tile_bytes(BLK, D);
  static constexpr uint32_t VT4 = fp4_tile_bytes(D, BLK);
  static constexpr uint32_t KT16 = f16_tile_bytes(BLK, D);
  static constexpr uint32_t VT16 = f16_tile_bytes(D, BLK);
  static constexpr uint32_t PT4 = fp4_tile_bytes(128, BLK);
  static constexpr uint32_t P16B = f16_tile_bytes(128, BLK);
  static constexpr uint32_t PT4A = align(PT4);  // one P slot
  // One region serves the NVFP4 phase and then the FP16 phase of a CTA (all
  // NVFP4 tiles come first); the producer enters the FP16 phase only after
  // the last NVFP4 PV has retired.
  //   NVFP4 view: Q4 | P4 x2 | NS4 stages (K4 + V4)
  //   FP16 view:  Q16 | P16 | 2 stages (K16 + V16)
  static constexpr uint32_t V4_OFF = align(KT4);
  static constexpr uint32_t STG4 = V4_OFF + align(VT4);
  static constexpr uint32_t V16_OFF = align(KT16);
  static constexpr uint32_t STG16 = V16_OFF + align(VT16);
  static constexpr uint32_t OFF4_Q = 0;
  static constexpr uint32_t OFF4_P = align(QT4);
  static constexpr uint32_t OFF4_STG = OFF4_P + 2 * PT4A;
  static constexpr uint32_t OFF16_Q = 0;
  static constexpr uint32_t OFF16_P = align(Q16B);
  static constexpr uint32_t OFF16_STG = OFF16_P + align(P16B);
  static constexpr uint32_t NS16 = 2;
  static constexpr uint32_t REGION = OFF16_STG + NS16 * STG16;
  static constexpr uint32_t NS4_FIT = (REGION - OFF4_STG) / STG4;
  static constexpr uint32_t NS4 = NS4_FIT > 12 ? 12 : NS4_FIT;
  static constexpr uint32_t OFF_LIST = REGION;
  static constexpr uint32_t MAX_TILES = 512;  // key tiles per sequence
  static constexpr uint32_t OFF_BAR = OFF_LIST + 2 * 2 * MAX_TILES;
  static constexpr uint32_t OFF_XCH = OFF_BAR + 1024;  // half-row maxima [group][slot][half][128]
  static constexpr uint32_t OFF_STA = OFF_XCH + 4 * 2 * 2 * 2 * 128;  // tile row max [4][128]
  static constexpr uint32_t OFF_STB = OFF_STA + 4 * 4 * 128;          // tile row sums [4][2][128]
  static constexpr uint32_t OFF_MR = OFF_STB + 4 * 4 * 2 * 128;       // running max [4][128]
  static constexpr uint32_t BYTES = OFF_MR + 4 * 4 * 128;
  static constexpr uint32_t SMEM_ALLOC = BYTES + 1024;  // base alignment slack
  // tensor-memory columns
  static constexpr uint32_t T_S = 0;
  static constexpr uint32_t T_O = 2 * BLK;
  static constexpr uint32_t T_QSF = T_O + D;
  static constexpr uint32_t T_KSF = T_QSF + (D / 64) * 4;
  static constexpr uint32_t T_PSF = T_KSF + 2 * (D / 64) * 4;
  static constexpr uint32_t T_VSF = T_PSF + 2 * (BLK / 64) * 4;
  static constexpr uint32_t T_END = T_VSF + 2 * (BLK / 64) * 4;
  static_assert(T_END <= 512, "tensor memory budget");
  static_assert(NS4 >= 2, "at least two NVFP4 stages");
  static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
};

// Barrier slots inside the barrier area.
//   SF/SE  S buffer full (MMA commit) / read (softmax group)
//   PF     P tile written (softmax group)
//   OD     PV(t) retired into O (MMA commit), one per P slot
//   STA    row max of tile t published (softmax), four slots
//   STB    row sums of tile t published (softmax), four slots
//   MR     running max through tile t published (correction), four slots
//   CF     O rescaled for tile t (correction)
//   XCH    half-row maxima exchanged, per (group, lane quarter, slot)
//   TURN   turn at the exponentials, one per softmax group
// Four-slot rings, each slot reused four tiles later:
//   STA(t+4) is written by the group of tiles t, t+2, t+4 after it stored
//   P(t+2), which waited for PV(t), issued after correction step t had read
//   STA(t);
//   STB(t) is read one correction step late (step t+1); STB(t+4) follows
//   the group's P(t+4), which waited for PV(t+2), issued after step t+2;
//   MR(t+4) is written by correction step t+4 after PV(t+3) retired; PV(t+1)
//   was issued earlier by the same thread, after the softmax of tile t+1
//   (the reader of MR(t)) had finished.
enum : int {
  B_Q4 = 0, B_Q16 = 1, B_SF = 2 /* 2,3 */, B_SE = 4 /* 4,5 */, B_PF = 6 /* 6,7 */,
  B_OD = 8 /* 8,9 */, B_DONE = 10, B_KVF16 = 11 /* 11,12 */, B_KVE16 = 13 /* 13,14 */,
  B_KVF4 = 15 /* 15..26 */, B_KVE4 = 27 /* 27..38 */, B_STA = 39 /* 39..42 */,
  B_STB = 43 /* 43..46 */, B_MR = 47 /* 47..50 */, B_CF = 51, B_XCH = 52 /* 52..67 */,
  B_TURN = 68 /* 68,69 */, B_N = 70
};

constexpr int kSoftmaxWarps = 16;
constexpr int kSoftmaxThreads = 32 * kSoftmaxWarps;
constexpr int kGroupThreads = kSoftmaxThreads / 2;
constexpr int kCorrWarp0 = kSoftmaxWarps;
constexpr int kCorrThreads = 128;
constexpr int kProducerWarp = kSoftmaxWarps + 4;
constexpr int kMmaWarp = kSoftmaxWarps + 5;
constexpr int kPvWarp = kSoftmaxWarps + 6;
constexpr int kAttnThreads = 32 * (kSoftmaxWarps + 7);

// Packed fp32 pairs (one instruction for two lanes' worth of fma / add;
// each half rounds exactly as the scalar operation).
__device__ __forceinline__ void fma2(float& d0, float& d1, float a0, float a1, float b0, float b1,
                                     float c0, float c1) {
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c0), "f"(c1));
}

__device__ __forceinline__ void add2(float& d0, float& d1, float a0, float a1, float b0,
                                     float b1) {
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

__device__ __forceinline__ float lg2_ftz(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// UE4M3 byte (0..126) -> value, with the subnormal case (m * 2^-9) formed by
// the 2^23 magic-number conversion instead of an integer-to-float convert.
__device__ __forceinline__ float ue4m3_decode_fast(uint32_t b) {
  const uint32_t e = b >> 3, mt = b & 7u;
  const float sub = (__uint_as_float(0x4B000000u | mt) - 8388608.0f) * 0.001953125f;
  return e ? __uint_as_float(((e + 120u) << 23) | (mt << 20)) : sub;
}

__device__ __forceinline__ float rcp_ftz(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float ex2_ftz(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Eight fp32 values -> eight E2M1 codes packed in 32 bits (value 2i in the
// low nibble of byte i), round to nearest even, saturating.
__device__ __forceinline__ uint32_t e2m1x8(const float* x) {
  uint32_t out;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(out)
      : "f"(x[0]), "f"(x[1]), "f"(x[2]), "f"(x[3]), "f"(x[4]), "f"(x[5]), "f"(x[6]),
        "f"(x[7]));
  return out;
}

// Two fp32 values -> packed 16-bit pair (lo in bits 0..15), nearest even.
template <int DT>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  if constexpr (DT == 1) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
  } else {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
  }
}

// Materialises a value at this point of the program (an empty asm that
// reads and rewrites it), so that it is not computed later.
__device__ __forceinline__ void pin64(uint64_t& x) { asm volatile("" : "+l"(x)); }

// Waits with every lane of the warp; the result is uniform across the warp.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort) {
  const bool ok = mbar_wait(bar, parity, abort);
  return __all_sync(0xffffffffu, ok);
}

template <int DT, int D, int BLK>
__global__ void __launch_bounds__(kAttnThreads, 1) attn_fwd_kernel(const AttnParams p) {
  using L = AttnLayout<D, BLK>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~(uintptr_t)1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::OFF_BAR);
  uint16_t* s_list = reinterpret_cast<uint16_t*>(sm + L::OFF_LIST);
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + L::OFF_BAR + 8 * B_N);
  int* s_n = reinterpret_cast<int*>(sm + L::OFF_BAR + 8 * B_N + 4);
  int* s_n4 = s_n + 1;
  volatile int* s_abort = s_n + 2;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qt = blockIdx.x, h = blockIdx.y, seq = blockIdx.z;
  int64_t start;
  int len;
  p.seqs.get(seq, start, len);
  if (qt * 128 >= len) return;
  const int hk = h / (p.H / p.Hkv);
  const int nb = (int)ceil_div(len, BLK);
  const int64_t nB2 = (int64_t)p.nB * p.nB;
  const uint8_t* mrow = p.mask + ((int64_t)seq * p.H + h) * nB2;

  if (tid == 0) {
    for (int i = 0; i < B_N; ++i) {
      uint32_t cnt = 1;
      if ((i >= B_SE && i < B_SE + 2) || (i >= B_PF && i < B_PF + 2) ||
          (i >= B_STB && i < B_STB + 4) || (i >= B_TURN && i < B_TURN + 2))
        cnt = kGroupThreads;
      if ((i >= B_STA && i < B_STA + 4) || (i >= B_MR && i < B_MR + 4) || i == B_CF) cnt = 128;
      if (i >= B_XCH && i < B_XCH + 16) cnt = 64;
      if (i == B_DONE) cnt = 2;  // one commit per MMA issuer
      mbar_init(&bars[i], cnt);
    }
    *s_abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    // Tile list: NVFP4 tiles ascending, then FP16 tiles ascending.  Entry:
    // key tile j (bits 0..12), bit 13 + b set when query block b of this CTA
    // (b = 0, 1; one block when BLK = 128) takes tile j on this path, bit 15
    // the path (1 = FP16).  Built by one warp, 32 key tiles per step.
    const int qb0 = BLK == 128 ? qt : 2 * qt;
    const int nqb = BLK == 128 ? 1 : min(2, nb - 2 * qt);
    int n = 0;
    for (int pass = 0; pass < 2; ++pass) {
      for (int j0 = 0; j0 < nb; j0 += 32) {
        const int j = j0 + lane;
        uint32_t bits = 0;
        if (j < nb) {
          for (int b = 0; b < nqb; ++b) {
            if (p.causal && j > qb0 + b) continue;
            if ((__ldg(mrow + (int64_t)(qb0 + b) * p.nB + j) != 0) == (pass == 1))
              bits |= 1u << (13 + b);
          }
        }
        const uint32_t vote = __ballot_sync(0xffffffffu, bits != 0);
        if (bits) s_list[n + __popc(vote & ((1u << lane) - 1u))] = (uint16_t)(j | bits | (pass << 15));
        n += __popc(vote);
      }
      if (pass == 0 && lane == 0) *s_n4 = n;
    }
    if (lane == 0) *s_n = n;
  }
  __syncthreads();
  if (warp == kMmaWarp) {
    tmem_alloc(s_tmem, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;
  const int n = *s_n, n4 = *s_n4;

  uint8_t* q4s = sm + L::OFF4_Q;
  uint8_t* q16s = sm + L::OFF16_Q;

  if (warp == kProducerWarp) {
    // ------------------------------------------------------- producer --
    if (lane == 0) {
      const int64_t qtile = ((int64_t)seq * p.H + h) * p.nTq + qt;
      bool q4_issued = false, q16_issued = false;
      int last4[L::NS4], last16[L::NS16];
      for (int i = 0; i < (int)L::NS4; ++i) last4[i] = -1;
      for (int i = 0; i < (int)L::NS16; ++i) last16[i] = -1;
      if (n4 > 0) {
        mbar_arrive_expect_tx(&bars[B_Q4], L::QT4);
        bulk_g2s(q4s, p.q4 + qtile * L::QT4, L::QT4, &bars[B_Q4]);
        q4_issued = true;
      }
      for (int t = 0; t < n && !*s_abort; ++t) {
        const int j = s_list[t] & 0x1FFF;
        const bool f16 = t >= n4;
        const int64_t ktile = ((int64_t)seq * p.Hkv + hk) * p.nB + j;
        if (!f16) {
          const int i = t, sl = i % L::NS4;
          if (i >= (int)L::NS4 &&
              !mbar_wait(&bars[B_KVE4 + sl], ((i / L::NS4) - 1) & 1, s_abort))
            break;
          uint8_t* stg = sm + L::OFF4_STG + sl * L::STG4;
          mbar_arrive_expect_tx(&bars[B_KVF4 + sl], L::KT4 + L::VT4);
          bulk_g2s(stg, p.k4 + ktile * L::KT4, L::KT4, &bars[B_KVF4 + sl]);
          bulk_g2s(stg + L::V4_OFF, p.v4 + ktile * L::VT4, L::VT4, &bars[B_KVF4 + sl]);
          last4[sl] = i;
        } else {
          const int i = t - n4, sl = i % L::NS16;
          if (i == 0) {
            // the region switches to its FP16 view: the last NVFP4 PV (and
            // with it every NVFP4 read of Q4, P4 and the stages) must be done
            if (n4 > 0 && !mbar_wait(&bars[B_KVE4 + (n4 - 1) % L::NS4],
                                     ((n4 - 1) / L::NS4) & 1, s_abort))
              break;
            mbar_arrive_expect_tx(&bars[B_Q16], L::Q16B);
            bulk_g2s(q16s, p.q16 + qtile * L::Q16B, L::Q16B, &bars[B_Q16]);
            q16_issued = true;
          }
          if (i >= (int)L::NS16 &&
              !mbar_wait(&bars[B_KVE16 + sl], ((i / L::NS16) - 1) & 1, s_abort))
            break;
          uint8_t* stg = sm + L::OFF16_STG + sl * L::STG16;
          mbar_arrive_expect_tx(&bars[B_KVF16 + sl], L::KT16 + L::VT16);
          bulk_g2s(stg, p.k16 + ktile * L::KT16, L::KT16, &bars[B_KVF16 + sl]);
          bulk_g2s(stg + L::V16_OFF, p.v16 + ktile * L::VT16, L::VT16, &bars[B_KVF16 + sl]);
          last16[sl] = i;
        }
      }
      // Drain: every copy this thread issued has landed before the CTA ends.
      int dummy = 0;
      volatile int* never = &dummy;
      if (q4_issued) mbar_wait(&bars[B_Q4], 0, never, 200000000ull);
      if (q16_issued) mbar_wait(&bars[B_Q16], 0, never, 200000000ull);
      for (int sl = 0; sl < (int)L::NS4; ++sl)
        if (last4[sl] >= 0)
          mbar_wait(&bars[B_KVF4 + sl], (last4[sl] / L::NS4) & 1, never, 200000000ull);
      for (int sl = 0; sl < (int)L::NS16; ++sl)
        if (last16[sl] >= 0)
          mbar_wait(&bars[B_KVF16 + sl], (last16[sl] / L::NS16) & 1, never, 200000000ull);
    }
  } else if (warp == kMmaWarp || warp == kPvWarp) {
    // ---------------------------------------------------- MMA issuers --
    // One warp issues QK^T for every tile in order (warp kMmaWarp), another
    // PV (warp kPvWarp), so scores for the next tiles never queue behind a PV
    // that waits for its P tile or for the correction step.  The whole warp
    // runs the loop and its waits, so the operand descriptors are uniform
    // across it; one elected lane issues the tensor instructions and their
    // commits.  QK^T(t) reads the K half of its stage before PV(t) is issued
    // (PV(t) follows P(t), which follows the scores of tile t), so the PV
    // side's commit alone frees the stage.  The lane is elected once, so
    // every tensor instruction of the warp and the commits that track them
    // come from the same thread.
    {
      const bool leader = elect_one();
      constexpr uint32_t id_qk4 = idesc_nvf4(128, BLK), id_pv4 = idesc_nvf4(128, D);
      constexpr uint32_t id_qk16 = idesc_f16(DT, 128, BLK), id_pv16 = idesc_f16(DT, 128, D);
      constexpr uint32_t swz_d = swz_mode_for_pitch(D / 2), swz_b = swz_mode_for_pitch(BLK / 2);
      // Descriptors of every operand at stage / slot 0, built once: a
      // descriptor's start field is the address in 16-byte units, so an
      // operand at byte offset o further on is the descriptor + (o >> 4).
      const uint32_t base = smem_u32(sm);
      const uint64_t d_sf = make_sdesc(base, 512, 128, SW_NONE);  // + (byte offset >> 4)
      int sl = 0, par = 0;  // stage ring position (NVFP4 ring, then FP16 ring)
      auto advance = [&](int t) {
        const int ns = t < n4 ? (int)L::NS4 : (int)L::NS16;
        if (t + 1 == n4) {
          sl = 0;
          par = 0;
        } else if (++sl == ns) {
          sl = 0;
          par ^= 1;
        }
      };
      bool ok = true;
      if (warp == kMmaWarp) {
        const uint64_t d_q4 = make_sdesc(base + L::OFF4_Q, 16, 8 * (D / 2), swz_d);
        const uint64_t d_k4 = make_sdesc(base + L::OFF4_STG, 16, 8 * (D / 2), swz_d);
        const uint64_t d_q16 = make_sdesc(base + L::OFF16_Q, 16, 1024, SW_128B);
        const uint64_t d_k16 = make_sdesc(base + L::OFF16_STG, 16, 1024, SW_128B);
        bool q4_ready = false, q16_ready = false;
        for (int t = 0; t < n && ok; ++t) {
          const int st = t & 1;
          const bool f16 = t >= n4;
          uint64_t* full = f16 ? &bars[B_KVF16 + sl] : &bars[B_KVF4 + sl];
          // NVFP4 operands first, then the waits
          const uint32_t dS = tmem + L::T_S + st * BLK;
          const uint32_t ksf = tmem + L::T_KSF + st * (D / 64) * 4;
          const uint32_t so = (uint32_t)sl * ((f16 ? L::STG16 : L::STG4) >> 4);
          uint64_t cpk[D / 64], db[D / 64];
#pragma unroll
          for (int s = 0; s < D / 64; ++s) {
            cpk[s] = d_sf + ((L::OFF4_STG + BLK * (D / 2) + 512 * s) >> 4) + so;
            db[s] = d_k4 + so + 2 * s;
            pin64(cpk[s]);
            pin64(db[s]);
          }
          if (!warp_wait(full, par, s_abort)) { ok = false; break; }
          if (!f16 && !q4_ready) {
            if (!warp_wait(&bars[B_Q4], 0, s_abort)) { ok = false; break; }
            tc_fence_after();
            if (leader) {
#pragma unroll
              for (int s = 0; s < D / 64; ++s)
                tc_cp_32x128b_x4(tmem + L::T_QSF + 4 * s,
                                 d_sf + ((L::OFF4_Q + 128 * (D / 2) + 512 * s) >> 4));
            }
            __syncwarp();
            q4_ready = true;
          }
          if (f16 && !q16_ready) {
            if (!warp_wait(&bars[B_Q16], 0, s_abort)) { ok = false; break; }
            q16_ready = true;
          }
          // the S buffer of tile t-2 has been read
          if (t >= 2 && !warp_wait(&bars[B_SE + st], ((t >> 1) - 1) & 1, s_abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (leader) {
            if (!f16) {
#pragma unroll
              for (int s = 0; s < D / 64; ++s) tc_cp_32x128b_x4(ksf + 4 * s, cpk[s]);
#pragma unroll
              for (int s = 0; s < D / 64; ++s)
                mma_nvf4(dS, d_q4 + 2 * s, db[s], id_qk4, tmem + L::T_QSF + 4 * s, ksf + 4 * s,
                         s > 0);
            } else {
#pragma unroll
              for (int s = 0; s < D / 16; ++s)
                mma_f16(dS, d_q16 + ((s / 4) * 128 * 128 >> 4) + 2 * (s % 4),
                        d_k16 + so + ((s / 4) * BLK * 128 >> 4) + 2 * (s % 4), id_qk16, s > 0);
            }
            tc_commit(&bars[B_SF + st]);
          }
          __syncwarp();
          advance(t);
        }
      } else {
        const uint64_t d_p4 = make_sdesc(base + L::OFF4_P, 16, 8 * (BLK / 2), swz_b);
        const uint64_t d_v4 = make_sdesc(base + L::OFF4_STG + L::V4_OFF, 16, 8 * (BLK / 2), swz_b);
        const uint64_t d_p16 = make_sdesc(base + L::OFF16_P, 16, 1024, SW_128B);
        const uint64_t d_v16 = make_sdesc(base + L::OFF16_STG + L::V16_OFF, 16, 1024, SW_128B);
        const uint32_t dO = tmem + L::T_O;
        for (int t = 0; t < n && ok; ++t) {
          const int st = t & 1;
          const bool f16 = t >= n4;
          uint64_t* empty = f16 ? &bars[B_KVE16 + sl] : &bars[B_KVE4 + sl];
          // NVFP4 operands first: the waits below end when the correction
          // step finishes, and from there on only the tensor instructions
          // remain.
          const uint32_t so = (uint32_t)sl * ((f16 ? L::STG16 : L::STG4) >> 4);
          const uint32_t po = (uint32_t)st * (L::PT4A >> 4);
          const uint32_t psf = tmem + L::T_PSF + st * (BLK / 64) * 4;
          const uint32_t vsf = tmem + L::T_VSF + st * (BLK / 64) * 4;
          uint64_t da[BLK / 64], db[BLK / 64], cpp[BLK / 64], cpv[BLK / 64];
#pragma unroll
          for (int s = 0; s < BLK / 64; ++s) {
            cpp[s] = d_sf + ((L::OFF4_P + 128 * (BLK / 2) + 512 * s) >> 4) + po;
            cpv[s] = d_sf + ((L::OFF4_STG + L::V4_OFF + D * (BLK / 2) + 512 * s) >> 4) + so;
            da[s] = d_p4 + po + 2 * s;
            db[s] = d_v4 + so + 2 * s;
            pin64(cpp[s]);
            pin64(cpv[s]);
            pin64(da[s]);
            pin64(db[s]);
          }
          if (!warp_wait(&bars[B_PF + st], (t >> 1) & 1, s_abort)) { ok = false; break; }
          if (!warp_wait(&bars[B_CF], t & 1, s_abort)) { ok = false; break; }  // O rescaled
          tc_fence_after();
          if (leader) {
            if (!f16) {
#pragma unroll
              for (int s = 0; s < BLK / 64; ++s) {
                tc_cp_32x128b_x4(psf + 4 * s, cpp[s]);
                tc_cp_32x128b_x4(vsf + 4 * s, cpv[s]);
              }
#pragma unroll
              for (int s = 0; s < BLK / 64; ++s)
                mma_nvf4(dO, da[s], db[s], id_pv4, psf + 4 * s, vsf + 4 * s, t > 0 || s > 0);
            } else {
#pragma unroll
              for (int s = 0; s < BLK / 16; ++s)
                mma_f16(dO, d_p16 + ((s / 4) * 128 * 128 >> 4) + 2 * (s % 4),
                        d_v16 + so + ((s / 4) * D * 128 >> 4) + 2 * (s % 4), id_pv16,
                        t > 0 || s > 0);
            }
            tc_commit(&bars[B_OD + st]);
            tc_commit(empty);
          }
          __syncwarp();
          advance(t);
        }
      }
      // every MMA of both issuers has completed before the CTA ends
      if (leader) tc_commit(&bars[B_DONE]);
      __syncwarp();
      int dummy = 0;
      volatile int* never = &dummy;
      mbar_wait(&bars[B_DONE], 0, never, 200000000ull);
    }
  } else if (warp >= kCorrWarp0) {
    // ----------------------------------------------------- correction --
    // One thread per query row; it owns the row's running max m and sum l.
    // The true output accumulator is ref * O, O being the tensor-memory
    // accumulator.  Tile t, taken by the softmax relative to its own row max
    // mt (NVFP4) or to the running max (FP16), asks for
    //   true O <- alpha * true O + sigma * PV(t)
    // with alpha = 2^(m - m_new) and sigma = 2^(mt - m_new) / 2688 * g_V
    // (NVFP4) or 1 (FP16).  The MMA only adds PV(t), so before it does, O is
    // multiplied by beta = alpha * ref / sigma and ref becomes sigma.  An
    // NVFP4 tile whose row factor is negligible (2^(mt - m_new) < 2^-60) or
    // not a normal float adds nothing: its row of P gets zero block scales.
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;
    const int row = qt * 128 + r;
    const bool row_ok = row < len;
    const uint32_t o_base = tmem + ((uint32_t)(q4 * 32) << 16) + L::T_O;
    const float* sta = reinterpret_cast<const float*>(sm + L::OFF_STA);
    const float* stb = reinterpret_cast<const float*>(sm + L::OFF_STB);
    float* mrw = reinterpret_cast<float*>(sm + L::OFF_MR);
    const float gv = tensor_scale_from_amax(p.amax[2]);
    float m = -INFINITY, l = 0.0f, ref = 1.0f;
    float pend_alpha = 1.0f, pend_sigma_raw = 0.0f;
    bool ok = true;
    // l <- alpha * l + sigma_raw * (row sum of tile u), in tile order
    auto accumulate_l = [&](int u) -> bool {
      const int s4 = u & 3;
      if (!warp_wait(&bars[B_STB + s4], (u >> 2) & 1, s_abort)) return false;
      const float ls = stb[(2 * s4) * 128 + r] + stb[(2 * s4 + 1) * 128 + r];
      l *= pend_alpha;
      l = u >= n4 ? l + ls : fmaf(ls, pend_sigma_raw, l);
      return true;
    };
    for (int t = 0; t < n; ++t) {
      const int s4 = t & 3;
      const bool f16 = t >= n4;
      if (!warp_wait(&bars[B_STA + s4], (t >> 2) & 1, s_abort)) { ok = false; break; }
      const float mt = sta[s4 * 128 + r];
      const float m_new = fmaxf(m, mt);
      const float alpha = (m == -INFINITY) ? 1.0f : ex2_ftz(m - m_new);
      float sigma = 1.0f, sigma_raw = 1.0f;
      bool drop = false;
      if (!f16) {
        const bool live = mt != -INFINITY;
        const float rowmax = live ? ex2_ftz(mt - m_new) : 0.0f;
        sigma_raw = (live && rowmax >= 8.6736174e-19f) ? rowmax * (1.0f / 2688.0f) : 0.0f;  // 2^-60
        sigma = sigma_raw * gv;
        if (!(sigma >= 1.17549435e-38f)) sigma = sigma_raw = 0.0f;
        drop = live && sigma == 0.0f;
      }
      // running max through tile t, for the FP16 softmax of tile t+1
      mrw[s4 * 128 + r] = m_new;
      mbar_arrive(&bars[B_MR + s4]);
      m = m_new;
      float beta = 1.0f;
      if (sigma > 0.0f) {
        if (t > 0) beta = alpha * ref * rcp_ftz(sigma);
        ref = sigma;
      } else {
        ref *= alpha;
      }
      // PV(t-1) has to be in O before O is rescaled.  The wait also keeps
      // this arrival on CF from running a phase ahead of the MMA issuer,
      // which consumed CF(t-1) before issuing PV(t-1).
      if (t > 0 && !warp_wait(&bars[B_OD + ((t - 1) & 1)], ((t - 1) >> 1) & 1, s_abort)) {
        ok = false;
        break;
      }
      if (t > 0 && __any_sync(0xffffffffu, beta != 1.0f)) {
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < D; c += 32) {
          float v[32];
          tmem_ld32(o_base + c, v);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; i += 2)
            fma2(v[i], v[i + 1], v[i], v[i + 1], beta, beta, 0.0f, 0.0f);
          tmem_st32(o_base + c, v);
        }
        tmem_st_wait();
      }
      if (__any_sync(0xffffffffu, drop)) {
        // zero this row's block scales once P(t) is in shared memory
        if (!warp_wait(&bars[B_PF + (t & 1)], (t >> 1) & 1, s_abort)) { ok = false; break; }
        if (drop) {
          uint8_t* psf = sm + L::OFF4_P + (t & 1) * L::PT4A + 128 * (BLK / 2);
#pragma unroll
          for (int a = 0; a < BLK / 64; ++a)
            *reinterpret_cast<uint32_t*>(psf + sf_offset(r, 4 * a)) = 0u;
        }
        fence_proxy_async_smem();
      }
      tc_fence_before();
      mbar_arrive(&bars[B_CF]);
      // the row sum of tile t-1 (two column halves), one step late: it is
      // published after P(t-1), which PV(t-1), waited for above, follows
      if (t > 0) {
        if (!accumulate_l(t - 1)) { ok = false; break; }
      }
      pend_alpha = alpha;
      pend_sigma_raw = sigma_raw;
    }
    if (ok && n > 0) ok = accumulate_l(n - 1);
    // epilogue: O * ref / l after the last PV
    if (ok && n > 0) ok = warp_wait(&bars[B_OD + ((n - 1) & 1)], ((n - 1) >> 1) & 1, s_abort);
    if (ok) {
      tc_fence_after();
      const float il = (l > 0.0f && n > 0) ? ref / l : 0.0f;
      uint16_t* orow = p.out + ((start + (row_ok ? row : 0)) * p.H + h) * D;
#pragma unroll 1
      for (int c = 0; c < D; c += 32) {
        float v[32];
        if (n > 0) {
          tmem_ld32(o_base + c, v);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = 0.0f;
        }
        if (row_ok) {
#pragma unroll
          for (int i = 0; i < 32; i += 8) {
            uint4 w;
            w.x = pack2<DT>(v[i] * il, v[i + 1] * il);
            w.y = pack2<DT>(v[i + 2] * il, v[i + 3] * il);
            w.z = pack2<DT>(v[i + 4] * il, v[i + 5] * il);
            w.w = pack2<DT>(v[i + 6] * il, v[i + 7] * il);
            *reinterpret_cast<uint4*>(orow + c + i) = w;
          }
        }
      }
      if (row_ok) {
        const float lse = l > 0.0f ? m * 0.6931471805599453f + logf(l) : -INFINITY;
        const int64_t li = p.lse_varlen ? (int64_t)h * p.total + start + row
                                        : ((int64_t)seq * p.H + h) * len + row;
        p.lse[li] = lse;
      }
    }
  } else {
    // -------------------------------------------------------- softmax --
    // Two groups of eight warps take alternate key tiles: group g = w / 8
    // the tiles t = g, g + 2, ... (S buffer and P slot g).  Within a group,
    // query row r (TMEM lane r) is shared by the warps r/32 + 4(2g + hf),
    // hf = 0, 1, each owning half of the key columns.  The groups take turns
    // at the exponentials, so one group's loads and reductions run while the
    // other keeps the MUFU busy.  No running state lives here: an NVFP4 tile
    // is taken relative to its own row max, an FP16 tile relative to the
    // running max published by the correction warps.
    constexpr int SC = BLK / 2;   // score columns per thread
    constexpr int NCH = SC / 32;  // 32-column chunks
    const int q4 = warp & 3, f = warp >> 2, g = f >> 1, hf = f & 1;
    const int r = q4 * 32 + lane;
    const int row = qt * 128 + r;
    const bool row_ok = row < len;
    const int mbit = 13 + ((BLK == 64 && r >= 64) ? 1 : 0);  // tile-list bit of this row's block
    const float gq = tensor_scale_from_amax(p.amax[0]);
    const float gk = tensor_scale_from_amax(p.amax[1]);
    const float cs4 = __fmul_rn(__fmul_rn(gq, gk), p.scale4);
    const float corr_r =
        (p.corr != nullptr && row_ok)
            ? __ldg(p.corr + ((int64_t)seq * p.H + h) * ((int64_t)p.nTq * 128) + row) * p.scale4
            : 0.0f;
    const uint32_t s_base = tmem + ((uint32_t)(q4 * 32) << 16) + L::T_S + g * BLK + hf * SC;
    float* xch = reinterpret_cast<float*>(sm + L::OFF_XCH) + g * 512;  // [2 slots][2 halves][128]
    float* sta = reinterpret_cast<float*>(sm + L::OFF_STA);
    float* stb = reinterpret_cast<float*>(sm + L::OFF_STB);
    const float* mr = reinterpret_cast<const float*>(sm + L::OFF_MR);
    uint64_t* xbar = &bars[B_XCH + (g * 4 + q4) * 2];
    // shared-memory offsets this thread writes every NVFP4 tile
    uint32_t p4_codes_off[NCH];
#pragma unroll
    for (int c = 0; c < NCH; ++c) p4_codes_off[c] = swz_offset(r, hf * (SC / 2) + 16 * c, BLK / 2);
    const uint32_t p4_sf_off = 128 * (BLK / 2) + sf_offset(r, hf * (SC / 16));
    uint8_t* p4 = sm + L::OFF4_P + g * L::PT4A;
    uint8_t* p16 = sm + L::OFF16_P;
    bool ok = true;
    // the first turn at the exponentials goes to group 0
    if (g == 1) mbar_arrive(&bars[B_TURN]);

    for (int t = g; t < n && ok; t += 2) {
      const int u = t >> 1;  // this group's tile count
      const uint32_t ent = s_list[t];
      const int j = ent & 0x1FFF;
      const bool f16 = (ent >> 15) != 0;
      const bool pair_ok = row_ok && ((ent >> mbit) & 1u);
      // last valid score column of this thread's half (negative: none)
      const int lim = (pair_ok ? min(len - 1, p.causal ? row : len - 1) - j * BLK : -1) - hf * SC;
      const bool full = __all_sync(0xffffffffu, lim >= SC - 1);
      const float cs = f16 ? p.scale16 : cs4;
      if (!warp_wait(&bars[B_SF + g], u & 1, s_abort)) { ok = false; break; }
      tc_fence_after();
      // pass 1: block maxima of the raw scores (the scale is positive)
      float bm[2 * NCH];
#pragma unroll
      for (int c = 0; c < NCH; ++c) {
        float a[32];
        tmem_ld32(s_base + 32 * c, a);
        tmem_ld_wait();
        if (!full) {
#pragma unroll
          for (int i = 0; i < 32; ++i) a[i] = i + 32 * c <= lim ? a[i] : -INFINITY;
        }
#pragma unroll
        for (int b = 0; b < 2; ++b) {
          const float* x = a + 16 * b;
          float x0 = fmaxf(x[0], x[1]), x1 = fmaxf(x[2], x[3]);
          float x2 = fmaxf(x[4], x[5]), x3 = fmaxf(x[6], x[7]);
          x0 = fmaxf(x0, fmaxf(x[8], x[9]));
          x1 = fmaxf(x1, fmaxf(x[10], x[11]));
          x2 = fmaxf(x2, fmaxf(x[12], x[13]));
          x3 = fmaxf(x3, fmaxf(x[14], x[15]));
          bm[2 * c + b] = fmaxf(fmaxf(x0, x1), fmaxf(x2, x3));
        }
      }
      float mh = bm[0];
#pragma unroll
      for (int b = 1; b < 2 * NCH; ++b) mh = fmaxf(mh, bm[b]);
      // exchange the half-row maxima with the partner warp
      float* xs = xch + (u & 1) * 256;
      xs[hf * 128 + r] = mh;
      mbar_arrive(&xbar[u & 1]);
      if (!warp_wait(&xbar[u & 1], (u >> 1) & 1, s_abort)) { ok = false; break; }
      const float mt_raw = fmaxf(xs[r], xs[128 + r]);
      const bool live = mt_raw != -INFINITY;  // this row has a valid key in the tile
      const float mt = mt_raw * cs;
      if (hf == 0) {
        // with K smoothing the NVFP4 scores miss q^ . mu, a constant of the
        // row: the probabilities (relative to mt) do not see it, the tile's
        // maximum handed to the correction warps does
        sta[(t & 3) * 128 + r] = (f16 || !live) ? mt : mt + corr_r;
        mbar_arrive(&bars[B_STA + (t & 3)]);
      }
      float ls = 0.0f;
      if (!f16) {
        // Two-level quantisation of P.  Relative to the tile max the scaled
        // probabilities are Phat = 2688 * 2^(s - mt); block b gets the UE4M3
        // scale S_b = ue4m3(max Phat / 6) and the codes E2M1(Phat / S_b),
        // computed as one exponential t = 2^(s + log2(2688) - mt - log2 S_b).
        // The row sum of the tile, relative to 2688 * 2^-mt, is
        // sum_b S_b * sum(t).
        // block scales first, outside the turn
        float dec[2 * NCH], cc[2 * NCH];
        uint32_t sfw = 0;
#pragma unroll
        for (int b = 0; b < 2 * NCH; ++b) {
          const float e = ex2_ftz(fmaf(bm[b], cs, -mt));  // block max / tile max
          const uint32_t S = live ? ue4m3(448.0f * e) : 0u;
          dec[b] = ue4m3_decode_fast(S);
          cc[b] = S ? 11.392317422778760f - mt - lg2_ftz(dec[b]) : -INFINITY;  // log2(2688)
          sfw |= S << (8 * b);
        }
        if (!warp_wait(&bars[B_TURN + g], u & 1, s_abort)) { ok = false; break; }
        uint32_t cw[NCH][4];
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
          float a[32];
          tmem_ld32(s_base + 32 * c, a);
          tmem_ld_wait();
          if (c == NCH - 1) {
            tc_fence_before();
            mbar_arrive(&bars[B_SE + g]);  // S buffer free for QK^T of tile t+2
          }
          if (!full) {
#pragma unroll
            for (int i = 0; i < 32; ++i) a[i] = i + 32 * c <= lim ? a[i] : -INFINITY;
          }
#pragma unroll
          for (int b2 = 0; b2 < 2; ++b2) {
            const int b = 2 * c + b2;
            float* x = a + 16 * b2;
            // all sixteen exponent arguments, then all sixteen exponentials
            // (independent, so they stream through the MUFU back to back),
            // then a sum tree
#pragma unroll
            for (int i = 0; i < 16; i += 2)
              fma2(x[i], x[i + 1], x[i], x[i + 1], cs, cs, cc[b], cc[b]);
#pragma unroll
            for (int i = 0; i < 16; ++i) x[i] = ex2_ftz(x[i]);  // masked (-inf) -> 0
            float y[8];
#pragma unroll
            for (int i = 0; i < 8; i += 2)
              add2(y[i], y[i + 1], x[2 * i], x[2 * i + 1], x[2 * i + 2], x[2 * i + 3]);
            add2(y[0], y[1], y[0], y[1], y[2], y[3]);
            add2(y[4], y[5], y[4], y[5], y[6], y[7]);
            add2(y[0], y[1], y[0], y[1], y[4], y[5]);
            ls = fmaf(y[0] + y[1], dec[b], ls);
            cw[c][2 * b2] = e2m1x8(x);
            cw[c][2 * b2 + 1] = e2m1x8(x + 8);
          }
        }
        if (t + 1 < n) mbar_arrive(&bars[B_TURN + (1 - g)]);
        // P slot g was last read by PV(t-2)
        if (u >= 1 && !warp_wait(&bars[B_OD + g], (u - 1) & 1, s_abort)) { ok = false; break; }
#pragma unroll
        for (int c = 0; c < NCH; ++c)
          *reinterpret_cast<uint4*>(p4 + p4_codes_off[c]) =
              make_uint4(cw[c][0], cw[c][1], cw[c][2], cw[c][3]);
        if constexpr (NCH == 2) {
          *reinterpret_cast<uint32_t*>(p4 + p4_sf_off) = sfw;
        } else {
          *reinterpret_cast<uint16_t*>(p4 + p4_sf_off) = (uint16_t)sfw;
        }
      } else {
        // FP16 tile: P = 2^(s - m_new) against the running max through t
        float m_prev = -INFINITY;
        if (t > 0) {
          if (!warp_wait(&bars[B_MR + ((t - 1) & 3)], ((t - 1) >> 2) & 1, s_abort)) {
            ok = false;
            break;
          }
          m_prev = mr[((t - 1) & 3) * 128 + r];
        }
        const float m_new = fmaxf(m_prev, mt);
        const float negm = m_new == -INFINITY ? 0.0f : -m_new;
        if (!warp_wait(&bars[B_TURN + g], u & 1, s_abort)) { ok = false; break; }
        uint32_t w[NCH][16];
        float l0 = 0.0f, l1 = 0.0f;
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
          float a[32];
          tmem_ld32(s_base + 32 * c, a);
          tmem_ld_wait();
          if (c == NCH - 1) {
            tc_fence_before();
            mbar_arrive(&bars[B_SE + g]);
          }
          if (!full) {
#pragma unroll
            for (int i = 0; i < 32; ++i) a[i] = i + 32 * c <= lim ? a[i] : -INFINITY;
          }
#pragma unroll
          for (int h16 = 0; h16 < 32; h16 += 16) {
            float* x = a + h16;
#pragma unroll
            for (int i = 0; i < 16; i += 2) fma2(x[i], x[i + 1], x[i], x[i + 1], cs, cs, negm, negm);
#pragma unroll
            for (int i = 0; i < 16; ++i) x[i] = ex2_ftz(x[i]);  // exp2(-inf) = 0 when masked
#pragma unroll
            for (int i = 0; i < 16; i += 2) {
              add2(l0, l1, l0, l1, x[i], x[i + 1]);
              w[c][(h16 + i) >> 1] = pack2<DT>(x[i], x[i + 1]);
            }
          }
        }
        ls = l0 + l1;
        if (t + 1 < n) mbar_arrive(&bars[B_TURN + (1 - g)]);
        // one P buffer: the previous FP16 PV must be done.  (The first FP16
        // tile needs no wait: its scores only arrive after the last NVFP4
        // PV has retired.)
        if (t > n4 && !warp_wait(&bars[B_OD + ((t - 1) & 1)], ((t - 1) >> 1) & 1, s_abort)) {
          ok = false;
          break;
        }
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
#pragma unroll
          for (int q8 = 0; q8 < 4; ++q8) {
            const uint32_t key0 = hf * SC + 32 * c + 8 * q8;
            *reinterpret_cast<uint4*>(p16 + (key0 / 64) * 128 * 128 +
                                      swz_offset(r, (key0 % 64) * 2, 128)) =
                make_uint4(w[c][4 * q8], w[c][4 * q8 + 1], w[c][4 * q8 + 2], w[c][4 * q8 + 3]);
          }
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(&bars[B_PF + g]);
      stb[(2 * (t & 3) + hf) * 128 + r] = ls;
      mbar_arrive(&bars[B_STB + (t & 3)]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace thrift
