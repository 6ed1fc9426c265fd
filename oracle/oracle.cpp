// CPU oracle for NVFP4 attention with ThriftAttention-style selective mixed
// precision.  TEST INFRASTRUCTURE ONLY: tests, the smoke check and the CPU
// baseline leg of the benchmark may load this library; the product path never
// does.  It shares no code, header or table with the CUDA path.
//
// Plain, slow and sequential on purpose.  Every rounding is an IEEE-754
// correctly rounded fp32/fp64 operation (built with -ffp-contract=off, no
// fast-math); fused multiply-adds are written out explicitly with fmaf/fma
// where the method's reading calls for them.
//
// Sources (the web pages this method is taken from):
//  * "Attn-QAT: 4-Bit Attention With Quantization-Aware Training",
//    Resumo tecnico section 1: the FP4 (E2M1) element has 15 distinct values.
//  * "ThriftAttention" (Resumen Tecnico), Metodologia step 1 (block-mean
//    importance S^_ij = qbar_i . kbar_j, top-k pairs) and step 2 (FP16 path for
//    the selected pairs, NVFP4 path for the rest, FlashAttention-2 style online
//    softmax merge, two-level quantisation of the probability blocks), and the
//    kernel paragraph after it (FP4 blocks first, FP16 helper afterwards).
//  * "Busca tus Escalas de Punto Flotante por Bloques" (ScaleSearch),
//    Declaracion del Problema (NVFP4 block scale is E4M3 with mantissa bits),
//    ScaleSearch "Mecanismo" (max scaling s = round(||x||_inf / 6) and the
//    bit-offset candidate s(f)), "Estrategia de Busqueda" (f in [-2, 6],
//    argmin of block MSE), and ScaleSearchAttention (Hadamard rotation of Q
//    and K; QK^T and PV in NVFP4 with FP32 accumulation).
//
// Readings taken where the pages are silent (each is a choice, stated once):
//  R1  block size 16, FP32 per-tensor scale g = amax/2688 (2688 = 6*448),
//      g = 1 when the tensor is all zero.
//  R2  E2M1 and UE4M3 conversions round to nearest, ties to even, saturating.
//  R3  max scaling: S = UE4M3(amax_b / (6 g)); codes = E2M1(x * (1/(S g))).
//  R4  ScaleSearch error of candidate f: fp32 sum, in element order, of
//      (t - q)^2 with fmaf, times S_f^2 in fp64; candidates visited in the
//      order 0,-2,-1,1,2,3,4,5,6; bytes outside 1..126 skipped; first strict
//      minimum kept; a block whose max-scaling byte is 0 keeps byte 0.
//  R5  Hadamard: unnormalised Sylvester transform, butterflies of stride
//      1,2,4,...,d/2 in fp32, (a,b) -> (a+b, a-b); the 1/d is folded into the
//      softmax scale.
//  R6  16-blocks run along the contraction axis: Q,K along d; V along tokens;
//      P along keys.
//  R7  P: per row and key tile sigma = rowmax/2688, Phat = P * (2688/rowmax),
//      NVFP4 with block scale UE4M3(amax/6) and no tensor scale.
//  R8  block means in fp64 over the unrotated 16-bit inputs; scores by a
//      sequential fp64 fma; k = ceil(frac * n_valid - 1e-9) per (batch, head)
//      over the valid pairs; ties go to the lower linear index i*nB + j.
//  R9  FP16 path: unrotated 16-bit Q, K, V; P rounded to the input dtype;
//      l accumulates the fp32 probabilities before rounding.
//  R14 sink-aware mixed precision (optional, off when both counts are 0):
//      the first `sink` key blocks, and the `recent` most recent key blocks a
//      query block can see, run on the FP16 path for every query block; the
//      fixed pairs are OR-ed with the top-k pairs, whose quota is unchanged.
//  R16 K smoothing (optional; "ThriftAttention" / Attn-QAT pages name Q/K
//      smoothing among the outlier mitigations of earlier FP4 attention):
//      mu = the mean of each K channel over the tokens of its sequence (per kv
//      head): fp64 sums in token order within 128-token blocks, the block
//      sums added in order, divided by the length, rounded to fp32.  The
//      NVFP4 path quantises K' = fl32(k - mu) (its own tensor scale) and
//      scores q^ . (k'^ + mu), i.e. the dequantised smoothed key with the
//      mean added back, so both paths keep the same scores; the FP16 path and
//      the selection use the raw K.  Not combined with the Hadamard rotation.
//  R17 Attn-QAT backward ("Attn-QAT", Metodologia, items 1 and 2): the forward
//      runs on fake-quantised NVFP4 Q^, K^, V^ (dequantised values) with the
//      probabilities quantised in two levels per (row, key tile) as in R7;
//      the backward treats every quantiser as the identity for gradients
//      (straight-through), recomputes P = exp(S - lse) and its FP4 image P^
//      from the same scales, and takes the scalar of the softmax gradient
//      from a high-precision output O' = P V^ (not from the FP4 output
//      O = P^ V^):  D = rowsum(dO o O'),  dV = P^T^ dO,  dP = dO V^T^,
//      dS = P o (dP - D),  dQ = dS K^ / sqrt(d),  dK = dS^T Q^ / sqrt(d).
//  R15 decode on the double cache (ThriftAttention, Resultados: decode
//      speed-up; Significado: the KV cache grows by 28% because every token
//      is cached in FP16 and in FP4): one new query token per sequence
//      attends to the len_b cached tokens of its sequence (its own key
//      included).  The cache holds K and V in 16 bits and in NVFP4 (K
//      blocks along d; V 16-token blocks along the tokens from token 0, the
//      last block zero-padded) under per-tensor scales g_K, g_V fixed by the
//      caller when the cache is filled (a growing cache cannot re-derive
//      its amax).  q is quantised with g_Q = amax(q of the step) / 2688.
//      Selection: the query block is the query itself (qbar = q), kbar_j
//      the mean of the cached 16-bit keys of block j; k = ceil(frac * nb)
//      per (sequence, head) over the nb key blocks, ties to the lower j;
//      fixed pairs: j < sink or j >= nb - recent.  The row then follows the
//      prefill steps: NVFP4 tiles ascending, then FP16 tiles ascending, one
//      online softmax.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <cstdlib>
#include <vector>
#include <thread>
#include <atomic>
#include <algorithm>
#include <limits>
#include <functional>

extern "C" {

// ---------------------------------------------------------------- formats --

// E2M1 magnitudes indexed by the 3-bit magnitude code (Attn-QAT, Resumo
// tecnico 1: sixteen codes, +0 and -0 coincide, so 15 distinct values).
static const float kE2M1Mag[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};

// Nearest E2M1 magnitude by exhaustive comparison; ties go to the even code.
// Values above 6 saturate to 6.  The sign bit copies the sign of t (so -0.0
// and tiny negatives give 0x8).
uint8_t orc_e2m1_encode(float t) {
  uint8_t sign = std::signbit(t) ? 0x8 : 0x0;
  double a = std::fabs((double)t);
  if (std::isnan(t)) return sign | 0x7;  // not produced by the method
  if (a >= 6.0) return sign | 0x7;       // saturation at the largest value
  int best = 0;
  double best_d = std::fabs(a - kE2M1Mag[0]);
  for (int c = 1; c < 8; ++c) {
    double dd = std::fabs(a - kE2M1Mag[c]);
    if (dd < best_d || (dd == best_d && (c % 2) == 0 && (best % 2) == 1)) {
      best = c;
      best_d = dd;
    }
  }
  return sign | (uint8_t)best;
}

float orc_e2m1_decode(uint8_t code) {
  float m = kE2M1Mag[code & 0x7];
  return (code & 0x8) ? -m : m;
}

// UE4M3 (unsigned E4M3FN: 4 exponent bits, bias 7, 3 mantissa bits,
// subnormals m * 2^-9, 0x7F is NaN, largest finite 448).
float orc_ue4m3_decode(uint8_t b) {
  b &= 0x7F;
  int e = b >> 3, m = b & 7;
  if (b == 0x7F) return std::numeric_limits<float>::quiet_NaN();
  if (e == 0) return std::ldexp((float)m, -9);
  return std::ldexp(1.0f + (float)m / 8.0f, e - 7);
}

// Nearest of the 127 finite UE4M3 values by exhaustive search, ties to the
// even byte, saturating at 448.  Negative inputs map to 0 (scales are >= 0).
uint8_t orc_ue4m3_encode(float v) {
  if (!(v > 0.0f)) return 0;
  if (v >= 448.0f) return 0x7E;
  int best = 0;
  double best_d = std::fabs((double)v);
  for (int b = 1; b <= 0x7E; ++b) {
    double dd = std::fabs((double)v - (double)orc_ue4m3_decode((uint8_t)b));
    if (dd < best_d || (dd == best_d && (b % 2) == 0 && (best % 2) == 1)) {
      best = b;
      best_d = dd;
    }
  }
  return (uint8_t)best;
}

void orc_e2m1_encode_array(const float* x, int64_t n, uint8_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_e2m1_encode(x[i]);
}
void orc_ue4m3_encode_array(const float* x, int64_t n, uint8_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_ue4m3_encode(x[i]);
}

// 16-bit storage types: 0 = IEEE fp16, 1 = bfloat16.  Both widen to fp32
// exactly.
float orc_half_to_float(uint16_t h, int dt) {
  if (dt == 1) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    std::memcpy(&f, &u, 4);
    return f;
  }
  int s = (h >> 15) & 1, e = (h >> 10) & 0x1F, m = h & 0x3FF;
  float v;
  if (e == 0) v = std::ldexp((float)m, -24);
  else if (e == 31) v = m ? std::numeric_limits<float>::quiet_NaN()
                           : std::numeric_limits<float>::infinity();
  else v = std::ldexp(1.0f + (float)m / 1024.0f, e - 15);
  return s ? -v : v;
}

// Round a double to the 16-bit type (nearest, ties to even, overflow to inf).
uint16_t orc_double_to_half(double x, int dt);

}  // extern "C"

extern "C" {

// Round to nearest, ties to even, on a grid whose spacing is 2^(e-p) for a
// value in [2^(e-1), 2^e), floored at the subnormal spacing 2^qmin; then
// encode.  p = 11, qmin = -24 for fp16; p = 8, qmin = -133 for bfloat16.
uint16_t orc_double_to_half(double x, int dt) {
  const int p = dt == 1 ? 8 : 11;
  const int qmin = dt == 1 ? -133 : -24;
  const double maxv = dt == 1 ? std::ldexp(255.0 / 128.0, 127) : 65504.0;
  uint16_t sign = std::signbit(x) ? 0x8000 : 0;
  double a = std::fabs(x);
  double r;
  if (std::isnan(x)) return dt == 1 ? 0x7FC0 : 0x7E00;
  if (a == 0.0) {
    r = 0.0;
  } else {
    int e;
    std::frexp(a, &e);  // a in [2^(e-1), 2^e)
    int qe = std::max(e - p, qmin);
    double scaled = std::ldexp(a, -qe);  // exact
    r = std::ldexp(std::nearbyint(scaled), qe);
  }
  if (dt == 1) {
    if (r > maxv) return sign | 0x7F80;
    float f = (float)r;  // exact: r has at most 8 significant bits
    uint32_t u;
    std::memcpy(&u, &f, 4);
    return sign | (uint16_t)((u >> 16) & 0x7FFF);
  }
  if (r > maxv) return sign | 0x7C00;
  if (r == 0.0) return sign;
  int e;
  std::frexp(r, &e);
  if (e - 1 < -14) {  // subnormal: r = m * 2^-24
    return sign | (uint16_t)std::ldexp(r, 24);
  }
  int ef = e - 1;                              // r in [2^ef, 2^(ef+1))
  double mant = std::ldexp(r, -ef) - 1.0;      // in [0, 1)
  return sign | (uint16_t)(((ef + 15) << 10) | (int)std::ldexp(mant, 10));
}

// Unnormalised Sylvester-Hadamard transform of one row of length d (power of
// two) in fp32 (ScaleSearchAttention, "Procesamiento de Incoherencia";
// reading R5).  Butterfly stride h = 1, 2, ..., d/2; (a, b) -> (a+b, a-b) with
// a at the lower index.
void orc_fwht_row(float* x, int d) {
  for (int h = 1; h < d; h *= 2) {
    for (int i = 0; i < d; i += 2 * h) {
      for (int j = i; j < i + h; ++j) {
        float a = x[j], b = x[j + h];
        x[j] = a + b;
        x[j + h] = a - b;
      }
    }
  }
}

// Load a [rows, cols] 16-bit matrix as fp32, optionally rotating every row.
static std::vector<float> load_rows(const uint16_t* x, int dt, int64_t rows,
                                    int64_t cols, int hadamard) {
  std::vector<float> v((size_t)(rows * cols));
  for (int64_t i = 0; i < rows * cols; ++i) v[(size_t)i] = orc_half_to_float(x[i], dt);
  if (hadamard)
    for (int64_t r = 0; r < rows; ++r) orc_fwht_row(&v[(size_t)(r * cols)], (int)cols);
  return v;
}

// Per-tensor FP32 scale g = amax / 2688 over all values (reading R1).
static float tensor_scale_of(const std::vector<float>& v) {
  float amax = 0.0f;
  for (float f : v) amax = std::max(amax, std::fabs(f));
  if (amax == 0.0f) return 1.0f;
  return amax / 2688.0f;
}

float orc_tensor_scale(const uint16_t* x, int dt, int64_t rows, int64_t cols, int hadamard) {
  return tensor_scale_of(load_rows(x, dt, rows, cols, hadamard));
}

// max |x| over a [rows, cols] 16-bit matrix (rows rotated first when
// hadamard): the quantity g = amax / 2688 of reading R1 is taken from.
float orc_tensor_absmax(const uint16_t* x, int dt, int64_t rows, int64_t cols, int hadamard) {
  float amax = 0.0f;
  for (float f : load_rows(x, dt, rows, cols, hadamard)) amax = std::max(amax, std::fabs(f));
  return amax;
}

// ScaleSearch error of one candidate scale byte for a block of 16 values x
// under tensor scale g (reading R4): t = x * (1/(S g)), q = E2M1 grid value
// of t, err = (sum over the block, in order, of (t-q)^2 with fmaf) * S^2.
double orc_block_err(const float* x, float g, uint8_t S) {
  float dec = orc_ue4m3_decode(S) * g;
  float r = 1.0f / dec;
  float acc = 0.0f;
  for (int e = 0; e < 16; ++e) {
    float t = x[e] * r;
    float q = orc_e2m1_decode(orc_e2m1_encode(t));
    float er = t - q;
    acc = std::fmaf(er, er, acc);
  }
  double s = (double)orc_ue4m3_decode(S);
  return (double)acc * (s * s);
}

// Quantise one 16-element block (readings R3, R4).  Writes 8 packed bytes
// (element 2c in the low nibble, 2c+1 in the high nibble), the scale byte and
// the chosen offset f.
//
// Max scaling (ScaleSearch "Mecanismo"): the block absmax is mapped to the
// top FP4 value 6.  ScaleSearch ("Estrategia de Busqueda"): the candidate
// bytes S0+f for f in [-2, 6], reinterpreted as UE4M3, and the one with the
// smallest block error wins.
void orc_quant_block(const float* x, float g, int use_ss, uint8_t* codes8,
                     uint8_t* scale, int* f_out) {
  float amax = 0.0f;
  for (int e = 0; e < 16; ++e) amax = std::max(amax, std::fabs(x[e]));
  float s_real = amax / (6.0f * g);
  uint8_t S = orc_ue4m3_encode(s_real);
  int best_f = 0;
  if (use_ss && S != 0) {
    static const int order[9] = {0, -2, -1, 1, 2, 3, 4, 5, 6};
    double best = 0.0;
    bool have = false;
    for (int oi = 0; oi < 9; ++oi) {
      int b = (int)S + order[oi];
      if (b < 1 || b > 126) continue;
      double err = orc_block_err(x, g, (uint8_t)b);
      if (!have || err < best) {
        best = err;
        best_f = order[oi];
        have = true;
      }
    }
    S = (uint8_t)((int)S + best_f);
  }
  *scale = S;
  if (f_out) *f_out = best_f;
  uint8_t c[16];
  if (S == 0) {
    for (int e = 0; e < 16; ++e) c[e] = 0;
  } else {
    float dec = orc_ue4m3_decode(S) * g;
    float r = 1.0f / dec;
    for (int e = 0; e < 16; ++e) c[e] = orc_e2m1_encode(x[e] * r);
  }
  for (int i = 0; i < 8; ++i) codes8[i] = (uint8_t)(c[2 * i] | (c[2 * i + 1] << 4));
}

// Quantise a [rows, cols] matrix with 16-blocks along cols.
// codes [rows, cols/2], scales [rows, cols/16].  g is read when
// tensor_scale_given != 0, else computed and written.  f_out (optional)
// receives the chosen offsets [rows, cols/16].  Returns 0, or -1 on bad sizes.
int orc_nvfp4_quantize(const uint16_t* x, int dt, int64_t rows, int64_t cols,
                       int use_ss, int hadamard, int tensor_scale_given,
                       uint8_t* codes, uint8_t* scales, float* g, int8_t* f_out) {
  if (rows < 0 || cols <= 0 || cols % 16) return -1;
  if (hadamard && (cols & (cols - 1))) return -1;
  std::vector<float> v = load_rows(x, dt, rows, cols, hadamard);
  if (!tensor_scale_given) *g = tensor_scale_of(v);
  const float gg = *g;
  const int64_t nb = cols / 16;
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t b = 0; b < nb; ++b) {
      int f;
      orc_quant_block(&v[(size_t)(r * cols + b * 16)], gg, use_ss,
                      &codes[r * (cols / 2) + b * 8], &scales[r * nb + b], &f);
      if (f_out) f_out[r * nb + b] = (int8_t)f;
    }
  return 0;
}

// Same with 16-blocks along rows (the token axis of V): the matrix is read
// transposed.  codes [cols, rows/2], scales [cols, rows/16].
int orc_nvfp4_quantize_colblocks(const uint16_t* x, int dt, int64_t rows, int64_t cols,
                                 int use_ss, int tensor_scale_given,
                                 uint8_t* codes, uint8_t* scales, float* g, int8_t* f_out) {
  if (rows <= 0 || cols <= 0 || rows % 16) return -1;
  std::vector<float> v = load_rows(x, dt, rows, cols, 0);
  if (!tensor_scale_given) *g = tensor_scale_of(v);
  const float gg = *g;
  const int64_t nb = rows / 16;
  float blk[16];
  for (int64_t c = 0; c < cols; ++c)
    for (int64_t b = 0; b < nb; ++b) {
      for (int e = 0; e < 16; ++e) blk[e] = v[(size_t)((b * 16 + e) * cols + c)];
      int f;
      orc_quant_block(blk, gg, use_ss, &codes[c * (rows / 2) + b * 8], &scales[c * nb + b], &f);
      if (f_out) f_out[c * nb + b] = (int8_t)f;
    }
  return 0;
}

}  // extern "C"

extern "C" {

// ------------------------------------------------------ block selection --
//
// ThriftAttention, Metodologia step 1: the sequence is cut into blocks, each
// block pair (i, j) is scored by the dot product of the block-mean query and
// key vectors, and the top-k pairs are computed in FP16 (reading R8).

struct SeqView {
  int64_t start;  // first token of the sequence in the packed token axis
  int len;        // tokens
};

// Block means of one head of one sequence: x is [tokens, heads, d] packed,
// blocks of blk tokens from the sequence start (the last may be partial).
static void block_means(const uint16_t* x, int dt, int64_t tok_stride, int64_t head_off,
                        const SeqView& s, int d, int blk, std::vector<double>& out) {
  int nb = (s.len + blk - 1) / blk;
  out.assign((size_t)nb * d, 0.0);
  for (int b = 0; b < nb; ++b) {
    int t0 = b * blk, t1 = std::min(s.len, t0 + blk);
    for (int c = 0; c < d; ++c) {
      double sum = 0.0;
      for (int t = t0; t < t1; ++t)
        sum += (double)orc_half_to_float(x[(s.start + t) * tok_stride + head_off + c], dt);
      out[(size_t)b * d + c] = sum / (double)(t1 - t0);
    }
  }
}

static double pair_score(const double* qm, const double* km, int d) {
  double acc = 0.0;
  for (int c = 0; c < d; ++c) acc = std::fma(qm[c], km[c], acc);
  return acc;
}

int64_t orc_topk_count(float frac, int64_t n_valid) {
  double kk = std::ceil((double)frac * (double)n_valid - 1e-9);
  if (kk < 0) kk = 0;
  if (kk > (double)n_valid) kk = (double)n_valid;
  return (int64_t)kk;
}

// Selection for one (sequence, head): mask [nB, nB] (1 = FP16 pair).
// Sink-aware fixed pairs (ScaleSearchAttention, the sink-aware mixed-
// precision paragraph; reading R14): key block j is kept at full precision
// for query block i when j is one of the first `sink` blocks, or one of the
// `recent` most recent blocks i can see (causal: i - recent < j <= i;
// non-causal: the last `recent` blocks of the sequence).
static bool fixed_pair(int i, int j, int nb, int causal, int sink, int recent) {
  if (j < sink) return true;
  return causal ? (j > i - recent) : (j >= nb - recent);
}

static void select_one(const uint16_t* q, const uint16_t* k, int dt, int H, int Hkv,
                       int h, const SeqView& s, int d, int blk, int causal, float frac,
                       int sink, int recent, uint8_t* mask, double* scores) {
  int nb = (s.len + blk - 1) / blk;
  int hk = h / (H / Hkv);
  std::vector<double> qm, km;
  block_means(q, dt, (int64_t)H * d, (int64_t)h * d, s, d, blk, qm);
  block_means(k, dt, (int64_t)Hkv * d, (int64_t)hk * d, s, d, blk, km);
  std::vector<std::pair<double, int64_t>> cand;
  for (int i = 0; i < nb; ++i)
    for (int j = 0; j < nb; ++j) {
      int64_t lin = (int64_t)i * nb + j;
      mask[lin] = 0;
      double sc = pair_score(&qm[(size_t)i * d], &km[(size_t)j * d], d);
      if (scores) scores[lin] = sc;
      if (causal && j > i) continue;
      cand.push_back({sc, lin});
    }
  int64_t kk = orc_topk_count(frac, (int64_t)cand.size());
  // Full sort: larger score first, then lower linear index.
  std::sort(cand.begin(), cand.end(), [](const std::pair<double, int64_t>& a,
                                         const std::pair<double, int64_t>& b) {
    if (a.first != b.first) return a.first > b.first;
    return a.second < b.second;
  });
  for (int64_t t = 0; t < kk; ++t) mask[cand[(size_t)t].second] = 1;
  // the fixed pairs are added to the top-k ones (the quota is unchanged)
  for (int i = 0; i < nb; ++i)
    for (int j = 0; j < nb && (!causal || j <= i); ++j)
      if (fixed_pair(i, j, nb, causal, sink, recent)) mask[(int64_t)i * nb + j] = 1;
}

// q [B, N, H, d], k [B, N, Hkv, d] 16-bit; mask out uint8 [B, H, nB, nB];
// scores (optional) fp64 [B, H, nB, nB] (every pair, valid or not).
int orc_block_mean_topk(const uint16_t* q, const uint16_t* k, int dt, int B, int H, int Hkv,
                        int N, int d, int blk, int causal, float frac, int sink, int recent,
                        uint8_t* mask, double* scores) {
  if (B <= 0 || H <= 0 || Hkv <= 0 || H % Hkv || N <= 0 || d <= 0 || blk <= 0) return -1;
  if (sink < 0 || recent < 0) return -1;
  int nb = (N + blk - 1) / blk;
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < H; ++h) {
      SeqView s{0, N};
      int64_t off = ((int64_t)b * H + h) * nb * nb;
      select_one(q + (int64_t)b * N * H * d, k + (int64_t)b * N * Hkv * d, dt, H, Hkv, h, s, d,
                 blk, causal, frac, sink, recent, mask + off, scores ? scores + off : nullptr);
    }
  return 0;
}

// Varlen: q [total, H, d], k [total, Hkv, d]; cu_seqlens [nseq+1].  Masks of
// sequence s are stored at mask_off(s) = H * sum_{s'<s} nB_{s'}^2, laid out
// [H, nB_s, nB_s].
int orc_block_mean_topk_varlen(const uint16_t* q, const uint16_t* k, int dt, int H, int Hkv,
                               const int32_t* cu, int nseq, int d, int blk, int causal,
                               float frac, int sink, int recent, uint8_t* mask) {
  if (sink < 0 || recent < 0) return -1;
  int64_t off = 0;
  for (int sq = 0; sq < nseq; ++sq) {
    SeqView s{cu[sq], cu[sq + 1] - cu[sq]};
    int nb = (s.len + blk - 1) / blk;
    for (int h = 0; h < H; ++h) {
      select_one(q, k, dt, H, Hkv, h, s, d, blk, causal, frac, sink, recent, mask + off,
                 nullptr);
      off += (int64_t)nb * nb;
    }
  }
  return 0;
}

// ------------------------------------------------------------ threading --

static void parallel_for(int64_t n, int nthreads, const std::function<void(int64_t)>& fn) {
  if (nthreads <= 1 || n <= 1) {
    for (int64_t i = 0; i < n; ++i) fn(i);
    return;
  }
  std::atomic<int64_t> next(0);
  std::vector<std::thread> pool;
  int nt = (int)std::min<int64_t>(nthreads, n);
  for (int t = 0; t < nt; ++t)
    pool.emplace_back([&]() {
      for (;;) {
        int64_t i = next.fetch_add(1);
        if (i >= n) break;
        fn(i);
      }
    });
  for (auto& th : pool) th.join();
}

// Threaded quantiser of a [rows, cols] matrix (blocks along cols), writing
// one unpacked 4-bit code per byte and one scale byte per block, for the
// attention emulation below.  Same arithmetic as orc_nvfp4_quantize.
static float quantize_rows_unpacked(const uint16_t* x, int dt, int64_t rows, int cols,
                                    int use_ss, int hadamard, int nthreads,
                                    std::vector<uint8_t>& codes, std::vector<uint8_t>& scales,
                                    const float* g_given = nullptr) {
  const int64_t chunk = 4096;
  const int64_t nchunks = (rows + chunk - 1) / chunk;
  std::vector<float> part(nchunks, 0.0f);
  parallel_for(nchunks, nthreads, [&](int64_t c) {
    std::vector<float> row(cols);
    float amax = 0.0f;
    for (int64_t r = c * chunk; r < std::min(rows, (c + 1) * chunk); ++r) {
      for (int e = 0; e < cols; ++e) row[e] = orc_half_to_float(x[r * cols + e], dt);
      if (hadamard) orc_fwht_row(row.data(), cols);
      for (int e = 0; e < cols; ++e) amax = std::max(amax, std::fabs(row[e]));
    }
    part[c] = amax;
  });
  float amax = 0.0f;
  for (float a : part) amax = std::max(amax, a);
  const float g = g_given ? *g_given : (amax == 0.0f ? 1.0f : amax / 2688.0f);
  codes.assign((size_t)(rows * cols), 0);
  scales.assign((size_t)(rows * (cols / 16)), 0);
  parallel_for(nchunks, nthreads, [&](int64_t c) {
    std::vector<float> row(cols);
    uint8_t packed[8];
    for (int64_t r = c * chunk; r < std::min(rows, (c + 1) * chunk); ++r) {
      for (int e = 0; e < cols; ++e) row[e] = orc_half_to_float(x[r * cols + e], dt);
      if (hadamard) orc_fwht_row(row.data(), cols);
      for (int b = 0; b < cols / 16; ++b) {
        orc_quant_block(&row[b * 16], g, use_ss, packed, &scales[(size_t)(r * (cols / 16) + b)],
                        nullptr);
        for (int e = 0; e < 8; ++e) {
          codes[(size_t)(r * cols + b * 16 + 2 * e)] = packed[e] & 0xF;
          codes[(size_t)(r * cols + b * 16 + 2 * e + 1)] = packed[e] >> 4;
        }
      }
    }
  });
  return g;
}

// ------------------------------------------------- attention emulation --
//
// ThriftAttention, Metodologia step 2 and the kernel paragraph after it:
// for every query block, the key blocks that were not selected are visited
// first on the NVFP4 path, then the selected ones on the FP16 path, all
// merged by one FlashAttention-2 online softmax (base-2 exponent, running
// max m, running sum l).  NVFP4 products follow ScaleSearchAttention
// ("Ejecucion Nativa NVFP4": QK^T and PV on block-scaled FP4 values).
// Arithmetic here is fp64 on exactly dequantised values; the probability
// tile is rounded to fp32 before it is quantised (reading R7).

struct AttnCtx {
  int dt, H, Hkv, d, blk, causal, use_had, smooth_k = 0;
  std::vector<float> mu;  // K channel means [nseq, Hkv, d] (reading R16)
  const int32_t* cu;
  int nseq;
  int64_t total, ptot;
  const uint16_t *q, *k, *v;
  std::vector<uint8_t> qc, qs, kc, ks, vc, vs;  // unpacked codes, scale bytes
  float gq, gk, gv;
  std::vector<int64_t> pstart;   // padded token start of each sequence (V)
  std::vector<int64_t> moff;     // mask offset of each sequence
  const uint8_t* mask;
};

static inline double deq(uint8_t code, uint8_t sc, float g) {
  return (double)orc_e2m1_decode(code) * (double)orc_ue4m3_decode(sc) * (double)g;
}

// ------------------------------------------ roundings that are not unique --
//
// The GPU evaluates the quantities of this emulation in another order: scores
// by fp32 accumulation in the tensor cores, the exponent argument of each
// probability in fp32, exp2 and log2 by the hardware approximations.  A
// probability whose E2M1 code, UE4M3 block scale or 16-bit value lies within
// that arithmetic's error of a rounding midpoint may round to either side,
// and both results are correct evaluations of the method.  The emulation
// reports, per output element, a bound `tol` on how far such roundings can
// move it.  The radius (relative) within which a rounding counts as not
// unique is taken per row and key tile from the error bounds of that
// arithmetic, in log2 units of the exponent argument:
//   * each score and the maximum it is taken against come from an fp32
//     accumulation of d exact products with at most one ulp of error per
//     addition: 2 d 2^-23 A, A = the tile's largest sum over channels of
//     |q_c k_c| (softmax scale included);
//   * the fp32 roundings of the scale product, the maximum, the constant part
//     of the argument (log2 2688 - log2 S_b, the log2 approximation adding at
//     most 2^-22 per unit of its result) and the fused argument itself:
//     2^-22 (|S|max + |m| + 24), 24 bounding |log2 2688| + |log2 S_b| <= 20.4;
// plus, relative, the exp2 approximation (2 ulp, 2^-22) and this emulation's
// own fp32 chain (P, 1/rowmax, P/rowmax, 1/S_b, t: five roundings of 2^-24):
//   rho = ln 2 (2 d 2^-23 A + 2^-22 (|S|max + |m| + 24)) + 2^-22 + 5 2^-24.
static double tile_radius(int d, double A, double smax_abs, double m_abs) {
  const double u23 = std::ldexp(1.0, -23), u22 = std::ldexp(1.0, -22);
  const double dx = 2.0 * d * u23 * A + u22 * (smax_abs + m_abs + 24.0);
  return 0.6931471805599453 * dx + u22 + 5.0 * std::ldexp(1.0, -24);
}

// Every rounding below is monotone, so the roundings a value x can take
// when it is changed by a factor in [1 - rho, 1 + rho] lie between the
// roundings of the two ends of that interval.  The ends carry 2^-23 of
// margin for the fp32 rounding of a changed value.
static double widen(double rho) { return rho + std::ldexp(1.0, -23); }

// E2M1 value of t (round to nearest even, saturating).
static double e2m1_val(double t) { return (double)orc_e2m1_decode(orc_e2m1_encode((float)t)); }

// How far the E2M1 value of t can move under a change of t within rho.
static double e2m1_reach(float t, double rho) {
  const double r = widen(rho), q0 = e2m1_val(t);
  return std::max(std::fabs(e2m1_val((double)t * (1.0 + r)) - q0),
                  std::fabs(e2m1_val((double)t * (1.0 - r)) - q0));
}

// How far the 16-bit rounding of x can move under a change of x within rho.
static double half_reach(double x, int dt, double rho) {
  const double r = widen(rho);
  const double q0 = orc_half_to_float(orc_double_to_half(x, dt), dt);
  const double qh = orc_half_to_float(orc_double_to_half(x * (1.0 + r), dt), dt);
  const double ql = orc_half_to_float(orc_double_to_half(x * (1.0 - r), dt), dt);
  return std::max(std::fabs(qh - q0), std::fabs(ql - q0));
}

// Test hooks (pins of `tol` only; off unless set by orc_set_test_hooks).
//   pert: every rounding input of the probabilities -- the scaled P whose
//     E2M1 code is taken, the block-scale argument, the P rounded to 16 bits
//     -- is multiplied by 1 + pert * rho * u, u in [-1, 1) a hash of (seed,
//     sequence, head, row, key, kind); with |pert| <= 1 only roundings within
//     the radius can change.
//   plant: on the NVFP4 path of one (sequence, head, row, key) the scaled
//     probability t takes the value plant_t, and its E2M1 code then moves
//     `force` grid steps (+1 up, -1 down, 0 none).
struct OrcHooks {
  double pert = 0.0;
  uint64_t seed = 0;
  int s = -1, h = -1, row = -1, key = -1;
  float plant_t = 0.0f;
  int force = 0;
};
static OrcHooks g_hooks;

void orc_set_test_hooks(double pert, uint64_t seed, int s, int h, int row, int key,
                        float plant_t, int force) {
  g_hooks.pert = pert;
  g_hooks.seed = seed;
  g_hooks.s = s;
  g_hooks.h = h;
  g_hooks.row = row;
  g_hooks.key = key;
  g_hooks.plant_t = plant_t;
  g_hooks.force = force;
}

// splitmix64 finaliser of the hooks' hash.
static uint64_t mix64(uint64_t z) {
  z += 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// fp32 x * (1 + pert * rho * u) for the hooks' perturbation (x when off).
static float hook_perturb(float x, double rho, int s, int h, int row, int key, int kind) {
  if (g_hooks.pert == 0.0) return x;
  uint64_t z = mix64(g_hooks.seed ^ ((uint64_t)(uint32_t)s << 40));
  z = mix64(z ^ ((uint64_t)(uint32_t)h << 20) ^ (uint64_t)(uint32_t)row);
  z = mix64(z ^ ((uint64_t)(uint32_t)key << 8) ^ (uint64_t)kind);
  const double u = (double)(z >> 11) * std::ldexp(1.0, -52) - 1.0;
  return (float)((double)x * (1.0 + g_hooks.pert * rho * u));
}

static bool hook_planted(int s, int h, int row, int key) {
  return s == g_hooks.s && h == g_hooks.h && row == g_hooks.row && key == g_hooks.key;
}

// Two-level quantisation of one row's probability tile (reading R7): Pt[t],
// t < nk, the fp32 probabilities relative to the running max; returns
// sigma = rowmax / 2688 (0 when the row has no live key: the tile adds
// nothing) and, for t < nk, Pq[t] = the value of P^ (E2M1 value times UE4M3
// block scale; the tile adds sigma * sum_t Pq[t] v[t]) and dq[t] = how far a
// rounding that is not unique within radius rho can move Pq[t].
// (s, h, row, key0) locate the tile for the test hooks.
static float p_tile_fp4(const float* Pt, int nk, int blk, double rho, int s, int h, int row,
                        int key0, double* Pq, double* dq) {
  float rowmax = 0.0f;
  for (int t = 0; t < nk; ++t) rowmax = std::max(rowmax, Pt[t]);
  if (rowmax == 0.0f) return 0.0f;
  const float inv = 2688.0f / rowmax;
  const float sigma = rowmax / 2688.0f;
  std::vector<float> Ph(blk);
  for (int t = 0; t < blk; ++t) Ph[t] = t < nk ? Pt[t] * inv : 0.0f;
  for (int b0 = 0; b0 < blk && b0 < nk; b0 += 16) {
    const int ne = std::min(16, nk - b0);
    float amax = 0.0f;
    for (int e = 0; e < 16; ++e) amax = std::max(amax, Ph[b0 + e]);
    const float s_real = hook_perturb(amax / 6.0f, rho, s, h, row, key0 + b0, 1);
    const uint8_t sp = orc_ue4m3_encode(s_real);
    const float dec = orc_ue4m3_decode(sp);
    const float rr = 1.0f / dec;
    for (int e = 0; e < ne; ++e) {
      const int key = key0 + b0 + e;
      float tq = Ph[b0 + e] * rr;
      const bool planted = hook_planted(s, h, row, key);
      if (planted) tq = g_hooks.plant_t;
      tq = hook_perturb(tq, rho, s, h, row, key, 0);
      uint8_t code = orc_e2m1_encode(tq);
      if (planted && g_hooks.force != 0) {
        const int mag = std::min(7, std::max(0, (int)(code & 7) + g_hooks.force));
        code = (uint8_t)((code & 8) | mag);
      }
      Pq[b0 + e] = sp == 0 ? 0.0 : (double)orc_e2m1_decode(code) * (double)dec;
      dq[b0 + e] = sp == 0 ? 0.0 : e2m1_reach(tq, rho) * (double)dec;
    }
    // block-scale bytes the scale argument can round to within the radius:
    // under each other byte, the block's codes (each within the radius too)
    const double rw = widen(rho);
    const int lo_b = orc_ue4m3_encode((float)((double)s_real * (1.0 - rw)));
    const int hi_b = orc_ue4m3_encode((float)((double)s_real * (1.0 + rw)));
    for (int alt = lo_b; alt <= hi_b; ++alt) {
      if (alt == (int)sp) continue;
      const float dec2 = orc_ue4m3_decode((uint8_t)alt);
      const float rr2 = alt == 0 ? 0.0f : 1.0f / dec2;
      for (int e = 0; e < ne; ++e) {
        const float t2 = Ph[b0 + e] * rr2;
        const double q2 = alt == 0 ? 0.0 : e2m1_val(t2) * (double)dec2;
        const double r2 = alt == 0 ? 0.0 : e2m1_reach(t2, rho) * (double)dec2;
        dq[b0 + e] = std::max(dq[b0 + e], std::fabs(q2 - Pq[b0 + e]) + r2);
      }
    }
  }
  return sigma;
}

// FP16 path of one row's tile (reading R9): P16[t] = Pt[t] rounded to the
// input type, dq[t] = how far that rounding can move under a change of Pt[t]
// within radius rho.
static void p_tile_16(const float* Pt, int nk, int dt, double rho, int s, int h, int row,
                      int key0, double* P16, double* dq) {
  for (int t = 0; t < nk; ++t) {
    const float x = hook_perturb(Pt[t], rho, s, h, row, key0 + t, 2);
    P16[t] = (double)orc_half_to_float(orc_double_to_half((double)x, dt), dt);
    dq[t] = half_reach((double)x, dt, rho);
  }
}

// One query block i of sequence s, head h.  Writes out rows and lse.
static void attn_unit(const AttnCtx& C, int s, int h, int i, uint16_t* out, float* lse,
                      double* out64, double* tol) {
  const int d = C.d, blk = C.blk, H = C.H, Hkv = C.Hkv;
  const int64_t st = C.cu[s];
  const int len = C.cu[s + 1] - C.cu[s];
  const int nb = (len + blk - 1) / blk;
  const int hk = h / (H / Hkv);
  const int r0 = i * blk, r1 = std::min(len, r0 + blk), nr = r1 - r0;
  const double l2e = 1.4426950408889634;  // log2(e)
  double s4 = l2e / std::sqrt((double)d);
  if (C.use_had) s4 /= (double)d;
  const double s16 = l2e / std::sqrt((double)d);
  const uint8_t* mk = C.mask + C.moff[s] + (int64_t)h * nb * nb + (int64_t)i * nb;

  std::vector<int> order;
  for (int pass = 0; pass < 2; ++pass)
    for (int j = 0; j < nb; ++j) {
      if (C.causal && j > i) continue;
      if ((mk[j] != 0) == (pass == 1)) order.push_back(pass == 0 ? j : -1 - j);
    }

  // Per-row query vectors: dequantised NVFP4 and the original 16-bit values.
  std::vector<double> qh((size_t)nr * d), q16((size_t)nr * d);
  for (int r = 0; r < nr; ++r)
    for (int c = 0; c < d; ++c) {
      int64_t e = ((st + r0 + r) * H + h) * d + c;
      qh[(size_t)r * d + c] = deq(C.qc[(size_t)e], C.qs[(size_t)(e / 16)], C.gq);
      q16[(size_t)r * d + c] = orc_half_to_float(C.q[e], C.dt);
    }
  std::vector<double> m(nr, -INFINITY), l(nr, 0.0), O((size_t)nr * d, 0.0);
  // amb: bound on how far the non-unique roundings can move O (before / l)
  std::vector<double> amb((size_t)nr * d, 0.0);
  // arun: the largest sum of |q_c k_c| of the row so far (error of its max)
  std::vector<double> arun(nr, 0.0);
  std::vector<double> dq(blk);
  std::vector<double> kt((size_t)blk * d), vt((size_t)blk * d), S(blk);
  std::vector<float> Pt(blk);
  std::vector<double> Pq(blk);

  for (int code : order) {
    const bool fp4 = code >= 0;
    const int j = fp4 ? code : -1 - code;
    const int k0 = j * blk, k1 = std::min(len, k0 + blk), nk = k1 - k0;
    for (int t = 0; t < nk; ++t)
      for (int c = 0; c < d; ++c) {
        int64_t e = ((st + k0 + t) * Hkv + hk) * d + c;
        if (fp4) {
          kt[(size_t)t * d + c] = deq(C.kc[(size_t)e], C.ks[(size_t)(e / 16)], C.gk);
          if (C.smooth_k) kt[(size_t)t * d + c] += (double)C.mu[((size_t)s * Hkv + hk) * d + c];
          int64_t ve = ((int64_t)hk * d + c) * C.ptot + C.pstart[s] + k0 + t;
          vt[(size_t)t * d + c] = deq(C.vc[(size_t)ve], C.vs[(size_t)(ve / 16)], C.gv);
        } else {
          kt[(size_t)t * d + c] = orc_half_to_float(C.k[e], C.dt);
          vt[(size_t)t * d + c] = orc_half_to_float(C.v[e], C.dt);
        }
      }
    for (int r = 0; r < nr; ++r) {
      const int row = r0 + r;
      const double* qv = fp4 ? &qh[(size_t)r * d] : &q16[(size_t)r * d];
      double mt = -INFINITY, amx = 0.0, smx = 0.0;
      for (int t = 0; t < nk; ++t) {
        if (C.causal && k0 + t > row) {
          S[t] = -INFINITY;
          continue;
        }
        double acc = 0.0, aabs = 0.0;
        for (int c = 0; c < d; ++c) {
          acc += qv[c] * kt[(size_t)t * d + c];
          aabs += std::fabs(qv[c] * kt[(size_t)t * d + c]);
        }
        S[t] = acc * (fp4 ? s4 : s16);
        mt = std::max(mt, S[t]);
        amx = std::max(amx, aabs * (fp4 ? s4 : s16));
        smx = std::max(smx, std::fabs(S[t]));
      }
      if (mt == -INFINITY) continue;
      const double mn = std::max(m[r], mt);
      const double alpha = std::exp2(m[r] - mn);  // 0 when m is still -inf
      arun[r] = std::max(arun[r], amx);
      l[r] *= alpha;
      for (int c = 0; c < d; ++c) {
        O[(size_t)r * d + c] *= alpha;
        amb[(size_t)r * d + c] *= alpha;
      }
      for (int t = 0; t < nk; ++t) {
        Pt[t] = S[t] == -INFINITY ? 0.0f : (float)std::exp2(S[t] - mn);
        l[r] += (double)Pt[t];
      }
      if (fp4) {
        // Two-level quantisation of the probability row tile (reading R7),
        // each row's P taken relative to the tile maximum on the GPU.
        const double rho = tile_radius(d, amx, smx, std::fabs(mt));
        const float sigma = p_tile_fp4(Pt.data(), nk, blk, rho, s, h, row, k0, Pq.data(),
                                       dq.data());
        if (sigma == 0.0f) { m[r] = mn; continue; }
        for (int c = 0; c < d; ++c) {
          double acc = 0.0, ab = 0.0;
          for (int t = 0; t < nk; ++t) {
            acc += Pq[t] * vt[(size_t)t * d + c];
            ab += dq[t] * std::fabs(vt[(size_t)t * d + c]);
          }
          O[(size_t)r * d + c] += (double)sigma * acc;
          amb[(size_t)r * d + c] += (double)sigma * ab;
        }
      } else {
        // FP16 path: P taken against the running max on the GPU
        const double rho = tile_radius(d, arun[r], smx, std::fabs(mn));
        p_tile_16(Pt.data(), nk, C.dt, rho, s, h, row, k0, Pq.data(), dq.data());
        for (int c = 0; c < d; ++c) {
          double acc = 0.0, ab = 0.0;
          for (int t = 0; t < nk; ++t) {
            acc += Pq[t] * vt[(size_t)t * d + c];
            ab += dq[t] * std::fabs(vt[(size_t)t * d + c]);
          }
          O[(size_t)r * d + c] += acc;
          amb[(size_t)r * d + c] += ab;
        }
      }
      m[r] = mn;
    }
  }
  const double ln2 = 0.6931471805599453;
  for (int r = 0; r < nr; ++r) {
    const int64_t tok = st + r0 + r;
    for (int c = 0; c < d; ++c) {
      double o = l[r] > 0.0 ? O[(size_t)r * d + c] / l[r] : 0.0;
      out[(tok * H + h) * d + c] = orc_double_to_half(o, C.dt);
      if (out64) out64[(tok * H + h) * d + c] = o;
      if (tol) tol[(tok * H + h) * d + c] = l[r] > 0.0 ? amb[(size_t)r * d + c] / l[r] : 0.0;
    }
    lse[(int64_t)h * C.total + tok] = l[r] > 0.0 ? (float)(m[r] * ln2 + std::log(l[r])) : -INFINITY;
  }
}

// Full emulation over packed sequences.  q [total, H, d], k/v [total, Hkv, d]
// 16-bit; cu [nseq+1].  out 16-bit [total, H, d]; lse fp32 [H, total].
// mask_io: if mask_given, the selection [per sequence: H, nB, nB] is read from
// it, else it is computed (reading R8) and written there.  units: optional
// list of (sequence, head, query block) triples to compute (n_units = 0 means
// every unit); rows of other units are left untouched.  gs_out (optional)
// receives g_Q, g_K, g_V.  out64 (optional) receives the fp64 output before
// its final rounding to the 16-bit type.  tol (optional) receives, per output
// element, a bound on how far roundings that are not unique can move it: a
// probability whose E2M1 code, UE4M3 block scale or 16-bit value lies within
// the radius of tile_radius() of a rounding midpoint may take either side in
// an implementation that evaluates the same arithmetic in another order.

// Quantiser of a [rows, cols] fp32 matrix (unpacked codes), tensor scale
// amax/2688 over the whole matrix: the same arithmetic as
// quantize_rows_unpacked on values that are not 16-bit.
static float quantize_rows_f32(const float* x, int64_t rows, int cols, int use_ss, int nthreads,
                               std::vector<uint8_t>& codes, std::vector<uint8_t>& scales,
                               const float* g_given = nullptr) {
  float amax = 0.0f;
  for (int64_t e = 0; e < rows * cols; ++e) amax = std::max(amax, std::fabs(x[e]));
  const float g = g_given ? *g_given : (amax == 0.0f ? 1.0f : amax / 2688.0f);
  codes.assign((size_t)(rows * cols), 0);
  scales.assign((size_t)(rows * (cols / 16)), 0);
  parallel_for((rows + 4095) / 4096, nthreads, [&](int64_t ch) {
    uint8_t packed[8];
    for (int64_t r = ch * 4096; r < std::min(rows, (ch + 1) * 4096); ++r)
      for (int b = 0; b < cols / 16; ++b) {
        orc_quant_block(&x[r * cols + b * 16], g, use_ss, packed,
                        &scales[(size_t)(r * (cols / 16) + b)], nullptr);
        for (int e = 0; e < 8; ++e) {
          codes[(size_t)(r * cols + b * 16 + 2 * e)] = packed[e] & 0xF;
          codes[(size_t)(r * cols + b * 16 + 2 * e + 1)] = packed[e] >> 4;
        }
      }
  });
  return g;
}

// K channel means of reading R16: [nseq, Hkv, d] fp32.
void orc_k_channel_means(const uint16_t* k, int dt, int Hkv, const int32_t* cu, int nseq, int d,
                         float* mu) {
  for (int s = 0; s < nseq; ++s) {
    const int64_t st = cu[s];
    const int len = cu[s + 1] - cu[s];
    for (int hk = 0; hk < Hkv; ++hk)
      for (int c = 0; c < d; ++c) {
        double total = 0.0;
        for (int b0 = 0; b0 < len; b0 += 128) {
          double sum = 0.0;
          for (int t = b0; t < std::min(len, b0 + 128); ++t)
            sum += (double)orc_half_to_float(k[((st + t) * Hkv + hk) * d + c], dt);
          total += sum;
        }
        mu[((size_t)s * Hkv + hk) * d + c] = len > 0 ? (float)(total / (double)len) : 0.0f;
      }
  }
}

int orc_thrift_attn_ex(const uint16_t* q, const uint16_t* k, const uint16_t* v, int dt, int H,
                       int Hkv, const int32_t* cu, int nseq, int d, int blk, int causal,
                       float frac, int sink, int recent, int use_ss, int use_had, int smooth_k,
                       uint8_t* mask_io, int mask_given,
                       const int32_t* units, int64_t n_units, int nthreads, uint16_t* out,
                       float* lse, float* gs_out, double* out64, double* tol);

int orc_thrift_attn(const uint16_t* q, const uint16_t* k, const uint16_t* v, int dt, int H,
                    int Hkv, const int32_t* cu, int nseq, int d, int blk, int causal,
                    float frac, int sink, int recent, int use_ss, int use_had,
                    uint8_t* mask_io, int mask_given,
                    const int32_t* units, int64_t n_units, int nthreads, uint16_t* out,
                    float* lse, float* gs_out, double* out64, double* tol) {
  return orc_thrift_attn_ex(q, k, v, dt, H, Hkv, cu, nseq, d, blk, causal, frac, sink, recent,
                            use_ss, use_had, 0, mask_io, mask_given, units, n_units, nthreads,
                            out, lse, gs_out, out64, tol);
}

int orc_thrift_attn_g(const uint16_t* q, const uint16_t* k, const uint16_t* v, int dt, int H,
                      int Hkv, const int32_t* cu, int nseq, int d, int blk, int causal,
                      float frac, int sink, int recent, int use_ss, int use_had, int smooth_k,
                      const float* g_in, uint8_t* mask_io, int mask_given,
                      const int32_t* units, int64_t n_units, int nthreads, uint16_t* out,
                      float* lse, float* gs_out, double* out64, double* tol);

// As orc_thrift_attn, with optional K smoothing (reading R16).
int orc_thrift_attn_ex(const uint16_t* q, const uint16_t* k, const uint16_t* v, int dt, int H,
                       int Hkv, const int32_t* cu, int nseq, int d, int blk, int causal,
                       float frac, int sink, int recent, int use_ss, int use_had, int smooth_k,
                       uint8_t* mask_io, int mask_given,
                       const int32_t* units, int64_t n_units, int nthreads, uint16_t* out,
                       float* lse, float* gs_out, double* out64, double* tol) {
  return orc_thrift_attn_g(q, k, v, dt, H, Hkv, cu, nseq, d, blk, causal, frac, sink, recent,
                           use_ss, use_had, smooth_k, nullptr, mask_io, mask_given, units,
                           n_units, nthreads, out, lse, gs_out, out64, tol);
}

// As orc_thrift_attn_ex, with the tensor scales g_Q, g_K, g_V given (g_in,
// 3 floats; NULL: computed from the tensors, reading R1): a shard of a larger
// problem quantised under that problem's scales.
int orc_thrift_attn_g(const uint16_t* q, const uint16_t* k, const uint16_t* v, int dt, int H,
                      int Hkv, const int32_t* cu, int nseq, int d, int blk, int causal,
                      float frac, int sink, int recent, int use_ss, int use_had, int smooth_k,
                      const float* g_in, uint8_t* mask_io, int mask_given,
                      const int32_t* units, int64_t n_units, int nthreads, uint16_t* out,
                      float* lse, float* gs_out, double* out64, double* tol) {
  if (H <= 0 || Hkv <= 0 || H % Hkv || nseq <= 0 || d % 16 || blk % 16 || blk <= 0) return -1;
  if (use_had && (d & (d - 1))) return -1;
  if (smooth_k && use_had) return -1;
  AttnCtx C;
  C.dt = dt; C.H = H; C.Hkv = Hkv; C.d = d; C.blk = blk; C.causal = causal; C.use_had = use_had;
  C.smooth_k = smooth_k;
  C.cu = cu; C.nseq = nseq; C.q = q; C.k = k; C.v = v;
  C.total = cu[nseq];
  C.pstart.resize(nseq + 1);
  C.moff.resize(nseq + 1);
  C.pstart[0] = 0;
  C.moff[0] = 0;
  for (int s = 0; s < nseq; ++s) {
    int len = cu[s + 1] - cu[s];
    if (len <= 0) return -1;
    int nb = (len + blk - 1) / blk;
    C.pstart[s + 1] = C.pstart[s] + (int64_t)nb * blk;
    C.moff[s + 1] = C.moff[s] + (int64_t)H * nb * nb;
  }
  C.ptot = C.pstart[nseq];
  C.gq = quantize_rows_unpacked(q, dt, C.total * H, d, use_ss, use_had, nthreads, C.qc, C.qs,
                                g_in ? &g_in[0] : nullptr);
  if (smooth_k) {
    C.mu.assign((size_t)nseq * Hkv * d, 0.0f);
    orc_k_channel_means(k, dt, Hkv, cu, nseq, d, C.mu.data());
    std::vector<float> ks((size_t)(C.total * Hkv * d));
    for (int s2 = 0; s2 < nseq; ++s2)
      for (int64_t t = cu[s2]; t < cu[s2 + 1]; ++t)
        for (int hk = 0; hk < Hkv; ++hk)
          for (int c = 0; c < d; ++c) {
            const int64_t e = (t * Hkv + hk) * d + c;
            ks[(size_t)e] = orc_half_to_float(k[e], dt) - C.mu[((size_t)s2 * Hkv + hk) * d + c];
          }
    C.gk = quantize_rows_f32(ks.data(), C.total * Hkv, d, use_ss, nthreads, C.kc, C.ks,
                             g_in ? &g_in[1] : nullptr);
  } else {
    C.gk = quantize_rows_unpacked(k, dt, C.total * Hkv, d, use_ss, use_had, nthreads, C.kc, C.ks,
                                  g_in ? &g_in[1] : nullptr);
  }
  // V: 16-blocks along tokens, every sequence zero-padded to a whole number of
  // key blocks (reading R6).  The tensor scale covers the real tokens only.
  {
    float amax = 0.0f;
    for (int64_t e = 0; e < C.total * Hkv * d; ++e) amax = std::max(amax, std::fabs(orc_half_to_float(v[e], dt)));
    C.gv = g_in ? g_in[2] : (amax == 0.0f ? 1.0f : amax / 2688.0f);
    C.vc.assign((size_t)(Hkv * d * C.ptot), 0);
    C.vs.assign((size_t)(Hkv * d * C.ptot / 16), 0);
    parallel_for((int64_t)Hkv * d, nthreads, [&](int64_t hc) {
      const int64_t hk = hc / d, c = hc % d;
      float col[16];
      uint8_t packed[8];
      for (int s = 0; s < nseq; ++s) {
        const int len = cu[s + 1] - cu[s];
        for (int64_t t0 = 0; t0 < C.pstart[s + 1] - C.pstart[s]; t0 += 16) {
          for (int e = 0; e < 16; ++e)
            col[e] = t0 + e < len ? orc_half_to_float(v[((cu[s] + t0 + e) * Hkv + hk) * d + c], dt) : 0.0f;
          const int64_t base = hc * C.ptot + C.pstart[s] + t0;
          orc_quant_block(col, C.gv, use_ss, packed, &C.vs[(size_t)(base / 16)], nullptr);
          for (int e = 0; e < 8; ++e) {
            C.vc[(size_t)(base + 2 * e)] = packed[e] & 0xF;
            C.vc[(size_t)(base + 2 * e + 1)] = packed[e] >> 4;
          }
        }
      }
    });
  }
  if (gs_out) { gs_out[0] = C.gq; gs_out[1] = C.gk; gs_out[2] = C.gv; }
  if (!mask_given)
    orc_block_mean_topk_varlen(q, k, dt, H, Hkv, cu, nseq, d, blk, causal, frac, sink, recent,
                               mask_io);
  C.mask = mask_io;
  std::vector<int32_t> all;
  if (n_units == 0) {
    for (int s = 0; s < nseq; ++s) {
      int nb = (cu[s + 1] - cu[s] + blk - 1) / blk;
      for (int h = 0; h < H; ++h)
        for (int i = 0; i < nb; ++i) { all.push_back(s); all.push_back(h); all.push_back(i); }
    }
    units = all.data();
    n_units = (int64_t)all.size() / 3;
  }
  parallel_for(n_units, nthreads, [&](int64_t u) {
    attn_unit(C, units[3 * u], units[3 * u + 1], units[3 * u + 2], out, lse, out64, tol);
  });
  return 0;
}

// ------------------------------------------------------------- decode --
//
// Reading R15.  q [B, H, d]; k, v [B, ncap, Hkv, d] 16-bit (token t of
// sequence b at row b * ncap + t); lens [B] cached tokens (0 <= len <= ncap).

// Rows of a [rows, cols] 16-bit matrix quantised under a given tensor scale,
// one unpacked 4-bit code per byte (same arithmetic as orc_nvfp4_quantize with
// the scale given).
static void quantize_rows_given(const uint16_t* x, int dt, int64_t rows, int cols, float g,
                                int use_ss, int nthreads, std::vector<uint8_t>& codes,
                                std::vector<uint8_t>& scales) {
  const int64_t chunk = 4096;
  const int64_t nchunks = (rows + chunk - 1) / chunk;
  codes.assign((size_t)(rows * cols), 0);
  scales.assign((size_t)(rows * (cols / 16)), 0);
  parallel_for(nchunks, nthreads, [&](int64_t c) {
    std::vector<float> row(cols);
    uint8_t packed[8];
    for (int64_t r = c * chunk; r < std::min(rows, (c + 1) * chunk); ++r) {
      for (int e = 0; e < cols; ++e) row[e] = orc_half_to_float(x[r * cols + e], dt);
      for (int b = 0; b < cols / 16; ++b) {
        orc_quant_block(&row[b * 16], g, use_ss, packed, &scales[(size_t)(r * (cols / 16) + b)],
                        nullptr);
        for (int e = 0; e < 8; ++e) {
          codes[(size_t)(r * cols + b * 16 + 2 * e)] = packed[e] & 0xF;
          codes[(size_t)(r * cols + b * 16 + 2 * e + 1)] = packed[e] >> 4;
        }
      }
    }
  });
}

// Selection of one (sequence, head) at decode (reading R15): mask [nbcap],
// 1 = FP16 key block; entries past the sequence are 0.
static void decode_select_one(const uint16_t* q, const uint16_t* k, int dt, int H, int Hkv,
                              int ncap, int d, int blk, int b, int h, int len, float frac,
                              int sink, int recent, uint8_t* mask, int nbcap) {
  const int nb = (len + blk - 1) / blk;
  const int hk = h / (H / Hkv);
  for (int j = 0; j < nbcap; ++j) mask[j] = 0;
  if (nb == 0) return;
  std::vector<double> qm(d), km(d);
  for (int c = 0; c < d; ++c) qm[c] = (double)orc_half_to_float(q[((int64_t)b * H + h) * d + c], dt);
  std::vector<std::pair<double, int64_t>> cand;
  for (int j = 0; j < nb; ++j) {
    const int t0 = j * blk, t1 = std::min(len, t0 + blk);
    for (int c = 0; c < d; ++c) {
      double sum = 0.0;
      for (int t = t0; t < t1; ++t)
        sum += (double)orc_half_to_float(k[(((int64_t)b * ncap + t) * Hkv + hk) * d + c], dt);
      km[c] = sum / (double)(t1 - t0);
    }
    cand.push_back({pair_score(qm.data(), km.data(), d), j});
  }
  const int64_t kk = orc_topk_count(frac, nb);
  std::sort(cand.begin(), cand.end(), [](const std::pair<double, int64_t>& a,
                                         const std::pair<double, int64_t>& bb) {
    if (a.first != bb.first) return a.first > bb.first;
    return a.second < bb.second;
  });
  for (int64_t t = 0; t < kk; ++t) mask[cand[(size_t)t].second] = 1;
  for (int j = 0; j < nb; ++j)
    if (j < sink || j >= nb - recent) mask[j] = 1;
}

struct DecCtx {
  int dt, B, H, Hkv, ncap, d, blk, nbcap;
  const int32_t* lens;
  const uint16_t *q, *k, *v;
  std::vector<uint8_t> qc, qs, kc, ks, vc, vs;  // unpacked codes, scale bytes
  float gq, gk, gv;
  const uint8_t* mask;  // [B, H, nbcap]
};

// One query row (sequence b, head h): the steps of attn_unit for a single,
// non-causal row over the cached tokens.
static void decode_row(const DecCtx& C, int b, int h, uint16_t* out, float* lse, double* out64,
                       double* tol) {
  const int d = C.d, blk = C.blk, H = C.H, Hkv = C.Hkv;
  const int len = C.lens[b];
  const int nb = (len + blk - 1) / blk;
  const int hk = h / (H / Hkv);
  const int64_t orow = ((int64_t)b * H + h) * d;
  const double l2e = 1.4426950408889634;
  const double s4 = l2e / std::sqrt((double)d), s16 = s4;
  const uint8_t* mk = C.mask + ((int64_t)b * H + h) * C.nbcap;
  std::vector<int> order;
  for (int pass = 0; pass < 2; ++pass)
    for (int j = 0; j < nb; ++j)
      if ((mk[j] != 0) == (pass == 1)) order.push_back(pass == 0 ? j : -1 - j);
  std::vector<double> qh(d), q16(d);
  for (int c = 0; c < d; ++c) {
    qh[c] = deq(C.qc[(size_t)(orow + c)], C.qs[(size_t)((orow + c) / 16)], C.gq);
    q16[c] = orc_half_to_float(C.q[orow + c], C.dt);
  }
  double m = -INFINITY, l = 0.0, arun = 0.0;
  std::vector<double> O(d, 0.0), amb(d, 0.0), dq(blk), kt((size_t)blk * d), vt((size_t)blk * d),
      S(blk), Pq(blk);
  std::vector<float> Pt(blk);
  const int64_t vcol = C.nbcap * (int64_t)blk;  // padded tokens per V column
  for (int code : order) {
    const bool fp4 = code >= 0;
    const int j = fp4 ? code : -1 - code;
    const int k0 = j * blk, k1 = std::min(len, k0 + blk), nk = k1 - k0;
    for (int t = 0; t < nk; ++t)
      for (int c = 0; c < d; ++c) {
        const int64_t e = (((int64_t)b * C.ncap + k0 + t) * Hkv + hk) * d + c;
        if (fp4) {
          kt[(size_t)t * d + c] = deq(C.kc[(size_t)e], C.ks[(size_t)(e / 16)], C.gk);
          const int64_t ve = (((int64_t)b * Hkv + hk) * d + c) * vcol + k0 + t;
          vt[(size_t)t * d + c] = deq(C.vc[(size_t)ve], C.vs[(size_t)(ve / 16)], C.gv);
        } else {
          kt[(size_t)t * d + c] = orc_half_to_float(C.k[e], C.dt);
          vt[(size_t)t * d + c] = orc_half_to_float(C.v[e], C.dt);
        }
      }
    const double* qv = fp4 ? qh.data() : q16.data();
    double mt = -INFINITY, amx = 0.0, smx = 0.0;
    for (int t = 0; t < nk; ++t) {
      double acc = 0.0, aabs = 0.0;
      for (int c = 0; c < d; ++c) {
        acc += qv[c] * kt[(size_t)t * d + c];
        aabs += std::fabs(qv[c] * kt[(size_t)t * d + c]);
      }
      S[t] = acc * (fp4 ? s4 : s16);
      mt = std::max(mt, S[t]);
      amx = std::max(amx, aabs * (fp4 ? s4 : s16));
      smx = std::max(smx, std::fabs(S[t]));
    }
    const double mn = std::max(m, mt);
    const double alpha = std::exp2(m - mn);  // 0 when m is still -inf
    arun = std::max(arun, amx);
    l *= alpha;
    for (int c = 0; c < d; ++c) {
      O[c] *= alpha;
      amb[c] *= alpha;
    }
    for (int t = 0; t < nk; ++t) {
      Pt[t] = (float)std::exp2(S[t] - mn);
      l += (double)Pt[t];
    }
    if (fp4) {
      const double rho = tile_radius(d, amx, smx, std::fabs(mt));
      const float sigma = p_tile_fp4(Pt.data(), nk, blk, rho, b, h, 0, k0, Pq.data(), dq.data());
      if (sigma == 0.0f) { m = mn; continue; }
      for (int c = 0; c < d; ++c) {
        double acc = 0.0, ab = 0.0;
        for (int t = 0; t < nk; ++t) {
          acc += Pq[t] * vt[(size_t)t * d + c];
          ab += dq[t] * std::fabs(vt[(size_t)t * d + c]);
        }
        O[c] += (double)sigma * acc;
        amb[c] += (double)sigma * ab;
      }
    } else {
      const double rho = tile_radius(d, arun, smx, std::fabs(mn));
      p_tile_16(Pt.data(), nk, C.dt, rho, b, h, 0, k0, Pq.data(), dq.data());
      for (int c = 0; c < d; ++c) {
        double acc = 0.0, ab = 0.0;
        for (int t = 0; t < nk; ++t) {
          acc += Pq[t] * vt[(size_t)t * d + c];
          ab += dq[t] * std::fabs(vt[(size_t)t * d + c]);
        }
        O[c] += acc;
        amb[c] += ab;
      }
    }
    m = mn;
  }
  const double ln2 = 0.6931471805599453;
  for (int c = 0; c < d; ++c) {
    const double o = l > 0.0 ? O[c] / l : 0.0;
    out[orow + c] = orc_double_to_half(o, C.dt);
    if (out64) out64[orow + c] = o;
    if (tol) tol[orow + c] = l > 0.0 ? amb[c] / l : 0.0;
  }
  lse[(int64_t)b * H + h] = l > 0.0 ? (float)(m * ln2 + std::log(l)) : -INFINITY;
}

// Decode step over the double cache (reading R15).  g_kv: g_K, g_V.
// mask [B, H, nbcap] (nbcap = ceil(ncap / blk)): read when mask_given, else
// computed and written.  out 16-bit [B, H, d]; lse fp32 [B, H] (natural log;
// -inf and a zero row for an empty sequence).  gq_in (optional) gives g_Q
// (for a sample of the sequences of a larger step), else it is amax(q) /
// 2688; gq_out (optional) receives it; out64 / tol (optional) as in
// orc_thrift_attn.
int orc_thrift_decode(const uint16_t* q, const uint16_t* k, const uint16_t* v, int dt, int B,
                      int H, int Hkv, int ncap, int d, int blk, const int32_t* lens,
                      const float* g_kv, float frac, int sink, int recent, int use_ss,
                      uint8_t* mask_io, int mask_given, const float* gq_in, int nthreads,
                      uint16_t* out, float* lse, float* gq_out, double* out64, double* tol) {
  if (B <= 0 || H <= 0 || Hkv <= 0 || H % Hkv || ncap <= 0 || d % 16 || blk % 16 || blk <= 0)
    return -1;
  if (sink < 0 || recent < 0 || !(frac >= 0.0f && frac <= 1.0f)) return -1;
  for (int b = 0; b < B; ++b)
    if (lens[b] < 0 || lens[b] > ncap) return -1;
  DecCtx C;
  C.dt = dt; C.B = B; C.H = H; C.Hkv = Hkv; C.ncap = ncap; C.d = d; C.blk = blk;
  C.nbcap = (ncap + blk - 1) / blk;
  C.lens = lens; C.q = q; C.k = k; C.v = v;
  C.gk = g_kv[0];
  C.gv = g_kv[1];
  if (gq_in) {
    C.gq = *gq_in;
    quantize_rows_given(q, dt, (int64_t)B * H, d, C.gq, use_ss, nthreads, C.qc, C.qs);
  } else {
    C.gq = quantize_rows_unpacked(q, dt, (int64_t)B * H, d, use_ss, 0, nthreads, C.qc, C.qs);
  }
  quantize_rows_given(k, dt, (int64_t)B * ncap * Hkv, d, C.gk, use_ss, nthreads, C.kc, C.ks);
  // V: per (sequence, kv head, channel) column of nbcap * blk tokens, 16-blocks
  // from token 0, tokens at or past len zero.
  const int64_t vcol = (int64_t)C.nbcap * blk;
  C.vc.assign((size_t)((int64_t)B * Hkv * d * vcol), 0);
  C.vs.assign((size_t)((int64_t)B * Hkv * d * vcol / 16), 0);
  parallel_for((int64_t)B * Hkv * d, nthreads, [&](int64_t bc) {
    const int64_t b = bc / ((int64_t)Hkv * d), hk = (bc / d) % Hkv, c = bc % d;
    float col[16];
    uint8_t packed[8];
    for (int64_t t0 = 0; t0 < vcol; t0 += 16) {
      for (int e = 0; e < 16; ++e)
        col[e] = t0 + e < lens[b]
                     ? orc_half_to_float(v[((b * ncap + t0 + e) * Hkv + hk) * d + c], dt)
                     : 0.0f;
      const int64_t base = bc * vcol + t0;
      orc_quant_block(col, C.gv, use_ss, packed, &C.vs[(size_t)(base / 16)], nullptr);
      for (int e = 0; e < 8; ++e) {
        C.vc[(size_t)(base + 2 * e)] = packed[e] & 0xF;
        C.vc[(size_t)(base + 2 * e + 1)] = packed[e] >> 4;
      }
    }
  });
  if (gq_out) *gq_out = C.gq;
  if (!mask_given)
    parallel_for((int64_t)B * H, nthreads, [&](int64_t u) {
      const int b = (int)(u / H), h = (int)(u % H);
      decode_select_one(q, k, dt, H, Hkv, ncap, d, blk, b, h, lens[b], frac, sink, recent,
                        mask_io + u * C.nbcap, C.nbcap);
    });
  C.mask = mask_io;
  parallel_for((int64_t)B * H, nthreads, [&](int64_t u) {
    decode_row(C, (int)(u / H), (int)(u % H), out, lse, out64, tol);
  });
  return 0;
}

// ------------------------------------------------ Attn-QAT backward --
//
// Reading R17.  q [total, H, d], k, v [total, Hkv, d], dout [total, H, d]
// 16-bit over packed sequences cu [nseq+1]; blk = key tile of the P
// quantisation.  Outputs (fp64): o (the FP4 forward output P^ V^), o_hp
// (O' = P V^), lse [H, total] (natural log), dq [total, H, d], dk, dv
// [total, Hkv, d] (summed over the query heads of a kv head).  g_in
// (optional, 3 floats): the tensor scales of Q, K, V to use instead of those
// of the given tensors (a slice of a larger problem keeps the whole tensor's
// scales, reading C3).
int orc_attn_qat_bwd(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                     const uint16_t* dout, int dt, int H, int Hkv, const int32_t* cu, int nseq,
                     int d, int blk, int causal, int use_ss, int nthreads, const float* g_in,
                     double* o, double* o_hp, double* lse, double* dq, double* dk, double* dv) {
  if (H <= 0 || Hkv <= 0 || H % Hkv || nseq <= 0 || d % 16 || blk % 16 || blk <= 0) return -1;
  const int64_t total = cu[nseq];
  std::vector<uint8_t> qc, qs, kc, ks, vc, vs;
  const float gq = quantize_rows_unpacked(q, dt, total * H, d, use_ss, 0, nthreads, qc, qs,
                                          g_in ? g_in + 0 : nullptr);
  const float gk = quantize_rows_unpacked(k, dt, total * Hkv, d, use_ss, 0, nthreads, kc, ks,
                                          g_in ? g_in + 1 : nullptr);
  // V: 16-blocks along the tokens of each sequence (zero-padded), reading R6
  std::vector<int64_t> pst(nseq + 1, 0);
  for (int s = 0; s < nseq; ++s) {
    const int len = cu[s + 1] - cu[s];
    if (len <= 0) return -1;
    pst[s + 1] = pst[s] + (len + 15) / 16 * 16;
  }
  const int64_t ptot = pst[nseq];
  float vamax = 0.0f;
  for (int64_t e = 0; e < total * Hkv * d; ++e) vamax = std::max(vamax, std::fabs(orc_half_to_float(v[e], dt)));
  const float gv = g_in ? g_in[2] : (vamax == 0.0f ? 1.0f : vamax / 2688.0f);
  std::vector<uint8_t> vcol((size_t)(Hkv * d * ptot), 0), vsc((size_t)(Hkv * d * ptot / 16), 0);
  for (int64_t hc = 0; hc < (int64_t)Hkv * d; ++hc) {
    const int64_t hk = hc / d, c = hc % d;
    float col[16];
    uint8_t packed[8];
    for (int s = 0; s < nseq; ++s) {
      const int len = cu[s + 1] - cu[s];
      for (int64_t t0 = 0; t0 < pst[s + 1] - pst[s]; t0 += 16) {
        for (int e = 0; e < 16; ++e)
          col[e] = t0 + e < len ? orc_half_to_float(v[((cu[s] + t0 + e) * Hkv + hk) * d + c], dt) : 0.0f;
        const int64_t base = hc * ptot + pst[s] + t0;
        orc_quant_block(col, gv, use_ss, packed, &vsc[(size_t)(base / 16)], nullptr);
        for (int e = 0; e < 8; ++e) {
          vcol[(size_t)(base + 2 * e)] = packed[e] & 0xF;
          vcol[(size_t)(base + 2 * e + 1)] = packed[e] >> 4;
        }
      }
    }
  }
  // dequantised values, tabulated once: Q^ [total, H, d], K^ and V^
  // [total, Hkv, d], and dO as fp64
  std::vector<double> qd((size_t)(total * H * d)), kd((size_t)(total * Hkv * d)),
      vd((size_t)(total * Hkv * d)), dod((size_t)(total * H * d));
  for (int64_t e = 0; e < total * H * d; ++e) {
    qd[(size_t)e] = deq(qc[(size_t)e], qs[(size_t)(e / 16)], gq);
    dod[(size_t)e] = (double)orc_half_to_float(dout[e], dt);
  }
  for (int64_t e = 0; e < total * Hkv * d; ++e) kd[(size_t)e] = deq(kc[(size_t)e], ks[(size_t)(e / 16)], gk);
  for (int s = 0; s < nseq; ++s)
    for (int64_t t = cu[s]; t < cu[s + 1]; ++t)
      for (int hk = 0; hk < Hkv; ++hk)
        for (int c = 0; c < d; ++c) {
          const int64_t ve = ((int64_t)hk * d + c) * ptot + pst[s] + (t - cu[s]);
          vd[(size_t)((t * Hkv + hk) * d + c)] = deq(vcol[(size_t)ve], vsc[(size_t)(ve / 16)], gv);
        }
  auto qhat = [&](int64_t t, int h, int c) { return qd[(size_t)((t * H + h) * d + c)]; };
  auto khat = [&](int64_t t, int hk, int c) { return kd[(size_t)((t * Hkv + hk) * d + c)]; };
  auto vhat = [&](int64_t t, int hk, int c) { return vd[(size_t)((t * Hkv + hk) * d + c)]; };
  for (int64_t e = 0; e < total * Hkv * d; ++e) dk[e] = dv[e] = 0.0;
  const double sc = 1.0 / std::sqrt((double)d);
  // one (sequence, head) at a time: the kv-head gradients of different
  // heads add into the same rows, so heads run in order
  for (int s = 0; s < nseq; ++s) {
    const int64_t st = cu[s];
    const int len = cu[s + 1] - cu[s];
    for (int h = 0; h < H; ++h) {
      const int hk = h / (H / Hkv);
      std::vector<double> P((size_t)len * len, 0.0), Ph((size_t)len * len, 0.0),
          dS((size_t)len * len, 0.0);
      parallel_for(len, nthreads, [&](int64_t i) {
        const int kend = causal ? (int)i + 1 : len;
        std::vector<double> srow(len, -INFINITY);
        double mx = -INFINITY;
        for (int j = 0; j < kend; ++j) {
          double acc = 0.0;
          for (int c = 0; c < d; ++c) acc += qhat(st + i, h, c) * khat(st + j, hk, c);
          srow[j] = acc * sc;
          mx = std::max(mx, srow[j]);
        }
        double den = 0.0;
        for (int j = 0; j < kend; ++j) den += std::exp(srow[j] - mx);
        const double lz = mx + std::log(den);
        lse[(int64_t)h * total + st + i] = lz;
        for (int j = 0; j < kend; ++j) P[(size_t)i * len + j] = std::exp(srow[j] - lz);
        // P^: two-level FP4 image per key tile (reading R7 on the normalised row)
        for (int j0 = 0; j0 < kend; j0 += blk) {
          const int j1 = std::min(kend, j0 + blk);
          std::vector<float> pt(blk, 0.0f);
          float rowmax = 0.0f;
          for (int j = j0; j < j1; ++j) {
            pt[j - j0] = (float)P[(size_t)i * len + j];
            rowmax = std::max(rowmax, pt[j - j0]);
          }
          if (rowmax == 0.0f) continue;
          const float inv = 2688.0f / rowmax, sigma = rowmax / 2688.0f;
          for (int b0 = 0; b0 < blk; b0 += 16) {
            float ph[16], amax = 0.0f;
            for (int e = 0; e < 16; ++e) {
              ph[e] = pt[b0 + e] * inv;
              amax = std::max(amax, ph[e]);
            }
            const uint8_t sp = orc_ue4m3_encode(amax / 6.0f);
            const float dec = orc_ue4m3_decode(sp);
            const float rr = 1.0f / dec;
            for (int e = 0; e < 16; ++e) {
              const int j = j0 + b0 + e;
              if (j >= j1 || sp == 0) continue;
              Ph[(size_t)i * len + j] = (double)orc_e2m1_decode(orc_e2m1_encode(ph[e] * rr)) *
                                        (double)dec * (double)sigma;
            }
          }
        }
      });
      // outputs, D, dP, dS and the gradients of this head
      parallel_for(len, nthreads, [&](int64_t i) {
        const int64_t ti = st + i;
        std::vector<double> oh(d, 0.0), ohp(d, 0.0);
        for (int j = 0; j < len; ++j) {
          const double p = P[(size_t)i * len + j], ph = Ph[(size_t)i * len + j];
          if (p == 0.0 && ph == 0.0) continue;
          for (int c = 0; c < d; ++c) {
            const double vv = vhat(st + j, hk, c);
            oh[c] += ph * vv;
            ohp[c] += p * vv;
          }
        }
        double D = 0.0;
        for (int c = 0; c < d; ++c) {
          o[(ti * H + h) * d + c] = oh[c];
          o_hp[(ti * H + h) * d + c] = ohp[c];
          D += dod[(size_t)((ti * H + h) * d + c)] * ohp[c];
        }
        std::vector<double> dqr(d, 0.0);
        for (int j = 0; j < len; ++j) {
          const double p = P[(size_t)i * len + j];
          if (p == 0.0) continue;
          double dp = 0.0;
          for (int c = 0; c < d; ++c)
            dp += dod[(size_t)((ti * H + h) * d + c)] * vhat(st + j, hk, c);
          const double ds = p * (dp - D);
          dS[(size_t)i * len + j] = ds;
          for (int c = 0; c < d; ++c) dqr[c] += ds * khat(st + j, hk, c) * sc;
        }
        for (int c = 0; c < d; ++c) dq[(ti * H + h) * d + c] = dqr[c];
      });
      // dK, dV rows of this head: key j sums over the queries in order
      // (blocks of 64 keys keep the row reads of P^ and dS contiguous)
      parallel_for((len + 63) / 64, nthreads, [&](int64_t jb) {
        const int j0 = (int)jb * 64, j1 = std::min(len, j0 + 64);
        for (int64_t i = 0; i < len; ++i) {
          const int64_t ti = st + i;
          for (int j = j0; j < j1; ++j) {
            const double p = P[(size_t)i * len + j], ph = Ph[(size_t)i * len + j];
            if (p == 0.0 && ph == 0.0) continue;
            const double ds = dS[(size_t)i * len + j];
            const int64_t tj = st + j;
            for (int c = 0; c < d; ++c) {
              const double g = dod[(size_t)((ti * H + h) * d + c)];
              dv[(tj * Hkv + hk) * d + c] += ph * g;
              dk[(tj * Hkv + hk) * d + c] += ds * qhat(ti, h, c) * sc;
            }
          }
        }
      });
    }
  }
  return 0;
}

// Unquantised attention in fp64 (softmax(Q K^T / sqrt(d)) V) over packed
// sequences; out fp64 [total, H, d], lse fp64 [H, total] (natural log).
// rows (optional): list of (token, head) pairs to compute; n_rows = 0 = all.
int orc_attn_fp64(const uint16_t* q, const uint16_t* k, const uint16_t* v, int dt, int H,
                  int Hkv, const int32_t* cu, int nseq, int d, int causal,
                  const int64_t* rows, int64_t n_rows, int nthreads, double* out, double* lse) {
  if (H <= 0 || Hkv <= 0 || H % Hkv) return -1;
  const int64_t total = cu[nseq];
  std::vector<int32_t> seq_of((size_t)total);
  for (int s = 0; s < nseq; ++s)
    for (int64_t t = cu[s]; t < cu[s + 1]; ++t) seq_of[(size_t)t] = s;
  const int64_t n = n_rows ? n_rows : total * H;
  parallel_for(n, nthreads, [&](int64_t u) {
    int64_t tok = n_rows ? rows[2 * u] : u / H;
    int h = n_rows ? (int)rows[2 * u + 1] : (int)(u % H);
    int s = seq_of[(size_t)tok];
    int hk = h / (H / Hkv);
    int64_t k0 = cu[s], k1 = causal ? tok + 1 : cu[s + 1];
    std::vector<double> sc((size_t)(k1 - k0));
    double mx = -INFINITY;
    for (int64_t t = k0; t < k1; ++t) {
      double acc = 0.0;
      for (int c = 0; c < d; ++c)
        acc += (double)orc_half_to_float(q[(tok * H + h) * d + c], dt) *
               (double)orc_half_to_float(k[(t * Hkv + hk) * d + c], dt);
      sc[(size_t)(t - k0)] = acc / std::sqrt((double)d);
      mx = std::max(mx, sc[(size_t)(t - k0)]);
    }
    double den = 0.0;
    for (auto& x : sc) { x = std::exp(x - mx); den += x; }
    for (int c = 0; c < d; ++c) {
      double acc = 0.0;
      for (int64_t t = k0; t < k1; ++t)
        acc += sc[(size_t)(t - k0)] * (double)orc_half_to_float(v[(t * Hkv + hk) * d + c], dt);
      out[(tok * H + h) * d + c] = acc / den;
    }
    lse[(int64_t)h * total + tok] = mx + std::log(den);
  });
  return 0;
}

}  // extern "C"
