// C-ABI entry points of libthrift_nvfp4.so: argument checks, workspace
// carving and kernel launches.  Declarations and the contract of every entry
// point are in include/thrift_nvfp4.h.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdio>
#include <mutex>
#include <utility>
#include <vector>

#include "attn.cuh"
#include "decode.cuh"
#include "qat.cuh"
#include "select.cuh"

namespace thrift {
namespace {

constexpr int kThreads = 256;

int grid_for(int64_t work_items, int per_block = kThreads) {
  int64_t g = ceil_div(work_items, per_block);
  if (g < 1) g = 1;
  if (g > 148 * 16) g = 148 * 16;
  return (int)g;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

thrift_status launch_status() {
  return cudaGetLastError() == cudaSuccess ? THRIFT_OK : THRIFT_ERR_CUDA;
}

// Bump allocator over the caller's workspace (1024-byte aligned slices).
struct Carve {
  uintptr_t base;
  size_t off = 0;
  explicit Carve(void* b) : base(reinterpret_cast<uintptr_t>(b)) {}
  template <class T>
  T* take(size_t bytes) {
    off = (off + 1023) & ~(size_t)1023;
    T* p = reinterpret_cast<T*>(base + off);
    off += bytes;
    return p;
  }
};

// Device-side settings (function attributes, occupancy queries) apply to
// the current device, so each is made once per device: bit `dev` of a
// DeviceSet records that it has succeeded there.
constexpr int kMaxDevices = 64;

int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return -1;
  return dev;
}

struct DeviceSet {
  std::atomic<uint64_t> bits{0};
  bool has(int dev) const { return (bits.load() >> dev) & 1u; }
  void add(int dev) { bits.fetch_or(1ull << dev); }
};

// Raises the dynamic shared-memory limit of `kernel` to `bytes` on the
// current device (once per device).
template <class Kernel>
bool smem_attr(Kernel kernel, size_t bytes, DeviceSet& done) {
  const int dev = current_device();
  if (dev < 0) return false;
  if (done.has(dev)) return true;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) !=
      cudaSuccess)
    return false;
  done.add(dev);
  return true;
}

// ------------------------------------------------------- quantiser glue --

int sm_count() {
  static std::atomic<int> n[kMaxDevices] = {};
  const int dev = current_device();
  if (dev < 0) return 148;
  if (n[dev].load() == 0) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
      v = 148;
    n[dev].store(v);
  }
  return n[dev].load();
}

// Grid for the streaming (grid-stride) kernels: enough CTAs for kKPT blocks
// per thread, capped at one full wave (resident CTAs per SM x SMs) so that no
// partial second wave trails the launch.
template <class Kernel>
int stream_grid(Kernel kernel, int64_t n_blocks, int kpt = kKPT) {
  static std::atomic<int> per_dev[kMaxDevices] = {};  // per kernel instantiation
  const int dev = current_device();
  int resident = dev < 0 ? 0 : per_dev[dev].load();
  if (resident == 0) {
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kThreads, 0) !=
            cudaSuccess || per_sm < 1)
      per_sm = 1;
    resident = per_sm * sm_count();
    if (dev >= 0) per_dev[dev].store(resident);
  }
  int64_t g = ceil_div(n_blocks, (int64_t)kThreads * kpt);
  if (g < 1) g = 1;
  if (g > resident) g = resident;
  return (int)g;
}

template <int DT, int G>
void launch_amax_t(const uint16_t* xp, int64_t n_blocks, uint32_t* out, cudaStream_t st) {
  amax_kernel<DT, G><<<stream_grid(amax_kernel<DT, G>, n_blocks), kThreads, 0, st>>>(
      xp, n_blocks, out);
}

template <int DT>
void launch_amax(const void* x, int64_t n_blocks, int G, uint32_t* out, cudaStream_t st) {
  const uint16_t* xp = static_cast<const uint16_t*>(x);
  if (G == 8) launch_amax_t<DT, 8>(xp, n_blocks, out, st);
  else if (G == 4) launch_amax_t<DT, 4>(xp, n_blocks, out, st);
  else launch_amax_t<DT, 0>(xp, n_blocks, out, st);
}

// Launch with programmatic dependent launch allowed: the kernel may start
// while the previous kernel of the stream finishes; it waits for it
// (pdl_wait) before touching anything that kernel may write.
template <class Kernel, class... Args>
cudaError_t launch_pdl(Kernel kernel, int grid, int threads, cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Quantiser workspace: from byte 256, the per-CTA maxima of the partial
// absmax kernel (one float each).  Every call that computes the tensor scale
// writes the slots it then reads, so no call depends on the workspace's
// earlier contents.
constexpr size_t kQuantWsBytes = 4096;
constexpr int kQuantMaxPartials = (int)((kQuantWsBytes - 256) / 4);

float* quant_partials(uint32_t* ws) {
  return reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(ws) + 256);
}

// The partial absmax kernel over n_blocks 16-element blocks of x (rows
// rotated when G > 0); returns its grid (the number of partial maxima).
template <int DT, int G>
int launch_amax_partial(const uint16_t* xp, int64_t nb, float* partial, cudaStream_t st,
                        thrift_status* s) {
  auto kern = amax_partial_kernel<DT, G>;
  const int grid = std::min(kQuantMaxPartials, stream_grid(kern, nb));
  *s = launch_pdl(kern, grid, kThreads, st, xp, nb, partial) == cudaSuccess ? THRIFT_OK
                                                                             : THRIFT_ERR_CUDA;
  return grid;
}

template <int DT, int G, bool SS>
thrift_status quantize_rows(const void* x, int64_t nb, uint32_t* ws, float* ts, int given,
                            uint8_t* codes, uint8_t* scales, cudaStream_t st) {
  const uint16_t* xp = static_cast<const uint16_t*>(x);
  float* partial = quant_partials(ws);
  int np = 0;
  thrift_status s = THRIFT_OK;
  if (!given) np = launch_amax_partial<DT, G>(xp, nb, partial, st, &s);
  if (s != THRIFT_OK) return s;
  auto kern = quant_rows_kernel<DT, G, SS>;
  return launch_pdl(kern, stream_grid(kern, nb, kQuantKPT), kThreads, st, xp, nb,
                    static_cast<const float*>(partial), np, ts, given, codes, scales) ==
                 cudaSuccess
             ? THRIFT_OK
             : THRIFT_ERR_CUDA;
}

template <int DT>
thrift_status launch_quantize(const void* x, int64_t nb, int G, bool ss, uint32_t* ws,
                              float* ts, int given, uint8_t* codes, uint8_t* scales,
                              cudaStream_t st) {
#define THRIFT_QUANT_CASE(GG, SSV) \
  if (G == GG && ss == SSV) return quantize_rows<DT, GG, SSV>(x, nb, ws, ts, given, codes, scales, st);
  THRIFT_QUANT_CASE(0, false)
  THRIFT_QUANT_CASE(0, true)
  THRIFT_QUANT_CASE(4, false)
  THRIFT_QUANT_CASE(4, true)
  THRIFT_QUANT_CASE(8, false)
  THRIFT_QUANT_CASE(8, true)
#undef THRIFT_QUANT_CASE
  return THRIFT_ERR_UNSUPPORTED;
}

// ---------------------------------------------------------- selection --

// The top-k pairs of every (sequence, head): one CTA each when its keys fit
// the CTA's shared-memory cache, else a cluster of kTopkCluster CTAs that
// split the keys (same selection, bit for bit).
thrift_status launch_topk(const double* scores, SeqInfo si, int nseq, int H, int blk, int nB,
                          int causal, float frac, int sink, int recent, uint8_t* mask,
                          cudaStream_t st) {
  if ((int64_t)nB * nB <= kTopkCache) {
    topk_kernel<<<nseq * H, kTopkThreads, topk_smem(nB), st>>>(scores, si, H, blk, nB, causal,
                                                               frac, sink, recent, mask);
    return launch_status();
  }
  static DeviceSet attr;
  const size_t smem = topk_cluster_smem(nB);
  if (!smem_attr(topk_cluster_kernel, kTopkClusterCacheBytes, attr)) return THRIFT_ERR_CUDA;
  topk_cluster_kernel<<<nseq * H * kTopkCluster, kTopkThreads, smem, st>>>(
      scores, si, H, blk, nB, causal, frac, sink, recent, mask, smem > 0 ? 1 : 0);
  return launch_status();
}

// ----------------------------------------------------- attention layout --

struct AttnWs {
  uint32_t* amax;
  double* means_q;
  double* means_k;
  double* scores;
  uint8_t* mask;
  uint8_t *q4, *k4, *v4, *q16, *k16, *v16;
  double* ksum;      // K smoothing: block sums [nseq, Hkv, nb128, d]
  float *kmin, *kmax;
  float* kmu;        // channel means [nseq, Hkv, d]
  float* qcorr;      // q^ . mu per query row [nseq, H, nTq * 128]
  size_t bytes;
};

AttnWs carve_attn(void* ws, int nseq, int maxlen, int H, int Hkv, int d, int blk) {
  Carve c(ws);
  AttnWs w;
  const int64_t nB = ceil_div(maxlen, blk), nTq = ceil_div(maxlen, 128);
  w.amax = c.take<uint32_t>(256);
  w.means_q = c.take<double>((size_t)nseq * H * nB * d * 8);
  w.means_k = c.take<double>((size_t)nseq * Hkv * nB * d * 8);
  w.scores = c.take<double>((size_t)nseq * H * nB * nB * 8);
  w.mask = c.take<uint8_t>((size_t)nseq * H * nB * nB);
  w.q4 = c.take<uint8_t>((size_t)nseq * H * nTq * fp4_tile_bytes(128, d));
  w.k4 = c.take<uint8_t>((size_t)nseq * Hkv * nB * fp4_tile_bytes(blk, d));
  w.v4 = c.take<uint8_t>((size_t)nseq * Hkv * nB * fp4_tile_bytes(d, blk));
  w.q16 = c.take<uint8_t>((size_t)nseq * H * nTq * f16_tile_bytes(128, d));
  w.k16 = c.take<uint8_t>((size_t)nseq * Hkv * nB * f16_tile_bytes(blk, d));
  w.v16 = c.take<uint8_t>((size_t)nseq * Hkv * nB * f16_tile_bytes(d, blk));
  const int64_t nb128 = ceil_div(maxlen, 128);
  w.ksum = c.take<double>((size_t)nseq * Hkv * nb128 * d * 8);
  w.kmin = c.take<float>((size_t)nseq * Hkv * nb128 * d * 4);
  w.kmax = c.take<float>((size_t)nseq * Hkv * nb128 * d * 4);
  w.kmu = c.take<float>((size_t)nseq * Hkv * d * 4);
  w.qcorr = c.take<float>((size_t)nseq * H * nTq * 128 * 4);
  w.bytes = c.off + 1024;
  return w;
}

// Image (and block-mean) launches: one CTA per (tile, head, sequence), the
// tile staged in shared memory.
struct TileArgs {
  const void* x;
  SeqInfo si;
  int nseq, nh, rows, ntiles, blk, nB;
  const uint32_t* amax;
  uint8_t *i4, *i16;
  double* means;
  const float* mu = nullptr;  // K smoothing (see qk_tile_kernel)
  int mu_group = 1;
  float* corr = nullptr;
};

template <int DT, int G, bool HAD, bool SS>
void launch_qk_tile(const TileArgs& a, cudaStream_t st) {
  dim3 grid(a.ntiles, a.nh, a.nseq);
  const size_t smem = (size_t)a.rows * G * 16 * 2;
  qk_tile_kernel<DT, G, HAD, SS><<<grid, kThreads, smem, st>>>(
      static_cast<const uint16_t*>(a.x), a.si, a.nh, a.rows, a.ntiles, a.blk, a.nB, a.amax, a.i4,
      a.i16, a.means, a.mu, a.mu_group, a.corr);
}

template <int DT, int G>
void dispatch_qk_tile(bool had, bool ss, const TileArgs& a, cudaStream_t st) {
  if (had) {
    if (ss) launch_qk_tile<DT, G, true, true>(a, st);
    else launch_qk_tile<DT, G, true, false>(a, st);
  } else {
    if (ss) launch_qk_tile<DT, G, false, true>(a, st);
    else launch_qk_tile<DT, G, false, false>(a, st);
  }
}

// Optional event pairs around the attention kernel (thrift_kernel_timer_*).
struct KernelTimer {
  bool enabled = false;
  std::vector<std::pair<cudaEvent_t, cudaEvent_t>> pool;
  size_t used = 0;
  cudaEvent_t* next_pair() {
    if (used == pool.size()) {
      cudaEvent_t a, b;
      if (cudaEventCreate(&a) != cudaSuccess) return nullptr;
      if (cudaEventCreate(&b) != cudaSuccess) return nullptr;
      pool.push_back({a, b});
    }
    return &pool[used++].first;
  }
};
KernelTimer g_timer;

template <int DT, int D, int BLK>
thrift_status launch_attn_kernel(const AttnParams& p, int nTq, cudaStream_t st) {
  using L = AttnLayout<D, BLK>;
  static DeviceSet attr;
  if (!smem_attr(attn_fwd_kernel<DT, D, BLK>, L::SMEM_ALLOC, attr)) return THRIFT_ERR_CUDA;
  dim3 grid(nTq, p.H, p.nseq);
  cudaEvent_t* ev = g_timer.enabled ? g_timer.next_pair() : nullptr;
  if (ev) cudaEventRecord(ev[0], st);
  attn_fwd_kernel<DT, D, BLK><<<grid, kAttnThreads, L::SMEM_ALLOC, st>>>(p);
  const thrift_status s = launch_status();
  if (ev) cudaEventRecord(ev[1], st);
  return s;
}

// The three tensor absmaxes of an attention call into amax[0..2] (bit
// patterns of non-negative floats): Q and K rotated when `had`, K - mu with
// K smoothing (whose channel means land in w.kmu on the way).
template <int DT>
thrift_status attn_absmax(const void* q, const void* k, const void* v, SeqInfo si, int nseq,
                          int64_t total, int maxlen, int H, int Hkv, int d, int had, int smooth,
                          const AttnWs& w, uint32_t* amax, cudaStream_t st) {
  const int G = d / 16;
  if (cudaMemsetAsync(amax, 0, 12, st) != cudaSuccess) return THRIFT_ERR_CUDA;
  launch_amax<DT>(q, total * H * d / 16, had ? G : 0, amax + 0, st);
  if (smooth) {
    // K smoothing: channel means per (sequence, kv head) and the absmax of
    // K - mu, from one pass of block statistics over K
    const int nb128 = (int)ceil_div(maxlen, 128);
    k_stats_kernel<DT><<<dim3(nb128, Hkv, nseq), 128, 0, st>>>(
        static_cast<const uint16_t*>(k), si, Hkv, d, nb128, w.ksum, w.kmin, w.kmax);
    k_mean_kernel<<<dim3(Hkv, nseq), 128, 0, st>>>(w.ksum, w.kmin, w.kmax, si, Hkv, d, nb128,
                                                   w.kmu, amax + 1);
  } else {
    launch_amax<DT>(k, total * Hkv * d / 16, had ? G : 0, amax + 1, st);
  }
  launch_amax<DT>(v, total * Hkv * d / 16, 0, amax + 2, st);
  return launch_status();
}

// One attention call.  amax_given (device, 3 floats) replaces the call's own
// tensor absmaxes when not null (a shard of a larger problem).
template <int DT>
thrift_status attn_impl(const void* q, const void* k, const void* v, SeqInfo si, int nseq,
                        int64_t total, int maxlen, int H, int Hkv, int d, int blk, int causal,
                        float frac, int sink, int recent, int ss, int had, int smooth, void* out,
                        float* lse, int lse_varlen, void* ws, cudaStream_t st,
                        const float* amax_given = nullptr) {
  AttnWs w = carve_attn(ws, nseq, maxlen, H, Hkv, d, blk);
  const int nB = (int)ceil_div(maxlen, blk), nTq = (int)ceil_div(maxlen, 128);
  const int G = d / 16;
  if (amax_given) {
    // the given absmaxes; K smoothing still needs this shard's channel means
    // (its own absmax goes to a spare word)
    if (smooth) {
      const thrift_status s0 = attn_absmax<DT>(q, k, v, si, nseq, total, maxlen, H, Hkv, d, had,
                                               smooth, w, w.amax + 4, st);
      if (s0 != THRIFT_OK) return s0;
    }
    if (cudaMemcpyAsync(w.amax, amax_given, 12, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
      return THRIFT_ERR_CUDA;
  } else {
    const thrift_status s0 = attn_absmax<DT>(q, k, v, si, nseq, total, maxlen, H, Hkv, d, had,
                                             smooth, w, w.amax, st);
    if (s0 != THRIFT_OK) return s0;
  }
  // Q and K images, with the block means of the selection on the way
  TileArgs aq{q, si, nseq, H, 128, nTq, blk, nB, w.amax + 0, w.q4, w.q16, w.means_q};
  TileArgs ak{k, si, nseq, Hkv, blk, nB, blk, nB, w.amax + 1, w.k4, w.k16, w.means_k};
  if (smooth) {
    aq.mu = w.kmu;
    aq.mu_group = H / Hkv;
    aq.corr = w.qcorr;
    ak.mu = w.kmu;
  }
  if (G == 8) {
    dispatch_qk_tile<DT, 8>(had, ss, aq, st);
    dispatch_qk_tile<DT, 8>(had, ss, ak, st);
  } else {
    dispatch_qk_tile<DT, 4>(had, ss, aq, st);
    dispatch_qk_tile<DT, 4>(had, ss, ak, st);
  }
  {
    // input tile, then the NVFP4 and 16-bit output images (128-byte aligned)
    dim3 grid(nB, Hkv, nseq);
    const size_t smem = (size_t)blk * d * 2 + ((fp4_tile_bytes(d, blk) + 127) & ~127u) +
                        f16_tile_bytes(d, blk);
    auto kern = ss ? v_tile_kernel<DT, true> : v_tile_kernel<DT, false>;
    static DeviceSet attr[2];
    if (!smem_attr(kern, 96 * 1024, attr[ss ? 1 : 0])) return THRIFT_ERR_CUDA;
    kern<<<grid, kThreads, smem, st>>>(static_cast<const uint16_t*>(v), si, Hkv, d, blk, nB,
                                       w.amax + 2, w.v4, w.v16);
  }
  // selection
  pair_scores_kernel<<<pair_scores_grid(nseq, H, nB), kThreads, pair_scores_smem(nB), st>>>(
      w.means_q, w.means_k, si, nseq, H, Hkv, d, blk, nB, causal, w.scores);
  if (launch_topk(w.scores, si, nseq, H, blk, nB, causal, frac, sink, recent, w.mask, st) !=
      THRIFT_OK)
    return THRIFT_ERR_CUDA;

  AttnParams p;
  p.q4 = w.q4; p.k4 = w.k4; p.v4 = w.v4; p.q16 = w.q16; p.k16 = w.k16; p.v16 = w.v16;
  p.mask = w.mask;
  p.amax = w.amax;
  p.out = static_cast<uint16_t*>(out);
  p.lse = lse;
  p.seqs = si;
  p.nseq = nseq; p.H = H; p.Hkv = Hkv; p.nB = nB; p.nTq = nTq; p.causal = causal;
  p.lse_varlen = lse_varlen;
  p.total = total;
  p.corr = smooth ? w.qcorr : nullptr;
  const double l2e = 1.4426950408889634;
  p.scale16 = (float)(l2e / std::sqrt((double)d));
  p.scale4 = (float)(l2e / std::sqrt((double)d) / (had ? (double)d : 1.0));
  if (d == 128 && blk == 128) return launch_attn_kernel<DT, 128, 128>(p, nTq, st);
  if (d == 128 && blk == 64) return launch_attn_kernel<DT, 128, 64>(p, nTq, st);
  if (d == 64 && blk == 128) return launch_attn_kernel<DT, 64, 128>(p, nTq, st);
  return launch_attn_kernel<DT, 64, 64>(p, nTq, st);
}

thrift_status check_attn_args(const void* q, const void* k, const void* v, int dt, int H, int Hkv,
                              int maxlen, int d, int blk, float frac, const void* out,
                              const float* lse) {
  if (!q || !k || !v || !out || !lse) return THRIFT_ERR_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return THRIFT_ERR_ARG;
  if (dt != THRIFT_F16 && dt != THRIFT_BF16) return THRIFT_ERR_ARG;
  if (H <= 0 || Hkv <= 0 || H % Hkv || maxlen <= 0) return THRIFT_ERR_ARG;
  if (!(frac >= 0.0f && frac <= 1.0f)) return THRIFT_ERR_ARG;
  if (d != 64 && d != 128) return THRIFT_ERR_UNSUPPORTED;
  if (blk != 64 && blk != 128) return THRIFT_ERR_UNSUPPORTED;
  if (ceil_div(maxlen, blk) > 512) return THRIFT_ERR_UNSUPPORTED;
  if (H > 65535) return THRIFT_ERR_UNSUPPORTED;
  return THRIFT_OK;
}

// Fixed scratch of block_mean_topk_noalloc.  In host code the array's name
// is only a stand-in; its device address is looked up once per device (with
// that device current) and cached.
constexpr size_t kNoAllocScratchBytes = THRIFT_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];
void* g_noalloc_ptr[kMaxDevices] = {};
std::mutex g_noalloc_mu;

thrift_status noalloc_scratch(void** out) {
  const int dev = current_device();
  if (dev < 0) return THRIFT_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return THRIFT_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return THRIFT_OK;
}

// ---------------------------------------------------------------- decode --

constexpr int kDecMaxSplit = 32;  // CTAs per (sequence, kv head)

bool decode_shape_ok(int H, int Hkv, int d, int blk, thrift_status* why) {
  if (H <= 0 || Hkv <= 0 || H % Hkv) { *why = THRIFT_ERR_ARG; return false; }
  if (d != kDecD || blk != kDecTile || H / Hkv > kDecMaxG || H > 65535 || Hkv > 65535) {
    *why = THRIFT_ERR_UNSUPPORTED;
    return false;
  }
  return true;
}

CacheGeom cache_geom(int B, int Hkv, int capacity) {
  CacheGeom cg;
  cg.B = B;
  cg.Hkv = Hkv;
  cg.ntc = (int)ceil_div(capacity, kDecTile);
  return cg;
}

struct DecWs {
  uint32_t* amax;
  uint8_t* q4;
  uint8_t* q16;
  double* scores;
  uint8_t* mask;
  float* part_o;
  float* part_ml;
  size_t bytes;
};

DecWs carve_decode(void* ws, int B, int H, int Hkv, int capacity) {
  Carve c(ws);
  DecWs w;
  const int64_t nbcap = ceil_div(capacity, kDecTile);
  w.amax = c.take<uint32_t>(16);
  w.q4 = c.take<uint8_t>((size_t)B * Hkv * kDecQ4Bytes);
  w.q16 = c.take<uint8_t>((size_t)B * Hkv * kDecQ16Bytes);
  w.scores = c.take<double>((size_t)B * H * nbcap * 8);
  w.mask = c.take<uint8_t>((size_t)B * H * nbcap);
  w.part_o = c.take<float>((size_t)B * H * 2 * kDecMaxSplit * kDecD * 4);
  w.part_ml = c.take<float>((size_t)B * H * 2 * kDecMaxSplit * 2 * 4);
  w.bytes = (c.off + 1023) & ~(size_t)1023;
  return w;
}

// CTAs per (sequence, kv head).  One CTA fits an SM, so the grid runs in
// waves of sm_count CTAs: take the fewest waves (two at least, when the
// problem has that many tiles) whose last wave is at least 90% full, else
// the fullest; never more than one CTA per key tile, never a CTA with more
// than 512 key tiles (each may appear in both lists).
int decode_splits(int B, int Hkv, int ntc) {
  const int64_t pairs = (int64_t)B * Hkv, sms = sm_count();
  const int lo = std::max(1, (int)ceil_div(ntc, (int64_t)DecLayout::MAX_TILES / 2));
  const int hi = std::max(lo, std::min(kDecMaxSplit, ntc));
  int best = lo;
  double best_eff = -1.0;
  for (int waves = 1; waves <= 16; ++waves) {
    int ns = (int)std::max<int64_t>(1, waves * sms / pairs);
    ns = std::min(std::max(ns, lo), hi);
    const int64_t ctas = pairs * ns;
    const double eff = (double)ctas / (double)(ceil_div(ctas, sms) * sms);
    if (waves >= 2 && eff >= 0.9) return ns;
    if (eff > best_eff + 1e-9) {
      best_eff = eff;
      best = ns;
    }
  }
  return best;
}

template <int DT, bool SS>
void launch_kv_append(const void* kn, const void* vn, const CacheGeom& cg, int max_new,
                      int capacity, const int32_t* cache_len, const int32_t* n_new,
                      const float* kv_scale, uint8_t* cache, cudaStream_t st) {
  kv_append_kernel<DT, SS><<<dim3(max_new, cg.Hkv, cg.B), kDecD, 0, st>>>(
      static_cast<const uint16_t*>(kn), static_cast<const uint16_t*>(vn), cg, max_new, capacity,
      cache_len, n_new, kv_scale, cache);
  const int nv16 = (int)ceil_div(max_new, 16) + 1, nmt = (int)ceil_div(max_new, kDecTile) + 1;
  kv_requant_kernel<DT, SS><<<dim3(nv16 + nmt, cg.Hkv, cg.B), kDecD, 0, st>>>(
      cg, max_new, capacity, cache_len, n_new, kv_scale, nv16, cache);
}

template <int DT, int GC>
thrift_status launch_decode_kernel(const DecParams& p, int B, int Hkv, cudaStream_t st) {
  static DeviceSet attr;
  if (!smem_attr(attn_decode_kernel<DT, GC>, DecLayout::SMEM_ALLOC, attr)) return THRIFT_ERR_CUDA;
  cudaEvent_t* ev = g_timer.enabled ? g_timer.next_pair() : nullptr;
  if (ev) cudaEventRecord(ev[0], st);
  attn_decode_kernel<DT, GC><<<dim3(p.nsplit, Hkv, B), kDecThreads, DecLayout::SMEM_ALLOC, st>>>(p);
  const thrift_status s = launch_status();
  if (ev) cudaEventRecord(ev[1], st);
  return s;
}

template <int DT>
thrift_status decode_impl(const void* q, int B, int H, int Hkv, int capacity, const void* cache,
                          const int32_t* seq_len, const float* kv_scale, float frac, int sink,
                          int recent, int ss, void* out, float* lse, void* ws, cudaStream_t st) {
  const DecWs w = carve_decode(ws, B, H, Hkv, capacity);
  const CacheGeom cg = cache_geom(B, Hkv, capacity);
  const int G = H / Hkv, nbcap = cg.ntc;
  const uint16_t* qp = static_cast<const uint16_t*>(q);
  const int64_t q_elems = (int64_t)B * H * kDecD;
  // small query tensors: reduced inside the image kernel
  const int self_amax = q_elems <= kDecQSelfAmaxMax ? 1 : 0;
  if (!self_amax) {
    if (cudaMemsetAsync(w.amax, 0, 4, st) != cudaSuccess) return THRIFT_ERR_CUDA;
    launch_amax<DT>(q, q_elems / 16, 0, w.amax, st);
  }
  if (ss)
    dec_q_image_kernel<DT, true><<<dim3(Hkv, B), 128, 0, st>>>(qp, H, G, w.amax, self_amax,
                                                               q_elems, w.q4, w.q16);
  else
    dec_q_image_kernel<DT, false><<<dim3(Hkv, B), 128, 0, st>>>(qp, H, G, w.amax, self_amax,
                                                                q_elems, w.q4, w.q16);
  const uint8_t* cp = static_cast<const uint8_t*>(cache);
  {
    static DeviceSet attr;
    if (!smem_attr(dec_scores_kernel<DT>, dec_scores_smem(kDecMaxG), attr)) return THRIFT_ERR_CUDA;
    const int threads = kDecScoreTiles * std::max(G, 4);
    dec_scores_kernel<DT><<<dim3((unsigned)ceil_div(nbcap, kDecScoreTiles), Hkv, B), threads,
                            dec_scores_smem(G), st>>>(qp, H, G, cg, cp, seq_len, capacity, nbcap,
                                                      w.scores);
  }
  const size_t tsm = nbcap <= kTopkCache ? (size_t)nbcap * 8 : 0;
  dec_topk_kernel<<<B * H, kDecTopkThreads, tsm, st>>>(w.scores, seq_len, capacity, H, nbcap,
                                                        frac, sink, recent, w.mask);
  thrift_status s = launch_status();
  if (s != THRIFT_OK) return s;
  DecParams p;
  p.cache = cp;
  p.cg = cg;
  p.q4img = w.q4;
  p.q16img = w.q16;
  p.mask = w.mask;
  p.seq_len = seq_len;
  p.amax_q = w.amax;
  p.kv_scale = kv_scale;
  p.part_o = w.part_o;
  p.part_ml = w.part_ml;
  p.nbcap = nbcap;
  p.capacity = capacity;
  p.H = H;
  p.G = G;
  p.nsplit = decode_splits(B, Hkv, cg.ntc);
  p.scale = (float)(1.4426950408889634 / std::sqrt((double)kDecD));
  if (G <= 4) s = launch_decode_kernel<DT, 4>(p, B, Hkv, st);
  else if (G <= 8) s = launch_decode_kernel<DT, 8>(p, B, Hkv, st);
  else s = launch_decode_kernel<DT, 16>(p, B, Hkv, st);
  if (s != THRIFT_OK) return s;
  dec_combine_kernel<DT><<<B * H, kDecD, 0, st>>>(w.part_o, w.part_ml, 2 * p.nsplit,
                                                  static_cast<uint16_t*>(out), lse);
  return launch_status();
}

// Failure-detection aid: one thread waits, with the library's own bounded
// waits, on something that never completes: an mbarrier that nothing arrives
// on (mode 0) or a global word that nothing writes (mode 1).  The wait gives
// up after limit_ns, sets the device status word and the kernel returns.
static __device__ unsigned g_never_written = 0u;

__global__ void wait_timeout_kernel(int mode, uint64_t limit_ns) {
  __shared__ uint64_t s_bar;
  __shared__ int s_abort;
  if (threadIdx.x == 0) {
    mbar_init(&s_bar, 1);
    s_abort = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x != 0) return;
  if (mode == 0)
    mbar_wait(&s_bar, 0, &s_abort, limit_ns);
  else
    spin_until_geq(&g_never_written, 1u, limit_ns);
}


// ---------------------------------------------------------- Attn-QAT glue --

struct QatWs {
  uint8_t* qt;   // fake-quantised tiles of Q [H][nslot], K, V [Hkv][nslot]
  uint8_t* kt;
  uint8_t* vt;
  uint8_t* dot;  // dO tiles [H][nslot]
  int64_t nslot;
  uint32_t* amax;  // [4]
  float* g;        // [4]
  float* dsum;     // [H, total]
  size_t bytes;
};

QatWs carve_qat(void* base, int64_t total, int nseq, int H, int Hkv, int d) {
  Carve c(base);
  QatWs w;
  w.nslot = qat_nslot(total, nseq);
  const size_t T = qt_tile_bytes(d);
  w.qt = c.take<uint8_t>((size_t)w.nslot * H * T);
  w.kt = c.take<uint8_t>((size_t)w.nslot * Hkv * T);
  w.vt = c.take<uint8_t>((size_t)w.nslot * Hkv * T);
  w.dot = c.take<uint8_t>((size_t)w.nslot * H * T);
  w.amax = c.take<uint32_t>(16);
  w.g = c.take<float>(16);
  w.dsum = c.take<float>((size_t)total * H * 4);
  w.bytes = c.off;
  return w;
}

template <int DT, bool SS, int D>
void qat_fq_tiles(const void* q, const void* k, const void* v, SeqInfo si, int nseq, int maxlen,
                  int H, int Hkv, const QatWs& w, cudaStream_t st) {
  const unsigned nt = (unsigned)ceil_div(maxlen, 128);
  const auto* qp = static_cast<const uint16_t*>(q);
  const auto* kp = static_cast<const uint16_t*>(k);
  const auto* vp = static_cast<const uint16_t*>(v);
  qat_fq_tile_kernel<DT, SS, D, false><<<dim3(nt, H, nseq), kThreads, 0, st>>>(
      qp, si, H, w.nslot, w.amax, w.g, w.qt);
  qat_fq_tile_kernel<DT, SS, D, false><<<dim3(nt, Hkv, nseq), kThreads, 0, st>>>(
      kp, si, Hkv, w.nslot, w.amax + 1, w.g + 1, w.kt);
  qat_fq_tile_kernel<DT, SS, D, true><<<dim3(nt, Hkv, nseq), kThreads, 0, st>>>(
      vp, si, Hkv, w.nslot, w.amax + 2, w.g + 2, w.vt);
}

// Fake-quantised tiles of Q, K, V and their tensor scales.
template <int DT>
thrift_status qat_images(const void* q, const void* k, const void* v, SeqInfo si, int nseq,
                         int64_t total, int maxlen, int H, int Hkv, int d, int ss, const QatWs& w,
                         cudaStream_t st) {
  if (cudaMemsetAsync(w.amax, 0, 16, st) != cudaSuccess) return THRIFT_ERR_CUDA;
  launch_amax<DT>(q, total * H * d / 16, 0, w.amax + 0, st);
  launch_amax<DT>(k, total * Hkv * d / 16, 0, w.amax + 1, st);
  launch_amax<DT>(v, total * Hkv * d / 16, 0, w.amax + 2, st);
  if (d == 128) {
    if (ss) qat_fq_tiles<DT, true, 128>(q, k, v, si, nseq, maxlen, H, Hkv, w, st);
    else qat_fq_tiles<DT, false, 128>(q, k, v, si, nseq, maxlen, H, Hkv, w, st);
  } else {
    if (ss) qat_fq_tiles<DT, true, 64>(q, k, v, si, nseq, maxlen, H, Hkv, w, st);
    else qat_fq_tiles<DT, false, 64>(q, k, v, si, nseq, maxlen, H, Hkv, w, st);
  }
  return launch_status();
}

template <int DT, int D, int BLK>
thrift_status qat_fwd_launch(const QatParams& p, int nseq, int maxlen, cudaStream_t st) {
  static DeviceSet attr;
  const size_t smem = QtFwdLayout<D>::SMEM_ALLOC;
  if (!smem_attr(qat_fwd_kernel<DT, D, BLK>, smem, attr)) return THRIFT_ERR_CUDA;
  const dim3 grid((unsigned)(ceil_div(maxlen, 128) * p.H), nseq);
  cudaEvent_t* ev = g_timer.enabled ? g_timer.next_pair() : nullptr;
  if (ev) cudaEventRecord(ev[0], st);
  qat_fwd_kernel<DT, D, BLK><<<grid, kQtThreads, smem, st>>>(p);
  const thrift_status s = launch_status();
  if (ev) cudaEventRecord(ev[1], st);
  return s;
}

template <int DT, int D, int BLK>
thrift_status qat_bwd_launch(const QatParams& p, const void* dout, int nseq, int maxlen,
                             cudaStream_t st) {
  static DeviceSet attr_kv, attr_q;
  const size_t skv = QtKvLayout<D>::SMEM_ALLOC, sq = QtQLayout<D>::SMEM_ALLOC;
  if (!smem_attr(qat_bwd_kv_kernel<DT, D, BLK>, skv, attr_kv)) return THRIFT_ERR_CUDA;
  if (!smem_attr(qat_bwd_q_kernel<DT, D>, sq, attr_q)) return THRIFT_ERR_CUDA;
  const unsigned nt = (unsigned)ceil_div(maxlen, 128);
  qat_rowdot_tile_kernel<DT, D><<<dim3(nt, p.H, nseq), kThreads, 0, st>>>(
      static_cast<const uint16_t*>(dout), p.out_hp, p.si, p.H, p.total, p.nslot,
      const_cast<float*>(p.dsum), const_cast<uint8_t*>(p.dot));
  cudaEvent_t* ev = g_timer.enabled ? g_timer.next_pair() : nullptr;
  if (ev) cudaEventRecord(ev[0], st);
  qat_bwd_kv_kernel<DT, D, BLK><<<dim3(nt * p.Hkv, nseq), kQtThreads, skv, st>>>(p);
  qat_bwd_q_kernel<DT, D><<<dim3(nt * p.H, nseq), kQtThreads, sq, st>>>(p);
  const thrift_status s = launch_status();
  if (ev) cudaEventRecord(ev[1], st);
  return s;
}

template <int DT>
thrift_status qat_fwd_dispatch(const QatParams& p, int nseq, int maxlen, int d, int blk,
                               cudaStream_t st) {
  if (d == 128 && blk == 128) return qat_fwd_launch<DT, 128, 128>(p, nseq, maxlen, st);
  if (d == 128 && blk == 64) return qat_fwd_launch<DT, 128, 64>(p, nseq, maxlen, st);
  if (d == 64 && blk == 128) return qat_fwd_launch<DT, 64, 128>(p, nseq, maxlen, st);
  return qat_fwd_launch<DT, 64, 64>(p, nseq, maxlen, st);
}

template <int DT>
thrift_status qat_bwd_dispatch(const QatParams& p, const void* dout, int nseq, int maxlen, int d,
                               int blk, cudaStream_t st) {
  if (d == 128 && blk == 128) return qat_bwd_launch<DT, 128, 128>(p, dout, nseq, maxlen, st);
  if (d == 128 && blk == 64) return qat_bwd_launch<DT, 128, 64>(p, dout, nseq, maxlen, st);
  if (d == 64 && blk == 128) return qat_bwd_launch<DT, 64, 128>(p, dout, nseq, maxlen, st);
  return qat_bwd_launch<DT, 64, 64>(p, dout, nseq, maxlen, st);
}

thrift_status check_qat_args(const void* q, const void* k, const void* v, int dt,
                             const int32_t* cu, int nseq, int64_t total, int maxlen, int H,
                             int Hkv, int d, int blk, const void* ws, size_t ws_bytes) {
  if (!q || !k || !v || !cu || !ws) return THRIFT_ERR_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(ws)) return THRIFT_ERR_ARG;
  if (dt != THRIFT_F16 && dt != THRIFT_BF16) return THRIFT_ERR_ARG;
  if (H <= 0 || Hkv <= 0 || H % Hkv || maxlen <= 0 || nseq <= 0 || total <= 0) return THRIFT_ERR_ARG;
  if (d != 64 && d != 128) return THRIFT_ERR_UNSUPPORTED;
  if (blk != 64 && blk != 128) return THRIFT_ERR_UNSUPPORTED;
  if (H > 65535 || nseq > 65535) return THRIFT_ERR_UNSUPPORTED;
  if (ws_bytes < carve_qat(nullptr, total, nseq, H, Hkv, d).bytes) return THRIFT_ERR_ARG;
  return THRIFT_OK;
}

}  // namespace
}  // namespace thrift

using namespace thrift;

extern "C" {

const char* thrift_status_string(int s) {
  switch (s) {
    case THRIFT_OK: return "ok";
    case THRIFT_ERR_ARG: return "invalid argument";
    case THRIFT_ERR_UNSUPPORTED: return "unsupported";
    case THRIFT_ERR_CUDA: return "CUDA error";
    case THRIFT_ERR_TIMEOUT: return "device wait timed out";
    case THRIFT_ERR_SCRATCH: return "problem exceeds the fixed scratch of the no-allocation entry point";
    default: return "unknown status";
  }
}

thrift_status thrift_device_status(int reset) {
  if (cudaDeviceSynchronize() != cudaSuccess) return THRIFT_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int)) != cudaSuccess)
    return THRIFT_ERR_CUDA;
  if (reset) {
    const int z = 0;
    if (cudaMemcpyToSymbol(g_device_status, &z, sizeof(int)) != cudaSuccess)
      return THRIFT_ERR_CUDA;
  }
  return (thrift_status)v;
}

thrift_status thrift_stream_status(void* stream, int reset) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int* word = nullptr;
  if (cudaGetSymbolAddress(reinterpret_cast<void**>(&word), g_device_status) != cudaSuccess)
    return THRIFT_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyAsync(&v, word, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return THRIFT_ERR_CUDA;
  if (reset && cudaMemsetAsync(word, 0, sizeof(int), st) != cudaSuccess) return THRIFT_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return THRIFT_ERR_CUDA;
  return (thrift_status)v;
}

thrift_status thrift_test_wait_timeout(int mode, int limit_us, void* stream) {
  if (mode != 0 && mode != 1) return THRIFT_ERR_ARG;
  if (limit_us < 1 || limit_us > 1000000) return THRIFT_ERR_ARG;
  wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      mode, (uint64_t)limit_us * 1000ull);
  return cudaGetLastError() == cudaSuccess ? THRIFT_OK : THRIFT_ERR_CUDA;
}

thrift_status thrift_kernel_timer_enable(int enable) {
  g_timer.enabled = enable != 0;
  return THRIFT_OK;
}

thrift_status thrift_kernel_timer_read(double* total_ms, int* launches) {
  if (!total_ms || !launches) return THRIFT_ERR_ARG;
  double sum = 0.0;
  for (size_t i = 0; i < g_timer.used; ++i) {
    auto& pr = g_timer.pool[i];
    if (cudaEventSynchronize(pr.second) != cudaSuccess) return THRIFT_ERR_CUDA;
    float ms = 0.0f;
    if (cudaEventElapsedTime(&ms, pr.first, pr.second) != cudaSuccess) return THRIFT_ERR_CUDA;
    sum += ms;
  }
  *total_ms = sum;
  *launches = (int)g_timer.used;
  g_timer.used = 0;
  return THRIFT_OK;
}

size_t nvfp4_quantize_workspace_size(void) { return kQuantWsBytes; }

thrift_status nvfp4_quantize(const void* x, thrift_dtype dt, int64_t rows, int64_t cols,
                             int use_scalesearch, int use_hadamard, int tensor_scale_given,
                             uint8_t* codes, uint8_t* scales, float* tensor_scale,
                             void* workspace, size_t ws_bytes, void* stream) {
  if (rows < 0 || cols <= 0 || cols % 16 || cols > 4096) return THRIFT_ERR_ARG;
  if (dt != THRIFT_F16 && dt != THRIFT_BF16) return THRIFT_ERR_ARG;
  if (!tensor_scale || !workspace || ws_bytes < nvfp4_quantize_workspace_size())
    return THRIFT_ERR_ARG;
  if (use_hadamard && cols != 64 && cols != 128) return THRIFT_ERR_UNSUPPORTED;
  if (rows == 0) return THRIFT_OK;
  if (!x || !codes || !scales || !aligned16(x) || !aligned16(workspace) ||
      (reinterpret_cast<uintptr_t>(codes) & 7))
    return THRIFT_ERR_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t* wsw = static_cast<uint32_t*>(workspace);
  const int64_t nb = rows * cols / 16;
  const int G = use_hadamard ? (int)(cols / 16) : 0;
  if (dt == THRIFT_BF16)
    return launch_quantize<1>(x, nb, G, use_scalesearch != 0, wsw, tensor_scale,
                              tensor_scale_given, codes, scales, st);
  return launch_quantize<0>(x, nb, G, use_scalesearch != 0, wsw, tensor_scale,
                            tensor_scale_given, codes, scales, st);
}

thrift_status nvfp4_quantize_colblocks(const void* x, thrift_dtype dt, int64_t rows,
                                       int64_t cols, int use_scalesearch,
                                       int tensor_scale_given, uint8_t* codes,
                                       uint8_t* scales, float* tensor_scale, void* workspace,
                                       size_t ws_bytes, void* stream) {
  if (rows < 0 || cols <= 0 || rows % 16) return THRIFT_ERR_ARG;
  if (dt != THRIFT_F16 && dt != THRIFT_BF16) return THRIFT_ERR_ARG;
  if (!tensor_scale || !workspace || ws_bytes < nvfp4_quantize_workspace_size())
    return THRIFT_ERR_ARG;
  if (rows == 0) return THRIFT_OK;
  if (!x || !codes || !scales || !aligned16(x) || !aligned16(workspace) ||
      (reinterpret_cast<uintptr_t>(codes) & 7) || ((rows / 2) % 8))
    return THRIFT_ERR_ARG;
  if ((rows * cols) % 16) return THRIFT_ERR_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const uint16_t* xp = static_cast<const uint16_t*>(x);
  float* partial = quant_partials(static_cast<uint32_t*>(workspace));
  int np = 0;
  thrift_status s = THRIFT_OK;
  if (!tensor_scale_given) {
    np = dt == THRIFT_BF16 ? launch_amax_partial<1, 0>(xp, rows * cols / 16, partial, st, &s)
                           : launch_amax_partial<0, 0>(xp, rows * cols / 16, partial, st, &s);
    if (s != THRIFT_OK) return s;
  }
  // one thread per (row block, column): kKPT * threads items per CTA
  const int64_t items = (rows / 16) * cols * kKPT;
  const float* pc = partial;
  cudaError_t e;
  if (dt == THRIFT_BF16) {
    if (use_scalesearch)
      e = launch_pdl(quant_cols_kernel<1, true>, stream_grid(quant_cols_kernel<1, true>, items),
                     kThreads, st, xp, rows, cols, pc, np, tensor_scale, tensor_scale_given, codes,
                     scales);
    else
      e = launch_pdl(quant_cols_kernel<1, false>, stream_grid(quant_cols_kernel<1, false>, items),
                     kThreads, st, xp, rows, cols, pc, np, tensor_scale, tensor_scale_given, codes,
                     scales);
  } else {
    if (use_scalesearch)
      e = launch_pdl(quant_cols_kernel<0, true>, stream_grid(quant_cols_kernel<0, true>, items),
                     kThreads, st, xp, rows, cols, pc, np, tensor_scale, tensor_scale_given, codes,
                     scales);
    else
      e = launch_pdl(quant_cols_kernel<0, false>, stream_grid(quant_cols_kernel<0, false>, items),
                     kThreads, st, xp, rows, cols, pc, np, tensor_scale, tensor_scale_given, codes,
                     scales);
  }
  return e == cudaSuccess ? THRIFT_OK : THRIFT_ERR_CUDA;
}

size_t block_mean_topk_workspace_size(int B, int H, int Hkv, int N, int d, int blk) {
  if (B <= 0 || H <= 0 || Hkv <= 0 || N <= 0 || d <= 0 || blk <= 0) return 0;
  const size_t nB = (size_t)ceil_div(N, blk);
  return 3 * 1024 + (size_t)B * H * nB * d * 8 + (size_t)B * Hkv * nB * d * 8 +
         (size_t)B * H * nB * nB * 8;
}

thrift_status block_mean_topk(const void* q, const void* k, thrift_dtype dt, int B, int H,
                              int Hkv, int N, int d, int blk, int causal, float topk_frac,
                              int sink_blocks, int recent_blocks, uint8_t* mask,
                              void* workspace, size_t ws_bytes, void* stream) {
  if (!q || !k || !mask || !workspace) return THRIFT_ERR_ARG;
  if (sink_blocks < 0 || recent_blocks < 0) return THRIFT_ERR_ARG;
  if (dt != THRIFT_F16 && dt != THRIFT_BF16) return THRIFT_ERR_ARG;
  if (B <= 0 || H <= 0 || Hkv <= 0 || H % Hkv || N <= 0) return THRIFT_ERR_ARG;
  if (!(topk_frac >= 0.0f && topk_frac <= 1.0f)) return THRIFT_ERR_ARG;
  if (d != 64 && d != 128) return THRIFT_ERR_UNSUPPORTED;
  if (blk != 64 && blk != 128) return THRIFT_ERR_UNSUPPORTED;
  if (ceil_div(N, blk) > 512) return THRIFT_ERR_UNSUPPORTED;
  if (ws_bytes < block_mean_topk_workspace_size(B, H, Hkv, N, d, blk)) return THRIFT_ERR_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int nB = (int)ceil_div(N, blk);
  Carve c(workspace);
  double* mq = c.take<double>((size_t)B * H * nB * d * 8);
  double* mk = c.take<double>((size_t)B * Hkv * nB * d * 8);
  double* sc = c.take<double>((size_t)B * H * nB * nB * 8);
  SeqInfo si{nullptr, N};
  const uint16_t* qp = static_cast<const uint16_t*>(q);
  const uint16_t* kp = static_cast<const uint16_t*>(k);
  if (dt == THRIFT_BF16) {
    block_means_kernel<1><<<grid_for((int64_t)B * H * nB * d), kThreads, 0, st>>>(qp, si, B, H, d, blk, nB, mq);
    block_means_kernel<1><<<grid_for((int64_t)B * Hkv * nB * d), kThreads, 0, st>>>(kp, si, B, Hkv, d, blk, nB, mk);
  } else {
    block_means_kernel<0><<<grid_for((int64_t)B * H * nB * d), kThreads, 0, st>>>(qp, si, B, H, d, blk, nB, mq);
    block_means_kernel<0><<<grid_for((int64_t)B * Hkv * nB * d), kThreads, 0, st>>>(kp, si, B, Hkv, d, blk, nB, mk);
  }
  pair_scores_kernel<<<pair_scores_grid(B, H, nB), kThreads, pair_scores_smem(nB), st>>>(
      mq, mk, si, B, H, Hkv, d, blk, nB, causal, sc);
  return launch_topk(sc, si, B, H, blk, nB, causal, topk_frac, sink_blocks, recent_blocks, mask,
                     st);
}

thrift_status block_mean_topk_noalloc(const void* q, const void* k, thrift_dtype dt, int B,
                                      int H, int Hkv, int N, int d, int blk, int causal,
                                      float topk_frac, int sink_blocks, int recent_blocks,
                                      uint8_t* mask, void* stream) {
  if (!q || !k || !mask) return THRIFT_ERR_ARG;
  const size_t need = block_mean_topk_workspace_size(B, H, Hkv, N, d, blk);
  if (need == 0) return THRIFT_ERR_ARG;
  if (need > kNoAllocScratchBytes) return THRIFT_ERR_SCRATCH;
  void* scratch = nullptr;
  const thrift_status s = noalloc_scratch(&scratch);
  if (s != THRIFT_OK) return s;
  return block_mean_topk(q, k, dt, B, H, Hkv, N, d, blk, causal, topk_frac, sink_blocks,
                         recent_blocks, mask, scratch, kNoAllocScratchBytes, stream);
}

size_t thrift_attn_workspace_size(int B, int H, int Hkv, int N, int d, int blk) {
  if (B <= 0 || H <= 0 || Hkv <= 0 || N <= 0 || (d != 64 && d != 128) ||
      (blk != 64 && blk != 128))
    return 0;
  return carve_attn(nullptr, B, N, H, Hkv, d, blk).bytes;
}

thrift_status thrift_attn_fwd(const void* q, const void* k, const void* v, thrift_dtype dt,
                              int B, int H, int Hkv, int N, int d, int blk, int causal,
                              float topk_frac, int sink_blocks, int recent_blocks,
                              int use_scalesearch, int use_hadamard, int smooth_k, void* out,
                              float* lse, void* workspace, size_t ws_bytes, void* stream) {
  thrift_status s = check_attn_args(q, k, v, dt, H, Hkv, N, d, blk, topk_frac, out, lse);
  if (sink_blocks < 0 || recent_blocks < 0) return THRIFT_ERR_ARG;
  if (s != THRIFT_OK) return s;
  if (smooth_k && use_hadamard) return THRIFT_ERR_UNSUPPORTED;
  if (B <= 0 || !workspace || !aligned16(workspace)) return THRIFT_ERR_ARG;
  if (ws_bytes < thrift_attn_workspace_size(B, H, Hkv, N, d, blk)) return THRIFT_ERR_ARG;
  if ((int64_t)B * ceil_div(N, 128) > 0x7FFFFFFF || B > 65535) return THRIFT_ERR_UNSUPPORTED;
  SeqInfo si{nullptr, N};
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t total = (int64_t)B * N;
  if (dt == THRIFT_BF16)
    return attn_impl<1>(q, k, v, si, B, total, N, H, Hkv, d, blk, causal, topk_frac,
                        sink_blocks, recent_blocks, use_scalesearch, use_hadamard, smooth_k, out,
                        lse, 0, workspace, st);
  return attn_impl<0>(q, k, v, si, B, total, N, H, Hkv, d, blk, causal, topk_frac, sink_blocks,
                      recent_blocks, use_scalesearch, use_hadamard, smooth_k, out, lse, 0,
                      workspace, st);
}

size_t thrift_attn_workspace_mask_offset(int nseq, int max_seqlen, int H, int Hkv, int d,
                                         int blk) {
  if (nseq <= 0 || max_seqlen <= 0 || H <= 0 || Hkv <= 0 || H % Hkv || (d != 64 && d != 128) ||
      (blk != 64 && blk != 128))
    return 0;
  const AttnWs w = carve_attn(nullptr, nseq, max_seqlen, H, Hkv, d, blk);
  return (size_t)reinterpret_cast<uintptr_t>(w.mask);
}

size_t thrift_attn_varlen_workspace_size(int nseq, int64_t total, int max_seqlen, int H,
                                         int Hkv, int d, int blk) {
  (void)total;
  if (nseq <= 0 || H <= 0 || Hkv <= 0 || max_seqlen <= 0 || (d != 64 && d != 128) ||
      (blk != 64 && blk != 128))
    return 0;
  return carve_attn(nullptr, nseq, max_seqlen, H, Hkv, d, blk).bytes;
}

thrift_status thrift_attn_fwd_varlen(const void* q, const void* k, const void* v,
                                     thrift_dtype dt, const int32_t* cu_seqlens, int nseq,
                                     int64_t total, int max_seqlen, int H, int Hkv, int d,
                                     int blk, int causal, float topk_frac, int sink_blocks,
                                     int recent_blocks, int use_scalesearch, int use_hadamard,
                                     int smooth_k, void* out, float* lse, void* workspace,
                                     size_t ws_bytes, void* stream) {
  thrift_status s = check_attn_args(q, k, v, dt, H, Hkv, max_seqlen, d, blk, topk_frac, out, lse);
  if (sink_blocks < 0 || recent_blocks < 0) return THRIFT_ERR_ARG;
  if (s != THRIFT_OK) return s;
  if (smooth_k && use_hadamard) return THRIFT_ERR_UNSUPPORTED;
  if (!cu_seqlens || nseq <= 0 || nseq > 65535 || total <= 0 || !workspace ||
      !aligned16(workspace))
    return THRIFT_ERR_ARG;
  if (ws_bytes < thrift_attn_varlen_workspace_size(nseq, total, max_seqlen, H, Hkv, d, blk))
    return THRIFT_ERR_ARG;
  SeqInfo si{cu_seqlens, 0};
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dt == THRIFT_BF16)
    return attn_impl<1>(q, k, v, si, nseq, total, max_seqlen, H, Hkv, d, blk, causal,
                        topk_frac, sink_blocks, recent_blocks, use_scalesearch, use_hadamard,
                        smooth_k, out, lse, 1, workspace, st);
  return attn_impl<0>(q, k, v, si, nseq, total, max_seqlen, H, Hkv, d, blk, causal, topk_frac,
                      sink_blocks, recent_blocks, use_scalesearch, use_hadamard, smooth_k, out,
                      lse, 1, workspace, st);
}

thrift_status thrift_attn_absmax(const void* q, const void* k, const void* v, thrift_dtype dt,
                                 const int32_t* cu_seqlens, int nseq, int64_t total,
                                 int max_seqlen, int H, int Hkv, int d, int blk, int use_hadamard,
                                 int smooth_k, float* amax_out, void* workspace, size_t ws_bytes,
                                 void* stream) {
  if (!q || !k || !v || !amax_out || !workspace || !aligned16(workspace)) return THRIFT_ERR_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v)) return THRIFT_ERR_ARG;
  if (dt != THRIFT_F16 && dt != THRIFT_BF16) return THRIFT_ERR_ARG;
  if (H <= 0 || Hkv <= 0 || H % Hkv || nseq <= 0 || max_seqlen <= 0 || total <= 0)
    return THRIFT_ERR_ARG;
  if (d != 64 && d != 128) return THRIFT_ERR_UNSUPPORTED;
  if (blk != 64 && blk != 128) return THRIFT_ERR_UNSUPPORTED;
  if (smooth_k && use_hadamard) return THRIFT_ERR_UNSUPPORTED;
  if (!cu_seqlens && total != (int64_t)nseq * max_seqlen) return THRIFT_ERR_ARG;
  if (ws_bytes < thrift_attn_varlen_workspace_size(nseq, total, max_seqlen, H, Hkv, d, blk))
    return THRIFT_ERR_ARG;
  const SeqInfo si{cu_seqlens, cu_seqlens ? 0 : max_seqlen};
  const AttnWs w = carve_attn(workspace, nseq, max_seqlen, H, Hkv, d, blk);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t* a = reinterpret_cast<uint32_t*>(amax_out);
  if (dt == THRIFT_BF16)
    return attn_absmax<1>(q, k, v, si, nseq, total, max_seqlen, H, Hkv, d, use_hadamard,
                          smooth_k, w, a, st);
  return attn_absmax<0>(q, k, v, si, nseq, total, max_seqlen, H, Hkv, d, use_hadamard, smooth_k,
                        w, a, st);
}

thrift_status thrift_attn_fwd_absmax(const void* q, const void* k, const void* v,
                                     thrift_dtype dt, const int32_t* cu_seqlens, int nseq,
                                     int64_t total, int max_seqlen, int H, int Hkv, int d,
                                     int blk, int causal, float topk_frac, int sink_blocks,
                                     int recent_blocks, int use_scalesearch, int use_hadamard,
                                     int smooth_k, const float* amax_in, void* out, float* lse,
                                     void* workspace, size_t ws_bytes, void* stream) {
  thrift_status s = check_attn_args(q, k, v, dt, H, Hkv, max_seqlen, d, blk, topk_frac, out, lse);
  if (s != THRIFT_OK) return s;
  if (sink_blocks < 0 || recent_blocks < 0 || !amax_in) return THRIFT_ERR_ARG;
  if (smooth_k && use_hadamard) return THRIFT_ERR_UNSUPPORTED;
  if (nseq <= 0 || nseq > 65535 || total <= 0 || !workspace || !aligned16(workspace))
    return THRIFT_ERR_ARG;
  if (!cu_seqlens && total != (int64_t)nseq * max_seqlen) return THRIFT_ERR_ARG;
  if (ws_bytes < thrift_attn_varlen_workspace_size(nseq, total, max_seqlen, H, Hkv, d, blk))
    return THRIFT_ERR_ARG;
  const SeqInfo si{cu_seqlens, cu_seqlens ? 0 : max_seqlen};
  const int lse_varlen = cu_seqlens ? 1 : 0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dt == THRIFT_BF16)
    return attn_impl<1>(q, k, v, si, nseq, total, max_seqlen, H, Hkv, d, blk, causal, topk_frac,
                        sink_blocks, recent_blocks, use_scalesearch, use_hadamard, smooth_k, out,
                        lse, lse_varlen, workspace, st, amax_in);
  return attn_impl<0>(q, k, v, si, nseq, total, max_seqlen, H, Hkv, d, blk, causal, topk_frac,
                      sink_blocks, recent_blocks, use_scalesearch, use_hadamard, smooth_k, out,
                      lse, lse_varlen, workspace, st, amax_in);
}

size_t thrift_kv_cache_size(int B, int Hkv, int capacity, int d, int blk) {
  thrift_status why;
  if (B <= 0 || capacity <= 0 || !decode_shape_ok(Hkv, Hkv, d, blk, &why)) return 0;
  return (size_t)cache_geom(B, Hkv, capacity).bytes();
}

thrift_status thrift_kv_cache_append(const void* k_new, const void* v_new, thrift_dtype dt, int B,
                                     int Hkv, int d, int blk, int capacity,
                                     const int32_t* cache_len, const int32_t* n_new, int max_new,
                                     const float* kv_scale, int use_scalesearch, void* cache,
                                     size_t cache_bytes, void* stream) {
  thrift_status why;
  if (!decode_shape_ok(Hkv, Hkv, d, blk, &why)) return why;
  if (dt != THRIFT_F16 && dt != THRIFT_BF16) return THRIFT_ERR_ARG;
  if (B <= 0 || B > 65535 || capacity <= 0 || max_new < 0) return THRIFT_ERR_ARG;
  if (!cache_len || !n_new || !kv_scale || !cache || !aligned16(cache)) return THRIFT_ERR_ARG;
  if (cache_bytes < thrift_kv_cache_size(B, Hkv, capacity, d, blk)) return THRIFT_ERR_ARG;
  if (max_new == 0) return THRIFT_OK;
  if (!k_new || !v_new || !aligned16(k_new) || !aligned16(v_new)) return THRIFT_ERR_ARG;
  if (max_new > 0x7FFFFFFF / 2) return THRIFT_ERR_UNSUPPORTED;
  const CacheGeom cg = cache_geom(B, Hkv, capacity);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* cp = static_cast<uint8_t*>(cache);
  const bool ss = use_scalesearch != 0;
  if (dt == THRIFT_BF16) {
    if (ss) launch_kv_append<1, true>(k_new, v_new, cg, max_new, capacity, cache_len, n_new, kv_scale, cp, st);
    else launch_kv_append<1, false>(k_new, v_new, cg, max_new, capacity, cache_len, n_new, kv_scale, cp, st);
  } else {
    if (ss) launch_kv_append<0, true>(k_new, v_new, cg, max_new, capacity, cache_len, n_new, kv_scale, cp, st);
    else launch_kv_append<0, false>(k_new, v_new, cg, max_new, capacity, cache_len, n_new, kv_scale, cp, st);
  }
  return launch_status();
}

size_t thrift_attn_decode_workspace_size(int B, int H, int Hkv, int capacity, int d, int blk) {
  thrift_status why;
  if (B <= 0 || capacity <= 0 || !decode_shape_ok(H, Hkv, d, blk, &why)) return 0;
  return carve_decode(nullptr, B, H, Hkv, capacity).bytes;
}

size_t thrift_attn_decode_mask_offset(int B, int H, int Hkv, int capacity, int d, int blk) {
  thrift_status why;
  if (B <= 0 || capacity <= 0 || !decode_shape_ok(H, Hkv, d, blk, &why)) return 0;
  return (size_t)reinterpret_cast<uintptr_t>(carve_decode(nullptr, B, H, Hkv, capacity).mask);
}

thrift_status thrift_attn_decode(const void* q, thrift_dtype dt, int B, int H, int Hkv, int d,
                                 int blk, int capacity, const void* cache, size_t cache_bytes,
                                 const int32_t* seq_len, const float* kv_scale, float topk_frac,
                                 int sink_blocks, int recent_blocks, int use_scalesearch,
                                 void* out, float* lse, void* workspace, size_t ws_bytes,
                                 void* stream) {
  thrift_status why;
  if (!decode_shape_ok(H, Hkv, d, blk, &why)) return why;
  if (dt != THRIFT_F16 && dt != THRIFT_BF16) return THRIFT_ERR_ARG;
  if (B <= 0 || B > 65535 || capacity <= 0) return THRIFT_ERR_ARG;
  if (!(topk_frac >= 0.0f && topk_frac <= 1.0f) || sink_blocks < 0 || recent_blocks < 0)
    return THRIFT_ERR_ARG;
  if (!q || !cache || !seq_len || !kv_scale || !out || !lse || !workspace) return THRIFT_ERR_ARG;
  if (!aligned16(q) || !aligned16(cache) || !aligned16(out) || !aligned16(workspace))
    return THRIFT_ERR_ARG;
  if (cache_bytes < thrift_kv_cache_size(B, Hkv, capacity, d, blk)) return THRIFT_ERR_ARG;
  if (ws_bytes < thrift_attn_decode_workspace_size(B, H, Hkv, capacity, d, blk))
    return THRIFT_ERR_ARG;
  if (ceil_div(cache_geom(B, Hkv, capacity).ntc, (int64_t)DecLayout::MAX_TILES / 2) > kDecMaxSplit)
    return THRIFT_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dt == THRIFT_BF16)
    return decode_impl<1>(q, B, H, Hkv, capacity, cache, seq_len, kv_scale, topk_frac,
                          sink_blocks, recent_blocks, use_scalesearch, out, lse, workspace, st);
  return decode_impl<0>(q, B, H, Hkv, capacity, cache, seq_len, kv_scale, topk_frac, sink_blocks,
                        recent_blocks, use_scalesearch, out, lse, workspace, st);
}

// ------------------------------------------------------------ Attn-QAT --

size_t thrift_qat_workspace_size(int64_t total, int nseq, int H, int Hkv, int d) {
  if (total <= 0 || nseq <= 0 || H <= 0 || Hkv <= 0 || (d != 64 && d != 128)) return 0;
  return carve_qat(nullptr, total, nseq, H, Hkv, d).bytes;
}

thrift_status thrift_qat_fwd_varlen(const void* q, const void* k, const void* v, thrift_dtype dt,
                                    const int32_t* cu_seqlens, int nseq, int64_t total,
                                    int max_seqlen, int H, int Hkv, int d, int blk, int causal,
                                    int use_scalesearch, void* out, float* out_hp, float* lse,
                                    void* workspace, size_t ws_bytes, void* stream) {
  thrift_status s = check_qat_args(q, k, v, dt, cu_seqlens, nseq, total, max_seqlen, H, Hkv, d,
                                   blk, workspace, ws_bytes);
  if (s != THRIFT_OK) return s;
  if (!out || !out_hp || !lse || !aligned16(out) || !aligned16(out_hp)) return THRIFT_ERR_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const QatWs w = carve_qat(workspace, total, nseq, H, Hkv, d);
  const SeqInfo si{cu_seqlens, 0};
  QatParams p{};
  p.qt = w.qt;
  p.kt = w.kt;
  p.vt = w.vt;
  p.nslot = w.nslot;
  p.g = w.g;
  p.si = si;
  p.H = H;
  p.Hkv = Hkv;
  p.total = total;
  p.causal = causal ? 1 : 0;
  p.sc = (float)(1.0 / std::sqrt((double)d));
  p.out = static_cast<uint16_t*>(out);
  p.out_hp = out_hp;
  p.lse = lse;
  if (dt == THRIFT_BF16) {
    s = qat_images<1>(q, k, v, si, nseq, total, max_seqlen, H, Hkv, d, use_scalesearch, w, st);
    return s != THRIFT_OK ? s : qat_fwd_dispatch<1>(p, nseq, max_seqlen, d, blk, st);
  }
  s = qat_images<0>(q, k, v, si, nseq, total, max_seqlen, H, Hkv, d, use_scalesearch, w, st);
  return s != THRIFT_OK ? s : qat_fwd_dispatch<0>(p, nseq, max_seqlen, d, blk, st);
}

thrift_status thrift_qat_bwd_varlen(const void* q, const void* k, const void* v, const void* dout,
                                    thrift_dtype dt, const int32_t* cu_seqlens, int nseq,
                                    int64_t total, int max_seqlen, int H, int Hkv, int d, int blk,
                                    int causal, int use_scalesearch, int reuse_images,
                                    const float* out_hp, const float* lse, float* dq, float* dk,
                                    float* dv, void* workspace, size_t ws_bytes, void* stream) {
  thrift_status s = check_qat_args(q, k, v, dt, cu_seqlens, nseq, total, max_seqlen, H, Hkv, d,
                                   blk, workspace, ws_bytes);
  if (s != THRIFT_OK) return s;
  if (!dout || !out_hp || !lse || !dq || !dk || !dv) return THRIFT_ERR_ARG;
  if (!aligned16(dout) || !aligned16(out_hp) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return THRIFT_ERR_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const QatWs w = carve_qat(workspace, total, nseq, H, Hkv, d);
  const SeqInfo si{cu_seqlens, 0};
  QatParams p{};
  p.qt = w.qt;
  p.kt = w.kt;
  p.vt = w.vt;
  p.dot = w.dot;
  p.nslot = w.nslot;
  p.g = w.g;
  p.si = si;
  p.H = H;
  p.Hkv = Hkv;
  p.total = total;
  p.causal = causal ? 1 : 0;
  p.sc = (float)(1.0 / std::sqrt((double)d));
  p.out_hp = const_cast<float*>(out_hp);
  p.lse = const_cast<float*>(lse);
  p.dsum = w.dsum;
  p.dq = dq;
  p.dk = dk;
  p.dv = dv;
  if (dt == THRIFT_BF16) {
    if (!reuse_images)
      s = qat_images<1>(q, k, v, si, nseq, total, max_seqlen, H, Hkv, d, use_scalesearch, w, st);
    return s != THRIFT_OK ? s : qat_bwd_dispatch<1>(p, dout, nseq, max_seqlen, d, blk, st);
  }
  if (!reuse_images)
    s = qat_images<0>(q, k, v, si, nseq, total, max_seqlen, H, Hkv, d, use_scalesearch, w, st);
  return s != THRIFT_OK ? s : qat_bwd_dispatch<0>(p, dout, nseq, max_seqlen, d, blk, st);
}

}  // extern "C"
