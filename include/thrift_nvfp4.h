/*
 * thrift_nvfp4.h -- C ABI of the B200 (sm_100a) NVFP4 attention library.
 *
 * Block-scaled 4-bit (NVFP4) attention forward with selective FP16 block
 * pairs.  Sources of the method (web pages):
 *   [AQ] "Attn-QAT: 4-Bit Attention With Quantization-Aware Training",
 *        Resumo tecnico 1 (E2M1: 15 distinct values).
 *   [TA] "ThriftAttention", Metodologia: step 1 (block-mean scores
 *        S^_ij = qbar_i . kbar_j, top-k pairs), step 2 (FP16 path for the
 *        selected pairs, NVFP4 for the rest, FlashAttention-2 online softmax
 *        merge, two-level quantisation of P), and the kernel paragraph that
 *        follows (FP4 blocks first, then the FP16 helper; tiles with no
 *        selected pair skip the FP16 path).
 *   [SS] "Busca tus Escalas de Punto Flotante por Bloques": Declaracion del
 *        Problema (NVFP4, E4M3 block scale), ScaleSearch Mecanismo and
 *        Estrategia de Busqueda (s = round(||x||_inf/6); offsets f in [-2,6]
 *        on the scale's bit pattern; least block MSE), ScaleSearchAttention
 *        (Hadamard rotation of Q/K; QK^T and PV on FP4 tensor cores with FP32
 *        accumulation).
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller; the
 *     library allocates no device memory.  Scratch lives in the caller's
 *     `workspace` (device memory of at least the size the matching
 *     *_workspace_size function returns, 256-byte aligned).
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream).  Arguments are validated on the host before any
 *     launch; a bad argument returns THRIFT_ERR_ARG / THRIFT_ERR_UNSUPPORTED
 *     and launches nothing.  A failed launch returns THRIFT_ERR_CUDA.
 *   - Device-side waits are bounded; a wait that gives up sets the device
 *     status word read by thrift_device_status() and the kernel returns.
 *   - 16-bit inputs: fp16 or bf16 (thrift_dtype).  Pointers must be 16-byte
 *     aligned.
 *   - FP4 codes are E2M1, two per byte: element 2c in the low nibble, 2c+1
 *     in the high nibble.  Block scales are UE4M3 bytes (bias 7, max 0x7E =
 *     448).  The per-tensor FP32 scale is g = amax/2688 (g = 1 for an all-zero
 *     tensor); dequantised value = e2m1(code) * ue4m3(scale) * g.
 */
#ifndef THRIFT_NVFP4_H
#define THRIFT_NVFP4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  THRIFT_OK = 0,
  THRIFT_ERR_ARG = -1,          /* bad pointer, size or flag */
  THRIFT_ERR_UNSUPPORTED = -2,  /* valid request the library does not handle */
  THRIFT_ERR_CUDA = -3,         /* a CUDA runtime call failed */
  THRIFT_ERR_TIMEOUT = -4,      /* a device-side wait gave up */
  THRIFT_ERR_SCRATCH = -5       /* problem too large for a fixed scratch area */
} thrift_status;

typedef enum { THRIFT_F16 = 0, THRIFT_BF16 = 1 } thrift_dtype;

/* Human-readable name of a status code (static string). */
const char* thrift_status_string(int status);

/*
 * Synchronises the calling thread with the current device and returns the
 * device status word: THRIFT_OK, or THRIFT_ERR_TIMEOUT if any kernel of this
 * library gave up on a bounded wait since the last reset.  reset != 0 clears
 * the word.  Returns THRIFT_ERR_CUDA if the synchronisation itself fails.
 */
thrift_status thrift_device_status(int reset);

/*
 * Per-stream form of thrift_device_status: waits only for the work already
 * queued on `stream` (cudaStreamSynchronize), then reads the device status
 * word through that stream, and with reset != 0 clears it (also on that
 * stream, before returning).  Other streams keep running.  The word itself
 * is shared by every stream of the current device: a timeout raised by a
 * kernel on another stream shows here too once it has happened.  Returns
 * THRIFT_ERR_CUDA if a CUDA call fails.
 */
thrift_status thrift_stream_status(void* stream, int reset);

/* ------------------------------------------------------------ quantiser --
 * [SS] ScaleSearch; [AQ] E2M1.  Quantises x [rows, cols] (row-major, 16-bit)
 * to NVFP4 with 16-element blocks along cols.
 *   codes  [rows, cols/2] uint8 out;   scales [rows, cols/16] uint8 out.
 *   tensor_scale: one float; read when tensor_scale_given != 0, else written
 *     (g = amax/2688 over the whole, possibly rotated, tensor).
 *   use_scalesearch: per block, among the bytes S0+f, f in {0,-2,-1,1,...,6}
 *     that stay in 1..126, keep the first one of least error
 *     (sum over the block, in order, of (t-q)^2 by fmaf) * S^2, where
 *     t = x * (1/(S*g)) and q is t rounded to the E2M1 grid.
 *   use_hadamard: rotate every row by the unnormalised Sylvester-Hadamard
 *     transform first (cols must be 64 or 128).
 * Requirements: rows >= 0, cols % 16 == 0, cols <= 4096.
 * Workspace: nvfp4_quantize_workspace_size() bytes, 16-byte aligned, no
 *   initial contents required (a call that computes the tensor scale writes
 *   every per-CTA maximum it then reads); one buffer serves any number of
 *   calls issued in stream order.  Calls that overlap on the GPU must not
 *   share a workspace.  nvfp4_quantize_colblocks takes the same workspace.
 * Execution: with the tensor scale computed, a partial-absmax kernel (one
 *   maximum per CTA into the workspace) and a quantise kernel that reduces
 *   those maxima to g and quantises (x read twice: from L2 the second time
 *   when it fits); with the scale given, the quantise kernel alone.  Both are
 *   launched with programmatic dependent launch: a kernel's first input loads
 *   may run while the previous kernel of the stream finishes, and whatever
 *   that kernel may write (the maxima, a given tensor scale, the outputs) is
 *   touched only after it has completed.  Hence x must already be final when
 *   the previous kernel of the stream lets its dependents start: x must not
 *   alias a previous quantiser call's codes, scales or tensor scale, and a
 *   predecessor that triggers its dependents early itself
 *   (griddepcontrol.launch_dependents) must have written x before it does;
 *   every other predecessor is waited for in full.
 */
size_t nvfp4_quantize_workspace_size(void);
thrift_status nvfp4_quantize(const void* x, thrift_dtype dt, int64_t rows, int64_t cols,
                             int use_scalesearch, int use_hadamard, int tensor_scale_given,
                             uint8_t* codes, uint8_t* scales, float* tensor_scale,
                             void* workspace, size_t ws_bytes, void* stream);

/* Same, with 16-element blocks along ROWS (the token axis of V):
 *   codes [cols, rows/2], scales [cols, rows/16].  rows % 16 == 0.
 * No Hadamard option (the rotation applies to Q and K only). */
thrift_status nvfp4_quantize_colblocks(const void* x, thrift_dtype dt, int64_t rows,
                                       int64_t cols, int use_scalesearch,
                                       int tensor_scale_given, uint8_t* codes,
                                       uint8_t* scales, float* tensor_scale, void* workspace,
                                       size_t ws_bytes, void* stream);

/* ------------------------------------------------------- block selection --
 * [TA] Metodologia step 1.  q [B,N,H,d], k [B,N,Hkv,d] 16-bit.  Blocks of
 * blk tokens from the sequence start (the last may be partial).  Block means
 * in fp64 (sequential sum in token order / count); scores by a sequential
 * fp64 fma over channels; per (batch, head) the k = ceil(frac*n_valid - 1e-9)
 * best valid pairs are selected (causal: j <= i), ties to the lower i*nB+j.
 *   mask [B, H, nB, nB] uint8 out, 1 = FP16 pair.
 * sink_blocks, recent_blocks >= 0 (0, 0: off): ScaleSearchAttention's
 * sink-aware mixed precision.  For every query block i the first
 * sink_blocks key blocks and the recent_blocks most recent key blocks i can
 * see (causal: i - recent_blocks < j <= i; non-causal: the last
 * recent_blocks blocks) are FP16 pairs too, added to the top-k pairs (whose
 * count k is unchanged).
 * Requirements: H % Hkv == 0, d in {64,128}, blk in {64,128}, 0<=frac<=1,
 * nB = ceil(N/blk) <= 512.
 */
size_t block_mean_topk_workspace_size(int B, int H, int Hkv, int N, int d, int blk);
thrift_status block_mean_topk(const void* q, const void* k, thrift_dtype dt, int B, int H,
                              int Hkv, int N, int d, int blk, int causal, float topk_frac,
                              int sink_blocks, int recent_blocks, uint8_t* mask,
                              void* workspace, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------- attention --
 * [TA] + [SS] ScaleSearchAttention.  q [B,N,H,d], k, v [B,N,Hkv,d] 16-bit,
 * contiguous.  Per (batch, head, query block of blk rows) the key blocks that
 * were not selected run first on the NVFP4 path (block-scaled FP4 MMA, fp32
 * accumulation; P quantised in two levels: a per-row, per-key-block fp32
 * factor rowmax/2688 and NVFP4 16-key blocks), then the selected ones on the
 * FP16 path (16-bit MMA with the unrotated inputs), merged by one online
 * softmax.  Q, K, V are quantised inside the call (Q, K along d; V along
 * tokens; use_scalesearch / use_hadamard as in nvfp4_quantize).
 *   out [B,N,H,d] 16-bit out;  lse [B,H,N] fp32 out (natural log).
 * The FP16 pairs are those of block_mean_topk with the same topk_frac,
 * sink_blocks and recent_blocks.
 * smooth_k != 0: K smoothing on the NVFP4 path (the Q/K smoothing the
 * "Attn-QAT" and "ThriftAttention" pages name among the outlier
 * mitigations of earlier FP4 attention; the pages give no formula, this is
 * the reading): mu = the mean of each K channel over its sequence's tokens
 * (per kv head; fp64 sums of 128-token blocks in token order, added in block
 * order, divided by the length, rounded to fp32) is subtracted from K before
 * the NVFP4 quantisation (own tensor scale for K - mu), and q^ . mu (the
 * dequantised NVFP4 query row against the means) is added back to every
 * NVFP4 score of the row, so the two paths keep one softmax scale.  The FP16
 * path and the selection use the raw K.  Not combined with use_hadamard
 * (THRIFT_ERR_UNSUPPORTED).
 * Requirements: H % Hkv == 0, d in {64,128}, blk in {64,128}, N >= 1,
 * 0 <= topk_frac <= 1, sink_blocks, recent_blocks >= 0,
 * nB = ceil(N/blk) <= 512.
 */
/* Same selection without a workspace argument.  For callers that cannot
 * allocate device memory: for example code that runs while a CUDA graph is
 * being captured (cudaMalloc is not allowed there), or a plug-in handed only
 * tensors and a stream by a host framework that owns all device memory.  The
 * scratch (block means and pair scores) lives in one fixed array of
 * THRIFT_NOALLOC_SCRATCH_BYTES in this library's device memory, held on every
 * device that loads the library until the process exits; nothing in it has
 * to start at zero.  The first call on a device looks up that array's device
 * address (cudaGetSymbolAddress, with that device current); make that first
 * call before any stream capture.  Calls that overlap on the GPU share the
 * array and race: issue them on one stream, or otherwise serialise them.
 * Returns THRIFT_ERR_SCRATCH, launching nothing, when
 * block_mean_topk_workspace_size(...) exceeds THRIFT_NOALLOC_SCRATCH_BYTES.
 * Other arguments and results as block_mean_topk.  The method has no
 * counterpart of this entry point; it only changes where scratch lives. */
#define THRIFT_NOALLOC_SCRATCH_BYTES (8u << 20)
thrift_status block_mean_topk_noalloc(const void* q, const void* k, thrift_dtype dt, int B,
                                      int H, int Hkv, int N, int d, int blk, int causal,
                                      float topk_frac, int sink_blocks, int recent_blocks,
                                      uint8_t* mask, void* stream);

size_t thrift_attn_workspace_size(int B, int H, int Hkv, int N, int d, int blk);
thrift_status thrift_attn_fwd(const void* q, const void* k, const void* v, thrift_dtype dt,
                              int B, int H, int Hkv, int N, int d, int blk, int causal,
                              float topk_frac, int sink_blocks, int recent_blocks,
                              int use_scalesearch, int use_hadamard, int smooth_k, void* out,
                              float* lse, void* workspace, size_t ws_bytes, void* stream);

/* Varlen: q [total,H,d], k, v [total,Hkv,d] packed; cu_seqlens int32
 * [nseq+1] on the DEVICE (cu_seqlens[0] = 0, cu_seqlens[nseq] = total,
 * every length in 1..max_seqlen).  Each sequence is an independent problem
 * (its own blocks and top-k); tensor scales cover the whole packed tensor.
 *   out [total,H,d];  lse [H,total] fp32.
 * Requirements as thrift_attn_fwd with N -> max_seqlen. */
size_t thrift_attn_varlen_workspace_size(int nseq, int64_t total, int max_seqlen, int H,
                                         int Hkv, int d, int blk);
thrift_status thrift_attn_fwd_varlen(const void* q, const void* k, const void* v,
                                     thrift_dtype dt, const int32_t* cu_seqlens, int nseq,
                                     int64_t total, int max_seqlen, int H, int Hkv, int d,
                                     int blk, int causal, float topk_frac, int sink_blocks,
                                     int recent_blocks, int use_scalesearch, int use_hadamard,
                                     int smooth_k, void* out, float* lse, void* workspace,
                                     size_t ws_bytes, void* stream);

/* ---------------------------------------------- one problem on several GPUs --
 * [TA] Metodologia step 1: block means, scores and selection are per
 * (sequence, head), and so are the NVFP4 blocks of Q, K and V and the
 * attention itself; the only quantity coupling the heads and sequences of one
 * problem is the per-tensor FP32 scale g = amax/2688 of Q, K and V.  A
 * problem split by (sequence, kv-head group) across GPUs therefore gives the
 * same codes, scales, selection and output as on one GPU once every shard
 * uses the whole problem's three absmaxes: each shard computes its own with
 * thrift_attn_absmax, the shards agree on the elementwise maximum (a 3-float
 * max all-reduce), and each runs thrift_attn_fwd_absmax with it.
 *
 * thrift_attn_absmax: amax_out[3] (device fp32, written) = the absmax of Q
 * and of K (after the Hadamard rotation when use_hadamard; of K - mu with
 * smooth_k, mu the per-sequence channel means of reading R16) and of V over
 * this call's tensors.  cu_seqlens: device [nseq+1] for packed sequences, or
 * NULL for nseq sequences of max_seqlen tokens each ([nseq, max_seqlen, .]
 * layout, total = nseq * max_seqlen).  workspace: as thrift_attn_fwd_absmax.
 *
 * thrift_attn_fwd_absmax: thrift_attn_fwd / thrift_attn_fwd_varlen (chosen
 * by cu_seqlens as above; lse [nseq, H, max_seqlen] without cu_seqlens,
 * [H, total] with them) with the three tensor absmaxes read from amax_in
 * (device fp32 [3]) instead of computed: g = amax/2688 (1 for 0) as always.
 * Workspace: thrift_attn_varlen_workspace_size(nseq, total, max_seqlen, H,
 * Hkv, d, blk) bytes.  Other arguments, requirements and errors as those
 * calls. */
thrift_status thrift_attn_absmax(const void* q, const void* k, const void* v, thrift_dtype dt,
                                 const int32_t* cu_seqlens, int nseq, int64_t total,
                                 int max_seqlen, int H, int Hkv, int d, int blk, int use_hadamard,
                                 int smooth_k, float* amax_out, void* workspace, size_t ws_bytes,
                                 void* stream);
thrift_status thrift_attn_fwd_absmax(const void* q, const void* k, const void* v,
                                     thrift_dtype dt, const int32_t* cu_seqlens, int nseq,
                                     int64_t total, int max_seqlen, int H, int Hkv, int d,
                                     int blk, int causal, float topk_frac, int sink_blocks,
                                     int recent_blocks, int use_scalesearch, int use_hadamard,
                                     int smooth_k, const float* amax_in, void* out, float* lse,
                                     void* workspace, size_t ws_bytes, void* stream);

/* Byte offset, inside the workspace of thrift_attn_fwd (nseq = B,
 * max_seqlen = N) or thrift_attn_fwd_varlen, of the block-pair selection the
 * call leaves there once it has completed on its stream: uint8
 * [nseq, H, nB, nB], nB = ceil(max_seqlen / blk), 1 = the pair ran on the
 * FP16 path ("ThriftAttention", Metodologia step 1); for a sequence with
 * fewer blocks only its leading nb x nb pairs are meaningful.  Returns 0 for
 * arguments the attention calls reject (0 is never a valid offset).  For
 * inspection and tests; the workspace stays owned by the caller. */
size_t thrift_attn_workspace_mask_offset(int nseq, int max_seqlen, int H, int Hkv, int d,
                                         int blk);

/* -------------------------------------------------------------- decode --
 * ThriftAttention decode over a double KV cache ("ThriftAttention",
 * Resultados: decode speed-up; Significado: the KV cache grows by 28%
 * because every token is kept in FP16 and in FP4).  One new query token per
 * sequence attends to the len_b tokens cached for that sequence (its own key
 * included: append it first).  Supported: d = 128, blk = 128, H % Hkv == 0,
 * H / Hkv <= 16; other shapes return THRIFT_ERR_UNSUPPORTED.
 *
 * The cache is caller-owned device memory of thrift_kv_cache_size() bytes,
 * ZERO-FILLED before its first use and before a sequence's slot is reused;
 * its content is defined by this library.  Per (sequence b, kv head, key
 * tile j of 128 tokens), in this order of regions, each region indexed by
 * tile = (b * Hkv + hk) * ntile + j, ntile = ceil(capacity / 128):
 *   K4   9216 B: NVFP4 K codes [128 tokens, 64 B] (byte 16i..16i+15 of a
 *        row's 64 stored at chunk i XOR ((row / 2) mod 4)), then the UE4M3
 *        scales of the 8 d-blocks in two 512-byte images (K-step s =
 *        d-blocks 4s..4s+3: byte 512 s + (row mod 32) 16 + (row / 32) 4 +
 *        (block mod 4));
 *   V4   9216 B: the same for V^T: rows = channels, 16-token blocks along
 *        the 128 tokens;
 *   K16  32768 B: the 16-bit K rows, two 64-column regions [128, 128 B],
 *        16-byte chunk i of a row at chunk i XOR (row mod 8);
 *   V16  32768 B: the 16-bit V^T, the same with rows = channels;
 *   MEAN 1024 B: fp64 mean over the cached tokens of the tile of each K
 *        channel (tokens summed in order from the tile start).
 * The 16-bit parts hold every cached value exactly; the NVFP4 parts are
 * their quantisation under the caller's per-tensor scales g_K, g_V (V in
 * 16-token blocks counted from token 0, the last block zero-padded).
 *
 * thrift_kv_cache_append: appends n_new[b] tokens (0 <= n_new[b] <=
 * max_new) after cache_len[b] tokens of sequence b: k_new, v_new 16-bit
 * [B, max_new, Hkv, 128] (token i of sequence b at [b, i]); cache_len,
 * n_new int32 [B] on the device, read only (the caller advances its own
 * lengths); kv_scale fp32 [2] on the device = (g_K, g_V).  Tokens that
 * would land at or past `capacity` are dropped.  use_scalesearch as in
 * nvfp4_quantize.  max_new = 0 launches nothing.  Appends to the same
 * sequence must not overlap on the GPU.
 *
 * thrift_attn_decode: q 16-bit [B, H, 128]; seq_len int32 [B] on the
 * device (tokens cached, clamped to [0, capacity]); kv_scale as above.
 * The query tensor is quantised with g_Q = amax(q) / 2688 (use_scalesearch
 * as in nvfp4_quantize); each (sequence, head) takes k = ceil(topk_frac *
 * nb) of its nb = ceil(len / 128) key tiles on the FP16 path by the score
 * q . kbar_j (fp64; ties to the lower tile), plus the first sink_blocks and
 * the last recent_blocks tiles; the rest on the NVFP4 path; one online
 * softmax (NVFP4 tiles, then FP16 tiles).
 *   out 16-bit [B, H, 128] out;  lse fp32 [B, H] out (natural log; an
 *   empty sequence gives a zero row and -inf).
 * The workspace (thrift_attn_decode_workspace_size bytes, no initial
 * content) also receives the selection, uint8 [B, H, ntile] (1 = FP16
 * tile; tiles past a sequence's end 0) at thrift_attn_decode_mask_offset().
 * Requirements: 0 <= topk_frac <= 1; sink_blocks, recent_blocks >= 0;
 * capacity <= 32 * 512 * 128 tokens.  The kernel timer covers the decode
 * attention kernel as well. */
size_t thrift_kv_cache_size(int B, int Hkv, int capacity, int d, int blk);
thrift_status thrift_kv_cache_append(const void* k_new, const void* v_new, thrift_dtype dt, int B,
                                     int Hkv, int d, int blk, int capacity,
                                     const int32_t* cache_len, const int32_t* n_new, int max_new,
                                     const float* kv_scale, int use_scalesearch, void* cache,
                                     size_t cache_bytes, void* stream);
size_t thrift_attn_decode_workspace_size(int B, int H, int Hkv, int capacity, int d, int blk);
size_t thrift_attn_decode_mask_offset(int B, int H, int Hkv, int capacity, int d, int blk);
thrift_status thrift_attn_decode(const void* q, thrift_dtype dt, int B, int H, int Hkv, int d,
                                 int blk, int capacity, const void* cache, size_t cache_bytes,
                                 const int32_t* seq_len, const float* kv_scale, float topk_frac,
                                 int sink_blocks, int recent_blocks, int use_scalesearch,
                                 void* out, float* lse, void* workspace, size_t ws_bytes,
                                 void* stream);

/* ------------------------------------------------------------ Attn-QAT --
 * "Attn-QAT: 4-Bit Attention With Quantization-Aware Training",
 * Metodologia: attention trained through a fake-quantised NVFP4 forward.
 * The forward quantises Q and K (16-blocks along d), V (16-blocks along the
 * tokens of each sequence, the last block zero-padded) with per-tensor
 * scales g = amax / 2688 and the block scales of max scaling (ScaleSearch
 * when use_scalesearch), computes S = Q^ K^T / sqrt(d),
 * lse = log sum_j exp S, P = exp(S - lse), its two-level FP4 image P^ per
 * (row, key tile of blk keys from the sequence start: sigma = tile row max /
 * 2688, 16-key blocks of P / sigma with scale E4M3(amax / 6)), the FP4
 * output O = P^ V^ and the high-precision output O' = P V^ (Metodologia 2).
 * The backward recomputes P and P^ at the forward's precision (Metodologia
 * 1) and returns, with every quantiser passing gradients straight through,
 *   D = rowsum(dO o O'),  dV = P^T dO,  dP = dO V^T,  dS = P o (dP - D),
 *   dQ = dS K^ / sqrt(d),  dK = dS^T Q^ / sqrt(d),
 * dK and dV summed over the query heads of each kv head (H % Hkv == 0).
 *
 * Layout: packed sequences as in thrift_attn_fwd_varlen: q, dout 16-bit
 * [total, H, d], k, v [total, Hkv, d], cu_seqlens int32 [nseq + 1] on the
 * device (cu[0] = 0, non-decreasing, cu[nseq] = total), all contiguous and
 * 16-byte aligned; max_seqlen >= every length.  causal: key j visible to
 * query i iff j <= i within a sequence.  d in {64, 128}, blk in {64, 128}
 * (else THRIFT_ERR_UNSUPPORTED).
 *
 * Outputs (caller-owned device memory): out [total, H, d] in the input
 * type (O), out_hp fp32 [total, H, d] (O'), lse fp32 [H, total] (natural
 * log); dq fp32 [total, H, d], dk, dv fp32 [total, Hkv, d].
 *
 * Workspace: thrift_qat_workspace_size(total, nseq, H, Hkv, d) bytes of
 * device memory, 16-byte aligned; it holds the fake-quantised images of Q,
 * K, V (each element E2M1 value x UE4M3 block scale, exact in the input
 * type) and the dO image as 128-row operand tiles (total / 128 + nseq tiles
 * per head), the tensor scales and D.  cu_seqlens must describe sequences
 * that partition [0, total): the tile slots of a sequence are derived from
 * its start.  thrift_qat_bwd_varlen with reuse_images != 0 takes the
 * images and scales from the workspace as a thrift_qat_fwd_varlen call on
 * the same q, k, v, flags and workspace left them; with 0 it recomputes them.
 *
 * Errors: THRIFT_ERR_ARG for null or misaligned pointers, bad shapes or a
 * short workspace (returned before any launch); THRIFT_ERR_CUDA if a launch
 * fails.  Asynchronous on `stream`. */
size_t thrift_qat_workspace_size(int64_t total, int nseq, int H, int Hkv, int d);
thrift_status thrift_qat_fwd_varlen(const void* q, const void* k, const void* v, thrift_dtype dt,
                                    const int32_t* cu_seqlens, int nseq, int64_t total,
                                    int max_seqlen, int H, int Hkv, int d, int blk, int causal,
                                    int use_scalesearch, void* out, float* out_hp, float* lse,
                                    void* workspace, size_t ws_bytes, void* stream);
thrift_status thrift_qat_bwd_varlen(const void* q, const void* k, const void* v, const void* dout,
                                    thrift_dtype dt, const int32_t* cu_seqlens, int nseq,
                                    int64_t total, int max_seqlen, int H, int Hkv, int d, int blk,
                                    int causal, int use_scalesearch, int reuse_images,
                                    const float* out_hp, const float* lse, float* dq, float* dk,
                                    float* dv, void* workspace, size_t ws_bytes, void* stream);

/* ----------------------------------------------------- kernel timing --
 * Measurement aid (not part of the method).  While enabled, every
 * thrift_attn_fwd / thrift_attn_fwd_varlen call records a CUDA event pair on
 * its stream around the attention kernel launch (thrift_qat_fwd_varlen:
 * around the forward kernel; thrift_qat_bwd_varlen: around its two
 * gradient kernels).  thrift_kernel_timer_read
 * waits for the recorded events, returns the summed kernel time in
 * milliseconds and the number of timed launches, and clears the record.
 * Host-side state shared by all threads of the process; not thread-safe.
 * Events are created on first use and kept for reuse. */
thrift_status thrift_kernel_timer_enable(int enable);
thrift_status thrift_kernel_timer_read(double* total_ms, int* launches);

/* Failure-detection aid (not part of the method).  Launches one small kernel
 * on `stream` whose single waiting thread uses the library's bounded waits on
 * something that never completes: mode 0 an mbarrier that nothing arrives
 * on (the wait every pipelined kernel here uses between its roles), mode 1
 * a global word that nothing writes (the quantiser's grid-wide exchange).
 * After limit_us microseconds (1 .. 1,000,000) the wait gives up, sets the
 * device status word to THRIFT_ERR_TIMEOUT and the kernel returns normally:
 * no trap, the context stays usable.  Returns THRIFT_ERR_ARG for a bad mode
 * or limit (nothing launched), THRIFT_ERR_CUDA if the launch fails. */
thrift_status thrift_test_wait_timeout(int mode, int limit_us, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* THRIFT_NVFP4_H */
