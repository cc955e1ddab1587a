/*
 * tq.h - C ABI of the TurboQuant codec library for NVIDIA B200 (sm_100a).
 *
 * The library quantizes key/value vectors with a random rotation (sign flips
 * then a Walsh-Hadamard transform), a per-vector norm, a Lloyd-Max scalar
 * code and a 1-bit QJL sketch of the residual, and computes attention logits,
 * decode attention and top-k inner-product search directly from the packed
 * codes.  A second stage-1 code rewrites the rotated vector in recursive
 * polar form and codes its angles with per-level tables (tq_polar_*).
 *
 * Sources (web articles about Google's TurboQuant; they print no code):
 *  [E1] "TurboQuant explainer" (m.163.com), section "TurboQuant 怎么做的",
 *       "第一步：PolarQuant": random rotation, then one precomputed Max-Lloyd
 *       table for every coordinate, b-1 bits, no per-block normalisation.
 *  [E2] same page, "第二步：QJL": JL transform of the residual kept as sign
 *       bits, estimator with E[<y, Q^-1(Q(x))>] = <y, x>.
 *  [E3] same page, "合起来": b-1 + 1 = b bits per value.
 *  [E4] same page, "速度": attention logits computed from 4-bit codes.
 *  [E5] same page, "向量搜索": inner-product nearest-neighbour search.
 *  [Z1] zhidx turboquant_plus article, "01 turboquant_plus：介绍与详解": WHT
 *       rotation; turbo4 = 4.25 bit/value; asymmetric K/V; block layout.
 *
 * Conventions (all entry points):
 *  - The caller owns every buffer; the library allocates no memory.  Device
 *    pointers must be device (or managed) memory of the current CUDA device.
 *  - Kernels are launched asynchronously on `stream` (NULL = legacy default
 *    stream).  The return value reports host-side validation and launch
 *    errors only.
 *  - Return value: TQ_OK or a negative TQ_E* status.  On error nothing is
 *    launched and no output is written; tq_last_error() gives a message
 *    (thread-local, valid until the next call on that thread).
 *  - Code buffers must be 16-byte aligned; float/fp16 arrays 4-byte/2-byte.
 *
 * Code layout (canonical; produced by tq_quantize, consumed by every reader):
 *   Vectors are grouped in tiles of 32 consecutive vectors; the last tile is
 *   zero-filled.  A tile holds kb bit-planes (plane p = bit p of each index),
 *   each 32 x d_pad/8 bytes with vector t at byte offset t*d_pad/8 and
 *   coordinate j at bit j%32 of little-endian 32-bit word j/32; then (product
 *   mode) the QJL signs, 32 x m/8 bytes, sign i at bit i%32 of word i/32.
 *   kb = bits-1 (TQ_MODE_PROD) or bits (TQ_MODE_MSE).  Norms ||x|| and
 *   residual norms ||r|| are separate fp16 arrays (IEEE half bit patterns),
 *   one per vector.  For multi-head data, vector index =
 *   (sequence*H_kv + head)*n_tokens + token.
 */
#ifndef TQ_H_
#define TQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* tq_stream_t; /* same type as cudaStream_t */

/* status codes */
#define TQ_OK 0
#define TQ_EINVAL (-1)        /* invalid argument (null, size, alignment) */
#define TQ_EUNSUPPORTED (-2)  /* valid but not implemented for this shape */
#define TQ_ECUDA (-3)         /* CUDA launch/runtime error; see tq_last_error */
#define TQ_ETIMEOUT (-4)      /* a bounded device-side wait gave up (tq_device_status) */

/* code modes */
#define TQ_MODE_PROD 0 /* (bits-1)-bit Lloyd-Max code + m QJL sign bits [E1][E2][E3] */
#define TQ_MODE_MSE 1  /* bits-bit Lloyd-Max code only (values; 2/pi-biased inner products) */

/* code layouts (tq_params.layout) */
#define TQ_LAYOUT_PLANES 0 /* canonical: per tile, plane p = 32 vectors x d_pad/8 bytes (above) */
#define TQ_LAYOUT_SLICED 1 /* token-sliced, MSE codes only: per tile, plane p = d_pad little-endian
                              32-bit words, word j's bit t = bit p of vector t's index at coordinate j
                              (same bytes per tile; the value cache tq_decode_attn scans on the tensor
                              cores).  Written by tq_quantize (d_pad 128, 16-bit input), read by
                              tq_decode_attn (values) and tq_dequantize; other calls return
                              TQ_EUNSUPPORTED. */

/* input element types */
#define TQ_F32 0
#define TQ_F16 1
#define TQ_BF16 2

/*
 * Quantizer description.  d: input dimension (1..d_pad); d_pad: rotation
 * size, 128 or 256; bits: total bits b (PROD: 2..4, MSE: 1..4); m: QJL rows
 * (PROD: a multiple of 32, 32..256; MSE: 0).  The four device arrays are
 * produced once by tq_make_codebook / tq_make_params and copied to the device
 * by the caller:
 *   centroids  [2^kb]   fp32, ascending, odd-symmetric
 *   thresholds [2^kb-1] fp32, midpoints of neighbouring centroids
 *   signs_D    [d_pad]  int8, +1 / -1
 *   S          [m*d_pad] fp16 bit patterns, row-major (NULL in MSE mode)
 */
typedef struct tq_params {
  int32_t d;
  int32_t d_pad;
  int32_t bits;
  int32_t mode;
  int32_t m;
  int32_t layout; /* TQ_LAYOUT_PLANES (0) or TQ_LAYOUT_SLICED (MSE codes only) */
  const float* centroids;
  const float* thresholds;
  const int8_t* signs_D;
  const uint16_t* S;
} tq_params;

/*
 * tq_make_codebook - Lloyd-Max codebook for the rotated-coordinate law [E1].
 * Host memory only; no device.  The law is that of one coordinate of a
 * uniform random unit vector in R^d_pad, density proportional to
 * (1-t^2)^((d_pad-3)/2) on (-1,1) (the "Beta" law of [E1]).  Writes 2^kb
 * centroids (fp64 Lloyd-Max fixed point rounded to fp32) and 2^kb-1
 * thresholds (fp32 rounding of the exact midpoints of the fp32 centroids).
 * d_pad: 4..4096 power of two; kb: 1..4.  Returns TQ_EINVAL on bad arguments.
 */
int tq_make_codebook(int d_pad, int kb, float* centroids, float* thresholds);

/*
 * tq_make_params - random sign flips D and QJL matrix S [E1][E2][Z1].
 * Host memory only.  Generator: Philox4x32-10 keyed by seed (low 32 bits,
 * high 32 bits); block i of stream s uses counter (i, s, 0, 0) and its four
 * words are words 4i..4i+3 of the stream.  D[j] = -1 if bit 0 of word j of
 * stream 0 is set, else +1.  S (m x d_pad, row-major) entries 2p, 2p+1 are
 * the Box-Muller pair of words 2p, 2p+1 of stream 1, u = (w + 0.5)/2^32,
 * (sqrt(-2 ln u_a) cos(2 pi u_b), sqrt(-2 ln u_a) sin(2 pi u_b)), rounded to
 * fp16 (nearest even).  S may be NULL when m == 0.
 */
int tq_make_params(int d_pad, int m, uint64_t seed, int8_t* D, uint16_t* S);

/* Bytes of a code buffer holding n_vec vectors (whole 32-vector tiles). */
int64_t tq_code_bytes(int d_pad, int kb, int m, int64_t n_vec);

/*
 * tq_quantize - encode n_vec vectors [E1][E2].
 *   x: device, n_vec rows of d elements of `dtype`, row stride ld elements
 *      (ld >= d; x and ld*elem_size must be 16-byte aligned, d*elem_size a
 *      multiple of 16).
 *   codes: device, tq_code_bytes(d_pad, kb, m, n_vec) bytes (tail zeroed).
 *   norms, rnorms: device fp16 [n_vec]; rnorms ignored (may be NULL) in MSE mode.
 * Per vector: n = ||x||, x_hat = x/n (0 for n = 0), zero-pad to d_pad,
 * y = H D x_hat / sqrt(d_pad), idx_j = #{l : y_j > t_l}, r = y - c[idx],
 * gamma = ||r||, sign_i = [(S r)_i >= 0].  Norms are stored as fp16 (nearest
 * even; values above 65504 become +inf).
 */
int tq_quantize(const tq_params* p, const void* x, int dtype, int64_t n_vec, int64_t ld,
                void* codes, uint16_t* norms, uint16_t* rnorms, tq_stream_t stream);

/*
 * tq_project_quantize - quantize-on-write: the K (or V) projection of an
 *   attention layer and tq_quantize of its output in one kernel, so the
 *   projected vectors never go to memory [Z1: the prefill path of the runtime
 *   port; E1][E2] for the code.
 *   Per head h and token t the vector is k = bf16(x_t . W_h^T), the 128
 *   projection outputs of head h rounded to bf16 as a bf16 cache write would
 *   round them (fp32 accumulation over `hidden`), then coded exactly as
 *   tq_quantize codes a bf16 row.
 *   p: d = d_pad = 128; product mode needs m = 128.
 *   x: device bf16 [n_tok][hidden], row stride ld_x elements; w: device bf16
 *      [n_heads*128][hidden] (the layer's weight in [out][in] order, head h =
 *      rows 128h .. 128h + 127), row stride ld_w.  hidden a positive multiple
 *      of 32; x, w 16-byte aligned; ld_x, ld_w >= hidden, multiples of 8.
 *   codes/norms/rnorms: as tq_quantize for n_heads*n_tok vectors, vector
 *      h*n_tok + t = token t of head h (the per-head key order tq_logits
 *      reads); code buffer tail zeroed.
 *   k_out: optional (NULL: not written) device bf16 [n_tok][ld_k], head h in
 *      columns 128h .. 128h + 127: the vectors that were coded.  ld_k >=
 *      128*n_heads, a multiple of 8; k_out 16-byte aligned.
 *   Returns TQ_EUNSUPPORTED for other shapes.
 */
int tq_project_quantize(const tq_params* p, const void* x, int64_t n_tok, int64_t ld_x, int hidden,
                        const void* w, int n_heads, int64_t ld_w, void* codes, uint16_t* norms,
                        uint16_t* rnorms, void* k_out, int64_t ld_k, tq_stream_t stream);

/*
 * tq_dequantize - the reconstruction x_hat = Q^-1(codes) [E2: the QJL part is
 *   sqrt(pi/2)/m * gamma * S^T sigma, sigma = 2s - 1, which makes
 *   E[<y, Q^-1(Q(x))>] = <y, x>]:
 *     product mode  x_hat = n D H (c[idx] + sqrt(pi/2)/m * gamma * S^T sigma) / sqrt(d_pad)
 *     MSE mode      x_hat = n D H c[idx] / sqrt(d_pad)
 *   first d coordinates.  <q, x_hat> equals the tq_logits estimate for every q
 *   (the estimate is linear in the key).  Re-encoding stored tokens at a lower
 *   bit width (temporal decay [Z1]) is tq_dequantize followed by tq_quantize
 *   with the lower-width parameters.
 *   codes, norms, rnorms: as written by tq_quantize for n_vec vectors (rnorms
 *   NULL in MSE mode).  out: device fp32 [n_vec][ld], ld >= d; columns d..ld-1
 *   are not written.  codes 16-byte aligned.
 */
int tq_dequantize(const tq_params* p, const void* codes, const uint16_t* norms,
                  const uint16_t* rnorms, int64_t n_vec, float* out, int64_t ld,
                  tq_stream_t stream);

/*
 * tq_logits - attention logits straight from the codes [E2][E4].
 *   q: device fp32 [n_q][d], n_q = n_kv_heads*group; query head h reads KV
 *      head h/group (GQA).
 *   codes/norms/rnorms: n_kv_heads*n_keys vectors; keys of head g are
 *      vectors g*n_keys .. g*n_keys+n_keys-1.
 *   logits: device fp32 [n_q][n_keys], raw inner-product estimates (no 1/sqrt(d)):
 *      l = n*( <q_rot, c[idx]> + gamma*sqrt(pi/2)/m*<S q_rot, 2s-1> ),
 *      q_rot = H D q / sqrt(d_pad).  MSE-mode codes give n*<q_rot, c[idx]>.
 *   workspace: device, >= tq_logits_workspace(p, n_q) bytes, 16-byte aligned.
 *      The tensor-core path (d_pad 128, group <= 4, n_keys a multiple of 32,
 *      16-byte aligned norms) prepares the queries inside its kernel and does
 *      not touch the workspace; the other shapes keep their query
 *      preparation there.
 * Supported: d_pad 128 with kb <= 3; d_pad 256 with kb <= 2; d_pad 256 with
 *   kb = 3 in MSE mode or with m = 256 (the tensor-memory scan of
 *   tq_search_topk writing every score; n_keys % 32 == 0 when n_kv_heads > 1).
 */
int64_t tq_logits_workspace(const tq_params* p, int n_q);
int tq_logits(const tq_params* p, const float* q, int n_q, int group, const void* codes,
              const uint16_t* norms, const uint16_t* rnorms, int64_t n_keys, int n_kv_heads,
              float* logits, void* workspace, int64_t workspace_bytes, tq_stream_t stream);

/*
 * tq_logits_ld - tq_logits writing row h of the logits at logits + h*ld_logits
 *   (ld_logits >= n_keys; columns past n_keys untouched).  Mixed bit widths
 *   along a sequence (older tokens re-encoded at a lower width, temporal decay
 *   [Z1]) are scanned with one call per width segment into one logits matrix:
 *   segment k's call gets its own parameters and codes, n_keys = the segment's
 *   length, logits + (segment start) and ld_logits = the whole length.
 */
int tq_logits_ld(const tq_params* p, const float* q, int n_q, int group, const void* codes,
                 const uint16_t* norms, const uint16_t* rnorms, int64_t n_keys, int n_kv_heads,
                 float* logits, int64_t ld_logits, void* workspace, int64_t workspace_bytes,
                 tq_stream_t stream);

/*
 * tq_logits_noalloc - tq_logits without a caller-provided workspace.
 * The pages have no counterpart: this is an interface for callers that cannot
 * allocate device memory when they call (for example code that runs while a
 * CUDA graph is being captured, or a plugin whose host framework owns every
 * device buffer and passes only inputs and outputs).  Same arguments and
 * results as tq_logits minus the workspace.  Shapes that tq_logits serves on
 * its tensor-core path need no scratch at all; the others keep their query
 * preparation in a static device array of tq_logits_noalloc_max_scratch()
 * bytes (1 MiB) that every device loading the library keeps until the
 * process exits.
 *  - The array's device address is looked up (cudaGetSymbolAddress, with the
 *    device current) on the first call on a device, and again whenever the
 *    current driver context differs from the one of the last lookup (after a
 *    cudaDeviceReset, or under a non-primary context); make the first call on
 *    a device before any stream capture.
 *  - Scratch needed on the other shapes: n_kv_heads * ceil(group / 4) chunks
 *    of 128*fr + 64 bytes, fr = 8 * 4 * (mma slots per bit class); at d_pad 128
 *    a chunk is 12352 bytes at b = 4 (product code, m = 128) and 8256 bytes at
 *    b = 3, so 1 MiB holds 84 and 127 chunks.  Calls needing more return
 *    TQ_EINVAL with a message; nothing is launched.
 *  - All calls share the one array: calls that may overlap on the GPU (other
 *    streams, other host threads) race and must be serialised by the caller.
 *    The scratch is fully rewritten by each call, so nothing needs clearing.
 *  - Allocates nothing (no cudaMalloc/cudaFree, no allocating library call).
 */
int64_t tq_logits_noalloc_max_scratch(void);
int tq_logits_noalloc(const tq_params* p, const float* q, int n_q, int group, const void* codes,
                      const uint16_t* norms, const uint16_t* rnorms, int64_t n_keys, int n_kv_heads,
                      float* logits, tq_stream_t stream);

/*
 * tq_decode_attn - one decode step of attention over compressed K (product
 * code) and V (MSE code) [E4][Z1 asymmetric K/V].
 *   q: device fp32 [batch][n_q_heads][d].  K/V vector index =
 *      (b*n_kv_heads + g)*max_tokens + t.  seq_lens: device int32 [batch],
 *      0 <= seq_lens[b] <= max_tokens.
 *   out[b][h] = sum_t softmax_t(scale*l_t) v_hat_t, v_hat = n_v D H c_v[idx_v] / sqrt(d_pad)
 *      (first d coordinates); scale 0 means 1/sqrt(d).  Rows with
 *      seq_lens[b] == 0 are zero.  out: device fp32 [batch][n_q_heads][d].
 *   workspace: device, >= tq_decode_attn_workspace(...) bytes, 16-byte aligned.
 * Supported: kp PROD kb <= 3 and vp MSE, same d/d_pad (128), n_q_heads a
 * multiple of n_kv_heads.
 */
int64_t tq_decode_attn_workspace(const tq_params* kp, int batch, int n_q_heads, int n_kv_heads,
                                 int64_t max_tokens);
int tq_decode_attn(const tq_params* kp, const tq_params* vp, const float* q, int batch,
                   int n_q_heads, int n_kv_heads, const void* kcodes, const uint16_t* knorms,
                   const uint16_t* krnorms, const void* vcodes, const uint16_t* vnorms,
                   const int32_t* seq_lens, int64_t max_tokens, float scale, float* out,
                   void* workspace, int64_t workspace_bytes, tq_stream_t stream);

/*
 * tq_decode_attn_sparse - tq_decode_attn with Sparse V [Z1 "Sparse V": skip
 *   the value work of tokens whose attention weight is negligible].  Same
 *   arguments plus v_eps >= 0.  Inside each 256-token split of a sequence, a
 *   token is dropped when its weight within the split, p_t / (split sum), is
 *   below v_eps for every query head sharing the KV head; since that bounds its
 *   final softmax weight from above, only tokens with final weight < v_eps are
 *   dropped.  A dropped token adds no value but keeps its weight in the
 *   normalisation, so |out - out_full| <= v_eps * sum over tokens with weight
 *   < v_eps of |v_hat_t|.  v_eps = 0 gives exactly tq_decode_attn's result.
 *   Returns TQ_EINVAL for negative or non-finite v_eps.
 */
int tq_decode_attn_sparse(const tq_params* kp, const tq_params* vp, const float* q, int batch,
                          int n_q_heads, int n_kv_heads, const void* kcodes, const uint16_t* knorms,
                          const uint16_t* krnorms, const void* vcodes, const uint16_t* vnorms,
                          const int32_t* seq_lens, int64_t max_tokens, float scale, float v_eps,
                          float* out, void* workspace, int64_t workspace_bytes, tq_stream_t stream);

/*
 * tq_search_topk - top-k inner-product search over quantized vectors [E5].
 *   q: device fp32 [n_q][d]; codes/norms/rnorms: n_db vectors.
 *   ids: device int32 [n_q][k], scores: device fp32 [n_q][k]: the k largest
 *   logit estimates (as tq_logits with group 1) per query, in descending
 *   order, ties to the lower id.  1 <= k <= 16.  When n_db < k the trailing
 *   slots hold id INT32_MAX and score -inf.
 *   workspace: device, >= tq_search_workspace(...) bytes, 16-byte aligned.
 */
int64_t tq_search_workspace(const tq_params* p, int n_q, int64_t n_db, int k);
int tq_search_topk(const tq_params* p, const float* q, int n_q, const void* codes,
                   const uint16_t* norms, const uint16_t* rnorms, int64_t n_db, int k,
                   int32_t* ids, float* scores, void* workspace, int64_t workspace_bytes,
                   tq_stream_t stream);

/*
 * Sharded forms: one process per GPU, each holding one shard; the only
 * exchange is one all-gather of the small per-shard results (the caller's,
 * e.g. torch.distributed over NCCL; see parallel.py of the Python package).
 *
 * tq_search_merge - global top-k of a database split across devices [E5:
 *   inner-product search over very large sets].  Each device runs
 *   tq_search_topk on its shard; the lists are gathered and merged here.
 *   ids, scores: device [n_parts][n_q][k], int32 shard-local ids and fp32
 *     estimates as tq_search_topk returns them (id < 0 or INT32_MAX, or
 *     score -inf: empty slot).
 *   id_offsets: HOST int64 [n_parts], the global id of each shard's first
 *     vector (0 <= offset < INT32_MAX); added to that shard's ids.
 *   out_ids / out_scores: device [n_q][k]: the k best by estimate, ties to the
 *     lower global id.  This equals tq_search_topk over the whole database
 *     when every shard returned its exact top-k.
 *   1 <= n_parts <= 64, 1 <= k <= 16, n_parts * k <= 1024.
 */
int tq_search_merge(const int32_t* ids, const float* scores, int n_parts, const int64_t* id_offsets, int n_q,
                    int k, int32_t* out_ids, float* out_scores, tq_stream_t stream);

/*
 * tq_decode_attn_partial - tq_decode_attn over the tokens this caller holds
 *   (a token range of every sequence, laid out as a KV cache of its own with
 *   max_tokens and per-sequence counts seq_lens of that range), returning the
 *   unnormalised partial instead of the output [E4, split over devices].
 *   partial: device fp32 [batch][n_q_heads][d_pad + 2], per row
 *     o_rot[0..d_pad) = sum_t 2^(s_t - m) n_v,t c_v[idx_t]  (rotated domain),
 *     then m = max_t s_t with s_t = scale * l_t * log2(e) (-inf: no token),
 *     then l = sum_t 2^(s_t - m) (0: no token).
 *   Other arguments and the workspace as tq_decode_attn;
 *   tq_decode_attn_partial_bytes gives the size of `partial`.
 */
int64_t tq_decode_attn_partial_bytes(const tq_params* vp, int batch, int n_q_heads);
int tq_decode_attn_partial(const tq_params* kp, const tq_params* vp, const float* q, int batch,
                           int n_q_heads, int n_kv_heads, const void* kcodes, const uint16_t* knorms,
                           const uint16_t* krnorms, const void* vcodes, const uint16_t* vnorms,
                           const int32_t* seq_lens, int64_t max_tokens, float scale, float* partial,
                           void* workspace, int64_t workspace_bytes, tq_stream_t stream);

/*
 * tq_decode_attn_merge - log-sum-exp merge of n_parts partials (device fp32
 *   [n_parts][batch][n_q_heads][d_pad + 2], e.g. all-gathered from the
 *   devices) and the inverse rotation: with M = max_k m_k and w_k = 2^(m_k - M),
 *   out[b][h] = D H (sum_k w_k o_k) / (sum_k w_k l_k) / sqrt(d_pad), first d
 *   coordinates; rows empty in every part are zero.  vp: the value
 *   parameters (MSE code, d_pad 128).  1 <= n_parts <= 2048.
 */
int tq_decode_attn_merge(const tq_params* vp, const float* partials, int n_parts, int batch, int n_q_heads,
                         float* out, tq_stream_t stream);

/*
 * tq_device_status - report (and optionally clear) device-side wait timeouts.
 *   The tensor-core kernels hand data between their warps on shared-memory
 *   barriers.  Every such wait has an iteration limit; a wait that reaches it
 *   sets a device fault word of its kernel family and the kernel returns
 *   early (its outputs are then undefined), so the context stays usable.
 *   This call synchronizes the current device, reads every family's fault
 *   word and returns TQ_OK if none is set, TQ_ETIMEOUT if one is (the
 *   message names the families), TQ_ECUDA on a CUDA error.  clear != 0
 *   resets the words.  The pages define no such call: it belongs to the
 *   library's error handling, not to the method.
 */
int tq_device_status(int clear);

/*
 * tq_diag_bounded_wait - diagnostic: one CTA waits `polls` times on a
 *   shared-memory barrier that nothing arrives at, then gives up the way the
 *   kernels' waits do (fault word of the diagnostic family set, kernel
 *   returns).  Lets a caller check, without any real failure, that timeouts
 *   reach tq_device_status.  1 <= polls <= 2^20.  Asynchronous on `stream`.
 */
int tq_diag_bounded_wait(int64_t polls, tq_stream_t stream);

/* ------------------------------------------------------------------------
 * Polar-coordinate stage 1 ("PolarQuant").
 *
 * [E1] same page, "第一步：PolarQuant", and "它到底怎么做到的？ / 第一步：
 * PolarQuant —— 换个坐标系压缩": after the random rotation the vector is
 * rewritten as a radius and angles; the angles follow a known, concentrated
 * Beta law, so they are coded with fixed tables and no normalisation constant.
 * The pages give no formulas; this library reads them as follows.
 *   - y = H D (x/||x||) / sqrt(d_pad) as in tq_quantize; ||x|| kept as fp16.
 *   - Recursive pairwise polar form: level 1 turns coordinates (2i, 2i+1) into
 *     a radius and a full angle theta = atan2(y_2i+1, y_2i) in [0, 2 pi);
 *     level l >= 2 turns radii (2i, 2i+1) of level l-1 into a radius and
 *     psi = atan2(r_2i+1, r_2i) in [0, pi/2]; the last radius is 1.
 *   - For a uniform direction theta is uniform and, at level l,
 *     sin^2 psi ~ Beta(2^(l-2), 2^(l-2)); each level has a Lloyd-Max table.
 *   - w bits per coordinate (1..3): a level-1 angle gets b1 = w+1 bits
 *     (2^b1 equal cells, centroids at their middles), a higher-level angle
 *     b2 = w-1 bits (w = 1: decoded at pi/4).
 *   - Decisions: theta -> floor(theta 2^b1 / 2 pi); psi -> #{t : psi > t}.
 * Code record: w*d_pad/8 bytes per vector, vectors consecutive; one
 * little-endian bit stream, LSB first: the d_pad/2 level-1 indices (b1 bits
 * each), then the level-2 indices (d_pad/4), ..., the last level (1), b2 bits
 * each; unused bits zero.
 *
 * Tables (fp32, tq_polar_table_floats(d_pad, w) values, L1 = 2^b1, L2 = 2^b2):
 *   [0, L1)            level-1 centroid angles (j + 1/2) 2 pi / L1
 *   [L1, 3 L1)         (cos, sin) of those, interleaved
 *   then for each level l = 2 .. log2(d_pad), 4 L2 - 1 values:
 *                      L2 centroid angles (Lloyd-Max fixed point, fp32),
 *                      L2 - 1 thresholds (fp32 midpoints of neighbouring
 *                      fp32 centroids), (cos, sin) of the centroids.
 * -------------------------------------------------------------------------*/
typedef struct tq_polar_params {
  int32_t d;      /* input dimension, 1..d_pad */
  int32_t d_pad;  /* rotation size, 128 or 256 */
  int32_t w;      /* bits per coordinate, 1..3 */
  int32_t reserved;
  const float* tables;    /* device, from tq_polar_make_tables */
  const int8_t* signs_D;  /* device, d_pad signs (tq_make_params) */
} tq_polar_params;

/* Number of fp32 table values for (d_pad, w); -1 on bad arguments. */
int64_t tq_polar_table_floats(int d_pad, int w);

/* tq_polar_make_tables - the tables above, host memory (d_pad: power of two
 * 4..4096, w: 1..3).  Lloyd-Max on each level's angle law by Gauss-Legendre
 * quadrature in fp64; centroids rounded to fp32.  TQ_EINVAL on bad arguments. */
int tq_polar_make_tables(int d_pad, int w, float* tables);

/* Bytes of a polar code buffer holding n_vec records of w * d_pad / 8 bytes
 * (d_pad a power of two >= 8; -1 for other arguments). */
int64_t tq_polar_code_bytes(int d_pad, int w, int64_t n_vec);

/*
 * tq_polar_quantize - encode n_vec vectors (x: device, rows of d elements of
 *   dtype, stride ld elements; x, ld*elem_size and d*elem_size 16-byte
 *   aligned, as tq_quantize).  codes: device, tq_polar_code_bytes bytes,
 *   16-byte aligned; norms: device fp16.
 */
int tq_polar_quantize(const tq_polar_params* p, const void* x, int dtype, int64_t n_vec, int64_t ld,
                      void* codes, uint16_t* norms, tq_stream_t stream);

/*
 * tq_polar_dequantize - x_hat = n D H y_hat / sqrt(d_pad) (first d
 *   coordinates), y_hat rebuilt from the table centroids, top radius 1.
 *   out: device fp32 rows of stride ld (>= d).
 */
int tq_polar_dequantize(const tq_polar_params* p, const void* codes, const uint16_t* norms, int64_t n_vec,
                        float* out, int64_t ld, tq_stream_t stream);

/*
 * tq_polar_logits - l[h][k] = n_k <q~_h, y_hat_k> with q~ = H D q / sqrt(d_pad)
 *   (= <q, x_hat_k>).  q: device fp32 [n_kv_heads*group][d]; query head h uses
 *   KV head h / group, whose keys are records h/group * n_keys .. + n_keys - 1.
 *   logits: device fp32 [n_kv_heads*group][n_keys].  1 <= group <= 8.
 */
int tq_polar_logits(const tq_polar_params* p, const float* q, int group, const void* codes,
                    const uint16_t* norms, int64_t n_keys, int n_kv_heads, float* logits, tq_stream_t stream);

/*
 * tq_polar_qjl - the QJL stage on the polar code's residual [E 第二步 applied
 *   to the polar stage 1 of E 第一步]: after tq_polar_quantize of the same x,
 *   r = y - y_hat (y the rotated unit vector, y_hat rebuilt from the records
 *   with unit radius), gamma = ||r||, and the sign bits of S r.  Together with
 *   the polar record this is the product code of the polar stage: w bits per
 *   coordinate plus one bit per projection.
 *   S: device fp16 [m][d_pad] (tq_make_params with the same d_pad), m a
 *      multiple of 32 in [32, d_pad].
 *   x, dtype, ld: as tq_polar_quantize; codes: its records (read).
 *   signs: device, n_vec * m / 8 bytes, 4-byte aligned: vector v's bits at
 *      byte v*m/8, bit i at bit i%32 of little-endian word i/32, bit = [(S r)_i >= 0].
 *   rnorms: device fp16 [n_vec], gamma.
 */
int tq_polar_qjl(const tq_polar_params* p, const uint16_t* S, int m, const void* x, int dtype, int64_t n_vec,
                 int64_t ld, const void* codes, void* signs, uint16_t* rnorms, tq_stream_t stream);

/*
 * tq_polar_logits_prod - logits of the polar product code, unbiased over S:
 *   l[h][k] = n_k ( <q~_h, y_hat_k> + gamma_k sqrt(pi/2)/m <S q~_h, 2 s_k - 1> ).
 *   Arguments as tq_polar_logits plus S, m (as tq_polar_qjl), signs and
 *   rnorms (from tq_polar_qjl).  Writes the stage-1 logits, then adds the QJL
 *   term in a second kernel.
 */
int tq_polar_logits_prod(const tq_polar_params* p, const uint16_t* S, int m, const float* q, int group,
                         const void* codes, const uint16_t* norms, const void* signs, const uint16_t* rnorms,
                         int64_t n_keys, int n_kv_heads, float* logits, tq_stream_t stream);

/* Message for the last failed call on this thread ("" if none). */
const char* tq_last_error(void);

/* Library version, e.g. 100 for 0.1.0. */
int tq_version(void);

#ifdef __cplusplus
}
#endif
#endif /* TQ_H_ */
