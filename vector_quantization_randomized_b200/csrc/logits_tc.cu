// tq_logits on the fifth-generation tensor cores, for d_pad 128 and up to four
// query heads per KV head ("TurboQuant explainer" (m.163.com), "第二步：QJL"
// estimator; "速度": logits straight from the compressed keys).
//
// Integer form of the estimator (scan.cuh): every product is "integer weight x
// code bit".  Weights 2 alpha_T q_rot_j (Walsh plane T of the codebook) and
// 2 u_i (u = S q_rot) are scaled by a per-query power of two to integers below
// 2^23, shifted left by 7 - c for bit class c = coordinate % 8 and split into
// four signed base-256 digits.  The code bits are the A operand of
// tcgen05.mma kind::i8 (u8 x s8 -> s32), held in tensor memory:
//
//   A[key][K = 128P + 16c + 4w + b] = byte b of (word w of plane P) & (1 << c)
//                                   = 2^c * bit(coordinate 32w + 8b + c),
//
// one 32-bit tensor-memory column per masked word.  The digits are the B
// operand in shared memory, 16 rows = 4 queries x 4 digits.  Centroid planes
// and the sign plane go to separate N = 16 MMAs with their own accumulator
// columns, so no MMA multiplies a zero block.  Per 128-key item: 4 NT centroid
// MMAs and 4 sign MMAs (M = 128, N = 16, K = 32 bytes).
//
// The query preparation (rotation, projection, scaling, digit split) runs
// inside this kernel: each CTA builds the B image of the KV heads it scans, so
// tq_logits is one launch and needs no workspace on this path.
//
// Warp roles, one persistent CTA per SM over a contiguous range of
// (KV head, 128-key tile) items, all hand-offs on mbarriers with bounded waits:
//   warp 0      bulk copies of the code tiles into a ring of stages, two items
//               per copy;
//   warps 1-2   MMA issue: warp 1 + p takes the items of parity p, all K steps
//               of an item into one accumulator set.  The loops are warp-uniform
//               and one lane, chosen by elect.sync, issues, with the
//               descriptors of a whole item unrolled from two base values;
//   warps 3-10  expansion: stage -> masked words -> tcgen05.st into one of two
//               or four A buffers (warp = lane quadrant; 3-6 even items, 7-10 odd;
//               with two buffers each is written and read in two halves).  They
//               first take a share of u = S q_rot for the CTA's first image;
//   warps 11-18 query preparation into a ring of two B images, then the
//               epilogue: tcgen05.ld of the item's accumulator set, digit
//               combination, norms (plain loads issued two items ahead), logits
//               (warp = lane quadrant; 11-14 even items, 15-18 odd).
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>

#include "common.h"
#include "prep.h"
#include "scan.cuh"
#include "tc.cuh"

namespace {
using namespace tqd;

constexpr int TK = 128;  // keys per item (MMA M)
constexpr int DP = 128;
constexpr int MAX_STAGES = 12;
constexpr int GI = 2;  // items per code copy (a bulk copy costs a few hundred cycles of the copy engine)

struct TArgs {
  const uint8_t* codes;
  const uint16_t* norms;
  const uint16_t* rnorms;
  int64_t n_keys;      // keys per KV head, a multiple of 32
  int group;           // query heads per KV head, 1..4
  int tb;              // bytes of one 32-key code tile
  int tiles_per_head;  // ceil(n_keys / 128)
  int64_t n_items;     // n_kv_heads * tiles_per_head (below 2^31)
  uint32_t per_cta, rem_cta;  // n_items = per_cta * gridDim.x + rem_cta
  const float* q;      // [n_kv_heads * group][d] fp32
  int d;
  int kb;
  int m;
  const float* cent;   // codebook centroids (2^kb)
  const int8_t* D;     // sign flips [128]
  const uint16_t* S;   // QJL matrix, fp16 [m][128]
  float* logits;
  int64_t ld;          // logits row stride
  float kappa;         // sqrt(pi/2) / m
  int stages;          // ring stages of GI items (<= MAX_STAGES)
};

template <int KB, int SI>
struct TL {
  static constexpr int NT = KB == 1 ? 1 : (KB == 2 ? 2 : 4);  // Walsh planes
  static constexpr int NP = NT + SI;                          // planes in A
  static constexpr int ACOLS = 32 * NP;                       // tensor-memory columns of one A buffer
  static constexpr int CSTEPS = 4 * NT;                       // centroid MMAs per item (K = 32 bytes each)
  static constexpr int SSTEPS = 4 * SI;                       // sign MMAs per item
  // B image of one KV head: 4 per-query float4 scalars, then the centroid digits
  // (16 rows x NT*128 bytes) and the sign digits (16 rows x 128 bytes), each in the
  // canonical K-major layout: 16-byte K chunk kc at kc*256, 8-row group g at g*128.
  static constexpr int IMG_C = 64;
  static constexpr int IMG_S = 64 + NT * 2048;
  static constexpr int IMG = (64 + NP * 2048 + 127) / 128 * 128;
  static constexpr int TILEB = 32 * 16 * (KB + SI);  // one 32-key code tile
  static constexpr int STAGE = GI * 4 * TILEB;       // the code tiles of GI items
  static constexpr int ACC = 32;                     // accumulator set: 16 centroid + 16 sign columns
  // Even buffer counts: item i and item i - NA (i - NB) have the same parity, so one MMA pair,
  // one expansion group and one epilogue group meet every phase of a buffer's barriers in turn.
  // (With an odd count a waiter could arrive two phases ahead, see the parity of the phase
  // before and pass without waiting.)
  static constexpr int NA = (4 * ACOLS + 2 * ACC <= 512) ? 4 : 2;
  static constexpr int NB = (NA * ACOLS + 4 * ACC <= 512) ? 4 : 2;
  static_assert(NA * ACOLS + NB * ACC <= 512, "tensor-memory budget");
  // With one A buffer per parity (NA = 2) a buffer is filled and consumed in two halves
  // (planes [0, NL) and [NL, NP)), each with its own barriers, so the expansion of an item's
  // first half can start once the MMAs of the previous item of its parity have read that half.
  static constexpr bool SPLIT = NA == 2;
  static constexpr int NL = SPLIT ? 3 : NP;
  static constexpr int W_EXP0 = 3, W_EPI0 = 11;
  static constexpr int NTHREADS = 19 * 32;
  static constexpr int OFF_IMG = 1024;
  static constexpr int OFF_PREP = OFF_IMG + 2 * IMG;  // q_rot [2][128], u [2][128], partial u [2][4][128] (float4)
  static constexpr int OFF_S = OFF_PREP + 12 * 128 * 16;     // S, fp16 [128][128], chunks swizzled (SI)
  static constexpr int OFF_RING = OFF_S + (SI ? 128 * 256 : 0);
  static constexpr int smem(int stages) { return OFF_RING + stages * STAGE; }
};

// frexpf's exponent (x = f 2^e, 0.5 <= f < 1) and 2^k from the fp32 bit pattern
// for normal values (exact), the library calls otherwise.
__device__ __forceinline__ int exponent_of(float x) {
  const uint32_t b = __float_as_uint(x) & 0x7FFFFFFFu;
  if (b >= 0x00800000u && b < 0x7F800000u) return (int)(b >> 23) - 126;
  int e;
  frexpf(x, &e);
  return e;
}
__device__ __forceinline__ float pow2(int k) {
  return (k >= -126 && k <= 127) ? __uint_as_float((uint32_t)(127 + k) << 23) : ldexpf(1.f, k);
}

// warp maximum of a float (redux.sync; finite, non-negative values here)
__device__ __forceinline__ float warp_max_redux(float v) {
  float r;
  asm volatile("redux.sync.max.NaN.f32 %0, %1, 0xffffffff;\n" : "=f"(r) : "f"(v));
  return r;
}

// Global loads of the query preparation, issued early so their latency overlaps
// other work: warp ew's query (image ew / 4, query ew % 4), the sign flips and
// 16-byte chunks et + 256 k of S (coalesced; make_images stores them to shared
// memory).  The loaded values are only stored here (no arithmetic or select on
// them), so the loads do not hold the warp before their first use; out-of-range
// elements load from a valid address and are zeroed by `ymask` in make_images.
struct PrepRegs {
  float y[4];
  int ds[4];
  uint32_t ymask;  // bit i: coordinate 32 i + lane of a real query
  uint4 sv[8];     // S chunks (SI; the first preparation of the CTA only)
  float cv;        // centroid et (et < 2^kb; other lanes hold centroid 0)
};

template <int SI>
__device__ __forceinline__ void prep_load(const TArgs& a, int64_t head0, int n_img, int et, PrepRegs& pr,
                                          bool with_s) {
  const int ew = et >> 5, lane = et & 31;
  const int k = ew >> 2, j = ew & 3;
  const bool valid = k < n_img && j < a.group;
  pr.cv = __ldg(a.cent + (et < (1 << a.kb) ? et : 0));
  const int64_t row = valid ? (head0 + k) * a.group + j : 0;
  pr.ymask = 0u;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int c = 32 * i + lane;
    const bool ok = valid && c < a.d;
    pr.ymask |= ok ? (1u << i) : 0u;
    pr.y[i] = __ldg(a.q + (ok ? row * a.d + c : 0));
    pr.ds[i] = __ldg(a.D + c);
  }
  if constexpr (SI) {  // m = 128: S is 32 KB
    if (with_s) {
#pragma unroll
      for (int k = 0; k < 8; ++k) pr.sv[k] = __ldg(reinterpret_cast<const uint4*>(a.S) + et + 256 * k);
    }
  }
}

// Partial sums of u = S q_rot for up to two query images: thread x of NQ * 128 takes row
// i = x % 128 and the 128 / NQ coordinates of part x / 128; up[(NQ im + part) 128 + i]
// receives its sums for the 4 queries of image im.  S sits in shared memory with 16-byte
// chunk c of row r at r * 16 + (c ^ (r & 15)) (8 consecutive rows read 8 banks apart).
template <int NQ>
__device__ __forceinline__ void sq_part(const float4* qT, const uint8_t* sS, float4* up, int n_img, int x) {
  constexpr int NC = 16 / NQ;  // 16-byte chunks (8 coordinates) per part
  const int i = x & 127, part = x >> 7;
  float2 acc[2][2];  // [image][queries 0-1, 2-3], packed fp32x2
#pragma unroll
  for (int im = 0; im < 2; ++im) acc[im][0] = acc[im][1] = make_float2(0.f, 0.f);
#pragma unroll
  for (int k = 0; k < NC; ++k) {
    const int c = NC * part + k;
    const uint4 sv = reinterpret_cast<const uint4*>(sS)[i * 16 + (c ^ (i & 15))];
    const uint32_t wv[4] = {sv.x, sv.y, sv.z, sv.w};
#pragma unroll
    for (int h2 = 0; h2 < 4; ++h2) {
      const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&wv[h2]));
      const float2 fx = make_float2(f.x, f.x), fy = make_float2(f.y, f.y);
      const int j = 8 * c + 2 * h2;
#pragma unroll
      for (int im = 0; im < 2; ++im) {
        if (im < n_img) {
          const float4 q0 = qT[128 * im + j], q1 = qT[128 * im + j + 1];
          acc[im][0] = __ffma2_rn(fy, make_float2(q1.x, q1.y), __ffma2_rn(fx, make_float2(q0.x, q0.y), acc[im][0]));
          acc[im][1] = __ffma2_rn(fy, make_float2(q1.z, q1.w), __ffma2_rn(fx, make_float2(q0.z, q0.w), acc[im][1]));
        }
      }
    }
  }
#pragma unroll
  for (int im = 0; im < 2; ++im)
    if (im < n_img) up[(NQ * im + part) * 128 + i] = make_float4(acc[im][0].x, acc[im][0].y, acc[im][1].x, acc[im][1].y);
}

// B images of n_img (1 or 2) consecutive KV heads into img0 / img1, by the 256
// threads of warps 11-18 (et = 0..255) from the loads in pr.  Steps:
// q_rot = H D q / sqrt(128) (warp per query: image ew / 4, query ew % 4);
// u = S q_rot (sq_part: a half row of S per thread, or, WIDE, a quarter row with
// the 8 expansion warps joining between two 512-thread named barriers);
// per-query scales 2^F, 2^G putting the largest weight just below 2^23; digits.
template <int KB, int SI, bool WIDE, class Sync>
__device__ void make_images(const TArgs& a, PrepRegs& pr, int n_img, uint8_t* img0, uint8_t* img1, float4* qT,
                            float4* uT, float4* up, const float* alpha, float* red, uint8_t* sS, bool with_s,
                            int et, Sync&& sync) {
  using L = TL<KB, SI>;
  const int ew = et >> 5, lane = et & 31;
  const int kq = ew >> 2, jq = ew & 3;  // this warp's image and query
  float* qTf = reinterpret_cast<float*>(qT);  // [2][128][4]
  float* uTf = reinterpret_cast<float*>(uT);  // [2][128][4]
  float* rd = red + 16 * kq;                  // per query of image kq: sum, max, 2^F, 2^G
  {
    float* y = pr.y;
#pragma unroll
    for (int i = 0; i < 4; ++i) y[i] = ((pr.ymask >> i) & 1u) ? y[i] * (float)pr.ds[i] : 0.f;
#pragma unroll
    for (int h = 1; h < 4; h <<= 1)
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if ((i & h) == 0) {
          const float u = y[i], w = y[i + h];
          y[i] = u + w;
          y[i + h] = u - w;
        }
#pragma unroll
    for (int sft = 1; sft < 32; sft <<= 1)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float o = __shfl_xor_sync(FULL, y[i], sft);
        y[i] = (lane & sft) ? (o - y[i]) : (y[i] + o);
      }
    float sum = 0.f, mx = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float v = y[i] * 0.08838834764831845f;  // 1/sqrt(128)
      qTf[512 * kq + 4 * (32 * i + lane) + jq] = v;
      sum += v;
      mx = fmaxf(mx, fabsf(v));
    }
    sum = warp_sum(sum);
    mx = warp_max_redux(mx);
    if (lane == 0) {
      rd[4 * jq] = sum;
      rd[4 * jq + 1] = mx;
    }
  }
  if constexpr (SI) {  // S into shared memory (kept for the CTA's later preparations): 16-byte chunk c of
    // row r at r * 16 + (c ^ (r & 15)), so both a row's 16 chunks (stored here) and one chunk of 8
    // consecutive rows (read below) fall in distinct banks
    if (with_s) {
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int g = et + 256 * k, r = g >> 4, c = g & 15;
        reinterpret_cast<uint4*>(sS)[r * 16 + (c ^ (r & 15))] = pr.sv[k];
      }
    }
  }
  if constexpr (SI && WIDE) {
    // u = S q_rot by the 8 expansion warps as well (threads 256 .. 511 of named barrier 2): a
    // quarter row each
    named_sync(2, 512);
    sq_part<4>(qT, sS, up, n_img, et);
    named_sync(2, 512);
  } else {
    sync();
    if constexpr (SI) {  // a half row per thread
      sq_part<2>(qT, sS, up, n_img, et);
      sync();
    }
  }
  if constexpr (SI) {
    constexpr int NQ = WIDE ? 4 : 2;
    const int im = et >> 7, r = et & 127;  // thread = (image, row)
    if (im < n_img) {
      float4 t = up[(NQ * im) * 128 + r];
#pragma unroll
      for (int pp = 1; pp < NQ; ++pp) {
        const float4 v = up[(NQ * im + pp) * 128 + r];
        t = make_float4(t.x + v.x, t.y + v.y, t.z + v.z, t.w + v.w);
      }
      uT[128 * im + r] = t;
    }
    sync();
  }
  if (kq < n_img) {  // scales and per-query scalars: warp = (image kq, query jq)
    float su = 0.f, mu = 0.f;
    if constexpr (SI) {  // m = 128 rows of S
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float v = uTf[512 * kq + 4 * (lane + 32 * k) + jq];
        su += v;
        mu = fmaxf(mu, fabsf(v));
      }
      su = warp_sum(su);
      mu = warp_max_redux(mu);
    }
    float amax = 0.f;
#pragma unroll
    for (int T = 0; T < L::NT; ++T) amax = fmaxf(amax, fabsf(alpha[T]));
    const float mc = 2.f * amax * rd[4 * jq + 1], ms = 2.f * mu;
    const int F = mc > 0.f ? 23 - exponent_of(mc) : 0;
    const int G = ms > 0.f ? 23 - exponent_of(ms) : 0;
    if (lane == 0) {
      rd[4 * jq + 2] = pow2(F);
      rd[4 * jq + 3] = pow2(G);
      // sum_T alpha_T = c[L-1] (all index bits set)
      reinterpret_cast<float4*>(kq ? img1 : img0)[jq] =
          make_float4(pow2(-(F + 7)), alpha[4] * rd[4 * jq], pow2(-(G + 7)), su);
    }
  }
  sync();
  // Digit words, one thread per (image, query q, plane P, bit class c, word w): the
  // weights of coordinates 32w + 8b + c (b = 0..3) give word w of K chunk c of plane P
  // in the 4 digit rows 4q + d.  Scaling by 2^F (2^G) is exact.
  constexpr int PER = 4 * L::NP * 32;
  for (int e = et; e < n_img * PER; e += 256) {
    const int im = e / PER, e2 = e - im * PER;
    // lanes run over (w, bit 0 of q, 4 bit classes): their word stores fall in 8 banks
    const int w = e2 & 3, c = (e2 >> 3) & 7, pq = e2 >> 6;
    const int qh = pq / L::NP, P = pq - qh * L::NP, q = 2 * qh + ((e2 >> 2) & 1);
    const bool cen = P < L::NT;
    const float* r2 = red + 16 * im;
    const float scale = cen ? 2.f * alpha[P] * r2[4 * q + 2] : 2.f * r2[4 * q + 3];
    const float* src = (cen ? qTf : uTf) + 512 * im;
    uint32_t W[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int j = 32 * w + 8 * b + c;
      int X = (cen || j < a.m) ? __float2int_rn(src[4 * j + q] * scale) * (1 << (7 - c)) : 0;
#pragma unroll
      for (int dd = 0; dd < 3; ++dd) {
        const int lowb = (int)(int8_t)(X & 0xFF);
        W[dd] |= (uint32_t)(uint8_t)lowb << (8 * b);
        X = (X - lowb) >> 8;
      }
      W[3] |= (uint32_t)(uint8_t)X << (8 * b);
    }
    const int kc = cen ? 8 * P + c : c;
    uint8_t* base = (im ? img1 : img0) + (cen ? L::IMG_C : L::IMG_S) + kc * 256 + (q >> 1) * 128 + 4 * w;
#pragma unroll
    for (int dd = 0; dd < 4; ++dd) *reinterpret_cast<uint32_t*>(base + (4 * (q & 1) + dd) * 16) = W[dd];
  }
  fence_async_smem();  // the images are read by the tensor core (async proxy)
  sync();
}

// The code tiles of the next GI items (or fewer, at the end of the CTA's range of nleft items)
// into one stage: one bulk copy when the tiles are contiguous in global memory (every item but
// the last of the group holds 128 keys), else one per item.  (head, t) is the next item's KV
// head and 128-key tile, advanced here (no integer division on the producer's path).
template <int KB, int SI>
__device__ __forceinline__ void copy_group(const TArgs& a, int nleft, int64_t& head, int& t, uint8_t* dst,
                                           uint64_t* bar) {
  using L = TL<KB, SI>;
  int64_t tile[GI];
  int nt[GI];
  uint32_t total = 0;
  bool whole = true;
#pragma unroll
  for (int j = 0; j < GI; ++j) {
    nt[j] = 0;
    tile[j] = 0;
    if (j < nleft) {
      const int64_t k0 = (int64_t)t * TK;
      const int64_t nk = a.n_keys - k0 < TK ? a.n_keys - k0 : TK;
      tile[j] = (head * a.n_keys + k0) >> 5;
      nt[j] = (int)(nk >> 5);
      total += (uint32_t)(nt[j] * L::TILEB);
      if (j + 1 < nleft && j + 1 < GI && nt[j] != 4) whole = false;
      if (++t == a.tiles_per_head) t = 0, ++head;
    }
  }
  mbar_expect_tx(bar, total);
  if (whole) {
    bulk_g2s(dst, a.codes + tile[0] * L::TILEB, total, bar);
  } else {
#pragma unroll
    for (int j = 0; j < GI; ++j)
      if (nt[j] > 0) bulk_g2s(dst + j * 4 * L::TILEB, a.codes + tile[j] * L::TILEB, nt[j] * L::TILEB, bar);
  }
}

template <int KB, int SI>
__global__ void __launch_bounds__(TL<KB, SI>::NTHREADS, 1) logits_tc_kernel(const TArgs a) {
  using L = TL<KB, SI>;
  constexpr int W_EXP0 = L::W_EXP0, W_EPI0 = L::W_EPI0;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);  // [MAX_STAGES] stage loaded
  uint64_t* empty = full + MAX_STAGES;                 // [MAX_STAGES] stage read by the 8 expansion warps
  uint64_t* afull = empty + MAX_STAGES;                // [4] A buffer (SPLIT: half 2b + h) written (4 arrivals)
  uint64_t* mdone = afull + 4;                         // [4] its MMAs done: the buffer (half) is free (1)
  uint64_t* cfull = mdone + 4;                         // [4] accumulator set full (1)
  uint64_t* accfree = cfull + 4;                       // [4] accumulator set read (4)
  uint64_t* imgfull = accfree + 4;                     // [2] B image ready (1)
  uint64_t* imgfree = imgfull + 2;                     // [2] no MMA reads the B image any more (2)
  uint64_t* gbar = imgfree + 2;                        // barrier of the 8 prep / epilogue warps (8)
  uint32_t* tbase = reinterpret_cast<uint32_t*>(gbar + 1);
  float* alpha = reinterpret_cast<float*>(tbase + 4);  // [5] Walsh coefficients, then c[L-1]
  float* red = alpha + 8;                              // [2][16] per image and query: sum, max, 2^F, 2^G
  uint8_t* imgs = smem + L::OFF_IMG;
  float4* qT = reinterpret_cast<float4*>(smem + L::OFF_PREP);
  float4* uT = qT + 256;
  float4* up = uT + 256;
  uint8_t* ring = smem + L::OFF_RING;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = a.stages;
  grid_dependents_launch();  // every global write below follows this grid's own dependency wait
  // this CTA's items [i0, i1) = [b n_items / G, (b + 1) n_items / G), in 32-bit arithmetic
  // (a 64-bit division costs hundreds of cycles on the start-up path)
  const uint32_t bx = blockIdx.x;
  const uint32_t u0 = bx * a.per_cta + bx * a.rem_cta / gridDim.x;
  const uint32_t u1 = (bx + 1) * a.per_cta + (bx + 1) * a.rem_cta / gridDim.x;
  const int64_t i0 = u0;
  const int n = (int)(u1 - u0);
  const uint32_t tph = (uint32_t)a.tiles_per_head;
  const int64_t h_first = u0 / tph;
  const int t_first = (int)(u0 - (uint32_t)h_first * tph);
  const int n_img = n > 0 ? (int)((u1 - 1) / tph - (uint32_t)h_first) + 1 : 0;
  const int n_groups = (n + GI - 1) / GI;

  if (threadIdx.x == 0) {
    for (int s = 0; s < MAX_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 8);  // the 4 expansion warps of each of the GI = 2 items
    }
    for (int b = 0; b < 4; ++b) {
      mbar_init(&afull[b], 4);
      mbar_init(&mdone[b], 1);
    }
    for (int c = 0; c < 4; ++c) {
      mbar_init(&cfull[c], 1);
      mbar_init(&accfree[c], 4);
    }
    for (int k = 0; k < 2; ++k) {
      mbar_init(&imgfull[k], 1);
      mbar_init(&imgfree[k], 2);
    }
    mbar_init(gbar, 8);
  }

  PrepRegs pr;
  // epilogue warps: the norms of key 32 qd + lane of an item, plain loads issued two of the warp's
  // items (four items) ahead; (nh, ntl) walks the items being loaded, nidx is the next one's index
  const int epar = ((warp - W_EPI0) >> 2) & 1;
  int64_t nh = h_first;
  int ntl = t_first, nidx = 0;
  // (raw fp16 bits, converted where used; keys past the range load key 0 and are never used)
  auto norms_next = [&](uint16_t& nr, uint16_t& ga) {  // item nidx, then advance the walk by 2
    const int64_t key = (int64_t)ntl * TK + 32 * (warp & 3) + lane;
    const int64_t at = (nidx < n && key < a.n_keys) ? nh * a.n_keys + key : 0;
    nr = __ldg(a.norms + at);
    if constexpr (SI) ga = __ldg(a.rnorms + at);
    nidx += 2;
    ntl += 2;
    while (ntl >= a.tiles_per_head) ntl -= a.tiles_per_head, ++nh;
  };
  uint16_t nrm0 = 0, gam0 = 0, nrm1 = 0, gam1 = 0;
  if (warp >= W_EPI0) {  // the first one or two heads' query loads overlap the set-up
    grid_dependency_wait();  // queries and norms may come from the preceding kernel in the stream
    prep_load<SI>(a, h_first, n_img < 2 ? n_img : 2, threadIdx.x - 32 * W_EPI0, pr, true);
    if (epar) {  // this group's first item is item 1
      nidx = 1;
      if (++ntl == a.tiles_per_head) ntl = 0, ++nh;
    }
    norms_next(nrm0, gam0);
    norms_next(nrm1, gam1);
  }
  if (warp == 0) tmem_alloc(tbase, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tbase;
  // tensor-memory columns: accumulator sets (64 each), then the A buffers
  auto acc_col = [&](int c) { return tmem + (uint32_t)(L::ACC * c); };
  auto a_col = [&](int b) { return tmem + (uint32_t)(L::ACC * L::NB + b * L::ACOLS); };

  if (warp == 0) {
    // ---------------- producer: code tiles into the ring, GI items per stage ----------------
    grid_dependency_wait();  // codes may come from the preceding kernel in the stream
    if (lane == 0) {
      int64_t ph = h_first;  // the next item's KV head and tile
      int pt = t_first;
      int issued = 0;
      for (int g = 0, s = 0, use = 0; g < n_groups; ++g) {
        if (use >= 1 && !mbar_wait(&empty[s], (use - 1) & 1)) break;
        copy_group<KB, SI>(a, n - GI * g, ph, pt, ring + s * L::STAGE, &full[s]);
        issued = g + 1;
        if (++s == S) s = 0, ++use;
      }
      // nothing may still be in flight into shared memory when the CTA ends
      for (int g = (issued > S ? issued - S : 0); g < issued; ++g) mbar_wait(&full[g % S], (g / S) & 1);
    }
  } else if (warp < W_EXP0) {
    // ---------------- MMA issue (warp-uniform, elected lane) ----------------
    const int par = warp - 1;
    constexpr uint32_t idesc = idesc_u8s8_s32(TK, 16);
    int t = t_first;
    int kimg = 0;
    bool ok = n > 0 && mbar_wait(&imgfull[0], 0);
    uint32_t simg = smem_u32(imgs);
    for (int i = 0; i < n && ok; ++i, ++t) {
      if (t == a.tiles_per_head) {  // next KV head: release the old image, wait for the next one
        t = 0;
        __syncwarp();
        umma_commit_elect(&imgfree[kimg & 1]);
        ++kimg;
        if (!mbar_wait(&imgfull[kimg & 1], (kimg >> 1) & 1)) break;
        simg = smem_u32(imgs + (kimg & 1) * L::IMG);
      }
      if ((i & 1) != par) continue;
      const int b = i % L::NA, ua = i / L::NA, c = i % L::NB, cu = i / L::NB;
      const int h0 = L::SPLIT ? 2 * b : b;  // barrier of the buffer's first half (or of the buffer)
      if (!mbar_wait(&afull[h0], ua & 1)) break;
      if (cu >= 1 && !mbar_wait(&accfree[c], (cu - 1) & 1)) break;
      __syncwarp();  // elect.sync needs the whole warp converged
      tc_fence_after();
      const uint32_t dacc = acc_col(c);
      const uint32_t abuf = a_col(b);
      const uint64_t dc = smem_desc(simg + L::IMG_C, 256, 128);
      const uint64_t ds = smem_desc(simg + L::IMG_S, 256, 128);
      // K step u of plane P = u / 4: 8 A columns (32 bytes), 512 bytes of image
      auto plane_mmas = [&](int P) {
        if (P < L::NT) {
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)
            umma_i8_ts_elect(dacc, abuf + 32u * P + 8u * ks, dc + (uint64_t)(32 * (4 * P + ks)), idesc,
                             (P > 0 || ks > 0) ? 1u : 0u);
        } else {
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)
            umma_i8_ts_elect(dacc + 16u, abuf + 32u * P + 8u * ks, ds + (uint64_t)(32 * ks), idesc, ks > 0 ? 1u : 0u);
        }
      };
#pragma unroll
      for (int P = 0; P < L::NL; ++P) plane_mmas(P);
      if constexpr (L::SPLIT) {
        umma_commit_elect(&mdone[h0]);
        if (!mbar_wait(&afull[h0 + 1], ua & 1)) break;
        __syncwarp();
        tc_fence_after();
#pragma unroll
        for (int P = L::NL; P < L::NP; ++P) plane_mmas(P);
        umma_commit_elect(&mdone[h0 + 1]);
      } else {
        umma_commit_elect(&mdone[b]);
      }
      umma_commit_elect(&cfull[c]);
    }
    __syncwarp();
  } else if (warp < W_EPI0) {
    // ---------------- expansion: code bits -> A in tensor memory ----------------
    // warps 3-6 take the even items, 7-10 the odd ones; each covers one lane quadrant
    // (a 32-key tile of the item) and all 8 bit classes of every plane.  First they take a
    // share of the CTA's first query preparation (u = S q_rot, between two named barriers
    // with the 8 preparation warps).
    const int ew = warp - W_EXP0;
    const int qd = warp & 3, par = ew >> 2;
    if constexpr (SI) {
      if (n_img > 0) {
        named_sync(2, 512);
        sq_part<4>(qT, smem + L::OFF_S, up, n_img < 2 ? n_img : 2, 256 + 32 * ew + lane);
        named_sync(2, 512);
      }
    }
    for (int i = par, s = 0, use = 0; i < n; i += 2) {  // item i sits in group i / 2: stage s, pass use
      const int b = i % L::NA, ua = i / L::NA;
      const int h0 = L::SPLIT ? 2 * b : b;
      if (!mbar_wait(&full[s], use & 1)) break;
      if (ua >= 1 && !mbar_wait(&mdone[h0], (ua - 1) & 1)) break;  // MMAs of item i - NA have read A[b] (half 0)
      const uint8_t* st = ring + s * L::STAGE + (i % GI) * 4 * L::TILEB + qd * L::TILEB + lane * 16;
      uint4 pw[KB + SI];
#pragma unroll
      for (int p = 0; p < KB + SI; ++p) pw[p] = *reinterpret_cast<const uint4*>(st + p * 512);
      release_to_copy(&empty[s], lane);  // the stage is refilled once its 8 readers release it
      if (++s == S) s = 0, ++use;
      uint4 it[L::NP];
#pragma unroll
      for (int T = 0; T < L::NT; ++T) it[T] = pw[T < KB ? T : 0];
      if constexpr (KB == 3)
        it[3] = make_uint4(pw[0].x ^ pw[1].x ^ pw[2].x, pw[0].y ^ pw[1].y ^ pw[2].y, pw[0].z ^ pw[1].z ^ pw[2].z,
                           pw[0].w ^ pw[1].w ^ pw[2].w);
      if constexpr (SI) it[L::NT] = pw[KB];
      const uint32_t lanebase = a_col(b) + ((uint32_t)(32 * qd) << 16);
      bool okh = true;
#pragma unroll
      for (int P = 0; P < L::NP; ++P) {
        if (L::SPLIT && P == L::NL) {  // first half done; the second half's previous MMAs must be done
          tmem_st_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&afull[h0]);
          if (ua >= 1 && !mbar_wait(&mdone[h0 + 1], (ua - 1) & 1)) {
            okh = false;
            break;
          }
          __syncwarp();
          tc_fence_after();
        }
#pragma unroll
        for (int cg = 0; cg < 2; ++cg) {
          uint32_t r[16];
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            const uint32_t mk = 0x01010101u << (4 * cg + cc);
            r[4 * cc + 0] = it[P].x & mk;
            r[4 * cc + 1] = it[P].y & mk;
            r[4 * cc + 2] = it[P].z & mk;
            r[4 * cc + 3] = it[P].w & mk;
          }
          tmem_st16(lanebase + 32 * P + 16 * cg, r);
        }
      }
      if (!okh) break;
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&afull[L::SPLIT ? h0 + 1 : b]);
    }
  } else {
    // ---------------- query preparation, then the epilogue ----------------
    // warps 11-14 take the even items, 15-18 the odd ones; each covers one lane quadrant
    // (32 keys) and all the query heads of the KV head
    const int et = threadIdx.x - 32 * W_EPI0;
    const int ew = warp - W_EPI0;
    const int qd = warp & 3, par = ew >> 2;
    if (et < 32) {  // Walsh coefficients of the odd-symmetric codebook (fp64), c[L-1]; lane l holds c[l]
      constexpr int Lv = 1 << KB;
      const int mask = et < L::NT ? walsh_mask(KB, et) : 0;
      double sacc = 0.0;
#pragma unroll
      for (int l = 0; l < Lv; ++l) {
        const float cl = __shfl_sync(FULL, pr.cv, l);
        sacc += (double)cl * ((__popc(l & mask) & 1) ? 1.0 : -1.0);
      }
      const float ctop = __shfl_sync(FULL, pr.cv, Lv - 1);
      if (et < L::NT) alpha[et] = (float)(sacc / Lv);
      if (et == 0) alpha[4] = ctop;
    }
    GroupSync gs{gbar, 0u};
    if (n_img > 0) {
      // every prep / epilogue warp gets here once, before any wait that can give up: a
      // named barrier (its first sync also publishes alpha)
      make_images<KB, SI, true>(a, pr, n_img < 2 ? n_img : 2, imgs, imgs + L::IMG, qT, uT, up, alpha, red,
                                smem + L::OFF_S, true, et,
                          [] { named_sync(1, 256); });
      if (et == 0) {
        mbar_arrive(&imgfull[0]);
        if (n_img > 1) mbar_arrive(&imgfull[1]);
      }
    }
    int64_t head = h_first;
    int t = t_first;
    int kimg = 0;
    for (int i = 0; i < n; ++i, ++t) {
      if (t == a.tiles_per_head) {
        t = 0, ++head, ++kimg;
        const int kn = kimg + 1;  // the next head's image, into the slot image kimg - 1 used
        if (kn >= 2 && kn < n_img) {
          mbar_wait(&imgfree[kn & 1], ((kn - 2) >> 1) & 1);  // on a time-out the fault word is set; go on
          PrepRegs pr2;
          prep_load<SI>(a, head + 1, 1, et, pr2, false);
          uint8_t* slot = imgs + (kn & 1) * L::IMG;
          make_images<KB, SI, false>(a, pr2, 1, slot, slot, qT, uT, up, alpha, red, smem + L::OFF_S, false, et,
                                     [&] { gs.sync(lane); });
          if (et == 0) mbar_arrive(&imgfull[kn & 1]);
        }
      }
      if ((i & 1) != par) continue;
      const int c = i % L::NB, cu = i / L::NB;
      const int64_t key = (int64_t)t * TK + 32 * qd + lane;
      const bool kvalid = key < a.n_keys;
      const float nrm = __half2float(__ushort_as_half(nrm0)), gam = SI ? __half2float(__ushort_as_half(gam0)) : 0.f;
      nrm0 = nrm1;
      gam0 = gam1;
      norms_next(nrm1, gam1);  // item i + 4
      if (!mbar_wait(&cfull[c], cu & 1)) break;
      tc_fence_after();
      const uint32_t lrow = acc_col(c) + ((uint32_t)(32 * qd) << 16);
      uint32_t C[16], Z[16];  // 4 queries x 4 digits, centroid and sign sums (exact int32, below 2^24)
      if constexpr (SI) {
        tmem_ld16_issue(lrow, C);
        tmem_ld16_issue(lrow + 16, Z);
        tmem_ld_wait16x2(C, Z);
      } else {
        tmem_ld16_issue(lrow, C);
        tmem_ld_wait16(C);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&accfree[c]);
      const float4* qs = reinterpret_cast<const float4*>(imgs + (kimg & 1) * L::IMG);
#pragma unroll
      for (int qi = 0; qi < 4; ++qi) {
        if (qi < a.group && kvalid) {
          const float4 sc = qs[qi];
          // sum_d 256^d C[d]: each C[d] an exact int32 below 2^24; one fp32 rounding per step
          const float cen = fmaf((float)(int)C[4 * qi + 3], 16777216.f,
                                 fmaf((float)(int)C[4 * qi + 2], 65536.f,
                                      fmaf((float)(int)C[4 * qi + 1], 256.f, (float)(int)C[4 * qi])));
          float l = fmaf(cen, sc.x, -sc.y);
          if constexpr (SI) {
            const float sg = fmaf((float)(int)Z[4 * qi + 3], 16777216.f,
                                  fmaf((float)(int)Z[4 * qi + 2], 65536.f,
                                       fmaf((float)(int)Z[4 * qi + 1], 256.f, (float)(int)Z[4 * qi])));
            l = fmaf(gam * a.kappa, fmaf(sg, sc.z, -sc.w), l);
          }
          a.logits[(head * a.group + qi) * a.ld + key] = nrm * l;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

template <int KB, int SI>
int launch_tc(const TArgs& a0, int sm, cudaStream_t st) {
  using L = TL<KB, SI>;
  TArgs a = a0;
  a.stages = MAX_STAGES;
  while (a.stages > 4 && L::smem(a.stages) > 200 * 1024) --a.stages;
  // at least 120 KB: one CTA per SM, so no second CTA waits for the SM's tensor memory
  const int bytes = std::max(L::smem(a.stages), 120 * 1024);
  auto kern = logits_tc_kernel<KB, SI>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return tq::set_error(TQ_ECUDA, "tq_logits: %s", cudaGetErrorString(e));
  cudaLaunchConfig_t cfg = {};
  const int64_t grid = std::max<int64_t>(1, std::min<int64_t>(sm, a.n_items));
  a.per_cta = (uint32_t)(a.n_items / grid);
  a.rem_cta = (uint32_t)(a.n_items % grid);
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(L::NTHREADS);
  cfg.dynamicSmemBytes = bytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, a);
  if (e != cudaSuccess) return tq::set_error(TQ_ECUDA, "tq_logits: launch failed: %s", cudaGetErrorString(e));
  return TQ_OK;
}

}  // namespace

namespace tq {

bool logits_tc_supported(int dp, int kb, int m, int group, int64_t n_keys, const void* norms, const void* rnorms) {
  return dp == 128 && kb >= 1 && kb <= 3 && (m == 0 || m == 128) && group >= 1 && group <= 4 && n_keys % 32 == 0 &&
         aligned(norms, 16) && (m == 0 || aligned(rnorms, 16));
}

// The fused scan: query preparation inside the kernel, no workspace.
int launch_logits_tc(int kb, int m, const float* q, int d, const float* cent, const int8_t* D, const uint16_t* S,
                     const void* codes, const uint16_t* norms, const uint16_t* rnorms, int64_t n_keys,
                     int n_kv_heads, int group, float* logits, int64_t ld, cudaStream_t st) {
  TArgs a;
  a.codes = static_cast<const uint8_t*>(codes);
  a.norms = norms;
  a.rnorms = rnorms;
  a.n_keys = n_keys;
  a.group = group;
  a.tb = tqd::tile_bytes(128, kb, m);
  a.tiles_per_head = (int)((n_keys + TK - 1) / TK);
  a.n_items = (int64_t)n_kv_heads * a.tiles_per_head;
  a.q = q;
  a.d = d;
  a.kb = kb;
  a.m = m;
  a.cent = cent;
  a.D = D;
  a.S = S;
  a.logits = logits;
  a.ld = ld;
  a.kappa = (float)(std::sqrt(M_PI / 2.0) / (m > 0 ? m : 1));
  a.stages = MAX_STAGES;
  if (a.n_items >= (int64_t(1) << 31)) return set_error(TQ_EINVAL, "tq_logits: more than 2^31 tiles of 128 keys");
  const int sm = sm_count();
  if (m > 0) {
    switch (kb) {
      case 1: return launch_tc<1, 1>(a, sm, st);
      case 2: return launch_tc<2, 1>(a, sm, st);
      default: return launch_tc<3, 1>(a, sm, st);
    }
  }
  switch (kb) {
    case 1: return launch_tc<1, 0>(a, sm, st);
    case 2: return launch_tc<2, 0>(a, sm, st);
    default: return launch_tc<3, 0>(a, sm, st);
  }
}

}  // namespace tq

namespace tq {
// Read (and optionally clear) this translation unit's device fault word.
int fault_word_logits(int clear, int* value) {
  cudaError_t e = cudaMemcpyFromSymbol(value, tqd::g_fault, sizeof(int));
  if (e == cudaSuccess && clear) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(tqd::g_fault, &zero, sizeof(int));
  }
  return e == cudaSuccess ? TQ_OK : set_error(TQ_ECUDA, "tq_device_status: %s", cudaGetErrorString(e));
}
}  // namespace tq
