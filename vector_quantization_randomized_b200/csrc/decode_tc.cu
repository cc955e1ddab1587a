// tq_decode_attn with token-sliced value codes, on the fifth-generation tensor
// cores ("TurboQuant explainer" (m.163.com), "速度": attention straight from the
// codes; zhidx turboquant_plus article: asymmetric K/V - keys in the product
// code, values MSE-only).
//
//   out[b][h] = sum_t softmax_t(scale * l_t) v_hat_t,  v_hat_t = n_v,t D H c_v[idx_t] / sqrt(128)
//
// Both contractions are integer MMAs (tcgen05.mma kind::i8) on code bits:
//  * logits, as in the logits scan: A = key code bits in tensor memory (lane =
//    token, one byte 2^c * bit per coordinate of bit class c), B = base-256
//    digits of the pre-shifted weights 2 alpha_T q_rot and 2 S q_rot of the
//    pair's 4 query heads (16 rows), prepared once per (sequence, KV head);
//  * the value sum in the rotated domain, o_rot[q][j] = sum_t w_t,q c[idx_t,j]
//    with w = p * n_v: with the odd-symmetric codebook c[idx] = sum_T alpha_T
//    (2 b_T - 1) over the Walsh planes b_T of the index bits, so
//    o_rot = sum_T 2 alpha_T sum_t w_t b_T,t,j - c[L-1] sum_t w_t.  A = value bits
//    in tensor memory with lane = coordinate: the token-sliced layout stores, per
//    tile of 32 tokens, one 32-bit word per coordinate, and (word & 0x01010101 << c)
//    is the K-major byte row of 4 tokens; B = 4 base-256 digits of the weights
//    w 2^F (23 bits) pre-shifted by 7 - (token class), one image per item, each
//    Walsh plane into a 16-column accumulator of its own (combined with 2 alpha_T
//    in the epilogue).
// Integer sums stay below 2^22, so their conversion to fp32 is exact.
//
// Work: pairs (sequence, KV head) x segments of 8 items of 128 tokens; each
// unit leaves (o_rot, m, l) partials that the log-sum-exp combine merges (and
// rotates back).  One persistent CTA per SM over a contiguous range of units,
// all hand-offs on mbarriers with bounded waits:
//   warp 0       bulk copies: code tiles and norms of every item into a ring of
//                stages, the pair's query image into one of two slots;
//   warp 1       MMA issue for the logits (per key plane, into a ring of plane slots);
//   warp 2       MMA issue for the value sum (per Walsh plane);
//   warps 3-6    key bits -> tensor-memory plane slots (lane quadrant = 32 tokens);
//   warps 7-10   value words -> tensor-memory plane slots (lane quadrant = 32 coordinates);
//   warps 11-18  softmax, two groups of 4 taking alternate items, each with a running
//                maximum, sum and weight sum of its own: logits from the
//                accumulators, the weights, their digit image for the value MMAs;
//   warps 19-22  value epilogue: accumulators -> rescaled fp32 sums per coordinate,
//                one set per softmax group; a unit leaves one partial per group.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>

#include "common.h"
#include "device.cuh"
#include "prep.h"
#include "scan.cuh"
#include "tc.cuh"

namespace {
using namespace tqd;

constexpr int DP = 128;
constexpr int TK = 128;       // tokens per item
constexpr int SEG = 8;        // items per unit (segment of 1024 tokens)
constexpr int NST = 8;        // code stages
constexpr int NSK = 4;        // key plane slots (32 columns each)
constexpr int NSV = 6;        // value plane slots (32 columns each)
constexpr int NBK = 2;        // logits accumulator sets (32 columns: 16 centroid + 16 sign)
constexpr int NBV = 2;        // value accumulator sets (per Walsh plane 16 columns)

template <int KB, int VKB>
struct DL {
  static constexpr int NTK = KB == 1 ? 1 : (KB == 2 ? 2 : 4);  // key Walsh planes
  static constexpr int NPK = NTK + 1;                           // + the sign plane
  static constexpr int NTV = VKB == 1 ? 1 : (VKB == 2 ? 2 : 4);  // value Walsh planes
  // query image of a pair: 4 float4 scalars, centroid digits (NTK planes of 8 K chunks), sign digits
  static constexpr int IMG_C = 64;
  static constexpr int IMG_S = 64 + NTK * 2048;
  static constexpr int IMG = (64 + NPK * 2048 + 127) / 128 * 128;
  static constexpr int KTILE = 32 * (KB * 16 + 16);  // a 32-token key tile (m = 128)
  static constexpr int VTILE = 32 * VKB * 16;         // a 32-token value tile
  static constexpr int OFF_KN = 4 * KTILE;            // key norms, residual norms, value norms (256 B each)
  static constexpr int OFF_V = OFF_KN + 768;
  static constexpr int STAGE = OFF_V + 4 * VTILE;
  static constexpr int BVB = 2048;                    // value weight digits of an item (16 rows x 128 B)
  static constexpr int OFF_IMG = 1024;
  static constexpr int OFF_BV = OFF_IMG + 2 * IMG;
  static constexpr int OFF_ST = OFF_BV + 2 * BVB;     // stats ring: [2][16 floats]
  static constexpr int OFF_X = OFF_ST + 2 * 64;       // per softmax group: 2 x [4 warps][8] item maxima, [4][8] sums
  static constexpr int OFF_RING = (OFF_X + 2 * 384 + 127) / 128 * 128;
  static constexpr int SMEM = OFF_RING + NST * STAGE;
  static constexpr int NTHREADS = 23 * 32;
  // tensor-memory columns
  static constexpr int C_KACC = 0, C_VACC = 64, C_KS = 192, C_VS = 320;
  static_assert(C_VS + NSV * 32 <= 512, "tensor memory");
  static_assert(SMEM <= 227 * 1024, "shared memory");
};

struct DTArgs {
  const uint8_t* kcodes;
  const uint16_t* knorms;
  const uint16_t* krnorms;
  const uint8_t* vcodes;
  const uint16_t* vnorms;
  const int32_t* seq_lens;
  int64_t max_tokens;
  int hkv, group, hq, nseg;
  int64_t n_units;
  const uint8_t* img;  // [pairs][IMG]
  float* part;         // [rows][nseg][DP + 2]
  float kappa, sl2;    // sqrt(pi/2)/m; scale * log2(e)
  const float* vco;    // value codebook terms, written by the prep kernel: alpha_T [4], c[L-1], max |alpha_T|
};

// ---------------------------------------------------------------------------
// Query images, one CTA (128 threads) per pair: q_rot = H D q / sqrt(128) (warp per
// query), u = S q_rot (thread per row of S), per-query scales 2^F, 2^G (largest
// weight just below 2^23), weights shifted by 7 - c and split into 4 signed base-256
// digits (the logits scan's layout: 16-byte K chunk kc at kc * 256, 8-row group at 128).
struct DPrepArgs {
  const float* q;
  int d, kb, group, hq, hkv;
  const float* vcent;  // value codebook (2^vkb centroids)
  int vkb;
  float* vco;          // out: alpha_T [4], c[L-1], max |alpha_T| of the value codebook
  const float* cent;
  const int8_t* D;
  const uint16_t* S;
  uint8_t* img;
  int img_bytes, ntk, img_s;
};

// warp maximum of a float (redux.sync; -inf and finite values only)
__device__ __forceinline__ float warp_max_f32(float v) {
  float r;
  asm volatile("redux.sync.max.NaN.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}
// int32 |x| < 2^22 to fp32, exactly, on the FP pipe (1.5 * 2^23 + x has x in its mantissa)
__device__ __forceinline__ float i2f_exact(uint32_t x) {
  return __uint_as_float(x + 0x4B400000u) - 12582912.f;
}

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

__global__ void __launch_bounds__(128) decode_prep_tc_kernel(const DPrepArgs a) {
  __shared__ float qt[4][DP];
  __shared__ float uu[4][DP];
  __shared__ float stat[4][4];  // sum q_rot, max |q_rot|, sum u, max |u|
  __shared__ float FG[4][2];
  __shared__ float alpha[5];
  const int pair = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int b = pair / a.hkv, g = pair - b * a.hkv;
  const int NT = a.ntk, L = 1 << a.kb, np = NT + 1;
  uint8_t* img = a.img + (int64_t)pair * a.img_bytes;
  if (tid < NT) {
    const int mask = walsh_mask(a.kb, tid);
    double s = 0.0;
    for (int l = 0; l < L; ++l) s += (double)__ldg(a.cent + l) * ((__popc(l & mask) & 1) ? 1.0 : -1.0);
    alpha[tid] = (float)(s / L);
  }
  if (tid == 32) alpha[4] = __ldg(a.cent + L - 1);
  if (pair == 0 && tid == 64) {  // the value codebook's Walsh coefficients (fp64), once
    const int Lv = 1 << a.vkb, ntv = walsh_planes(a.vkb);
    float amax = 0.f;
    for (int T = 0; T < 4; ++T) {
      double s = 0.0;
      if (T < ntv) {
        const int mask = walsh_mask(a.vkb, T);
        for (int l = 0; l < Lv; ++l) s += (double)__ldg(a.vcent + l) * ((__popc(l & mask) & 1) ? 1.0 : -1.0);
        s /= Lv;
      }
      a.vco[T] = (float)s;
      amax = fmaxf(amax, fabsf((float)s));
    }
    a.vco[4] = __ldg(a.vcent + Lv - 1);
    a.vco[5] = amax;
  }
  {  // warp j: query j of the pair
    const int j = warp;
    const bool valid = j < a.group;
    const int64_t row = (int64_t)b * a.hq + (int64_t)g * a.group + j;
    float y[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int c = 32 * i + lane;
      y[i] = (valid && c < a.d) ? __ldg(a.q + row * a.d + c) * (float)__ldg(a.D + c) : 0.f;
    }
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
      qt[j][32 * i + lane] = v;
      sum += v;
      mx = fmaxf(mx, fabsf(v));
    }
    sum = warp_sum(sum);
    mx = warp_max(mx);
    if (lane == 0) {
      stat[j][0] = sum;
      stat[j][1] = mx;
    }
  }
  __syncthreads();
  {  // u = S q_rot: thread = row of S
    const int i = tid;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    const uint4* srow = reinterpret_cast<const uint4*>(a.S + (size_t)i * DP);
#pragma unroll 4
    for (int k = 0; k < DP / 8; ++k) {
      const uint4 v = __ldg(srow + k);
      const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int h2 = 0; h2 < 4; ++h2) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&wv[h2]));
        const int c = 8 * k + 2 * h2;
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[j] = fmaf(f.y, qt[j][c + 1], fmaf(f.x, qt[j][c], acc[j]));
      }
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) uu[j][i] = acc[j];
  }
  __syncthreads();
  {
    const int j = warp;
    float su = 0.f, mu = 0.f;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const float v = uu[j][lane + 32 * r];
      su += v;
      mu = fmaxf(mu, fabsf(v));
    }
    su = warp_sum(su);
    mu = warp_max(mu);
    if (lane == 0) {
      float amax = 0.f;
      for (int T = 0; T < NT; ++T) amax = fmaxf(amax, fabsf(alpha[T]));
      const float mc = 2.f * amax * stat[j][1], ms = 2.f * mu;
      const int F = mc > 0.f ? 23 - exponent_of(mc) : 0;
      const int G = ms > 0.f ? 23 - exponent_of(ms) : 0;
      FG[j][0] = pow2(F);
      FG[j][1] = pow2(G);
      reinterpret_cast<float4*>(img)[j] = make_float4(pow2(-(F + 7)), alpha[4] * stat[j][0], pow2(-(G + 7)), su);
    }
  }
  __syncthreads();
  // digit words: item (query j, plane P, bit class c, word w): the weights of coordinates
  // 32w + 8bb + c (bb = 0..3) are bytes 4w + bb of K chunk c of plane P, rows 4j + digit
  for (int e = tid; e < 4 * np * 32; e += 128) {
    const int w = e & 3, c = (e >> 2) & 7, pq = e >> 5;
    const int j = pq / np, P = pq - j * np;
    const bool cen = P < NT;
    const float scale = cen ? 2.f * alpha[P] * FG[j][0] : 2.f * FG[j][1];
    const float* src = cen ? qt[j] : uu[j];
    uint32_t W[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int bb = 0; bb < 4; ++bb) {
      const int co = 32 * w + 8 * bb + c;
      int X = __float2int_rn(src[co] * scale) * (1 << (7 - c));
#pragma unroll
      for (int dd = 0; dd < 3; ++dd) {
        const int lowb = (int)(int8_t)(X & 0xFF);
        W[dd] |= (uint32_t)(uint8_t)lowb << (8 * bb);
        X = (X - lowb) >> 8;
      }
      W[3] |= (uint32_t)(uint8_t)X << (8 * bb);
    }
    const int kc = cen ? 8 * P + c : c;
    uint8_t* base = img + (cen ? 64 : a.img_s) + kc * 256 + (j >> 1) * 128 + 4 * w;
#pragma unroll
    for (int dd = 0; dd < 4; ++dd) *reinterpret_cast<uint32_t*>(base + (4 * (j & 1) + dd) * 16) = W[dd];
  }
}

// ---------------------------------------------------------------------------
// the item walk shared by every role: unit u -> (pair, segment) -> items
struct Walk {
  const DTArgs* a;
  __device__ __forceinline__ void unit(int64_t u, int64_t& pair, int& seg, int& n_items, int& len) const {
    pair = u / a->nseg;
    seg = (int)(u - pair * a->nseg);
    const int b = (int)(pair / a->hkv);
    len = (int)min((int64_t)max(a->seq_lens[b], 0), a->max_tokens);
    const int t0 = seg * SEG * TK;
    n_items = len > t0 ? min(SEG, (len - t0 + TK - 1) / TK) : 0;
  }
};

template <int KB, int VKB>
__global__ void __launch_bounds__(DL<KB, VKB>::NTHREADS, 1) decode_tc_kernel(const DTArgs a) {
  using L = DL<KB, VKB>;
  constexpr int NTK = L::NTK, NPK = L::NPK, NTV = L::NTV;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);  // [NST] stage loaded (1 + tx)
  uint64_t* empty = full + NST;                        // [NST] stage read (4 key + 4 value expansion + 4 softmax warps)
  uint64_t* ksf = empty + NST;                         // [NSK] key plane slot written (4)
  uint64_t* ksr = ksf + NSK;                           // [NSK] key plane slot read by its MMAs (1)
  uint64_t* vsf = ksr + NSK;                           // [NSV] value plane slot written (4)
  uint64_t* vsr = vsf + NSV;                           // [NSV] value plane slot read (1)
  uint64_t* kaf = vsr + NSV;                           // [NBK] logits accumulators complete (1)
  uint64_t* kar = kaf + NBK;                           // [NBK] logits accumulators read (4)
  uint64_t* bvf = kar + NBK;                           // [2] value digit images written (4)
  uint64_t* bvr = bvf + 2;                             // [2] value digit images read (1)
  uint64_t* vaf = bvr + 2;                             // [NBV] value accumulators complete (1)
  uint64_t* var_ = vaf + NBV;                          // [NBV] value accumulators read (4)
  uint64_t* stf = var_ + NBV;                          // [2] item stats written (1)
  uint64_t* str_ = stf + 2;                            // [2] item stats read (4)
  uint64_t* imf = str_ + 2;                            // [2] query image loaded (1 + tx)
  uint64_t* imr = imf + 2;                             // [2] query image no longer read by the MMAs (1)
  uint64_t* imq = imr + 2;                             // [2] query image scalars copied by the softmax (4)
  uint64_t* sbar = imq + 2;                            // [2] barrier of each softmax group (4)
  uint32_t* tbase = reinterpret_cast<uint32_t*>(sbar + 2);
  uint8_t* imgs = smem + L::OFF_IMG;
  uint8_t* bv = smem + L::OFF_BV;
  float* stats = reinterpret_cast<float*>(smem + L::OFF_ST);  // [2][16]: alpha[4], 2^-(F_q+7)[4], sum w[4], last
  float* xch = reinterpret_cast<float*>(smem + L::OFF_X);     // [4 warps][8]
  uint8_t* ring = smem + L::OFF_RING;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t u0 = (int64_t)blockIdx.x * a.n_units / gridDim.x;
  const int64_t u1 = (int64_t)(blockIdx.x + 1) * a.n_units / gridDim.x;
  const Walk walk{&a};

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 12);
    }
    for (int s = 0; s < NSK; ++s) {
      mbar_init(&ksf[s], 4);
      mbar_init(&ksr[s], 1);
    }
    for (int s = 0; s < NSV; ++s) {
      mbar_init(&vsf[s], 4);
      mbar_init(&vsr[s], 1);
    }
    for (int c = 0; c < NBK; ++c) {
      mbar_init(&kaf[c], 1);
      mbar_init(&kar[c], 4);
    }
    for (int c = 0; c < NBV; ++c) {
      mbar_init(&vaf[c], 1);
      mbar_init(&var_[c], 4);
    }
    for (int k = 0; k < 2; ++k) {
      mbar_init(&bvf[k], 4);
      mbar_init(&bvr[k], 1);
      mbar_init(&stf[k], 1);
      mbar_init(&str_[k], 4);
      mbar_init(&imf[k], 1);
      mbar_init(&imr[k], 1);
      mbar_init(&imq[k], 8);
    }
    mbar_init(&sbar[0], 4);
    mbar_init(&sbar[1], 4);
  }
  fence_async_smem();
  if (warp == 0) tmem_alloc(tbase, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tbase;
  grid_dependency_wait();  // codes, lengths, query images and coefficients come from earlier kernels

  if (warp == 0) {
    // ---------------- producer ----------------
    if (lane == 0) {
      int64_t gi = 0, kimg = 0, prev_pair = -1;
      bool ok = true;
      for (int64_t u = u0; u < u1 && ok; ++u) {
        int64_t pair;
        int seg, n_items, len;
        walk.unit(u, pair, seg, n_items, len);
        if (n_items == 0) continue;
        if (pair != prev_pair) {  // this pair's query image into slot kimg & 1
          const int sl = (int)(kimg & 1);
          if (kimg >= 2 && (!mbar_wait(&imr[sl], (uint32_t)(((kimg - 2) >> 1) & 1)) ||
                            !mbar_wait(&imq[sl], (uint32_t)(((kimg - 2) >> 1) & 1))))
            break;
          mbar_expect_tx(&imf[sl], L::IMG);
          bulk_g2s(imgs + sl * L::IMG, a.img + pair * L::IMG, L::IMG, &imf[sl]);
          prev_pair = pair;
          ++kimg;
        }
        const int64_t vbase = pair * a.max_tokens;
        for (int it = 0; it < n_items; ++it, ++gi) {
          const int s = (int)(gi % NST);
          if (gi >= NST && !mbar_wait(&empty[s], (uint32_t)(((gi - NST) / NST) & 1))) {
            ok = false;
            break;
          }
          const int t0 = (seg * SEG + it) * TK;
          const int nt = min(TK, len - t0);
          const int ntiles = (nt + 31) >> 5;
          const uint32_t nb = (uint32_t)(((nt + 7) >> 3) * 16);  // norms, whole 16-byte chunks
          uint8_t* st = ring + s * L::STAGE;
          mbar_expect_tx(&full[s], (uint32_t)(ntiles * (L::KTILE + L::VTILE)) + 3 * nb);
          bulk_g2s(st, a.kcodes + ((vbase + t0) >> 5) * L::KTILE, ntiles * L::KTILE, &full[s]);
          bulk_g2s(st + L::OFF_KN, a.knorms + vbase + t0, nb, &full[s]);
          bulk_g2s(st + L::OFF_KN + 256, a.krnorms + vbase + t0, nb, &full[s]);
          bulk_g2s(st + L::OFF_KN + 512, a.vnorms + vbase + t0, nb, &full[s]);
          bulk_g2s(st + L::OFF_V, a.vcodes + ((vbase + t0) >> 5) * L::VTILE, ntiles * L::VTILE, &full[s]);
        }
      }
      for (int64_t i = (gi > NST ? gi - NST : 0); i < gi; ++i) mbar_wait(&full[i % NST], (uint32_t)((i / NST) & 1));
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------- logits MMAs ----------------
    constexpr uint32_t idesc = idesc_u8s8_s32(TK, 16);
    int64_t gi = 0, gp = 0, kimg = 0, prev_pair = -1;
    uint32_t simg = 0;
    bool ok = true;
    for (int64_t u = u0; u < u1 && ok; ++u) {
      int64_t pair;
      int seg, n_items, len;
      walk.unit(u, pair, seg, n_items, len);
      if (n_items == 0) continue;
      if (pair != prev_pair) {
        if (kimg >= 1) {  // the previous pair's image is no longer read once these MMAs complete
          __syncwarp();
          umma_commit_elect(&imr[(kimg - 1) & 1]);
        }
        if (!mbar_wait(&imf[kimg & 1], (uint32_t)((kimg >> 1) & 1))) break;
        simg = smem_u32(imgs + (kimg & 1) * L::IMG);
        prev_pair = pair;
        ++kimg;
      }
      for (int it = 0; it < n_items && ok; ++it, ++gi) {
        const int c = (int)(gi % NBK);
        if (gi >= NBK && !mbar_wait(&kar[c], (uint32_t)(((gi - NBK) / NBK) & 1))) {
          ok = false;
          break;
        }
        const uint32_t dacc = tmem + L::C_KACC + 32u * c;
#pragma unroll 1
        for (int P = 0; P < NPK; ++P, ++gp) {
          const int s = (int)(gp % NSK);
          if (!mbar_wait(&ksf[s], (uint32_t)((gp / NSK) & 1))) {
            ok = false;
            break;
          }
          __syncwarp();
          tc_fence_after();
          const bool cen = P < NTK;
          const uint64_t bd = smem_desc(simg + (cen ? L::IMG_C + 2048 * P : L::IMG_S), 256, 128);
          const uint32_t d = dacc + (cen ? 0u : 16u);
          const uint32_t acol = tmem + L::C_KS + 32u * s;
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)  // K = 32 bytes: bit classes 2ks, 2ks + 1
            umma_i8_ts_elect(d, acol + 8u * ks, bd + (uint64_t)(32 * ks), idesc,
                             ((P == 0 || P == NTK) && ks == 0) ? 0u : 1u);
          umma_commit_elect(&ksr[s]);
        }
        if (!ok) break;
        umma_commit_elect(&kaf[c]);
      }
    }
    __syncwarp();
  } else if (warp == 2) {
    // ---------------- value MMAs ----------------
    constexpr uint32_t idesc = idesc_u8s8_s32(TK, 16);
    int64_t gi = 0, gp = 0;
    bool ok = true;
    for (int64_t u = u0; u < u1 && ok; ++u) {
      int64_t pair;
      int seg, n_items, len;
      walk.unit(u, pair, seg, n_items, len);
      for (int it = 0; it < n_items && ok; ++it, ++gi) {
        const int c = (int)(gi % NBV), sb = (int)(gi & 1);
        if (gi >= NBV && !mbar_wait(&var_[c], (uint32_t)(((gi - NBV) / NBV) & 1))) {
          ok = false;
          break;
        }
        if (!mbar_wait(&bvf[sb], (uint32_t)((gi >> 1) & 1))) {
          ok = false;
          break;
        }
        const uint32_t d = tmem + L::C_VACC + 64u * c;
        const uint32_t sbv = smem_u32(bv + sb * L::BVB);
#pragma unroll 1
        for (int T = 0; T < NTV; ++T, ++gp) {
          const int s = (int)(gp % NSV);
          if (!mbar_wait(&vsf[s], (uint32_t)((gp / NSV) & 1))) {
            ok = false;
            break;
          }
          __syncwarp();
          tc_fence_after();
          const uint64_t bd = smem_desc(sbv, 256, 128);
          const uint32_t acol = tmem + L::C_VS + 32u * s;
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)  // K = 32 tokens: 2 K chunks of the digit image
            umma_i8_ts_elect(d + 16u * T, acol + 8u * ks, bd + (uint64_t)(32 * ks), idesc, ks == 0 ? 0u : 1u);
          umma_commit_elect(&vsr[s]);
        }
        if (!ok) break;
        umma_commit_elect(&vaf[c]);
        umma_commit_elect(&bvr[sb]);
      }
    }
    __syncwarp();
  } else if (warp < 7) {
    // ---------------- key bits -> plane slots (lane = token 32 qd + lane) ----------------
    const int qd = warp & 3;
    int64_t gi = 0, gp = 0;
    bool ok = true;
    for (int64_t u = u0; u < u1 && ok; ++u) {
      int64_t pair;
      int seg, n_items, len;
      walk.unit(u, pair, seg, n_items, len);
      for (int it = 0; it < n_items && ok; ++it, ++gi) {
        const int st = (int)(gi % NST);
        if (!mbar_wait(&full[st], (uint32_t)((gi / NST) & 1))) {
          ok = false;
          break;
        }
        const uint8_t* src = ring + st * L::STAGE + qd * L::KTILE + lane * 16;
        uint4 pw[KB + 1];
#pragma unroll
        for (int p = 0; p < KB + 1; ++p) pw[p] = *reinterpret_cast<const uint4*>(src + p * 512);
        release_to_copy(&empty[st], lane);
        uint4 itp[NPK];
#pragma unroll
        for (int T = 0; T < NTK; ++T) itp[T] = pw[T < KB ? T : 0];
        if constexpr (KB == 3)
          itp[3] = make_uint4(pw[0].x ^ pw[1].x ^ pw[2].x, pw[0].y ^ pw[1].y ^ pw[2].y, pw[0].z ^ pw[1].z ^ pw[2].z,
                              pw[0].w ^ pw[1].w ^ pw[2].w);
        itp[NTK] = pw[KB];
#pragma unroll
        for (int P = 0; P < NPK; ++P, ++gp) {
          const int s = (int)(gp % NSK);
          if (gp >= NSK && !mbar_wait(&ksr[s], (uint32_t)(((gp - NSK) / NSK) & 1))) {
            ok = false;
            break;
          }
          __syncwarp();
          tc_fence_after();
          const uint32_t base = tmem + L::C_KS + 32u * s + ((uint32_t)(32 * qd) << 16);
#pragma unroll
          for (int cg = 0; cg < 2; ++cg) {
            uint32_t r[16];
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
              const uint32_t mk = 0x01010101u << (4 * cg + cc);
              r[4 * cc + 0] = itp[P].x & mk;
              r[4 * cc + 1] = itp[P].y & mk;
              r[4 * cc + 2] = itp[P].z & mk;
              r[4 * cc + 3] = itp[P].w & mk;
            }
            tmem_st16(base + 16 * cg, r);
          }
          tmem_st_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&ksf[s]);
        }
      }
    }
  } else if (warp < 11) {
    // ---------------- value words -> plane slots (lane = coordinate 32 qd + lane) ----------------
    const int qd = warp & 3;
    const int j = 32 * qd + lane;
    int64_t gi = 0, gp = 0;
    bool ok = true;
    for (int64_t u = u0; u < u1 && ok; ++u) {
      int64_t pair;
      int seg, n_items, len;
      walk.unit(u, pair, seg, n_items, len);
      for (int it = 0; it < n_items && ok; ++it, ++gi) {
        const int st = (int)(gi % NST);
        if (!mbar_wait(&full[st], (uint32_t)((gi / NST) & 1))) {
          ok = false;
          break;
        }
        // word j of plane p of the item's 4 tiles (tiles past the item's end hold stale words; their
        // tokens have weight 0)
        const uint32_t* src = reinterpret_cast<const uint32_t*>(ring + st * L::STAGE + L::OFF_V) + j;
        uint32_t w[4][VKB];
#pragma unroll
        for (int t4 = 0; t4 < 4; ++t4)
#pragma unroll
          for (int p = 0; p < VKB; ++p) w[t4][p] = src[t4 * (L::VTILE / 4) + p * DP];
        release_to_copy(&empty[st], lane);
#pragma unroll
        for (int T = 0; T < NTV; ++T, ++gp) {
          const int s = (int)(gp % NSV);
          if (gp >= NSV && !mbar_wait(&vsr[s], (uint32_t)(((gp - NSV) / NSV) & 1))) {
            ok = false;
            break;
          }
          __syncwarp();
          tc_fence_after();
          const uint32_t base = tmem + L::C_VS + 32u * s + ((uint32_t)(32 * qd) << 16);
#pragma unroll
          for (int half = 0; half < 2; ++half) {  // tiles 2 half, 2 half + 1: columns 8 t4 + class
            uint32_t r[16];
#pragma unroll
            for (int tt = 0; tt < 2; ++tt) {
              const int t4 = 2 * half + tt;
              uint32_t wt;
              if constexpr (VKB == 3) {
                wt = T < 3 ? w[t4][T < 3 ? T : 0] : (w[t4][0] ^ w[t4][1] ^ w[t4][2]);
              } else {
                wt = w[t4][T < VKB ? T : 0];
              }
#pragma unroll
              for (int c = 0; c < 8; ++c) r[8 * tt + c] = wt & (0x01010101u << c);
            }
            tmem_st16(base + 16 * half, r);
          }
          tmem_st_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&vsf[s]);
        }
      }
    }
  } else if (warp < 19) {
    // ---------------- softmax (lane = token 32 qd + lane), group sg takes the items of parity sg ----------------
    const int sg = (warp - 11) >> 2, sw = (warp - 11) & 3;
    const int qd = warp & 3;
    const int tk = 32 * qd + lane;
    const int cls = lane & 7;                           // bit class of the token inside its 32-token tile
    const int kpos = 32 * qd + 4 * cls + (lane >> 3);  // its K byte in the value MMAs
    const int sh = 7 - cls;
    GroupSync gs{&sbar[sg], 0u};
    float* xg = xch + sg * 96;  // this group's exchange: [2][4 warps][8] item maxima, then [4][8] sums
    int64_t gi = 0, kimg = 0, prev_pair = -1;
    float4 qsc[4];
    bool ok = true;
    for (int64_t u = u0; u < u1 && ok; ++u) {
      int64_t pair;
      int seg, n_items, len;
      walk.unit(u, pair, seg, n_items, len);
      const int b = (int)(pair / a.hkv), g = (int)(pair - (int64_t)b * a.hkv);
      const int sub = (int)((sg ^ gi) & 1);  // this group's items in the unit: it = sub, sub + 2, ...
      float mrun[4], lw[4], ww[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        mrun[q] = -INFINITY;
        lw[q] = 0.f;
        ww[q] = 0.f;
      }
      if (n_items > 0 && pair != prev_pair) {  // the query image's scalars, copied; the slot may then be reloaded
        if (!mbar_wait(&imf[kimg & 1], (uint32_t)((kimg >> 1) & 1))) break;
        const float4* qs = reinterpret_cast<const float4*>(imgs + (kimg & 1) * L::IMG);
#pragma unroll
        for (int q = 0; q < 4; ++q) qsc[q] = qs[q];
        __syncwarp();
        if (lane == 0) mbar_arrive(&imq[kimg & 1]);
        prev_pair = pair;
        ++kimg;
      }
      for (int it = 0; it < n_items && ok; ++it, ++gi) {
        if ((gi & 1) != sg) continue;
        const int st = (int)(gi % NST), c = (int)(gi % NBK), sb = (int)(gi & 1);
        const int t0 = (seg * SEG + it) * TK;
        const bool valid = t0 + tk < len;
        if (!mbar_wait(&full[st], (uint32_t)((gi / NST) & 1))) {
          ok = false;
          break;
        }
        const __half* nst = reinterpret_cast<const __half*>(ring + st * L::STAGE + L::OFF_KN);
        const float kn = __half2float(nst[tk]), gam = __half2float(nst[128 + tk]), vn = __half2float(nst[256 + tk]);
        release_to_copy(&empty[st], lane);
        if (!mbar_wait(&kaf[c], (uint32_t)((gi / NBK) & 1))) {
          ok = false;
          break;
        }
        __syncwarp();
        tc_fence_after();
        uint32_t C[16], Z[16];
        {
          const uint32_t lrow = tmem + L::C_KACC + 32u * c + ((uint32_t)(32 * qd) << 16);
          tmem_ld16_issue(lrow, C);
          tmem_ld16_issue(lrow + 16, Z);
          tmem_ld_wait16x2(C, Z);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&kar[c]);
        float s[4];
        float xm[5];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float4 sc = qsc[q];
          // sum_d 256^d C[d]: each C[d] an exact int32 below 2^22; one fp32 rounding per step
          const float cen = fmaf((float)(int)C[4 * q + 3], 16777216.f,
                                 fmaf((float)(int)C[4 * q + 2], 65536.f,
                                      fmaf((float)(int)C[4 * q + 1], 256.f, (float)(int)C[4 * q])));
          const float sg2 = fmaf((float)(int)Z[4 * q + 3], 16777216.f,
                                 fmaf((float)(int)Z[4 * q + 2], 65536.f,
                                      fmaf((float)(int)Z[4 * q + 1], 256.f, (float)(int)Z[4 * q])));
          const float l = fmaf(gam * a.kappa, fmaf(sg2, sc.z, -sc.w), fmaf(cen, sc.x, -sc.y));
          s[q] = (valid && q < a.group) ? kn * l * a.sl2 : -INFINITY;
          xm[q] = warp_max_f32(s[q]);
        }
        xm[4] = warp_max_f32(valid ? vn : 0.f);
        // item maxima over the group's 4 warps
        float* xb = xg + ((gi >> 1) & 1) * 32;  // two buffers: a fast warp may reach the group's next item
        if (lane == 0) {
#pragma unroll
          for (int q = 0; q < 5; ++q) xb[8 * sw + q] = xm[q];
        }
        gs.sync(lane);
        float vmax = 0.f;
#pragma unroll
        for (int k = 0; k < 4; ++k) vmax = fmaxf(vmax, xb[8 * k + 4]);
        // per query: weights w 2^F_q below 2^23, F_q from the bound w <= 2^(item max - running max) * max n_v
        float mnew[4], alf[4], fq[4];
        int Fq[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float mi = -INFINITY;
#pragma unroll
          for (int k = 0; k < 4; ++k) mi = fmaxf(mi, xb[8 * k + q]);
          mnew[q] = fmaxf(mrun[q], mi);
          alf[q] = mrun[q] == -INFINITY ? 0.f : exp2f(mrun[q] - mnew[q]);
          const float mc = mi == -INFINITY ? 0.f : vmax * exp2f(mi - mnew[q]);
          Fq[q] = mc > 0.f ? 23 - exponent_of(mc) : 0;
          fq[q] = pow2(Fq[q]);
        }
        float wq[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float p = (s[q] == -INFINITY) ? 0.f : exp2f(s[q] - mnew[q]);
          wq[q] = valid ? p * vn : 0.f;  // norms past the sequence end are stale
          lw[q] = fmaf(lw[q], alf[q], p);
          ww[q] = fmaf(ww[q], alf[q], wq[q]);
          mrun[q] = mnew[q];
        }
        // the value MMAs' weight image: row 4q + d, K byte kpos; 4 base-256 digits of w 2^F_q << (7 - class)
        if (gi >= 2 && !mbar_wait(&bvr[sb], (uint32_t)(((gi - 2) >> 1) & 1))) {
          ok = false;
          break;
        }
        uint8_t* img = bv + sb * L::BVB + (kpos >> 4) * 256 + (kpos & 15);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          int X = __float2int_rn(wq[q] * fq[q]) << sh;
#pragma unroll
          for (int dd = 0; dd < 4; ++dd) {
            const int r = 4 * q + dd;
            const int lowb = dd < 3 ? (int)(int8_t)(X & 0xFF) : X;
            img[(r >> 3) * 128 + (r & 7) * 16] = (uint8_t)lowb;
            X = (X - lowb) >> 8;
          }
        }
        fence_async_smem();  // the image is read by the tensor core
        __syncwarp();
        if (lane == 0) mbar_arrive(&bvf[sb]);
        const bool last = it + 2 >= n_items;  // the group's last item of the unit
        if (last) {  // the group's sums over its 4 warps
          float* xs = xg + 64;  // [4][8]
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float l1 = warp_sum(lw[q]), w1 = warp_sum(ww[q]);
            if (lane == 0) {
              xs[8 * sw + q] = l1;
              xs[8 * sw + 4 + q] = w1;
            }
          }
          gs.sync(lane);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            lw[q] = xs[q] + xs[8 + q] + xs[16 + q] + xs[24 + q];
            ww[q] = xs[4 + q] + xs[12 + q] + xs[20 + q] + xs[28 + q];
          }
          gs.sync(lane);  // xs is reused by the group's next unit
        }
        // item stats for the value epilogue (one writer per group)
        if (sw == 0) {
          if (gi >= 2 && !mbar_wait(&str_[sb], (uint32_t)(((gi - 2) >> 1) & 1))) {
            ok = false;
            break;
          }
          if (lane == 0) {
            float* sp = stats + 16 * sb;  // alpha[4], 2^-(F_q+7) [4], sum w [4], last
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              sp[q] = alf[q];
              sp[4 + q] = pow2(-(Fq[q] + 7));
              sp[8 + q] = ww[q];
            }
            sp[12] = last ? 1.f : 0.f;
            mbar_arrive(&stf[sb]);
          }
          __syncwarp();
        }
      }
      if (!ok) break;
      // the group's partial of the unit (m, l in log2 units): chunk 2 seg + sub, one writer per query
      if (sw == 0 && lane < a.group) {
        const bool has = n_items > sub;
        const int q = lane;
        float mq = -INFINITY, lq = 0.f;
#pragma unroll
        for (int k = 0; k < 4; ++k)
          if (k == q) {
            mq = has ? mrun[k] : -INFINITY;
            lq = has ? lw[k] : 0.f;
          }
        const int64_t row = (int64_t)b * a.hq + (int64_t)g * a.group + q;
        float* dst = a.part + (row * (2 * a.nseg) + 2 * seg + sub) * (DP + 2);
        dst[DP] = mq;
        dst[DP + 1] = lq;
      }
    }
  } else {
    // ---------------- value epilogue (lane = coordinate 32 qd + lane), one sum set per item parity ----------------
    const int qd = warp & 3;
    const int j = 32 * qd + lane;
    const float va2[4] = {2.f * a.vco[0], 2.f * a.vco[1], 2.f * a.vco[2], 2.f * a.vco[3]};
    const float vctop = a.vco[4];
    int64_t gi = 0;
    bool ok = true;
    for (int64_t u = u0; u < u1 && ok; ++u) {
      int64_t pair;
      int seg, n_items, len;
      walk.unit(u, pair, seg, n_items, len);
      const int b = (int)(pair / a.hkv), g = (int)(pair - (int64_t)b * a.hkv);
      float o[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
      float wsum[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
      for (int it = 0; it < n_items && ok; ++it, ++gi) {
        const int c = (int)(gi % NBV), sb = (int)(gi & 1), sub = it & 1;
        if (!mbar_wait(&vaf[c], (uint32_t)((gi / NBV) & 1))) {
          ok = false;
          break;
        }
        __syncwarp();
        tc_fence_after();
        // sum_T 2 alpha_T sum_d 256^d D_T[4q + d] = 2^(7+F_q) sum_T 2 alpha_T sum_t w b_T (each D exact,
        // below 2^22), two planes (32 columns) at a time
        float v[4] = {0.f, 0.f, 0.f, 0.f};
        {
          const uint32_t lrow = tmem + L::C_VACC + 64u * c + ((uint32_t)(32 * qd) << 16);
#pragma unroll
          for (int T0 = 0; T0 < NTV; T0 += 2) {
            uint32_t d0[16], d1[16];
            tmem_ld16_issue(lrow + 16 * T0, d0);
            if (T0 + 1 < NTV) {
              tmem_ld16_issue(lrow + 16 * T0 + 16, d1);
              tmem_ld_wait16x2(d0, d1);
            } else {
              tmem_ld_wait16(d0);
            }
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              if (T0 + h < NTV) {
                const uint32_t* dt = h ? d1 : d0;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                  const float cT = fmaf(i2f_exact(dt[4 * q + 3]), 16777216.f,
                                        fmaf(i2f_exact(dt[4 * q + 2]), 65536.f,
                                             fmaf(i2f_exact(dt[4 * q + 1]), 256.f, i2f_exact(dt[4 * q]))));
                  v[q] = fmaf(va2[T0 + h], cT, v[q]);
                }
              }
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&var_[c]);
        if (!mbar_wait(&stf[sb], (uint32_t)((gi >> 1) & 1))) {
          ok = false;
          break;
        }
        const float* sp = stats + 16 * sb;
        float alf[4], inv[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          alf[q] = sp[q];
          inv[q] = sp[4 + q];
        }
        if (sp[12] != 0.f) {
#pragma unroll
          for (int q = 0; q < 4; ++q) wsum[sub][q] = sp[8 + q];
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&str_[sb]);
#pragma unroll
        for (int q = 0; q < 4; ++q) o[sub][q] = fmaf(o[sub][q], alf[q], v[q] * inv[q]);
      }
      if (!ok) break;
      // o_rot = sum_T 2 alpha_T sum_t w b_T - c[L-1] sum_t w, one partial per item parity
#pragma unroll
      for (int sbb = 0; sbb < 2; ++sbb) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          if (q < a.group) {
            const int64_t row = (int64_t)b * a.hq + (int64_t)g * a.group + q;
            a.part[(row * (2 * a.nseg) + 2 * seg + sbb) * (DP + 2) + j] =
                n_items > sbb ? fmaf(-vctop, wsum[sbb][q], o[sbb][q]) : 0.f;
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

template <int KB, int VKB>
int launch_dtc(const DTArgs& a, int sm, cudaStream_t st) {
  using L = DL<KB, VKB>;
  auto kern = decode_tc_kernel<KB, VKB>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::SMEM);
  if (e != cudaSuccess) return tq::set_error(TQ_ECUDA, "tq_decode_attn: %s", cudaGetErrorString(e));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)std::max<int64_t>(1, std::min<int64_t>(sm, a.n_units)));
  cfg.blockDim = dim3(L::NTHREADS);
  cfg.dynamicSmemBytes = L::SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, a);
  if (e != cudaSuccess) return tq::set_error(TQ_ECUDA, "tq_decode_attn: launch failed: %s", cudaGetErrorString(e));
  return TQ_OK;
}

template <int KB>
int dispatch_vkb(int vkb, const DTArgs& a, int sm, cudaStream_t st) {
  switch (vkb) {
    case 1: return launch_dtc<KB, 1>(a, sm, st);
    case 2: return launch_dtc<KB, 2>(a, sm, st);
    default: return launch_dtc<KB, 3>(a, sm, st);
  }
}

int image_bytes(int kb) {
  const int ntk = walsh_planes(kb);
  return (64 + (ntk + 1) * 2048 + 127) / 128 * 128;
}

}  // namespace

namespace tq {

int64_t decode_sliced_workspace(int kb, int m, int batch, int n_q_heads, int n_kv_heads, int64_t max_tokens) {
  if (kb < 1 || kb > 3 || m != 128 || batch < 0 || n_kv_heads < 1 || max_tokens < 0) return 0;
  const int64_t pairs = (int64_t)batch * n_kv_heads;
  const int64_t nseg = std::max<int64_t>(1, (max_tokens + SEG * TK - 1) / (SEG * TK));
  int64_t img = pairs * image_bytes(kb);
  img = (img + 255) & ~(int64_t)255;
  return img + 256 + (int64_t)batch * n_q_heads * 2 * nseg * (DP + 2) * 4;
}

int launch_combine(const float* part, int64_t row_stride, int64_t chunk_stride, const int8_t* vD,
                   const int32_t* seq_lens, float* out, int nch, int d, int dp, int hq, int64_t rows,
                   cudaStream_t st);

int decode_attn_sliced(const tq_params* kp, const tq_params* vp, const float* q, int batch, int n_q_heads,
                       int n_kv_heads, const void* kcodes, const uint16_t* knorms, const uint16_t* krnorms,
                       const void* vcodes, const uint16_t* vnorms, const int32_t* seq_lens, int64_t max_tokens,
                       float scale, float* out, void* workspace, int64_t workspace_bytes, cudaStream_t st) {
  const int kb = index_bits(kp), vkb = index_bits(vp);
  if (kp->mode != TQ_MODE_PROD || kp->m != 128 || kp->d_pad != 128 || vp->d_pad != 128 || kp->d != vp->d ||
      kb > 3 || vkb > 3 || n_q_heads % n_kv_heads != 0 || n_q_heads / n_kv_heads > 4)
    return set_error(TQ_EUNSUPPORTED, "tq_decode_attn: token-sliced values need d_pad 128, keys with m = 128 and "
                                      "at most 3 index bits each, and at most 4 query heads per KV head");
  if (batch < 0 || n_kv_heads < 1 || max_tokens < 0) return set_error(TQ_EINVAL, "tq_decode_attn: bad sizes");
  if (batch == 0) {
    clear_error();
    return TQ_OK;
  }
  if (max_tokens % 32 != 0)
    return set_error(TQ_EUNSUPPORTED, "tq_decode_attn: token-sliced values need max_tokens %% 32 == 0");
  if (!q || !kcodes || !knorms || !krnorms || !vcodes || !vnorms || !seq_lens || !out || !workspace)
    return set_error(TQ_EINVAL, "tq_decode_attn: NULL pointer argument");
  if (!aligned(kcodes, 16) || !aligned(vcodes, 16) || !aligned(knorms, 16) || !aligned(krnorms, 16) ||
      !aligned(vnorms, 16) || !aligned(workspace, 16))
    return set_error(TQ_EINVAL, "tq_decode_attn: code and norm arrays and the workspace must be 16-byte aligned");
  const int64_t need = decode_sliced_workspace(kb, kp->m, batch, n_q_heads, n_kv_heads, max_tokens);
  if (workspace_bytes < need)
    return set_error(TQ_EINVAL, "tq_decode_attn: workspace too small (%lld < %lld)", (long long)workspace_bytes,
                     (long long)need);
  const int group = n_q_heads / n_kv_heads;
  const int64_t pairs = (int64_t)batch * n_kv_heads;
  const int nseg = (int)std::max<int64_t>(1, (max_tokens + SEG * TK - 1) / (SEG * TK));
  if (2 * nseg > 2048) return set_error(TQ_EUNSUPPORTED, "tq_decode_attn: max_tokens too large for the combine");
  const int ib = image_bytes(kb);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int64_t img_total = (pairs * ib + 255) & ~(int64_t)255;
  float* vco = reinterpret_cast<float*>(ws + img_total);
  float* part = reinterpret_cast<float*>(ws + img_total + 256);

  DPrepArgs pa;
  pa.q = q;
  pa.d = kp->d;
  pa.kb = kb;
  pa.group = group;
  pa.hq = n_q_heads;
  pa.hkv = n_kv_heads;
  pa.vcent = vp->centroids;
  pa.vkb = vkb;
  pa.vco = vco;
  pa.cent = kp->centroids;
  pa.D = kp->signs_D;
  pa.S = kp->S;
  pa.img = ws;
  pa.img_bytes = ib;
  pa.ntk = walsh_planes(kb);
  pa.img_s = 64 + pa.ntk * 2048;
  decode_prep_tc_kernel<<<(unsigned)pairs, 128, 0, st>>>(pa);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(TQ_ECUDA, "tq_decode_attn: prep launch failed: %s", cudaGetErrorString(e));

  DTArgs a;
  a.kcodes = static_cast<const uint8_t*>(kcodes);
  a.knorms = knorms;
  a.krnorms = krnorms;
  a.vcodes = static_cast<const uint8_t*>(vcodes);
  a.vnorms = vnorms;
  a.seq_lens = seq_lens;
  a.max_tokens = max_tokens;
  a.hkv = n_kv_heads;
  a.group = group;
  a.hq = n_q_heads;
  a.nseg = nseg;
  a.n_units = pairs * nseg;
  a.img = ws;
  a.part = part;
  a.kappa = (float)(std::sqrt(M_PI / 2.0) / kp->m);
  const float sc = scale > 0.f ? scale : 1.f / std::sqrt((float)kp->d);
  a.sl2 = sc * 1.4426950408889634f;
  a.vco = vco;
  int rc;
  const int sm = sm_count();
  switch (kb) {
    case 1: rc = dispatch_vkb<1>(vkb, a, sm, st); break;
    case 2: rc = dispatch_vkb<2>(vkb, a, sm, st); break;
    default: rc = dispatch_vkb<3>(vkb, a, sm, st); break;
  }
  if (rc) return rc;
  rc = launch_combine(part, (int64_t)2 * nseg * (DP + 2), DP + 2, vp->signs_D, seq_lens, out, 2 * nseg, vp->d, DP,
                      n_q_heads, (int64_t)batch * n_q_heads, st);
  if (rc == TQ_OK) clear_error();
  return rc;
}

}  // namespace tq
