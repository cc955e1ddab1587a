// tq_quantize for d_pad = 128 (m <= 128): two threads per vector, QJL
// projection on the 5th-generation tensor cores.
//
// Method ("TurboQuant explainer" (m.163.com), "第一步：PolarQuant" and
// "第二步：QJL"): norm, random sign flips + Walsh-Hadamard rotation, Lloyd-Max
// code at b-1 bits, residual and its norm, sign bits of S r.
//
// Design (B200, sm_100a):
//  * A CTA of 512 threads runs two independent groups of 256 threads; a group
//    owns a tile of 128 vectors (the M of one MMA) and runs its own pipeline
//    (input staging, encode, MMA, read-back) with named barriers and its own
//    mbarrier, so one group's encode overlaps the other's tensor-core work.
//  * Two threads per vector (lanes l and l + 16 of a warp): thread h holds the
//    64 rotated coordinates 64h .. 64h + 63 in registers (<= 128 registers a
//    thread, 16 warps per SM).  Input rows are staged in shared memory with
//    cp.async (16-byte chunks, XOR-swizzled per row); the copies of a group's
//    next tile are issued when its current tile starts (two buffers in
//    product mode, three in MSE mode, where the copies run two tiles ahead).
//  * Rotation: both threads read the whole row; the Walsh-Hadamard stage on
//    coordinate bit 6 is taken first, while unpacking (thread h keeps
//    x_c + (-1)^h x_{c+64}), so the other six stages stay inside the thread
//    (bit 0 on scalars, bits 1..5 on Blackwell's packed f32x2 add/fma).  The
//    squared norm is half the sum of both threads' squared stage-6 values.
//  * Code: with p_k = [|y| > t_{L/2+k}] (monotone in k) and s = [y > 0] the
//    index is idx = s ? L/2 + m : L/2-1 - m with m = sum_k p_k; bit b of m is
//    the XOR of the p_k at which bit b of k+1 differs from bit b of k.  Each
//    predicate is packed into a 32-bit word with one predicated OR, and the
//    bit-planes are a few word-wide XORs.  The residual is |y| - mag[m] with
//    the sign of s.
//  * QJL: the residual (scaled by 2^14) is split into fp16 hi and lo parts,
//    written in the UMMA K-major canonical layout: the hi part over the
//    staged input rows themselves (the canonical tile of 8 rows takes the same
//    2 KB as their staged input, and one warp owns those rows, so a __syncwarp
//    after the rotation has read them suffices), the lo part to a buffer of
//    its own.  One thread of the group issues tcgen05.mma (M=128, N=m, K=16)
//    x 16 against S (fp16, exact) with fp32 accumulation in tensor memory
//    (S r_hi + S r_lo, so z is exact to ~2^-22 before fp32 accumulation).
//    Each warp of the group reads back 64 columns of 32 rows with
//    tcgen05.ld.32x32b; a projection with |z| below the accumulation bound
//    (about 0.03 per vector) is recomputed in fp32 from hi+lo by the warp.
#include <cuda_runtime.h>

#include <algorithm>

#include "common.h"
#include "device.cuh"
#include "tc.cuh"

namespace {

using namespace tqd;

constexpr int NG = 2;          // independent thread groups per CTA
constexpr int GV = 128;        // vectors per group tile (the M of one MMA)
constexpr int GT = 256;        // threads per group: two per vector
constexpr int NT = NG * GT;    // threads per CTA
constexpr int DP = 128;        // rotation size handled here
constexpr int ROWB = 256;      // staged bytes per input row (2-byte elements, d <= 128)
constexpr int KCH = DP / 8;    // 16-byte K chunks of a 128-element fp16 row

struct Q2Args {
  const uint8_t* x;
  int64_t n_vec, n_pad, ld_bytes;
  int d, m, row_bytes;
  uint8_t* codes;
  uint16_t* norms;
  uint16_t* rnorms;
  const float* cent;
  const float* thr;
  const int8_t* D;
  const uint16_t* S;
};

// shared-memory carve-up; product mode: a staged tile turns into the hi part of the MMA's A operand
template <bool PROD>
struct Lay {
  static constexpr int NB = PROD ? 2 : 3;                    // staging depth (tiles per group)
  static constexpr int XS = 0;                               // [NB][NG][GV][ROWB] staged input (swizzled chunks)
  static constexpr int RL = XS + NB * NG * GV * ROWB;        // [NG] residual lo parts, canonical (product mode)
  static constexpr int SS = RL + (PROD ? NG * GV * DP * 2 : 0);  // S, canonical K-major fp16 (product mode)
  static constexpr int DM = SS + (PROD ? 128 * DP * 2 : 0);  // sign-flip masks, 64 x uint32 (bits 15, 31)
  static constexpr int BND = DM + 64 * 4;                    // [NG][GV] fix-up bound of each vector
  static constexpr int MISC = BND + NG * GV * 4;             // mbarriers (+0, +8), tmem base (+16), max ||S_i|| (+20), 16 floats (+32)
  static constexpr int TOTAL = MISC + 96;
};

// byte offset of element (row, k) in a K-major canonical fp16 tile of 128 rows
__device__ __forceinline__ int canon(int row, int k) {
  return (row >> 3) * (KCH * 128) + (k >> 3) * 128 + (row & 7) * 16 + (k & 7) * 2;
}

template <int DT>
__device__ __forceinline__ void unpack_pair(uint32_t w, uint32_t dm, float& x0, float& x1) {
  if constexpr (DT == TQ_BF16) {
    const uint32_t s = w ^ dm;  // sign flips on the raw bits
    x0 = __uint_as_float(s << 16);
    x1 = __uint_as_float(s & 0xFFFF0000u);
  } else {  // fp16
    const uint32_t s = w ^ dm;
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&s));
    x0 = f.x;
    x1 = f.y;
  }
}

// Rotation of this thread's half of one staged row: y[k] (32 float2) holds
// coordinates 64h + 2k, 64h + 2k + 1 of H (D o x), unnormalized.  Returns the
// sum of squares of the stage-6 values x_c + (-1)^h x_{c+64} (the two threads
// of a vector together hold 2 ||x||^2).  Chunks past d were zeroed at CTA start.
template <int DT>
__device__ __forceinline__ float rotate_half(const uint8_t* xrow, int sw, int h, const uint32_t* dmask,
                                             float2 (&y)[32]) {
  const float2 sg = h ? make_float2(-1.f, -1.f) : make_float2(1.f, 1.f);
  float2 ss = make_float2(0.f, 0.f);
#pragma unroll
  for (int c = 0; c < 8; ++c) {  // chunk c = elements 8c..8c+7, chunk c + 8 = elements 64 + 8c ..
    const uint4 va = *reinterpret_cast<const uint4*>(xrow + ((c ^ sw) << 4));
    const uint4 vb = *reinterpret_cast<const uint4*>(xrow + (((c + 8) ^ sw) << 4));
    const uint32_t wa[4] = {va.x, va.y, va.z, va.w}, wb[4] = {vb.x, vb.y, vb.z, vb.w};
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      float a0, a1, b0, b1;
      unpack_pair<DT>(wa[w], dmask[4 * c + w], a0, a1);
      unpack_pair<DT>(wb[w], dmask[32 + 4 * c + w], b0, b1);
      const float2 z = __ffma2_rn(make_float2(b0, b1), sg, make_float2(a0, a1));  // stage on bit 6
      ss = __ffma2_rn(z, z, ss);
      y[4 * c + w] = make_float2(z.x + z.y, z.x - z.y);  // stage on bit 0
    }
  }
  const float2 neg1 = make_float2(-1.f, -1.f);
#pragma unroll
  for (int hs = 1; hs < 32; hs <<= 1) {  // stages on bits 1..5 (pairs of pairs)
#pragma unroll
    for (int k = 0; k < 32; ++k) {
      if ((k & hs) == 0) {
        const float2 u = y[k], w = y[k + hs];
        y[k] = __fadd2_rn(u, w);
        y[k + hs] = __ffma2_rn(w, neg1, u);
      }
    }
  }
  return ss.x + ss.y;
}

// a * b clamped to [0, 1] in one instruction
__device__ __forceinline__ float mul_sat(float a, float b) {
  float r;
  asm("mul.rn.sat.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
  return r;
}

// Scalar code of one coordinate.  The predicate bits are shifted in at the
// bottom of 32-bit words (one funnel shift of a sign bit each), so a word is
// filled from its highest coordinate down; the centroid magnitude is picked
// with saturated multiplies and FMAs.  Both keep compares and selects off the
// integer pipe, which is the busier one here; every decision is exactly the
// comparison it stands for (see code()).
template <int KB>
struct Coder {
  static constexpr int L = 1 << KB;
  static constexpr int NPT = L / 2 - 1;  // positive thresholds t_{L/2} .. t_{L-2}
  static constexpr int NP1 = NPT > 0 ? NPT : 1;
  float tp[NP1];    // positive thresholds
  float dmag[NP1];  // c[L/2 + k + 1] - c[L/2 + k]
  float mag0;       // c[L/2]

  __device__ __forceinline__ void init(const float* thr, const float* cent) {
#pragma unroll
    for (int k = 0; k < NPT; ++k) {
      tp[k] = thr[L / 2 + k];
      dmag[k] = cent[L / 2 + k + 1] - cent[L / 2 + k];
    }
    mag0 = cent[L / 2];
  }
  // Shifts [y <= 0] into wn and [|y| > t_{L/2+k}] into wp[k].  Returns y - c[idx]
  // (RES) or 0.
  //  * e = t - |y| is < 0 exactly when |y| > t (a zero difference is +0), so its
  //    sign bit is the predicate, and sat(-2^126 e) is 1 or 0 with it (a nonzero
  //    e is at least an ulp of t, far above 2^-126).
  //  * y - 2^-149 (no flush to zero) has its sign bit set exactly when y <= 0.
  template <bool RES>
  __device__ __forceinline__ float code(float y, uint32_t& wn, uint32_t (&wp)[NP1]) const {
    const float a = fabsf(y);
    float mg = mag0;
#pragma unroll
    for (int k = 0; k < NPT; ++k) {
      const float e = tp[k] - a;
      wp[k] = __funnelshift_l(__float_as_uint(e), wp[k], 1);
      if constexpr (RES) mg = fmaf(mul_sat(e, -0x1p126f), dmag[k], mg);
    }
    const float ys = y - 0x1p-149f;
    wn = __funnelshift_l(__float_as_uint(ys), wn, 1);
    if constexpr (RES) return y - copysignf(mg, ys);  // c[idx] = (y > 0) ? +mag[m] : -mag[m]
    return 0.f;
  }
  // bit-plane words from the predicate words (ws = [y > 0])
  __device__ __forceinline__ void planes(uint32_t ws, const uint32_t (&wp)[NP1], uint32_t (&pl)[KB]) const {
#pragma unroll
    for (int b = 0; b < KB - 1; ++b) {
      uint32_t x = 0;
#pragma unroll
      for (int k = 0; k < NPT; ++k)
        if ((((k + 1) >> b) & 1) != ((k >> b) & 1)) x ^= wp[k];
      pl[b] = x ^ ~ws;  // m XOR (s ? 0 : all ones)
    }
    pl[KB - 1] = ws;
  }
};

// Code of this thread's half of one rotated row (y from rotate_half, ss its
// return value).  Both threads of the vector (lanes l and l ^ 16) must call it
// together: the norms are completed with a shuffle.  With RES, the residual
// pair of coordinates (64h + 2k, 64h + 2k + 1) is handed to sink(k, r) as soon
// as it is known (k descending within each code word) and g2 is its squared
// norm; pl[b][w] is plane b's word 2h + w.
template <int KB, bool RES, class Sink>
__device__ __forceinline__ void code_half(float2 (&y)[32], float ss, const Coder<KB>& cd, uint32_t (&pl)[KB][2],
                                          float& n, float& g2, Sink&& sink) {
  ss += __shfl_xor_sync(FULL, ss, 16);
  n = sqrtf(0.5f * ss);
  const float sc = (n > 0.f) ? 0.08838834764831845f / n : 0.f;  // 1/(sqrt(128) n)
  const float2 sc2 = make_float2(sc, sc);
  float2 acc = make_float2(0.f, 0.f);
#pragma unroll
  for (int w = 0; w < 2; ++w) {  // 32 coordinates per code word, highest bit first
    uint32_t wn = 0, wp[Coder<KB>::NP1];
#pragma unroll
    for (int k = 0; k < Coder<KB>::NP1; ++k) wp[k] = 0;
#pragma unroll
    for (int k = 15; k >= 0; --k) {
      const float2 v = __fmul2_rn(y[16 * w + k], sc2);
      const float r1 = cd.template code<RES>(v.y, wn, wp);  // bit 2k + 1
      const float r0 = cd.template code<RES>(v.x, wn, wp);  // bit 2k
      if constexpr (RES) {
        const float2 rv = make_float2(r0, r1);
        acc = __ffma2_rn(rv, rv, acc);
        sink(16 * w + k, rv);
      }
    }
    uint32_t p[KB];
    cd.planes(~wn, wp, p);
#pragma unroll
    for (int b = 0; b < KB; ++b) pl[b][w] = p[b];
  }
  if constexpr (RES) {
    g2 = acc.x + acc.y;
    g2 += __shfl_xor_sync(FULL, g2, 16);
  }
}

// Rare path, run by the whole warp: every projection whose two-pass
// tensor-core value lies within the rounding bound of zero is recomputed in
// fp32 from the hi+lo residual parts (2^-22 relative), four coordinates per
// lane and a shuffle reduction, and the owning lane overwrites its sign bit.
// need[u] / sgn[u] cover S rows 32 (wbase + u) .. + 31; `lanes` (warp-uniform)
// holds the lanes with at least one such projection.
__device__ __forceinline__ void fixup_signs(const uint8_t* Ss, const uint8_t* rh, const uint8_t* rl, int row,
                                            int wbase, const uint32_t (&need)[2], uint32_t (&sgn)[2],
                                            uint32_t lanes) {
  const int lane = threadIdx.x & 31;
  while (lanes) {
    const int src = __ffs(lanes) - 1;
    lanes &= lanes - 1;
    const int srow = __shfl_sync(FULL, row, src);
    const uint2 hv = *reinterpret_cast<const uint2*>(rh + canon(srow, 4 * lane));
    const uint2 lv = *reinterpret_cast<const uint2*>(rl + canon(srow, 4 * lane));
    const float2 h0 = __half22float2(*reinterpret_cast<const __half2*>(&hv.x));
    const float2 h1 = __half22float2(*reinterpret_cast<const __half2*>(&hv.y));
    const float2 l0 = __half22float2(*reinterpret_cast<const __half2*>(&lv.x));
    const float2 l1 = __half22float2(*reinterpret_cast<const __half2*>(&lv.y));
    const float r0 = h0.x + l0.x, r1 = h0.y + l0.y, r2 = h1.x + l1.x, r3 = h1.y + l1.y;
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      uint32_t nd = __shfl_sync(FULL, need[u], src);
      while (nd) {
        const int j = __ffs(nd) - 1;
        nd &= nd - 1;
        const uint2 sv = *reinterpret_cast<const uint2*>(Ss + canon(32 * (wbase + u) + j, 4 * lane));
        const float2 s0 = __half22float2(*reinterpret_cast<const __half2*>(&sv.x));
        const float2 s1 = __half22float2(*reinterpret_cast<const __half2*>(&sv.y));
        float s = fmaf(s0.x, r0, fmaf(s0.y, r1, fmaf(s1.x, r2, s1.y * r3)));
        s = warp_sum(s);
        if (lane == src) sgn[u] = s >= 0.f ? (sgn[u] | (1u << j)) : (sgn[u] & ~(1u << j));
      }
    }
  }
}

__device__ __forceinline__ void group_sync(int g) {
  asm volatile("bar.sync %0, %1;\n" ::"r"(1 + g), "n"(GT) : "memory");
}

template <int KB, bool PROD, int DT>
__global__ void __launch_bounds__(NT, 1) quantize128_kernel(const Q2Args a) {
  using L = Lay<PROD>;
  constexpr int NB = L::NB;
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = tid / GT, lt = tid % GT, wg = lt >> 5;  // group, thread and warp within the group
  const int q = wg & 3, sub = wg >> 2;                  // tensor-memory lane quadrant of the warp, its half
  const int vt = 32 * q + 16 * sub + (lane & 15);      // encode: vector of the group tile (a warp owns 16 rows)
  const int h = lane >> 4;                              // encode: coordinate half
  uint8_t* Ss = smem + L::SS;
  uint8_t* rl = smem + L::RL + g * (GV * DP * 2);
  uint32_t* dmask = reinterpret_cast<uint32_t*>(smem + L::DM);
  float* bnd = reinterpret_cast<float*>(smem + L::BND) + g * GV;
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + L::MISC) + g;  // this group's MMA-done barrier
  uint32_t* tbase = reinterpret_cast<uint32_t*>(smem + L::MISC + 16);
  float* smax = reinterpret_cast<float*>(smem + L::MISC + 20);
  auto xbuf = [&](int64_t i) { return smem + L::XS + ((int)(i % NB) * NG + g) * (GV * ROWB); };
  const int64_t n_tiles = (a.n_pad + GV - 1) / GV;
  const int64_t stride = (int64_t)gridDim.x * NG;
  const int tbytes = tile_bytes(DP, KB, a.m);
  const int cpr = a.row_bytes / 16;  // input chunks per row

  // ---- per-CTA constants -------------------------------------------------
  for (int j = tid; j < 64; j += NT) {
    uint32_t mk = 0;
    if (a.D[2 * j] < 0) mk |= 0x8000u;
    if (a.D[2 * j + 1] < 0) mk |= 0x80000000u;
    dmask[j] = mk;
  }
  if constexpr (PROD) {
    // S rows -> canonical K-major fp16 layout
    for (int e = tid; e < a.m * KCH; e += NT) {
      const int row = e / KCH, kc = e % KCH;
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(a.S + (size_t)row * DP) + kc);
      *reinterpret_cast<uint4*>(Ss + canon(row, 8 * kc)) = v;
    }
    if (warp == 0) tmem_alloc(tbase, NG * 128);
    if (tid == 0) {
      mbar_init(bar, 1);
      mbar_init(bar + 1, 1);
    }
  }
  Coder<KB> cd;
  cd.init(a.thr, a.cent);

  // stage the rows of the group's i-th tile (if any) in its buffer; rows past n_vec and
  // chunks past d are zero-filled (a buffer also serves as MMA operand, so every time)
  const int64_t tile0 = (int64_t)blockIdx.x * NG + g;
  auto issue = [&](int64_t i) {
    const int64_t tile = tile0 + i * stride;
    if (tile < n_tiles) {
      uint8_t* xs = xbuf(i);
      for (int e = lt; e < GV * KCH; e += GT) {
        const int row = e / KCH, c = e % KCH;
        const int64_t v = tile * GV + row;
        uint8_t* dst = xs + row * ROWB + ((c ^ (row & 7)) << 4);
        if (c < cpr && v < a.n_vec)
          cp_async16(dst, a.x + v * a.ld_bytes + c * 16);
        else
          *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
      }
    }
    cp_async_commit();  // possibly empty: one group per tile slot keeps the wait counts uniform
  };

#pragma unroll
  for (int i = 0; i < NB - 1; ++i) issue(i);
  __syncthreads();
  if constexpr (PROD) {
    // max_i ||S_i|| (slightly inflated so the bound stays a bound): two threads per
    // row, 16-byte reads of the canonical layout, then a block-wide maximum
    float s = 0.f;
    if (tid < 2 * a.m) {
      const int row = tid >> 1, k0 = (tid & 1) * (DP / 2);
#pragma unroll 4
      for (int k = k0; k < k0 + DP / 2; k += 8) {
        const uint4 v = *reinterpret_cast<const uint4*>(Ss + canon(row, k));
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int hh = 0; hh < 4; ++hh) {
          const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[hh]));
          s = fmaf(f.x, f.x, fmaf(f.y, f.y, s));
        }
      }
    }
    s += __shfl_xor_sync(FULL, s, 1);  // the row's two halves
    const float wmx = warp_max(s);
    float* wmax = reinterpret_cast<float*>(smem + L::MISC + 32);  // 16 floats after the barriers
    if (lane == 0) wmax[warp] = wmx;
    __syncthreads();
    if (tid == 0) {
      float mx = 0.f;
      for (int w = 0; w < NT / 32; ++w) mx = fmaxf(mx, wmax[w]);
      *smax = sqrtf(mx) * 1.0001f;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  }
  const uint32_t tmem = PROD ? *tbase + (uint32_t)(g * 128) : 0u;  // this group's accumulator columns
  const uint32_t idesc = idesc_f16_f32(128, a.m > 0 ? a.m : 128);
  const float smx = PROD ? *smax : 0.f;
  uint32_t phase = 0;

  for (int64_t i = 0; tile0 + i * stride < n_tiles; ++i) {
    const int64_t tile = tile0 + i * stride;
    uint8_t* xs = xbuf(i);
    cp_async_wait<NB - 2>();
    group_sync(g);  // tile i is staged; the buffer of tile i - 1 is free
    issue(i + NB - 1);
    const int64_t v = tile * GV + vt;
    const bool valid = v < a.n_vec, inpad = v < a.n_pad;
    uint32_t pl[KB][2];
    float n = 0.f, g2 = 0.f;
    float2 y[32];
    const float ss = rotate_half<DT>(xs + vt * ROWB, vt & 7, h, dmask, y);
    // Residuals, scaled by 2^14 (|r| < 2 for a unit vector, so no fp16 overflow and no
    // subnormal hi/lo parts), go straight into the canonical A tiles of the QJL MMA as
    // an fp16 hi part (over this warp's own staged rows, read above) and an fp16 lo part.
    if constexpr (PROD) __syncwarp();
    uint32_t hq[4], lq[4];
    auto sink = [&](int k, float2 rv) {
      if constexpr (PROD) {
        const float2 sr = __fmul2_rn(rv, make_float2(16384.f, 16384.f));
        const __half2 hv = __floats2half2_rn(sr.x, sr.y);
        const float2 dl = __ffma2_rn(__half22float2(hv), make_float2(-1.f, -1.f), sr);  // exact
        const __half2 lv = __floats2half2_rn(dl.x, dl.y);
        hq[k & 3] = *reinterpret_cast<const uint32_t*>(&hv);
        lq[k & 3] = *reinterpret_cast<const uint32_t*>(&lv);
        if ((k & 3) == 0) {  // pairs k + 3 .. k done (k descends)
          const int col = 64 * h + 2 * k;
          *reinterpret_cast<uint4*>(xs + canon(vt, col)) = make_uint4(hq[0], hq[1], hq[2], hq[3]);
          *reinterpret_cast<uint4*>(rl + canon(vt, col)) = make_uint4(lq[0], lq[1], lq[2], lq[3]);
        }
      }
    };
    // every thread codes (rows past n_vec hold zeros), so the pair's shuffles are full-warp
    code_half<KB, PROD>(y, ss, cd, pl, n, g2, sink);
    if constexpr (PROD) {
      // |z - S_i.r'| <= max||S_i|| (2^-21 + 2^-15) gamma' covers the lo-part rounding and the
      // fp32 accumulation of 256 exact products (gamma' = 2^14 gamma)
      if (h == 0) bnd[vt] = smx * (16384.f * sqrtf(g2)) * 3.1471252e-05f;  // 2^-15 + 2^-21
      fence_async_smem();
      tc_fence_before();
      group_sync(g);  // every residual written
      if (lt == 0) {
        tc_fence_after();
        const uint32_t lbo = 128, sbo = KCH * 128;
        const uint32_t sB = smem_u32(Ss);
#pragma unroll
        for (int part = 0; part < 2; ++part) {  // z = S r_hi + S r_lo
          const uint32_t sA = smem_u32(part ? rl : xs);
#pragma unroll
          for (int ks = 0; ks < DP / 16; ++ks)
            umma_f16(tmem, smem_desc(sA + ks * 256, lbo, sbo), smem_desc(sB + ks * 256, lbo, sbo), idesc,
                     (part | ks) ? 1u : 0u);
        }
        umma_commit(bar);
      }
    }

    // codes and norms of this thread's vector (plane words 2h, 2h + 1)
    if (inpad) {
      uint8_t* tb = a.codes + (v >> 5) * tbytes + (int)(v & 31) * (DP / 8) + 8 * h;
#pragma unroll
      for (int b = 0; b < KB; ++b)
        *reinterpret_cast<uint2*>(tb + b * TILE * (DP / 8)) =
            valid ? make_uint2(pl[b][0], pl[b][1]) : make_uint2(0, 0);
    }
    if (valid && h == 0) {
      a.norms[v] = __half_as_ushort(__float2half_rn(n));
      if constexpr (PROD) a.rnorms[v] = __half_as_ushort(__float2half_rn(sqrtf(g2)));
    }

    if constexpr (PROD) {
      mbar_wait(bar, phase);
      phase ^= 1u;
      tc_fence_after();
      // read back: warp wg takes rows 32q .. 32q + 31 (its lane quadrant) and columns
      // 64 sub .. + 63, i.e. sign words 2 sub and 2 sub + 1
      const int row = 32 * q + lane, wbase = 2 * sub;
      const int64_t vr = tile * GV + row;
      const bool rvalid = vr < a.n_vec;
      const float bound = bnd[row];
      const uint32_t taddr = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(32 * wbase);
      uint32_t zr[2][32];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        if (32 * (wbase + u) < a.m) {  // uniform over the warp
          tmem_ld32_issue(taddr + 32 * u, zr[u]);
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) zr[u][j] = 0u;
        }
      }
      tmem_ld_wait(zr[0]);
      tmem_ld_wait(zr[1]);
      // Sign words: the sign bits of z shifted in from the top column down (z = -0 is
      // within the bound, so the fix-up decides it).  Doubt test: |z| - max(bound, FLT_MIN)
      // is negative whenever |z| <= bound, so the OR of those differences has its sign bit
      // set when the word needs a fix-up; the exact mask is then taken by comparison.
      const float bnd2 = fmaxf(bound, 0x1p-126f);
      uint32_t sgn[2] = {0, 0}, need[2] = {0, 0};
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        uint32_t word = 0, any = 0;
#pragma unroll
        for (int j = 31; j >= 0; --j) {
          word = __funnelshift_l(zr[u][j], word, 1);
          any |= __float_as_uint(fabsf(__uint_as_float(zr[u][j])) - bnd2);
        }
        sgn[u] = ~word;
        if ((int)any < 0 && rvalid && 32 * (wbase + u) < a.m) {
          uint32_t nd = 0;
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (fabsf(__uint_as_float(zr[u][j])) <= bound) nd |= 1u << j;
          need[u] = nd;
        }
      }
      const uint32_t doubt_lanes = __ballot_sync(FULL, (need[0] | need[1]) != 0u);
      if (doubt_lanes) fixup_signs(Ss, xs, rl, row, wbase, need, sgn, doubt_lanes);  // warp-uniform
      if (vr < a.n_pad) {
        uint32_t* sd = reinterpret_cast<uint32_t*>(a.codes + (vr >> 5) * tbytes + KB * TILE * (DP / 8) +
                                                   (int)(vr & 31) * (a.m / 8));
#pragma unroll
        for (int u = 0; u < 2; ++u)
          if (32 * (wbase + u) < a.m) sd[wbase + u] = rvalid ? sgn[u] : 0u;
      }
      tc_fence_before();
    }
  }
  cp_async_wait<0>();
  if constexpr (PROD) {
    __syncthreads();
    if (warp == 0) tmem_dealloc(*tbase, NG * 128);
  }
}

template <int KB, bool PROD, int DT>
int launch_q2(const Q2Args& a, int sm_count, cudaStream_t st) {
  auto kern = quantize128_kernel<KB, PROD, DT>;
  constexpr int smem = Lay<PROD>::TOTAL;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return tq::set_error(TQ_ECUDA, "tq_quantize: %s", cudaGetErrorString(e));
  const int64_t tiles = (a.n_pad + GV - 1) / GV;
  const int blocks = (int)std::max<int64_t>(1, std::min<int64_t>((tiles + NG - 1) / NG, sm_count));
  kern<<<blocks, NT, smem, st>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return tq::set_error(TQ_ECUDA, "tq_quantize: launch failed: %s", cudaGetErrorString(e));
  return TQ_OK;
}

template <bool PROD, int DT>
int dispatch_kb2(int kb, const Q2Args& a, int smc, cudaStream_t st) {
  switch (kb) {
    case 1: return launch_q2<1, PROD, DT>(a, smc, st);
    case 2: return launch_q2<2, PROD, DT>(a, smc, st);
    case 3: return launch_q2<3, PROD, DT>(a, smc, st);
    default: return launch_q2<4, PROD, DT>(a, smc, st);
  }
}

}  // namespace

namespace tq {

// Whether the one-thread-per-vector tensor-core kernel handles this call.
bool quantize128_supported(const tq_params* p, int dtype) {
  return p->d_pad == 128 && (dtype == TQ_BF16 || dtype == TQ_F16) && (p->mode == TQ_MODE_MSE || p->m <= 128);
}

int launch_quantize128(const tq_params* p, const void* x, int dtype, int64_t n_vec, int64_t ld_bytes, void* codes,
                       uint16_t* norms, uint16_t* rnorms, int smc, cudaStream_t st) {
  Q2Args a;
  a.x = static_cast<const uint8_t*>(x);
  a.n_vec = n_vec;
  a.n_pad = (n_vec + 31) / 32 * 32;
  a.ld_bytes = ld_bytes;
  a.d = p->d;
  a.m = p->mode == TQ_MODE_PROD ? p->m : 0;
  a.row_bytes = p->d * 2;
  a.codes = static_cast<uint8_t*>(codes);
  a.norms = norms;
  a.rnorms = rnorms;
  a.cent = p->centroids;
  a.thr = p->thresholds;
  a.D = p->signs_D;
  a.S = p->S;
  const int kb = index_bits(p);
  const bool prod = p->mode == TQ_MODE_PROD;
  if (dtype == TQ_BF16)
    return prod ? dispatch_kb2<true, TQ_BF16>(kb, a, smc, st) : dispatch_kb2<false, TQ_BF16>(kb, a, smc, st);
  return prod ? dispatch_kb2<true, TQ_F16>(kb, a, smc, st) : dispatch_kb2<false, TQ_F16>(kb, a, smc, st);
}

}  // namespace tq

namespace tq {
// Read (and optionally clear) this translation unit's device fault word.
int fault_word_quantize(int clear, int* value) {
  cudaError_t e = cudaMemcpyFromSymbol(value, tqd::g_fault, sizeof(int));
  if (e == cudaSuccess && clear) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(tqd::g_fault, &zero, sizeof(int));
  }
  return e == cudaSuccess ? TQ_OK : set_error(TQ_ECUDA, "tq_device_status: %s", cudaGetErrorString(e));
}
}  // namespace tq
