// tq_quantize for d_pad = 128 (m <= 128): one thread per vector, QJL projection
// on the 5th-generation tensor cores.
//
// Method ("TurboQuant explainer" (m.163.com), "第一步：PolarQuant" and
// "第二步：QJL"): norm, random sign flips + Walsh-Hadamard rotation, Lloyd-Max
// code at b-1 bits, residual and its norm, sign bits of S r.
//
// Design (B200, sm_100a):
//  * A CTA of 256 threads owns a tile of 256 vectors; thread v encodes vector
//    v of the tile entirely in registers: no shuffles and no cross-lane
//    reductions.  The tile's input rows are staged in shared memory with
//    cp.async (16-byte chunks, XOR-swizzled per row so that a thread reading
//    its own row is bank-conflict free); the next tile is fetched as soon as
//    the current rows are in registers.
//  * Rotation: the first Walsh-Hadamard stage is fused with the bf16/fp16
//    unpacking and the sign flips (applied to the raw bits); the other six
//    stages run on Blackwell's packed f32x2 add/fma.  y is scaled once by
//    1/(||x|| sqrt(128)).
//  * Code: with p_k = [|y| > t_{L/2+k}] (monotone in k) and s = [y > 0] the
//    index is idx = s ? L/2 + m : L/2-1 - m with m = sum_k p_k; bit b of m is
//    the XOR of the p_k at which bit b of k+1 differs from bit b of k.  Each
//    predicate is packed into a 32-bit word with one predicated OR, and the
//    bit-planes are a few word-wide XORs.  The residual is |y| - mag[m] with
//    the sign of s.
//  * QJL: residuals are written to shared memory in the UMMA K-major
//    canonical layout; one thread issues tcgen05.mma (M=128, N=m, K=16)
//    x 16 per half tile against S (fp16, exact) with fp32
//    accumulation in tensor memory; every thread reads its own row back with
//    tcgen05.ld.32x32b.  The residual (scaled by 2^14) is split into fp16 hi
//    and lo parts and the MMA runs twice into the same accumulator
//    (S r_hi + S r_lo), so z is exact to ~2^-22 before fp32 accumulation.  A
//    projection with |z| below the accumulation bound (about 0.03 per vector)
//    is recomputed in fp32 from hi+lo by its thread.
#include <cuda_runtime.h>

#include <algorithm>

#include "common.h"
#include "device.cuh"
#include "tc.cuh"

namespace {

using namespace tqd;

constexpr int NV = 256;        // vectors per tile (threads per CTA)
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

// shared-memory carve-up
struct Lay {
  static constexpr int XS = 0;                    // [NV][ROWB] staged input (swizzled chunks)
  static constexpr int SS = XS + NV * ROWB;       // S, canonical K-major fp16, 128 rows max
  static constexpr int RS = SS + 128 * DP * 2;    // residuals (hi part) fp16, canonical, two 128-row halves
  static constexpr int RL = RS + NV * DP * 2;     // residuals (lo part), same layout
  static constexpr int DM = RL + NV * DP * 2;     // sign-flip masks, 64 x uint32 (bits 15, 31)
  static constexpr int MISC = DM + 64 * 4;        // mbarriers (+0, +16), tmem base (+8), max ||S_i|| (+12), 8 floats (+32)
  static constexpr int TOTAL = MISC + 64;
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

// Rotation of one staged row: y (64 float2 = 128 values) = H (D o x), unnormalized; returns ||x||^2.
template <int DT>
__device__ __forceinline__ float rotate_row(const uint8_t* xrow, int sw, int d, const uint32_t* dmask,
                                            float2 (&y)[64]) {
  float ss = 0.f;
#pragma unroll
  for (int c = 0; c < KCH; ++c) {  // chunk c = elements 8c..8c+7
    uint4 v = make_uint4(0, 0, 0, 0);
    if (8 * c < d) v = *reinterpret_cast<const uint4*>(xrow + ((c ^ sw) << 4));
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      float x0, x1;
      unpack_pair<DT>(w[h], dmask[4 * c + h], x0, x1);
      if (8 * c + 2 * h >= d) x0 = 0.f;
      if (8 * c + 2 * h + 1 >= d) x1 = 0.f;
      ss = fmaf(x0, x0, fmaf(x1, x1, ss));
      y[4 * c + h] = make_float2(x0 + x1, x0 - x1);  // Walsh-Hadamard stage on bit 0
    }
  }
  const float2 neg1 = make_float2(-1.f, -1.f);
#pragma unroll
  for (int hs = 1; hs < 64; hs <<= 1) {  // stages on bits 1..6 (pairs of pairs)
#pragma unroll
    for (int k = 0; k < 64; ++k) {
      if ((k & hs) == 0) {
        const float2 u = y[k], w = y[k + hs];
        y[k] = __fadd2_rn(u, w);
        y[k + hs] = __ffma2_rn(w, neg1, u);
      }
    }
  }
  return ss;
}

// Scalar code of one coordinate: returns the residual and ORs the predicate bits into the words.
template <int KB>
struct Coder {
  static constexpr int L = 1 << KB;
  static constexpr int NPT = L / 2 - 1;  // positive thresholds t_{L/2} .. t_{L-2}
  static constexpr int NP1 = NPT > 0 ? NPT : 1;
  float tp[NP1];        // positive thresholds
  float mag[NPT + 1];   // c[L/2 .. L-1]

  __device__ __forceinline__ void init(const float* thr, const float* cent) {
#pragma unroll
    for (int k = 0; k < NPT; ++k) tp[k] = thr[L / 2 + k];
#pragma unroll
    for (int k = 0; k <= NPT; ++k) mag[k] = cent[L / 2 + k];
  }
  // ws: word of [y > 0]; wp[k]: word of [|y| > t_{L/2+k}].  Returns y - c[idx].
  __device__ __forceinline__ float code(float y, uint32_t bit, uint32_t& ws, uint32_t (&wp)[NP1]) const {
    const float a = fabsf(y);
    float mg = mag[0];
#pragma unroll
    for (int k = 0; k < NPT; ++k) {
      if (a > tp[k]) {
        wp[k] |= bit;
        mg = mag[k + 1];
      }
    }
    const bool s = y > 0.f;
    if (s) ws |= bit;
    return s ? (y - mg) : (y + mg);  // c[idx] = s ? +mag[m] : -mag[m]
  }
  // bit-plane words from the predicate words
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

// Full encode of one row - shared by the main path and the fix-up path.  The
// residual pair of coordinates (2k, 2k+1) is handed to sink(k, r0, r1) as soon
// as it is known, so the main path never holds all 128 residuals.
template <int KB, int DT, class Sink>
__device__ __forceinline__ void encode_row(const uint8_t* xrow, int sw, int d, const uint32_t* dmask,
                                           const Coder<KB>& cd, uint32_t (&pl)[KB][4], float& n, float& g2,
                                           Sink&& sink) {
  float2 y[64];
  const float ss = rotate_row<DT>(xrow, sw, d, dmask, y);
  n = sqrtf(ss);
  const float sc = (n > 0.f) ? 0.08838834764831845f / n : 0.f;  // 1/(sqrt(128) n)
  const float2 sc2 = make_float2(sc, sc);
  float2 acc = make_float2(0.f, 0.f);
#pragma unroll
  for (int w = 0; w < 4; ++w) {  // 32 coordinates per code word
    uint32_t ws = 0, wp[Coder<KB>::NP1];
#pragma unroll
    for (int k = 0; k < Coder<KB>::NP1; ++k) wp[k] = 0;
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const float2 v = __fmul2_rn(y[16 * w + k], sc2);
      const float r0 = cd.code(v.x, 1u << (2 * k), ws, wp);
      const float r1 = cd.code(v.y, 1u << (2 * k + 1), ws, wp);
      const float2 rv = make_float2(r0, r1);
      acc = __ffma2_rn(rv, rv, acc);
      sink(16 * w + k, rv);
    }
    uint32_t p[KB];
    cd.planes(ws, wp, p);
#pragma unroll
    for (int b = 0; b < KB; ++b) pl[b][w] = p[b];
  }
  g2 = acc.x + acc.y;
}

// Rare path, run by the whole warp: every projection whose two-pass
// tensor-core value lies within the rounding bound of zero is recomputed in
// fp32 from the hi+lo residual parts (2^-22 relative), four coordinates per
// lane and a shuffle reduction, and the owning lane overwrites its sign bit.
// `lanes` (warp-uniform) holds the lanes with at least one such projection.
__device__ __forceinline__ void fixup_signs(const uint8_t* Ss, const uint8_t* rh, const uint8_t* rl, int row,
                                         const uint32_t (&need)[4], uint32_t (&sgn)[4], uint32_t lanes) {
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
    for (int w = 0; w < 4; ++w) {
      uint32_t nd = __shfl_sync(FULL, need[w], src);
      while (nd) {
        const int j = __ffs(nd) - 1;
        nd &= nd - 1;
        const uint2 sv = *reinterpret_cast<const uint2*>(Ss + canon(32 * w + j, 4 * lane));
        const float2 s0 = __half22float2(*reinterpret_cast<const __half2*>(&sv.x));
        const float2 s1 = __half22float2(*reinterpret_cast<const __half2*>(&sv.y));
        float s = fmaf(s0.x, r0, fmaf(s0.y, r1, fmaf(s1.x, r2, s1.y * r3)));
        s = warp_sum(s);
        if (lane == src) sgn[w] = s >= 0.f ? (sgn[w] | (1u << j)) : (sgn[w] & ~(1u << j));
      }
    }
  }
}

template <int KB, bool PROD, int DT>
__global__ void __launch_bounds__(NV, 1) quantize128_kernel(const Q2Args a) {
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* xs = smem + Lay::XS;
  uint8_t* Ss = smem + Lay::SS;
  uint8_t* Rs = smem + Lay::RS;
  uint32_t* dmask = reinterpret_cast<uint32_t*>(smem + Lay::DM);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + Lay::MISC);  // [0]: half 0 done, [2]: half 1 done
  uint32_t* tbase = reinterpret_cast<uint32_t*>(smem + Lay::MISC + 8);
  float* smax = reinterpret_cast<float*>(smem + Lay::MISC + 12);
  const int tid = threadIdx.x, warp = tid >> 5;
  const int64_t n_tiles = (a.n_pad + NV - 1) / NV;
  const int tbytes = tile_bytes(DP, KB, a.m);

  // ---- per-CTA constants -------------------------------------------------
  for (int j = tid; j < 64; j += NV) {
    uint32_t mk = 0;
    if (a.D[2 * j] < 0) mk |= 0x8000u;
    if (a.D[2 * j + 1] < 0) mk |= 0x80000000u;
    dmask[j] = mk;
  }
  if constexpr (PROD) {
    // S rows -> canonical K-major fp16 layout
    for (int e = tid; e < a.m * KCH; e += NV) {
      const int row = e / KCH, kc = e % KCH;
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(a.S + (size_t)row * DP) + kc);
      *reinterpret_cast<uint4*>(Ss + canon(row, 8 * kc)) = v;
    }
    if (warp == 0) tmem_alloc(tbase, 256);
    if (tid == 0) {
      mbar_init(bar, 1);
      mbar_init(bar + 2, 1);
    }
  }
  Coder<KB> cd;
  cd.init(a.thr, a.cent);

  auto issue = [&](int64_t tile) {
    const int cpr = a.row_bytes / 16;
    for (int e = tid; e < NV * 16; e += NV) {
      const int row = e >> 4, c = e & 15;
      const int64_t v = tile * NV + row;
      if (c < cpr && v < a.n_vec)
        cp_async16(xs + row * ROWB + ((c ^ (row & 7)) << 4), a.x + v * a.ld_bytes + c * 16);
    }
    cp_async_commit();
  };

  int64_t tile = blockIdx.x;
  if (tile < n_tiles) issue(tile);
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
        for (int h = 0; h < 4; ++h) {
          const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[h]));
          s = fmaf(f.x, f.x, fmaf(f.y, f.y, s));
        }
      }
    }
    s += __shfl_xor_sync(FULL, s, 1);  // the row's two halves
    const float wmx = warp_max(s);
    float* wmax = reinterpret_cast<float*>(smem + Lay::MISC + 32);  // 8 floats after the barriers
    if ((tid & 31) == 0) wmax[warp] = wmx;
    __syncthreads();
    if (tid == 0) {
      float mx = 0.f;
      for (int w = 0; w < NV / 32; ++w) mx = fmaxf(mx, wmax[w]);
      *smax = sqrtf(mx) * 1.0001f;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  }
  const uint32_t tmem = PROD ? *tbase : 0u;
  const uint32_t idesc = idesc_f16_f32(128, a.m > 0 ? a.m : 128);
  uint32_t phase = 0;

  for (; tile < n_tiles; tile += gridDim.x) {
    cp_async_wait<0>();
    __syncthreads();
    const int64_t v = tile * NV + tid;
    const bool valid = v < a.n_vec, inpad = v < a.n_pad;
    uint32_t pl[KB][4];
    float n = 0.f, g2 = 0.f;
    // Residuals, scaled by 2^14 (|r| < 2 for a unit vector, so no fp16 overflow and no
    // subnormal hi/lo parts), go straight into the canonical A tiles of the QJL MMA as
    // an fp16 hi part and an fp16 lo part (zeros for rows without a vector).
    const int half = tid >> 7, row = tid & 127;
    uint8_t* ra = Rs + half * (128 * DP * 2);
    uint8_t* rl = smem + Lay::RL + half * (128 * DP * 2);
    uint32_t hq[4], lq[4];
    auto sink = [&](int k, float2 rv) {
      if constexpr (PROD) {
        const float2 sr = __fmul2_rn(rv, make_float2(16384.f, 16384.f));
        const __half2 hv = __floats2half2_rn(sr.x, sr.y);
        const float2 dl = __ffma2_rn(__half22float2(hv), make_float2(-1.f, -1.f), sr);  // exact
        const __half2 lv = __floats2half2_rn(dl.x, dl.y);
        hq[k & 3] = *reinterpret_cast<const uint32_t*>(&hv);
        lq[k & 3] = *reinterpret_cast<const uint32_t*>(&lv);
        if ((k & 3) == 3) {
          *reinterpret_cast<uint4*>(ra + canon(row, 2 * (k - 3))) = make_uint4(hq[0], hq[1], hq[2], hq[3]);
          *reinterpret_cast<uint4*>(rl + canon(row, 2 * (k - 3))) = make_uint4(lq[0], lq[1], lq[2], lq[3]);
        }
      }
    };
    if (valid) {
      encode_row<KB, DT>(xs + tid * ROWB, tid & 7, a.d, dmask, cd, pl, n, g2, sink);
    } else if (PROD) {
#pragma unroll
      for (int kc = 0; kc < KCH; ++kc) {
        *reinterpret_cast<uint4*>(ra + canon(row, 8 * kc)) = make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4*>(rl + canon(row, 8 * kc)) = make_uint4(0, 0, 0, 0);
      }
    }
    __syncthreads();  // every row is consumed: refill the staging buffer with the next tile
    if (tile + gridDim.x < n_tiles) issue(tile + gridDim.x);

    uint8_t* tb = a.codes + (v >> 5) * tbytes;
    const int slot = (int)(v & 31);
    if (inpad) {
#pragma unroll
      for (int b = 0; b < KB; ++b) {
        const uint4 w = valid ? make_uint4(pl[b][0], pl[b][1], pl[b][2], pl[b][3]) : make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4*>(tb + b * TILE * (DP / 8) + slot * (DP / 8)) = w;
      }
    }
    if (valid) a.norms[v] = __half_as_ushort(__float2half_rn(n));
    if constexpr (PROD) {
      const float gm = sqrtf(g2);
      if (valid) a.rnorms[v] = __half_as_ushort(__float2half_rn(gm));
      // |z - S_i.r'| <= max||S_i|| (2^-21 + 2^-15) gamma' covers the lo-part rounding and the
      // fp32 accumulation of 256 exact products (gamma' = 2^14 gamma)
      const float bound = (*smax) * (16384.f * gm) * 3.1471252e-05f;  // 2^-15 + 2^-21
      fence_async_smem();
      tc_fence_before();
      __syncthreads();
      tc_fence_after();
      if (tid == 0) {
        const uint32_t lbo = 128, sbo = KCH * 128;
        const uint32_t sB = smem_u32(Ss);
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
#pragma unroll
          for (int part = 0; part < 2; ++part) {  // z = S r_hi + S r_lo
            const uint32_t sA = smem_u32(smem + (part ? Lay::RL : Lay::RS) + hf * (128 * DP * 2));
#pragma unroll
            for (int ks = 0; ks < DP / 16; ++ks)
              umma_f16(tmem + hf * 128, smem_desc(sA + ks * 256, lbo, sbo), smem_desc(sB + ks * 256, lbo, sbo),
                       idesc, (part | ks) ? 1u : 0u);
          }
          // these MMAs keep the tensor pipe busy (~64 cycles each), so one issuing thread
          // suffices; committing per half lets the first half's warps read while the second computes
          umma_commit(bar + 2 * hf);
        }
      }
      mbar_wait(bar + 2 * half, phase);
      phase ^= 1u;
      tc_fence_after();
      // read back this vector's projections: lane = row within its half, columns [half*128, half*128 + m)
      const uint32_t taddr = tmem + ((uint32_t)((warp & 3) * 32) << 16) + (uint32_t)(half * 128);
      // two loads in flight per wait; sign bits and the doubt mask (|z| within the bound) in one sweep
      uint32_t sgn[4] = {0, 0, 0, 0}, need[4] = {0, 0, 0, 0};
#pragma unroll
      for (int w2 = 0; w2 < 4; w2 += 2) {
        uint32_t zr[2][32];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          if (32 * (w2 + u) < a.m) {  // uniform over the warp
            tmem_ld32_issue(taddr + 32 * (w2 + u), zr[u]);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) zr[u][j] = 0u;
          }
        }
        tmem_ld_wait(zr[0]);
        tmem_ld_wait(zr[1]);
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          if (32 * (w2 + u) < a.m) {
            uint32_t word = 0, nd = 0;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const float z = __uint_as_float(zr[u][j]);
              if (z >= 0.f) word |= 1u << j;
              if (fabsf(z) <= bound) nd |= 1u << j;
            }
            sgn[w2 + u] = word;
            need[w2 + u] = valid ? nd : 0u;
          }
        }
      }
      const bool doubt = (need[0] | need[1] | need[2] | need[3]) != 0u;
      const uint32_t doubt_lanes = __ballot_sync(FULL, doubt);
      if (doubt_lanes) fixup_signs(Ss, ra, rl, row, need, sgn, doubt_lanes);  // warp-uniform
      if (inpad) {
        uint32_t* sd = reinterpret_cast<uint32_t*>(tb + KB * TILE * (DP / 8) + slot * (a.m / 8));
#pragma unroll
        for (int w = 0; w < 4; ++w)
          if (32 * w < a.m) sd[w] = valid ? sgn[w] : 0u;
      }
      tc_fence_before();
    }
  }
  cp_async_wait<0>();
  if constexpr (PROD) {
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 256);
  }
}

template <int KB, bool PROD, int DT>
int launch_q2(const Q2Args& a, int sm_count, cudaStream_t st) {
  auto kern = quantize128_kernel<KB, PROD, DT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Lay::TOTAL);
  if (e != cudaSuccess) return tq::set_error(TQ_ECUDA, "tq_quantize: %s", cudaGetErrorString(e));
  const int64_t tiles = (a.n_pad + NV - 1) / NV;
  const int blocks = (int)std::max<int64_t>(1, std::min<int64_t>(tiles, sm_count));
  kern<<<blocks, NV, Lay::TOTAL, st>>>(a);
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
