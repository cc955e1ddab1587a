// Polar-coordinate stage 1 ("TurboQuant explainer" (m.163.com),
// "第一步：PolarQuant" and "第一步：PolarQuant —— 换个坐标系压缩"): the
// rotated unit vector y is rewritten in recursive pairwise polar form - level 1
// turns coordinate pairs into (radius, full angle theta), level l >= 2 turns
// pairs of level-(l-1) radii into (radius, psi in [0, pi/2]) - and every
// angle is coded with its level's Lloyd-Max table (level 1: 2^(w+1) equal
// cells; higher levels: 2^(w-1) cells of the law sin^2 psi ~ Beta).
//
//  * tq_polar_quantize: a warp per vector, lane l holding coordinates
//    NI l .. NI l + NI - 1 (NI = d_pad / 32).  Rotation by in-lane and
//    shuffle Walsh-Hadamard stages; the levels whose pairs lie inside a lane
//    are formed there, the others across lanes with shuffles.  No angle is
//    computed: a level-1 cell is the quadrant (signs) and the position inside
//    it (cross products with the cell boundaries), a higher-level decision
//    psi > t is rb cos t > ra sin t.  Indices are OR-ed into the warp's
//    record in shared memory and stored by the first lanes as consecutive
//    words.
//  * tq_polar_dequantize: a warp per vector; each lane rebuilds its radius
//    from the root down (cos / sin of its ancestors' centroids), then its
//    coordinates, then the inverse rotation.
//  * tq_polar_logits: a thread per key; the record is held in registers and
//    the tree is walked depth first (every bit position is a compile-time
//    constant), accumulating <q~, y_hat> for the key's query group from
//    rotated queries in shared memory.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>

#include "common.h"
#include "device.cuh"
#include "prep.h"

namespace {
using namespace tqd;

template <int DP, int W>
struct PL {
  static constexpr int NI = DP / 32;                          // coordinates per lane
  static constexpr int LV = DP == 128 ? 7 : 8;                // levels
  static constexpr int LI = NI == 4 ? 2 : 3;                  // levels formed inside a lane
  static constexpr int B1 = W + 1, B2 = W - 1;
  static constexpr int L1 = 1 << B1, L2 = 1 << B2;
  static constexpr int NW = W * DP / 32;                      // 32-bit words of a record
  static constexpr int T1 = 3 * L1;                           // table offset of level 2
  static constexpr int TL = 4 * L2 - 1;                       // table values per level >= 2
  // bit position of index u of level l (l = 1: pair u)
  static constexpr __host__ __device__ int pos(int l, int u) {
    int p = l == 1 ? B1 * u : B1 * (DP / 2);
    for (int k = 2; k < l; ++k) p += B2 * (DP >> k);
    return l == 1 ? p : p + B2 * u;
  }
};

struct PArgs {
  const uint8_t* x;
  int64_t n_vec, ld;  // ld in elements (quantize) or floats (dequantize)
  int d;
  const float* tables;
  const int8_t* D;
  uint8_t* codes;
  const uint8_t* ccodes;
  uint16_t* norms;
  const uint16_t* cnorms;
  float* out;
  // logits
  const float* q;
  float* logits;
  int64_t n_keys;
  int group;
};

// ---- quantize ---------------------------------------------------------------
template <int DP, int W, int DT>
__global__ void __launch_bounds__(256) polar_quantize_kernel(const PArgs a) {
  using P = PL<DP, W>;
  constexpr int NI = P::NI;
  __shared__ uint32_t rec[8][P::NW];
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  // (cos t, sin t) of the higher levels' thresholds t: psi > t exactly when rb cos t > ra sin t
  // (psi = atan2(rb, ra) and t both in [0, pi/2])
  float thc[P::LV - 1][P::L2 > 1 ? P::L2 - 1 : 1], ths[P::LV - 1][P::L2 > 1 ? P::L2 - 1 : 1];
#pragma unroll
  for (int l = 2; l <= P::LV; ++l)
#pragma unroll
    for (int j = 0; j < P::L2 - 1; ++j) sincosf(__ldg(a.tables + P::T1 + (l - 2) * P::TL + P::L2 + j), &ths[l - 2][j], &thc[l - 2][j]);
  float dsg[NI];
#pragma unroll
  for (int k = 0; k < NI; ++k) dsg[k] = (float)a.D[NI * lane + k];
  if (lane < P::NW) rec[wib][lane] = 0u;
  __syncwarp();
  const float rs = rsqrtf((float)DP);
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t v = (int64_t)blockIdx.x * (blockDim.x >> 5) + wib; v < a.n_vec; v += warps) {
    const uint8_t* row = a.x + v * a.ld * (DT == TQ_F32 ? 4 : 2);
    float y[NI];
    float ss = 0.f;
    // groups of 4 elements (d is a multiple of 4, of 8 for 16-bit types): one 8- or 16-byte load each
#pragma unroll
    for (int g4 = 0; g4 < NI / 4; ++g4) {
      const int j = NI * lane + 4 * g4;
      float e[4] = {0.f, 0.f, 0.f, 0.f};
      if (j < a.d) {
        if constexpr (DT == TQ_F32) {
          const float4 f = __ldg(reinterpret_cast<const float4*>(row) + (j >> 2));
          e[0] = f.x, e[1] = f.y, e[2] = f.z, e[3] = f.w;
        } else {
          const uint2 u = __ldg(reinterpret_cast<const uint2*>(row) + (j >> 2));
          const uint32_t wd[2] = {u.x, u.y};
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            if constexpr (DT == TQ_BF16) {
              e[2 * h] = __uint_as_float(wd[h] << 16);
              e[2 * h + 1] = __uint_as_float(wd[h] & 0xFFFF0000u);
            } else {
              const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&wd[h]));
              e[2 * h] = f.x, e[2 * h + 1] = f.y;
            }
          }
        }
      }
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        y[4 * g4 + k] = e[k] * dsg[4 * g4 + k];
        ss = fmaf(y[4 * g4 + k], y[4 * g4 + k], ss);
      }
    }
    ss = warp_sum(ss);
    const float n = sqrtf(ss);
    // Walsh-Hadamard: in-lane stages, then across lanes
#pragma unroll
    for (int hs = 1; hs < NI; hs <<= 1)
#pragma unroll
      for (int k = 0; k < NI; ++k)
        if ((k & hs) == 0) {
          const float u = y[k], w = y[k + hs];
          y[k] = u + w;
          y[k + hs] = u - w;
        }
#pragma unroll
    for (int s = 1; s < 32; s <<= 1)
#pragma unroll
      for (int k = 0; k < NI; ++k) {
        const float o = __shfl_xor_sync(FULL, y[k], s);
        y[k] = (lane & s) ? (o - y[k]) : (y[k] + o);
      }
    const float sc = n > 0.f ? rs / n : 0.f;
#pragma unroll
    for (int k = 0; k < NI; ++k) y[k] *= sc;

    uint32_t* r = rec[wib];
    auto put = [&](int p, uint32_t idx) {  // OR `idx` in at bit position p
      if (idx == 0u) return;
      atomicOr(&r[p >> 5], idx << (p & 31));
      if ((p & 31) != 0 && (idx >> (32 - (p & 31))) != 0u) atomicOr(&r[(p >> 5) + 1], idx >> (32 - (p & 31)));
    };
    auto angle_index = [&](int l, float ra, float rb) {
      int ix = 0;
#pragma unroll
      for (int j = 0; j < P::L2 - 1; ++j) ix += rb * thc[l - 2][j] > ra * ths[l - 2][j] ? 1 : 0;
      return (uint32_t)ix;
    };
    // level 1: cell floor(theta L1 / 2 pi) of theta = atan2(x1, x0) in [0, 2 pi), by the quadrant
    // (signs) and the position inside it (cross products with the cell boundaries)
    float rad[NI / 2];
#pragma unroll
    for (int j = 0; j < NI / 2; ++j) {
      const float x0 = y[2 * j], x1 = y[2 * j + 1];
      const int qd = x1 > 0.f ? (x0 > 0.f ? 0 : 1) : (x1 < 0.f ? (x0 < 0.f ? 2 : 3) : (x0 < 0.f ? 2 : 0));
      const float u = qd == 0 ? x0 : qd == 1 ? x1 : qd == 2 ? -x0 : -x1;  // rotated into [0, pi/2)
      const float w = qd == 0 ? x1 : qd == 1 ? -x0 : qd == 2 ? -x1 : x0;
      int sub = 0;
      if constexpr (P::L1 == 8) sub = w >= u ? 1 : 0;
      if constexpr (P::L1 == 16)
        sub = (w * 0.92387953f >= u * 0.38268343f ? 1 : 0) + (w >= u ? 1 : 0) +
              (w * 0.38268343f >= u * 0.92387953f ? 1 : 0);  // boundaries pi/8, pi/4, 3 pi/8
      put(P::pos(1, (NI / 2) * lane + j), (uint32_t)(qd * (P::L1 / 4) + sub));
      rad[j] = sqrtf(fmaf(x0, x0, x1 * x1));
    }
    // levels inside the lane
#pragma unroll
    for (int l = 2; l <= P::LI; ++l) {
      const int cnt = NI >> l;  // nodes of level l in this lane
#pragma unroll
      for (int j = 0; j < cnt; ++j) {
        const float ra = rad[2 * j], rb = rad[2 * j + 1];
        if constexpr (P::B2 > 0) put(P::pos(l, cnt * lane + j), angle_index(l, ra, rb));
        rad[j] = sqrtf(fmaf(ra, ra, rb * rb));
      }
    }
    // levels across lanes: node = lane >> (l - LI), partner lane differs in bit l - LI - 1
    float R = rad[0];
#pragma unroll
    for (int l = P::LI + 1; l <= P::LV; ++l) {
      const int s = 1 << (l - P::LI - 1);
      const float o = __shfl_xor_sync(FULL, R, s);
      const float ra = (lane & s) ? o : R, rb = (lane & s) ? R : o;
      if constexpr (P::B2 > 0)
        if ((lane & (2 * s - 1)) == 0) put(P::pos(l, lane >> (l - P::LI)), angle_index(l, ra, rb));
      R = sqrtf(fmaf(ra, ra, rb * rb));
    }
    __syncwarp();
    if (lane < P::NW) {
      reinterpret_cast<uint32_t*>(a.codes + v * (P::NW * 4))[lane] = r[lane];
      r[lane] = 0u;
    }
    if (lane == 0) a.norms[v] = __half_as_ushort(__float2half_rn(n));
    __syncwarp();
  }
}

// ---- dequantize ---------------------------------------------------------------
template <int DP, int W>
__global__ void __launch_bounds__(256) polar_dequantize_kernel(const PArgs a) {
  using P = PL<DP, W>;
  constexpr int NI = P::NI;
  __shared__ uint32_t rec[8][P::NW + 1];
  __shared__ float tab[P::T1 + (P::LV - 1) * P::TL];
  for (int i = threadIdx.x; i < P::T1 + (P::LV - 1) * P::TL; i += blockDim.x) tab[i] = a.tables[i];
  __syncthreads();
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  float dsg[NI];
#pragma unroll
  for (int k = 0; k < NI; ++k) dsg[k] = (float)a.D[NI * lane + k];
  if (lane == 0) rec[wib][P::NW] = 0u;
  const float rs = rsqrtf((float)DP);
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t v = (int64_t)blockIdx.x * (blockDim.x >> 5) + wib; v < a.n_vec; v += warps) {
    uint32_t* r = rec[wib];
    if (lane < P::NW) r[lane] = __ldg(reinterpret_cast<const uint32_t*>(a.ccodes + v * (P::NW * 4)) + lane);
    __syncwarp();
    auto get = [&](int p, int width) {
      const uint64_t w64 = (uint64_t)r[p >> 5] | ((uint64_t)r[(p >> 5) + 1] << 32);
      return (int)((w64 >> (p & 31)) & ((1u << width) - 1u));
    };
    auto cs = [&](int l, int ix) {  // (cos, sin) of the centroid ix of level l >= 2
      const float* t = tab + P::T1 + (l - 2) * P::TL + 2 * P::L2 - 1;
      return make_float2(t[2 * ix], t[2 * ix + 1]);
    };
    // root to this lane's node of level LI
    float R = 1.f;
#pragma unroll
    for (int l = P::LV; l > P::LI; --l) {
      const int ix = P::B2 > 0 ? get(P::pos(l, lane >> (l - P::LI)), P::B2) : 0;
      const float2 c = cs(l, ix);
      R *= ((lane >> (l - P::LI - 1)) & 1) ? c.y : c.x;
    }
    // levels inside the lane, from LI down to 2
    float rad[NI / 2];
    rad[0] = R;
#pragma unroll
    for (int l = P::LI; l >= 2; --l) {
      const int cnt = NI >> l;
#pragma unroll
      for (int j = cnt - 1; j >= 0; --j) {
        const int ix = P::B2 > 0 ? get(P::pos(l, cnt * lane + j), P::B2) : 0;
        const float2 c = cs(l, ix);
        const float pr = rad[j];
        rad[2 * j] = pr * c.x;
        rad[2 * j + 1] = pr * c.y;
      }
    }
    float y[NI];
#pragma unroll
    for (int j = 0; j < NI / 2; ++j) {
      const int ix = get(P::pos(1, (NI / 2) * lane + j), P::B1);
      y[2 * j] = rad[j] * tab[P::L1 + 2 * ix];
      y[2 * j + 1] = rad[j] * tab[P::L1 + 2 * ix + 1];
    }
    __syncwarp();
    // inverse rotation D H y / sqrt(DP), times the norm
#pragma unroll
    for (int hs = 1; hs < NI; hs <<= 1)
#pragma unroll
      for (int k = 0; k < NI; ++k)
        if ((k & hs) == 0) {
          const float u = y[k], w = y[k + hs];
          y[k] = u + w;
          y[k + hs] = u - w;
        }
#pragma unroll
    for (int s = 1; s < 32; s <<= 1)
#pragma unroll
      for (int k = 0; k < NI; ++k) {
        const float o = __shfl_xor_sync(FULL, y[k], s);
        y[k] = (lane & s) ? (o - y[k]) : (y[k] + o);
      }
    const float nrm = __half2float(__ushort_as_half(__ldg(a.cnorms + v))) * rs;
    float* orow = a.out + v * a.ld;
#pragma unroll
    for (int k = 0; k < NI; ++k) {
      const int c = NI * lane + k;
      if (c < a.d) orow[c] = y[k] * nrm * dsg[k];
    }
  }
}

// ---- logits ---------------------------------------------------------------------
template <int DP, int W, int G>
__global__ void __launch_bounds__(128) polar_logits_kernel(const PArgs a) {
  using P = PL<DP, W>;
  __shared__ float qt[G][DP];
  __shared__ float2 cs1[P::L1];
  __shared__ float2 csh[P::LV - 1][P::L2];
  const int tid = threadIdx.x;
  const int kv = blockIdx.y;
  for (int i = tid; i < P::L1; i += blockDim.x) cs1[i] = make_float2(a.tables[P::L1 + 2 * i], a.tables[P::L1 + 2 * i + 1]);
  for (int i = tid; i < (P::LV - 1) * P::L2; i += blockDim.x) {
    const int l = i / P::L2, j = i % P::L2;
    const float* t = a.tables + P::T1 + l * P::TL + 2 * P::L2 - 1;
    csh[l][j] = make_float2(t[2 * j], t[2 * j + 1]);
  }
  // rotated queries q~ = H D q / sqrt(DP) of this KV head's group
  for (int i = tid; i < G * DP; i += blockDim.x) {
    const int g = i / DP, j = i % DP;
    qt[g][j] = (g < a.group && j < a.d) ? a.q[((int64_t)kv * a.group + g) * a.d + j] * (float)a.D[j] : 0.f;
  }
  __syncthreads();
  for (int hs = 1; hs < DP; hs <<= 1) {
    for (int i = tid; i < G * DP / 2; i += blockDim.x) {
      const int g = i / (DP / 2), p = i % (DP / 2);
      const int j = ((p & ~(hs - 1)) << 1) | (p & (hs - 1));
      const float u = qt[g][j], w = qt[g][j + hs];
      qt[g][j] = u + w;
      qt[g][j + hs] = u - w;
    }
    __syncthreads();
  }
  const int64_t key = (int64_t)blockIdx.x * blockDim.x + tid;
  if (key >= a.n_keys) return;
  const int64_t vi = (int64_t)kv * a.n_keys + key;
  uint32_t r[P::NW + 1];
  {
    const uint4* src = reinterpret_cast<const uint4*>(a.ccodes + vi * (P::NW * 4));
#pragma unroll
    for (int i = 0; i < P::NW / 4; ++i) {
      const uint4 u = __ldg(src + i);
      r[4 * i] = u.x;
      r[4 * i + 1] = u.y;
      r[4 * i + 2] = u.z;
      r[4 * i + 3] = u.w;
    }
    r[P::NW] = 0u;
  }
  auto get = [&](int p, int width) {  // p is a compile-time constant after unrolling
    const uint64_t w64 = (uint64_t)r[p >> 5] | ((uint64_t)r[(p >> 5) + 1] << 32);
    return (int)((w64 >> (p & 31)) & ((1u << width) - 1u));
  };
  float acc[G];
#pragma unroll
  for (int g = 0; g < G; ++g) acc[g] = 0.f;
  float st[P::LV + 1];  // radius of the current node of each level, root first
  st[P::LV] = 1.f;
#pragma unroll
  for (int u = 0; u < DP / 4; ++u) {  // level-2 nodes in order
    // refresh the levels whose node changes at u (all indices are constants here)
#pragma unroll
    for (int l = P::LV; l >= 3; --l) {
      if ((u & ((1 << (l - 3)) - 1)) == 0) {  // a new node of level l - 1 starts at u
        const int node = u >> (l - 3);         // node of level l - 1; its parent is node >> 1 of level l
        const int ix = P::B2 > 0 ? get(P::pos(l, node >> 1), P::B2) : 0;
        const float2 c = csh[l - 2][ix];
        st[l - 1] = st[l] * ((node & 1) ? c.y : c.x);
      }
    }
    const int ix2 = P::B2 > 0 ? get(P::pos(2, u), P::B2) : 0;
    const float2 c2 = csh[0][ix2];
    const float ra = st[2] * c2.x, rb = st[2] * c2.y;
    const float2 t0 = cs1[get(P::pos(1, 2 * u), P::B1)];
    const float2 t1 = cs1[get(P::pos(1, 2 * u + 1), P::B1)];
    const float y0 = ra * t0.x, y1 = ra * t0.y, y2 = rb * t1.x, y3 = rb * t1.y;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float4 qq = *reinterpret_cast<const float4*>(&qt[g][4 * u]);
      acc[g] = fmaf(y0, qq.x, fmaf(y1, qq.y, fmaf(y2, qq.z, fmaf(y3, qq.w, acc[g]))));
    }
  }
  const float n = __half2float(__ushort_as_half(__ldg(a.cnorms + vi))) * rsqrtf((float)DP);
#pragma unroll
  for (int g = 0; g < G; ++g)
    if (g < a.group) a.logits[((int64_t)kv * a.group + g) * a.n_keys + key] = acc[g] * n;
}

// ---- QJL stage on the polar residual ---------------------------------------------
// "TurboQuant explainer" (m.163.com), "第二步：QJL" applied to the polar stage 1:
// r = y - y_hat (y the rotated unit vector, y_hat the unit-radius reconstruction
// from the stored tables), gamma = ||r||, sign bits of S r.  A warp per vector:
// the rotation as in the quantize kernel, y_hat as in the dequantize kernel, r
// staged in shared memory, then lane l computes the projections l + 32 j in
// fp64 (exact products of fp16 S and fp32 r) from S stored transposed in shared
// memory, and a ballot per 32 projections packs the sign words.
template <int DP, int W, int DT>
__global__ void __launch_bounds__(256) polar_qjl_kernel(const PArgs a, const uint16_t* S, int m, uint32_t* signs,
                                                        uint16_t* rnorms) {
  using P = PL<DP, W>;
  constexpr int NI = P::NI;
  extern __shared__ __align__(16) uint8_t qsm[];
  __half* St = reinterpret_cast<__half*>(qsm);                      // [DP][m]: St[k][i] = S[i][k]
  float* rw = reinterpret_cast<float*>(qsm + (size_t)DP * m * 2);   // [8][DP] residual of each warp's vector
  float* tab = rw + 8 * DP;                                         // the tables
  uint32_t* rec = reinterpret_cast<uint32_t*>(tab + P::T1 + (P::LV - 1) * P::TL);  // [8][NW + 1]
  for (int e = threadIdx.x; e < m * DP; e += blockDim.x) {
    const int i = e / DP, k = e % DP;
    St[k * m + i] = __ushort_as_half(__ldg(S + e));
  }
  for (int i = threadIdx.x; i < P::T1 + (P::LV - 1) * P::TL; i += blockDim.x) tab[i] = a.tables[i];
  __syncthreads();
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  float dsg[NI];
#pragma unroll
  for (int k = 0; k < NI; ++k) dsg[k] = (float)a.D[NI * lane + k];
  uint32_t* r = rec + wib * (P::NW + 1);
  if (lane == 0) r[P::NW] = 0u;
  float* rv = rw + wib * DP;
  const float rs = rsqrtf((float)DP);
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t v = (int64_t)blockIdx.x * (blockDim.x >> 5) + wib; v < a.n_vec; v += warps) {
    // ---- y: rotation of the unit vector (as polar_quantize_kernel)
    const uint8_t* row = a.x + v * a.ld * (DT == TQ_F32 ? 4 : 2);
    float y[NI];
    float ss = 0.f;
#pragma unroll
    for (int g4 = 0; g4 < NI / 4; ++g4) {
      const int j = NI * lane + 4 * g4;
      float e[4] = {0.f, 0.f, 0.f, 0.f};
      if (j < a.d) {
        if constexpr (DT == TQ_F32) {
          const float4 f = __ldg(reinterpret_cast<const float4*>(row) + (j >> 2));
          e[0] = f.x, e[1] = f.y, e[2] = f.z, e[3] = f.w;
        } else {
          const uint2 u = __ldg(reinterpret_cast<const uint2*>(row) + (j >> 2));
          const uint32_t wd[2] = {u.x, u.y};
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            if constexpr (DT == TQ_BF16) {
              e[2 * h] = __uint_as_float(wd[h] << 16);
              e[2 * h + 1] = __uint_as_float(wd[h] & 0xFFFF0000u);
            } else {
              const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&wd[h]));
              e[2 * h] = f.x, e[2 * h + 1] = f.y;
            }
          }
        }
      }
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        y[4 * g4 + k] = e[k] * dsg[4 * g4 + k];
        ss = fmaf(y[4 * g4 + k], y[4 * g4 + k], ss);
      }
    }
    ss = warp_sum(ss);
    const float n = sqrtf(ss);
#pragma unroll
    for (int hs = 1; hs < NI; hs <<= 1)
#pragma unroll
      for (int k = 0; k < NI; ++k)
        if ((k & hs) == 0) {
          const float u = y[k], w = y[k + hs];
          y[k] = u + w;
          y[k + hs] = u - w;
        }
#pragma unroll
    for (int sft = 1; sft < 32; sft <<= 1)
#pragma unroll
      for (int k = 0; k < NI; ++k) {
        const float o = __shfl_xor_sync(FULL, y[k], sft);
        y[k] = (lane & sft) ? (o - y[k]) : (y[k] + o);
      }
    const float sc = n > 0.f ? rs / n : 0.f;
    // ---- y_hat from the record (as polar_dequantize_kernel, without the inverse rotation)
    if (lane < P::NW) r[lane] = __ldg(reinterpret_cast<const uint32_t*>(a.ccodes + v * (P::NW * 4)) + lane);
    __syncwarp();
    auto get = [&](int p, int width) {
      const uint64_t w64 = (uint64_t)r[p >> 5] | ((uint64_t)r[(p >> 5) + 1] << 32);
      return (int)((w64 >> (p & 31)) & ((1u << width) - 1u));
    };
    auto cs = [&](int l, int ix) {
      const float* t = tab + P::T1 + (l - 2) * P::TL + 2 * P::L2 - 1;
      return make_float2(t[2 * ix], t[2 * ix + 1]);
    };
    float R = 1.f;
#pragma unroll
    for (int l = P::LV; l > P::LI; --l) {
      const int ix = P::B2 > 0 ? get(P::pos(l, lane >> (l - P::LI)), P::B2) : 0;
      const float2 c = cs(l, ix);
      R *= ((lane >> (l - P::LI - 1)) & 1) ? c.y : c.x;
    }
    float rad[NI / 2];
    rad[0] = R;
#pragma unroll
    for (int l = P::LI; l >= 2; --l) {
      const int cnt = NI >> l;
#pragma unroll
      for (int j = cnt - 1; j >= 0; --j) {
        const int ix = P::B2 > 0 ? get(P::pos(l, cnt * lane + j), P::B2) : 0;
        const float2 c = cs(l, ix);
        const float pr = rad[j];
        rad[2 * j] = pr * c.x;
        rad[2 * j + 1] = pr * c.y;
      }
    }
    float g2 = 0.f;
#pragma unroll
    for (int j = 0; j < NI / 2; ++j) {
      const int ix = get(P::pos(1, (NI / 2) * lane + j), P::B1);
      const float r0 = y[2 * j] * sc - rad[j] * tab[P::L1 + 2 * ix];
      const float r1 = y[2 * j + 1] * sc - rad[j] * tab[P::L1 + 2 * ix + 1];
      rv[NI * lane + 2 * j] = r0;
      rv[NI * lane + 2 * j + 1] = r1;
      g2 = fmaf(r0, r0, fmaf(r1, r1, g2));
    }
    g2 = warp_sum(g2);
    __syncwarp();
    // ---- z = S r in fp64, a ballot per 32 projections
    for (int jw = 0; jw < m / 32; ++jw) {
      const int i = 32 * jw + lane;
      double acc = 0.0;
#pragma unroll 8
      for (int k = 0; k < DP; ++k) acc = fma((double)__half2float(St[k * m + i]), (double)rv[k], acc);
      const uint32_t word = __ballot_sync(FULL, acc >= 0.0);
      if (lane == 0) signs[v * (m / 32) + jw] = word;
    }
    if (lane == 0) rnorms[v] = __half_as_ushort(__float2half_rn(sqrtf(g2)));
    __syncwarp();
  }
}

// QJL term of the polar product-code logits, added to the stage-1 logits:
// l += n gamma sqrt(pi/2)/m <S q~, 2 s - 1>.  A CTA of 128 threads takes 128
// keys of one KV head: it rotates the group's queries and projects them
// (u = S q~) into shared memory, then each thread walks its key's sign bits.
template <int DP>
__global__ void __launch_bounds__(128) polar_qjl_logits_kernel(const PArgs a, const uint16_t* S, int m,
                                                               const uint32_t* signs, const uint16_t* rnorms,
                                                               float kappa) {
  __shared__ float qt[8][DP];
  __shared__ float u[8][DP];
  const int kv = blockIdx.y;
  const int tid = threadIdx.x;
  // q~ = H D q / sqrt(DP): butterflies in shared memory
  for (int e = tid; e < a.group * DP; e += blockDim.x) {
    const int g = e / DP, c = e % DP;
    qt[g][c] = c < a.d ? a.q[((int64_t)kv * a.group + g) * a.d + c] * (float)a.D[c] : 0.f;
  }
  __syncthreads();
  for (int hs = 1; hs < DP; hs <<= 1) {
    for (int e = tid; e < a.group * DP / 2; e += blockDim.x) {
      const int g = e / (DP / 2), p = e % (DP / 2);
      const int lo = (p / hs) * 2 * hs + (p % hs), hi = lo + hs;
      const float x0 = qt[g][lo], x1 = qt[g][hi];
      qt[g][lo] = x0 + x1;
      qt[g][hi] = x0 - x1;
    }
    __syncthreads();
  }
  const float rs = rsqrtf((float)DP);
  for (int e = tid; e < a.group * m; e += blockDim.x) {
    const int g = e / m, i = e % m;
    float acc = 0.f;
    const uint16_t* srow = S + (size_t)i * DP;
    for (int k = 0; k < DP; ++k) acc = fmaf(__half2float(__ushort_as_half(__ldg(srow + k))), qt[g][k], acc);
    u[g][i] = acc * rs;
  }
  __syncthreads();
  const int64_t key = (int64_t)blockIdx.x * blockDim.x + tid;
  if (key >= a.n_keys) return;
  const int64_t vi = (int64_t)kv * a.n_keys + key;
  const float n = __half2float(__ushort_as_half(__ldg(a.cnorms + vi)));
  const float gm = __half2float(__ushort_as_half(__ldg(rnorms + vi)));
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  for (int w = 0; w < m / 32; ++w) {
    const uint32_t word = __ldg(signs + vi * (m / 32) + w);
    for (int b = 0; b < 32; ++b) {
      const bool pos = (word >> b) & 1u;
      for (int g = 0; g < a.group; ++g) acc[g] += pos ? u[g][32 * w + b] : -u[g][32 * w + b];
    }
  }
  for (int g = 0; g < a.group; ++g) a.logits[((int64_t)kv * a.group + g) * a.n_keys + key] += n * gm * kappa * acc[g];
}

int launch_err(const char* who) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return tq::set_error(TQ_ECUDA, "%s: launch failed: %s", who, cudaGetErrorString(e));
  return TQ_OK;
}

int check_polar(const tq_polar_params* p, const char* who) {
  if (!p) return tq::set_error(TQ_EINVAL, "%s: NULL params", who);
  if (p->d_pad != 128 && p->d_pad != 256) return tq::set_error(TQ_EUNSUPPORTED, "%s: d_pad must be 128 or 256", who);
  if (p->d < 1 || p->d > p->d_pad) return tq::set_error(TQ_EINVAL, "%s: d out of range", who);
  if (p->w < 1 || p->w > 3) return tq::set_error(TQ_EINVAL, "%s: w must be 1..3", who);
  if (!p->tables || !p->signs_D) return tq::set_error(TQ_EINVAL, "%s: NULL tables or signs", who);
  return TQ_OK;
}

int grid_for(int64_t n_vec) {
  return (int)std::max<int64_t>(1, std::min<int64_t>((n_vec + 7) / 8, (int64_t)tq::sm_count() * 16));
}

template <int DP, int W>
int quantize_dw(int dtype, const PArgs& a, cudaStream_t st) {
  const int g = grid_for(a.n_vec);
  if (dtype == TQ_F32)
    polar_quantize_kernel<DP, W, TQ_F32><<<g, 256, 0, st>>>(a);
  else if (dtype == TQ_F16)
    polar_quantize_kernel<DP, W, TQ_F16><<<g, 256, 0, st>>>(a);
  else
    polar_quantize_kernel<DP, W, TQ_BF16><<<g, 256, 0, st>>>(a);
  return launch_err("tq_polar_quantize");
}

template <int DP, int W>
int dequantize_dw(const PArgs& a, cudaStream_t st) {
  polar_dequantize_kernel<DP, W><<<grid_for(a.n_vec), 256, 0, st>>>(a);
  return launch_err("tq_polar_dequantize");
}

template <int DP, int W>
int logits_dw(const PArgs& a, int n_kv, cudaStream_t st) {
  const dim3 grid((unsigned)((a.n_keys + 127) / 128), (unsigned)n_kv);
  if (a.group <= 1)
    polar_logits_kernel<DP, W, 1><<<grid, 128, 0, st>>>(a);
  else if (a.group <= 2)
    polar_logits_kernel<DP, W, 2><<<grid, 128, 0, st>>>(a);
  else if (a.group <= 4)
    polar_logits_kernel<DP, W, 4><<<grid, 128, 0, st>>>(a);
  else
    polar_logits_kernel<DP, W, 8><<<grid, 128, 0, st>>>(a);
  return launch_err("tq_polar_logits");
}

template <int DP, int W>
int qjl_dw(int dtype, const PArgs& a, const uint16_t* S, int m, uint32_t* signs, uint16_t* rnorms, cudaStream_t st) {
  using P = PL<DP, W>;
  const size_t smem = (size_t)DP * m * 2 + 8 * DP * 4 + (P::T1 + (P::LV - 1) * P::TL) * 4 + 8 * (P::NW + 1) * 4;
  void (*kern)(const PArgs, const uint16_t*, int, uint32_t*, uint16_t*) =
      dtype == TQ_F32 ? polar_qjl_kernel<DP, W, TQ_F32>
                      : (dtype == TQ_F16 ? polar_qjl_kernel<DP, W, TQ_F16> : polar_qjl_kernel<DP, W, TQ_BF16>);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return tq::set_error(TQ_ECUDA, "tq_polar_qjl: %s", cudaGetErrorString(e));
  kern<<<grid_for(a.n_vec), 256, smem, st>>>(a, S, m, signs, rnorms);
  return launch_err("tq_polar_qjl");
}

#define TQ_POLAR_DISPATCH(dp, w, CALL) \
  ((dp) == 128 ? ((w) == 1 ? CALL(128, 1) : (w) == 2 ? CALL(128, 2) : CALL(128, 3)) \
               : ((w) == 1 ? CALL(256, 1) : (w) == 2 ? CALL(256, 2) : CALL(256, 3)))

}  // namespace

extern "C" int tq_polar_quantize(const tq_polar_params* p, const void* x, int dtype, int64_t n_vec, int64_t ld,
                                 void* codes, uint16_t* norms, tq_stream_t stream) {
  using namespace tq;
  int rc = check_polar(p, "tq_polar_quantize");
  if (rc) return rc;
  if (n_vec < 0) return set_error(TQ_EINVAL, "tq_polar_quantize: n_vec < 0");
  if (n_vec == 0) {
    clear_error();
    return TQ_OK;
  }
  if (dtype != TQ_F32 && dtype != TQ_F16 && dtype != TQ_BF16) return set_error(TQ_EINVAL, "tq_polar_quantize: dtype");
  if (!x || !codes || !norms) return set_error(TQ_EINVAL, "tq_polar_quantize: NULL pointer argument");
  if (ld < p->d) return set_error(TQ_EINVAL, "tq_polar_quantize: ld < d");
  const int es = dtype == TQ_F32 ? 4 : 2;
  if (!aligned(x, 16) || ((ld * es) % 16) != 0 || ((int64_t)p->d * es) % 16 != 0 || !aligned(codes, 16) ||
      !aligned(norms, 2))
    return set_error(TQ_EINVAL, "tq_polar_quantize: x, ld*elem, d*elem and codes must be 16-byte aligned");
  PArgs a{};
  a.x = static_cast<const uint8_t*>(x);
  a.n_vec = n_vec;
  a.ld = ld;
  a.d = p->d;
  a.tables = p->tables;
  a.D = p->signs_D;
  a.codes = static_cast<uint8_t*>(codes);
  a.norms = norms;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
#define Q_CALL(DP, W) quantize_dw<DP, W>(dtype, a, st)
  rc = TQ_POLAR_DISPATCH(p->d_pad, p->w, Q_CALL);
#undef Q_CALL
  if (rc == TQ_OK) clear_error();
  return rc;
}

extern "C" int tq_polar_dequantize(const tq_polar_params* p, const void* codes, const uint16_t* norms, int64_t n_vec,
                                   float* out, int64_t ld, tq_stream_t stream) {
  using namespace tq;
  int rc = check_polar(p, "tq_polar_dequantize");
  if (rc) return rc;
  if (n_vec < 0) return set_error(TQ_EINVAL, "tq_polar_dequantize: n_vec < 0");
  if (n_vec == 0) {
    clear_error();
    return TQ_OK;
  }
  if (!codes || !norms || !out) return set_error(TQ_EINVAL, "tq_polar_dequantize: NULL pointer argument");
  if (ld < p->d) return set_error(TQ_EINVAL, "tq_polar_dequantize: ld < d");
  if (!aligned(codes, 16) || !aligned(out, 4)) return set_error(TQ_EINVAL, "tq_polar_dequantize: misaligned pointer");
  PArgs a{};
  a.n_vec = n_vec;
  a.ld = ld;
  a.d = p->d;
  a.tables = p->tables;
  a.D = p->signs_D;
  a.ccodes = static_cast<const uint8_t*>(codes);
  a.cnorms = norms;
  a.out = out;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
#define D_CALL(DP, W) dequantize_dw<DP, W>(a, st)
  rc = TQ_POLAR_DISPATCH(p->d_pad, p->w, D_CALL);
#undef D_CALL
  if (rc == TQ_OK) clear_error();
  return rc;
}

extern "C" int tq_polar_logits(const tq_polar_params* p, const float* q, int group, const void* codes,
                               const uint16_t* norms, int64_t n_keys, int n_kv_heads, float* logits,
                               tq_stream_t stream) {
  using namespace tq;
  int rc = check_polar(p, "tq_polar_logits");
  if (rc) return rc;
  if (group < 1 || group > 8) return set_error(TQ_EINVAL, "tq_polar_logits: group must be 1..8");
  if (n_keys < 0 || n_kv_heads < 0) return set_error(TQ_EINVAL, "tq_polar_logits: negative size");
  if (n_keys == 0 || n_kv_heads == 0) {
    clear_error();
    return TQ_OK;
  }
  if (n_kv_heads > 65535) return set_error(TQ_EUNSUPPORTED, "tq_polar_logits: more than 65535 KV heads");
  if (!q || !codes || !norms || !logits) return set_error(TQ_EINVAL, "tq_polar_logits: NULL pointer argument");
  if (!aligned(codes, 16) || !aligned(q, 4) || !aligned(logits, 4))
    return set_error(TQ_EINVAL, "tq_polar_logits: misaligned pointer");
  PArgs a{};
  a.d = p->d;
  a.tables = p->tables;
  a.D = p->signs_D;
  a.ccodes = static_cast<const uint8_t*>(codes);
  a.cnorms = norms;
  a.q = q;
  a.logits = logits;
  a.n_keys = n_keys;
  a.group = group;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
#define L_CALL(DP, W) logits_dw<DP, W>(a, n_kv_heads, st)
  rc = TQ_POLAR_DISPATCH(p->d_pad, p->w, L_CALL);
#undef L_CALL
  if (rc == TQ_OK) clear_error();
  return rc;
}

extern "C" int tq_polar_qjl(const tq_polar_params* p, const uint16_t* S, int m, const void* x, int dtype,
                            int64_t n_vec, int64_t ld, const void* codes, void* signs, uint16_t* rnorms,
                            tq_stream_t stream) {
  using namespace tq;
  int rc = check_polar(p, "tq_polar_qjl");
  if (rc) return rc;
  if (m < 32 || m > p->d_pad || m % 32 != 0)
    return set_error(TQ_EINVAL, "tq_polar_qjl: m must be a multiple of 32 in [32, d_pad]");
  if (n_vec < 0) return set_error(TQ_EINVAL, "tq_polar_qjl: n_vec < 0");
  if (n_vec == 0) {
    clear_error();
    return TQ_OK;
  }
  if (dtype != TQ_F32 && dtype != TQ_F16 && dtype != TQ_BF16) return set_error(TQ_EINVAL, "tq_polar_qjl: dtype");
  if (!S || !x || !codes || !signs || !rnorms) return set_error(TQ_EINVAL, "tq_polar_qjl: NULL pointer argument");
  if (ld < p->d) return set_error(TQ_EINVAL, "tq_polar_qjl: ld < d");
  const int es = dtype == TQ_F32 ? 4 : 2;
  if (!aligned(x, 16) || ((ld * es) % 16) != 0 || ((int64_t)p->d * es) % 16 != 0 || !aligned(codes, 16) ||
      !aligned(signs, 4) || !aligned(rnorms, 2))
    return set_error(TQ_EINVAL, "tq_polar_qjl: x, ld*elem, d*elem and codes must be 16-byte aligned, signs 4-byte");
  PArgs a{};
  a.x = static_cast<const uint8_t*>(x);
  a.n_vec = n_vec;
  a.ld = ld;
  a.d = p->d;
  a.tables = p->tables;
  a.D = p->signs_D;
  a.ccodes = static_cast<const uint8_t*>(codes);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint32_t* sg = static_cast<uint32_t*>(signs);
#define J_CALL(DP, W) qjl_dw<DP, W>(dtype, a, S, m, sg, rnorms, st)
  rc = TQ_POLAR_DISPATCH(p->d_pad, p->w, J_CALL);
#undef J_CALL
  if (rc == TQ_OK) clear_error();
  return rc;
}

extern "C" int tq_polar_logits_prod(const tq_polar_params* p, const uint16_t* S, int m, const float* q, int group,
                                    const void* codes, const uint16_t* norms, const void* signs,
                                    const uint16_t* rnorms, int64_t n_keys, int n_kv_heads, float* logits,
                                    tq_stream_t stream) {
  using namespace tq;
  if (!p) return set_error(TQ_EINVAL, "tq_polar_logits_prod: NULL params");
  if (m < 32 || m > p->d_pad || m % 32 != 0)
    return set_error(TQ_EINVAL, "tq_polar_logits_prod: m must be a multiple of 32 in [32, d_pad]");
  if (!S || !signs || !rnorms) return set_error(TQ_EINVAL, "tq_polar_logits_prod: NULL pointer argument");
  if (!aligned(signs, 4)) return set_error(TQ_EINVAL, "tq_polar_logits_prod: signs must be 4-byte aligned");
  int rc = tq_polar_logits(p, q, group, codes, norms, n_keys, n_kv_heads, logits, stream);
  if (rc) return rc;
  if (n_keys == 0 || n_kv_heads == 0) return TQ_OK;
  PArgs a{};
  a.d = p->d;
  a.D = p->signs_D;
  a.cnorms = norms;
  a.q = q;
  a.logits = logits;
  a.n_keys = n_keys;
  a.group = group;
  const float kappa = (float)(std::sqrt(M_PI / 2.0) / m);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const dim3 grid((unsigned)((n_keys + 127) / 128), (unsigned)n_kv_heads);
  if (p->d_pad == 128)
    polar_qjl_logits_kernel<128><<<grid, 128, 0, st>>>(a, S, m, static_cast<const uint32_t*>(signs), rnorms, kappa);
  else
    polar_qjl_logits_kernel<256><<<grid, 128, 0, st>>>(a, S, m, static_cast<const uint32_t*>(signs), rnorms, kappa);
  rc = launch_err("tq_polar_logits_prod");
  if (rc == TQ_OK) clear_error();
  return rc;
}
