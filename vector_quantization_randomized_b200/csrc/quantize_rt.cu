// tq_quantize for d_pad = 128 with 16-bit input: the rotation and the QJL
// projection both on the fifth-generation tensor cores.
//
// Method ("TurboQuant explainer" (m.163.com), "第一步：PolarQuant" and
// "第二步：QJL"): norm, random sign flips + Walsh-Hadamard rotation, Lloyd-Max
// code at b-1 bits (b bits in MSE mode), residual and its norm, sign bits of S r.
//
// Design (B200, sm_100a), one persistent CTA per SM over tiles of 128 vectors:
//  * warp 0 loads each tile with TMA: 16 boxes of 8 elements x 128 rows, which
//    land as the K-major canonical layout of an MMA operand (K chunk k8 of
//    every row in one 2 KB slab); rows past the end and columns past d read 0.
//  * warp 1 issues, per tile, the rotation y = X (H D)^T (M = 128 vectors,
//    N = 128 coordinates, K = 128; the +-1 entries of H D are exact in 16 bits,
//    fp32 accumulation) into one of two tensor-memory buffers, and, once the
//    residual of the tile is written, the projection z = R S^T on its fp16 hi
//    and lo parts (S r to about 2^-22 before fp32 accumulation).  Warp-uniform
//    loops, elect-issued MMAs.
//  * warps 2-9 encode: two threads per vector (the two warps of a lane
//    quadrant take coordinates 0-63 and 64-127), y read back with tcgen05.ld;
//    the squared norms of the two halves meet in shared memory; the code and the
//    residual as in the two-thread kernel (quantize_tc.cu), with the thresholds
//    scaled per vector so that no value needs the 1/(sqrt(128) n) multiply; the
//    residual (x 2^14) goes to the hi / lo operand tiles.
//  * warps 10-13 (product mode) read z back (a thread per vector, all
//    projections), pack the sign words, and recompute in fp32 from the hi + lo
//    parts the projections within the fp32 accumulation bound of zero.  They run
//    one tile behind the encode warps, which wait for them only before writing
//    the next residual.
// Every hand-off is an mbarrier with an iteration limit.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "common.h"
#include "device.cuh"
#include "prep.h"
#include "tc.cuh"
#include "tmap.h"

namespace {

using namespace tqd;

constexpr int TV = 128;       // vectors per tile (M of the MMAs)
constexpr int DP = 128;
constexpr int SLAB = 2048;    // one K chunk (8 elements) of 128 rows
constexpr int TILE_B = 16 * SLAB;  // a 128 x 128 16-bit operand tile

struct RArgs {
  int64_t n_vec, n_pad;
  int d, m;
  uint8_t* codes;
  uint16_t* norms;
  uint16_t* rnorms;
  const float* cent;
  const float* thr;
  const int8_t* D;
  const uint16_t* S;
  int tbytes;  // bytes of one 32-vector code tile
};

// byte offset of element (row, k) of a canonical K-major 128 x 128 16-bit tile
__device__ __forceinline__ int cofs(int row, int k) { return (k >> 3) * SLAB + (row >> 3) * 128 + (row & 7) * 16 + (k & 7) * 2; }

template <bool PROD>
struct RL {
  static constexpr int NX = PROD ? 2 : 4;  // input stages
  static constexpr int HD = 0;                                  // H D, canonical (N = out coordinate, K = in)
  static constexpr int SS = HD + TILE_B;                        // S, canonical (N = projection, K = coordinate)
  static constexpr int XS = SS + (PROD ? TILE_B : 0);           // [NX] input tiles
  static constexpr int RH = XS + NX * TILE_B;                   // residual hi / lo (A of the projection)
  static constexpr int RLO = RH + (PROD ? TILE_B : 0);
  static constexpr int NSQ = RLO + (PROD ? TILE_B : 0);         // [2 tile parities][2 halves][128] squared norms
  static constexpr int GSQ = NSQ + 4 * TV * 4;                  // [2 halves][128] squared residual norms
  static constexpr int BND = GSQ + 2 * TV * 4;                  // [2][128] fix-up bound per vector (per tile parity)
  static constexpr int BAR = BND + 2 * TV * 4;
  static constexpr int TOTAL = BAR + 256;
  static constexpr int W_MMA = 1, W_ENC0 = 2, W_RB0 = 10;
  static constexpr int NTHREADS = (PROD ? 14 : 10) * 32;
};

__device__ __forceinline__ float mul_sat(float a, float b) {
  float r;
  asm("mul.rn.sat.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
  return r;
}

// 2-D tiled TMA load: box at (x, y) of the tensor map into shared memory, completing on `bar`.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];\n" ::
          "r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// kind::f16 instruction descriptor with A, B 16-bit floats (bf16 when BF is set), fp32 D, K-major.
__host__ __device__ constexpr uint32_t idesc_16(int M, int N, bool bf) {
  return (1u << 4) | ((bf ? 1u : 0u) << 7) | ((bf ? 1u : 0u) << 10) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void umma_16_ss_elect(uint32_t d, uint64_t ad, uint64_t bd, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p, e;\n setp.ne.b32 p, %4, 0;\n elect.sync _|e, 0xffffffff;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d),
      "l"(ad), "l"(bd), "r"(idesc), "r"(acc));
}

// Scalar code of one coordinate against thresholds scaled to the unnormalised
// rotated value (tps = t * sqrt(128) n): the predicates [|y| > t_k] and [y <= 0]
// are shifted into 32-bit words (sign bits of tps_k - |y| and of y - 2^-149),
// the centroid magnitude (x 2^14, scaled like the thresholds' inverse) is picked
// with saturated multiplies; returns the residual x 2^14.
template <int KB>
struct CoderR {
  static constexpr int L = 1 << KB;
  static constexpr int NPT = L / 2 - 1;
  static constexpr int NP1 = NPT > 0 ? NPT : 1;
  float tps[NP1];
  float dmag[NP1];  // (c[L/2 + k + 1] - c[L/2 + k]) * 2^14
  float mag0;       // c[L/2] * 2^14
  template <bool RES>
  __device__ __forceinline__ float code(float y, float ysc, uint32_t& wn, uint32_t (&wp)[NP1]) const {
    const float a = fabsf(y);
    float mg = mag0;
#pragma unroll
    for (int k = 0; k < NPT; ++k) {
      const float e = tps[k] - a;
      wp[k] = __funnelshift_l(__float_as_uint(e), wp[k], 1);
      if constexpr (RES) mg = fmaf(mul_sat(e, -0x1p126f), dmag[k], mg);
    }
    const float ys = y - 0x1p-149f;
    wn = __funnelshift_l(__float_as_uint(ys), wn, 1);
    if constexpr (RES) return fmaf(y, ysc, -copysignf(mg, ys));  // 2^14 (y / (sqrt(128) n) - c[idx])
    return 0.f;
  }
  __device__ __forceinline__ void planes(uint32_t ws, const uint32_t (&wp)[NP1], uint32_t (&pl)[KB]) const {
#pragma unroll
    for (int b = 0; b < KB - 1; ++b) {
      uint32_t x = 0;
#pragma unroll
      for (int k = 0; k < NPT; ++k)
        if ((((k + 1) >> b) & 1) != ((k >> b) & 1)) x ^= wp[k];
      pl[b] = x ^ ~ws;
    }
    pl[KB - 1] = ws;
  }
};

template <int KB, bool PROD, bool BF>
__global__ void __launch_bounds__(RL<PROD>::NTHREADS, 1) quantize_rt_kernel(const __grid_constant__ CUtensorMap tmap,
                                                                            const RArgs a) {
  using L = RL<PROD>;
  constexpr int NX = L::NX;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* hd = smem + L::HD;
  uint8_t* Ss = smem + L::SS;
  uint8_t* rh = smem + L::RH;
  uint8_t* rlo = smem + L::RLO;
  float* nsq = reinterpret_cast<float*>(smem + L::NSQ);
  float* gsq = reinterpret_cast<float*>(smem + L::GSQ);
  float* bnd = reinterpret_cast<float*>(smem + L::BND);
  uint64_t* xfull = reinterpret_cast<uint64_t*>(smem + L::BAR);  // [4] input tile landed (1 + tx)
  uint64_t* xfree = xfull + 4;                                     // [4] rotation MMAs read it (1)
  uint64_t* yfull = xfree + 4;                                     // [2] rotation done (1)
  uint64_t* yfree = yfull + 2;                                     // [2] y read by the encode warps (8)
  uint64_t* rfull = yfree + 2;                                     // residual tiles written (8)
  uint64_t* rfree = rfull + 1;                                     // residual tiles no longer needed (4)
  uint64_t* zfull = rfree + 1;                                     // [2] projection done (1)
  uint64_t* zfree = zfull + 2;                                     // [2] z read back (4)
  uint64_t* gbar = zfree + 2;                                      // encode warps' barrier (8)
  uint32_t* tbase = reinterpret_cast<uint32_t*>(gbar + 1);
  float* smax = reinterpret_cast<float*>(tbase + 1);
  float* wmax = smax + 1;  // [14]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t n_tiles = (a.n_pad + TV - 1) / TV;

  // ---- per-CTA constants: H D (and S) in the canonical layout ----
  for (int e = threadIdx.x; e < DP * DP / 2; e += blockDim.x) {  // two elements of a row per thread
    const int n = e / (DP / 2), k = 2 * (e % (DP / 2));
    uint32_t w = 0;
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const int kk = k + t;
      const float v = ((__popc(n & kk) & 1) ? -1.f : 1.f) * (float)__ldg(a.D + kk);
      const uint16_t bits = BF ? __bfloat16_as_ushort(__float2bfloat16(v)) : __half_as_ushort(__float2half(v));
      w |= (uint32_t)bits << (16 * t);
    }
    *reinterpret_cast<uint32_t*>(hd + cofs(n, k)) = w;
  }
  if constexpr (PROD) {
    for (int e = threadIdx.x; e < a.m * (DP / 8); e += blockDim.x) {
      const int row = e / (DP / 8), kc = e % (DP / 8);
      *reinterpret_cast<uint4*>(Ss + cofs(row, 8 * kc)) = __ldg(reinterpret_cast<const uint4*>(a.S + (size_t)row * DP) + kc);
    }
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < 4; ++s) {
      mbar_init(&xfull[s], 1);
      mbar_init(&xfree[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&yfull[b], 1);
      mbar_init(&yfree[b], 8);
      mbar_init(&zfull[b], 1);
      mbar_init(&zfree[b], 4);
    }
    mbar_init(rfull, 8);
    mbar_init(rfree, 4);
    mbar_init(gbar, 8);
  }
  if (warp == 0) tmem_alloc(tbase, 512);
  // max_i ||S_i|| (inflated slightly so the bound stays a bound): 2 threads per row
  if constexpr (PROD) {
    float s = 0.f;
    if (threadIdx.x < 2 * a.m) {
      const int row = threadIdx.x >> 1, k0 = (threadIdx.x & 1) * (DP / 2);
      const uint4* srow = reinterpret_cast<const uint4*>(a.S + (size_t)row * DP + k0);
#pragma unroll 2
      for (int kc = 0; kc < DP / 16; ++kc) {
        const uint4 v = __ldg(srow + kc);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int hh = 0; hh < 4; ++hh) {
          const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[hh]));
          s = fmaf(f.x, f.x, fmaf(f.y, f.y, s));
        }
      }
    }
    s += __shfl_xor_sync(FULL, s, 1);
    const float wm = warp_max(s);
    if (lane == 0) wmax[warp] = wm;
  }
  fence_async_smem();  // H D and S are read by the tensor core
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if constexpr (PROD) {
    if (threadIdx.x == 0) {
      float mx = 0.f;
      for (int w = 0; w < L::NTHREADS / 32; ++w) mx = fmaxf(mx, wmax[w]);
      *smax = sqrtf(mx) * 1.0001f;
    }
    __syncthreads();
  }
  const uint32_t tmem = *tbase;
  auto ycol = [&](int b) { return tmem + (uint32_t)(128 * b); };
  auto zcol = [&](int b) { return tmem + 256u + (uint32_t)(128 * b); };
  const int64_t t0 = blockIdx.x, ts = gridDim.x;
  const int nt = t0 < n_tiles ? (int)((n_tiles - 1 - t0) / ts) + 1 : 0;  // tiles of this CTA

  if (warp == 0) {
    // ---------------- producer: input tiles by TMA ----------------
    if (lane == 0) {
      int issued = 0;
      for (int i = 0; i < nt; ++i) {
        const int s = i % NX;
        if (i >= NX && !mbar_wait(&xfree[s], ((i - NX) / NX) & 1)) break;
        uint8_t* dst = smem + L::XS + s * TILE_B;
        mbar_expect_tx(&xfull[s], TILE_B);
        const int y = (int)((t0 + (int64_t)i * ts) * TV);
#pragma unroll 1
        for (int kc = 0; kc < DP / 8; ++kc) tma_load_2d(dst + kc * SLAB, &tmap, 8 * kc, y, &xfull[s]);
        issued = i + 1;
      }
      for (int i = (issued > NX ? issued - NX : 0); i < issued; ++i) mbar_wait(&xfull[i % NX], (i / NX) & 1);
    }
    __syncwarp();
  } else if (warp == L::W_MMA) {
    // ---------------- MMA issue: rotation, then the projection one tile behind ----------------
    constexpr uint32_t id1 = idesc_16(TV, DP, BF);
    const uint32_t id2 = idesc_16(TV, a.m > 0 ? a.m : 128, false);
    const uint32_t shd = smem_u32(hd);
    auto projection = [&](int j) {  // z = R S^T of tile j (R: hi then lo)
      if (!mbar_wait(rfull, j & 1)) return false;
      if (j >= 2 && !mbar_wait(&zfree[j & 1], ((j - 2) >> 1) & 1)) return false;
      __syncwarp();
      tc_fence_after();
      const uint32_t d = zcol(j & 1);
#pragma unroll
      for (int part = 0; part < 2; ++part) {
        const uint64_t ad = smem_desc(smem_u32(part ? rlo : rh), SLAB, 128);
        const uint64_t bd = smem_desc(smem_u32(Ss), SLAB, 128);
#pragma unroll
        for (int ks = 0; ks < DP / 16; ++ks)
          umma_16_ss_elect(d, ad + (uint64_t)(ks * (2 * SLAB >> 4)), bd + (uint64_t)(ks * (2 * SLAB >> 4)), id2,
                           (part | ks) ? 1u : 0u);
      }
      umma_commit_elect(&zfull[j & 1]);
      return true;
    };
    bool ok = true;
    for (int i = 0; i < nt && ok; ++i) {
      const int s = i % NX, b = i & 1;
      if (!mbar_wait(&xfull[s], (i / NX) & 1)) break;
      if (i >= 2 && !mbar_wait(&yfree[b], ((i - 2) >> 1) & 1)) break;
      __syncwarp();
      tc_fence_after();
      const uint64_t ad = smem_desc(smem_u32(smem + L::XS + s * TILE_B), SLAB, 128);
      const uint64_t bd = smem_desc(shd, SLAB, 128);
#pragma unroll
      for (int ks = 0; ks < DP / 16; ++ks)
        umma_16_ss_elect(ycol(b), ad + (uint64_t)(ks * (2 * SLAB >> 4)), bd + (uint64_t)(ks * (2 * SLAB >> 4)), id1,
                         ks ? 1u : 0u);
      umma_commit_elect(&yfull[b]);
      umma_commit_elect(&xfree[s]);
      if constexpr (PROD)
        if (i >= 1) ok = projection(i - 1);
    }
    if constexpr (PROD)
      if (ok && nt >= 1) projection(nt - 1);
    __syncwarp();
  } else if (warp < L::W_RB0) {
    // ---------------- encode: two threads per vector ----------------
    const int ew = warp - L::W_ENC0;
    const int qd = warp & 3, h = ew >> 2;  // lane quadrant; coordinate half
    const int v = 32 * qd + lane;          // vector within the tile
    CoderR<KB> cd;
    float tpr[CoderR<KB>::NP1];
#pragma unroll
    for (int k = 0; k < CoderR<KB>::NPT; ++k) {
      tpr[k] = __ldg(a.thr + CoderR<KB>::L / 2 + k);
      cd.dmag[k] = (__ldg(a.cent + CoderR<KB>::L / 2 + k + 1) - __ldg(a.cent + CoderR<KB>::L / 2 + k)) * 16384.f;
    }
    cd.mag0 = __ldg(a.cent + CoderR<KB>::L / 2) * 16384.f;
    const float smx = PROD ? *smax : 0.f;
    GroupSync gs{gbar, 0u};
    for (int i = 0; i < nt; ++i) {
      const int b = i & 1;
      const int64_t tile = t0 + (int64_t)i * ts;
      const int64_t vg = tile * TV + v;
      if (!mbar_wait(&yfull[b], (i >> 1) & 1)) break;
      tc_fence_after();
      uint32_t yr[64];
      {
        uint32_t (&y0)[32] = *reinterpret_cast<uint32_t(*)[32]>(yr);
        uint32_t (&y1)[32] = *reinterpret_cast<uint32_t(*)[32]>(yr + 32);
        const uint32_t ta = ycol(b) + ((uint32_t)(32 * qd) << 16) + 64 * h;
        tmem_ld32_issue(ta, y0);
        tmem_ld32_issue(ta + 32, y1);
        tmem_ld_wait(y0);
        tmem_ld_wait(y1);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&yfree[b]);
      float ss = 0.f;
#pragma unroll
      for (int k = 0; k < 64; ++k) ss = fmaf(__uint_as_float(yr[k]), __uint_as_float(yr[k]), ss);
      // the partner half may still read the previous tile's sums: those sit in the other parity
      float* nsb = nsq + b * 2 * TV;
      nsb[h * TV + v] = ss;
      gs.sync(lane);
      const float tot = nsb[v] + nsb[TV + v];  // = 128 ||x||^2
      const float n = sqrtf(tot * 0.0078125f);
      const float s128n = sqrtf(tot);          // sqrt(128) n
      const float ysc = tot > 0.f ? 16384.f / s128n : 0.f;  // 2^14 / (sqrt(128) n)
#pragma unroll
      for (int k = 0; k < CoderR<KB>::NPT; ++k) cd.tps[k] = tpr[k] * s128n;
      if (PROD && i >= 1 && !mbar_wait(rfree, (i - 1) & 1)) break;  // the previous residual has been read back
      uint32_t pl[KB][2];
      float g2 = 0.f;
#pragma unroll
      for (int w = 0; w < 2; ++w) {  // 32 coordinates per code word, highest bit first
        uint32_t wn = 0, wp[CoderR<KB>::NP1];
#pragma unroll
        for (int k = 0; k < CoderR<KB>::NP1; ++k) wp[k] = 0;
#pragma unroll
        for (int kk = 3; kk >= 0; --kk) {  // 8-coordinate chunks, descending
          uint32_t hq[4], lq[4];
#pragma unroll
          for (int j = 7; j >= 0; j -= 2) {
            const float y1 = __uint_as_float(yr[32 * w + 8 * kk + j]);
            const float y0 = __uint_as_float(yr[32 * w + 8 * kk + j - 1]);
            const float r1 = cd.template code<PROD>(y1, ysc, wn, wp);
            const float r0 = cd.template code<PROD>(y0, ysc, wn, wp);
            if constexpr (PROD) {
              g2 = fmaf(r0, r0, fmaf(r1, r1, g2));
              const __half2 hv = __floats2half2_rn(r0, r1);
              const float2 hf = __half22float2(hv);
              const __half2 lv = __floats2half2_rn(r0 - hf.x, r1 - hf.y);  // exact differences
              hq[j >> 1] = *reinterpret_cast<const uint32_t*>(&hv);
              lq[j >> 1] = *reinterpret_cast<const uint32_t*>(&lv);
            }
          }
          if constexpr (PROD) {
            const int col = 64 * h + 32 * w + 8 * kk;
            *reinterpret_cast<uint4*>(rh + cofs(v, col)) = make_uint4(hq[0], hq[1], hq[2], hq[3]);
            *reinterpret_cast<uint4*>(rlo + cofs(v, col)) = make_uint4(lq[0], lq[1], lq[2], lq[3]);
          }
        }
        uint32_t p[KB];
        cd.planes(~wn, wp, p);
#pragma unroll
        for (int bb = 0; bb < KB; ++bb) pl[bb][w] = p[bb];
      }
      if constexpr (PROD) {
        gsq[h * TV + v] = g2;
        gs.sync(lane);
        const float g2t = gsq[v] + gsq[TV + v];  // (2^14 gamma)^2
        // |z - S_i.r'| <= max||S_i|| (2^-21 + 2^-15) gamma' covers the lo-part rounding and the
        // fp32 accumulation of 256 exact products (gamma' = 2^14 gamma)
        if (h == 0) bnd[b * TV + v] = smx * sqrtf(g2t) * 3.1471252e-05f;
        fence_async_smem();  // the residual tiles are read by the tensor core
        __syncwarp();
        if (lane == 0) mbar_arrive(rfull);  // releases the residual and the bounds to the read-back warps
        if (h == 0 && vg < a.n_vec) a.rnorms[vg] = __half_as_ushort(__float2half_rn(sqrtf(g2t) * (1.f / 16384.f)));
      }
      if (vg < a.n_pad) {
        uint8_t* tb = a.codes + (vg >> 5) * a.tbytes + (int)(vg & 31) * (DP / 8) + 8 * h;
        const bool valid = vg < a.n_vec;
#pragma unroll
        for (int bb = 0; bb < KB; ++bb)
          *reinterpret_cast<uint2*>(tb + bb * TILE * (DP / 8)) = valid ? make_uint2(pl[bb][0], pl[bb][1]) : make_uint2(0, 0);
      }
      if (h == 0 && vg < a.n_vec) a.norms[vg] = __half_as_ushort(__float2half_rn(n));
    }
  } else {
    // ---------------- read-back of z: sign words and fix-ups (product mode) ----------------
    const int qd = warp & 3;
    const int v = 32 * qd + lane;
    for (int i = 0; i < nt; ++i) {
      const int b = i & 1;
      const int64_t tile = t0 + (int64_t)i * ts;
      const int64_t vg = tile * TV + v;
      // rfull of this tile completed before its projection was issued; waiting on it here as
      // well orders the encode warps' shared-memory writes (bounds, residual) before the reads below
      if (!mbar_wait(rfull, i & 1)) break;
      if (!mbar_wait(&zfull[b], (i >> 1) & 1)) break;
      tc_fence_after();
      const float bound = bnd[b * TV + v];
      const float bnd2 = fmaxf(bound, 0x1p-126f);
      uint32_t sgn[4], need[4];
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t zr[2][32];
        const uint32_t ta = zcol(b) + ((uint32_t)(32 * qd) << 16) + 64 * half;
        tmem_ld32_issue(ta, zr[0]);
        tmem_ld32_issue(ta + 32, zr[1]);
        tmem_ld_wait(zr[0]);
        tmem_ld_wait(zr[1]);
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          uint32_t word = 0, any = 0;
#pragma unroll
          for (int j = 31; j >= 0; --j) {
            word = __funnelshift_l(zr[u][j], word, 1);
            any |= __float_as_uint(fabsf(__uint_as_float(zr[u][j])) - bnd2);
          }
          const int wi = 2 * half + u;
          sgn[wi] = ~word;
          uint32_t nd = 0;
          if ((int)any < 0 && vg < a.n_vec && 32 * wi < a.m) {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (fabsf(__uint_as_float(zr[u][j])) <= bound) nd |= 1u << j;
          }
          need[wi] = nd;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&zfree[b]);
      // projections within the bound: recomputed in fp32 from hi + lo by the whole warp
      uint32_t lanes = __ballot_sync(FULL, (need[0] | need[1] | need[2] | need[3]) != 0u);
      while (lanes) {
        const int src = __ffs(lanes) - 1;
        lanes &= lanes - 1;
        const int srow = 32 * qd + src;
        const uint2 hv = *reinterpret_cast<const uint2*>(rh + cofs(srow, 4 * lane));
        const uint2 lv = *reinterpret_cast<const uint2*>(rlo + cofs(srow, 4 * lane));
        const float2 h0 = __half22float2(*reinterpret_cast<const __half2*>(&hv.x));
        const float2 h1 = __half22float2(*reinterpret_cast<const __half2*>(&hv.y));
        const float2 l0 = __half22float2(*reinterpret_cast<const __half2*>(&lv.x));
        const float2 l1 = __half22float2(*reinterpret_cast<const __half2*>(&lv.y));
        const float r0 = h0.x + l0.x, r1 = h0.y + l0.y, r2 = h1.x + l1.x, r3 = h1.y + l1.y;
#pragma unroll
        for (int wi = 0; wi < 4; ++wi) {
          uint32_t nd = __shfl_sync(FULL, need[wi], src);
          while (nd) {
            const int j = __ffs(nd) - 1;
            nd &= nd - 1;
            const uint2 sv = *reinterpret_cast<const uint2*>(Ss + cofs(32 * wi + j, 4 * lane));
            const float2 s0 = __half22float2(*reinterpret_cast<const __half2*>(&sv.x));
            const float2 s1 = __half22float2(*reinterpret_cast<const __half2*>(&sv.y));
            float sdot = fmaf(s0.x, r0, fmaf(s0.y, r1, fmaf(s1.x, r2, s1.y * r3)));
            sdot = warp_sum(sdot);
            if (lane == src) sgn[wi] = sdot >= 0.f ? (sgn[wi] | (1u << j)) : (sgn[wi] & ~(1u << j));
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(rfree);  // the residual tiles may be overwritten
      if (vg < a.n_pad) {
        uint32_t* sd = reinterpret_cast<uint32_t*>(a.codes + (vg >> 5) * a.tbytes + KB * TILE * (DP / 8) +
                                                   (int)(vg & 31) * (a.m / 8));
        const bool valid = vg < a.n_vec;
#pragma unroll
        for (int wi = 0; wi < 4; ++wi)
          if (32 * wi < a.m) sd[wi] = valid ? sgn[wi] : 0u;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

template <int KB, bool PROD, bool BF>
int launch_rt(const CUtensorMap& map, const RArgs& a, int sm, cudaStream_t st) {
  using L = RL<PROD>;
  auto kern = quantize_rt_kernel<KB, PROD, BF>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::TOTAL);
  if (e != cudaSuccess) return tq::set_error(TQ_ECUDA, "tq_quantize: %s", cudaGetErrorString(e));
  const int64_t tiles = (a.n_pad + TV - 1) / TV;
  const int blocks = (int)std::max<int64_t>(1, std::min<int64_t>(tiles, sm));
  kern<<<blocks, L::NTHREADS, L::TOTAL, st>>>(map, a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return tq::set_error(TQ_ECUDA, "tq_quantize: launch failed: %s", cudaGetErrorString(e));
  return TQ_OK;
}

template <bool PROD, bool BF>
int dispatch_rt(int kb, const CUtensorMap& map, const RArgs& a, int sm, cudaStream_t st) {
  switch (kb) {
    case 1: return launch_rt<1, PROD, BF>(map, a, sm, st);
    case 2: return launch_rt<2, PROD, BF>(map, a, sm, st);
    case 3: return launch_rt<3, PROD, BF>(map, a, sm, st);
    default: return launch_rt<4, PROD, BF>(map, a, sm, st);
  }
}

}  // namespace

namespace tq {

// Whether the tensor-core rotation kernel handles this call: d_pad 128, 16-bit input,
// m 0 or 128, index bits up to 4 (3 in product mode).
bool quantize_rt_supported(const tq_params* p, int dtype) {
  const int kb = index_bits(p);
  return p->d_pad == 128 && (dtype == TQ_BF16 || dtype == TQ_F16) && kb >= 1 && kb <= 4 &&
         (p->mode == TQ_MODE_MSE || p->m == 128);
}

int launch_quantize_rt(const tq_params* p, const void* x, int dtype, int64_t n_vec, int64_t ld_bytes, void* codes,
                       uint16_t* norms, uint16_t* rnorms, int smc, cudaStream_t st) {
  CUtensorMap map;
  int rc = make_tmap_2d_u16(&map, x, (uint64_t)p->d, (uint64_t)n_vec, (uint64_t)ld_bytes, 8, TV);
  if (rc) return rc;
  RArgs a;
  a.n_vec = n_vec;
  a.n_pad = (n_vec + 31) / 32 * 32;
  a.d = p->d;
  a.m = p->mode == TQ_MODE_PROD ? p->m : 0;
  a.codes = static_cast<uint8_t*>(codes);
  a.norms = norms;
  a.rnorms = rnorms;
  a.cent = p->centroids;
  a.thr = p->thresholds;
  a.D = p->signs_D;
  a.S = p->S;
  a.tbytes = tqd::tile_bytes(DP, index_bits(p), a.m);
  const int kb = index_bits(p);
  const bool prod = p->mode == TQ_MODE_PROD;
  if (dtype == TQ_BF16)
    return prod ? dispatch_rt<true, true>(kb, map, a, smc, st) : dispatch_rt<false, true>(kb, map, a, smc, st);
  return prod ? dispatch_rt<true, false>(kb, map, a, smc, st) : dispatch_rt<false, false>(kb, map, a, smc, st);
}

}  // namespace tq

namespace tq {
// Read (and optionally clear) this translation unit's device fault word.
int fault_word_quantize_rt(int clear, int* value) {
  cudaError_t e = cudaMemcpyFromSymbol(value, tqd::g_fault, sizeof(int));
  if (e == cudaSuccess && clear) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(tqd::g_fault, &zero, sizeof(int));
  }
  return e == cudaSuccess ? TQ_OK : set_error(TQ_ECUDA, "tq_device_status: %s", cudaGetErrorString(e));
}
}  // namespace tq
