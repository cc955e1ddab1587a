// tq_quantize for d_pad = 128 with 16-bit input, and the fused projection +
// quantize (tq_project_quantize): the rotation and the QJL projection on the
// fifth-generation tensor cores.
//
// Method ("TurboQuant explainer" (m.163.com), "第一步：PolarQuant" and
// "第二步：QJL"): norm, random sign flips + Walsh-Hadamard rotation, Lloyd-Max
// code at b-1 bits (b bits in MSE mode), residual and its norm, sign bits of S r.
// The fused form takes the vectors straight from the K/V projection of an
// attention layer (x W^T per head, rounded to bf16 as a cache write would be)
// without writing them to memory: quantize-on-write ("turboquant_plus", the
// prefill path of the runtime port).
//
// Design (B200, sm_100a), one persistent CTA per SM over tiles of 128 vectors:
//  * source of a tile, one of
//    - TMA: warp 0 loads the tile as 16 boxes of 8 elements x 128 rows, which
//      land as the K-major canonical layout of an MMA operand (K chunk k8 of
//      every row in one 2 KB slab); rows past the end and columns past d read 0;
//    - projection: warp 0 streams K blocks of 64 of the layer input x (128
//      tokens) and of the head's weight rows into a ring, one TMA box with
//      128-byte swizzle per operand and block (tiles numbered head-fastest, so
//      the CTAs running together share their token rows); warp 1 runs the
//      bf16 GEMM x W_h^T into tensor memory (M = 128 tokens, N = 128, fp32), and
//      warps 10-13 read the accumulator back, round it to bf16 and write the
//      tile in the canonical layout (optionally also to memory);
//  * warp 1 issues, per tile, the rotation y = X (H D)^T (M = 128 vectors,
//    N = 128 coordinates, K = 128; the +-1 entries of H D are exact in 16 bits,
//    fp32 accumulation) into one of two tensor-memory buffers, and, once the
//    residual of the tile is written, the projection z = R S^T on its fp16 hi
//    and lo parts (S r to about 2^-22 before fp32 accumulation).  Warp-uniform
//    loops, elect-issued MMAs.  In the projection form these small MMAs are
//    slotted in between the GEMM's K blocks as soon as their inputs are ready,
//    so the tensor pipe never waits for an epilogue;
//  * warps 2-9 encode: two threads per vector (the two warps of a lane
//    quadrant take coordinates 0-63 and 64-127), y read back with tcgen05.ld;
//    the squared norms of the two halves meet in shared memory; the code and the
//    residual as in the two-thread kernel (quantize_tc.cu), with the thresholds
//    scaled per vector so that no value needs the 1/(sqrt(128) n) multiply; the
//    residual (x 2^14) goes to the hi / lo operand tiles;
//  * warps 10-13 (product mode) read z back (a thread per vector, all
//    projections), pack the sign words, and recompute in fp32 from the hi + lo
//    parts the projections within the fp32 accumulation bound of zero.  They run
//    one tile behind the encode warps, which wait for them only before writing
//    the next residual.
// Every hand-off is an mbarrier with an iteration limit.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <climits>

#include <cuda_bf16.h>

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
  int sliced;  // token-sliced layout (MSE codes): per tile and plane, word j holds coordinate j of the 32 vectors
  // projection source: vector v = head * n_tok + token, tiles of 128 tokens of one head
  int64_t n_tok;
  int n_heads, hidden;
  uint16_t* k_out;  // optional bf16 copy of the projected vectors, [n_tok][n_heads * 128] (row stride ld_k)
  int64_t ld_k;
};

// byte offset of element (row, k) of a canonical K-major 128 x 128 16-bit tile
__device__ __forceinline__ int cofs(int row, int k) { return (k >> 3) * SLAB + (row >> 3) * 128 + (row & 7) * 16 + (k & 7) * 2; }

template <bool PROD, bool GEMM>
struct RL {
  static constexpr int NX = GEMM ? 1 : (PROD ? 2 : 4);  // input tiles (TMA source) / the projected tile
  static constexpr int NG = GEMM ? (PROD ? 2 : 4) : 0;   // GEMM K-block stages
  static constexpr int KBLK = 64;                        // GEMM K block (elements): one 128-byte swizzled row
  static constexpr int GSTAGE = 2 * (KBLK / 8) * SLAB;   // x block + weight block (16 KB each), 1 TMA copy each
  static constexpr int HD = 0;                           // H D, canonical (N = out coordinate, K = in)
  static constexpr int SS = HD + TILE_B;                 // S, canonical (N = projection, K = coordinate)
  static constexpr int XS = SS + (PROD ? TILE_B : 0);    // [NX] input tiles
  static constexpr int GS = XS + NX * TILE_B;            // GEMM stages
  // residual (A of the projection): the hi part is written over the tile's own input buffer,
  // which the rotation has read by then; the lo part has buffers of its own, one per tile
  // parity with the TMA source (so a tile's encode does not wait for the previous read-back)
  static constexpr int NRL = PROD ? (GEMM ? 1 : 2) : 0;
  static constexpr int RLO = GS + NG * GSTAGE;
  static constexpr int NSQ = RLO + NRL * TILE_B;         // [2 tile parities][2 halves][128] squared norms
  static constexpr int GSQ = NSQ + 4 * TV * 4;           // [2 halves][128] squared residual norms
  static constexpr int BND = GSQ + 2 * TV * 4;           // [2][128] fix-up bound per vector (per tile parity)
  static constexpr int BAR = BND + 2 * TV * 4;
  static constexpr int TOTAL = BAR + 512;
  static constexpr int W_MMA = 1, W_ENC0 = 2, W_RB0 = 10;
  static constexpr int NTHREADS = (PROD || GEMM ? 14 : 10) * 32;
  static_assert(TOTAL <= 227 * 1024, "shared memory");
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

// A tile's rows: vector index, whether it holds data, whether this CTA writes its code slot.
template <bool GEMM>
__device__ __forceinline__ void row_vector(const RArgs& a, int64_t tile, int r, int64_t& vg, bool& valid, bool& own) {
  if constexpr (GEMM) {
    // GEMM tiles are numbered head-fastest (tile = m-tile * n_heads + head), so the CTAs that run
    // at the same time share their token rows and read them from HBM once
    const int64_t h = tile % a.n_heads, t = (tile / a.n_heads) * TV + r;
    vg = h * a.n_tok + t;
    valid = t < a.n_tok;
    own = valid || (h == a.n_heads - 1 && vg < a.n_pad);  // the zero tail of the last code tile
  } else {
    vg = tile * TV + r;
    valid = vg < a.n_vec;
    own = vg < a.n_pad;
  }
}

// test_wait without blocking, made warp-uniform
__device__ __forceinline__ bool mbar_ready(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(done)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return __all_sync(FULL, done != 0u);
}

// 32 x 32 bit transpose across a warp: on return, bit t of lane j's word is bit j of
// lane t's word on entry (five exchange stages of s x s blocks between lanes l, l ^ s).
__device__ __forceinline__ uint32_t warp_transpose32(uint32_t x, int lane) {
  const uint32_t masks[5] = {0x0000FFFFu, 0x00FF00FFu, 0x0F0F0F0Fu, 0x33333333u, 0x55555555u};
#pragma unroll
  for (int k = 0; k < 5; ++k) {
    const int sft = 16 >> k;
    const uint32_t m = masks[k];
    const uint32_t y = __shfl_xor_sync(FULL, x, sft);
    x = (lane & sft) ? ((x & ~m) | ((y >> sft) & m)) : ((x & m) | ((y & m) << sft));
  }
  return x;
}

template <int KB, bool PROD, bool BF, bool GEMM>
__global__ void __launch_bounds__(RL<PROD, GEMM>::NTHREADS, 1)
    quantize_rt_kernel(const __grid_constant__ CUtensorMap tmap, const __grid_constant__ CUtensorMap tmap_w,
                       const RArgs a) {
  using L = RL<PROD, GEMM>;
  constexpr int NX = L::NX, NG = L::NG;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* hd = smem + L::HD;
  uint8_t* Ss = smem + L::SS;
  auto rh_of = [&](int j) { return smem + L::XS + (j % NX) * TILE_B; };         // residual hi of tile j
  auto rlo_of = [&](int j) { return smem + L::RLO + (L::NRL > 1 ? (j & 1) : 0) * TILE_B; };  // residual lo of tile j
  float* nsq = reinterpret_cast<float*>(smem + L::NSQ);
  float* gsq = reinterpret_cast<float*>(smem + L::GSQ);
  float* bnd = reinterpret_cast<float*>(smem + L::BND);
  uint64_t* xfull = reinterpret_cast<uint64_t*>(smem + L::BAR);  // [4] input tile ready (TMA: 1 + tx; GEMM: 4)
  uint64_t* xfree = xfull + 4;                                     // [4] rotation MMAs read it (1)
  uint64_t* yfull = xfree + 4;                                     // [2] rotation done (1)
  uint64_t* yfree = yfull + 2;                                     // [2] y read by the encode warps (8)
  uint64_t* rfull = yfree + 2;                                     // residual tiles written (8)
  uint64_t* rfree = rfull + 1;                                     // [2] residual tiles read back (4)
  uint64_t* zfull = rfree + 2;                                     // [2] projection done (1)
  uint64_t* zfree = zfull + 2;                                     // [2] z read back (4)
  uint64_t* gbar = zfree + 2;                                      // encode warps' barrier (8)
  uint64_t* gfull = gbar + 1;                                      // [8] GEMM stage loaded (1 + tx)
  uint64_t* gempty = gfull + 8;                                    // [8] GEMM stage read (1)
  uint64_t* accfull = gempty + 8;                                  // [2] GEMM accumulator complete (1)
  uint32_t* tbase = reinterpret_cast<uint32_t*>(accfull + 2);
  float* smax = reinterpret_cast<float*>(tbase + 1);
  float* wmax = smax + 1;  // [14]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t n_tiles = GEMM ? (int64_t)a.n_heads * ((a.n_tok + TV - 1) / TV) : (a.n_pad + TV - 1) / TV;

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
      mbar_init(&xfull[s], GEMM ? 4 : 1);
      mbar_init(&xfree[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&yfull[b], 1);
      mbar_init(&yfree[b], 8);
      mbar_init(&zfull[b], 1);
      mbar_init(&zfree[b], 4);
      mbar_init(&accfull[b], 1);
    }
    for (int s = 0; s < 8; ++s) {
      mbar_init(&gfull[s], 1);
      mbar_init(&gempty[s], 1);
    }
    mbar_init(rfull, 8);
    mbar_init(&rfree[0], 4);
    mbar_init(&rfree[1], 4);
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
  auto tile_of = [&](int i) { return t0 + (int64_t)i * ts; };
  const int nkb = GEMM ? (a.hidden + L::KBLK - 1) / L::KBLK : 0;  // a last half block reads zeros past hidden

  if (warp == 0) {
    // ---------------- producer: input tiles, or the GEMM's K blocks, by TMA ----------------
    if (lane == 0) {
      if constexpr (GEMM) {
        int64_t g = 0;
        bool ok = true;
        for (int i = 0; i < nt && ok; ++i) {
          const int64_t tile = tile_of(i), h = tile % a.n_heads;
          const int y = (int)((tile / a.n_heads) * TV), yw = (int)(h * TV);
          for (int kb = 0; kb < nkb; ++kb, ++g) {
            const int s = (int)(g % NG);
            if (g >= NG && !mbar_wait(&gempty[s], (uint32_t)(((g - NG) / NG) & 1))) {
              ok = false;
              break;
            }
            uint8_t* dst = smem + L::GS + s * L::GSTAGE;
            mbar_expect_tx(&gfull[s], L::GSTAGE);
            tma_load_2d(dst, &tmap, L::KBLK * kb, y, &gfull[s]);  // 128 rows x 128 bytes, swizzled
            tma_load_2d(dst + L::GSTAGE / 2, &tmap_w, L::KBLK * kb, yw, &gfull[s]);
          }
        }
        for (int64_t i = (g > NG ? g - NG : 0); i < g; ++i) mbar_wait(&gfull[i % NG], (uint32_t)((i / NG) & 1));
      } else {
        int issued = 0;
        for (int i = 0; i < nt; ++i) {
          const int s = i % NX;
          if (i >= NX && !mbar_wait(&xfree[s], ((i - NX) / NX) & 1)) break;
          // product mode: the residual hi part of tile i - 2, written over this slot, has been read back
          if (PROD && i >= NX && !mbar_wait(&rfree[(i - NX) & 1], ((i - NX) >> 1) & 1)) break;
          uint8_t* dst = smem + L::XS + s * TILE_B;
          mbar_expect_tx(&xfull[s], TILE_B);
          const int y = (int)(tile_of(i) * TV);
#pragma unroll 1
          for (int kc = 0; kc < DP / 8; ++kc) tma_load_2d(dst + kc * SLAB, &tmap, 8 * kc, y, &xfull[s]);
          issued = i + 1;
        }
        for (int i = (issued > NX ? issued - NX : 0); i < issued; ++i) mbar_wait(&xfull[i % NX], (i / NX) & 1);
      }
    }
    __syncwarp();
  } else if (warp == L::W_MMA) {
    // ---------------- MMA issue ----------------
    constexpr uint32_t id1 = idesc_16(TV, DP, BF);
    const uint32_t id2 = idesc_16(TV, a.m > 0 ? a.m : 128, false);
    const uint32_t shd = smem_u32(hd);
    // rotation of tile j: y = X (H D)^T into y buffer j & 1 (the projection source's
    // accumulator of that tile, already read back)
    auto rotation = [&](int j) {
      const int s = j % NX;
      const uint64_t ad = smem_desc(smem_u32(smem + L::XS + s * TILE_B), SLAB, 128);
      const uint64_t bd = smem_desc(shd, SLAB, 128);
#pragma unroll
      for (int ks = 0; ks < DP / 16; ++ks)
        umma_16_ss_elect(ycol(j & 1), ad + (uint64_t)(ks * (2 * SLAB >> 4)), bd + (uint64_t)(ks * (2 * SLAB >> 4)),
                         id1, ks ? 1u : 0u);
      umma_commit_elect(&yfull[j & 1]);
      umma_commit_elect(&xfree[s]);
    };
    // z = R S^T of tile j (R: hi then lo) into z buffer j & 1
    auto projection = [&](int j) {
      const uint32_t d = zcol(j & 1);
#pragma unroll
      for (int part = 0; part < 2; ++part) {
        const uint64_t ad = smem_desc(smem_u32(part ? rlo_of(j) : rh_of(j)), SLAB, 128);
        const uint64_t bd = smem_desc(smem_u32(Ss), SLAB, 128);
#pragma unroll
        for (int ks = 0; ks < DP / 16; ++ks)
          umma_16_ss_elect(d, ad + (uint64_t)(ks * (2 * SLAB >> 4)), bd + (uint64_t)(ks * (2 * SLAB >> 4)), id2,
                           (part | ks) ? 1u : 0u);
      }
      umma_commit_elect(&zfull[j & 1]);
    };
    bool ok = true;
    if constexpr (!GEMM) {
      auto proj_wait = [&](int j) {
        if (!mbar_wait(rfull, j & 1)) return false;
        if (j >= 2 && !mbar_wait(&zfree[j & 1], ((j - 2) >> 1) & 1)) return false;
        __syncwarp();
        tc_fence_after();
        projection(j);
        return true;
      };
      for (int i = 0; i < nt && ok; ++i) {
        const int s = i % NX, b = i & 1;
        if (!mbar_wait(&xfull[s], (i / NX) & 1)) break;
        if (i >= 2 && !mbar_wait(&yfree[b], ((i - 2) >> 1) & 1)) break;
        __syncwarp();
        tc_fence_after();
        rotation(i);
        if constexpr (PROD)
          if (i >= 1) ok = proj_wait(i - 1);
      }
      if constexpr (PROD)
        if (ok && nt >= 1) proj_wait(nt - 1);
    } else {
      // GEMM of tile i into accumulator i & 1; rotations and projections of earlier tiles
      // go in between K blocks once their inputs are ready (non-blocking tests), and are
      // forced, in dependency order, only where the next GEMM or the end needs them.
      constexpr uint32_t idg = idesc_16(TV, DP, true);
      int nrot = 0, nproj = 0;
      int64_t g = 0;
      auto rot_ready = [&](int j) { return mbar_ready(&xfull[0], j & 1); };
      auto proj_ready = [&](int j) {
        return mbar_ready(rfull, j & 1) && (j < 2 || mbar_ready(&zfree[j & 1], ((j - 2) >> 1) & 1));
      };
      auto try_small = [&](int limit_rot) {  // issue whatever is ready, in order
        for (;;) {
          if (PROD && nproj < nrot && proj_ready(nproj)) {
            tc_fence_after();
            projection(nproj++);
          } else if (nrot < limit_rot && (!PROD || nproj >= nrot - 1) && rot_ready(nrot)) {
            tc_fence_after();
            rotation(nrot++);
          } else {
            break;
          }
        }
      };
      // blocking: every rotation below `upto` issued (projections first where a rotation needs them)
      auto force = [&](int upto_rot, int upto_proj) {
        while (ok && (nrot < upto_rot || nproj < upto_proj)) {
          if (PROD && nproj < nrot && (nproj < upto_proj || nproj < nrot - 1 + (nrot < upto_rot ? 1 : 0))) {
            const int j = nproj;
            if (!mbar_wait(rfull, j & 1) || (j >= 2 && !mbar_wait(&zfree[j & 1], ((j - 2) >> 1) & 1))) {
              ok = false;
              break;
            }
            __syncwarp();
            tc_fence_after();
            projection(nproj++);
          } else if (nrot < upto_rot) {
            if (!mbar_wait(&xfull[0], nrot & 1)) {
              ok = false;
              break;
            }
            __syncwarp();
            tc_fence_after();
            rotation(nrot++);
          } else {
            break;
          }
        }
      };
      for (int i = 0; i < nt && ok; ++i) {
        const int b = i & 1;
        if (i >= 2) {
          force(i - 1, 0);  // y of tile i - 2 exists, so it can be consumed
          if (!ok || !mbar_wait(&yfree[b], ((i - 2) >> 1) & 1)) break;
        }
        __syncwarp();
        tc_fence_after();
        for (int kb = 0; kb < nkb; ++kb, ++g) {
          const int s = (int)(g % NG);
          if (!mbar_wait(&gfull[s], (uint32_t)((g / NG) & 1))) {
            ok = false;
            break;
          }
          __syncwarp();
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + L::GS + s * L::GSTAGE);
          const uint64_t ad = smem_desc_sw128(sa);
          const uint64_t bd = smem_desc_sw128(sa + L::GSTAGE / 2);
#pragma unroll
          for (int ks = 0; ks < L::KBLK / 16; ++ks)  // K step: 32 bytes along the swizzled rows
            umma_16_ss_elect(ycol(b), ad + (uint64_t)(2 * ks), bd + (uint64_t)(2 * ks), idg, (kb | ks) ? 1u : 0u);
          umma_commit_elect(&gempty[s]);
          try_small(i);
        }
        if (!ok) break;
        umma_commit_elect(&accfull[b]);
      }
      force(nt, PROD ? nt : 0);
    }
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
      int64_t vg;
      bool valid, own;
      row_vector<GEMM>(a, tile_of(i), v, vg, valid, own);
      if (!mbar_wait(&yfull[b], (i >> 1) & 1)) break;
      __syncwarp();
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
      // the residual buffers of this tile are free: the tile that used them last has been read back
      if (PROD && i >= L::NRL && !mbar_wait(&rfree[(i - L::NRL) & 1], ((i - L::NRL) >> 1) & 1)) break;
      uint8_t* rh = rh_of(i);
      uint8_t* rlo = rlo_of(i);
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
        if (h == 0 && valid) a.rnorms[vg] = __half_as_ushort(__float2half_rn(sqrtf(g2t) * (1.f / 16384.f)));
      }
      if (!PROD && !GEMM && a.sliced) {
        // the warp's 32 lanes are the 32 vectors of one code tile: transpose each 32-coordinate
        // block of each plane, so lane j holds coordinate 64h + 32w + j of the 32 vectors
        uint32_t* tw = reinterpret_cast<uint32_t*>(a.codes + (vg >> 5) * a.tbytes) + 64 * h + lane;
#pragma unroll
        for (int bb = 0; bb < KB; ++bb)
#pragma unroll
          for (int w = 0; w < 2; ++w) {
            const uint32_t t = warp_transpose32(valid ? pl[bb][w] : 0u, lane);
            if (own) tw[bb * DP + 32 * w] = t;  // every lane of a warp shares `own` (whole tiles)
          }
      } else if (own) {
        uint8_t* tb = a.codes + (vg >> 5) * a.tbytes + (int)(vg & 31) * (DP / 8) + 8 * h;
#pragma unroll
        for (int bb = 0; bb < KB; ++bb)
          *reinterpret_cast<uint2*>(tb + bb * TILE * (DP / 8)) = valid ? make_uint2(pl[bb][0], pl[bb][1]) : make_uint2(0, 0);
      }
      if (h == 0 && valid) a.norms[vg] = __half_as_ushort(__float2half_rn(n));
    }
  } else {
    // ---------------- warps 10-13: the projected tile (GEMM source), read-back of z (product mode) ----------------
    const int qd = warp & 3;
    const int v = 32 * qd + lane;
    // accumulator of tile i -> bf16 -> canonical tile (+ optional copy to memory)
    auto convert = [&](int i) {
      const int b = i & 1;
      if (!mbar_wait(&accfull[b], (i >> 1) & 1)) return false;
      // the tile buffer is free once the previous tile's rotation has read it and, in product
      // mode, its residual hi part (written over it) has been read back
      if (i >= 1) {
        if (PROD ? !mbar_wait(&rfree[(i - 1) & 1], ((i - 1) >> 1) & 1)
                 : !mbar_wait(&yfull[(i - 1) & 1], ((i - 1) >> 1) & 1))
          return false;
      }
      __syncwarp();
      tc_fence_after();
      int64_t vg;
      bool valid, own;
      row_vector<GEMM>(a, tile_of(i), v, vg, valid, own);
      const int64_t hh = tile_of(i) % a.n_heads, tok = vg - hh * a.n_tok;
      uint8_t* xs = smem + L::XS;
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        uint32_t c[32];
        tmem_ld32_issue(ycol(b) + ((uint32_t)(32 * qd) << 16) + 32 * q4, c);
        tmem_ld_wait(c);
#pragma unroll
        for (int k8 = 0; k8 < 4; ++k8) {
          uint32_t wv[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const __nv_bfloat162 h2 = __floats2bfloat162_rn(__uint_as_float(c[8 * k8 + 2 * e]),
                                                            __uint_as_float(c[8 * k8 + 2 * e + 1]));
            wv[e] = *reinterpret_cast<const uint32_t*>(&h2);
          }
          const uint4 w4 = make_uint4(wv[0], wv[1], wv[2], wv[3]);
          *reinterpret_cast<uint4*>(xs + cofs(v, 32 * q4 + 8 * k8)) = w4;
          if (a.k_out && valid)
            *reinterpret_cast<uint4*>(a.k_out + tok * a.ld_k + hh * DP + 32 * q4 + 8 * k8) = w4;
        }
      }
      fence_async_smem();  // the tile is read by the tensor core
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&xfull[0]);
      return true;
    };
    auto readback = [&](int i) {
      const int b = i & 1;
      int64_t vg;
      bool valid, own;
      row_vector<GEMM>(a, tile_of(i), v, vg, valid, own);
      // rfull of this tile completed before its projection was issued; waiting on it here as
      // well orders the encode warps' shared-memory writes (bounds, residual) before the reads below
      if (!mbar_wait(rfull, i & 1)) return false;
      if (!mbar_wait(&zfull[b], (i >> 1) & 1)) return false;
      __syncwarp();
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
          if ((int)any < 0 && valid && 32 * wi < a.m) {
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
        const uint2 hv = *reinterpret_cast<const uint2*>(rh_of(i) + cofs(srow, 4 * lane));
        const uint2 lv = *reinterpret_cast<const uint2*>(rlo_of(i) + cofs(srow, 4 * lane));
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
      if (lane == 0) mbar_arrive(&rfree[i & 1]);  // the residual tiles may be overwritten
      if (own) {
        uint32_t* sd = reinterpret_cast<uint32_t*>(a.codes + (vg >> 5) * a.tbytes + KB * TILE * (DP / 8) +
                                                   (int)(vg & 31) * (a.m / 8));
#pragma unroll
        for (int wi = 0; wi < 4; ++wi)
          if (32 * wi < a.m) sd[wi] = valid ? sgn[wi] : 0u;
      }
      return true;
    };
    // one tile behind in each role: readback(i - 1) frees the buffer convert(i) writes
    for (int i = 0; i < nt; ++i) {
      if (PROD && i >= 1 && !readback(i - 1)) break;
      if (GEMM && !convert(i)) break;
      if (PROD && i == nt - 1) readback(i);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

template <int KB, bool PROD, bool BF, bool GEMM>
int launch_rt(const CUtensorMap& map, const CUtensorMap& map_w, const RArgs& a, int64_t n_tiles, int sm,
              cudaStream_t st) {
  using L = RL<PROD, GEMM>;
  auto kern = quantize_rt_kernel<KB, PROD, BF, GEMM>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::TOTAL);
  if (e != cudaSuccess) return tq::set_error(TQ_ECUDA, "tq_quantize: %s", cudaGetErrorString(e));
  const int blocks = (int)std::max<int64_t>(1, std::min<int64_t>(n_tiles, sm));
  kern<<<blocks, L::NTHREADS, L::TOTAL, st>>>(map, map_w, a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return tq::set_error(TQ_ECUDA, "tq_quantize: launch failed: %s", cudaGetErrorString(e));
  return TQ_OK;
}

template <bool PROD, bool BF, bool GEMM>
int dispatch_rt(int kb, const CUtensorMap& map, const CUtensorMap& map_w, const RArgs& a, int64_t n_tiles, int sm,
                cudaStream_t st) {
  switch (kb) {
    case 1: return launch_rt<1, PROD, BF, GEMM>(map, map_w, a, n_tiles, sm, st);
    case 2: return launch_rt<2, PROD, BF, GEMM>(map, map_w, a, n_tiles, sm, st);
    case 3: return launch_rt<3, PROD, BF, GEMM>(map, map_w, a, n_tiles, sm, st);
    default:
      if constexpr (PROD) return tq::set_error(TQ_EUNSUPPORTED, "tq_quantize: product mode uses at most 3 index bits");
      else return launch_rt<4, PROD, BF, GEMM>(map, map_w, a, n_tiles, sm, st);
  }
}

}  // namespace

namespace tq {

// Whether tq_quantize runs on the tensor-core rotation kernel: d_pad 128, 16-bit input, MSE
// codes (either layout).  Product codes stay on the register kernel (quantize_tc.cu), which is
// faster there (72 against 101 us for 2^18 keys at b = 3): with the sign read-back added, this
// kernel issues about 108 warp-instructions per vector at an IPC near 1.  The product form of
// this kernel serves the fused projection path.
bool quantize_rt_supported(const tq_params* p, int dtype) {
  const int kb = index_bits(p);
  return p->d_pad == 128 && (dtype == TQ_BF16 || dtype == TQ_F16) && kb >= 1 && kb <= 4 && p->mode == TQ_MODE_MSE;
}

int launch_quantize_rt(const tq_params* p, const void* x, int dtype, int64_t n_vec, int64_t ld_bytes, void* codes,
                       uint16_t* norms, uint16_t* rnorms, int smc, cudaStream_t st) {
  CUtensorMap map;
  int rc = make_tmap_2d_u16(&map, x, (uint64_t)p->d, (uint64_t)n_vec, (uint64_t)ld_bytes, 8, TV);
  if (rc) return rc;
  RArgs a = {};
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
  a.sliced = p->layout == TQ_LAYOUT_SLICED;
  const int kb = index_bits(p);
  const bool prod = p->mode == TQ_MODE_PROD;
  const int64_t tiles = (a.n_pad + TV - 1) / TV;
  if (dtype == TQ_BF16)
    return prod ? dispatch_rt<true, true, false>(kb, map, map, a, tiles, smc, st)
                : dispatch_rt<false, true, false>(kb, map, map, a, tiles, smc, st);
  return prod ? dispatch_rt<true, false, false>(kb, map, map, a, tiles, smc, st)
              : dispatch_rt<false, false, false>(kb, map, map, a, tiles, smc, st);
}

int sm_count();

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

extern "C" int tq_project_quantize(const tq_params* p, const void* x, int64_t n_tok, int64_t ld_x, int hidden,
                                   const void* w, int n_heads, int64_t ld_w, void* codes, uint16_t* norms,
                                   uint16_t* rnorms, void* k_out, int64_t ld_k, tq_stream_t stream) {
  using namespace tq;
  int rc = check_params(p, "tq_project_quantize");
  if (!rc) rc = check_planes(p, "tq_project_quantize");
  if (rc) return rc;
  const bool prod = p->mode == TQ_MODE_PROD;
  if (p->d != 128 || p->d_pad != 128 || (prod && p->m != 128))
    return set_error(TQ_EUNSUPPORTED, "tq_project_quantize: needs d = d_pad = 128 and m = 128 in product mode");
  if (n_tok < 0 || n_tok > (int64_t)INT32_MAX - 256 || n_heads < 1 || hidden < 32 || hidden % 32 != 0)
    return set_error(TQ_EINVAL, "tq_project_quantize: bad n_tok / n_heads / hidden (hidden a positive multiple of 32)");
  if ((int64_t)n_heads * n_tok > (int64_t)INT32_MAX)
    return set_error(TQ_EINVAL, "tq_project_quantize: n_heads * n_tok too large");
  if (n_tok == 0) {
    clear_error();
    return TQ_OK;
  }
  if (!x || !w || !codes || !norms || (prod && !rnorms))
    return set_error(TQ_EINVAL, "tq_project_quantize: NULL x/w/codes/norms/rnorms");
  if (ld_x < hidden || ld_w < hidden || !aligned(x, 16) || !aligned(w, 16) || (ld_x * 2) % 16 != 0 ||
      (ld_w * 2) % 16 != 0)
    return set_error(TQ_EINVAL, "tq_project_quantize: x / w need 16-byte alignment and row strides >= hidden, "
                                "multiples of 8 elements");
  if (k_out && (ld_k < (int64_t)n_heads * 128 || !aligned(k_out, 16) || (ld_k * 2) % 16 != 0))
    return set_error(TQ_EINVAL, "tq_project_quantize: k_out needs 16-byte alignment and ld_k >= 128 * n_heads, "
                                "a multiple of 8");
  if (!aligned(codes, 16) || !aligned(norms, 2) || (rnorms && !aligned(rnorms, 2)))
    return set_error(TQ_EINVAL, "tq_project_quantize: codes must be 16-byte aligned, norms 2-byte aligned");
  CUtensorMap mx, mw;
  rc = make_tmap_2d_u16(&mx, x, (uint64_t)hidden, (uint64_t)n_tok, (uint64_t)ld_x * 2, 64, TV, true);
  if (rc) return rc;
  rc = make_tmap_2d_u16(&mw, w, (uint64_t)hidden, (uint64_t)n_heads * 128, (uint64_t)ld_w * 2, 64, TV, true);
  if (rc) return rc;
  RArgs a = {};
  a.n_vec = (int64_t)n_heads * n_tok;
  a.n_pad = (a.n_vec + 31) / 32 * 32;
  a.d = 128;
  a.m = prod ? p->m : 0;
  a.codes = static_cast<uint8_t*>(codes);
  a.norms = norms;
  a.rnorms = rnorms;
  a.cent = p->centroids;
  a.thr = p->thresholds;
  a.D = p->signs_D;
  a.S = p->S;
  a.tbytes = tqd::tile_bytes(DP, index_bits(p), a.m);
  a.n_tok = n_tok;
  a.n_heads = n_heads;
  a.hidden = hidden;
  a.k_out = static_cast<uint16_t*>(k_out);
  a.ld_k = ld_k;
  const int64_t tiles = (int64_t)n_heads * ((n_tok + TV - 1) / TV);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int kb = index_bits(p);
  rc = prod ? dispatch_rt<true, true, true>(kb, mx, mw, a, tiles, sm_count(), st)
            : dispatch_rt<false, true, true>(kb, mx, mw, a, tiles, sm_count(), st);
  if (rc == TQ_OK) clear_error();
  return rc;
}
