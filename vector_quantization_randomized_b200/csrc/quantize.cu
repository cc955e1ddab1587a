// tq_quantize: norm, random rotation, Lloyd-Max code, residual and QJL signs.
//
// Method ("TurboQuant explainer" (m.163.com), "TurboQuant 怎么做的"):
//  "第一步：PolarQuant" - random rotation (here sign flips D then the
//  Walsh-Hadamard transform, per the zhidx turboquant_plus article), then one
//  fixed Lloyd-Max table for every coordinate, b-1 bits;
//  "第二步：QJL" - sign bits of a Gaussian JL projection of the residual.
//
// Kernel design (B200, sm_100a):
//  * A warp owns 16 vectors at a time.  Their rows are staged into shared
//    memory with cp.async (double-buffered across groups) so HBM reads are
//    16-byte and stay in flight while the previous group is computed.
//  * One vector per warp pass: lane l holds coordinates l + 32 i.  The WHT is
//    log2(d_pad/32) in-register butterfly stages plus 5 shuffle stages.  The
//    norm is folded into one final scale: y = WHT(D o x) * (1/(n sqrt(d_pad))).
//  * Index bit-planes come straight out of __ballot_sync: ballot over lanes of
//    bit p of register i is word i of plane p in the canonical layout.
//  * The residuals of the 16 vectors (fp32, shared memory) times S^T (fp16,
//    shared memory, loaded once per CTA) run on the tensor cores
//    (mma.sync m16n8k16, fp32 accumulate).  A projection whose magnitude is
//    below the rounding bound of the fp16 residual, 2^-10 ||S_i|| gamma +
//    2^-20 ||S_i||, is recomputed exactly in fp32 by the whole warp, so every
//    stored sign is the sign of the fp32 projection of the fp32 residual.
#include <cuda_runtime.h>

#include <algorithm>

#include "common.h"
#include "device.cuh"

namespace {

using namespace tqd;

struct QArgs {
  const uint8_t* x;
  int64_t n_vec, n_pad, ld_bytes;
  int d, m, row_bytes, nbuf;
  uint8_t* codes;
  uint16_t* norms;
  uint16_t* rnorms;
  const float* cent;
  const float* thr;
  const int8_t* D;
  const uint16_t* S;
};

constexpr int GROUP = 16;  // vectors per warp batch (= MMA M)

template <int DT>
__device__ __forceinline__ float load_elem(const uint8_t* row, int j) {
  if constexpr (DT == TQ_F32) return reinterpret_cast<const float*>(row)[j];
  if constexpr (DT == TQ_F16) return __half2float(reinterpret_cast<const __half*>(row)[j]);
  return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(row)[j]);
}

// Shared-memory carve-up (bytes), identical on host and device.
struct QSmem {
  int s_off, sn_off, x_off, r_off, g_off, total;
  __host__ __device__ QSmem(int dp, int m, bool prod, int nw, int row_bytes, int nbuf) {
    int o = 0;
    s_off = o;
    o += prod ? m * (dp + 8) * 2 : 0;
    sn_off = o;
    o += prod ? m * 4 : 0;
    o = (o + 15) & ~15;
    x_off = o;
    o += nw * nbuf * GROUP * row_bytes;
    r_off = o;
    o += prod ? nw * GROUP * (dp + 4) * 4 : 0;
    g_off = o;
    o += prod ? nw * GROUP * 4 : 0;
    total = o;
  }
};

template <int DP, int KB, bool PROD, int DT, int NW>
__global__ void __launch_bounds__(NW * 32) quantize_kernel(const QArgs a) {
  constexpr int NI = DP / 32;        // coordinates per lane
  constexpr int L = 1 << KB;         // codebook levels
  constexpr int SST = DP + 8;        // S row stride (halves)
  constexpr int RST = DP + 4;        // residual row stride (floats)
  extern __shared__ __align__(16) uint8_t smem[];
  const QSmem lay(DP, a.m, PROD, NW, a.row_bytes, a.nbuf);
  __half* S_s = reinterpret_cast<__half*>(smem + lay.s_off);
  float* Sn_s = reinterpret_cast<float*>(smem + lay.sn_off);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t* xs = smem + lay.x_off + warp * a.nbuf * GROUP * a.row_bytes;
  float* R = reinterpret_cast<float*>(smem + lay.r_off) + warp * GROUP * RST;
  float* gam = reinterpret_cast<float*>(smem + lay.g_off) + warp * GROUP;

  // per-CTA constants: S (fp16) and its row norms
  if constexpr (PROD) {
    const int chunks_per_row = DP / 8;  // 16-byte chunks
    for (int c = threadIdx.x; c < a.m * chunks_per_row; c += NW * 32) {
      int row = c / chunks_per_row, col = c % chunks_per_row;
      uint4 v = reinterpret_cast<const uint4*>(a.S + (size_t)row * DP)[col];
      *reinterpret_cast<uint4*>(S_s + row * SST + col * 8) = v;
    }
    __syncthreads();
    for (int row = warp; row < a.m; row += NW) {
      float s = 0.f;
#pragma unroll
      for (int i = 0; i < NI; ++i) {
        float v = __half2float(S_s[row * SST + 32 * i + lane]);
        s = fmaf(v, v, s);
      }
      s = warp_sum(s);
      if (lane == 0) Sn_s[row] = sqrtf(s) * 1.0001f;  // tiny inflation: bound stays a bound
    }
    __syncthreads();
  }

  float thr[L - 1], Dv[NI];
#pragma unroll
  for (int l = 0; l < L - 1; ++l) thr[l] = a.thr[l];
#pragma unroll
  for (int i = 0; i < NI; ++i) Dv[i] = (float)a.D[32 * i + lane];
  const float rs = rsqrtf((float)DP);
  const int tb = tile_bytes(DP, KB, a.m);
  const int64_t n_groups = (a.n_pad + GROUP - 1) / GROUP;
  const int64_t gstride = (int64_t)gridDim.x * NW;

  auto issue = [&](int64_t g, int buf) {
    uint8_t* dst = xs + buf * GROUP * a.row_bytes;
    const int cpr = a.row_bytes / 16;
    for (int c = lane; c < GROUP * cpr; c += 32) {
      int r = c / cpr, col = c % cpr;
      int64_t v = g * GROUP + r;
      if (v < a.n_vec) cp_async16(dst + r * a.row_bytes + col * 16, a.x + v * a.ld_bytes + col * 16);
    }
    cp_async_commit();
  };

  int64_t g = (int64_t)blockIdx.x * NW + warp;
  int buf = 0;
  if (g < n_groups) issue(g, 0);
  for (; g < n_groups; g += gstride) {
    const int64_t gn = g + gstride;
    if (a.nbuf == 2) {  // prefetch the next group into the other buffer
      if (gn < n_groups) issue(gn, buf ^ 1);
      else cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncwarp();
    const uint8_t* xb = xs + buf * GROUP * a.row_bytes;

    for (int r = 0; r < GROUP; ++r) {
      const int64_t v = g * GROUP + r;
      if (v >= a.n_pad) break;
      const int64_t tile = v >> 5;
      const int slot = (int)(v & 31);
      uint8_t* tbase = a.codes + tile * tb;
      if (v >= a.n_vec) {  // zero-fill the tail of the last tile
        for (int k = lane; k < KB * DP / 32; k += 32) {
          int p = k / NI, w = k % NI;
          reinterpret_cast<uint32_t*>(tbase + p * TILE * (DP / 8) + slot * (DP / 8))[w] = 0u;
        }
        if constexpr (PROD) {
          for (int w = lane; w < a.m / 32; w += 32)
            reinterpret_cast<uint32_t*>(tbase + KB * TILE * (DP / 8) + slot * (a.m / 8))[w] = 0u;
#pragma unroll
          for (int i = 0; i < NI; ++i) R[r * RST + 32 * i + lane] = 0.f;
          if (lane == 0) gam[r] = 0.f;
        }
        continue;
      }
      const uint8_t* row = xb + r * a.row_bytes;
      float y[NI];
      float ss = 0.f;
#pragma unroll
      for (int i = 0; i < NI; ++i) {
        const int j = 32 * i + lane;
        float xv = (j < a.d) ? load_elem<DT>(row, j) : 0.f;
        ss = fmaf(xv, xv, ss);
        y[i] = xv * Dv[i];
      }
      ss = warp_sum(ss);
      const float n = sqrtf(ss);
      // Walsh-Hadamard transform (natural order): register bits, then lane bits
#pragma unroll
      for (int h = 1; h < NI; h <<= 1) {
#pragma unroll
        for (int i = 0; i < NI; ++i) {
          if ((i & h) == 0) {
            float u = y[i], w = y[i + h];
            y[i] = u + w;
            y[i + h] = u - w;
          }
        }
      }
#pragma unroll
      for (int s = 1; s < 32; s <<= 1) {
#pragma unroll
        for (int i = 0; i < NI; ++i) {
          float o = __shfl_xor_sync(FULL, y[i], s);
          y[i] = (lane & s) ? (o - y[i]) : (y[i] + o);
        }
      }
      const float scale = (n > 0.f) ? rs / n : 0.f;
      int idx[NI];
      float r2 = 0.f;
#pragma unroll
      for (int i = 0; i < NI; ++i) {
        y[i] *= scale;
        int c = 0;
#pragma unroll
        for (int l = 0; l < L - 1; ++l) c += (y[i] > thr[l]) ? 1 : 0;
        idx[i] = c;
        const float res = y[i] - __ldg(a.cent + c);
        if constexpr (PROD) R[r * RST + 32 * i + lane] = res;
        r2 = fmaf(res, res, r2);
      }
      // bit-planes: ballot over lanes of bit p of register i = word i of plane p
#pragma unroll
      for (int p = 0; p < KB; ++p) {
        uint32_t wds[NI];
#pragma unroll
        for (int i = 0; i < NI; ++i) wds[i] = __ballot_sync(FULL, (idx[i] >> p) & 1);
        uint4* dst = reinterpret_cast<uint4*>(tbase + p * TILE * (DP / 8) + slot * (DP / 8));
#pragma unroll
        for (int q = 0; q < NI / 4; ++q)
          if (lane == p * (NI / 4) + q) dst[q] = make_uint4(wds[4 * q], wds[4 * q + 1], wds[4 * q + 2], wds[4 * q + 3]);
      }
      if (lane == 0) a.norms[v] = __half_as_ushort(__float2half_rn(n));
      if constexpr (PROD) {
        r2 = warp_sum(r2);
        const float gm = sqrtf(r2);
        if (lane == 0) {
          a.rnorms[v] = __half_as_ushort(__float2half_rn(gm));
          gam[r] = gm;
        }
      }
    }
    __syncwarp();

    if constexpr (PROD) {
      const int gq = lane >> 2, t = lane & 3;
      const int64_t v0 = g * GROUP + gq, v1 = v0 + 8;
      const bool ok0 = v0 < a.n_vec, ok1 = v1 < a.n_vec;
      const float g0 = gam[gq], g1 = gam[gq + 8];
      const int n_half = (a.m + 127) / 128;
      for (int hf = 0; hf < n_half; ++hf) {
        const int ncol = min(128, a.m - 128 * hf);
        const int nt_cnt = ncol / 8;
        float acc[16][4];
#pragma unroll
        for (int nt = 0; nt < 16; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
#pragma unroll 2
        for (int ks = 0; ks < DP / 16; ++ks) {
          const int k0 = 16 * ks + 2 * t;
          uint32_t af[4];
          af[0] = pack_half2(R[gq * RST + k0], R[gq * RST + k0 + 1]);
          af[1] = pack_half2(R[(gq + 8) * RST + k0], R[(gq + 8) * RST + k0 + 1]);
          af[2] = pack_half2(R[gq * RST + k0 + 8], R[gq * RST + k0 + 9]);
          af[3] = pack_half2(R[(gq + 8) * RST + k0 + 8], R[(gq + 8) * RST + k0 + 9]);
#pragma unroll
          for (int nt = 0; nt < 16; ++nt) {
            if (nt < nt_cnt) {
              const __half* srow = S_s + (128 * hf + 8 * nt + gq) * SST + k0;
              uint32_t b0 = *reinterpret_cast<const uint32_t*>(srow);
              uint32_t b1 = *reinterpret_cast<const uint32_t*>(srow + 8);
              mma_f16_16816(acc[nt], af, b0, b1);
            }
          }
        }
        // sign bits and the fp32 fix-up of projections inside the fp16 bound
        uint32_t sb0 = 0, sb1 = 0, nd0 = 0, nd1 = 0;
#pragma unroll
        for (int nt = 0; nt < 16; ++nt) {
          if (nt < nt_cnt) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int col = 128 * hf + 8 * nt + 2 * t + e;
              const float sn = Sn_s[col];
              const float z0 = acc[nt][e], z1 = acc[nt][2 + e];
              const int bit = 2 * nt + e;
              sb0 |= (z0 >= 0.f ? 1u : 0u) << bit;
              sb1 |= (z1 >= 0.f ? 1u : 0u) << bit;
              if (ok0 && fabsf(z0) <= sn * fmaf(0.0009765625f, g0, 9.5367431640625e-07f)) nd0 |= 1u << bit;
              if (ok1 && fabsf(z1) <= sn * fmaf(0.0009765625f, g1, 9.5367431640625e-07f)) nd1 |= 1u << bit;
            }
          }
        }
        while (true) {
          const unsigned any = __ballot_sync(FULL, (nd0 | nd1) != 0u);
          if (!any) break;
          const int leader = __ffs(any) - 1;
          int item = 0;
          if (lane == leader) item = nd0 ? (__ffs(nd0) - 1) : (32 + __ffs(nd1) - 1);
          item = __shfl_sync(FULL, item, leader);
          const int row = (leader >> 2) + ((item >= 32) ? 8 : 0);
          const int bit = item & 31;
          const int col = 128 * hf + 8 * (bit >> 1) + 2 * (leader & 3) + (bit & 1);
          float part = 0.f;
#pragma unroll
          for (int i = 0; i < NI; ++i) {
            const int j = 32 * i + lane;
            part = fmaf(R[row * RST + j], __half2float(S_s[col * SST + j]), part);
          }
          part = warp_sum(part);
          if (lane == leader) {
            const uint32_t m1 = 1u << bit;
            if (item < 32) {
              sb0 = (part >= 0.f) ? (sb0 | m1) : (sb0 & ~m1);
              nd0 &= ~m1;
            } else {
              sb1 = (part >= 0.f) ? (sb1 | m1) : (sb1 & ~m1);
              nd1 &= ~m1;
            }
          }
        }
        // assemble 32-bit sign words: word w covers columns 32w..32w+31 of this half
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          uint32_t w0 = 0, w1 = 0;
#pragma unroll
          for (int qq = 0; qq < 4; ++qq) {
            const int nt = 4 * w + qq;
            w0 |= ((sb0 >> (2 * nt)) & 3u) << (8 * qq + 2 * t);
            w1 |= ((sb1 >> (2 * nt)) & 3u) << (8 * qq + 2 * t);
          }
          w0 |= __shfl_xor_sync(FULL, w0, 1);
          w0 |= __shfl_xor_sync(FULL, w0, 2);
          w1 |= __shfl_xor_sync(FULL, w1, 1);
          w1 |= __shfl_xor_sync(FULL, w1, 2);
          if (t == w && 32 * w < ncol) {
            const int widx = 4 * hf + w;
            if (ok0) {
              uint8_t* tb0 = a.codes + (v0 >> 5) * tb + KB * TILE * (DP / 8) + (int)(v0 & 31) * (a.m / 8);
              reinterpret_cast<uint32_t*>(tb0)[widx] = w0;
            }
            if (ok1) {
              uint8_t* tb1 = a.codes + (v1 >> 5) * tb + KB * TILE * (DP / 8) + (int)(v1 & 31) * (a.m / 8);
              reinterpret_cast<uint32_t*>(tb1)[widx] = w1;
            }
          }
        }
      }
      __syncwarp();
    }
    if (a.nbuf == 2) {
      buf ^= 1;
    } else if (gn < n_groups) {  // single buffer: load the next group once this one is done
      issue(gn, 0);
    }
  }
  cp_async_wait<0>();
}

template <int DP, int KB, bool PROD, int DT>
int launch_q(const QArgs& a, int sm_count, cudaStream_t st) {
  constexpr int NW = (DP == 256) ? 2 : 4;  // keeps S (fp16) + staging + residuals in 227 KB
  QArgs args = a;
  QSmem lay(DP, a.m, PROD, NW, a.row_bytes, 2);
  args.nbuf = 2;
  if (lay.total > 227 * 1024) {
    args.nbuf = 1;
    lay = QSmem(DP, a.m, PROD, NW, a.row_bytes, 1);
    if (lay.total > 227 * 1024) return tq::set_error(TQ_EUNSUPPORTED, "tq_quantize: shape needs too much shared memory");
  }
  auto kern = quantize_kernel<DP, KB, PROD, DT, NW>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, lay.total);
  if (e != cudaSuccess) return tq::set_error(TQ_ECUDA, "tq_quantize: %s", cudaGetErrorString(e));
  int per_sm = 1;
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, NW * 32, lay.total);
  per_sm = std::max(per_sm, 1);
  const int64_t groups = (a.n_pad + GROUP - 1) / GROUP;
  const int64_t want = (groups + NW - 1) / NW;
  const int blocks = (int)std::max<int64_t>(1, std::min<int64_t>(want, (int64_t)sm_count * per_sm));
  kern<<<blocks, NW * 32, lay.total, st>>>(args);
  e = cudaGetLastError();
  if (e != cudaSuccess) return tq::set_error(TQ_ECUDA, "tq_quantize: launch failed: %s", cudaGetErrorString(e));
  return TQ_OK;
}

template <int DP, int KB, bool PROD>
int dispatch_dt(int dt, const QArgs& a, int smc, cudaStream_t st) {
  switch (dt) {
    case TQ_F32: return launch_q<DP, KB, PROD, TQ_F32>(a, smc, st);
    case TQ_F16: return launch_q<DP, KB, PROD, TQ_F16>(a, smc, st);
    default: return launch_q<DP, KB, PROD, TQ_BF16>(a, smc, st);
  }
}

template <int DP>
int dispatch_kb(int kb, bool prod, int dt, const QArgs& a, int smc, cudaStream_t st) {
  if (prod) {
    switch (kb) {
      case 1: return dispatch_dt<DP, 1, true>(dt, a, smc, st);
      case 2: return dispatch_dt<DP, 2, true>(dt, a, smc, st);
      default: return dispatch_dt<DP, 3, true>(dt, a, smc, st);
    }
  }
  switch (kb) {
    case 1: return dispatch_dt<DP, 1, false>(dt, a, smc, st);
    case 2: return dispatch_dt<DP, 2, false>(dt, a, smc, st);
    case 3: return dispatch_dt<DP, 3, false>(dt, a, smc, st);
    default: return dispatch_dt<DP, 4, false>(dt, a, smc, st);
  }
}

}  // namespace

namespace tq {
bool quantize128_supported(const tq_params* p, int dtype);
bool quantize_rt_supported(const tq_params* p, int dtype);
int launch_quantize_rt(const tq_params* p, const void* x, int dtype, int64_t n_vec, int64_t ld_bytes, void* codes,
                       uint16_t* norms, uint16_t* rnorms, int smc, cudaStream_t st);
int launch_quantize128(const tq_params* p, const void* x, int dtype, int64_t n_vec, int64_t ld_bytes, void* codes,
                       uint16_t* norms, uint16_t* rnorms, int smc, cudaStream_t st);
int sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}
}  // namespace tq

extern "C" int tq_quantize(const tq_params* p, const void* x, int dtype, int64_t n_vec, int64_t ld, void* codes,
                           uint16_t* norms, uint16_t* rnorms, tq_stream_t stream) {
  using namespace tq;
  int rc = check_params(p, "tq_quantize");
  if (rc) return rc;
  if (dtype != TQ_F32 && dtype != TQ_F16 && dtype != TQ_BF16) return set_error(TQ_EINVAL, "tq_quantize: bad dtype");
  if (n_vec < 0) return set_error(TQ_EINVAL, "tq_quantize: n_vec < 0");
  if (n_vec == 0) {
    clear_error();
    return TQ_OK;
  }
  const int es = dtype == TQ_F32 ? 4 : 2;
  if (!x || !codes || !norms) return set_error(TQ_EINVAL, "tq_quantize: NULL x/codes/norms");
  if (p->mode == TQ_MODE_PROD && !rnorms) return set_error(TQ_EINVAL, "tq_quantize: NULL rnorms in product mode");
  if (ld < p->d) return set_error(TQ_EINVAL, "tq_quantize: ld < d");
  if (!aligned(x, 16) || ((ld * es) % 16) != 0 || ((p->d * es) % 16) != 0)
    return set_error(TQ_EINVAL, "tq_quantize: x, ld*elem and d*elem must be 16-byte aligned");
  if (!aligned(codes, 16)) return set_error(TQ_EINVAL, "tq_quantize: codes must be 16-byte aligned");
  if (!aligned(norms, 2) || (rnorms && !aligned(rnorms, 2))) return set_error(TQ_EINVAL, "tq_quantize: norms misaligned");
  const int kb = index_bits(p);
  QArgs a;
  a.x = static_cast<const uint8_t*>(x);
  a.n_vec = n_vec;
  a.n_pad = (n_vec + 31) / 32 * 32;
  a.ld_bytes = ld * es;
  a.d = p->d;
  a.m = p->mode == TQ_MODE_PROD ? p->m : 0;
  a.row_bytes = p->d * es;
  a.nbuf = 2;
  a.codes = static_cast<uint8_t*>(codes);
  a.norms = norms;
  a.rnorms = rnorms;
  a.cent = p->centroids;
  a.thr = p->thresholds;
  a.D = p->signs_D;
  a.S = p->S;
  const bool prod = p->mode == TQ_MODE_PROD;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (p->layout == TQ_LAYOUT_SLICED && !quantize_rt_supported(p, dtype))
    return set_error(TQ_EUNSUPPORTED, "tq_quantize: the token-sliced layout needs d_pad 128 and 16-bit input");
  if (quantize_rt_supported(p, dtype)) {
    rc = launch_quantize_rt(p, x, dtype, n_vec, ld * es, codes, norms, rnorms, sm_count(), st);
    if (rc == TQ_OK) clear_error();
    return rc;
  }
  if (quantize128_supported(p, dtype)) {
    rc = launch_quantize128(p, x, dtype, n_vec, ld * es, codes, norms, rnorms, sm_count(), st);
    if (rc == TQ_OK) clear_error();
    return rc;
  }
  rc = (p->d_pad == 128) ? dispatch_kb<128>(kb, prod, dtype, a, sm_count(), st)
                         : dispatch_kb<256>(kb, prod, dtype, a, sm_count(), st);
  if (rc == TQ_OK) clear_error();
  return rc;
}
