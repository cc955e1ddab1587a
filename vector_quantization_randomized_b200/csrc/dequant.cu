// tq_dequantize: the reconstruction x_hat = Q^-1(codes) ("TurboQuant explainer"
// (m.163.com), "第二步：QJL": the QJL part is sqrt(pi/2)/m * gamma * S^T sigma,
// sigma = 2s - 1, so that E[<y, Q^-1(Q(x))>] = <y, x>):
//   x_hat = n * D H (c[idx] + sqrt(pi/2)/m * gamma * S^T sigma) / sqrt(d_pad),
// first d coordinates (MSE mode: no QJL term).  <q, x_hat> is exactly the logit
// estimate of tq_logits for every q, since that estimate is linear in the key.
//
// One warp per vector; lane l holds coordinates NI*l .. NI*l + NI - 1 (NI = 4 at
// d_pad 128, 8 at 256): the code words are warp-uniform loads, the centroid
// lookup is a shuffle from the lane that holds c[idx], S^T sigma accumulates
// S rows staged once per CTA in shared memory (each lane reads its NI
// consecutive fp16 entries of a row in one load), the inverse rotation takes
// log2(NI) in-register Walsh-Hadamard stages and five shuffle stages, and the
// output row is written by the warp as one contiguous run.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>

#include "common.h"
#include "device.cuh"
#include "prep.h"

namespace {
using namespace tqd;

struct QArgs {
  const uint8_t* codes;
  const uint16_t* norms;
  const uint16_t* rnorms;
  const float* cent;
  const int8_t* D;
  const uint16_t* S;
  int64_t n_vec, ld;
  int d, m, tb;
  int sliced;   // token-sliced layout (MSE codes): plane p of a tile = DP words, word j bit t
  float kappa;  // sqrt(pi/2) / m
  float* out;
};

template <int DP, int KB, bool PROD>
__global__ void __launch_bounds__(256) dequant_kernel(const QArgs a) {
  constexpr int NI = DP / 32;          // coordinates per lane
  extern __shared__ __align__(16) uint8_t smem[];
  const __half* Ss = reinterpret_cast<const __half*>(smem);  // [m][DP]
  const int lane = threadIdx.x & 31;
  if constexpr (PROD) {
    for (int e = threadIdx.x; e < a.m * DP / 8; e += blockDim.x)
      reinterpret_cast<uint4*>(smem)[e] = __ldg(reinterpret_cast<const uint4*>(a.S) + e);
    __syncthreads();
  }
  const float cent_lane = lane < (1 << KB) ? a.cent[lane] : 0.f;
  float dsign[NI];
#pragma unroll
  for (int k = 0; k < NI; ++k) dsign[k] = (float)a.D[NI * lane + k];
  const float rs = rsqrtf((float)DP);
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t v = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); v < a.n_vec; v += warps) {
    const uint8_t* tile = a.codes + (v >> 5) * a.tb;
    const int slot = (int)(v & 31);
    // index bits of this lane's coordinates: word NI*lane/32, bits (NI*lane) % 32 ..
    const int wsel = (NI * lane) >> 5, sh = (NI * lane) & 31;
    int idx[NI] = {};
    if (!PROD && a.sliced) {  // words NI*lane .. of each plane, bit `slot`
#pragma unroll
      for (int p = 0; p < KB; ++p) {
        const uint32_t* wp = reinterpret_cast<const uint32_t*>(tile + p * (DP * 4)) + NI * lane;
#pragma unroll
        for (int k = 0; k < NI; ++k) idx[k] |= (int)((__ldg(wp + k) >> slot) & 1u) << p;
      }
    } else {
#pragma unroll
      for (int p = 0; p < KB; ++p) {
        const uint32_t w = __ldg(reinterpret_cast<const uint32_t*>(tile + p * TILE * (DP / 8) + slot * (DP / 8)) + wsel);
#pragma unroll
        for (int k = 0; k < NI; ++k) idx[k] |= (int)((w >> (sh + k)) & 1u) << p;
      }
    }
    float y[NI];
#pragma unroll
    for (int k = 0; k < NI; ++k) y[k] = __shfl_sync(FULL, cent_lane, idx[k]);
    if constexpr (PROD) {
      // S^T sigma for this lane's coordinates; sigma_i = +1 where sign bit i is set
      const uint32_t* sw = reinterpret_cast<const uint32_t*>(tile + KB * TILE * (DP / 8) + slot * (a.m / 8));
      float acc[NI] = {};
      for (int w32 = 0; w32 < a.m / 32; ++w32) {
        const uint32_t bits = __ldg(sw + w32);
#pragma unroll 4
        for (int j = 0; j < 32; ++j) {
          const int i = 32 * w32 + j;
          const uint32_t flip = ((bits >> j) & 1u) ? 0u : 0x80008000u;  // -S_i where sigma_i = -1
          const __half* row = Ss + (size_t)i * DP + NI * lane;
#pragma unroll
          for (int h = 0; h < NI / 4; ++h) {
            const uint2 sv = *reinterpret_cast<const uint2*>(row + 4 * h);
            const uint32_t s0 = sv.x ^ flip, s1 = sv.y ^ flip;
            const float2 f0 = __half22float2(*reinterpret_cast<const __half2*>(&s0));
            const float2 f1 = __half22float2(*reinterpret_cast<const __half2*>(&s1));
            acc[4 * h + 0] += f0.x;
            acc[4 * h + 1] += f0.y;
            acc[4 * h + 2] += f1.x;
            acc[4 * h + 3] += f1.y;
          }
        }
      }
      const float g = __half2float(__ushort_as_half(__ldg(a.rnorms + v))) * a.kappa;
#pragma unroll
      for (int k = 0; k < NI; ++k) y[k] = fmaf(g, acc[k], y[k]);
    }
    // inverse rotation D H y / sqrt(DP): stages on the in-lane bits, then on the lane bits
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
    const float nrm = __half2float(__ushort_as_half(__ldg(a.norms + v))) * rs;
    float* orow = a.out + v * a.ld;
#pragma unroll
    for (int k = 0; k < NI; ++k) {
      const int c = NI * lane + k;
      if (c < a.d) orow[c] = y[k] * nrm * dsign[k];
    }
  }
}

template <int DP, int KB, bool PROD>
int launch_dq(const QArgs& a, cudaStream_t st) {
  const int smem = PROD ? a.m * DP * 2 : 0;
  auto kern = dequant_kernel<DP, KB, PROD>;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return tq::set_error(TQ_ECUDA, "tq_dequantize: %s", cudaGetErrorString(e));
  }
  const int blocks = (int)std::max<int64_t>(1, std::min<int64_t>((a.n_vec + 7) / 8, (int64_t)tq::sm_count() * 8));
  kern<<<blocks, 256, smem, st>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return tq::set_error(TQ_ECUDA, "tq_dequantize: launch failed: %s", cudaGetErrorString(e));
  return TQ_OK;
}

template <int DP, bool PROD>
int dispatch_kb(int kb, const QArgs& a, cudaStream_t st) {
  switch (kb) {
    case 1: return launch_dq<DP, 1, PROD>(a, st);
    case 2: return launch_dq<DP, 2, PROD>(a, st);
    case 3: return launch_dq<DP, 3, PROD>(a, st);
    default: return launch_dq<DP, 4, PROD>(a, st);
  }
}

}  // namespace

extern "C" int tq_dequantize(const tq_params* p, const void* codes, const uint16_t* norms, const uint16_t* rnorms,
                             int64_t n_vec, float* out, int64_t ld, tq_stream_t stream) {
  using namespace tq;
  int rc = check_params(p, "tq_dequantize");
  if (rc) return rc;
  const bool prod = p->mode == TQ_MODE_PROD;
  if (n_vec < 0) return set_error(TQ_EINVAL, "tq_dequantize: n_vec < 0");
  if (n_vec == 0) {
    clear_error();
    return TQ_OK;
  }
  if (!codes || !norms || !out || (prod && !rnorms)) return set_error(TQ_EINVAL, "tq_dequantize: NULL pointer argument");
  if (ld < p->d) return set_error(TQ_EINVAL, "tq_dequantize: ld (%lld) < d (%d)", (long long)ld, p->d);
  if (!aligned(codes, 16) || !aligned(out, 4)) return set_error(TQ_EINVAL, "tq_dequantize: misaligned pointer");
  const int kb = index_bits(p);
  QArgs a;
  a.codes = static_cast<const uint8_t*>(codes);
  a.norms = norms;
  a.rnorms = rnorms;
  a.cent = p->centroids;
  a.D = p->signs_D;
  a.S = p->S;
  a.n_vec = n_vec;
  a.ld = ld;
  a.d = p->d;
  a.m = prod ? p->m : 0;
  a.tb = tqd::tile_bytes(p->d_pad, kb, a.m);
  a.sliced = p->layout == TQ_LAYOUT_SLICED;
  a.kappa = prod ? (float)(std::sqrt(M_PI / 2.0) / p->m) : 0.f;
  a.out = out;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (p->d_pad == 128)
    rc = prod ? dispatch_kb<128, true>(kb, a, st) : dispatch_kb<128, false>(kb, a, st);
  else
    rc = prod ? dispatch_kb<256, true>(kb, a, st) : dispatch_kb<256, false>(kb, a, st);
  if (rc == TQ_OK) clear_error();
  return rc;
}
