// Query preparation for the code scans (tq_logits, tq_decode_attn,
// tq_search_topk): rotated query q_rot = H D q / sqrt(d_pad), projection
// u = S q_rot ("TurboQuant explainer" (m.163.com), "第二步：QJL"), the Walsh
// weights of the odd-symmetric codebook, integer scaling and the int8 digit
// split laid out as mma.sync A fragments (see scan.cuh).
#include <cuda_runtime.h>

#include "common.h"
#include "prep.h"
#include "scan.cuh"

namespace {
using namespace tqd;

__global__ void __launch_bounds__(256) qprep_kernel(const PrepArgs a) {
  __shared__ float qt[QCHUNK][256];
  __shared__ float uu[QCHUNK][256];
  __shared__ int W[QCHUNK][4][256];
  __shared__ int V[QCHUNK][256];
  __shared__ float alpha[4];
  __shared__ float qstat[QCHUNK][2];  // sum q_rot, max |q_rot|
  __shared__ int FG[QCHUNK][2];
  // the scan kernel may be scheduled now; it waits for this grid before reading the output
  asm volatile("griddepcontrol.launch_dependents;\n" ::);
  const int chunk = blockIdx.x;
  const int outer = chunk / a.nqc, qc = chunk % a.nqc;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int NT = walsh_planes(a.kb);
  const int L = 1 << a.kb;
  const int NI = a.dp / 32;

  if (threadIdx.x < NT) {  // Walsh coefficients of the odd-symmetric codebook (fp64)
    const int mask = walsh_mask(a.kb, threadIdx.x);
    double s = 0.0;
    for (int l = 0; l < L; ++l) s += (double)a.cent[l] * ((__popc(l & mask) & 1) ? 1.0 : -1.0);
    alpha[threadIdx.x] = (float)(s / L);
  }
  if (warp < QCHUNK) {  // q_rot = H D q / sqrt(dp); warp = query, lane holds coordinates lane + 32 i
    const int qi = warp;
    const bool valid = QCHUNK * qc + qi < a.group;
    const int64_t row = (int64_t)outer * a.group + QCHUNK * qc + qi;
    float y[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int j = 32 * i + lane;
      float x = 0.f;
      if (i < NI && valid && j < a.d) x = a.q[row * a.d + j];
      y[i] = (i < NI) ? x * (float)a.D[j] : 0.f;
    }
#pragma unroll
    for (int h = 1; h < 8; h <<= 1)
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if ((i & h) == 0) {
          float u = y[i], w = y[i + h];
          y[i] = u + w;
          y[i + h] = u - w;
        }
#pragma unroll
    for (int sft = 1; sft < 32; sft <<= 1)
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float o = __shfl_xor_sync(FULL, y[i], sft);
        y[i] = (lane & sft) ? (o - y[i]) : (y[i] + o);
      }
    const float rs = rsqrtf((float)a.dp);
    float sq = 0.f, mq = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (i < NI) {
        const float v = y[i] * rs;
        qt[qi][32 * i + lane] = v;
        sq += v;
        mq = fmaxf(mq, fabsf(v));
      }
    }
    sq = warp_sum(sq);
    mq = warp_max(mq);
    if (lane == 0) {
      qstat[qi][0] = sq;
      qstat[qi][1] = mq;
    }
  }
  __syncthreads();
  // u = S q_rot: thread i owns projection row i for all four queries
  for (int i = threadIdx.x; i < a.m; i += blockDim.x) {
    float acc[QCHUNK] = {0.f, 0.f, 0.f, 0.f};
    const uint4* srow = reinterpret_cast<const uint4*>(a.S + (size_t)i * a.dp);
    for (int k = 0; k < a.dp / 8; ++k) {
      const uint4 v = __ldg(srow + k);
      const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&wv[e]));
#pragma unroll
        for (int qq = 0; qq < QCHUNK; ++qq) {
          acc[qq] = fmaf(f.x, qt[qq][8 * k + 2 * e], acc[qq]);
          acc[qq] = fmaf(f.y, qt[qq][8 * k + 2 * e + 1], acc[qq]);
        }
      }
    }
#pragma unroll
    for (int qq = 0; qq < QCHUNK; ++qq) uu[qq][i] = acc[qq];
  }
  __syncthreads();
  if (warp < QCHUNK) {  // scales: weights 2 alpha q_rot and 2 u become integers below 2^23
    const int qi = warp;
    float su = 0.f, mu = 0.f;
    for (int i = lane; i < a.m; i += 32) {
      su += uu[qi][i];
      mu = fmaxf(mu, fabsf(uu[qi][i]));
    }
    su = warp_sum(su);
    mu = warp_max(mu);
    float amax = 0.f;
    for (int T = 0; T < NT; ++T) amax = fmaxf(amax, fabsf(alpha[T]));
    int F = 0, G = 0;
    const float mc = 2.f * amax * qstat[qi][1], ms = 2.f * mu;
    if (mc > 0.f) {
      int e;
      frexpf(mc, &e);
      F = 23 - e;
    }
    if (ms > 0.f) {
      int e;
      frexpf(ms, &e);
      G = 23 - e;
    }
    if (lane == 0) {
      FG[qi][0] = F;
      FG[qi][1] = G;
      float4* scal = reinterpret_cast<float4*>(a.out + (int64_t)chunk * prep_chunk_bytes(a.fr) + (int64_t)a.fr * 128);
      // sum_T alpha_T = c[L-1] (all index bits set)
      scal[qi] = make_float4(ldexpf(1.f, -(F + 7)), a.cent[L - 1] * qstat[qi][0], ldexpf(1.f, -(G + 7)), su);
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < QCHUNK * NT * a.dp; e += blockDim.x) {
    const int qq = e / (NT * a.dp), r = e % (NT * a.dp), T = r / a.dp, j = r % a.dp;
    W[qq][T][j] = __float2int_rn(ldexpf(2.f * alpha[T] * qt[qq][j], FG[qq][0]));
  }
  for (int e = threadIdx.x; e < QCHUNK * a.m; e += blockDim.x) {
    const int qq = e / a.m, i = e % a.m;
    V[qq][i] = __float2int_rn(ldexpf(2.f * uu[qq][i], FG[qq][1]));
  }
  __syncthreads();

  // A fragments (layout in scan.cuh)
  const ScanShape sh(a.dp, a.kb, a.m);
  const int NH = a.dp / 128;
  uint32_t* frag = reinterpret_cast<uint32_t*>(a.out + (int64_t)chunk * prep_chunk_bytes(a.fr));
  for (int widx = threadIdx.x; widx < 32 * a.fr; widx += blockDim.x) {
    const int L2 = widx & 31, w = widx >> 5;
    uint32_t word = 0u;
    if (w < 8 * sh.per_c) {
      const int c = w / sh.per_c, o = w % sh.per_c;
      const int g = L2 >> 2, t = L2 & 3;
      int reg, item;
      bool sign;
      if (o < 4 * sh.ncp) {
        sign = false;
        reg = o & 3;
        item = 2 * (o >> 2) + (reg >= 2 ? 1 : 0);
      } else if (o < 4 * sh.ncp + 2 * sh.ncs) {
        sign = false;
        reg = o - 4 * sh.ncp;
        item = sh.nci - 1;
      } else if (o < 4 * sh.ncp + 2 * sh.ncs + 4 * sh.nsp) {
        sign = true;
        reg = (o - 4 * sh.ncp - 2 * sh.ncs) & 3;
        item = reg >= 2 ? 1 : 0;
      } else {
        sign = true;
        reg = o - 4 * sh.ncp - 2 * sh.ncs - 4 * sh.nsp;
        item = 0;
      }
      const int r = (reg & 1) ? g + 8 : g;
      const int digit = r >> 2, qq = r & 3;
      for (int jj = 0; jj < 4; ++jj) {
        int X = 0;
        if (sign) {
          const int wi = t + 4 * item;
          const int j = 32 * wi + c + 8 * jj;
          X = (j < a.m) ? V[qq][j] : 0;
        } else {
          const int T = item / NH, hh = item % NH;
          const int wi = t + 4 * hh;
          X = W[qq][T][32 * wi + c + 8 * jj];
        }
        X *= (1 << (7 - c));
        int dv[4];  // balanced base-256 digits
        for (int k = 0; k < 3; ++k) {
          const int lowb = (int)(int8_t)(X & 0xFF);
          dv[k] = lowb;
          X = (X - lowb) >> 8;
        }
        dv[3] = X;
        word |= ((uint32_t)(uint8_t)(int8_t)dv[digit]) << (8 * jj);
      }
    }
    frag[((int64_t)(w >> 2) * 32 + L2) * 4 + (w & 3)] = word;
  }
}

}  // namespace

namespace tq {

int launch_prep(const tqd::PrepArgs& a, cudaStream_t st) {
  const int chunks = a.n_outer * a.nqc;
  if (chunks <= 0) return TQ_OK;
  qprep_kernel<<<chunks, 256, 0, st>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(TQ_ECUDA, "query prep launch failed: %s", cudaGetErrorString(e));
  return TQ_OK;
}

}  // namespace tq
