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

constexpr int PREP_SPLIT = 4;  // CTAs per chunk (each writes a quarter of the fragment words)

__global__ void __launch_bounds__(256) qprep_kernel(const PrepArgs a) {
  __shared__ float qt[QCHUNK][256];
  __shared__ float uu[QCHUNK][256];
  // int8 digits of the shifted integer weights: dw[digit][query][plane][coordinate], ds[digit][query][row]
  __shared__ int8_t dw[4][QCHUNK][4][256];
  __shared__ int8_t ds[4][QCHUNK][256];
  __shared__ float alpha[4];
  __shared__ float cent_s[16];
  __shared__ float qstat[QCHUNK][2];  // sum q_rot, max |q_rot|
  __shared__ int FG[QCHUNK][2];
  // the scan kernel may be scheduled now; it waits for this grid before reading the output
  asm volatile("griddepcontrol.launch_dependents;\n" ::);
  const int chunk = blockIdx.x / PREP_SPLIT, part = blockIdx.x % PREP_SPLIT;
  const int outer = chunk / a.nqc, qc = chunk % a.nqc;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int NT = walsh_planes(a.kb);
  const int L = 1 << a.kb;
  const int NI = a.dp / 32;

  if (threadIdx.x < L) cent_s[threadIdx.x] = a.cent[threadIdx.x];  // one load per thread, all in flight
  __syncthreads();
  if (threadIdx.x < NT) {  // Walsh coefficients of the odd-symmetric codebook (fp64)
    const int mask = walsh_mask(a.kb, threadIdx.x);
    double s = 0.0;
    for (int l = 0; l < L; ++l) s += (double)cent_s[l] * ((__popc(l & mask) & 1) ? 1.0 : -1.0);
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
  // u = S q_rot: thread (row i, query pair) -- 2 x 128 FMA per thread for m <= 128
  for (int e = threadIdx.x; e < 2 * a.m; e += blockDim.x) {
    const int i = e % a.m, qp = e / a.m;  // queries 2qp, 2qp+1
    float acc0 = 0.f, acc1 = 0.f;
    const uint4* srow = reinterpret_cast<const uint4*>(a.S + (size_t)i * a.dp);
    const float* q0 = qt[2 * qp];
    const float* q1 = qt[2 * qp + 1];
    for (int k0 = 0; k0 < a.dp / 8; k0 += 16) {  // 16 row loads in flight, then their FMAs
      uint4 v[16];
#pragma unroll
      for (int kk = 0; kk < 16; ++kk) v[kk] = (k0 + kk < a.dp / 8) ? __ldg(srow + k0 + kk) : make_uint4(0, 0, 0, 0);
#pragma unroll
      for (int kk = 0; kk < 16; ++kk) {
        const int k = min(k0 + kk, a.dp / 8 - 1);  // rows past d_pad carry zeros
        const uint32_t wv[4] = {v[kk].x, v[kk].y, v[kk].z, v[kk].w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&wv[h]));
          acc0 = fmaf(f.x, q0[8 * k + 2 * h], acc0);
          acc0 = fmaf(f.y, q0[8 * k + 2 * h + 1], acc0);
          acc1 = fmaf(f.x, q1[8 * k + 2 * h], acc1);
          acc1 = fmaf(f.y, q1[8 * k + 2 * h + 1], acc1);
        }
      }
    }
    uu[2 * qp][i] = acc0;
    uu[2 * qp + 1][i] = acc1;
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
      if (part == 0) {
        // sum_T alpha_T = c[L-1] (all index bits set)
        float4* scal = reinterpret_cast<float4*>(a.out + (int64_t)chunk * prep_chunk_bytes(a.fr) + (int64_t)a.fr * 128);
        scal[qi] = make_float4(ldexpf(1.f, -(F + 7)), cent_s[L - 1] * qstat[qi][0], ldexpf(1.f, -(G + 7)), su);
      }
    }
  }
  __syncthreads();
  // Each weight is used with one bit class only (c = coordinate % 8): shift by 7-c once and
  // split into balanced base-256 digits.
  auto digits = [](int X, int8_t* d0, int stride) {
    for (int k = 0; k < 3; ++k) {
      const int lowb = (int)(int8_t)(X & 0xFF);
      d0[k * stride] = (int8_t)lowb;
      X = (X - lowb) >> 8;
    }
    d0[3 * stride] = (int8_t)X;
  };
  for (int e = threadIdx.x; e < QCHUNK * NT * a.dp; e += blockDim.x) {
    const int qq = e / (NT * a.dp), r = e % (NT * a.dp), T = r / a.dp, j = r % a.dp;
    const int X = __float2int_rn(ldexpf(2.f * alpha[T] * qt[qq][j], FG[qq][0])) * (1 << (7 - (j & 7)));
    digits(X, &dw[0][qq][T][j], QCHUNK * 4 * 256);
  }
  for (int e = threadIdx.x; e < QCHUNK * 256; e += blockDim.x) {
    const int qq = e / 256, i = e % 256;
    const int X = (i < a.m) ? __float2int_rn(ldexpf(2.f * uu[qq][i], FG[qq][1])) * (1 << (7 - (i & 7))) : 0;
    digits(X, &ds[0][qq][i], QCHUNK * 256);
  }
  __syncthreads();

  // A fragments (layout in scan.cuh); this CTA writes words w = part, part + PREP_SPLIT, ...
  const ScanShape sh(a.dp, a.kb, a.m);
  const int NH = a.dp / 128;
  uint32_t* frag = reinterpret_cast<uint32_t*>(a.out + (int64_t)chunk * prep_chunk_bytes(a.fr));
  for (int widx = threadIdx.x; widx < 32 * a.fr / PREP_SPLIT; widx += blockDim.x) {
    const int L2 = widx & 31, w = (widx >> 5) * PREP_SPLIT + part;
    uint32_t word = 0u;
    if (w < sh.fr) {
      const int c = w / sh.per_c, o = w % sh.per_c;
      const int g = L2 >> 2, t = L2 & 3;
      const int slot = o >> 2;
      int reg = o & 3, item = 0;
      bool sign, pad = false;
      if (slot < sh.ncp) {  // centroid k32 pair: a0,a1 -> first item, a2,a3 -> second
        sign = false;
        item = 2 * slot + (reg >= 2 ? 1 : 0);
      } else if (slot < sh.ncp + sh.ncs) {  // centroid k16 single
        sign = false;
        item = sh.nci - 1;
        pad = reg >= 2;
      } else if (slot < sh.ncp + sh.ncs + sh.nsp) {  // sign k32 pair
        sign = true;
        item = reg >= 2 ? 1 : 0;
      } else {  // sign k16 single
        sign = true;
        item = 0;
        pad = reg >= 2;
      }
      if (!pad) {
        const int r = (reg & 1) ? g + 8 : g;
        const int digit = r >> 2, qq = r & 3;
        const int8_t* src;
        if (sign) {
          src = &ds[digit][qq][32 * (t + 4 * item) + c];
        } else {
          const int T = item / NH, hh = item % NH;
          src = &dw[digit][qq][T][32 * (t + 4 * hh) + c];
        }
        word = (uint32_t)(uint8_t)src[0] | ((uint32_t)(uint8_t)src[8] << 8) | ((uint32_t)(uint8_t)src[16] << 16) |
               ((uint32_t)(uint8_t)src[24] << 24);
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
  qprep_kernel<<<chunks * PREP_SPLIT, 256, 0, st>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(TQ_ECUDA, "query prep launch failed: %s", cudaGetErrorString(e));
  return TQ_OK;
}

}  // namespace tq
