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
        float4* scal;
        // sum_T alpha_T = c[L-1] (all index bits set)
        const int64_t cb = a.layout ? prep_chunk_bytes_tc(a.kc) : prep_chunk_bytes(a.fr);
        const int64_t sc_off = a.layout ? (int64_t)a.kc * 512 : (int64_t)a.fr * 128;
        scal = reinterpret_cast<float4*>(a.out + (int64_t)chunk * cb + sc_off);
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

  if (a.layout == 1) {  // tcgen05 B image (layout in scan.cuh); this CTA writes every PREP_SPLIT-th word
    const int NTc = NT;
    uint32_t* img = reinterpret_cast<uint32_t*>(a.out + (int64_t)chunk * prep_chunk_bytes_tc(a.kc));
    const int words = 128 * a.kc;
    for (int widx = threadIdx.x * PREP_SPLIT + part; widx < words; widx += blockDim.x * PREP_SPLIT) {
      const int o = 4 * widx;
      const int qq = o / (a.kc * 128), rem = o % (a.kc * 128);
      const int kc = rem >> 7, r = (rem >> 4) & 7, e0 = rem & 15;
      const int c = kc & 7, P = kc >> 3;
      uint32_t word = 0u;
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const int j = 32 * (e0 >> 2) + 8 * b + c;
        int8_t v = 0;
        if (P < NTc) {
          if (r < 4) v = dw[r][qq][P][j];
        } else if (r >= 4) {
          v = ds[r - 4][qq][j];
        }
        word |= (uint32_t)(uint8_t)v << (8 * b);
      }
      img[widx] = word;
    }
    return;
  }
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

// frexpf's exponent (x = f 2^e, 0.5 <= f < 1) and ldexpf(1, k), read from / written
// into the fp32 bit pattern for normal values (exact), the library calls otherwise.
__device__ __forceinline__ int frexp_exponent(float x) {
  const uint32_t b = __float_as_uint(x) & 0x7FFFFFFFu;
  if (b >= 0x00800000u && b < 0x7F800000u) return (int)(b >> 23) - 126;
  int e;
  frexpf(x, &e);
  return e;
}
__device__ __forceinline__ float pow2f(int k) {
  return (k >= -126 && k <= 127) ? __uint_as_float((uint32_t)(127 + k) << 23) : ldexpf(1.f, k);
}

// Query prep for the tensor-memory scan (d_pad 128): one CTA of 512 threads per
// chunk of 4 queries writes the B image of layout 1 (scan.cuh) and the per-query
// scalars.  Same integer weights as qprep_kernel: X = round(2 alpha_T q_rot_j 2^F)
// 2^(7-c) and round(2 u_i 2^G) 2^(7-c), split into balanced base-256 digits.
// The kernel is a chain of short phases, each a memory latency or a dependent
// arithmetic chain, so every phase keeps its shared-memory reads broadcast and
// its stores whole: S rows are fetched first (their latency overlaps the query
// rotation); u takes one row per thread in four coordinate quarters; the image is
// written as whole 16-byte rows, one thread per (query, plane, bit class).
__global__ void __launch_bounds__(512) qprep_tc_kernel(const PrepArgs a) {
  constexpr int DP = 128;
  __shared__ float4 qT[DP];            // q_rot of the 4 queries, per coordinate
  __shared__ float4 upart[4][DP];      // u partial sums per coordinate quarter
  __shared__ float4 uT[DP];            // u = S q_rot, per row
  __shared__ float alpha[4];
  __shared__ float cent_s[16];
  __shared__ float qstat[QCHUNK][2];   // sum q_rot, max |q_rot|
  __shared__ float FGs[QCHUNK][2];     // 2^F, 2^G
  asm volatile("griddepcontrol.launch_dependents;\n" ::);
  const int chunk = blockIdx.x;
  const int outer = chunk / a.nqc, qc = chunk % a.nqc;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int NT = walsh_planes(a.kb), NP = NT + (a.m > 0 ? 1 : 0), KC = a.kc;
  const int L = 1 << a.kb;
  float* qTf = reinterpret_cast<float*>(qT);
  float* uTf = reinterpret_cast<float*>(uT);

  // S row si, coordinates 32 sq .. 32 sq + 31, fetched before anything else
  const int si = tid & (DP - 1), sq = tid >> 7;
  uint4 sv[4] = {};
  if (si < a.m) {
    const uint4* srow = reinterpret_cast<const uint4*>(a.S + (size_t)si * DP) + 4 * sq;
#pragma unroll
    for (int k = 0; k < 4; ++k) sv[k] = __ldg(srow + k);
  }
  // the centroid load stays in flight while the query warps rotate
  const float cent_r = tid < L ? __ldg(a.cent + tid) : 0.f;
  if (warp < QCHUNK) {  // q_rot = H D q / sqrt(128): warp = query, lane holds coordinates lane + 32 i
    const int qi = warp;
    const bool valid = QCHUNK * qc + qi < a.group;
    const int64_t row = (int64_t)outer * a.group + QCHUNK * qc + qi;
    float y[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int j = 32 * i + lane;
      y[i] = (valid && j < a.d) ? __ldg(a.q + row * a.d + j) * (float)__ldg(a.D + j) : 0.f;
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
      qTf[4 * (32 * i + lane) + qi] = v;
      sum += v;
      mx = fmaxf(mx, fabsf(v));
    }
    sum = warp_sum(sum);
    mx = warp_max(mx);
    if (lane == 0) {
      qstat[qi][0] = sum;
      qstat[qi][1] = mx;
    }
  }
  if (tid < L) cent_s[tid] = cent_r;
  __syncthreads();
  if (tid < NT) {  // Walsh coefficients of the odd-symmetric codebook (fp64)
    const int mask = walsh_mask(a.kb, tid);
    double sum = 0.0;
    for (int l = 0; l < L; ++l) sum += (double)cent_s[l] * ((__popc(l & mask) & 1) ? 1.0 : -1.0);
    alpha[tid] = (float)(sum / L);
  }
  if (a.m > 0) {  // partial u over one coordinate quarter: a warp = 32 rows, same coordinates (broadcast)
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f), acc2 = acc;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint32_t wv[4] = {sv[k].x, sv[k].y, sv[k].z, sv[k].w};
#pragma unroll
      for (int h2 = 0; h2 < 4; ++h2) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&wv[h2]));
        const int j = 32 * sq + 8 * k + 2 * h2;
        const float4 q0 = qT[j], q1 = qT[j + 1];
        acc.x = fmaf(f.x, q0.x, acc.x);
        acc.y = fmaf(f.x, q0.y, acc.y);
        acc.z = fmaf(f.x, q0.z, acc.z);
        acc.w = fmaf(f.x, q0.w, acc.w);
        acc2.x = fmaf(f.y, q1.x, acc2.x);
        acc2.y = fmaf(f.y, q1.y, acc2.y);
        acc2.z = fmaf(f.y, q1.z, acc2.z);
        acc2.w = fmaf(f.y, q1.w, acc2.w);
      }
    }
    upart[sq][si] = make_float4(acc.x + acc2.x, acc.y + acc2.y, acc.z + acc2.z, acc.w + acc2.w);
    __syncthreads();
    if (tid < DP) {
      const float4 p0 = upart[0][tid], p1 = upart[1][tid], p2 = upart[2][tid], p3 = upart[3][tid];
      uT[tid] = make_float4((p0.x + p1.x) + (p2.x + p3.x), (p0.y + p1.y) + (p2.y + p3.y),
                            (p0.z + p1.z) + (p2.z + p3.z), (p0.w + p1.w) + (p2.w + p3.w));
    }
  }
  __syncthreads();
  if (warp < QCHUNK) {  // scales: weights 2 alpha q_rot and 2 u become integers below 2^23
    const int qi = warp;
    float su = 0.f, mu = 0.f;
    for (int i = lane; i < a.m; i += 32) {
      const float v = uTf[4 * i + qi];
      su += v;
      mu = fmaxf(mu, fabsf(v));
    }
    su = warp_sum(su);
    mu = warp_max(mu);
    float amax = 0.f;
    for (int T = 0; T < NT; ++T) amax = fmaxf(amax, fabsf(alpha[T]));
    const float mc = 2.f * amax * qstat[qi][1], ms = 2.f * mu;
    const int F = mc > 0.f ? 23 - frexp_exponent(mc) : 0;
    const int G = ms > 0.f ? 23 - frexp_exponent(ms) : 0;
    if (lane == 0) {
      FGs[qi][0] = pow2f(F);
      FGs[qi][1] = pow2f(G);
      float4* scal = reinterpret_cast<float4*>(a.out + (int64_t)chunk * prep_chunk_bytes_tc(KC) + (int64_t)KC * 512);
      // sum_T alpha_T = c[L-1] (all index bits set)
      scal[qi] = make_float4(pow2f(-(F + 7)), cent_s[L - 1] * qstat[qi][0], pow2f(-(G + 7)), su);
    }
  }
  __syncthreads();
  // B image words, one thread per (query q, plane P, bit class c, word w): the 4
  // weights of coordinates 32w + 8b + c (bytes 4w + b of K chunk 8P + c) give word
  // w of the 4 digit rows 8q + r0 + d (r0 = 0 centroid, 4 sign); the same word of
  // the chunk's other 4 rows is zero.  Scaling by the power of two 2^F (2^G) is
  // exact, as in ldexpf.
  for (int e = tid; e < QCHUNK * NP * 32; e += 512) {
    const int w = e & 3, c = (e >> 2) & 7, pq = e >> 5;
    const int q = pq / NP, P = pq - q * NP;
    const bool cen = P < NT;
    const float scale = cen ? 2.f * alpha[P] * FGs[q][0] : 2.f * FGs[q][1];
    const float* src = cen ? qTf : uTf;
    uint32_t W[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int j = 32 * w + 8 * b + c;
      int X = (cen || j < a.m) ? __float2int_rn(src[4 * j + q] * scale) * (1 << (7 - c)) : 0;
#pragma unroll
      for (int d = 0; d < 3; ++d) {
        const int lowb = (int)(int8_t)(X & 0xFF);
        W[d] |= (uint32_t)(uint8_t)lowb << (8 * b);
        X = (X - lowb) >> 8;
      }
      W[3] |= (uint32_t)(uint8_t)X << (8 * b);
    }
    uint32_t* dst = reinterpret_cast<uint32_t*>(a.out + (int64_t)chunk * prep_chunk_bytes_tc(KC) + q * (KC * 128) +
                                                (8 * P + c) * 128) + w;
    const int r0 = cen ? 0 : 4;
#pragma unroll
    for (int d = 0; d < 4; ++d) {
      dst[4 * (r0 + d)] = W[d];
      dst[4 * ((r0 ^ 4) + d)] = 0u;
    }
  }
}

}  // namespace

namespace tq {

int launch_prep(const tqd::PrepArgs& a, cudaStream_t st) {
  const int chunks = a.n_outer * a.nqc;
  if (chunks <= 0) return TQ_OK;
  if (a.layout == 1) {
    if (a.dp != 128 || a.kc > 40) return set_error(TQ_EUNSUPPORTED, "query prep: tensor-memory layout needs d_pad 128");
    qprep_tc_kernel<<<chunks, 512, 0, st>>>(a);
  } else {
    qprep_kernel<<<chunks * PREP_SPLIT, 256, 0, st>>>(a);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(TQ_ECUDA, "query prep launch failed: %s", cudaGetErrorString(e));
  return TQ_OK;
}

}  // namespace tq
