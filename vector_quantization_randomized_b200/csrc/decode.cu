// tq_decode_attn: one decode step of attention over compressed K and V
// ("TurboQuant explainer" (m.163.com), "速度": attention from the codes;
// zhidx turboquant_plus article: asymmetric K/V - keys in the product code,
// values MSE-only).
//
//   out[b][h] = sum_t softmax_t(scale * l_t) * v_hat_t,
//   v_hat_t = n_v D H c_v[idx_t] / sqrt(d_pad).
//
// Split-K over tokens ("flash-decoding"): CTA (b, kv head, query chunk,
// token chunk of 256) computes the logits of its 4 query heads with the
// tensor-core code scan (scan.cuh), the chunk's softmax statistics, and the
// value sum in the *rotated* domain, o_rot = sum_t p_t n_v,t c_v[idx_t]
// (the rotation is linear, so it is applied once per output row instead of
// once per token).  A combine kernel merges the chunks (log-sum-exp) and
// applies the inverse rotation D H / sqrt(d_pad).
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>

#include "common.h"
#include "prep.h"
#include "scan.cuh"

namespace {
using namespace tqd;

constexpr int CH = 256;  // tokens per split-K chunk

struct DArgs {
  const uint8_t* kcodes;
  const uint16_t* knorms;
  const uint16_t* krnorms;
  const uint8_t* vcodes;
  const uint16_t* vnorms;
  const int32_t* seq_lens;
  const float* vcent;
  int64_t max_tokens;
  int hkv, group, nqc, nch, km, ktb, vtb, vkb, dp;
  const uint8_t* prep;
  int64_t prep_bytes;
  float* part;  // [b][h][chunk][dp + 2]
  float kappa, sl2;  // sqrt(pi/2)/m, scale*log2(e)
  float veps;        // Sparse V threshold (0: off)
};

// Value weights p_j * n_v,j of token j for the 4 query heads of the chunk.
// Sparse V ("zhidx turboquant_plus article", "Sparse V": skip the value work of
// tokens with negligible attention weight): with veps > 0 the token is dropped
// when p_j < veps * (chunk sum of p) for every query head of the chunk.  The
// chunk-normalised weight bounds the final softmax weight from above (the other
// chunks only add to the denominator), so a dropped token has final weight
// below veps; its weight stays in the normalisation.
__device__ __forceinline__ float4 value_weights(const float (*sl)[CH], const float (*stat)[2], int j, float nv,
                                                float veps, int nq) {
  float4 w = make_float4(sl[0][j] * nv, sl[1][j] * nv, sl[2][j] * nv, sl[3][j] * nv);
  if (veps > 0.f) {
    bool keep = false;
#pragma unroll
    for (int qq = 0; qq < QCHUNK; ++qq) keep |= qq < nq && sl[qq][j] >= veps * stat[qq][1];
    if (!keep) w = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  return w;
}

template <int KB, int SI, int VKB>
__global__ void __launch_bounds__(128) decode_kernel(const DArgs a) {
  constexpr int DP = 128;
  using SC = Scan<DP, KB, SI>;
  constexpr int SW = SI > 0 ? SI : 1;
  __shared__ float sl[QCHUNK][CH];
  __shared__ float4 wv[CH];
  __shared__ float stat[QCHUNK][2];
  __shared__ float vc[16];
  __shared__ uint4 afrag[SC::FR / 4 * 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int chunk_id = blockIdx.x % a.nch;
  const int rest = blockIdx.x / a.nch;
  const int qc = rest % a.nqc;
  const int bg = rest / a.nqc;  // b * hkv + g
  const int b = bg / a.hkv;
  const int L = (int)min((int64_t)a.seq_lens[b], a.max_tokens);
  const int t0 = chunk_id * CH;
  const int ntok = max(0, min(CH, L - t0));
  if (threadIdx.x < (1 << VKB)) vc[threadIdx.x] = a.vcent[threadIdx.x];
  const int64_t vbase = (int64_t)bg * a.max_tokens;

  // 1) logits of the chunk's tokens for the 4 query heads
  grid_dependency_wait();  // query prep (previous grid) complete
  const uint8_t* prep = a.prep + (int64_t)(bg * a.nqc + qc) * a.prep_bytes;
  if (ntok > 0) SC::stage(afrag, prep);
  __syncthreads();
  if (ntok > 0) {
    SC sc;
    sc.load(reinterpret_cast<const uint8_t*>(afrag), lane);
    const int g = lane >> 2, t = lane & 3;
    const float4 qs = reinterpret_cast<const float4*>(prep + SC::FR * 128)[g & 3];
    const int nsub = (ntok + 7) / 8;
    for (int s = warp; s < nsub; s += 4) {
      uint32_t bw[KB][1], sw[SW];
      const int tk = 8 * s + g;
      load_words<DP, KB, SI>(a.kcodes, a.ktb, a.km, vbase + t0 + tk, tk < ntok, t, bw, sw);
      int accC[2][SC::NCSL][4] = {}, accS[2][4] = {}, accF[2][4];
      sc.run(accC, accS, bw, sw);
      SC::fold(accC, accF);
      float c0, c1, z0 = 0.f, z1 = 0.f;
      combine_digits(accF, lane, c0, c1);
      if constexpr (SI > 0) combine_digits(accS, lane, z0, z1);
      if (lane < 16) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int tok = 8 * s + 2 * t + e;
          float val = -INFINITY;
          if (tok < ntok) {
            const int64_t v = vbase + t0 + tok;
            const float n = __half2float(__ushort_as_half(a.knorms[v]));
            float l = fmaf(e ? c1 : c0, qs.x, -qs.y);
            if constexpr (SI > 0) {
              const float gm = __half2float(__ushort_as_half(a.krnorms[v]));
              l = fmaf(gm * a.kappa, fmaf(e ? z1 : z0, qs.z, -qs.w), l);
            }
            val = n * l * a.sl2;
          }
          sl[g][tok] = val;
        }
      }
    }
  }
  __syncthreads();

  // 2) softmax statistics per query (warp q), weights p * n_v
  if (ntok > 0) {
    const int qq = warp;
    float mx = -INFINITY;
    for (int j = lane; j < ntok; j += 32) mx = fmaxf(mx, sl[qq][j]);
    mx = warp_max(mx);
    float sum = 0.f;
    for (int j = lane; j < ntok; j += 32) {
      const float p = exp2f(sl[qq][j] - mx);
      sl[qq][j] = p;
      sum += p;
    }
    sum = warp_sum(sum);
    if (lane == 0) {
      stat[qq][0] = mx;
      stat[qq][1] = sum;
    }
  }
  __syncthreads();
  for (int j = threadIdx.x; j < ntok; j += 128) {
    const float nv = __half2float(__ushort_as_half(a.vnorms[vbase + t0 + j]));
    wv[j] = value_weights(sl, stat, j, nv, a.veps, min(QCHUNK, a.group - QCHUNK * qc));
  }
  __syncthreads();

  // 3) value sum in the rotated domain: thread = coordinate c
  const int c = threadIdx.x;  // DP == blockDim.x
  float acc0 = 0.f, acc1 = 0.f, acc2 = 0.f, acc3 = 0.f;
  const int w = c >> 5, bit = c & 31;
  auto vstep = [&](int j, const float4 ww) {
    const int64_t v = vbase + t0 + j;
    const uint8_t* tbase = a.vcodes + (v >> 5) * a.vtb + (int)(v & 31) * (DP / 8);
    int idx = 0;
#pragma unroll
    for (int p = 0; p < VKB; ++p) {
      const uint32_t word = __ldg(reinterpret_cast<const uint32_t*>(tbase + p * TILE * (DP / 8)) + w);
      idx |= ((word >> bit) & 1u) << p;
    }
    const float cv = vc[idx];
    acc0 = fmaf(ww.x, cv, acc0);
    acc1 = fmaf(ww.y, cv, acc1);
    acc2 = fmaf(ww.z, cv, acc2);
    acc3 = fmaf(ww.w, cv, acc3);
  };
  if (a.veps > 0.f) {  // Sparse V: dropped tokens (all four weights zero) are skipped, uniformly over the CTA
    for (int j = 0; j < ntok; ++j) {
      const float4 ww = wv[j];
      if (ww.x != 0.f || ww.y != 0.f || ww.z != 0.f || ww.w != 0.f) vstep(j, ww);
    }
  } else {
    for (int j = 0; j < ntok; ++j) vstep(j, wv[j]);
  }

  // 4) partials: [b][h][chunk][dp + 2] = (o_rot[0..dp), max (log2 units), sum)
  const int hq0 = (bg % a.hkv) * a.group + QCHUNK * qc;
  const int nq = min(QCHUNK, a.group - QCHUNK * qc);
  const float accs[4] = {acc0, acc1, acc2, acc3};
#pragma unroll
  for (int qq = 0; qq < QCHUNK; ++qq) {
    if (qq < nq) {
      const int64_t h = (int64_t)b * (a.hkv * a.group) + hq0 + qq;
      float* dst = a.part + (h * a.nch + chunk_id) * (DP + 2);
      dst[c] = accs[qq];
      if (c == 0) {
        dst[DP] = ntok > 0 ? stat[qq][0] : -INFINITY;
        dst[DP + 1] = ntok > 0 ? stat[qq][1] : 0.f;
      }
    }
  }
}

// Staged variant (max_tokens a multiple of 32, 16-byte aligned norm arrays): the
// chunk's K and V code tiles and its norms are copied to shared memory with
// cp.async before any compute, so all of a CTA's HBM reads are in flight at
// once; the scan and the value loop then read shared memory only.
template <int KB, int SI, int VKB>
constexpr int staged_smem() {
  return (CH / TILE) * TILE * (KB * 16 + 16 * SI) + (CH / TILE) * TILE * (VKB * 16) + 3 * CH * 2 + QCHUNK * CH * 4;
}

template <int KB, int SI, int VKB>
__global__ void __launch_bounds__(128) decode_staged_kernel(const DArgs a) {
  constexpr int DP = 128;
  using SC = Scan<DP, KB, SI>;
  constexpr int SW = SI > 0 ? SI : 1;
  constexpr int KTB = TILE * (KB * DP / 8 + 16 * SI);  // m == 128 * SI
  constexpr int VTB = TILE * (VKB * DP / 8);
  constexpr int NT = CH / TILE;
  __shared__ float stat[QCHUNK][2];
  __shared__ __half vch[16];
  __shared__ uint4 afrag[SC::FR / 4 * 32];
  // dynamic: K tiles (later reused for the weights), V tiles, norms, scores
  extern __shared__ __align__(16) uint8_t dsm[];
  uint8_t* kbuf = dsm;
  uint8_t* vbuf = dsm + NT * KTB;
  __half (*nbuf)[CH] = reinterpret_cast<__half (*)[CH]>(vbuf + NT * VTB);  // K norms, K residual norms, V norms
  float (*sl)[CH] = reinterpret_cast<float (*)[CH]>(vbuf + NT * VTB + 3 * CH * 2);
  float4* wv = reinterpret_cast<float4*>(kbuf);  // written after the scan no longer reads kbuf
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int chunk_id = blockIdx.x % a.nch;
  const int rest = blockIdx.x / a.nch;
  const int qc = rest % a.nqc;
  const int bg = rest / a.nqc;
  const int b = bg / a.hkv;
  const int L = (int)min((int64_t)a.seq_lens[b], a.max_tokens);
  const int t0 = chunk_id * CH;
  const int ntok = max(0, min(CH, L - t0));
  const int64_t vbase = (int64_t)bg * a.max_tokens;
  if (threadIdx.x < (1 << VKB)) vch[threadIdx.x] = __float2half_rn(a.vcent[threadIdx.x]);

  if (ntok > 0) {  // stage codes and norms (whole tiles; max_tokens % 32 == 0)
    const int ntiles = (ntok + TILE - 1) / TILE;
    const int64_t tile0 = (vbase + t0) / TILE;
    const uint8_t* ks = a.kcodes + tile0 * KTB;
    const uint8_t* vs = a.vcodes + tile0 * VTB;
    for (int e = threadIdx.x; e < ntiles * KTB / 16; e += 128) cp_async16(kbuf + 16 * e, ks + 16 * e);
    for (int e = threadIdx.x; e < ntiles * VTB / 16; e += 128) cp_async16(vbuf + 16 * e, vs + 16 * e);
    const int nch16 = (ntok + 7) / 8;  // 16-byte chunks of 8 norms
    for (int e = threadIdx.x; e < 3 * nch16; e += 128) {
      const int arr = e / nch16, c = e % nch16;
      const uint16_t* src = arr == 0 ? a.knorms : (arr == 1 ? a.krnorms : a.vnorms);
      cp_async16(&nbuf[arr][8 * c], src + vbase + t0 + 8 * c);
    }
  }
  cp_async_commit();
  grid_dependency_wait();  // query prep (previous grid) complete
  const uint8_t* prep = a.prep + (int64_t)(bg * a.nqc + qc) * a.prep_bytes;
  if (ntok > 0) SC::stage(afrag, prep);
  cp_async_wait<0>();
  __syncthreads();

  // 1) logits of the chunk's tokens for the 4 query heads
  if (ntok > 0) {
    SC sc;
    sc.load(reinterpret_cast<const uint8_t*>(afrag), lane);
    const int g = lane >> 2, t = lane & 3;
    const float4 qs = reinterpret_cast<const float4*>(prep + SC::FR * 128)[g & 3];
    const int nsub = (ntok + 7) / 8;
    for (int s = warp; s < nsub; s += 4) {
      const int tk = 8 * s + g;
      const uint8_t* tb = kbuf + (tk >> 5) * KTB;
      const int slot = tk & 31;
      uint32_t bw[KB][1], sw[SW];
#pragma unroll
      for (int p = 0; p < KB; ++p) bw[p][0] = reinterpret_cast<const uint32_t*>(tb + p * TILE * 16 + slot * 16)[t];
#pragma unroll
      for (int i = 0; i < SW; ++i)
        sw[i] = SI ? reinterpret_cast<const uint32_t*>(tb + KB * TILE * 16 + slot * 16 * SI)[t + 4 * i] : 0u;
      int accC[2][SC::NCSL][4] = {}, accS[2][4] = {}, accF[2][4];
      sc.run(accC, accS, bw, sw);
      SC::fold(accC, accF);
      float c0, c1, z0 = 0.f, z1 = 0.f;
      combine_digits(accF, lane, c0, c1);
      if constexpr (SI > 0) combine_digits(accS, lane, z0, z1);
      if (lane < 16) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int tok = 8 * s + 2 * t + e;
          float val = -INFINITY;
          if (tok < ntok) {
            const float n = __half2float(nbuf[0][tok]);
            float l = fmaf(e ? c1 : c0, qs.x, -qs.y);
            if constexpr (SI > 0) {
              const float gm = __half2float(nbuf[1][tok]);
              l = fmaf(gm * a.kappa, fmaf(e ? z1 : z0, qs.z, -qs.w), l);
            }
            val = n * l * a.sl2;
          }
          sl[g][tok] = val;
        }
      }
    }
  }
  __syncthreads();

  // 2) softmax statistics per query (warp q), weights p * n_v
  if (ntok > 0) {
    const int qq = warp;
    float mx = -INFINITY;
    for (int j = lane; j < ntok; j += 32) mx = fmaxf(mx, sl[qq][j]);
    mx = warp_max(mx);
    float sum = 0.f;
    for (int j = lane; j < ntok; j += 32) {
      const float p = exp2f(sl[qq][j] - mx);
      sl[qq][j] = p;
      sum += p;
    }
    sum = warp_sum(sum);
    if (lane == 0) {
      stat[qq][0] = mx;
      stat[qq][1] = sum;
    }
  }
  __syncthreads();
  for (int j = threadIdx.x; j < ntok; j += 128) {
    const float nv = __half2float(nbuf[2][j]);
    wv[j] = value_weights(sl, stat, j, nv, a.veps, min(QCHUNK, a.group - QCHUNK * qc));
  }
  // tokens past ntok up to the next multiple of 16 take part in the last MMA step with weight 0
  // (their codes are staged: whole 32-token tiles)
  for (int j = ntok + threadIdx.x; j < ((ntok + 15) & ~15); j += 128) wv[j] = make_float4(0.f, 0.f, 0.f, 0.f);
  __syncthreads();

  // 3) value sum in the rotated domain on the tensor cores: o_rot[q][c] = sum_t w_{t,q} c[idx_{t,c}]
  //    as mma.sync m16n8k16, A = centroids of 16 coordinates (rows) x 16 tokens in fp16, B = the
  //    weights p n_v of those tokens for the query heads (columns; 4 of 8 used) in fp16, fp32
  //    accumulation.  Block j covers coordinates 16j .. 16j + 15, so thread (g, t4) needs
  //    coordinates 32w + g + 8k of each token: one shift and mask per plane word gives their
  //    index bits, one byte each.  Warp wp takes the 16-token steps wp, wp + 4, ...
  const int g = lane >> 2, t4 = lane & 3;
  float acc[8][4] = {};
  const float* wf = reinterpret_cast<const float*>(wv);
  const int nstep = (ntok + 15) >> 4;
  for (int st = warp; st < nstep; st += 4) {
    const int tb0 = 16 * st + 2 * t4;  // this thread's tokens: tb0, tb0 + 1, tb0 + 8, tb0 + 9
    uint32_t b0 = 0u, b1 = 0u;
    if (g < QCHUNK) {
      b0 = pack_half2(wf[4 * tb0 + g], wf[4 * (tb0 + 1) + g]);
      b1 = pack_half2(wf[4 * (tb0 + 8) + g], wf[4 * (tb0 + 9) + g]);
    }
    if (a.veps > 0.f && __all_sync(FULL, (b0 | b1) == 0u)) continue;  // Sparse V: every weight dropped
    uint32_t ib[4][4];  // [token][word]: byte k = index of coordinate 32 word + g + 8k
#pragma unroll
    for (int tk = 0; tk < 4; ++tk) {
      const int tok = tb0 + (tk & 1) + 8 * (tk >> 1);
      const uint8_t* tb = vbuf + (tok >> 5) * VTB + (tok & 31) * 16;
#pragma unroll
      for (int w = 0; w < 4; ++w) ib[tk][w] = 0u;
#pragma unroll
      for (int p = 0; p < VKB; ++p) {
        const uint4 v = *reinterpret_cast<const uint4*>(tb + p * TILE * 16);
        const uint32_t wd[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int w = 0; w < 4; ++w) ib[tk][w] |= ((wd[w] >> g) & 0x01010101u) << p;
      }
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int w = j >> 1, k0 = 2 * (j & 1);  // rows g and g + 8: bytes k0 and k0 + 1 of word w
      auto val = [&](int tk, int k) { return vch[(ib[tk][w] >> (8 * k)) & 0xFFu]; };
      const __half2 h0 = __halves2half2(val(0, k0), val(1, k0));
      const __half2 h1 = __halves2half2(val(0, k0 + 1), val(1, k0 + 1));
      const __half2 h2 = __halves2half2(val(2, k0), val(3, k0));
      const __half2 h3 = __halves2half2(val(2, k0 + 1), val(3, k0 + 1));
      const uint32_t af[4] = {*reinterpret_cast<const uint32_t*>(&h0), *reinterpret_cast<const uint32_t*>(&h1),
                              *reinterpret_cast<const uint32_t*>(&h2), *reinterpret_cast<const uint32_t*>(&h3)};
      mma_f16_16816(acc[j], af, b0, b1);
    }
  }
  __syncthreads();  // every warp is done with the weights and the V tiles
  float* red = reinterpret_cast<float*>(kbuf);  // [4 warps][QCHUNK][DP], over the weights
  if (2 * t4 < QCHUNK) {  // D: rows g, g + 8 of block j; columns (query heads) 2 t4, 2 t4 + 1
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      float* r0 = red + (warp * QCHUNK + 2 * t4) * DP + 16 * j + g;
      r0[0] = acc[j][0];
      r0[DP] = acc[j][1];
      r0[8] = acc[j][2];
      r0[DP + 8] = acc[j][3];
    }
  }
  __syncthreads();
  const int c = threadIdx.x;
  float accs[4];
#pragma unroll
  for (int qq = 0; qq < QCHUNK; ++qq)
    accs[qq] = (red[(0 * QCHUNK + qq) * DP + c] + red[(1 * QCHUNK + qq) * DP + c]) +
               (red[(2 * QCHUNK + qq) * DP + c] + red[(3 * QCHUNK + qq) * DP + c]);

  // 4) partials
  const int hq0 = (bg % a.hkv) * a.group + QCHUNK * qc;
  const int nq = min(QCHUNK, a.group - QCHUNK * qc);
#pragma unroll
  for (int qq = 0; qq < QCHUNK; ++qq) {
    if (qq < nq) {
      const int64_t h = (int64_t)b * (a.hkv * a.group) + hq0 + qq;
      float* dst = a.part + (h * a.nch + chunk_id) * (DP + 2);
      dst[c] = accs[qq];
      if (c == 0) {
        dst[DP] = ntok > 0 ? stat[qq][0] : -INFINITY;
        dst[DP + 1] = ntok > 0 ? stat[qq][1] : 0.f;
      }
    }
  }
}

struct CArgs {
  const float* part;       // partial rows: o_rot[dp], m, l
  int64_t row_stride;      // floats between consecutive output rows' first partial
  int64_t chunk_stride;    // floats between the partials of one row
  const int8_t* vD;
  const int32_t* seq_lens;  // NULL: a row is empty when no partial has weight
  float* out;              // final mode: [rows][d]
  float* part_out;         // partial mode (non-NULL): [rows][dp + 2], unnormalised, no rotation
  int nch, d, dp, hq;
};

// Log-sum-exp merge of the partials of one output row (b, h): weights
// 2^(m_k - M) over the partials k, then either the normalised output with the
// inverse rotation D H / sqrt(dp) (final mode), or the merged partial itself.
__global__ void __launch_bounds__(128) combine_kernel(const CArgs a) {
  __shared__ float o[256];
  __shared__ float wts[2048];
  __shared__ float tot;
  __shared__ float red[4];
  const int64_t h = blockIdx.x;  // b * hq + head
  const int b = (int)(h / a.hq);
  const float* src = a.part + h * a.row_stride;
  // chunk weights 2^(m_k - M)
  float mx = -INFINITY;
  for (int k = threadIdx.x; k < a.nch; k += blockDim.x) mx = fmaxf(mx, src[(int64_t)k * a.chunk_stride + a.dp]);
  mx = warp_max(mx);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
  __syncthreads();
  mx = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
  __syncthreads();
  float lsum = 0.f;
  for (int k = threadIdx.x; k < a.nch; k += blockDim.x) {
    const float mk = src[(int64_t)k * a.chunk_stride + a.dp];
    const float wk = (mk == -INFINITY) ? 0.f : exp2f(mk - mx);
    wts[k] = wk;
    lsum += wk * src[(int64_t)k * a.chunk_stride + a.dp + 1];
  }
  lsum = warp_sum(lsum);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = lsum;
  __syncthreads();
  if (threadIdx.x == 0) tot = red[0] + red[1] + red[2] + red[3];
  __syncthreads();
  const bool empty = (a.seq_lens != nullptr && a.seq_lens[b] <= 0) || !(tot > 0.f);
  if (a.part_out) {
    float* dst = a.part_out + h * (a.dp + 2);
    for (int c = threadIdx.x; c < a.dp; c += blockDim.x) {
      float s = 0.f;
      for (int k = 0; k < a.nch; ++k) s = fmaf(wts[k], src[(int64_t)k * a.chunk_stride + c], s);
      dst[c] = empty ? 0.f : s;
    }
    if (threadIdx.x == 0) {
      dst[a.dp] = empty ? -INFINITY : mx;
      dst[a.dp + 1] = empty ? 0.f : tot;
    }
    return;
  }
  for (int c = threadIdx.x; c < a.dp; c += blockDim.x) {
    float s = 0.f;
    for (int k = 0; k < a.nch; ++k) s = fmaf(wts[k], src[(int64_t)k * a.chunk_stride + c], s);
    o[c] = empty ? 0.f : s / tot;
  }
  __syncthreads();
  // inverse rotation: x_hat = D o (H o_rot) / sqrt(dp)
  const float rs = rsqrtf((float)a.dp);
  for (int c = threadIdx.x; c < a.d; c += blockDim.x) {
    float s = 0.f;
    for (int j = 0; j < a.dp; ++j) s += (__popc(c & j) & 1) ? -o[j] : o[j];
    a.out[h * a.d + c] = s * rs * (float)a.vD[c];
  }
}

template <int KB, int SI, int VKB>
int launch_decode(const DArgs& a, int blocks, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(blocks);
  cfg.blockDim = dim3(128);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const bool staged = (a.max_tokens % TILE) == 0 && a.km == 128 * SI && tq::aligned(a.knorms, 16) &&
                      tq::aligned(a.krnorms, 16) && tq::aligned(a.vnorms, 16);
  cudaError_t e;
  if (staged) {
    constexpr int smem = staged_smem<KB, SI, VKB>();
    static_assert((CH / TILE) * TILE * (KB * 16 + 16 * SI) >= CH * 16 &&
                      (CH / TILE) * TILE * (KB * 16 + 16 * SI) >= 4 * QCHUNK * 128 * 4,
                  "the weights and, after them, the warp sums alias the K tiles");
    e = cudaFuncSetAttribute(decode_staged_kernel<KB, SI, VKB>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return tq::set_error(TQ_ECUDA, "tq_decode_attn: %s", cudaGetErrorString(e));
    cfg.dynamicSmemBytes = smem;
    e = cudaLaunchKernelEx(&cfg, decode_staged_kernel<KB, SI, VKB>, a);
  } else {
    e = cudaLaunchKernelEx(&cfg, decode_kernel<KB, SI, VKB>, a);
  }
  if (e != cudaSuccess) return tq::set_error(TQ_ECUDA, "tq_decode_attn: launch failed: %s", cudaGetErrorString(e));
  return TQ_OK;
}

template <int KB, int SI>
int dispatch_vkb(int vkb, const DArgs& a, int blocks, cudaStream_t st) {
  switch (vkb) {
    case 1: return launch_decode<KB, SI, 1>(a, blocks, st);
    case 2: return launch_decode<KB, SI, 2>(a, blocks, st);
    case 3: return launch_decode<KB, SI, 3>(a, blocks, st);
    default: return launch_decode<KB, SI, 4>(a, blocks, st);
  }
}

int64_t decode_ws_parts(int batch, int hq, int64_t max_tokens) {
  const int64_t nch = (max_tokens + CH - 1) / CH;
  return (int64_t)batch * hq * std::max<int64_t>(nch, 1) * (128 + 2) * 4;
}

}  // namespace

extern "C" int64_t tq_decode_attn_workspace(const tq_params* kp, int batch, int n_q_heads, int n_kv_heads,
                                            int64_t max_tokens) {
  if (!kp || batch < 0 || n_q_heads < 1 || n_kv_heads < 1 || max_tokens < 0) return -1;
  const int kb = kp->mode == TQ_MODE_PROD ? kp->bits - 1 : kp->bits;
  if (kb < 1 || kb > 4) return -1;
  const tqd::ScanShape sh(kp->d_pad, kb, kp->mode == TQ_MODE_PROD ? kp->m : 0);
  const int group = n_q_heads / n_kv_heads;
  const int nqc = (group + tqd::QCHUNK - 1) / tqd::QCHUNK;
  int64_t prep = (int64_t)batch * n_kv_heads * nqc * tqd::prep_chunk_bytes(sh.fr);
  prep = (prep + 255) & ~(int64_t)255;
  // the values' layout is not known here: enough for either decode
  const int64_t sliced = tq::decode_sliced_workspace(kb, kp->mode == TQ_MODE_PROD ? kp->m : 0, batch, n_q_heads,
                                                     n_kv_heads, max_tokens);
  return std::max<int64_t>(prep + decode_ws_parts(batch, n_q_heads, max_tokens), sliced);
}

namespace {
int decode_attn(const tq_params* kp, const tq_params* vp, const float* q, int batch, int n_q_heads, int n_kv_heads,
                const void* kcodes, const uint16_t* knorms, const uint16_t* krnorms, const void* vcodes,
                const uint16_t* vnorms, const int32_t* seq_lens, int64_t max_tokens, float scale, float v_eps,
                float* out, float* partial_out, void* workspace, int64_t workspace_bytes, tq_stream_t stream) {
  using namespace tq;
  int rc = check_params(kp, "tq_decode_attn(kp)");
  if (!rc) rc = check_planes(kp, "tq_decode_attn(kp)");
  if (rc) return rc;
  rc = check_params(vp, "tq_decode_attn(vp)");
  if (rc) return rc;
  if (vp->layout != TQ_LAYOUT_PLANES) {  // token-sliced values: the tensor-memory decode
    if (partial_out || v_eps != 0.f)
      return set_error(TQ_EUNSUPPORTED, "tq_decode_attn: token-sliced values take the full decode only");
    return decode_attn_sliced(kp, vp, q, batch, n_q_heads, n_kv_heads, kcodes, knorms, krnorms, vcodes, vnorms,
                              seq_lens, max_tokens, scale, out, workspace, workspace_bytes,
                              reinterpret_cast<cudaStream_t>(stream));
  }
  if (kp->mode != TQ_MODE_PROD || vp->mode != TQ_MODE_MSE)
    return set_error(TQ_EUNSUPPORTED, "tq_decode_attn: needs product-code keys and MSE-code values");
  if (kp->d_pad != 128 || vp->d_pad != 128 || kp->d != vp->d)
    return set_error(TQ_EUNSUPPORTED, "tq_decode_attn: keys and values need d_pad = 128 and equal d");
  const int kkb = index_bits(kp), vkb = index_bits(vp);
  if (kkb > 3) return set_error(TQ_EUNSUPPORTED, "tq_decode_attn: key codes need <= 3 index bits");
  if (batch < 0 || n_kv_heads < 1 || n_q_heads < 1 || (n_q_heads % n_kv_heads) != 0)
    return set_error(TQ_EINVAL, "tq_decode_attn: n_q_heads must be a positive multiple of n_kv_heads");
  if (max_tokens < 0 || max_tokens > (int64_t)1 << 31) return set_error(TQ_EINVAL, "tq_decode_attn: bad max_tokens");
  if (batch == 0) {
    clear_error();
    return TQ_OK;
  }
  if (!q || !kcodes || !knorms || !krnorms || !vcodes || !vnorms || !seq_lens || (!out && !partial_out) || !workspace)
    return set_error(TQ_EINVAL, "tq_decode_attn: NULL pointer argument");
  if (!aligned(kcodes, 16) || !aligned(vcodes, 16) || !aligned(workspace, 16))
    return set_error(TQ_EINVAL, "tq_decode_attn: codes and workspace must be 16-byte aligned");
  const int64_t need = tq_decode_attn_workspace(kp, batch, n_q_heads, n_kv_heads, max_tokens);
  if (workspace_bytes < need)
    return set_error(TQ_EINVAL, "tq_decode_attn: workspace too small (%lld < %lld)", (long long)workspace_bytes,
                     (long long)need);
  const int group = n_q_heads / n_kv_heads;
  const int nqc = (group + tqd::QCHUNK - 1) / tqd::QCHUNK;
  const tqd::ScanShape sh(128, kkb, kp->m);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  tqd::PrepArgs pa;
  pa.q = q;
  pa.d = kp->d;
  pa.dp = 128;
  pa.kb = kkb;
  pa.m = kp->m;
  pa.n_outer = batch * n_kv_heads;
  pa.group = group;
  pa.nqc = nqc;
  pa.cent = kp->centroids;
  pa.D = kp->signs_D;
  pa.S = kp->S;
  pa.out = static_cast<uint8_t*>(workspace);
  pa.fr = sh.fr;
  rc = launch_prep(pa, st);
  if (rc) return rc;
  int64_t prep_total = (int64_t)batch * n_kv_heads * nqc * tqd::prep_chunk_bytes(sh.fr);
  prep_total = (prep_total + 255) & ~(int64_t)255;
  const int nch = (int)std::max<int64_t>(1, (max_tokens + CH - 1) / CH);
  if (nch > 2048) return set_error(TQ_EUNSUPPORTED, "tq_decode_attn: max_tokens above 524288 is not supported");
  DArgs a;
  a.kcodes = static_cast<const uint8_t*>(kcodes);
  a.knorms = knorms;
  a.krnorms = krnorms;
  a.vcodes = static_cast<const uint8_t*>(vcodes);
  a.vnorms = vnorms;
  a.seq_lens = seq_lens;
  a.vcent = vp->centroids;
  a.max_tokens = max_tokens;
  a.hkv = n_kv_heads;
  a.group = group;
  a.nqc = nqc;
  a.nch = nch;
  a.km = kp->m;
  a.ktb = tqd::tile_bytes(128, kkb, kp->m);
  a.vtb = tqd::tile_bytes(128, vkb, 0);
  a.vkb = vkb;
  a.dp = 128;
  a.prep = pa.out;
  a.prep_bytes = tqd::prep_chunk_bytes(sh.fr);
  a.part = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + prep_total);
  a.kappa = (float)(std::sqrt(M_PI / 2.0) / kp->m);
  const float sc = scale != 0.f ? scale : (float)(1.0 / std::sqrt((double)kp->d));
  a.sl2 = sc * 1.4426950408889634f;
  a.veps = v_eps;
  const int64_t blocks64 = (int64_t)batch * n_kv_heads * nqc * nch;
  if (blocks64 > 0x7fffffff) return set_error(TQ_EUNSUPPORTED, "tq_decode_attn: grid too large");
  const int blocks = (int)blocks64;
  const int si = sh.nsi;
  switch (kkb) {
    case 1: rc = si == 2 ? dispatch_vkb<1, 2>(vkb, a, blocks, st) : dispatch_vkb<1, 1>(vkb, a, blocks, st); break;
    case 2: rc = si == 2 ? dispatch_vkb<2, 2>(vkb, a, blocks, st) : dispatch_vkb<2, 1>(vkb, a, blocks, st); break;
    default: rc = si == 2 ? dispatch_vkb<3, 2>(vkb, a, blocks, st) : dispatch_vkb<3, 1>(vkb, a, blocks, st); break;
  }
  if (rc) return rc;
  CArgs ca;
  ca.part = a.part;
  ca.row_stride = (int64_t)nch * (128 + 2);
  ca.chunk_stride = 128 + 2;
  ca.vD = vp->signs_D;
  ca.seq_lens = seq_lens;
  ca.out = out;
  ca.part_out = partial_out;
  ca.nch = nch;
  ca.d = kp->d;
  ca.dp = 128;
  ca.hq = n_q_heads;
  combine_kernel<<<batch * n_q_heads, 128, 0, st>>>(ca);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(TQ_ECUDA, "tq_decode_attn: combine launch failed: %s", cudaGetErrorString(e));
  clear_error();
  return TQ_OK;
}
}  // namespace

extern "C" int tq_decode_attn(const tq_params* kp, const tq_params* vp, const float* q, int batch, int n_q_heads,
                              int n_kv_heads, const void* kcodes, const uint16_t* knorms, const uint16_t* krnorms,
                              const void* vcodes, const uint16_t* vnorms, const int32_t* seq_lens,
                              int64_t max_tokens, float scale, float* out, void* workspace,
                              int64_t workspace_bytes, tq_stream_t stream) {
  return decode_attn(kp, vp, q, batch, n_q_heads, n_kv_heads, kcodes, knorms, krnorms, vcodes, vnorms, seq_lens,
                     max_tokens, scale, 0.f, out, nullptr, workspace, workspace_bytes, stream);
}

extern "C" int tq_decode_attn_sparse(const tq_params* kp, const tq_params* vp, const float* q, int batch,
                                     int n_q_heads, int n_kv_heads, const void* kcodes, const uint16_t* knorms,
                                     const uint16_t* krnorms, const void* vcodes, const uint16_t* vnorms,
                                     const int32_t* seq_lens, int64_t max_tokens, float scale, float v_eps,
                                     float* out, void* workspace, int64_t workspace_bytes, tq_stream_t stream) {
  if (!(v_eps >= 0.f) || !std::isfinite(v_eps))
    return tq::set_error(TQ_EINVAL, "tq_decode_attn_sparse: v_eps must be finite and >= 0");
  return decode_attn(kp, vp, q, batch, n_q_heads, n_kv_heads, kcodes, knorms, krnorms, vcodes, vnorms, seq_lens,
                     max_tokens, scale, v_eps, out, nullptr, workspace, workspace_bytes, stream);
}

extern "C" int64_t tq_decode_attn_partial_bytes(const tq_params* vp, int batch, int n_q_heads) {
  if (!vp || batch < 0 || n_q_heads < 1) return -1;
  return (int64_t)batch * n_q_heads * (vp->d_pad + 2) * 4;
}

extern "C" int tq_decode_attn_partial(const tq_params* kp, const tq_params* vp, const float* q, int batch,
                                      int n_q_heads, int n_kv_heads, const void* kcodes, const uint16_t* knorms,
                                      const uint16_t* krnorms, const void* vcodes, const uint16_t* vnorms,
                                      const int32_t* seq_lens, int64_t max_tokens, float scale, float* partial,
                                      void* workspace, int64_t workspace_bytes, tq_stream_t stream) {
  if (!partial) return tq::set_error(TQ_EINVAL, "tq_decode_attn_partial: NULL partial");
  if (!tq::aligned(partial, 4)) return tq::set_error(TQ_EINVAL, "tq_decode_attn_partial: misaligned partial");
  return decode_attn(kp, vp, q, batch, n_q_heads, n_kv_heads, kcodes, knorms, krnorms, vcodes, vnorms, seq_lens,
                     max_tokens, scale, 0.f, nullptr, partial, workspace, workspace_bytes, stream);
}

extern "C" int tq_decode_attn_merge(const tq_params* vp, const float* partials, int n_parts, int batch,
                                    int n_q_heads, float* out, tq_stream_t stream) {
  using namespace tq;
  int rc = check_params(vp, "tq_decode_attn_merge");
  if (rc) return rc;
  if (vp->mode != TQ_MODE_MSE || vp->d_pad != 128)
    return set_error(TQ_EUNSUPPORTED, "tq_decode_attn_merge: needs the MSE-code value parameters with d_pad 128");
  if (n_parts < 1 || n_parts > 2048 || batch < 0 || n_q_heads < 1)
    return set_error(TQ_EINVAL, "tq_decode_attn_merge: need 1 <= n_parts <= 2048, batch >= 0, n_q_heads >= 1");
  if (batch == 0) {
    clear_error();
    return TQ_OK;
  }
  if (!partials || !out) return set_error(TQ_EINVAL, "tq_decode_attn_merge: NULL pointer argument");
  if (!aligned(partials, 4) || !aligned(out, 4)) return set_error(TQ_EINVAL, "tq_decode_attn_merge: misaligned pointer");
  const int64_t rows = (int64_t)batch * n_q_heads;
  if (rows > 0x7fffffff) return set_error(TQ_EUNSUPPORTED, "tq_decode_attn_merge: too many rows");
  CArgs ca;
  ca.part = partials;
  ca.row_stride = 128 + 2;
  ca.chunk_stride = rows * (128 + 2);
  ca.vD = vp->signs_D;
  ca.seq_lens = nullptr;
  ca.out = out;
  ca.part_out = nullptr;
  ca.nch = n_parts;
  ca.d = vp->d;
  ca.dp = 128;
  ca.hq = n_q_heads;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  combine_kernel<<<(unsigned)rows, 128, 0, st>>>(ca);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(TQ_ECUDA, "tq_decode_attn_merge: launch failed: %s", cudaGetErrorString(e));
  clear_error();
  return TQ_OK;
}

namespace tq {
// The log-sum-exp combine (and inverse rotation) over partial rows, for the
// tensor-memory decode (decode_tc.cu).
int launch_combine(const float* part, int64_t row_stride, int64_t chunk_stride, const int8_t* vD,
                   const int32_t* seq_lens, float* out, int nch, int d, int dp, int hq, int64_t rows,
                   cudaStream_t st) {
  if (rows > 0x7fffffff || nch > 2048) return set_error(TQ_EUNSUPPORTED, "tq_decode_attn: combine shape too large");
  CArgs ca;
  ca.part = part;
  ca.row_stride = row_stride;
  ca.chunk_stride = chunk_stride;
  ca.vD = vD;
  ca.seq_lens = seq_lens;
  ca.out = out;
  ca.part_out = nullptr;
  ca.nch = nch;
  ca.d = d;
  ca.dp = dp;
  ca.hq = hq;
  combine_kernel<<<(unsigned)rows, 128, 0, st>>>(ca);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(TQ_ECUDA, "tq_decode_attn: combine launch failed: %s", cudaGetErrorString(e));
  return TQ_OK;
}
}  // namespace tq
