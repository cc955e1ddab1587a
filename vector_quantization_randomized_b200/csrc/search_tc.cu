// tq_search_topk on the fifth-generation tensor cores for d_pad 256 ("TurboQuant
// explainer" (m.163.com), "向量搜索": top-k inner-product search straight from
// the codes; the estimator is the logit of "第二步：QJL").
//
// Same integer form as the logits scan (scan.cuh, logits_tc.cu): the code bits
// of 128 database vectors are the A operand of tcgen05.mma kind::i8 in tensor
// memory, one byte per bit (2^c * bit for bit class c = coordinate % 8), and
// the digits of 16 queries' weights are the B operand in shared memory (64
// rows = 16 queries x 4 signed base-256 digits).  One plane of 128 vectors is
// 64 tensor-memory columns; an item (128 vectors) is NT Walsh planes and the
// sign plane, 8 MMAs each (M = 128, N = 64, K = 32 bytes), into accumulator
// columns of its own for the centroid and the sign sums.
//
// Work is split into units (database split x chunk of 16 queries), ordered
// split-major so the CTAs running at the same time read the same split and
// share it in L2.  Per CTA, one persistent loop over its units:
//   warp 0      bulk copies of the code tiles of every item into a ring of stages;
//   warp 1      MMA issue (warp-uniform, elected lane); at a unit boundary it
//               waits for its last MMAs and bulk-loads the next chunk's B image;
//   warps 2-9   expansion: code words -> masked bytes -> tcgen05.st into a ring of
//               four plane slots (warp = lane quadrant x 4 bit classes);
//   warps 10-17 epilogue: tcgen05.ld of the item's sums, digits, norms, scores;
//               warp = lane quadrant x 8 queries, one sorted top-16 per query
//               across lanes 0..15 (insertions only when a score beats the 16th);
//               at a unit's end the four quadrant lists of a query are merged
//               into the unit's candidates.  A last kernel merges the splits.
// The B images (every chunk of 16 queries) are built once per call by
// search_prep_kernel into the workspace.
#include <cuda_runtime.h>

#include <algorithm>
#include <climits>
#include <cmath>

#include "common.h"
#include "prep.h"
#include "scan.cuh"
#include "tc.cuh"

namespace {
using namespace tqd;

constexpr int DP = 256;
constexpr int QC = 16;          // queries per chunk
constexpr int NR = 4 * QC;      // B rows: 16 queries x 4 digits
constexpr int KEEP = 16;        // candidates kept per (query, split)
constexpr int TK = 128;         // vectors per item
constexpr int NSLOT = 4;        // plane slots in tensor memory
constexpr int STAGES = 6;       // code stages in shared memory
constexpr int MAX_SPLITS = 64;  // the split merge takes up to 1024 candidates per query

// chunk image: scalars (16 x float4), then per plane 16 K chunks of 16 bytes,
// each chunk 64 rows x 16 bytes (8-row groups 128 bytes apart, K chunks 1024 apart)
template <int KB, int SI>
struct SL {
  static constexpr int NT = KB == 1 ? 1 : (KB == 2 ? 2 : 4);
  static constexpr int NP = NT + SI;
  static constexpr int IMG_PLANE = 16 * 1024;
  static constexpr int IMG = 256 + NP * IMG_PLANE;
  static constexpr int TILEB = 32 * 32 * (KB + SI);  // 32-vector tile, d_pad 256, m = 256
  static constexpr int STAGE = 4 * TILEB;
  static constexpr int W_MMA = 1, W_EXP0 = 2, W_EPI0 = 10, NTHREADS = 18 * 32;
  static constexpr int OFF_IMG = 1024;
  static constexpr int OFF_RING = OFF_IMG + IMG;
  static constexpr int OFF_LIST = OFF_RING + STAGES * STAGE;       // [8 warps][8 queries][16] (score, id)
  static constexpr int SMEM = OFF_LIST + 8 * 8 * KEEP * 8;
};

struct PrepS {
  const float* q;
  int n_q, d, kb, m;
  int group, n_chunks;  // queries per head; 16-query chunks per head (image i = head * n_chunks + chunk)
  const float* cent;
  const int8_t* D;
  const uint16_t* S;
  uint8_t* img;  // [n_chunks][IMG]
  int img_bytes, np;
};

__device__ __forceinline__ int exponent_of(float x) {
  const uint32_t b = __float_as_uint(x) & 0x7FFFFFFFu;
  if (b >= 0x00800000u && b < 0x7F800000u) return (int)(b >> 23) - 126;
  int e;
  frexpf(x, &e);
  return e;
}
__device__ __forceinline__ float pow2(int k) {
  return (k >= -126 && k <= 127) ? __uint_as_float((uint32_t)(127 + k) << 23) : ldexpf(1.f, k);
}

// B image of one chunk of 16 queries (256 threads): q_rot = H D q / 16 (warp per
// 2 queries), u = S q_rot (thread = row of S), per-query scales 2^F, 2^G (the
// largest weight just below 2^23), weights shifted by 7 - c and split into 4
// signed base-256 digits; row 4j + digit of query j.
__global__ void __launch_bounds__(256) search_prep_kernel(const PrepS a) {
  __shared__ float qt[QC][DP];
  __shared__ float uu[QC][DP];
  __shared__ float alpha[5];
  __shared__ float stat[QC][4];  // sum q_rot, max |q_rot|, sum u, max |u|
  __shared__ float FG[QC][2];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int head = blockIdx.x / a.n_chunks, chunk = blockIdx.x - head * a.n_chunks;
  const int NT = walsh_planes(a.kb), L = 1 << a.kb;
  uint8_t* img = a.img + (int64_t)blockIdx.x * a.img_bytes;
  if (tid < NT) {
    const int mask = walsh_mask(a.kb, tid);
    double s = 0.0;
    for (int l = 0; l < L; ++l) s += (double)__ldg(a.cent + l) * ((__popc(l & mask) & 1) ? 1.0 : -1.0);
    alpha[tid] = (float)(s / L);
  }
  if (tid == 32) alpha[4] = __ldg(a.cent + L - 1);
  for (int jq = 0; jq < 2; ++jq) {  // warp = queries 2 warp, 2 warp + 1; lane holds coordinates lane + 32 i
    const int j = 2 * warp + jq, qi = head * a.group + chunk * QC + j;
    const bool valid = chunk * QC + j < a.group;
    float y[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int c = 32 * i + lane;
      y[i] = (valid && c < a.d) ? __ldg(a.q + (int64_t)qi * a.d + c) * (float)__ldg(a.D + c) : 0.f;
    }
#pragma unroll
    for (int h = 1; h < 8; h <<= 1)
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if ((i & h) == 0) {
          const float u = y[i], w = y[i + h];
          y[i] = u + w;
          y[i + h] = u - w;
        }
#pragma unroll
    for (int sft = 1; sft < 32; sft <<= 1)
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float o = __shfl_xor_sync(FULL, y[i], sft);
        y[i] = (lane & sft) ? (o - y[i]) : (y[i] + o);
      }
    float sum = 0.f, mx = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float v = y[i] * 0.0625f;  // 1/sqrt(256)
      qt[j][32 * i + lane] = v;
      sum += v;
      mx = fmaxf(mx, fabsf(v));
    }
    sum = warp_sum(sum);
    mx = warp_max(mx);
    if (lane == 0) {
      stat[j][0] = sum;
      stat[j][1] = mx;
    }
  }
  __syncthreads();
  if (a.m > 0) {  // u = S q_rot: thread = row of S, all 16 queries
    const int i = tid;
    float acc[QC];
#pragma unroll
    for (int j = 0; j < QC; ++j) acc[j] = 0.f;
    if (i < a.m) {
      const uint4* srow = reinterpret_cast<const uint4*>(a.S + (size_t)i * DP);
      for (int k = 0; k < DP / 8; ++k) {
        const uint4 v = __ldg(srow + k);
        const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int h2 = 0; h2 < 4; ++h2) {
          const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&wv[h2]));
          const int c = 8 * k + 2 * h2;
#pragma unroll
          for (int j = 0; j < QC; ++j) acc[j] = fmaf(f.y, qt[j][c + 1], fmaf(f.x, qt[j][c], acc[j]));
        }
      }
    }
#pragma unroll
    for (int j = 0; j < QC; ++j) uu[j][i] = acc[j];
    __syncthreads();
    for (int jq = 0; jq < 2; ++jq) {
      const int j = 2 * warp + jq;
      float su = 0.f, mu = 0.f;
      for (int r = lane; r < a.m; r += 32) {
        su += uu[j][r];
        mu = fmaxf(mu, fabsf(uu[j][r]));
      }
      su = warp_sum(su);
      mu = warp_max(mu);
      if (lane == 0) {
        stat[j][2] = su;
        stat[j][3] = mu;
      }
    }
  }
  __syncthreads();
  if (tid < QC) {
    const int j = tid;
    float amax = 0.f;
    for (int T = 0; T < NT; ++T) amax = fmaxf(amax, fabsf(alpha[T]));
    const float mc = 2.f * amax * stat[j][1], ms = a.m > 0 ? 2.f * stat[j][3] : 0.f;
    const int F = mc > 0.f ? 23 - exponent_of(mc) : 0;
    const int G = ms > 0.f ? 23 - exponent_of(ms) : 0;
    FG[j][0] = pow2(F);
    FG[j][1] = pow2(G);
    reinterpret_cast<float4*>(img)[j] =
        make_float4(pow2(-(F + 7)), alpha[4] * stat[j][0], pow2(-(G + 7)), a.m > 0 ? stat[j][2] : 0.f);
  }
  __syncthreads();
  // digit words: item (query j, plane P, bit class c, word w of 8): the weights of
  // coordinates 32w + 8b + c (b = 0..3) = bytes 4(w&3) + b of K chunk 16P + 2c + (w>>2)
  const int items = QC * a.np * 64;
  for (int e = tid; e < items; e += 256) {
    const int w = e & 7, c = (e >> 3) & 7, pj = e >> 6;
    const int j = pj / a.np, P = pj - j * a.np;
    const bool cen = P < NT;
    const float scale = cen ? 2.f * alpha[P] * FG[j][0] : 2.f * FG[j][1];
    uint32_t W[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int co = 32 * w + 8 * b + c;
      const float src = cen ? qt[j][co] : (co < a.m ? uu[j][co] : 0.f);
      int X = __float2int_rn(src * scale) * (1 << (7 - c));
#pragma unroll
      for (int dd = 0; dd < 3; ++dd) {
        const int lowb = (int)(int8_t)(X & 0xFF);
        W[dd] |= (uint32_t)(uint8_t)lowb << (8 * b);
        X = (X - lowb) >> 8;
      }
      W[3] |= (uint32_t)(uint8_t)X << (8 * b);
    }
    const int kc = 2 * c + (w >> 2);
    uint8_t* base = img + 256 + P * 16384 + kc * 1024 + 4 * (w & 3);
#pragma unroll
    for (int dd = 0; dd < 4; ++dd) {
      const int row = 4 * j + dd;
      *reinterpret_cast<uint32_t*>(base + (row >> 3) * 128 + (row & 7) * 16) = W[dd];
    }
  }
}

struct SArgsTC {
  const uint8_t* codes;
  const uint16_t* norms;
  const uint16_t* rnorms;
  int64_t n_db;         // keys per head (the database in search)
  int n_q, n_chunks, nsplit, tb;
  int group;            // queries per head (search: n_q, one head)
  int64_t split_keys;   // keys per split (a multiple of 32)
  int64_t n_units;      // heads * nsplit * n_chunks: head-major, then split-major
  const uint8_t* img;   // [heads][n_chunks][img_bytes]
  int img_bytes;
  float2* cand;         // top-k: [n_q][nsplit][KEEP] (score, id bits)
  float* logits;        // all scores: row head * group + query, stride ld
  int64_t ld;
  float kappa;
};

__device__ __forceinline__ bool better(float s, int i, float s2, int i2) { return s > s2 || (s == s2 && i < i2); }

// ALL: write every score to the logits rows instead of keeping a top-16 per query
template <int KB, int SI, bool ALL>
__global__ void __launch_bounds__(SL<KB, SI>::NTHREADS, 1) search_tc_kernel(const SArgsTC a) {
  using L = SL<KB, SI>;
  constexpr int NP = L::NP, NT = L::NT;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);  // [STAGES] code stage loaded (1 + tx)
  uint64_t* empty = full + STAGES;                     // [STAGES] code stage read (8 expansion warps)
  uint64_t* afull = empty + STAGES;                    // [NSLOT] plane slot written (8)
  uint64_t* afree = afull + NSLOT;                     // [NSLOT] plane slot read by its MMAs (1)
  uint64_t* cfull = afree + NSLOT;                     // [2] accumulator set complete (1)
  uint64_t* accfree = cfull + 2;                       // [2] accumulator set read (8)
  uint64_t* bfull = accfree + 2;                       // B image loaded (1 + tx)
  uint64_t* bdone = bfull + 1;                         // the MMA warp's MMAs so far completed (1)
  uint64_t* gbar = bdone + 1;                          // epilogue group barrier (8)
  uint32_t* tbase = reinterpret_cast<uint32_t*>(gbar + 1);
  uint8_t* img = smem + L::OFF_IMG;
  uint8_t* ring = smem + L::OFF_RING;
  float2* lists = reinterpret_cast<float2*>(smem + L::OFF_LIST);  // [8 warps][8 queries][KEEP]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 8);
    }
    for (int s = 0; s < NSLOT; ++s) {
      mbar_init(&afull[s], 8);
      mbar_init(&afree[s], 1);
    }
    for (int c = 0; c < 2; ++c) {
      mbar_init(&cfull[c], 1);
      mbar_init(&accfree[c], 8);
    }
    mbar_init(bfull, 1);
    mbar_init(bdone, 1);
    mbar_init(gbar, 8);
  }
  if (warp == 0) tmem_alloc(tbase, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tbase;
  // tensor-memory columns: accumulator sets 0, 1 (128 each: 64 centroid + 64 sign), then the plane slots
  auto acc_col = [&](int c) { return tmem + (uint32_t)(128 * c); };
  auto slot_col = [&](int s) { return tmem + 256u + (uint32_t)(64 * s); };

  // the units of this CTA: u = blockIdx.x + k * gridDim.x; unit -> (head, split, chunk);
  // k0 = first key of the unit (global over heads), nk = its key count
  const int64_t per_head = (int64_t)a.nsplit * a.n_chunks;
  auto unit_keys = [&](int64_t u, int64_t& k0, int64_t& nk) {
    const int64_t head = u / per_head;
    const int64_t split = (u - head * per_head) / a.n_chunks;
    const int64_t kl = split * a.split_keys;
    nk = std::min<int64_t>(a.split_keys, a.n_db - kl);
    if (nk < 0) nk = 0;
    k0 = head * a.n_db + kl;
  };
  auto unit_image = [&](int64_t u) {  // image index head * n_chunks + chunk
    const int64_t head = u / per_head;
    return head * a.n_chunks + (u - head * per_head) % a.n_chunks;
  };

  if (warp == 0) {
    // ---------------- producer: code tiles of every item ----------------
    grid_dependency_wait();
    if (lane == 0) {
      int64_t gi = 0;  // global item counter
      bool ok = true;
      for (int64_t u = blockIdx.x; u < a.n_units && ok; u += gridDim.x) {
        int64_t k0, nk;
        unit_keys(u, k0, nk);
        for (int64_t i0 = 0; i0 < nk; i0 += TK, ++gi) {
          const int s = (int)(gi % STAGES);
          const int use = (int)(gi / STAGES);
          if (use >= 1 && !mbar_wait(&empty[s], (use - 1) & 1)) {
            ok = false;
            break;
          }
          const int64_t nki = std::min<int64_t>(TK, nk - i0);
          const uint32_t bytes = (uint32_t)(((nki + 31) >> 5) * a.tb);
          mbar_expect_tx(&full[s], bytes);
          bulk_g2s(ring + s * L::STAGE, a.codes + ((k0 + i0) >> 5) * a.tb, bytes, &full[s]);
        }
      }
      // nothing may still be in flight into shared memory when the CTA ends
      for (int64_t i = (gi > STAGES ? gi - STAGES : 0); i < gi; ++i) mbar_wait(&full[i % STAGES], (i / STAGES) & 1);
    }
  } else if (warp == L::W_MMA) {
    // ---------------- MMA issue and B images ----------------
    constexpr uint32_t idesc = idesc_u8s8_s32(TK, NR);
    grid_dependency_wait();  // the B images come from the prep kernel
    int64_t gi = 0, gp = 0;  // global item and plane counters
    uint32_t bph = 0, dph = 0;
    bool ok = true;
    for (int64_t u = blockIdx.x; u < a.n_units && ok; u += gridDim.x) {
      const int64_t chunk = unit_image(u);
      int64_t k0, nk;
      unit_keys(u, k0, nk);
      if (u != blockIdx.x) {  // every MMA reading the old image has completed
        __syncwarp();
        umma_commit_elect(bdone);
        if (!mbar_wait(bdone, dph)) break;
        dph ^= 1u;
      }
      if (lane == 0) {
        mbar_expect_tx(bfull, (uint32_t)L::IMG);
        bulk_g2s(img, a.img + chunk * a.img_bytes, (uint32_t)L::IMG, bfull);
      }
      if (!mbar_wait(bfull, bph)) break;
      bph ^= 1u;
      const uint32_t simg = smem_u32(img);
      for (int64_t i0 = 0; i0 < nk; i0 += TK, ++gi) {
        const int c = (int)(gi & 1);
        if (gi >= 2 && !mbar_wait(&accfree[c], ((gi - 2) >> 1) & 1)) {
          ok = false;
          break;
        }
#pragma unroll 1
        for (int P = 0; P < NP; ++P, ++gp) {
          const int s = (int)(gp % NSLOT);
          if (!mbar_wait(&afull[s], (gp / NSLOT) & 1)) {
            ok = false;
            break;
          }
          __syncwarp();
          tc_fence_after();
          const uint32_t d = acc_col(c) + (P < NT ? 0u : 64u);
          const uint64_t bd = smem_desc(simg + 256 + P * L::IMG_PLANE, 1024, 128);
          const bool first = P == 0 || P == NT;
#pragma unroll
          for (int ks = 0; ks < 8; ++ks)  // K step = bit class ks: 2 K chunks of the image
            umma_i8_ts_elect(d, slot_col(s) + 8u * ks, bd + (uint64_t)(128 * ks), idesc,
                             (first && ks == 0) ? 0u : 1u);
          umma_commit_elect(&afree[s]);
        }
        if (!ok) break;
        umma_commit_elect(&cfull[c]);
      }
    }
    __syncwarp();
  } else if (warp < L::W_EPI0) {
    // ---------------- expansion: code bits -> plane slots ----------------
    const int ew = warp - L::W_EXP0;
    const int qd = warp & 3;  // lane quadrant = 32-vector tile of the item
    const int cg = ew >> 2;   // bit classes 4cg .. 4cg+3
    int64_t gi = 0, gp = 0;
    bool ok = true;
    for (int64_t u = blockIdx.x; u < a.n_units && ok; u += gridDim.x) {
      int64_t k0, nk;
      unit_keys(u, k0, nk);
      for (int64_t i0 = 0; i0 < nk; i0 += TK, ++gi) {
        const int st = (int)(gi % STAGES);
        if (!mbar_wait(&full[st], (gi / STAGES) & 1)) {
          ok = false;
          break;
        }
        // plane words of vector 32 qd + lane (tiles past the item's end hold stale bytes; never scored)
        const uint8_t* src = ring + st * L::STAGE + qd * L::TILEB + lane * 32;
        uint4 pw[KB + SI][2];
#pragma unroll
        for (int p = 0; p < KB + SI; ++p) {
          pw[p][0] = *reinterpret_cast<const uint4*>(src + p * 1024);
          pw[p][1] = *reinterpret_cast<const uint4*>(src + p * 1024 + 16);
        }
        release_to_copy(&empty[st], lane);  // the stage is refilled once all 8 warps release it
#pragma unroll
        for (int P = 0; P < NP; ++P, ++gp) {
          uint32_t wv[8];
          {
            uint4 lo, hi;
            if (P < NT) {
              if constexpr (KB == 3) {
                if (P == 3) {  // sigma_0 sigma_1 sigma_2: parity of the three planes
                  lo = make_uint4(pw[0][0].x ^ pw[1][0].x ^ pw[2][0].x, pw[0][0].y ^ pw[1][0].y ^ pw[2][0].y,
                                  pw[0][0].z ^ pw[1][0].z ^ pw[2][0].z, pw[0][0].w ^ pw[1][0].w ^ pw[2][0].w);
                  hi = make_uint4(pw[0][1].x ^ pw[1][1].x ^ pw[2][1].x, pw[0][1].y ^ pw[1][1].y ^ pw[2][1].y,
                                  pw[0][1].z ^ pw[1][1].z ^ pw[2][1].z, pw[0][1].w ^ pw[1][1].w ^ pw[2][1].w);
                } else {
                  lo = pw[P][0];
                  hi = pw[P][1];
                }
              } else {
                lo = pw[P][0];
                hi = pw[P][1];
              }
            } else {  // the sign plane
              lo = pw[KB + SI - 1][0];
              hi = pw[KB + SI - 1][1];
            }
            wv[0] = lo.x, wv[1] = lo.y, wv[2] = lo.z, wv[3] = lo.w;
            wv[4] = hi.x, wv[5] = hi.y, wv[6] = hi.z, wv[7] = hi.w;
          }
          const int s = (int)(gp % NSLOT);
          if (gp >= NSLOT && !mbar_wait(&afree[s], ((gp - NSLOT) / NSLOT) & 1)) {
            ok = false;
            break;
          }
          const uint32_t base = slot_col(s) + ((uint32_t)(32 * qd) << 16) + 32 * cg;
#pragma unroll
          for (int half = 0; half < 2; ++half) {  // classes 4cg + 2half, 4cg + 2half + 1
            uint32_t r[16];
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
              const uint32_t mk = 0x01010101u << (4 * cg + 2 * half + cc);
#pragma unroll
              for (int w = 0; w < 8; ++w) r[8 * cc + w] = wv[w] & mk;
            }
            tmem_st16(base + 16 * half, r);
          }
          tmem_st_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&afull[s]);
        }
      }
    }
  } else {
    // ---------------- epilogue: scores and top-16 per query ----------------
    const int ew = warp - L::W_EPI0;
    const int qd = warp & 3, hq = ew >> 2;  // vectors 32 qd + lane; queries 8 hq .. 8 hq + 7 of the chunk
    grid_dependency_wait();
    GroupSync gs{gbar, 0u};
    int64_t gi = 0;
    bool ok = true;
    for (int64_t u = blockIdx.x; u < a.n_units && ok; u += gridDim.x) {
      const int64_t img_i = unit_image(u), head = u / per_head;
      const int64_t chunk = img_i - head * a.n_chunks, split = (u - head * per_head) / a.n_chunks;
      int64_t k0, nk;
      unit_keys(u, k0, nk);
      const float4* scal = reinterpret_cast<const float4*>(a.img + img_i * a.img_bytes) + 8 * hq;
      // per query: entry `lane` (< 16) of the sorted list; the 16th entry is the threshold
      float ls[8];
      int li[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        ls[j] = -INFINITY;
        li[j] = INT_MAX;
      }
      for (int64_t i0 = 0; i0 < nk; i0 += TK, ++gi) {
        const int c = (int)(gi & 1);
        const int64_t key = k0 + i0 + 32 * qd + lane;
        const bool kvalid = (i0 + 32 * qd + lane) < nk;
        const float nrm = kvalid ? __half2float(__ushort_as_half(__ldg(a.norms + key))) : 0.f;
        const float gam = (SI && kvalid) ? __half2float(__ushort_as_half(__ldg(a.rnorms + key))) : 0.f;
        if (!mbar_wait(&cfull[c], (gi >> 1) & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t lrow = acc_col(c) + ((uint32_t)(32 * qd) << 16) + 32 * hq;
        float lv[8];
        {
          uint32_t rc[32];
          tmem_ld32_issue(lrow, rc);
          tmem_ld_wait(rc);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float4 scj = __ldg(scal + j);  // per-query scalars (same address on every lane)
            // sum_d 256^d C[d]: each C[d] an exact int32 below 2^24; one fp32 rounding per step
            const float cen = fmaf((float)(int)rc[4 * j + 3], 16777216.f,
                                   fmaf((float)(int)rc[4 * j + 2], 65536.f,
                                        fmaf((float)(int)rc[4 * j + 1], 256.f, (float)(int)rc[4 * j])));
            lv[j] = fmaf(cen, scj.x, -scj.y);
          }
        }
        if constexpr (SI) {
          uint32_t rs[32];
          tmem_ld32_issue(lrow + 64, rs);
          tmem_ld_wait(rs);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float4 scj = __ldg(scal + j);
            const float sg = fmaf((float)(int)rs[4 * j + 3], 16777216.f,
                                  fmaf((float)(int)rs[4 * j + 2], 65536.f,
                                       fmaf((float)(int)rs[4 * j + 1], 256.f, (float)(int)rs[4 * j])));
            lv[j] = fmaf(gam * a.kappa, fmaf(sg, scj.z, -scj.w), lv[j]);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&accfree[c]);
        if constexpr (ALL) {
          const int64_t kl = key - head * a.n_db;  // key within the head
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int qj = (int)chunk * QC + 8 * hq + j;
            if (kvalid && qj < a.group) a.logits[(head * a.group + qj) * a.ld + kl] = nrm * lv[j];
          }
          continue;
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float l = lv[j];
          const float score = nrm * l;
          const int id = (int)key;
          const float ts = __shfl_sync(FULL, ls[j], KEEP - 1);
          const int ti = __shfl_sync(FULL, li[j], KEEP - 1);
          uint32_t hit = __ballot_sync(FULL, kvalid && better(score, id, ts, ti));
          while (hit) {  // insert the hitting lanes one by one into the sorted list of lanes 0..15
            const int src = __ffs(hit) - 1;
            hit &= hit - 1;
            const float s2 = __shfl_sync(FULL, score, src);
            const int i2 = __shfl_sync(FULL, id, src);
            const float t15 = __shfl_sync(FULL, ls[j], KEEP - 1);
            const int i15 = __shfl_sync(FULL, li[j], KEEP - 1);
            if (!better(s2, i2, t15, i15)) continue;  // the list moved on since the ballot
            // position = number of entries better than the new one
            const bool above = lane < KEEP && better(ls[j], li[j], s2, i2);
            const int pos = __popc(__ballot_sync(FULL, above));
            const float us = __shfl_up_sync(FULL, ls[j], 1);
            const int ui = __shfl_up_sync(FULL, li[j], 1);
            if (lane < KEEP && lane > pos) {
              ls[j] = us;
              li[j] = ui;
            }
            if (lane == pos) {
              ls[j] = s2;
              li[j] = i2;
            }
          }
        }
      }
      if (!ok) break;
      if constexpr (ALL) continue;
      // unit end: the four quadrant lists of each query -> one top-16 per (query, split)
      if (lane < KEEP) {
#pragma unroll
        for (int j = 0; j < 8; ++j) lists[(ew * 8 + j) * KEEP + lane] = make_float2(ls[j], __int_as_float(li[j]));
      }
      gs.sync(lane);
      // warp ew merges queries 2 ew, 2 ew + 1 of the chunk: 4 lists of 16 each
#pragma unroll 1
      for (int jj = 0; jj < 2; ++jj) {
        const int jq = 2 * ew + jj, h = jq >> 3, jl = jq & 7;
        // candidates: warps with hq == h are ew' = 4h + q' (q' = 0..3)
        float cs0 = -INFINITY, cs1 = -INFINITY;
        int ci0 = INT_MAX, ci1 = INT_MAX;
        {
          const int e0 = lane, e1 = lane + 32;  // 64 candidates: list q' = e / 16, entry e % 16
          const float2 v0 = lists[((4 * h + e0 / KEEP) * 8 + jl) * KEEP + e0 % KEEP];
          const float2 v1 = lists[((4 * h + e1 / KEEP) * 8 + jl) * KEEP + e1 % KEEP];
          cs0 = v0.x, ci0 = __float_as_int(v0.y);
          cs1 = v1.x, ci1 = __float_as_int(v1.y);
        }
        bool t0 = false, t1 = false;
        const int64_t qrow = chunk * QC + jq;
        for (int r = 0; r < KEEP; ++r) {  // 16 rounds of a warp-wide maximum
          float bs;
          int bi, bl;
          if (!t0 && (t1 || better(cs0, ci0, cs1, ci1))) {
            bs = cs0, bi = ci0, bl = 0;
          } else if (!t1) {
            bs = cs1, bi = ci1, bl = 1;
          } else {
            bs = -INFINITY, bi = INT_MAX, bl = 2;
          }
          float ws = bs;
          int wi = bi, wl = bl == 2 ? 64 : lane + 32 * bl;
#pragma unroll
          for (int o = 16; o; o >>= 1) {
            const float s2 = __shfl_xor_sync(FULL, ws, o);
            const int i2 = __shfl_xor_sync(FULL, wi, o);
            const int l2 = __shfl_xor_sync(FULL, wl, o);
            if (l2 < 64 && (wl == 64 || better(s2, i2, ws, wi) || (s2 == ws && i2 == wi && l2 < wl))) {
              ws = s2;
              wi = i2;
              wl = l2;
            }
          }
          if (wl < 64 && (wl & 31) == lane) {
            if (wl < 32) t0 = true;
            else t1 = true;
          }
          if (lane == 0 && qrow < a.n_q)
            a.cand[(qrow * a.nsplit + split) * KEEP + r] = make_float2(wl < 64 ? ws : -INFINITY,
                                                                        __int_as_float(wl < 64 ? wi : INT_MAX));
        }
      }
      gs.sync(lane);  // the lists buffer is free for the next unit
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

template <int KB, int SI, bool ALL>
int launch_stc(const SArgsTC& a, int sm, cudaStream_t st) {
  using L = SL<KB, SI>;
  auto kern = search_tc_kernel<KB, SI, ALL>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::SMEM);
  if (e != cudaSuccess) return tq::set_error(TQ_ECUDA, "tq_search_topk: %s", cudaGetErrorString(e));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)std::max<int64_t>(1, std::min<int64_t>(sm, a.n_units)));
  cfg.blockDim = dim3(L::NTHREADS);
  cfg.dynamicSmemBytes = L::SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, a);
  if (e != cudaSuccess) return tq::set_error(TQ_ECUDA, "tq_search_topk: launch failed: %s", cudaGetErrorString(e));
  return TQ_OK;
}

template <bool ALL>
int dispatch_stc(int kb, int si, const SArgsTC& a, int sm, cudaStream_t st) {
  if (si) {
    switch (kb) {
      case 1: return launch_stc<1, 1, ALL>(a, sm, st);
      case 2: return launch_stc<2, 1, ALL>(a, sm, st);
      default: return launch_stc<3, 1, ALL>(a, sm, st);
    }
  }
  switch (kb) {
    case 1: return launch_stc<1, 0, ALL>(a, sm, st);
    case 2: return launch_stc<2, 0, ALL>(a, sm, st);
    default: return launch_stc<3, 0, ALL>(a, sm, st);
  }
}

int image_bytes(int kb, int si) {
  const int nt = walsh_planes(kb);
  return 256 + (nt + si) * 16 * 1024;
}

int splits_for(int64_t n_db) { return (int)std::max<int64_t>(1, std::min<int64_t>(MAX_SPLITS, (n_db + 16383) / 16384)); }

// The images of every (head, 16-query chunk), then the scan.
int run_stc(const tq_params* p, int kb, const float* q, int n_heads, int group, const void* codes,
            const uint16_t* norms, const uint16_t* rnorms, int64_t n_keys, void* workspace, bool all, float* logits,
            int64_t ld, float2** cand, int* nsplit, cudaStream_t st) {
  const int m = p->mode == TQ_MODE_PROD ? p->m : 0;
  const int si = m > 0 ? 1 : 0;
  const int n_chunks = (group + QC - 1) / QC;
  const int ib = image_bytes(kb, si);
  PrepS pa;
  pa.q = q;
  pa.n_q = n_heads * group;
  pa.d = p->d;
  pa.kb = kb;
  pa.m = m;
  pa.group = group;
  pa.n_chunks = n_chunks;
  pa.cent = p->centroids;
  pa.D = p->signs_D;
  pa.S = p->S;
  pa.img = static_cast<uint8_t*>(workspace);
  pa.img_bytes = ib;
  pa.np = walsh_planes(kb) + si;
  search_prep_kernel<<<n_heads * n_chunks, 256, 0, st>>>(pa);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return tq::set_error(TQ_ECUDA, "tensor-core scan: prep launch failed: %s", cudaGetErrorString(e));
  SArgsTC a;
  a.codes = static_cast<const uint8_t*>(codes);
  a.norms = norms;
  a.rnorms = rnorms;
  a.n_db = n_keys;
  a.n_q = n_heads * group;
  a.n_chunks = n_chunks;
  a.group = group;
  a.nsplit = all ? (int)std::max<int64_t>(1, std::min<int64_t>(MAX_SPLITS, (n_keys + 4095) / 4096)) : splits_for(n_keys);
  a.tb = tqd::tile_bytes(256, kb, m);
  a.split_keys = ((n_keys + a.nsplit - 1) / a.nsplit + TK - 1) / TK * TK;
  a.n_units = (int64_t)n_heads * a.nsplit * n_chunks;
  a.img = pa.img;
  a.img_bytes = ib;
  const int64_t img_total = ((int64_t)n_heads * n_chunks * ib + 255) & ~(int64_t)255;
  a.cand = all ? nullptr : reinterpret_cast<float2*>(static_cast<uint8_t*>(workspace) + img_total);
  a.logits = logits;
  a.ld = ld;
  a.kappa = (float)(std::sqrt(M_PI / 2.0) / (m > 0 ? m : 1));
  if (cand) *cand = a.cand;
  if (nsplit) *nsplit = a.nsplit;
  const int sm = tq::sm_count();
  return all ? dispatch_stc<true>(kb, si, a, sm, st) : dispatch_stc<false>(kb, si, a, sm, st);
}

}  // namespace

namespace tq {

bool search_tc_supported(int dp, int kb, int m) { return dp == 256 && kb >= 1 && kb <= 3 && (m == 0 || m == 256); }

// Workspace of the tensor-core search: the chunk images, then the split candidates.
int64_t search_tc_workspace(int kb, int m, int n_q, int64_t n_db) {
  const int n_chunks = (n_q + QC - 1) / QC;
  const int64_t img = ((int64_t)n_chunks * image_bytes(kb, m > 0 ? 1 : 0) + 255) & ~(int64_t)255;
  return img + (int64_t)n_q * splits_for(n_db) * KEEP * 8;
}

// Prep + scan; the candidates [n_q][*nsplit][16] (score, id bits) are left in the workspace for the split merge.
int launch_search_tc(const tq_params* p, int kb, const float* q, int n_q, const void* codes, const uint16_t* norms,
                     const uint16_t* rnorms, int64_t n_db, void* workspace, float2** cand, int* nsplit,
                     cudaStream_t st) {
  return run_stc(p, kb, q, 1, n_q, codes, norms, rnorms, n_db, workspace, false, nullptr, 0, cand, nsplit, st);
}

// Logits on the same scan (d_pad 256): bytes of the query images for n_q = n_heads * group queries
// (an upper bound over every split of n_q into heads and groups).
int64_t logits_stc_workspace(int kb, int m, int n_q) { return (int64_t)n_q * image_bytes(kb, m > 0 ? 1 : 0) + 256; }

int launch_logits_stc(const tq_params* p, int kb, const float* q, int n_heads, int group, const void* codes,
                      const uint16_t* norms, const uint16_t* rnorms, int64_t n_keys, float* logits, int64_t ld,
                      void* workspace, cudaStream_t st) {
  return run_stc(p, kb, q, n_heads, group, codes, norms, rnorms, n_keys, workspace, true, logits, ld, nullptr,
                 nullptr, st);
}

}  // namespace tq

namespace tq {
// Read (and optionally clear) this translation unit's device fault word.
int fault_word_search(int clear, int* value) {
  cudaError_t e = cudaMemcpyFromSymbol(value, tqd::g_fault, sizeof(int));
  if (e == cudaSuccess && clear) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(tqd::g_fault, &zero, sizeof(int));
  }
  return e == cudaSuccess ? TQ_OK : set_error(TQ_ECUDA, "tq_device_status: %s", cudaGetErrorString(e));
}
}  // namespace tq
