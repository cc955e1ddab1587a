// tq_search_topk: top-k inner-product search over quantized vectors
// ("TurboQuant explainer" (m.163.com), "向量搜索": nearest-neighbour search
// by inner product on TurboQuant codes, no training or tuning of the codebook).
//
// Scores are the logit estimator of tq_logits (scan.cuh) with each query on
// its own.  A CTA takes one chunk of 4 queries and one contiguous database
// split; CTAs are ordered split-major so the chunks that share a split run
// together and re-read it from L2.  The chunk's A fragments sit in shared
// memory (one 16-byte slot per MMA), and each warp applies every slot to
// NB = 4 subtiles (32 keys) before moving on, so one shared-memory load feeds
// four MMAs.  Each lane keeps a sorted top-16 (score desc, id asc) for its
// query in registers; the CTA merges its 16 lists per query into one, and a
// final kernel merges the splits.
#include <cuda_runtime.h>

#include <algorithm>
#include <cfloat>
#include <climits>
#include <cmath>

#include "common.h"
#include "prep.h"
#include "scan.cuh"

namespace {
using namespace tqd;

constexpr int KM = 16;  // candidates kept per list
constexpr int NB = 4;   // subtiles per warp step

struct SArgs {
  const uint8_t* codes;
  const uint16_t* norms;
  const uint16_t* rnorms;
  int64_t n_db;
  int n_q, nqc, nsplit, m, tb;
  const uint8_t* prep;
  int64_t prep_bytes;
  float2* cand;  // [n_q][nsplit][KM] (score, id bits)
  float kappa;
};

__device__ __forceinline__ bool better(float s, int i, float s2, int i2) { return s > s2 || (s == s2 && i < i2); }

__device__ __forceinline__ void topk_insert(float (&ts)[KM], int (&ti)[KM], float s, int id) {
  if (!better(s, id, ts[KM - 1], ti[KM - 1])) return;
  ts[KM - 1] = s;
  ti[KM - 1] = id;
#pragma unroll
  for (int j = KM - 1; j > 0; --j) {
    if (better(ts[j], ti[j], ts[j - 1], ti[j - 1])) {
      const float a = ts[j];
      ts[j] = ts[j - 1];
      ts[j - 1] = a;
      const int b = ti[j];
      ti[j] = ti[j - 1];
      ti[j - 1] = b;
    }
  }
}

// Warp-wide selection of the best `k` of n candidates in smem (cs, ci); results to out_s/out_i (lane 0 writes).
__device__ void warp_select(const float* cs, const int* ci, int n, int k, float* out_s, int* out_i, int lane) {
  unsigned taken_lo = 0;  // per lane: candidates lane + 32 j, j < 32, already chosen
  for (int r = 0; r < k; ++r) {
    float bs = -INFINITY;
    int bi = INT_MAX, bj = -1;
    for (int j = 0; j * 32 + lane < n && j < 32; ++j) {
      if (taken_lo & (1u << j)) continue;
      const float s = cs[j * 32 + lane];
      const int id = ci[j * 32 + lane];
      if (bj < 0 || better(s, id, bs, bi)) {
        bs = s;
        bi = id;
        bj = j;
      }
    }
    float ws = bs;
    int wi = bi, wl = (bj >= 0) ? lane : 32;
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      const float s2 = __shfl_xor_sync(FULL, ws, o);
      const int i2 = __shfl_xor_sync(FULL, wi, o);
      const int l2 = __shfl_xor_sync(FULL, wl, o);
      if (l2 < 32 && (wl == 32 || better(s2, i2, ws, wi))) {
        ws = s2;
        wi = i2;
        wl = l2;
      }
    }
    if (wl == lane) taken_lo |= 1u << bj;
    if (lane == 0) {
      out_s[r] = (wl < 32) ? ws : -INFINITY;
      out_i[r] = (wl < 32) ? wi : INT_MAX;
    }
  }
}

template <int DP, int KB, int SI>
__global__ void __launch_bounds__(128) search_kernel(const SArgs a) {
  using SC = Scan<DP, KB, SI>;
  constexpr int NH = DP / 128;
  constexpr int SW = SI > 0 ? SI : 1;
  extern __shared__ uint4 afrag[];  // SC::FR / 4 * 32
  __shared__ float ms[QCHUNK][16 * KM];
  __shared__ int mi[QCHUNK][16 * KM];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int chunk = blockIdx.x % a.nqc, split = blockIdx.x / a.nqc;
  const int g = lane >> 2, t = lane & 3;
  const int qrow = QCHUNK * chunk + (g & 3);
  const int64_t n_sub = (a.n_db + 7) / 8;
  const int64_t per = (n_sub + a.nsplit - 1) / a.nsplit;
  const int64_t s_begin = (int64_t)split * per;
  const int64_t s_end = min(n_sub, s_begin + per);

  grid_dependency_wait();
  const uint8_t* prep = a.prep + (int64_t)chunk * a.prep_bytes;
  SC::stage(afrag, prep);
  const float4 qs = reinterpret_cast<const float4*>(prep + SC::FR * 128)[g & 3];
  __syncthreads();

  float ts[KM];
  int ti[KM];
#pragma unroll
  for (int j = 0; j < KM; ++j) {
    ts[j] = -INFINITY;
    ti[j] = INT_MAX;
  }
  for (int64_t s0 = s_begin + (int64_t)warp * NB; s0 < s_end; s0 += 4 * NB) {
    uint32_t bw[NB][KB][NH], sw[NB][SW];
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      const int64_t kk = 8 * (s0 + b) + g;
      load_words<DP, KB, SI>(a.codes, a.tb, a.m, kk, (s0 + b < s_end) && kk < a.n_db, t, bw[b], sw[b]);
    }
    int accC[NB][2][4] = {}, accS[NB][2][4] = {};
    uint32_t it[NB][SC::NCI];
#pragma unroll
    for (int b = 0; b < NB; ++b)
#pragma unroll
      for (int T = 0; T < SC::NT; ++T)
#pragma unroll
        for (int h = 0; h < NH; ++h)
          it[b][T * NH + h] = (KB == 3 && T == 3) ? (bw[b][0][h] ^ bw[b][1][h] ^ bw[b][2][h]) : bw[b][T][h];
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const uint32_t mk = 0x01010101u << c;
      const uint4* slot = afrag + c * SC::NSLOT * 32 + lane;
#pragma unroll
      for (int p = 0; p < SC::NCP; ++p) {
        const uint4 A = slot[p * 32];
#pragma unroll
        for (int b = 0; b < NB; ++b)
          mma_s8u8_16832(accC[b][c & 1], A.x, A.y, A.z, A.w, it[b][2 * p] & mk, it[b][2 * p + 1] & mk);
      }
      if constexpr (SC::NCS) {
        const uint4 A = slot[SC::NCP * 32];
#pragma unroll
        for (int b = 0; b < NB; ++b) mma_s8u8_16816(accC[b][c & 1], A.x, A.y, it[b][SC::NCI - 1] & mk);
      }
      if constexpr (SC::NSP) {
        const uint4 A = slot[(SC::NCP + SC::NCS) * 32];
#pragma unroll
        for (int b = 0; b < NB; ++b)
          mma_s8u8_16832(accS[b][c & 1], A.x, A.y, A.z, A.w, sw[b][0] & mk, sw[b][SI > 1 ? 1 : 0] & mk);
      }
      if constexpr (SC::NSS) {
        const uint4 A = slot[(SC::NCP + SC::NCS) * 32];
#pragma unroll
        for (int b = 0; b < NB; ++b) mma_s8u8_16816(accS[b][c & 1], A.x, A.y, sw[b][0] & mk);
      }
    }
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      float c0, c1, z0 = 0.f, z1 = 0.f;
      combine_digits(accC[b], lane, c0, c1);
      if constexpr (SI > 0) combine_digits(accS[b], lane, z0, z1);
      if (lane < 16 && qrow < a.n_q) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int64_t key = 8 * (s0 + b) + 2 * t + e;
          if (s0 + b < s_end && key < a.n_db) {
            const float n = __half2float(__ushort_as_half(a.norms[key]));
            float l = fmaf(e ? c1 : c0, qs.x, -qs.y);
            if constexpr (SI > 0) {
              const float gm = __half2float(__ushort_as_half(a.rnorms[key]));
              l = fmaf(gm * a.kappa, fmaf(e ? z1 : z0, qs.z, -qs.w), l);
            }
            topk_insert(ts, ti, n * l, (int)key);
          }
        }
      }
    }
  }
  // merge: 16 lists per query (4 warps x 4 lanes) -> one list per (query, split)
  if (lane < 16) {
    const int list = warp * 4 + t;
#pragma unroll
    for (int j = 0; j < KM; ++j) {
      ms[g][list * KM + j] = ts[j];
      mi[g][list * KM + j] = ti[j];
    }
  }
  __syncthreads();
  {
    const int q = warp;  // warp q merges query q of the chunk
    __shared__ float os[QCHUNK][KM];
    __shared__ int oi[QCHUNK][KM];
    warp_select(ms[q], mi[q], 16 * KM, KM, os[q], oi[q], lane);
    __syncwarp();
    const int qr = QCHUNK * chunk + q;
    if (qr < a.n_q && lane < KM) {
      float2 v;
      v.x = os[q][lane];
      v.y = __int_as_float(oi[q][lane]);
      a.cand[((int64_t)qr * a.nsplit + split) * KM + lane] = v;
    }
  }
}

struct MArgs {
  const float2* cand;
  int n_q, nsplit, k;
  int32_t* ids;
  float* scores;
};

__global__ void __launch_bounds__(32) merge_kernel(const MArgs a) {
  extern __shared__ float buf[];
  const int q = blockIdx.x, lane = threadIdx.x;
  const int n = a.nsplit * KM;
  float* cs = buf;
  int* ci = reinterpret_cast<int*>(buf + n);
  float* os = reinterpret_cast<float*>(ci + n);
  int* oi = reinterpret_cast<int*>(os + KM);
  const float2* src = a.cand + (int64_t)q * n;
  for (int j = lane; j < n; j += 32) {
    const float2 v = src[j];
    cs[j] = v.x;
    ci[j] = __float_as_int(v.y);
  }
  __syncwarp();
  // candidates per lane may exceed 32 words of the taken mask: select in rounds of 1024
  warp_select(cs, ci, min(n, 1024), a.k, os, oi, lane);
  __syncwarp();
  if (lane < a.k) {
    a.ids[(int64_t)q * a.k + lane] = oi[lane];
    a.scores[(int64_t)q * a.k + lane] = os[lane];
  }
}

// Merge of per-shard top-k lists (a database split across devices, "TurboQuant
// explainer" (m.163.com), "向量搜索"): one warp per query gathers the n_parts x k
// candidates with their shard offsets and selects the k best, ties to the lower id.
constexpr int MAX_SHARDS = 64;
struct ShardMergeArgs {
  const int32_t* ids;    // [n_parts][n_q][k] shard-local
  const float* scores;   // [n_parts][n_q][k]
  int n_parts, n_q, k;
  int64_t offs[MAX_SHARDS];
  int32_t* out_ids;
  float* out_scores;
};

__global__ void __launch_bounds__(32) shard_merge_kernel(const ShardMergeArgs a) {
  extern __shared__ float sbuf[];
  const int q = blockIdx.x, lane = threadIdx.x;
  const int n = a.n_parts * a.k;
  float* cs = sbuf;
  int* ci = reinterpret_cast<int*>(sbuf + n);
  float* os = reinterpret_cast<float*>(ci + n);
  int* oi = reinterpret_cast<int*>(os + KM);
  for (int j = lane; j < n; j += 32) {
    const int part = j / a.k, r = j - part * a.k;
    const int64_t src = ((int64_t)part * a.n_q + q) * a.k + r;
    const int id = a.ids[src];
    const float sc = a.scores[src];
    const bool empty = id < 0 || id == INT_MAX || !(sc > -INFINITY);
    cs[j] = empty ? -INFINITY : sc;
    ci[j] = empty ? INT_MAX : (int)(id + a.offs[part]);
  }
  __syncwarp();
  warp_select(cs, ci, n, a.k, os, oi, lane);
  __syncwarp();
  if (lane < a.k) {
    a.out_ids[(int64_t)q * a.k + lane] = oi[lane];
    a.out_scores[(int64_t)q * a.k + lane] = os[lane];
  }
}

int search_nsplit(int64_t n_db) {
  // each split should give every warp a few hundred keys; at most 32 splits (merge handles 1024 candidates)
  const int64_t per = 8192;
  return (int)std::max<int64_t>(1, std::min<int64_t>(32, (n_db + per - 1) / per));
}

template <int DP, int KB, int SI>
int launch_search(const SArgs& a, cudaStream_t st) {
  using SC = Scan<DP, KB, SI>;
  const int smem = SC::FR / 4 * 32 * 16;
  auto kern = search_kernel<DP, KB, SI>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return tq::set_error(TQ_ECUDA, "tq_search_topk: %s", cudaGetErrorString(e));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((int64_t)a.nqc * a.nsplit));
  cfg.blockDim = dim3(128);
  cfg.dynamicSmemBytes = smem;
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

template <int DP, int KB>
int dispatch_si(int si, const SArgs& a, cudaStream_t st) {
  switch (si) {
    case 0: return launch_search<DP, KB, 0>(a, st);
    case 1: return launch_search<DP, KB, 1>(a, st);
    default: return launch_search<DP, KB, 2>(a, st);
  }
}

int64_t prep_bytes_for(const tq_params* p, int n_q) {
  const int kb = p->mode == TQ_MODE_PROD ? p->bits - 1 : p->bits;
  const tqd::ScanShape sh(p->d_pad, kb, p->mode == TQ_MODE_PROD ? p->m : 0);
  const int nqc = (n_q + tqd::QCHUNK - 1) / tqd::QCHUNK;
  return ((int64_t)nqc * tqd::prep_chunk_bytes(sh.fr) + 255) & ~(int64_t)255;
}

}  // namespace

extern "C" int64_t tq_search_workspace(const tq_params* p, int n_q, int64_t n_db, int k) {
  if (!p || n_q < 0 || n_db < 0 || k < 1) return -1;
  const int kb = p->mode == TQ_MODE_PROD ? p->bits - 1 : p->bits;
  if (kb < 1 || kb > 4 || (p->d_pad != 128 && p->d_pad != 256)) return -1;
  const int m = p->mode == TQ_MODE_PROD ? p->m : 0;
  if (tq::search_tc_supported(p->d_pad, kb, m)) return tq::search_tc_workspace(kb, m, n_q, n_db);
  return prep_bytes_for(p, n_q) + (int64_t)n_q * search_nsplit(n_db) * KM * 8;
}

extern "C" int tq_search_topk(const tq_params* p, const float* q, int n_q, const void* codes, const uint16_t* norms,
                              const uint16_t* rnorms, int64_t n_db, int k, int32_t* ids, float* scores,
                              void* workspace, int64_t workspace_bytes, tq_stream_t stream) {
  using namespace tq;
  int rc = check_params(p, "tq_search_topk");
  if (!rc) rc = check_planes(p, "tq_search_topk");
  if (rc) return rc;
  const int kb = index_bits(p);
  const bool prod = p->mode == TQ_MODE_PROD;
  if (kb > 3) return set_error(TQ_EUNSUPPORTED, "tq_search_topk: at most 3 index bits");
  if (k < 1 || k > KM) return set_error(TQ_EUNSUPPORTED, "tq_search_topk: k must be in 1..%d", KM);
  if (n_q < 0 || n_db < 0 || n_db > INT_MAX) return set_error(TQ_EINVAL, "tq_search_topk: bad n_q/n_db");
  if (n_q == 0) {
    clear_error();
    return TQ_OK;
  }
  if (n_db < k) return set_error(TQ_EINVAL, "tq_search_topk: n_db < k");
  if (!q || !codes || !norms || !ids || !scores || !workspace || (prod && !rnorms))
    return set_error(TQ_EINVAL, "tq_search_topk: NULL pointer argument");
  if (!aligned(codes, 16) || !aligned(workspace, 16))
    return set_error(TQ_EINVAL, "tq_search_topk: codes and workspace must be 16-byte aligned");
  const int64_t need = tq_search_workspace(p, n_q, n_db, k);
  if (workspace_bytes < need)
    return set_error(TQ_EINVAL, "tq_search_topk: workspace too small (%lld < %lld)", (long long)workspace_bytes,
                     (long long)need);
  const int m = prod ? p->m : 0;
  const tqd::ScanShape sh(p->d_pad, kb, m);
  const int nqc = (n_q + tqd::QCHUNK - 1) / tqd::QCHUNK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (search_tc_supported(p->d_pad, kb, m)) {  // tensor-memory scan, then the split merge
    float2* cand = nullptr;
    int nsplit = 0;
    rc = launch_search_tc(p, kb, q, n_q, codes, norms, rnorms, n_db, workspace, &cand, &nsplit, st);
    if (rc) return rc;
    MArgs ma;
    ma.cand = cand;
    ma.n_q = n_q;
    ma.nsplit = nsplit;
    ma.k = k;
    ma.ids = ids;
    ma.scores = scores;
    const int msmem = (2 * nsplit * KM + 2 * KM) * 4;
    merge_kernel<<<n_q, 32, msmem, st>>>(ma);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return set_error(TQ_ECUDA, "tq_search_topk: merge launch failed: %s", cudaGetErrorString(e));
    clear_error();
    return TQ_OK;
  }
  tqd::PrepArgs pa;
  pa.q = q;
  pa.d = p->d;
  pa.dp = p->d_pad;
  pa.kb = kb;
  pa.m = m;
  pa.n_outer = 1;
  pa.group = n_q;
  pa.nqc = nqc;
  pa.cent = p->centroids;
  pa.D = p->signs_D;
  pa.S = p->S;
  pa.out = static_cast<uint8_t*>(workspace);
  pa.fr = sh.fr;
  rc = launch_prep(pa, st);
  if (rc) return rc;
  SArgs a;
  a.codes = static_cast<const uint8_t*>(codes);
  a.norms = norms;
  a.rnorms = rnorms;
  a.n_db = n_db;
  a.n_q = n_q;
  a.nqc = nqc;
  a.nsplit = search_nsplit(n_db);
  a.m = m;
  a.tb = tqd::tile_bytes(p->d_pad, kb, m);
  a.prep = pa.out;
  a.prep_bytes = tqd::prep_chunk_bytes(sh.fr);
  a.cand = reinterpret_cast<float2*>(static_cast<uint8_t*>(workspace) + prep_bytes_for(p, n_q));
  a.kappa = (float)(std::sqrt(M_PI / 2.0) / (m > 0 ? m : 1));
  const int si = sh.nsi;
  if (p->d_pad == 128) {
    switch (kb) {
      case 1: rc = dispatch_si<128, 1>(si, a, st); break;
      case 2: rc = dispatch_si<128, 2>(si, a, st); break;
      default: rc = dispatch_si<128, 3>(si, a, st); break;
    }
  } else {
    switch (kb) {
      case 1: rc = dispatch_si<256, 1>(si, a, st); break;
      case 2: rc = dispatch_si<256, 2>(si, a, st); break;
      default: rc = dispatch_si<256, 3>(si, a, st); break;
    }
  }
  if (rc) return rc;
  MArgs ma;
  ma.cand = a.cand;
  ma.n_q = n_q;
  ma.nsplit = a.nsplit;
  ma.k = k;
  ma.ids = ids;
  ma.scores = scores;
  const int msmem = a.nsplit * KM * 8 + KM * 8;
  merge_kernel<<<n_q, 32, msmem, st>>>(ma);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(TQ_ECUDA, "tq_search_topk: merge launch failed: %s", cudaGetErrorString(e));
  clear_error();
  return TQ_OK;
}

extern "C" int tq_search_merge(const int32_t* ids, const float* scores, int n_parts, const int64_t* id_offsets,
                               int n_q, int k, int32_t* out_ids, float* out_scores, tq_stream_t stream) {
  using namespace tq;
  if (n_parts < 1 || n_parts > MAX_SHARDS || k < 1 || k > KM || n_parts * k > 1024 || n_q < 0)
    return set_error(TQ_EINVAL, "tq_search_merge: need 1 <= n_parts <= %d, 1 <= k <= %d, n_parts * k <= 1024",
                     MAX_SHARDS, KM);
  if (n_q == 0) {
    clear_error();
    return TQ_OK;
  }
  if (!ids || !scores || !id_offsets || !out_ids || !out_scores)
    return set_error(TQ_EINVAL, "tq_search_merge: NULL pointer argument");
  if (!aligned(ids, 4) || !aligned(scores, 4) || !aligned(out_ids, 4) || !aligned(out_scores, 4))
    return set_error(TQ_EINVAL, "tq_search_merge: misaligned pointer");
  ShardMergeArgs a;
  a.ids = ids;
  a.scores = scores;
  a.n_parts = n_parts;
  a.n_q = n_q;
  a.k = k;
  for (int p = 0; p < MAX_SHARDS; ++p) a.offs[p] = 0;
  for (int p = 0; p < n_parts; ++p) {
    if (id_offsets[p] < 0 || id_offsets[p] >= INT_MAX)
      return set_error(TQ_EINVAL, "tq_search_merge: id offset %lld out of range", (long long)id_offsets[p]);
    a.offs[p] = id_offsets[p];
  }
  a.out_ids = out_ids;
  a.out_scores = out_scores;
  const int n = n_parts * k;
  const int smem = (2 * n + 2 * KM) * 4;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  shard_merge_kernel<<<n_q, 32, smem, st>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(TQ_ECUDA, "tq_search_merge: launch failed: %s", cudaGetErrorString(e));
  clear_error();
  return TQ_OK;
}
