// tq_logits: attention logits straight from the packed codes
// ("TurboQuant explainer" (m.163.com), "第二步：QJL" estimator; "速度":
// logits from 4-bit codes).
//
// One CTA (4 warps) scans a contiguous key range for one KV head and one
// chunk of 4 query heads; each warp takes 8-key subtiles.  Per subtile a lane
// loads its key's plane words with plain coalesced 32-bit loads (a warp reads
// 8 keys x 16 B per plane = 128 contiguous bytes), the next subtile's words
// are prefetched while the current one runs on the tensor cores (int8
// mma.sync, exact integer sums, see scan.cuh), and lanes 0..15 write the
// logits of their (query, key pair).
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <mutex>

#include "common.h"
#include "prep.h"
#include "scan.cuh"

namespace {
using namespace tqd;

struct LArgs {
  const uint8_t* codes;
  const uint16_t* norms;
  const uint16_t* rnorms;
  int64_t n_keys;
  int group, nqc, nsplit, m, tb;
  const uint8_t* prep;
  int64_t prep_bytes;
  float* logits;
  int64_t ld;  // logits row stride (>= n_keys)
  float kappa;
};

template <int DP, int KB, int SI>
__global__ void __launch_bounds__(128) logits_kernel(const LArgs a) {
  using SC = Scan<DP, KB, SI>;
  constexpr int NH = DP / 128;
  constexpr int SW = SI > 0 ? SI : 1;
  __shared__ uint4 afrag[SC::FR / 4 * 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int chunk = blockIdx.x / a.nsplit, split = blockIdx.x % a.nsplit;
  const int head = chunk / a.nqc, qc = chunk % a.nqc;
  const int g = lane >> 2, t = lane & 3;
  const int qrow = QCHUNK * qc + (g & 3);
  const bool qvalid = (lane < 16) && (qrow < a.group);
  const int64_t n_sub = (a.n_keys + 7) / 8;
  const int64_t per = (n_sub + a.nsplit - 1) / a.nsplit;
  const int64_t s_begin = (int64_t)split * per;
  const int64_t s_end = min(n_sub, s_begin + per);
  const int64_t vbase = (int64_t)head * a.n_keys;
  float* out = a.logits + ((int64_t)head * a.group + qrow) * a.ld;

  // first code words do not depend on the query prep: fetch them before waiting for it
  uint32_t bw[KB][NH], sw[SW];
  int64_t s = s_begin + warp;
  if (s < s_end) {
    const int64_t kk = 8 * s + g;
    load_words<DP, KB, SI>(a.codes, a.tb, a.m, vbase + kk, kk < a.n_keys, t, bw, sw);
  }
  grid_dependency_wait();
  const uint8_t* prep = a.prep + (int64_t)chunk * a.prep_bytes;
  SC::stage(afrag, prep);
  const float4 qs = reinterpret_cast<const float4*>(prep + SC::FR * 128)[g & 3];
  __syncthreads();
  SC sc;
  sc.load(reinterpret_cast<const uint8_t*>(afrag), lane);

  for (; s < s_end; s += 4) {
    uint32_t cbw[KB][NH], csw[SW];
#pragma unroll
    for (int p = 0; p < KB; ++p)
#pragma unroll
      for (int h = 0; h < NH; ++h) cbw[p][h] = bw[p][h];
#pragma unroll
    for (int i = 0; i < SW; ++i) csw[i] = sw[i];
    const int64_t sn = s + 4;
    if (sn < s_end) {
      const int64_t kk = 8 * sn + g;
      load_words<DP, KB, SI>(a.codes, a.tb, a.m, vbase + kk, kk < a.n_keys, t, bw, sw);
    }
    int accC[2][SC::NCSL][4] = {}, accS[2][4] = {}, accF[2][4];
    sc.run(accC, accS, cbw, csw);
    SC::fold(accC, accF);
    float c0, c1, z0 = 0.f, z1 = 0.f;
    combine_digits(accF, lane, c0, c1);
    if constexpr (SI > 0) combine_digits(accS, lane, z0, z1);
    if (qvalid) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int64_t key = 8 * s + 2 * t + e;
        if (key < a.n_keys) {
          const int64_t v = vbase + key;
          const float n = __half2float(__ushort_as_half(a.norms[v]));
          float l = fmaf(e ? c1 : c0, qs.x, -qs.y);
          if constexpr (SI > 0) {
            const float gm = __half2float(__ushort_as_half(a.rnorms[v]));
            l = fmaf(gm * a.kappa, fmaf(e ? z1 : z0, qs.z, -qs.w), l);
          }
          out[key] = n * l;
        }
      }
    }
  }
}

// Streaming variant for key ranges whose 8-key subtiles never straddle a
// 32-vector tile (head offsets that are multiples of 8): each warp keeps a
// ring of RS subtiles in shared memory filled by cp.async (16-byte copies of
// the plane rows, sign rows and the 8 norms / residual norms), so RS-1
// subtiles (~3.8 KB per warp) are always in flight from HBM.
constexpr int RS = 8;

template <int DP, int KB, int SI>
struct Ring {
  static constexpr int PLANE = 8 * (DP / 8);         // bytes of one plane for 8 keys
  static constexpr int SIGN = SI ? 8 * 32 * SI : 0;  // bytes reserved for 8 keys' sign rows (m <= 128*SI)
  static constexpr int STAGE = KB * PLANE + SIGN + 32;
};

template <int DP, int KB, int SI>
__global__ void __launch_bounds__(128) logits_ring_kernel(const LArgs a) {
  using SC = Scan<DP, KB, SI>;
  using RG = Ring<DP, KB, SI>;
  constexpr int NH = DP / 128;
  constexpr int SW = SI > 0 ? SI : 1;
  __shared__ uint4 afrag[SC::FR / 4 * 32];
  __shared__ __align__(16) uint8_t ring[4][RS][RG::STAGE];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int chunk = blockIdx.x / a.nsplit, split = blockIdx.x % a.nsplit;
  const int head = chunk / a.nqc, qc = chunk % a.nqc;
  const int g = lane >> 2, t = lane & 3;
  const int qrow = QCHUNK * qc + (g & 3);
  const bool qvalid = (lane < 16) && (qrow < a.group);
  const int64_t n_sub = (a.n_keys + 7) / 8;
  const int64_t per = (n_sub + a.nsplit - 1) / a.nsplit;
  const int64_t s_begin = (int64_t)split * per;
  const int64_t s_end = min(n_sub, s_begin + per);
  const int64_t vbase = (int64_t)head * a.n_keys;
  float* out = a.logits + ((int64_t)head * a.group + qrow) * a.ld;
  const int sbytes = a.m / 8;  // sign bytes per key
  const int n_sign_cp = SI ? (8 * sbytes) / 16 : 0;
  const int n_cp = KB * 8 + n_sign_cp + 2;

  // copy subtile s into ring stage st (whole subtile lies in one tile; tail keys of the
  // last tile are zero-filled codes, their logits are not written)
  auto issue = [&](int64_t s, int st) {
    if (s < s_end) {
      const int64_t v0 = vbase + 8 * s;
      const uint8_t* tb = a.codes + (v0 >> 5) * a.tb;
      const int slot0 = (int)(v0 & 31);
      uint8_t* dst = ring[warp][st];
      for (int c = lane; c < n_cp; c += 32) {
        const uint8_t* src;
        uint8_t* d;
        if (c < KB * 8) {
          const int p = c >> 3, r = c & 7;
          src = tb + p * TILE * (DP / 8) + (slot0 + r) * (DP / 8);
          d = dst + p * RG::PLANE + r * (DP / 8);
          if (DP == 256) {  // two 16-byte halves per 32-byte row
            cp_async16(d, src);
            cp_async16(d + 16, src + 16);
            continue;
          }
        } else if (c < KB * 8 + n_sign_cp) {
          const int k = c - KB * 8;
          src = tb + KB * TILE * (DP / 8) + slot0 * sbytes + 16 * k;
          d = dst + KB * RG::PLANE + 16 * k;
        } else if (c == KB * 8 + n_sign_cp) {
          src = reinterpret_cast<const uint8_t*>(a.norms + v0);
          d = dst + KB * RG::PLANE + RG::SIGN;
        } else {
          if (!SI) continue;
          src = reinterpret_cast<const uint8_t*>(a.rnorms + v0);
          d = dst + KB * RG::PLANE + RG::SIGN + 16;
        }
        cp_async16(d, src);
      }
    }
    cp_async_commit();
  };

  int64_t s = s_begin + warp;
#pragma unroll 1
  for (int i = 0; i < RS - 1; ++i) issue(s + 4 * i, i);
  grid_dependency_wait();
  const uint8_t* prep = a.prep + (int64_t)chunk * a.prep_bytes;
  SC::stage(afrag, prep);
  const float4 qs = reinterpret_cast<const float4*>(prep + SC::FR * 128)[g & 3];
  __syncthreads();
  SC sc;
  sc.load(reinterpret_cast<const uint8_t*>(afrag), lane);

  int st = 0;
  for (; s < s_end; s += 4) {
    issue(s + 4 * (RS - 1), (st + RS - 1) % RS);
    cp_async_wait<RS - 1>();
    __syncwarp();
    const uint8_t* src = ring[warp][st];
    uint32_t bw[KB][NH], sw[SW];
#pragma unroll
    for (int p = 0; p < KB; ++p)
#pragma unroll
      for (int h = 0; h < NH; ++h)
        bw[p][h] = reinterpret_cast<const uint32_t*>(src + p * RG::PLANE + g * (DP / 8))[t + 4 * h];
#pragma unroll
    for (int i = 0; i < SW; ++i) {
      const int w = t + 4 * i;
      sw[i] = (SI && 32 * w < a.m) ? reinterpret_cast<const uint32_t*>(src + KB * RG::PLANE + g * sbytes)[w] : 0u;
    }
    int accC[2][SC::NCSL][4] = {}, accS[2][4] = {}, accF[2][4];
    sc.run(accC, accS, bw, sw);
    SC::fold(accC, accF);
    float c0, c1, z0 = 0.f, z1 = 0.f;
    combine_digits(accF, lane, c0, c1);
    if constexpr (SI > 0) combine_digits(accS, lane, z0, z1);
    if (qvalid) {
      const __half* nn = reinterpret_cast<const __half*>(src + KB * RG::PLANE + RG::SIGN);
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int64_t key = 8 * s + 2 * t + e;
        if (key < a.n_keys) {
          float l = fmaf(e ? c1 : c0, qs.x, -qs.y);
          if constexpr (SI > 0) {
            const float gm = __half2float(nn[8 + 2 * t + e]);
            l = fmaf(gm * a.kappa, fmaf(e ? z1 : z0, qs.z, -qs.w), l);
          }
          out[key] = __half2float(nn[2 * t + e]) * l;
        }
      }
    }
    __syncwarp();
    st = (st + 1) % RS;
  }
  cp_async_wait<0>();
}

template <int DP, int KB, int SI>
int launch_logits(const LArgs& a, int chunks, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(chunks * a.nsplit);
  cfg.blockDim = dim3(128);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // the streaming kernel needs 8-key subtiles inside one tile and 16-byte aligned norm rows
  const bool ring_ok = (a.n_keys % 8) == 0 && tq::aligned(a.norms, 16) && (!SI || tq::aligned(a.rnorms, 16)) &&
                       (a.m % 128 == 0 || SI == 0);
  cudaError_t e = ring_ok ? cudaLaunchKernelEx(&cfg, logits_ring_kernel<DP, KB, SI>, a)
                          : cudaLaunchKernelEx(&cfg, logits_kernel<DP, KB, SI>, a);
  if (e != cudaSuccess) return tq::set_error(TQ_ECUDA, "tq_logits: launch failed: %s", cudaGetErrorString(e));
  return TQ_OK;
}

template <int DP, int KB>
int dispatch_si(int si, const LArgs& a, int chunks, cudaStream_t st) {
  switch (si) {
    case 0: return launch_logits<DP, KB, 0>(a, chunks, st);
    case 1: return launch_logits<DP, KB, 1>(a, chunks, st);
    default: return launch_logits<DP, KB, 2>(a, chunks, st);
  }
}

}  // namespace

namespace tq {
// Whether the register-fed scan supports this (d_pad, kb).
bool scan_supported(int dp, int kb) { return (dp == 128 && kb >= 1 && kb <= 3) || (dp == 256 && kb >= 1 && kb <= 2); }

int64_t prep_chunk_bytes_max(int dp, int kb, int m) {
  const tqd::ScanShape sh(dp, kb, m);
  return tqd::prep_chunk_bytes(sh.fr);
}
}  // namespace tq

// d_pad 256 with 3 index bits runs on the tensor-memory search scan in all-scores mode.
static bool logits_on_stc(const tq_params* p, int kb) {
  return p->d_pad == 256 && kb == 3 && tq::search_tc_supported(256, kb, p->mode == TQ_MODE_PROD ? p->m : 0);
}

extern "C" int64_t tq_logits_workspace(const tq_params* p, int n_q) {
  if (!p || n_q < 0) return -1;
  const int kb = p->mode == TQ_MODE_PROD ? p->bits - 1 : p->bits;
  if (kb < 1 || kb > 4 || (p->d_pad != 128 && p->d_pad != 256)) return -1;
  const int m = p->mode == TQ_MODE_PROD ? p->m : 0;
  if (logits_on_stc(p, kb)) return tq::logits_stc_workspace(kb, m, n_q);
  return (int64_t)n_q * tq::prep_chunk_bytes_max(p->d_pad, kb, m);
}

extern "C" int tq_logits_ld(const tq_params* p, const float* q, int n_q, int group, const void* codes,
                            const uint16_t* norms, const uint16_t* rnorms, int64_t n_keys, int n_kv_heads,
                            float* logits, int64_t ld_logits, void* workspace, int64_t workspace_bytes,
                            tq_stream_t stream) {
  using namespace tq;
  int rc = check_params(p, "tq_logits");
  if (!rc) rc = check_planes(p, "tq_logits");
  if (rc) return rc;
  if (ld_logits < n_keys) return set_error(TQ_EINVAL, "tq_logits: ld_logits < n_keys");
  const int kb = index_bits(p);
  const bool prod = p->mode == TQ_MODE_PROD;
  const bool stc = logits_on_stc(p, kb);
  if (!scan_supported(p->d_pad, kb) && !stc)
    return set_error(TQ_EUNSUPPORTED, "tq_logits: d_pad=%d with %d index bits (m=%d) is not supported", p->d_pad,
                     kb, p->m);
  if (group < 1 || n_kv_heads < 1 || (int64_t)n_kv_heads * group != n_q)
    return set_error(TQ_EINVAL, "tq_logits: need n_q == n_kv_heads * group (n_q=%d, heads=%d, group=%d)", n_q,
                     n_kv_heads, group);
  if (n_keys < 0) return set_error(TQ_EINVAL, "tq_logits: n_keys < 0");
  if (n_keys == 0) {
    clear_error();
    return TQ_OK;
  }
  if (!q || !codes || !norms || !logits || !workspace || (prod && !rnorms))
    return set_error(TQ_EINVAL, "tq_logits: NULL pointer argument");
  if (!aligned(codes, 16) || !aligned(workspace, 16) || !aligned(q, 4) || !aligned(logits, 4))
    return set_error(TQ_EINVAL, "tq_logits: misaligned pointer (codes/workspace need 16 bytes)");
  const int m = prod ? p->m : 0;
  cudaStream_t st0 = reinterpret_cast<cudaStream_t>(stream);
  if (stc) {  // tensor-memory scan of the search kernel, every score written
    if (n_kv_heads > 1 && n_keys % 32 != 0)
      return set_error(TQ_EUNSUPPORTED, "tq_logits: d_pad 256 with 3 index bits needs n_keys %% 32 == 0 for "
                                        "more than one KV head");
    const int64_t need = logits_stc_workspace(kb, m, n_q);
    if (workspace_bytes < need)
      return set_error(TQ_EINVAL, "tq_logits: workspace too small (%lld < %lld bytes)", (long long)workspace_bytes,
                       (long long)need);
    rc = launch_logits_stc(p, kb, q, n_kv_heads, group, codes, norms, rnorms, n_keys, logits, ld_logits, workspace,
                           st0);
    if (rc == TQ_OK) clear_error();
    return rc;
  }
  const tqd::ScanShape sh(p->d_pad, kb, m);
  const int nqc = (group + tqd::QCHUNK - 1) / tqd::QCHUNK;
  const int chunks = n_kv_heads * nqc;
  const int64_t need = (int64_t)chunks * tqd::prep_chunk_bytes(sh.fr);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (logits_tc_supported(p->d_pad, kb, m, group, n_keys, norms, rnorms)) {
    // tensor-memory scan with the query preparation inside the kernel: the workspace is not used
    rc = launch_logits_tc(kb, m, q, p->d, p->centroids, p->signs_D, p->S, codes, norms, rnorms, n_keys, n_kv_heads,
                          group, logits, ld_logits, st);
    if (rc == TQ_OK) clear_error();
    return rc;
  }
  if (workspace_bytes < need)  // the other scans keep their query preparation in the workspace
    return set_error(TQ_EINVAL, "tq_logits: workspace too small (%lld < %lld bytes)", (long long)workspace_bytes,
                     (long long)need);
  tqd::PrepArgs pa;
  pa.q = q;
  pa.d = p->d;
  pa.dp = p->d_pad;
  pa.kb = kb;
  pa.m = m;
  pa.n_outer = n_kv_heads;
  pa.group = group;
  pa.nqc = nqc;
  pa.cent = p->centroids;
  pa.D = p->signs_D;
  pa.S = p->S;
  pa.out = static_cast<uint8_t*>(workspace);
  pa.fr = sh.fr;
  rc = launch_prep(pa, st);
  if (rc) return rc;

  LArgs a;
  a.codes = static_cast<const uint8_t*>(codes);
  a.norms = norms;
  a.rnorms = rnorms;
  a.n_keys = n_keys;
  a.group = group;
  a.nqc = nqc;
  a.m = m;
  a.tb = tqd::tile_bytes(p->d_pad, kb, m);
  a.prep = pa.out;
  a.prep_bytes = tqd::prep_chunk_bytes(sh.fr);
  a.logits = logits;
  a.ld = ld_logits;
  a.kappa = (float)(std::sqrt(M_PI / 2.0) / (m > 0 ? m : 1));
  // about four 128-thread CTAs per SM, each with at least 16 subtiles per warp
  const int64_t n_sub = (n_keys + 7) / 8;
  const int64_t target = (int64_t)sm_count() * 4;
  a.nsplit = (int)std::max<int64_t>(1, std::min<int64_t>((target + chunks - 1) / chunks, (n_sub + 63) / 64));
  const int si = sh.nsi;
  if (p->d_pad == 128) {
    switch (kb) {
      case 1: rc = dispatch_si<128, 1>(si, a, chunks, st); break;
      case 2: rc = dispatch_si<128, 2>(si, a, chunks, st); break;
      default: rc = dispatch_si<128, 3>(si, a, chunks, st); break;
    }
  } else {
    switch (kb) {
      case 1: rc = dispatch_si<256, 1>(si, a, chunks, st); break;
      default: rc = dispatch_si<256, 2>(si, a, chunks, st); break;
    }
  }
  if (rc == TQ_OK) clear_error();
  return rc;
}

extern "C" int tq_logits(const tq_params* p, const float* q, int n_q, int group, const void* codes,
                         const uint16_t* norms, const uint16_t* rnorms, int64_t n_keys, int n_kv_heads,
                         float* logits, void* workspace, int64_t workspace_bytes, tq_stream_t stream) {
  return tq_logits_ld(p, q, n_q, group, codes, norms, rnorms, n_keys, n_kv_heads, logits, n_keys, workspace,
                      workspace_bytes, stream);
}

// ---------------------------------------------------------------------------
// Allocation-free variant of tq_logits.
//
// Some callers cannot allocate device memory at call time: code running while
// a CUDA graph is being captured, plugins hosted by a framework that owns every
// device buffer and hands out only inputs and outputs, or runtimes whose device
// heap is a fixed pool.  For them the query-prep scratch that tq_logits takes as
// `workspace` lives in a static device array instead.  Every device that loads
// the library holds this array until the process exits.
// ---------------------------------------------------------------------------
namespace {

constexpr int64_t kNoAllocScratchBytes = int64_t(1) << 20;  // 1 MiB
__device__ __align__(256) uint8_t g_logits_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};
void* g_scratch_ctx[kMaxDevices] = {};  // the driver context the address was looked up in

// The current driver context (cuCtxGetCurrent through the runtime's driver entry point, so
// the library does not link the driver library itself); nullptr when unavailable.
void* current_context() {
  using GetCtx = int (*)(void**);
  static GetCtx fn = [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      f = nullptr;
    return reinterpret_cast<GetCtx>(f);
  }();
  void* ctx = nullptr;
  if (fn && fn(&ctx) != 0) ctx = nullptr;
  return ctx;
}

// Device address of the static scratch on the current device.  It is looked up once per
// device and looked up again when the current driver context is not the one it was found
// in (after cudaDeviceReset, or under a context other than the device's primary one).
int scratch_on_current_device(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return tq::set_error(TQ_ECUDA, "tq_logits_noalloc: cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return tq::set_error(TQ_EUNSUPPORTED, "tq_logits_noalloc: device index %d", dev);
  void* ctx = current_context();
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev] || g_scratch_ctx[dev] != ctx) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_logits_scratch);
    if (e != cudaSuccess || !ptr)
      return tq::set_error(TQ_ECUDA, "tq_logits_noalloc: cudaGetSymbolAddress: %s", cudaGetErrorString(e));
    g_scratch_ptr[dev] = ptr;
    g_scratch_ctx[dev] = ctx;
  }
  *out = g_scratch_ptr[dev];
  return TQ_OK;
}

}  // namespace

extern "C" int64_t tq_logits_noalloc_max_scratch(void) { return kNoAllocScratchBytes; }

extern "C" int tq_logits_noalloc(const tq_params* p, const float* q, int n_q, int group, const void* codes,
                                 const uint16_t* norms, const uint16_t* rnorms, int64_t n_keys, int n_kv_heads,
                                 float* logits, tq_stream_t stream) {
  using namespace tq;
  int rc = check_params(p, "tq_logits_noalloc");
  if (!rc) rc = check_planes(p, "tq_logits_noalloc");
  if (rc) return rc;
  if (group < 1 || n_kv_heads < 1 || (int64_t)n_kv_heads * group != n_q)
    return set_error(TQ_EINVAL, "tq_logits_noalloc: need n_q == n_kv_heads * group");
  const int kb = index_bits(p);
  const int m = p->mode == TQ_MODE_PROD ? p->m : 0;
  // the tensor-core path prepares its queries inside the kernel; the other shapes use the scratch
  const bool tc = logits_tc_supported(p->d_pad, kb, m, group, n_keys, norms, rnorms);
  const int64_t need =
      tc ? 0 : (int64_t)n_kv_heads * ((group + tqd::QCHUNK - 1) / tqd::QCHUNK) * prep_chunk_bytes_max(p->d_pad, kb, m);
  if (need > kNoAllocScratchBytes)
    return set_error(TQ_EINVAL,
                     "tq_logits_noalloc: %d query heads need %lld bytes of scratch, above the static %lld; "
                     "use tq_logits with a caller-owned workspace",
                     n_q, (long long)need, (long long)kNoAllocScratchBytes);
  void* scratch = nullptr;
  rc = scratch_on_current_device(&scratch);
  if (rc) return rc;
  return tq_logits(p, q, n_q, group, codes, norms, rnorms, n_keys, n_kv_heads, logits, scratch,
                   kNoAllocScratchBytes, stream);
}
