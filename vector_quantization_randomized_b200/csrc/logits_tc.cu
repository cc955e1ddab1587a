// tq_logits on the fifth-generation tensor cores, for d_pad 128 and up to four
// query heads per KV head ("TurboQuant explainer" (m.163.com), "第二步：QJL"
// estimator; "速度": logits straight from the compressed keys).
//
// The integer form of the estimator is the one in scan.cuh: every product is
// "integer weight x code bit", the weights split into signed base-256 digits.
// Here the code bits are the A operand of tcgen05.mma kind::i8 (u8 x s8 ->
// s32), held in tensor memory, and the prepared query digits are the B operand
// in shared memory:
//
//   A[key][chunk 8P + c][4w + b] = byte b of (plane word w of plane P) & (1 << c)
//                                = 2^c * bit(coordinate 32w + 8b + c),
//
// i.e. bit class c of a plane is the plane's four words masked with
// 0x01010101 << c, one 32-bit tensor-memory column per masked word; the B
// image (prep.cu) holds at the same K position the digit of the weight of
// that coordinate, pre-shifted by 7 - c.  One MMA of M = 128 keys, N = 32
// (4 queries x 4 digits x {centroid, sign}), K = 32 bytes.
//
// Warp-specialised pipeline, one persistent CTA per SM over (KV head, 128-key
// tile) items, all hand-offs on mbarriers (waits bounded):
//   warp 0      bulk copies of the code tiles and norms into a ring of shared-memory stages;
//   warps 1-4   tcgen05.mma issue: two pairs take alternate items, each warp of a
//               pair every other K step into its own partial accumulator of a ring
//               of accumulator sets (one thread issues an MMA only every ~50
//               cycles and waits for them to be taken before its next item); the
//               pair that meets a new KV head first loads its B image (bulk copy);
//   8 warps     expansion: stage -> masked words -> tcgen05.st into one of two or
//               three A buffers in tensor memory (warp = lane quadrant x 4 bit classes);
//   8 warps     epilogue: tcgen05.ld of the partial accumulators, digit
//               combination, norms, logits (warp = lane quadrant x 2 queries).
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>

#include "common.h"
#include "prep.h"
#include "scan.cuh"
#include "tc.cuh"

namespace {
using namespace tqd;

constexpr int TK = 128;  // keys per item (MMA M)
constexpr int MAX_STAGES = 16;
constexpr int HDR = 1024;  // barriers + tensor-memory base, ahead of the B image

struct TArgs {
  const uint8_t* codes;
  const uint16_t* norms;
  const uint16_t* rnorms;
  int64_t n_keys;        // keys per KV head, a multiple of 32
  int group;             // query heads per KV head, 1..4
  int tb;                // bytes of one 32-key code tile
  int tiles_per_head;    // ceil(n_keys / 128)
  int64_t n_items;       // n_kv_heads * tiles_per_head
  const uint8_t* prep;   // per KV head: B image + per-query scalars
  int64_t prep_bytes;
  float* logits;
  int64_t ld;            // logits row stride
  float kappa;           // sqrt(pi/2) / m
  int stages;            // ring stages (<= MAX_STAGES)
};

template <int KB, int SI>
struct TL {
  static constexpr int NT = KB == 1 ? 1 : (KB == 2 ? 2 : 4);  // Walsh planes
  static constexpr int NP = NT + SI;                          // planes in A
  static constexpr int KC = 8 * NP;                           // 16-byte K chunks
  static constexpr int ACOLS = 4 * KC;                        // tensor-memory columns of one A buffer
  static constexpr int KSTEPS = ACOLS / 8;                    // MMAs per item (K = 32 bytes each)
  static constexpr int BBYTES = 512 * KC;                     // B image
  static constexpr int TILEB = 32 * 16 * (KB + SI);           // one 32-key code tile
  static constexpr int NORMB = 256 * (1 + SI);                // fp16 norms (+ residual norms) of 128 keys
  static constexpr int STAGE = 4 * TILEB + NORMB;             // one item: code tiles, then norms
  // Two partial accumulators per item, one per MMA-issuing warp: a thread issues a
  // tcgen05.mma only every ~50 cycles while the tensor pipe finishes one of these
  // in ~17, so two warps issue in parallel (K steps j, j + 2, ...) and the epilogue
  // adds the two partial sums (exact int32).  NB accumulator sets in a ring, so the
  // MMAs of item i wait for the epilogue of item i - NB, not i - 2.
  static constexpr int NACC = 2;
  static constexpr int NISS = 2 * NACC;  // two pairs of issuing warps, alternate items
  static constexpr int COLS = 512;
  // A buffers: three where they fit beside three accumulator sets (b <= 3), else two;
  // the expansion of item i then waits for the MMAs of item i - NA
  static constexpr int NA = 3 * ACOLS + 3 * 32 * NACC <= COLS ? 3 : 2;
  static constexpr int NB = (COLS - NA * ACOLS) / (32 * NACC) < 4 ? (COLS - NA * ACOLS) / (32 * NACC) : 4;
  static_assert(NB >= 2 && 32 * NACC * NB + NA * ACOLS <= COLS, "tensor-memory budget");
  static constexpr int W_EXP0 = 1 + NISS, W_EPI0 = W_EXP0 + 8;  // first expansion / epilogue warp
  static constexpr int NTHREADS = (W_EPI0 + 8) * 32;
  static_assert(KSTEPS >= NACC, "every accumulator is written by each item");
  static constexpr int smem(int stages) { return HDR + BBYTES + stages * STAGE; }
};

template <int KB, int SI>
__global__ void __launch_bounds__(TL<KB, SI>::NTHREADS, 1) logits_tc_kernel(const TArgs a) {
  using L = TL<KB, SI>;
  constexpr int W_EXP0 = L::W_EXP0, W_EPI0 = L::W_EPI0;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);   // [MAX_STAGES] stage loaded
  uint64_t* empty = full + MAX_STAGES;                  // [MAX_STAGES] stage read by the expansion and epilogue warps
  uint64_t* afull = empty + MAX_STAGES;                 // [3] A buffer written (8 arrivals)
  uint64_t* mdone = afull + 3;                          // [3] MMAs of the item done: its A buffer is free
  uint64_t* cfull = mdone + 3;                          // [4] MMAs done: accumulator set full
  uint64_t* accfree = cfull + 4;                        // [4] accumulator set read (8 arrivals)
  uint64_t* bfull = accfree + 4;                        // B image loaded
  uint32_t* tbase = reinterpret_cast<uint32_t*>(bfull + 1);
  uint8_t* Bsm = smem + HDR;
  uint8_t* ring = Bsm + L::BBYTES;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = a.stages;
  const int64_t i0 = (int64_t)blockIdx.x * a.n_items / gridDim.x;
  const int64_t i1 = (int64_t)(blockIdx.x + 1) * a.n_items / gridDim.x;
  const int n = (int)(i1 - i0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < MAX_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 16);
    }
    for (int b = 0; b < 3; ++b) {
      mbar_init(&afull[b], 8);
      mbar_init(&mdone[b], L::NACC);
    }
    for (int c = 0; c < 4; ++c) {
      mbar_init(&cfull[c], L::NACC);
      mbar_init(&accfree[c], 8);
    }
    mbar_init(bfull, 1);
  }
  if (warp == 0) tmem_alloc(tbase, L::COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tbase;
  // tensor-memory columns: accumulator set c = NACC x 32 columns from c * NACC * 32,
  // then the two A buffers
  auto acc_col = [&](int c, int k) { return tmem + (uint32_t)(32 * (c * L::NACC + k)); };
  auto a_col = [&](int b) { return tmem + (uint32_t)(32 * L::NACC * L::NB + b * L::ACOLS); };

  if (warp == 0) {
    // ---------------- producer: code tiles into the ring ----------------
    if (lane == 0) {
      int issued = 0;
      int64_t head = i0 / a.tiles_per_head;  // (head, t) advance by one item per iteration: no division in the loop
      int t = (int)(i0 % a.tiles_per_head);
      for (int i = 0, s = 0, use = 0; i < n; ++i) {
        if (i >= S && !mbar_wait(&empty[s], (use - 1) & 1)) break;
        const int64_t k0 = (int64_t)t * TK;
        const int nk = (int)((a.n_keys - k0) < TK ? (a.n_keys - k0) : TK);
        const int64_t tile0 = (head * a.n_keys + k0) >> 5;
        const uint32_t bytes = (uint32_t)((nk >> 5) * a.tb);
        uint8_t* dst = ring + s * L::STAGE;
        mbar_expect_tx(&full[s], bytes + (uint32_t)(2 * nk * (1 + SI)));
        bulk_g2s(dst, a.codes + tile0 * a.tb, bytes, &full[s]);
        bulk_g2s(dst + 4 * L::TILEB, a.norms + head * a.n_keys + k0, 2 * nk, &full[s]);
        if constexpr (SI) bulk_g2s(dst + 4 * L::TILEB + 256, a.rnorms + head * a.n_keys + k0, 2 * nk, &full[s]);
        issued = i + 1;
        if (++t == a.tiles_per_head) t = 0, ++head;
        if (++s == S) s = 0, ++use;
      }
      // nothing may still be in flight into shared memory when the CTA ends
      for (int i = (issued > S ? issued - S : 0); i < issued; ++i) mbar_wait(&full[i % S], (i / S) & 1);
    }
  } else if (warp < W_EXP0) {
    // ---------------- B image + MMA issue ----------------
    // Two pairs of issuing warps take alternate items (pair p: items i with i % 2 == p),
    // each warp of a pair every other K step into its own partial accumulator.  A
    // thread cannot go on to its next item until the tensor core has taken its MMAs,
    // so the other pair keeps the tensor pipe busy meanwhile.
    const int j = warp - 1, par = j >> 1, k = j & 1;
    if (lane == 0) {
      grid_dependency_wait();  // the B image comes from the query-prep kernel
      constexpr uint32_t idesc = idesc_u8s8_s32(TK, 32);
      const uint32_t sB = smem_u32(Bsm);
      int64_t cur = -1, head = i0 / a.tiles_per_head;
      int t = (int)(i0 % a.tiles_per_head);
      uint32_t loads = 0, waited = 0;  // B images requested so far / waited for
      int done = -1;
      bool ok = true;
      for (int i = 0, c = 0, cu = 0; i < n && ok; ++i, ++t, (++c == L::NB ? (c = 0, ++cu) : 0)) {
        const int b = i % L::NA, ua = i / L::NA;  // A buffer and its use count
        if (t == a.tiles_per_head) t = 0, ++head;
        const bool mine = (i & 1) == par;
        if (head != cur) {
          if (mine && k == 0) {  // reload B once no MMA of either pair still reads the old one
            if (i >= 1 && !mbar_wait(&mdone[(i - 1) % L::NA], ((i - 1) / L::NA) & 1)) break;
            if (i >= 2 && !mbar_wait(&mdone[(i - 2) % L::NA], ((i - 2) / L::NA) & 1)) break;
            mbar_expect_tx(bfull, L::BBYTES);
            bulk_g2s(Bsm, a.prep + head * a.prep_bytes, L::BBYTES, bfull);
          }
          ++loads;
          cur = head;
        }
        if (!mine) continue;
        if (waited != loads) {  // the latest B image (load number loads - 1) has landed
          if (!mbar_wait(bfull, (loads - 1) & 1)) break;
          waited = loads;
        }
        if (!mbar_wait(&afull[b], ua & 1)) break;
        if (cu >= 1 && !mbar_wait(&accfree[c], (cu - 1) & 1)) break;
        tc_fence_after();
        for (int ks = k; ks < L::KSTEPS; ks += 2)
          umma_i8_ts(acc_col(c, k), a_col(b) + 8 * ks, smem_desc(sB + ks * 256, 128, L::KC * 128), idesc,
                     ks >= 2 ? 1u : 0u);
        umma_commit(&mdone[b]);
        umma_commit(&cfull[c]);
        done = i;
      }
      if (done >= 0) mbar_wait(&mdone[done % L::NA], (done / L::NA) & 1);  // no MMA left in flight
    }
  } else if (warp < W_EPI0) {
    // ---------------- expansion: code bits -> A in tensor memory ----------------
    const int ew = warp - W_EXP0;
    const int qd = warp & 3;   // tensor-memory lane quadrant = 32-key code tile within the item
    const int cg = ew >> 2;    // bit classes 4cg .. 4cg+3
    for (int i = 0, s = 0, use = 0; i < n; ++i, (++s == S ? (s = 0, ++use) : 0)) {
      const int b = i % L::NA, ua = i / L::NA;
      if (!mbar_wait(&full[s], use & 1)) break;
      if (ua >= 1 && !mbar_wait(&mdone[b], (ua - 1) & 1)) break;  // MMAs of item i - NA have read A[b]
      const uint8_t* st = ring + s * L::STAGE + qd * L::TILEB + lane * 16;
      uint4 pw[KB + SI];
#pragma unroll
      for (int p = 0; p < KB + SI; ++p) pw[p] = *reinterpret_cast<const uint4*>(st + p * 512);
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
      uint4 it[L::NP];
#pragma unroll
      for (int T = 0; T < L::NT; ++T) it[T] = pw[T];
      if constexpr (KB == 3)
        it[3] = make_uint4(pw[0].x ^ pw[1].x ^ pw[2].x, pw[0].y ^ pw[1].y ^ pw[2].y, pw[0].z ^ pw[1].z ^ pw[2].z,
                           pw[0].w ^ pw[1].w ^ pw[2].w);
      if constexpr (SI) it[L::NT] = pw[KB];
      const uint32_t lanebase = a_col(b) + ((uint32_t)(32 * qd) << 16) + 16 * cg;
#pragma unroll
      for (int P = 0; P < L::NP; ++P) {
        uint32_t r[16];
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          const uint32_t mk = 0x01010101u << (4 * cg + cc);
          r[4 * cc + 0] = it[P].x & mk;
          r[4 * cc + 1] = it[P].y & mk;
          r[4 * cc + 2] = it[P].z & mk;
          r[4 * cc + 3] = it[P].w & mk;
        }
        tmem_st16(lanebase + 32 * P, r);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&afull[b]);
    }
  } else {
    // ---------------- epilogue: accumulators -> logits ----------------
    grid_dependency_wait();  // per-query scalars come from the query-prep kernel
    const int ew = warp - W_EPI0;
    const int qd = warp & 3, qp = ew >> 2;  // keys 32qd + lane; queries 2qp, 2qp+1
    int64_t cur = -1, head = i0 / a.tiles_per_head;
    int t = (int)(i0 % a.tiles_per_head);
    float4 sc[2] = {};
    for (int i = 0, s = 0, use = 0, c = 0, cu = 0; i < n;
         ++i, ++t, (++s == S ? (s = 0, ++use) : 0), (++c == L::NB ? (c = 0, ++cu) : 0)) {
      if (t == a.tiles_per_head) t = 0, ++head;
      if (head != cur) {
        const float4* qs = reinterpret_cast<const float4*>(a.prep + head * a.prep_bytes + L::BBYTES);
        sc[0] = qs[2 * qp];
        sc[1] = qs[2 * qp + 1];
        cur = head;
      }
      const int64_t key = (int64_t)t * TK + 32 * qd + lane;
      const bool kvalid = key < a.n_keys;
      if (!mbar_wait(&full[s], use & 1)) break;  // long complete: makes the stage's norms visible here
      const __half* nst = reinterpret_cast<const __half*>(ring + s * L::STAGE + 4 * L::TILEB);
      const float nrm = __half2float(nst[32 * qd + lane]);
      const float gam = SI ? __half2float(nst[128 + 32 * qd + lane]) : 0.f;
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
      if (!mbar_wait(&cfull[c], cu & 1)) break;
      tc_fence_after();
      uint32_t r[16], rp[16];
      const uint32_t lrow = ((uint32_t)(32 * qd) << 16) + 16 * qp;
      tmem_ld16_issue(acc_col(c, 0) + lrow, r);
      tmem_ld16_issue(acc_col(c, 1) + lrow, rp);
      tmem_ld_wait16(r);
      tmem_ld_wait16(rp);
#pragma unroll
      for (int e = 0; e < 16; ++e) r[e] += rp[e];  // exact: the full sums stay below 2^24
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&accfree[c]);
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int q = 2 * qp + j;
        if (q < a.group && kvalid) {
          // sum_d 256^d C[d]: each C[d] an exact int32 below 2^24; one fp32 rounding per step
          const float cen = fmaf((float)(int)r[8 * j + 3], 16777216.f,
                                 fmaf((float)(int)r[8 * j + 2], 65536.f,
                                      fmaf((float)(int)r[8 * j + 1], 256.f, (float)(int)r[8 * j])));
          float l = fmaf(cen, sc[j].x, -sc[j].y);
          if constexpr (SI) {
            const float sg = fmaf((float)(int)r[8 * j + 7], 16777216.f,
                                  fmaf((float)(int)r[8 * j + 6], 65536.f,
                                       fmaf((float)(int)r[8 * j + 5], 256.f, (float)(int)r[8 * j + 4])));
            l = fmaf(gam * a.kappa, fmaf(sg, sc[j].z, -sc[j].w), l);
          }
          a.logits[(head * a.group + q) * a.ld + key] = nrm * l;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, L::COLS);
}

template <int KB, int SI>
int launch_tc(const TArgs& a0, int sm, cudaStream_t st) {
  using L = TL<KB, SI>;
  TArgs a = a0;
  a.stages = MAX_STAGES;
  while (a.stages > 4 && L::smem(a.stages) > 227 * 1024) --a.stages;
  // at least 120 KB: one CTA per SM, so no second CTA waits for the SM's tensor memory
  const int bytes = std::max(L::smem(a.stages), 120 * 1024);
  auto kern = logits_tc_kernel<KB, SI>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return tq::set_error(TQ_ECUDA, "tq_logits: %s", cudaGetErrorString(e));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)std::max<int64_t>(1, std::min<int64_t>(sm, a.n_items)));
  cfg.blockDim = dim3(L::NTHREADS);
  cfg.dynamicSmemBytes = bytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, a);
  if (e != cudaSuccess) return tq::set_error(TQ_ECUDA, "tq_logits: launch failed: %s", cudaGetErrorString(e));
  return TQ_OK;
}

}  // namespace

namespace tq {

bool logits_tc_supported(int dp, int kb, int m, int group, int64_t n_keys, const void* norms, const void* rnorms) {
  return dp == 128 && kb >= 1 && kb <= 3 && (m == 0 || m == 128) && group >= 1 && group <= 4 && n_keys % 32 == 0 &&
         aligned(norms, 16) && (m == 0 || aligned(rnorms, 16));
}

// Scan with the query-prep output `prep` (layout 1, one chunk per KV head).
int launch_logits_tc(int kb, int m, const void* codes, const uint16_t* norms, const uint16_t* rnorms,
                     int64_t n_keys, int n_kv_heads, int group, const uint8_t* prep, int64_t prep_bytes,
                     float* logits, int64_t ld, cudaStream_t st) {
  TArgs a;
  a.codes = static_cast<const uint8_t*>(codes);
  a.norms = norms;
  a.rnorms = rnorms;
  a.n_keys = n_keys;
  a.group = group;
  a.tb = tqd::tile_bytes(128, kb, m);
  a.tiles_per_head = (int)((n_keys + TK - 1) / TK);
  a.n_items = (int64_t)n_kv_heads * a.tiles_per_head;
  a.prep = prep;
  a.prep_bytes = prep_bytes;
  a.logits = logits;
  a.ld = ld;
  a.kappa = (float)(std::sqrt(M_PI / 2.0) / (m > 0 ? m : 1));
  a.stages = MAX_STAGES;
  const int sm = sm_count();
  if (m > 0) {
    switch (kb) {
      case 1: return launch_tc<1, 1>(a, sm, st);
      case 2: return launch_tc<2, 1>(a, sm, st);
      default: return launch_tc<3, 1>(a, sm, st);
    }
  }
  switch (kb) {
    case 1: return launch_tc<1, 0>(a, sm, st);
    case 2: return launch_tc<2, 0>(a, sm, st);
    default: return launch_tc<3, 0>(a, sm, st);
  }
}

}  // namespace tq

namespace tq {
// Read (and optionally clear) this translation unit's device fault word.
int fault_word_logits(int clear, int* value) {
  cudaError_t e = cudaMemcpyFromSymbol(value, tqd::g_fault, sizeof(int));
  if (e == cudaSuccess && clear) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(tqd::g_fault, &zero, sizeof(int));
  }
  return e == cudaSuccess ? TQ_OK : set_error(TQ_ECUDA, "tq_device_status: %s", cudaGetErrorString(e));
}
}  // namespace tq
