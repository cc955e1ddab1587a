// Query preparation and the per-key code scan shared by tq_logits,
// tq_decode_attn and tq_search_topk.
//
// Estimator ("TurboQuant explainer" (m.163.com), "第二步：QJL"):
//   l = n * ( <q_rot, c[idx]> + gamma*sqrt(pi/2)/m * <u, 2s-1> ),
//   q_rot = H D q / sqrt(d_pad),  u = S q_rot.
//
// Evaluation on the tensor cores.  The stored codebook is odd-symmetric
// (c[L-1-l] = -c[l]) and indices are sorted by value, so as a function of the
// index bits it has only odd-degree Walsh terms:
//   c[idx] = sum_T alpha_T * sigma_T,  sigma_T = 2*parity(bits of idx in T) - 1,
//   alpha_T = (1/L) sum_l c_l * prod_{p in T} (2 bit_p(l) - 1),  |T| odd
// (kb=1: {0}; kb=2: {0},{1}; kb=3: {0},{1},{2},{0,1,2}).  With b_T the parity
// bit-plane,
//   <q_rot, c[idx]> = 2 sum_T alpha_T <q_rot, b_T> - c[L-1] * sum_j q_rot_j
//   <u, 2s-1>       = 2 <u, s> - sum_i u_i.
// Every remaining product is "integer weight x bit", evaluated exactly with
// int8 MMA (mma.sync m16n8k32 / m16n8k16, s8 x u8 -> s32):
//  * weights 2 alpha_T q_rot_j and 2 u_i are scaled by 2^F (per query) to
//    integers below 2^23, shifted left by 7-c for bit class c, and split into
//    four signed base-256 digits; MMA row r = 4*digit + query;
//  * the B operand is the code word itself: (word & (0x01010101 << c)) puts
//    the bits c, c+8, c+16, c+24 of a 32-bit plane word into four bytes of
//    value 2^c - no unpacking.  Bit class c's factor 2^c and the weight's
//    2^(7-c) give every product the same factor 2^7;
//  * sum_r 256^digit(r) C[r] = 2^(F+7) * sum weight*bit, exactly.
// The query-side arithmetic (rotation, projection, scaling, digit split) is
// done once per query by qprep_kernel and stored as ready-made A fragments.
#pragma once

#include "device.cuh"

namespace tqd {

constexpr int QCHUNK = 4;  // queries per MMA row block (4 queries x 4 digits = 16 rows)

// Walsh plane T (0..nt-1) as a mask over index bits.
__host__ __device__ __forceinline__ int walsh_mask(int kb, int T) {
  if (kb == 3 && T == 3) return 7;
  return 1 << T;
}
__host__ __device__ __forceinline__ int walsh_planes(int kb) { return kb == 1 ? 1 : (kb == 2 ? 2 : 4); }

// Fragment words per lane for a scan configuration.  Per bit class c there is
// one 4-word slot per MMA: centroid k32 pairs, then a centroid k16 single,
// then the sign k32 pair or k16 single (k16 slots use words 0 and 1).
struct ScanShape {
  int nt, nci, ncp, ncs, nsi, nsp, nss, per_c, fr;
  __host__ __device__ ScanShape(int dp, int kb, int m) {
    nt = walsh_planes(kb);
    nci = nt * (dp / 128);
    ncp = nci / 2;
    ncs = nci % 2;
    nsi = m == 0 ? 0 : (m > 128 ? 2 : 1);
    nsp = nsi / 2;
    nss = nsi % 2;
    per_c = 4 * (ncp + ncs + nsp + nss);  // one 16-byte slot per MMA (k16 uses half of it)
    fr = 8 * per_c;
  }
};

// Query-prep output per chunk of 4 queries: A fragments (uint4 [fr/4][32])
// followed by per-query scalars (float4 [4]: 2^-(F+7), c[L-1]*sum q_rot,
// 2^-(G+7), sum u).
__host__ __device__ __forceinline__ int64_t prep_chunk_bytes(int fr) { return (int64_t)fr * 32 * 4 + 4 * 16; }

struct PrepArgs {
  const float* q;       // query rows, stride d
  int d, dp, kb, m;
  int n_outer, group, nqc;  // chunk = outer*nqc + qc; query row = outer*group + 4*qc + j
  const float* cent;
  const int8_t* D;
  const uint16_t* S;
  uint8_t* out;         // n_outer*nqc chunks of prep_chunk_bytes(fr)
  int fr;
};

// Compile-time scan over one 8-key subtile.
template <int DP, int KB, int SI>
struct Scan {
  static constexpr int NT = KB == 1 ? 1 : (KB == 2 ? 2 : 4);
  static constexpr int NH = DP / 128;  // plane words per lane
  static constexpr int NCI = NT * NH;
  static constexpr int NCP = NCI / 2, NCS = NCI % 2;
  static constexpr int NSP = SI / 2, NSS = SI % 2;
  static constexpr int NSLOT = NCP + NCS + NSP + NSS;  // MMAs per bit class
  static constexpr int PER_C = 4 * NSLOT;
  static constexpr int FR = 8 * PER_C;

  uint32_t A[FR];

  // A fragments of a chunk: fr/4 x 32 uint4, lane-interleaved (global or shared memory)
  __device__ __forceinline__ void load(const uint8_t* chunk, int lane) {
    const uint4* f = reinterpret_cast<const uint4*>(chunk);
#pragma unroll
    for (int k = 0; k < FR / 4; ++k) {
      uint4 v = f[k * 32 + lane];
      A[4 * k] = v.x;
      A[4 * k + 1] = v.y;
      A[4 * k + 2] = v.z;
      A[4 * k + 3] = v.w;
    }
  }

  // Stage a chunk's fragments in shared memory (whole CTA), then every warp loads from there.
  __device__ __forceinline__ static void stage(uint4* smem, const uint8_t* chunk) {
    const uint4* f = reinterpret_cast<const uint4*>(chunk);
    for (int k = threadIdx.x; k < FR / 4 * 32; k += blockDim.x) smem[k] = __ldg(f + k);
  }

  // bw[p][h]: word (t + 4h) of bit-plane p of this lane's key; sw[i]: sign word (t + 4i).
  // Every MMA slot accumulates into its own register set, separately for even and
  // odd bit classes, so a subtile carries 2*NSLOT independent MMA chains.
  static constexpr int NCSL = NCP + NCS;  // centroid slots
  __device__ __forceinline__ void run(int (&accC)[2][NCSL][4], int (&accS)[2][4], const uint32_t (&bw)[KB][NH],
                                      const uint32_t (&sw)[SI > 0 ? SI : 1]) const {
    uint32_t it[NCI];
#pragma unroll
    for (int T = 0; T < NT; ++T) {
#pragma unroll
      for (int h = 0; h < NH; ++h) {
        if (KB == 3 && T == 3) it[T * NH + h] = bw[0][h] ^ bw[1][h] ^ bw[2][h];
        else it[T * NH + h] = bw[T][h];
      }
    }
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const uint32_t mk = 0x01010101u << c;
      const int base = c * PER_C;
#pragma unroll
      for (int p = 0; p < NCP; ++p)
        mma_s8u8_16832(accC[c & 1][p], A[base + 4 * p], A[base + 4 * p + 1], A[base + 4 * p + 2],
                       A[base + 4 * p + 3], it[2 * p] & mk, it[2 * p + 1] & mk);
      if constexpr (NCS) mma_s8u8_16816(accC[c & 1][NCP], A[base + 4 * NCP], A[base + 4 * NCP + 1], it[NCI - 1] & mk);
      constexpr int o = 4 * (NCP + NCS);
      if constexpr (NSP) mma_s8u8_16832(accS[c & 1], A[base + o], A[base + o + 1], A[base + o + 2], A[base + o + 3],
                                        sw[0] & mk, sw[SI > 1 ? 1 : 0] & mk);
      if constexpr (NSS) mma_s8u8_16816(accS[c & 1], A[base + o], A[base + o + 1], sw[0] & mk);
    }
  }

  // Fold the centroid chains into one [2][4] set (exact integer sums).
  __device__ __forceinline__ static void fold(const int (&accC)[2][NCSL][4], int (&out)[2][4]) {
#pragma unroll
    for (int par = 0; par < 2; ++par)
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        int v = 0;
#pragma unroll
        for (int p = 0; p < NCSL; ++p) v += accC[par][p][r];
        out[par][r] = v;
      }
  }
};

// Programmatic dependent launch: wait until the preceding grid (query prep)
// has completed and its writes are visible.
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
// Let the next grid in the stream (launched with programmatic stream serialization) be
// scheduled now: its CTAs take each SM as this grid's CTAs leave it, and wait in their own
// grid_dependency_wait for this grid to complete before they read its outputs.
__device__ __forceinline__ void grid_dependents_launch() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }

// Combine the digit rows of an accumulator pair: thread (g, t) holds rows g,
// g+8 (digits g>>2 and 2+(g>>2) of query g&3) for keys 2t, 2t+1.  Returns, in
// lanes 0..15, sum_r 256^digit C[r] for query g, keys 2t, 2t+1.  Each row sum
// is an exact int32 below 2^24 in magnitude (so exact in fp32); the weighted
// sum is rounded to fp32 (relative 2^-24, far inside the logit tolerance).
__device__ __forceinline__ void combine_digits(const int (&acc)[2][4], int lane, float& k0, float& k1) {
  const int g = lane >> 2;
  const float lo = (g >> 2) ? 256.f : 1.f;
  const float hi = (g >> 2) ? 16777216.f : 65536.f;
  k0 = fmaf((float)(acc[0][2] + acc[1][2]), hi, (float)(acc[0][0] + acc[1][0]) * lo);
  k1 = fmaf((float)(acc[0][3] + acc[1][3]), hi, (float)(acc[0][1] + acc[1][1]) * lo);
  k0 += __shfl_xor_sync(FULL, k0, 16);
  k1 += __shfl_xor_sync(FULL, k1, 16);
}

// Load this lane's code words for key vector v (or zeros when !valid).
template <int DP, int KB, int SI>
__device__ __forceinline__ void load_words(const uint8_t* codes, int tb, int m, int64_t v, bool valid, int t,
                                           uint32_t (&bw)[KB][DP / 128], uint32_t (&sw)[SI > 0 ? SI : 1]) {
  if (valid) {
    const uint8_t* base = codes + (v >> 5) * tb;
    const int slot = (int)(v & 31);
#pragma unroll
    for (int p = 0; p < KB; ++p)
#pragma unroll
      for (int h = 0; h < DP / 128; ++h)
        bw[p][h] = __ldg(reinterpret_cast<const uint32_t*>(base + p * TILE * (DP / 8) + slot * (DP / 8)) + t + 4 * h);
#pragma unroll
    for (int i = 0; i < SI; ++i) {
      const int w = t + 4 * i;
      sw[i] = (32 * w < m)
                  ? __ldg(reinterpret_cast<const uint32_t*>(base + KB * TILE * (DP / 8) + slot * (m / 8)) + w)
                  : 0u;
    }
  } else {
#pragma unroll
    for (int p = 0; p < KB; ++p)
#pragma unroll
      for (int h = 0; h < DP / 128; ++h) bw[p][h] = 0u;
#pragma unroll
    for (int i = 0; i < (SI > 0 ? SI : 1); ++i) sw[i] = 0u;
  }
}

}  // namespace tqd
