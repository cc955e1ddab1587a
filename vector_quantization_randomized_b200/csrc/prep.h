// Internal host-side interface between the entry points and the query-prep
// kernel (not part of the public C ABI).
#pragma once

#include <cuda_runtime.h>

#include "scan.cuh"

namespace tq {
// Launch qprep_kernel for a.n_outer * a.nqc chunks of 4 queries.
int launch_prep(const tqd::PrepArgs& a, cudaStream_t st);
// Number of SMs of the current device.
int sm_count();
// The tensor-memory logits scan (logits_tc.cu): supported shapes, and the launch
// (query preparation inside the kernel, no workspace).
bool logits_tc_supported(int dp, int kb, int m, int group, int64_t n_keys, const void* norms, const void* rnorms);
int launch_logits_tc(int kb, int m, const float* q, int d, const float* cent, const int8_t* D, const uint16_t* S,
                     const void* codes, const uint16_t* norms, const uint16_t* rnorms, int64_t n_keys,
                     int n_kv_heads, int group, float* logits, int64_t ld, cudaStream_t st);
// The tensor-memory search (search_tc.cu): supported shapes, workspace, and the
// prep + scan launch that leaves [n_q][*nsplit][16] candidates for the split merge.
bool search_tc_supported(int dp, int kb, int m);
int64_t search_tc_workspace(int kb, int m, int n_q, int64_t n_db);
int launch_search_tc(const tq_params* p, int kb, const float* q, int n_q, const void* codes, const uint16_t* norms,
                     const uint16_t* rnorms, int64_t n_db, void* workspace, float2** cand, int* nsplit,
                     cudaStream_t st);
// Logits on the tensor-memory search scan (d_pad 256): every score of n_kv_heads x group
// queries against their head's n_keys keys, into rows of stride ld; query images in the workspace.
int64_t logits_stc_workspace(int kb, int m, int n_q);
int launch_logits_stc(const tq_params* p, int kb, const float* q, int n_heads, int group, const void* codes,
                      const uint16_t* norms, const uint16_t* rnorms, int64_t n_keys, float* logits, int64_t ld,
                      void* workspace, cudaStream_t st);
// tq_decode_attn with token-sliced value codes (decode_tc.cu): workspace bytes and the call.
int64_t decode_sliced_workspace(int kb, int m, int batch, int n_q_heads, int n_kv_heads, int64_t max_tokens);
int decode_attn_sliced(const tq_params* kp, const tq_params* vp, const float* q, int batch, int n_q_heads,
                       int n_kv_heads, const void* kcodes, const uint16_t* knorms, const uint16_t* krnorms,
                       const void* vcodes, const uint16_t* vnorms, const int32_t* seq_lens, int64_t max_tokens,
                       float scale, float* out, void* workspace, int64_t workspace_bytes, cudaStream_t st);
// Bytes of query-prep scratch per chunk of 4 queries, the larger of both layouts.
int64_t prep_chunk_bytes_max(int dp, int kb, int m);
}  // namespace tq
