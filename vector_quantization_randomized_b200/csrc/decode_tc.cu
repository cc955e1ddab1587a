// tq_decode_attn with token-sliced value codes on the fifth-generation tensor
// cores ("TurboQuant explainer" (m.163.com), "速度": attention from the codes;
// zhidx turboquant_plus article: asymmetric K/V).
#include <cuda_runtime.h>

#include <algorithm>

#include "common.h"
#include "prep.h"

namespace tq {

int64_t decode_sliced_workspace(int kb, int m, int batch, int n_q_heads, int n_kv_heads, int64_t max_tokens) {
  (void)kb;
  (void)m;
  (void)batch;
  (void)n_q_heads;
  (void)n_kv_heads;
  (void)max_tokens;
  return 0;
}

int decode_attn_sliced(const tq_params* kp, const tq_params* vp, const float* q, int batch, int n_q_heads,
                       int n_kv_heads, const void* kcodes, const uint16_t* knorms, const uint16_t* krnorms,
                       const void* vcodes, const uint16_t* vnorms, const int32_t* seq_lens, int64_t max_tokens,
                       float scale, float* out, void* workspace, int64_t workspace_bytes, cudaStream_t st) {
  return set_error(TQ_EUNSUPPORTED, "tq_decode_attn: token-sliced values are not served yet");
}

}  // namespace tq
