// tq_search_topk: top-k inner-product search over quantized vectors
// ("TurboQuant explainer" (m.163.com), "向量搜索").
#include <cuda_runtime.h>

#include "common.h"

extern "C" int64_t tq_search_workspace(const tq_params* p, int n_q, int64_t n_db, int k) {
  (void)p;
  (void)n_q;
  (void)n_db;
  (void)k;
  return 0;
}

extern "C" int tq_search_topk(const tq_params* p, const float* q, int n_q, const void* codes, const uint16_t* norms,
                              const uint16_t* rnorms, int64_t n_db, int k, int32_t* ids, float* scores,
                              void* workspace, int64_t workspace_bytes, tq_stream_t stream) {
  (void)p; (void)q; (void)n_q; (void)codes; (void)norms; (void)rnorms; (void)n_db; (void)k; (void)ids;
  (void)scores; (void)workspace; (void)workspace_bytes; (void)stream;
  return tq::set_error(TQ_EUNSUPPORTED, "tq_search_topk: not built yet");
}
