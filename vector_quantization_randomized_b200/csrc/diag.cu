// Device status: the fault words that bounded device-side waits set when they
// give up, and a diagnostic kernel whose wait runs out on purpose (a barrier
// that nothing arrives at), so the reporting path can be checked without any
// real failure.
#include <cuda_runtime.h>

#include "common.h"
#include "tc.cuh"

namespace {

__global__ void bounded_wait_probe_kernel(uint32_t polls) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) tqd::mbar_init(&bar, 1);
  __syncthreads();
  if (threadIdx.x == 0) tqd::mbar_wait(&bar, 0, polls);  // never completes: gives up after `polls`
  __syncthreads();
}

}  // namespace

namespace tq {
int fault_word_quantize(int clear, int* value);
int fault_word_quantize_rt(int clear, int* value);
int fault_word_logits(int clear, int* value);
int fault_word_search(int clear, int* value);

int fault_word_diag(int clear, int* value) {
  cudaError_t e = cudaMemcpyFromSymbol(value, tqd::g_fault, sizeof(int));
  if (e == cudaSuccess && clear) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(tqd::g_fault, &zero, sizeof(int));
  }
  return e == cudaSuccess ? TQ_OK : set_error(TQ_ECUDA, "tq_device_status: %s", cudaGetErrorString(e));
}
}  // namespace tq

extern "C" int tq_device_status(int clear) {
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return tq::set_error(TQ_ECUDA, "tq_device_status: %s", cudaGetErrorString(e));
  struct {
    const char* name;
    int (*read)(int, int*);
  } fam[] = {{"quantize", tq::fault_word_quantize},
             {"quantize (tensor-core rotation)", tq::fault_word_quantize_rt},
             {"logits", tq::fault_word_logits},
             {"search", tq::fault_word_search},
             {"diagnostic", tq::fault_word_diag}};
  std::string which;
  for (auto& f : fam) {
    int v = 0;
    const int rc = f.read(clear, &v);
    if (rc) return rc;
    if (v) which += (which.empty() ? "" : ", ") + std::string(f.name);
  }
  if (!which.empty()) return tq::set_error(TQ_ETIMEOUT, "tq_device_status: bounded device wait gave up in: %s", which.c_str());
  tq::clear_error();
  return TQ_OK;
}

extern "C" int tq_diag_bounded_wait(int64_t polls, tq_stream_t stream) {
  if (polls < 1 || polls > (int64_t(1) << 20)) return tq::set_error(TQ_EINVAL, "tq_diag_bounded_wait: polls out of range");
  bounded_wait_probe_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>((uint32_t)polls);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return tq::set_error(TQ_ECUDA, "tq_diag_bounded_wait: %s", cudaGetErrorString(e));
  tq::clear_error();
  return TQ_OK;
}
