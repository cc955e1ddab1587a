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
}  // namespace tq
