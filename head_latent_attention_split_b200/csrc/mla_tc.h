// tcgen05 / TMA decode kernel for r = 512, d_r = 64, block_size = 64 (sm_100a).
#pragma once

#include "mla_internal.h"

namespace mla {

// Whether MLA_KERNEL_AUTO picks the tensor-core kernel for the shapes it supports.
constexpr bool kTcAuto = true;

// True when the tensor-core kernel handles this problem (rows = Sq * H).
bool tc_supported(int r, int d_r, int block_size, int q_dtype, int cache_dtype, int out_dtype, int rows);
// Default worker count for `sms` SMs.
int tc_auto_workers(int sms, int rows);
// True when W workers fit the kernel's persistent grid.
bool tc_workers_ok(int W, int rows);
cudaError_t launch_tc_decode(const DecodeArgs& a, cudaStream_t s);

// Split-role pair kernel (mla_pair.cu): bf16 cache, dense token ranges.
cudaError_t launch_pair_decode(const DecodeArgs& a, cudaStream_t s);

}  // namespace mla
