// The contiguous forward kernels alone (the hot path of fa_fwd), compiled by
// tests/test_kernel_resources.py with ptxas's resource report.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "fa_fwd_tc.cuh"

template __global__ void fa::fa_fwd_tc_kernel<128, __nv_bfloat16>(const __grid_constant__ CUtensorMap,
                                                                  const __grid_constant__ CUtensorMap,
                                                                  const __grid_constant__ CUtensorMap, fa::TcParams,
                                                                  unsigned int*);
template __global__ void fa::fa_fwd_tc_kernel<64, __nv_bfloat16>(const __grid_constant__ CUtensorMap,
                                                                 const __grid_constant__ CUtensorMap,
                                                                 const __grid_constant__ CUtensorMap, fa::TcParams,
                                                                 unsigned int*);
