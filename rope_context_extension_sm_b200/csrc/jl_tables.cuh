// jl_tables.cuh -- RoPE cos/sin tables, fp64 angles rounded once to fp32.
// theta_c = base^(-2c/d); row p holds cos/sin(p * theta_c), c < d/2 (rotate-half
// pairing).  The bifocal kernels read row x for base rotations R(x), row f(x)
// for remote rotations R(f(x)) and row x - f(x) for decode corrections.
#pragma once

#include "jl_device.cuh"

namespace jl {

__global__ void __launch_bounds__(256) jl_rope_table_kernel(float* __restrict__ cos_out, float* __restrict__ sin_out,
                                                            int64_t n_pos, int half, double rope_base) {
  const int64_t total = n_pos * half;
  for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t pos = idx / half;
    const int c = static_cast<int>(idx % half);
    const double theta = pow(rope_base, -2.0 * static_cast<double>(c) / static_cast<double>(2 * half));
    double s, co;
    sincos(static_cast<double>(pos) * theta, &s, &co);
    cos_out[idx] = static_cast<float>(co);
    sin_out[idx] = static_cast<float>(s);
  }
}

// Scaled tables: cos/sin(p * theta_c * lambda_c), fp64 angle, rounded to fp32 once.
struct FreqScale {
  double lambda[64];
};

__global__ void __launch_bounds__(256) jl_rope_table_scaled_kernel(float* __restrict__ cos_out,
                                                                   float* __restrict__ sin_out, int64_t n_pos,
                                                                   int half, double rope_base, const FreqScale fs) {
  const int64_t total = n_pos * half;
  for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t pos = idx / half;
    const int c = static_cast<int>(idx % half);
    const double theta = pow(rope_base, -2.0 * static_cast<double>(c) / static_cast<double>(2 * half));
    double s, co;
    sincos(static_cast<double>(pos) * theta * fs.lambda[c], &s, &co);
    cos_out[idx] = static_cast<float>(co);
    sin_out[idx] = static_cast<float>(s);
  }
}

// Waits on a barrier nobody arrives at, for at most `limit` cycles, then records
// a timeout exactly as the attention kernels' bounded waits do.
__global__ void jl_selftest_wait_kernel(long long limit) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const long long t0 = clock64();
    while (!mbar_try_wait(&bar, 0)) {
      if (clock64() - t0 > limit) {
        atomicOr(&g_status, kDevErrTimeout);
        break;
      }
    }
  }
}

}  // namespace jl
