// Throughput of exponentials on this GPU, the co-roofline of the SA forward
// (k exponentials per token in each of its two kernels, next to 2kd flop of
// tensor-core work).  Measurement support, not part of the method.
//
// Every thread keeps 16 independent values v <- 2^(v - 1) (bounded in (1/2, 1]),
// so the loop is limited by exponential throughput, not latency.  Mode 0: all
// on the MUFU (ex2.approx); mode 1: the forward kernels' mix, one pair in eight
// by the cubic on the FMA pipe (exp2_poly.cuh).
#include <algorithm>

#include "exp2_poly.cuh"
#include "sa_internal.cuh"
#include "tc_ptx.cuh"

namespace sa {

namespace {
constexpr int kThreads = 512, kIters = 2048, kPairs = 8;

template <int MODE>
__global__ void __launch_bounds__(kThreads) exp2_rate_kernel(float* __restrict__ sink) {
  float2 v[kPairs];
#pragma unroll
  for (int j = 0; j < kPairs; ++j)
    v[j] = make_float2(0.5f + 0.001f * (threadIdx.x % 97) + 0.01f * j, 0.75f - 0.001f * (threadIdx.x % 89));
  const float2 m1 = make_float2(-1.f, -1.f);
  for (int it = 0; it < kIters; ++it) {
#pragma unroll
    for (int j = 0; j < kPairs; ++j) {
      const float2 e = __fadd2_rn(v[j], m1);
      v[j] = (MODE == 1 && (j & 7) == 1) ? exp2_poly2(e) : make_float2(tc::ex2(e.x), tc::ex2(e.y));
    }
  }
  float s = 0.f;
#pragma unroll
  for (int j = 0; j < kPairs; ++j) s += v[j].x + v[j].y;
  sink[(int64_t)blockIdx.x * kThreads + threadIdx.x] = s;
}
// One thread waits on an mbarrier that nothing arrives at, with the bounded wait
// every kernel of the library uses; on expiry the wait sets the abort flag and the
// device error word and returns, and so does the kernel (no trap, no fault).
__global__ void bounded_wait_kernel(long long budget, int* err) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x != 0) return;
  tc::mbar_init(&bar, 1);
  abort_flag = 0;
  tc::fence_mbar_init();
  tc::mbar_wait(&bar, 0, &abort_flag, err, budget);
}
}  // namespace

sa_status selftest_bounded_wait(long long budget_cycles, cudaStream_t st) {
  bounded_wait_kernel<<<1, 32, 0, st>>>(budget_cycles, device_status_word());
  SA_CUDA(cudaGetLastError());
  return SA_OK;
}

sa_status measure_exp2_rate(int mode, double* per_second, cudaStream_t st) {
  const int blocks = device_info().sm_count * 4;
  float* sink = nullptr;
  SA_CUDA(cudaMallocAsync(&sink, sizeof(float) * blocks * kThreads, st));
  cudaEvent_t a, b;
  SA_CUDA(cudaEventCreate(&a));
  SA_CUDA(cudaEventCreate(&b));
  auto launch = [&]() {
    if (mode == 0) exp2_rate_kernel<0><<<blocks, kThreads, 0, st>>>(sink);
    else exp2_rate_kernel<1><<<blocks, kThreads, 0, st>>>(sink);
  };
  launch();                       // warm-up
  SA_CUDA(cudaEventRecord(a, st));
  constexpr int reps = 5;
  for (int r = 0; r < reps; ++r) launch();
  SA_CUDA(cudaGetLastError());
  SA_CUDA(cudaEventRecord(b, st));
  SA_CUDA(cudaEventSynchronize(b));
  float ms = 0.f;
  SA_CUDA(cudaEventElapsedTime(&ms, a, b));
  cudaEventDestroy(a);
  cudaEventDestroy(b);
  SA_CUDA(cudaFreeAsync(sink, st));
  SA_CUDA(cudaStreamSynchronize(st));
  const double exps = (double)reps * blocks * kThreads * kIters * kPairs * 2;
  *per_second = exps / (ms / 1e3);
  return SA_OK;
}

}  // namespace sa
