// Small fp32 GEMM for the projections around the hot loops (prototype
// folding, value projection, STCA head projections, weight gradients).
// These are O(k d^2) or O(C D^2) per call, far below the token loops.
#pragma once
#include "common.cuh"

namespace sa {

struct Gemm {
  // C[m, n] = alpha * sum_k A[m, k] B[k, n] (+ bias[n]) (+ Cin[m, n])
  int M = 0, N = 0, K = 0;
  const float* A = nullptr; int64_t lda = 0; bool transA = false;   // A[m*lda+k] or A[k*lda+m]
  const float* B = nullptr; int64_t ldb = 0; bool transB = false;   // B[k*ldb+n] or B[n*ldb+k]
  float* C = nullptr; int64_t ldc = 0;                               // fp32 out (may be NULL)
  __nv_bfloat16* C16 = nullptr; int64_t ldc16 = 0;                   // optional bf16 copy
  bool c16_half = false;    // C16 holds fp16 values instead of bf16; |v| > 65504 sets the range bit in *err
  int* err = nullptr;
  const float* Cin = nullptr; int64_t ldcin = 0;                     // optional addend
  const float* bias = nullptr;                                        // optional [N]
  float alpha = 1.f;
  int batch = 1;
  int64_t sA = 0, sB = 0, sC = 0, sC16 = 0, sCin = 0;                // batch strides
  // split-K: split_k CTAs share one output tile, each summing a slice of K
  // into split_ws ([batch * split_k, M, N] fp32); a second kernel adds the
  // slices in a fixed order and applies alpha, bias and Cin.
  int split_k = 1;
  float* split_ws = nullptr;
  // profiler label of the call site (a string literal); NULL = "gemm_kernel"
  const char* tag = nullptr;
};

// Split count for a GEMM with a long K and few output tiles (1 = no split).
int gemm_split_for(int M, int N, int K, int max_split);

sa_status gemm(const Gemm& g, cudaStream_t stream);

}  // namespace sa
