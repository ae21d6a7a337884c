// Internal interfaces of the STCA kernels.
#pragma once
#include "common.cuh"
#include "gemm.cuh"

namespace sa {

struct StcaArgs {
  const void* q; sa_dtype dtype;
  const int64_t* cand_dev; int B; int64_t C_total;
  const void* kv; int64_t kv_rows;
  const int64_t* kvb_dev; const int64_t* kve_dev;
  int D, heads, d_h, n_layers;
  const stca_layer* layers;   // host array
  float* out;
  int64_t max_rows_per_user;  // max over users of C_u * heads (host-computed)
};

struct StcaWork {
  float* Qh;           // [C, heads*d_h]
  float* U;            // [C*heads, D]   fp32 (CUDA-core attention)
  __nv_bfloat16* Ub;   // [C*heads, D]   bf16 (tensor-core attention)
  float* Y;            // [C*heads, D]
  float* O;            // [C, heads*d_h]
  int* tile_prefix;    // [B+1]
  int max_tiles;       // upper bound on the number of query tiles
};

sa_status stca_run(const StcaArgs& a, const StcaWork& w, cudaStream_t st);

bool stca_tc_supported(sa_dtype dtype, int D);
sa_status stca_tc_attention(const StcaArgs& a, const StcaWork& w, cudaStream_t st);

}  // namespace sa
