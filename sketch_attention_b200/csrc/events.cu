// Event embeddings for Sketch Attention's input rows: x_i = item_table[id_i] +
// action_table[a_i] (the workloads' events, an item embedding plus the
// embedding of the feedback type; SequenceO1 Sec. 3.5, the sum that eq. (20)'s
// fusion adds a SwiGLU term to), gathered on the device so that a step ships
// 5 bytes of ids per event instead of its 256-byte row.
//
// bf16 tables; the sum is formed in fp32 and rounded to nearest even bf16.
// Each thread writes 16 bytes (8 columns) of one row; a row is read from the
// tables once (popular items stay in L2).  An id outside its table zeroes the
// row and sets the device error word instead of reading out of bounds.
#include <algorithm>

#include "sa_internal.cuh"

namespace sa {

namespace {
__device__ __forceinline__ uint32_t add_bf16x2(uint32_t a, uint32_t b) {
  // bf16 -> fp32 is exact (the bf16 bits are the high half of the fp32)
  const float lo = __uint_as_float(a << 16) + __uint_as_float(b << 16);
  const float hi = __uint_as_float(a & 0xFFFF0000u) + __uint_as_float(b & 0xFFFF0000u);
  const __nv_bfloat162 r = __floats2bfloat162_rn(lo, hi);
  return *(const uint32_t*)&r;
}

__global__ void __launch_bounds__(256) gather_events_kernel(const uint4* __restrict__ item, int64_t vocab,
                                                            const uint4* __restrict__ action, int n_actions,
                                                            const int32_t* __restrict__ ids,
                                                            const uint8_t* __restrict__ acts, int64_t n,
                                                            int pieces, uint4* __restrict__ X, int* err) {
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n * pieces;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = e / pieces;
    const int c = (int)(e % pieces);
    const int64_t id = ids[r];
    const int a = acts[r];
    uint4 out = make_uint4(0, 0, 0, 0);
    if (id >= 0 && id < vocab && a < n_actions) {
      const uint4 x = item[id * pieces + c], y = action[(int64_t)a * pieces + c];
      out = make_uint4(add_bf16x2(x.x, y.x), add_bf16x2(x.y, y.y), add_bf16x2(x.z, y.z), add_bf16x2(x.w, y.w));
    } else if (c == 0) {
      atomicOr(err, DEV_ERR_INDEX);
    }
    X[e] = out;
  }
}
}  // namespace

sa_status gather_events_run(const void* item, int64_t vocab, const void* action, int n_actions,
                            const int32_t* ids, const uint8_t* acts, int64_t n, int d, void* X,
                            cudaStream_t st) {
  if (n == 0) return SA_OK;
  const int pieces = d / 8;
  const int64_t total = n * pieces;
  const unsigned grid = (unsigned)std::max<int64_t>(1, std::min<int64_t>((total + 255) / 256, 148 * 16));
  SA_TIMED("gather_events_kernel", st,
           (gather_events_kernel<<<grid, 256, 0, st>>>((const uint4*)item, vocab, (const uint4*)action, n_actions,
                                                        ids, acts, n, pieces, (uint4*)X, device_status_word())));
  return SA_OK;
}

}  // namespace sa
