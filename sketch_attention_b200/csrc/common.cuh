// Shared helpers of the CUDA sources: status plumbing, bf16 loads, the
// chunk decomposition of a ragged token stream, and the host-side launch
// helpers.  Nothing here is method arithmetic.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>
#include <string>

#include "../../include/sketch_attn.h"

namespace sa {

// ---------------------------------------------------------------- errors
void set_error(const std::string& msg);
sa_status fail(sa_status st, const std::string& msg);
sa_status cuda_fail(cudaError_t e, const char* what);

#define SA_CUDA(call)                                                  \
  do {                                                                 \
    cudaError_t _e = (call);                                           \
    if (_e != cudaSuccess) return ::sa::cuda_fail(_e, #call);          \
  } while (0)

#define SA_LAUNCH_CHECK(what)                                          \
  do {                                                                 \
    ::sa::note_launch();                                               \
    cudaError_t _e = cudaGetLastError();                               \
    if (_e != cudaSuccess) return ::sa::cuda_fail(_e, what);           \
  } while (0)

// Measurement support: a count of kernel launches, and (when enabled) a CUDA
// event pair recorded on the launch stream around each timed launch.
void note_launch();
void prof_begin(const char* name, cudaStream_t st);
void prof_end(const char* name, cudaStream_t st);

// Launch `stmt` (a kernel launch on stream `st`) between profiling events.
#define SA_TIMED(name, st, stmt)                                       \
  do {                                                                 \
    ::sa::prof_begin(name, st);                                        \
    stmt;                                                              \
    SA_LAUNCH_CHECK(name);                                             \
    ::sa::prof_end(name, st);                                          \
  } while (0)

// Device error word (defined in api.cu): kernels whose bounded waits expire
// OR in a code; sa_poll_device_status reads and clears it.
// bits of the device status word: a bounded wait expired; an embedding id was out of
// range; a value stored as fp16 exceeded the fp16 range (|x| > 65504)
enum : int { DEV_ERR_TIMEOUT = 1, DEV_ERR_INDEX = 2, DEV_ERR_RANGE = 4 };
int* device_status_word();

// ---------------------------------------------------------------- device info
struct DeviceInfo {
  int device = 0;
  int sm_count = 0;
  int max_smem_optin = 0;
  int cc_major = 0, cc_minor = 0;
};
const DeviceInfo& device_info();   // current device, cached per device

// ---------------------------------------------------------------- loads
__device__ __forceinline__ float load_as_f32(const float* p, int64_t i) { return p[i]; }
__device__ __forceinline__ float load_as_f32(const __nv_bfloat16* p, int64_t i) {
  return __bfloat162float(p[i]);
}
__device__ __forceinline__ void store_from_f32(float* p, int64_t i, float v) { p[i] = v; }
__device__ __forceinline__ void store_from_f32(__nv_bfloat16* p, int64_t i, float v) {
  p[i] = __float2bfloat16_rn(v);
}

// ---------------------------------------------------------------- decomposition
// The concatenated token stream [0, n_total) is cut into G chunks of T
// tokens (the last may be shorter).  A chunk is worked on by one CTA (or one
// cluster); it visits the users that overlap it as "pieces".  A piece's
// partial result goes to:
//   slot (g, 0)  if its user started before the chunk,
//   slot (g, 1)  else if its user continues past the chunk,
//   the user's own output row block otherwise (the user lies in one chunk).
// The reduction then adds, per user and in a fixed order, slot (g_first, 1),
// the slots (g, 0) of the chunks in between, and slot (g_last, 0).
struct Chunking {
  int64_t n_total;
  int64_t T;       // tokens per chunk (>= 1)
  int G;           // number of chunks
};

inline Chunking make_chunking(int64_t n_total, int target_chunks, int64_t align = 1) {
  Chunking c;
  c.n_total = n_total;
  if (n_total <= 0) { c.T = 1; c.G = 0; return c; }
  if (target_chunks < 1) target_chunks = 1;
  int64_t T = (n_total + target_chunks - 1) / target_chunks;
  T = ((T + align - 1) / align) * align;
  if (T < 1) T = 1;
  c.T = T;
  c.G = (int)((n_total + T - 1) / T);
  return c;
}

enum PieceDest : int { DEST_SLOT0 = 0, DEST_SLOT1 = 1, DEST_USER = 2 };

// Largest u in [0, B) with off[u] <= t (t < off[B]); that user is non-empty.
__device__ __forceinline__ int user_of_token(const int64_t* __restrict__ off, int B, int64_t t) {
  int lo = 0, hi = B - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (off[mid] <= t) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ int piece_dest(int64_t u_begin, int64_t u_end, int64_t c_begin,
                                          int64_t c_end) {
  if (u_begin < c_begin) return DEST_SLOT0;
  if (u_end > c_end) return DEST_SLOT1;
  return DEST_USER;
}

// ---------------------------------------------------------------- misc
inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Bump allocator over the caller's workspace (host-side arithmetic only).
struct Carve {
  char* base;
  size_t off = 0;
  explicit Carve(void* p) : base((char*)p) {}
  template <class T>
  T* take(size_t count) {
    off = align_up(off, 256);
    T* p = base ? (T*)(base + off) : nullptr;
    off += count * sizeof(T);
    return p;
  }
  size_t bytes() const { return align_up(off, 256); }
};

inline bool aligned16(const void* p) { return ((uintptr_t)p & 15) == 0; }

}  // namespace sa
