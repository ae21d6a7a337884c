// Tensor-core SA forward (tcgen05 / TMEM / TMA).  Not enabled yet.
#include "sa_internal.cuh"

namespace sa {
bool sa_tc_supported(sa_dtype, int, int) { return false; }
int sa_tc_num_chunks(int) { return 1; }
sa_status sa_tc_forward(const SaFwdArgs&, const SaFwdWork&, cudaStream_t) {
  return fail(SA_ERR_UNSUPPORTED, "tensor-core SA forward not built");
}
}  // namespace sa
