// Tensor-core STCA attention (tcgen05 / TMEM / TMA).  Not enabled yet.
#include "stca_internal.cuh"

namespace sa {
bool stca_tc_supported(sa_dtype, int) { return false; }
sa_status stca_tc_attention(const StcaArgs&, const StcaWork&, cudaStream_t) {
  return fail(SA_ERR_UNSUPPORTED, "tensor-core STCA attention not built");
}
}  // namespace sa
