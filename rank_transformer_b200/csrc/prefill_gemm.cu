// Prefill-regime factorized linear (tcgen05).  Placeholder until the
// tensor-core kernel lands.
#include "kernels.h"

namespace fsvd {
int prefill_linear_launch(const PfLinear&, cudaStream_t) { return FLASHSVD_ERR_UNSUPPORTED_SHAPE; }
int prefill_dense_launch(const PfLinear&, cudaStream_t) { return FLASHSVD_ERR_UNSUPPORTED_SHAPE; }
}  // namespace fsvd
