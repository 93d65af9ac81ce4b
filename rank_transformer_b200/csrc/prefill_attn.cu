// Prefill attention.  Placeholder until the kernel lands.
#include "kernels.h"

namespace fsvd {
int attn_prefill_launch(const AttnPfParams&, cudaStream_t) { return FLASHSVD_ERR_UNSUPPORTED_SHAPE; }
}  // namespace fsvd
