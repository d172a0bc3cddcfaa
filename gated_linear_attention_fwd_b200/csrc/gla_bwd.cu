// gla_bwd.cu -- placeholder until the backward kernel lands.
#include "gla.h"
namespace dig {
cudaError_t launch_gla_bwd(const GlaVariant&, const GlaArgs&, int, bool, cudaStream_t) { return cudaErrorNotSupported; }
int gla_bwd_blocks_per_sm(const GlaVariant&) { return 0; }
}  // namespace dig
