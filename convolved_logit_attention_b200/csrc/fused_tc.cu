// Fused tcgen05 MTA forward (placeholder until the kernel lands).
#include "mta_internal.h"

namespace mta {

bool fused_supported(const mta_shape &) { return false; }
size_t fused_workspace_bytes(const mta_shape &) { return 0; }
int fused_kernel_count(const mta_shape &) { return 0; }
const char *fused_kernel_name(const mta_shape &, int) { return nullptr; }
mta_status launch_fused(const mta_shape &, const ForwardArgs &, void *, cudaStream_t,
                        const Trace &)
{
    return MTA_ERR_UNSUPPORTED;
}
unsigned int fused_take_error() { return 0; }

}  // namespace mta
