// usp_attn_bwd.cu -- backward of the blockwise attention (placeholder until the kernel lands).
#include "usp_internal.h"

namespace usp {
cudaError_t launch_attn_bwd(const BwdLaunch&, cudaStream_t) { return cudaErrorNotSupported; }
}  // namespace usp
