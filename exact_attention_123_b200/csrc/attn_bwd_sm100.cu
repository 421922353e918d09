// attn_bwd_sm100.cu -- placeholder until the backward kernels land.
#include "attn_launch.h"
namespace attn {
cudaError_t launch_bwd(const BwdLaunch &, cudaStream_t) { return cudaErrorNotSupported; }
}  // namespace attn
