// scan_fwd_bf16.cu -- instantiations of the fused forward kernel for
// __nv_bfloat16 inputs and __nv_bfloat16 outputs (one translation unit per dtype pair so the
// variants compile in parallel).
#include "scan_fwd_kernel.cuh"

namespace ssm {

cudaError_t fwd_dispatch_bf16(const LaunchShape *ls, const TmaMaps *maps, const FwdParams *p,
                            cudaStream_t st, VariantInfo *vi) {
  return by_ns<__nv_bfloat16, __nv_bfloat16>(ls, maps, p, st, vi);
}

}  // namespace ssm
