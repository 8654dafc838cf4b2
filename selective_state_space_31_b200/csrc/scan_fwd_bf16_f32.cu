// scan_fwd_bf16_f32.cu -- instantiations of the fused forward kernel for
// __nv_bfloat16 inputs and float outputs (one translation unit per dtype pair so the
// variants compile in parallel).
#include "scan_fwd_kernel.cuh"

namespace ssm {

cudaError_t fwd_dispatch_bf16_f32(const LaunchShape *ls, const TmaMaps *maps, const FwdParams *p,
                            cudaStream_t st, VariantInfo *vi) {
  return by_ns<__nv_bfloat16, float>(ls, maps, p, st, vi);
}

}  // namespace ssm
