// scan_fwd_f32.cu -- instantiations of the fused forward kernel for
// float inputs and float outputs (one translation unit per dtype pair so the
// variants compile in parallel).
#include "scan_fwd_kernel.cuh"

namespace ssm {

cudaError_t fwd_dispatch_f32(const LaunchShape *ls, const TmaMaps *maps, const FwdParams *p,
                            cudaStream_t st, VariantInfo *vi) {
  return by_ns<float, float>(ls, maps, p, st, vi);
}

}  // namespace ssm
