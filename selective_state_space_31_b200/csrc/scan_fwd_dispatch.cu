// scan_fwd_dispatch.cu -- dtype dispatch of the fused forward kernel.
#include "scan_fwd_kernel.cuh"

namespace ssm {

static cudaError_t dispatch(int in_dtype, int out_dtype, const LaunchShape *ls,
                            const TmaMaps *maps, const FwdParams *p, cudaStream_t st,
                            size_t *sm, int *oc) {
  if (in_dtype == 0 && out_dtype == 0) return fwd_dispatch_f32(ls, maps, p, st, sm, oc);
  if (in_dtype == 1 && out_dtype == 1) return fwd_dispatch_bf16(ls, maps, p, st, sm, oc);
  if (in_dtype == 1 && out_dtype == 0) return fwd_dispatch_bf16_f32(ls, maps, p, st, sm, oc);
  return cudaErrorInvalidValue;
}

cudaError_t launch_fwd_tma(int in_dtype, int out_dtype, const LaunchShape &ls,
                           const TmaMaps &maps, const FwdParams &p, cudaStream_t stream) {
  return dispatch(in_dtype, out_dtype, &ls, &maps, &p, stream, nullptr, nullptr);
}

cudaError_t fwd_tma_smem_and_occupancy(int in_dtype, int out_dtype, const LaunchShape &ls,
                                       size_t *smem, int *blocks_per_sm) {
  return dispatch(in_dtype, out_dtype, &ls, nullptr, nullptr, nullptr, smem, blocks_per_sm);
}

}  // namespace ssm
