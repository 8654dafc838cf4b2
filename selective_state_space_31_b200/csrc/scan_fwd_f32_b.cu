// scan_fwd_f32_b.cu -- compiled variants of the fused forward kernel for fp32 inputs and outputs, dstate 8 and 4
// (the variant tables are split over translation units so they compile in
// parallel).
#include "scan_fwd_kernel.cuh"
#include "scan_fwd_variants.h"

namespace ssm {

cudaError_t fwd_table_f32_b(const LaunchShape *ls, const TmaMaps *maps, const FwdParams *p,
                           cudaStream_t st, VariantInfo *vi) {
#define SSM_X(NS, LPC, KC, W, TT, ZOH, CARRY, CONV, OPT)                                  \
  if (shape_is(ls, NS, LPC, KC, W, TT, ZOH, CARRY, CONV, OPT))                              \
    return run_variant<float, float, NS, LPC, KC, W, TT, ZOH, CARRY, CONV, OPT>(ls, maps, p, st, vi);
  SSM_FWD_F32_N8_N4(SSM_X)
#undef SSM_X
  return cudaErrorNotSupported;
}

int fwd_list_f32_b(VariantDesc *out, int max) {
  int n = 0;
#define SSM_X(NS, LPC, KC, W, TT, ZOH, CARRY, CONV, OPT)                                  \
  if (n < max) out[n] = VariantDesc{NS, LPC, KC, W, TT, ZOH, CARRY, CONV, OPT};              \
  ++n;
  SSM_FWD_F32_N8_N4(SSM_X)
#undef SSM_X
  return n;
}

}  // namespace ssm
