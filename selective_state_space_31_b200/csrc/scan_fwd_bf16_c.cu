// scan_fwd_bf16_c.cu -- compiled variants of the fused forward kernel for bf16 inputs and outputs, dstate 8
// (the variant tables are split over translation units so they compile in
// parallel).
#include "scan_fwd_kernel.cuh"
#include "scan_fwd_variants.h"

namespace ssm {

cudaError_t fwd_table_bf16_c(const LaunchShape *ls, const TmaMaps *maps, const FwdParams *p,
                           cudaStream_t st, VariantInfo *vi) {
#define SSM_X(NS, LPC, KC, W, TT, ZOH, CARRY, CONV, OPT)                                  \
  if (shape_is(ls, NS, LPC, KC, W, TT, ZOH, CARRY, CONV, OPT))                              \
    return run_variant<__nv_bfloat16, __nv_bfloat16, NS, LPC, KC, W, TT, ZOH, CARRY, CONV, OPT>(ls, maps, p, st, vi);
  SSM_FWD_BF16_N8(SSM_X)
#undef SSM_X
  return cudaErrorNotSupported;
}

int fwd_list_bf16_c(VariantDesc *out, int max) {
  int n = 0;
#define SSM_X(NS, LPC, KC, W, TT, ZOH, CARRY, CONV, OPT)                                  \
  if (n < max) out[n] = VariantDesc{NS, LPC, KC, W, TT, ZOH, CARRY, CONV, OPT};              \
  ++n;
  SSM_FWD_BF16_N8(SSM_X)
#undef SSM_X
  return n;
}

}  // namespace ssm
