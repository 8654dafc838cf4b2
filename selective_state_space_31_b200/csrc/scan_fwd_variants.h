// scan_fwd_variants.h -- the compiled variants of the fused forward kernel,
// X(NS, LPC, KC, WARPS, TT, ZOH, CARRY, CONV, OPT), one list per dtype pair and dstate
// (OPT bit 0: software-pipelined scan loop; bit 1: five CTAs per SM; bit 2:
// B and C widened to fp32 once per CTA by the load warp, bf16 inputs only;
// bit 3: a quarter of the state exponentials on the FMA pipe; bit 4: the
// pipelined loop prepares two tokens ahead).
// Only these shapes exist in the library; the planner chooses among them.
// Row tiles need DT = WARPS * (32 / LPC) * KC channels whose bytes are a
// multiple of 16 (TMA rows); two channels per lane need an even NPL.
#pragma once

// ---- bf16 in, bf16 out ----
#define SSM_FWD_BF16_N16(X)                                                              \
  X(16, 4, 1, 4, 32, false, false, false, 1) X(16, 8, 1, 4, 64, false, false, false, 1)  \
  X(16, 4, 1, 4, 64, false, false, false, 1) X(16, 8, 1, 4, 32, false, false, false, 1)  \
  X(16, 4, 1, 4, 32, false, false, false, 2) X(16, 8, 1, 4, 64, false, false, false, 2)  \
  X(16, 4, 1, 4, 32, false, false, false, 3) X(16, 8, 1, 4, 64, false, false, false, 3)  \
  X(16, 8, 1, 4, 64, false, false, false, 5) X(16, 4, 1, 4, 32, false, false, false, 4)  \
  X(16, 4, 1, 4, 32, false, false, false, 8)                                              \
  X(16, 8, 1, 4, 64, false, false, false, 17)                                             \
  X(16, 1, 1, 4, 32, false, false, false, 0) X(16, 2, 1, 4, 32, false, false, false, 0)                      \
  X(16, 4, 1, 4, 32, false, false, false, 0) X(16, 4, 1, 4, 64, false, false, false, 0)                      \
  X(16, 8, 1, 4, 32, false, false, false, 0) X(16, 8, 1, 4, 64, false, false, false, 0)                      \
  X(16, 16, 1, 4, 32, false, false, false, 0) X(16, 16, 1, 4, 64, false, false, false, 0)                    \
  X(16, 4, 1, 2, 32, false, false, false, 0) X(16, 8, 1, 2, 32, false, false, false, 0)                      \
  X(16, 8, 1, 8, 32, false, false, false, 0) X(16, 16, 1, 8, 32, false, false, false, 0)                     \
  X(16, 2, 2, 4, 32, false, false, false, 0)                                                       \
  X(16, 4, 2, 4, 32, false, false, false, 0) X(16, 4, 2, 4, 64, false, false, false, 0)                      \
  X(16, 8, 2, 4, 32, false, false, false, 0) X(16, 8, 2, 4, 64, false, false, false, 0)                      \
  X(16, 4, 2, 8, 32, false, false, false, 0) X(16, 8, 2, 8, 32, false, false, false, 0)
#define SSM_FWD_BF16_N16_ZOH_CARRY(X)                                                    \
  X(16, 4, 1, 4, 32, false, true, false, 4)                                              \
  X(16, 4, 1, 4, 32, true, false, false, 0) X(16, 4, 1, 4, 64, true, false, false, 0)                        \
  X(16, 8, 1, 4, 32, true, false, false, 0) X(16, 8, 1, 4, 64, true, false, false, 0)                        \
  X(16, 16, 1, 4, 32, true, false, false, 0) X(16, 16, 1, 4, 64, true, false, false, 0)                      \
  X(16, 4, 2, 4, 32, true, false, false, 0) X(16, 8, 2, 4, 32, true, false, false, 0)                        \
  X(16, 4, 1, 4, 32, false, true, false, 0) X(16, 4, 1, 4, 64, false, true, false, 0)                        \
  X(16, 8, 1, 4, 32, false, true, false, 0) X(16, 8, 1, 4, 64, false, true, false, 0)                        \
  X(16, 16, 1, 4, 32, false, true, false, 0) X(16, 16, 1, 4, 64, false, true, false, 0)                      \
  X(16, 4, 2, 4, 32, false, true, false, 0) X(16, 4, 2, 4, 64, false, true, false, 0)                        \
  X(16, 8, 2, 4, 32, false, true, false, 0) X(16, 8, 2, 4, 64, false, true, false, 0)                        \
  X(16, 4, 1, 4, 32, true, true, false, 0) X(16, 4, 1, 4, 64, true, true, false, 0)                          \
  X(16, 8, 1, 4, 32, true, true, false, 0) X(16, 8, 1, 4, 64, true, true, false, 0)                          \
  X(16, 16, 1, 4, 32, true, true, false, 0) X(16, 16, 1, 4, 64, true, true, false, 0)                        \
  X(16, 4, 1, 4, 32, false, true, false, 8)
#define SSM_FWD_BF16_N8(X)                                                               \
  X(8, 2, 1, 4, 32, false, false, false, 0) X(8, 2, 1, 4, 64, false, false, false, 0)                        \
  X(8, 4, 1, 4, 32, false, false, false, 0) X(8, 4, 1, 4, 64, false, false, false, 0)                        \
  X(8, 8, 1, 4, 32, false, false, false, 0) X(8, 8, 1, 4, 64, false, false, false, 0)                        \
  X(8, 4, 1, 2, 32, false, false, false, 0) X(8, 8, 1, 2, 32, false, false, false, 0)                        \
  X(8, 2, 2, 4, 32, false, false, false, 0) X(8, 4, 2, 4, 32, false, false, false, 0)                        \
  X(8, 4, 1, 4, 32, true, false, false, 0) X(8, 4, 1, 4, 64, true, false, false, 0)                          \
  X(8, 8, 1, 4, 32, true, false, false, 0) X(8, 8, 1, 4, 64, true, false, false, 0)                          \
  X(8, 4, 1, 4, 32, false, true, false, 0) X(8, 4, 1, 4, 64, false, true, false, 0)                          \
  X(8, 8, 1, 4, 32, false, true, false, 0) X(8, 8, 1, 4, 64, false, true, false, 0)                          \
  X(8, 4, 1, 4, 64, true, true, false, 0) X(8, 8, 1, 4, 64, true, true, false, 0)                            \
  X(8, 4, 1, 4, 32, true, true, false, 0) X(8, 8, 1, 4, 32, true, true, false, 0)

// ---- bf16 in, fp32 out ----
#define SSM_FWD_BF16_F32(X)                                                              \
  X(16, 4, 1, 4, 32, false, false, false, 0) X(16, 4, 1, 4, 64, false, false, false, 0)                      \
  X(16, 8, 1, 4, 32, false, false, false, 0) X(16, 8, 1, 4, 64, false, false, false, 0)                      \
  X(16, 16, 1, 4, 32, false, false, false, 0) X(16, 16, 1, 4, 64, false, false, false, 0)                    \
  X(16, 4, 2, 4, 32, false, false, false, 0) X(16, 8, 2, 4, 32, false, false, false, 0)                      \
  X(16, 4, 1, 4, 64, true, false, false, 0) X(16, 8, 1, 4, 64, true, false, false, 0)                        \
  X(16, 4, 1, 4, 32, false, true, false, 0) X(16, 4, 1, 4, 64, false, true, false, 0)                        \
  X(16, 8, 1, 4, 32, false, true, false, 0) X(16, 8, 1, 4, 64, false, true, false, 0)                        \
  X(16, 16, 1, 4, 32, false, true, false, 0) X(16, 16, 1, 4, 64, false, true, false, 0)                      \
  X(16, 4, 1, 4, 64, true, true, false, 0) X(16, 8, 1, 4, 64, true, true, false, 0)                          \
  X(8, 4, 1, 4, 32, false, false, false, 0) X(8, 4, 1, 4, 64, false, false, false, 0)                        \
  X(8, 8, 1, 4, 32, false, false, false, 0) X(8, 8, 1, 4, 64, false, false, false, 0)                        \
  X(8, 4, 2, 4, 32, false, false, false, 0)                                                        \
  X(8, 4, 1, 4, 32, false, true, false, 0) X(8, 4, 1, 4, 64, false, true, false, 0)                          \
  X(8, 8, 1, 4, 32, false, true, false, 0) X(8, 8, 1, 4, 64, false, true, false, 0)

// ---- fp32 in, fp32 out ----
#define SSM_FWD_F32_N16(X)                                                               \
  X(16, 4, 1, 4, 32, false, false, false, 1)                                          \
  X(16, 1, 1, 4, 32, false, false, false, 0) X(16, 2, 1, 4, 32, false, false, false, 0)                      \
  X(16, 4, 1, 4, 32, false, false, false, 0) X(16, 8, 1, 4, 32, false, false, false, 0)                      \
  X(16, 16, 1, 4, 32, false, false, false, 0) X(16, 4, 1, 4, 64, false, false, false, 0)                     \
  X(16, 8, 1, 4, 64, false, false, false, 0) X(16, 16, 1, 4, 64, false, false, false, 0)                     \
  X(16, 4, 1, 2, 32, false, false, false, 0) X(16, 8, 1, 2, 32, false, false, false, 0)                      \
  X(16, 16, 1, 2, 32, false, false, false, 0)                                                      \
  X(16, 2, 2, 4, 32, false, false, false, 0) X(16, 4, 2, 4, 32, false, false, false, 0)                      \
  X(16, 8, 2, 4, 32, false, false, false, 0)                                                       \
  X(16, 4, 1, 4, 32, true, false, false, 0) X(16, 4, 1, 4, 64, true, false, false, 0)                        \
  X(16, 8, 1, 4, 32, true, false, false, 0) X(16, 8, 1, 4, 64, true, false, false, 0)                        \
  X(16, 16, 1, 4, 32, true, false, false, 0) X(16, 16, 1, 4, 64, true, false, false, 0)                      \
  X(16, 4, 2, 4, 32, true, false, false, 0)                                                        \
  X(16, 4, 1, 4, 32, false, true, false, 0) X(16, 4, 1, 4, 64, false, true, false, 0)                        \
  X(16, 8, 1, 4, 32, false, true, false, 0) X(16, 8, 1, 4, 64, false, true, false, 0)                        \
  X(16, 16, 1, 4, 32, false, true, false, 0) X(16, 16, 1, 4, 64, false, true, false, 0)                      \
  X(16, 4, 2, 4, 32, false, true, false, 0)                                                        \
  X(16, 4, 1, 4, 32, true, true, false, 0) X(16, 4, 1, 4, 64, true, true, false, 0)                          \
  X(16, 8, 1, 4, 32, true, true, false, 0) X(16, 8, 1, 4, 64, true, true, false, 0)                          \
  X(16, 16, 1, 4, 32, true, true, false, 0) X(16, 16, 1, 4, 64, true, true, false, 0)
#define SSM_FWD_F32_N8_N4(X)                                                             \
  X(8, 2, 1, 4, 32, false, false, false, 0) X(8, 2, 1, 4, 64, false, false, false, 0)                        \
  X(8, 4, 1, 4, 32, false, false, false, 0) X(8, 4, 1, 4, 64, false, false, false, 0)                        \
  X(8, 8, 1, 4, 32, false, false, false, 0) X(8, 8, 1, 4, 64, false, false, false, 0)                        \
  X(8, 4, 1, 2, 32, false, false, false, 0) X(8, 8, 1, 2, 32, false, false, false, 0)                        \
  X(8, 2, 2, 4, 32, false, false, false, 0) X(8, 4, 2, 4, 32, false, false, false, 0)                        \
  X(8, 4, 1, 4, 32, true, false, false, 0) X(8, 4, 1, 4, 64, true, false, false, 0)                          \
  X(8, 8, 1, 4, 32, true, false, false, 0) X(8, 8, 1, 4, 64, true, false, false, 0)                          \
  X(8, 4, 1, 4, 32, false, true, false, 0) X(8, 4, 1, 4, 64, false, true, false, 0)                          \
  X(8, 8, 1, 4, 32, false, true, false, 0) X(8, 8, 1, 4, 64, false, true, false, 0)                          \
  X(8, 4, 1, 4, 64, true, true, false, 0) X(8, 8, 1, 4, 64, true, true, false, 0)                            \
  X(8, 4, 1, 4, 32, true, true, false, 0) X(8, 8, 1, 4, 32, true, true, false, 0)                            \
  X(4, 1, 1, 4, 32, false, false, false, 0) X(4, 2, 1, 4, 32, false, false, false, 0)                        \
  X(4, 4, 1, 4, 32, false, false, false, 0) X(4, 4, 1, 4, 64, false, false, false, 0)                        \
  X(4, 4, 1, 2, 32, false, false, false, 0) X(4, 2, 2, 4, 32, false, false, false, 0)                        \
  X(4, 2, 1, 4, 32, true, false, false, 0) X(4, 2, 1, 4, 64, true, false, false, 0)                          \
  X(4, 4, 1, 4, 32, true, false, false, 0) X(4, 4, 1, 4, 64, true, false, false, 0)                          \
  X(4, 2, 1, 4, 32, false, true, false, 0) X(4, 2, 1, 4, 64, false, true, false, 0)                          \
  X(4, 4, 1, 4, 32, false, true, false, 0) X(4, 4, 1, 4, 64, false, true, false, 0)                          \
  X(4, 2, 1, 4, 64, true, true, false, 0) X(4, 4, 1, 4, 64, true, true, false, 0)                            \
  X(4, 2, 1, 4, 32, true, true, false, 0) X(4, 4, 1, 4, 32, true, true, false, 0)

// ---- the causal conv front-end of the x branch (CONV) ----
#define SSM_FWD_BF16_CONV(X)                                                             \
  X(16, 4, 1, 4, 32, false, false, true, 0) X(16, 8, 1, 4, 32, false, false, true, 0)          \
  X(16, 4, 2, 4, 32, false, false, true, 0) X(16, 8, 2, 4, 32, false, false, true, 0)          \
  X(16, 4, 1, 4, 32, false, true, true, 0) X(16, 8, 1, 4, 32, false, true, true, 0)            \
  X(16, 4, 2, 4, 32, false, true, true, 0) X(16, 8, 2, 4, 32, false, true, true, 0)
#define SSM_FWD_F32_CONV(X)                                                              \
  X(16, 4, 1, 4, 32, false, false, true, 0) X(16, 4, 2, 4, 32, false, false, true, 0)          \
  X(16, 4, 1, 4, 32, false, true, true, 0) X(16, 4, 2, 4, 32, false, true, true, 0)
