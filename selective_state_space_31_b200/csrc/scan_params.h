// scan_params.h -- parameter blocks passed from the C-ABI layer to the
// kernel launchers (internal to the library).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ssm {

// Device-resident control block of one plan.  The last CTA of each chunked
// launch resets `done` and advances `epoch`, so consecutive calls
// need no memset and work under stream capture.
struct Control {
  unsigned long long reserved;
  unsigned int done;        // CTAs finished in the current launch
  unsigned int epoch;       // launch counter, tags the carry flags
  int status;               // 0 or a timeout code, sticky until read
  unsigned int ticket;      // next work item to hand out in the current launch
  int pad[2];
};
static_assert(sizeof(Control) == 32, "control block layout");

struct FwdParams {
  int Bsz, L, D, N;
  int DT;       // channels per row tile
  int nDT;      // row tiles per batch element
  int rows;     // Bsz * nDT
  int S;        // stages (of the kernel's stage length) per row
  int PL;       // stages per part (work item) of a row
  int items;    // rows * parts per row
  bool softplus, has_z, has_D, has_bias, has_h0, want_hlast;
  bool zoh;            // zero-order-hold Bbar (selects the kernel template too)
  const float *A;      // (D, N)
  const float *Dv;     // (D) or null
  const float *bias;   // (D) or null
  const float *h0;     // (B, D, N) or null
  float *h_last;       // (B, D, N) or null
  void *y;             // (B, L, D) output
  float *ws_state;     // rows * DT * N carried states
  unsigned long long *ws_flags;  // rows * warps carry flags
  Control *ctl;
  unsigned long long timeout_ns;
  long long drop_unit;  // test hook: the run ending at this unit does not hand on its state
};

struct TmaMaps {
  CUtensorMap x, dt, z, B, C;
};

struct LaunchShape {
  int lpc, warps, tt, stages, ns;
  int grid;
  size_t smem;
  bool zoh;  // zero-order-hold variant of the kernel
};

// Fused forward kernel (scan_fwd_kernel.cuh, instantiated per dtype pair).
cudaError_t launch_fwd_tma(int in_dtype, int out_dtype, const LaunchShape &ls,
                           const TmaMaps &maps, const FwdParams &p, cudaStream_t stream);
// What one fused-kernel variant needs and gets on the device.
struct VariantInfo {
  size_t smem;  // dynamic shared memory per CTA
  int occ;      // CTAs resident per SM
  int ring;     // stage slots in the TMA ring
};
cudaError_t fwd_variant_info(int in_dtype, int out_dtype, const LaunchShape &ls,
                             VariantInfo *vi);

// Pipeline tag every fused-kernel LaunchShape carries (`stages`).
constexpr int kStages = 2;

// Launch-shape overrides (0 = free choice).
struct FwdOverrides {
  int lpc, warps, tt, grid;
};
// (the zero-order-hold variants exist for 32- and 64-token stages only)
// A launch shape of the fused kernel with its work split.
struct FwdShape {
  LaunchShape ls;  // lpc, warps, tt, stages, ns, grid, smem
  int DT;          // channels per row tile
  int64_t rows;    // batch * ceil(dim / DT)
  int S;           // stages per row
  int PL;          // stages per part
  int parts;       // parts per row
  int ring;        // stage slots in the TMA ring
};
// Choose the fused kernel's launch shape for a problem (scan_fwd_dispatch.cu).
// Returns cudaErrorInvalidValue when no variant fits the overrides.
cudaError_t choose_fwd_shape(int in_dtype, int out_dtype, int64_t batch, int64_t seqlen,
                             int64_t dim, int ns, bool zoh, int sms, const FwdOverrides &o,
                             FwdShape *out);

struct GenericParams {
  int Bsz, L, D, N;
  bool softplus, has_z, has_D, has_bias, has_h0, want_hlast, zoh;
  int in_bf16, out_bf16;
  const void *x, *dt, *z, *B, *C;
  const float *A, *Dv, *bias, *h0;
  void *y;
  float *h_last;
};
// General forward kernel: any shape and alignment (scan_general.cu).
cudaError_t launch_fwd_general(const GenericParams &p, cudaStream_t stream);

struct DirectParams {
  int Bsz, L, D;
  int in_bf16, out_bf16;
  const void *x, *A, *B, *C;
  const float *h0;
  void *y;
  float *h_last;
};
// Elementwise (N = 1, A given per token) variant (scan_general.cu).
cudaError_t launch_direct(const DirectParams &p, cudaStream_t stream);

struct StepParams {
  int Bsz, D, N;
  bool softplus, has_z, has_D, has_bias, zoh;
  int in_bf16, out_bf16;
  const void *x, *dt, *z, *B, *C;
  const float *A, *Dv, *bias;
  float *state;
  void *y;
};
// Decode step (scan_step.cu).
cudaError_t launch_step(const StepParams &p, cudaStream_t stream);

}  // namespace ssm
