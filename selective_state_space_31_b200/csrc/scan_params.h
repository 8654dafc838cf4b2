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
  int M;        // segments per row (1 = the row is one chain of parts)
  int SPS;      // stages per segment (the last one may be shorter)
  int PL;       // stages per part (work item) of a segment; carry pass: per sub-chunk
  int items;    // work items of the launch
  int nq;       // carry sub-chunks per segment
  int nsub_row; // carry sub-chunks per row ((M - 1) * nq)
  bool softplus, has_z, has_D, has_bias, has_h0, want_hlast;
  bool zoh;            // zero-order-hold Bbar (selects the kernel template too)
  const float *A;      // (D, N)
  const float *Dv;     // (D) or null
  const float *bias;   // (D) or null
  const float *h0;     // (B, D, N) or null
  float *h_last;       // (B, D, N) or null
  void *y;             // (B, L, D) output
  float *ws_state;     // rows * M * DT * N carried states
  unsigned long long *ws_flags;  // rows * M * warps carry flags
  float *agg_h;        // (B, nsub_row, D, N) states each carry sub-chunk reaches from 0
  float *agg_s;        // (B, nsub_row, D) sum of Delta over each carry sub-chunk
  const float *conv_w; // (D, 4) taps of the x branch's causal conv (conv variants)
  const float *conv_b; // (D) or null
  void *xconv;         // (B, L, D) out dtype: the conv output, or null
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
  bool zoh;    // zero-order-hold variant of the kernel
  int kc = 1;  // channels per lane
  bool carry = false;  // the carry pass of a segmented launch
  bool conv = false;   // the x branch comes through the causal conv front-end
  int opt = 0;         // bit 0: software-pipelined scan loop; bit 1: five CTAs per SM
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
  int kc = 0;        // channels per lane
  int segments = 0;  // segments per row (1 = none)
  int opt = 0;       // 1 + the variant's OPT bits (0 = free choice)
  int carry_lpc = 0;  // carry pass: lanes per channel (0 = free choice)
  int carry_opt = 0;  // carry pass: 1 + its OPT bits (0 = free choice)
  int carry_kc = 0;   // carry pass: channels per lane (0 = free choice)
};
// A launch shape of the fused kernel with its work split.
struct FwdShape {
  LaunchShape ls;  // lpc, warps, tt, stages, ns, grid, smem, zoh, kc
  int DT;          // channels per row tile
  int64_t rows;    // batch * ceil(dim / DT)
  int S;           // stages per row
  int M;           // segments per row
  int SPS;         // stages per segment
  int PL;          // stages per part
  int parts;       // parts per segment
  int ring;        // stage slots in the TMA ring
  // carry pass (M > 1): its launch shape and sub-chunk split
  LaunchShape cls;
  int cDT;         // channels per row tile of the carry pass
  int64_t crows;   // its rows
  int Q;           // stages per carry sub-chunk
  int nq;          // sub-chunks per segment
};
// The carry pass run over a whole sequence (the map of a sequence): its
// launch shape and the sub-chunks the sequence is cut into.
struct MapShape {
  LaunchShape ls;
  int DT;          // channels per row tile
  int64_t rows;    // batch * ceil(dim / DT)
  int Q;           // stages per sub-chunk
  int nsub;        // sub-chunks per row
};
// Choose the map pass for a fused-kernel shape (same stage length).
cudaError_t choose_map_shape(int in_dtype, int out_dtype, int64_t batch, int64_t dim,
                             const FwdShape &fs, int sms, MapShape *out);

// One compiled variant of the fused kernel (for listing and tests).
struct VariantDesc {
  int ns, lpc, kc, warps, tt;
  bool zoh, carry, conv;
  int opt;
};
// The variants compiled for a dtype pair; returns how many (fills up to max).
int fwd_variants(int in_dtype, int out_dtype, VariantDesc *out, int max);
// Choose the fused kernel's launch shape for a problem (scan_fwd_dispatch.cu).
// Returns cudaErrorInvalidValue when no variant fits the overrides.
cudaError_t choose_fwd_shape(int in_dtype, int out_dtype, int64_t batch, int64_t seqlen,
                             int64_t dim, int ns, bool zoh, bool conv, int sms,
                             const FwdOverrides &o, FwdShape *out);

struct GenericParams {
  int Bsz, L, D, N;
  bool softplus, has_z, has_D, has_bias, has_h0, want_hlast, zoh;
  int in_bf16, out_bf16;
  const void *x, *dt, *z, *B, *C;
  const float *A, *Dv, *bias, *h0;
  void *y;
  float *h_last;
  // conv front-end of the x branch (x holds x_in when conv_w is set)
  const float *conv_w = nullptr;  // (D, kConvWidth)
  const float *conv_b = nullptr;  // (D) or null
  void *xconv = nullptr;          // (B, L, D) out dtype, or null
};

// Taps of the causal conv front-end of the x branch.
constexpr int kConvWidth = 4;
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

// Map (sum of Delta, state from 0) of a whole sequence, general kernel.
struct MapParams {
  int Bsz, L, D, N;
  bool softplus, zoh;
  int in_bf16;
  const void *x, *dt, *B;
  const float *A, *bias;
  float *map_h;  // (B, D, N)
  float *map_s;  // (B, D)
};
cudaError_t launch_map_general(const MapParams &p, cudaStream_t stream);

// Composition of `count` maps onto h0 (scan_carry.cu).  Map j of channel
// (b, d) sits at element b * stride_b + j * stride_j + d of maps_s (times N,
// plus n, in maps_h).
struct FoldParams {
  int Bsz, D, N, count;
  long long stride_b, stride_j;
  const float *A;
  const float *maps_h, *maps_s;
  const float *h0;  // (B, D, N) or null (0)
  float *h_out;     // (B, D, N)
  float *s_out;     // (B, D) sum of the maps' Delta sums, or null
};
cudaError_t launch_fold_maps(const FoldParams &p, cudaStream_t stream);

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
