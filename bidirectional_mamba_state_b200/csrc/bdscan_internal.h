// Internal launch interface between the C-ABI layer (api.cu) and the kernels.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

namespace bdscan {

enum class Mode : int { Prefix = 0, Step = 1, AllBlock = 2 };

// Process-wide options (bdscan_set_option); read from the environment once,
// at the first use, not per call.
unsigned long long opt_wait_timeout_ns();
bool opt_force_generic();
bool opt_verbose();
bool opt_cb_prepass();

struct DirArgs {
  const void *x, *dt, *B, *C, *z;  // z == nullptr: no gate
  const float *A, *D;
};

// One fully validated call.  Step is expressed as a prefix over a single block
// (h0 = state_in, final_state = state_out).
struct ScanArgs {
  int64_t Bsz, L, H, P, N, G, T, Q;
  bool in_bf16, out_bf16;
  Mode mode;
  DirArgs cf, cr, nf, nr;  // clean fwd/rev, noisy fwd/rev (noisy: AllBlock only)
  bool has_cr, has_nr;
  const float *h0;         // nullptr = zeros
  void *y_clean;           // may be nullptr (AllBlock)
  void *y_noisy;           // AllBlock only
  float *states;           // [B][K][H][P][N] or nullptr
  float *final_state;      // [B][H][P][N] or nullptr
  void *ws;                // workspace (>= 256 B); first word: device status
  size_t ws_bytes;
  int *status;             // == ws
};

// Generic path: direct sequential recurrence on CUDA cores (any supported
// shape, fp32 or bf16 inputs, gated or not).
cudaError_t launch_seq(const ScanArgs &a, cudaStream_t stream);

// Workspace: [0, kWsHeader) status word (first int); the tensor-core path's
// C B^T tiles follow.
constexpr size_t kWsHeader = 1024;

// Tensor-core path (sm_100a): bf16 inputs, P = 64, N = 128, T = 32, no gate.
bool tc_shape_ok(int64_t P, int64_t N, int64_t T, bool in_bf16);
size_t tc_workspace_bytes(int64_t Bsz, int64_t L, int64_t G, int64_t H, bool allblock);
int tc_plan_segments(int64_t Bsz, int64_t H, int64_t K, bool allblock);
bool tc_supported(const ScanArgs &a);
// Small-batch step without a state chain: C B^T computed in the scan kernel,
// one launch (see scan_tc.cu).
bool tc_one_launch_step(const ScanArgs &a);
cudaError_t launch_tc(const ScanArgs &a, cudaStream_t stream);

// Backward of the all-block pass (generic kernel, any accepted ungated shape
// whose block fits the shared-memory plan).
struct GradArgs {
  float *dx, *ddt, *dB, *dC, *dA, *dD;
};
struct BwdArgs {
  int64_t Bsz, L, H, P, N, G, T;
  bool in_bf16, dy_bf16;
  DirArgs dir[4];   // clean fwd, clean rev, noisy fwd, noisy rev (x == nullptr: absent)
  GradArgs grad[4];
  const float *h0, *states, *dstates;
  const void *dy_clean, *dy_noisy;
  float *dh0;
  void *ws;         // partial sums (bwd_workspace_bytes)
};
size_t bwd_smem_bytes(int64_t P, int64_t N, int64_t T);
size_t bwd_workspace_bytes(int64_t Bsz, int64_t L, int64_t H, int64_t N);
cudaError_t launch_bwd(const BwdArgs &a, cudaStream_t stream);

// Short convolution (+SiLU) in front of the scan.
struct ConvDirArgs {
  const void *x, *B, *C;         // pre-convolution inputs (x == nullptr: absent direction)
  const float *weight, *bias;    // [Cx][W], [Cx] or nullptr
  void *x_out, *B_out, *C_out;
};
struct ConvArgs {
  int64_t Bsz, L, H, P, N, G, T;
  int W;
  bool in_bf16, silu;
  ConvDirArgs dir[4];  // clean (or prefix) fwd, its rev, noisy fwd, noisy rev
  const void *state_in;  // [B][W-1][Cx] or nullptr
  void *state_out;       // [B][W-1][Cx] or nullptr (dir[0]'s last rows)
};
int conv_tile(const ConvArgs &a);
cudaError_t launch_conv(const ConvArgs &a, cudaStream_t stream);

// Gated RMSNorm of the summed output, bf16 result.
struct NormArgs {
  int64_t Bsz, L, C, groups;  // rows = Bsz * L, C = H * P channels per row
  float eps;
  const void *y, *z;          // y: out_dtype, z: in_dtype or nullptr
  const float *weight;        // [C]
  void *out;                  // bf16 [rows][C]
  bool y_bf16, z_bf16;
};
size_t norm_smem_bytes(int64_t C, int64_t groups);
cudaError_t launch_norm(const NormArgs &a, cudaStream_t stream);

}  // namespace bdscan
