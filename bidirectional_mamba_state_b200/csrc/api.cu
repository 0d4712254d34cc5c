// api.cu -- the C ABI of libbdscan: argument validation, workspace sizing,
// dispatch to the kernels, status reporting.  See include/bdscan.h.
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <utility>
#include <vector>

#include "bdscan.h"
#include "bdscan_internal.h"
#include <nvtx3/nvToolsExt.h>

// ---- process-wide options ------------------------------------------------------
namespace bdscan {
namespace {

struct Options {
  std::atomic<unsigned long long> wait_timeout_ns{2000000000ull};
  std::atomic<int> force_generic{0};
  std::atomic<int> verbose{0};
  std::atomic<int> cb_prepass{0};
  Options() {
    // initial values from the environment, read once
    if (const char *v = std::getenv("BDSCAN_WAIT_TIMEOUT_NS"); v && *v)
      wait_timeout_ns = std::strtoull(v, nullptr, 10);
    if (const char *v = std::getenv("BDSCAN_FORCE_GENERIC"); v && v[0] == '1') force_generic = 1;
    if (const char *v = std::getenv("BDSCAN_VERBOSE"); v && v[0] == '1') verbose = 1;
    if (const char *v = std::getenv("BDSCAN_CB_PREPASS"); v && v[0] == '1') cb_prepass = 1;
  }
};

Options &options() {
  static Options o;
  return o;
}

}  // namespace

unsigned long long opt_wait_timeout_ns() { return options().wait_timeout_ns.load(std::memory_order_relaxed); }
bool opt_force_generic() { return options().force_generic.load(std::memory_order_relaxed) != 0; }
bool opt_verbose() { return options().verbose.load(std::memory_order_relaxed) != 0; }
bool opt_cb_prepass() { return options().cb_prepass.load(std::memory_order_relaxed) != 0; }

}  // namespace bdscan

using bdscan::DirArgs;
using bdscan::Mode;
using bdscan::ScanArgs;

namespace {

// An NVTX range around each compute entry point, so that a timeline tool
// (Nsight Systems and the like) shows the library's calls by name; without a
// tool attached the calls cost a pointer check.
struct NvtxScope {
  explicit NvtxScope(const char *name) { nvtxRangePushA(name); }
  ~NvtxScope() { nvtxRangePop(); }
  NvtxScope(const NvtxScope &) = delete;
  NvtxScope &operator=(const NvtxScope &) = delete;
};


constexpr size_t kStatusBytes = 256;

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct Range {
  uintptr_t lo, hi;  // [lo, hi)
};

Range range_of(const void *p, size_t bytes) {
  uintptr_t lo = reinterpret_cast<uintptr_t>(p);
  return {lo, lo + bytes};
}

bool overlaps(Range a, Range b) { return a.lo < b.hi && b.lo < a.hi && a.hi > a.lo && b.hi > b.lo; }

int check_shape(const bdscan_shape_t *s) {
  if (!s) return BDSCAN_ERR_INVALID_ARG;
  if (s->batch < 0 || s->seqlen < 0 || s->nheads < 1 || s->headdim < 1 || s->dstate < 1 ||
      s->ngroups < 1 || s->block_len < 1 || s->chunk_len < 1)
    return BDSCAN_ERR_INVALID_ARG;
  if ((s->in_dtype != BDSCAN_BF16 && s->in_dtype != BDSCAN_FP32) ||
      (s->out_dtype != BDSCAN_BF16 && s->out_dtype != BDSCAN_FP32))
    return BDSCAN_ERR_INVALID_ARG;
  if (s->nheads % s->ngroups) return BDSCAN_ERR_UNSUPPORTED_SHAPE;
  if (s->seqlen % s->block_len) return BDSCAN_ERR_UNSUPPORTED_SHAPE;
  if (s->chunk_len % s->block_len) return BDSCAN_ERR_UNSUPPORTED_SHAPE;
  if (!(s->block_len <= 32 || (s->block_len % 32 == 0 && s->block_len <= 256)))
    return BDSCAN_ERR_UNSUPPORTED_SHAPE;
  if (!(s->headdim == 16 || s->headdim == 32 || s->headdim == 64 || s->headdim == 128))
    return BDSCAN_ERR_UNSUPPORTED_SHAPE;
  if (s->dstate > 256) return BDSCAN_ERR_UNSUPPORTED_SHAPE;
  // 32-bit grid limits of the kernels
  if (s->batch * s->nheads * (s->headdim / 16) > (int64_t)INT32_MAX) return BDSCAN_ERR_UNSUPPORTED_SHAPE;
  return BDSCAN_OK;
}

struct Sizes {
  size_t x, dt, bc, y, state, states, ad;
};

Sizes sizes_of(const bdscan_shape_t *s) {
  const size_t in = s->in_dtype == BDSCAN_BF16 ? 2 : 4, out = s->out_dtype == BDSCAN_BF16 ? 2 : 4;
  const size_t B = (size_t)s->batch, L = (size_t)s->seqlen, H = (size_t)s->nheads,
               P = (size_t)s->headdim, N = (size_t)s->dstate, G = (size_t)s->ngroups,
               K = (size_t)(s->seqlen / s->block_len);
  Sizes z;
  z.x = B * L * H * P * in;
  z.dt = B * L * H * in;
  z.bc = B * L * G * N * in;
  z.y = B * L * H * P * out;
  z.state = B * H * P * N * 4;
  z.states = B * K * H * P * N * 4;
  z.ad = H * 4;
  return z;
}

// Validates one direction; appends its input ranges to `ins`.
int check_dir(const bdscan_dir_t *d, const Sizes &z, std::vector<Range> &ins) {
  // A pointer to a zero-byte tensor may be NULL (empty batch or sequence).
  if (!d || !d->A || !d->D) return BDSCAN_ERR_INVALID_ARG;
  if (z.x && (!d->x || !d->dt || !d->B || !d->C)) return BDSCAN_ERR_INVALID_ARG;
  const void *ptrs[] = {d->x, d->dt, d->B, d->C, d->z, d->A, d->D};
  for (const void *p : ptrs)
    if (p && !aligned16(p)) return BDSCAN_ERR_MISALIGNED;
  ins.push_back(range_of(d->x, z.x));
  ins.push_back(range_of(d->dt, z.dt));
  ins.push_back(range_of(d->B, z.bc));
  ins.push_back(range_of(d->C, z.bc));
  if (d->z) ins.push_back(range_of(d->z, z.x));
  ins.push_back(range_of(d->A, z.ad));
  ins.push_back(range_of(d->D, z.ad));
  return BDSCAN_OK;
}

DirArgs to_args(const bdscan_dir_t *d) {
  DirArgs a{};
  if (d) {
    a.x = d->x; a.dt = d->dt; a.B = d->B; a.C = d->C; a.z = d->z; a.A = d->A; a.D = d->D;
  }
  return a;
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// One direction's convolved x, B and C (the scan's inputs), each 256-aligned.
size_t conv_scratch_bytes(const bdscan_shape_t *s) {
  const size_t in = s->in_dtype == BDSCAN_BF16 ? 2 : 4;
  const size_t BL = (size_t)s->batch * (size_t)s->seqlen;
  return align256(BL * (size_t)(s->nheads * s->headdim) * in) + 2 * align256(BL * (size_t)(s->ngroups * s->dstate) * in);
}

ScanArgs base_args(const bdscan_shape_t *s) {
  ScanArgs a{};
  a.Bsz = s->batch; a.L = s->seqlen; a.H = s->nheads; a.P = s->headdim; a.N = s->dstate;
  a.G = s->ngroups; a.T = s->block_len; a.Q = s->chunk_len;
  a.in_bf16 = s->in_dtype == BDSCAN_BF16;
  a.out_bf16 = s->out_dtype == BDSCAN_BF16;
  return a;
}

int check_outputs(const std::vector<Range> &ins, const std::vector<Range> &outs) {
  for (size_t i = 0; i < outs.size(); ++i) {
    for (const Range &r : ins)
      if (overlaps(outs[i], r)) return BDSCAN_ERR_INVALID_ARG;
    for (size_t j = i + 1; j < outs.size(); ++j)
      if (overlaps(outs[i], outs[j])) return BDSCAN_ERR_INVALID_ARG;
  }
  return BDSCAN_OK;
}

int check_ws(void *ws, size_t ws_bytes, size_t need) {
  if (!ws || ws_bytes < need) return BDSCAN_ERR_WORKSPACE;
  if (!aligned16(ws)) return BDSCAN_ERR_MISALIGNED;
  return BDSCAN_OK;
}

int launch(ScanArgs &a, cudaStream_t stream) {
  a.status = reinterpret_cast<int *>(a.ws);
  // The tensor-core path clears the status word in its first kernel (a
  // memset here would stand between that kernel and the one before it and
  // stop their launches from overlapping); every other path clears it here.
  const bool tc = a.Bsz > 0 && a.L > 0 && bdscan::tc_supported(a);
  if (!tc && cudaMemsetAsync(a.ws, 0, sizeof(int), stream) != cudaSuccess) return BDSCAN_ERR_CUDA;
  if (a.Bsz == 0) return BDSCAN_OK;
  if (a.L == 0) {
    // Nothing to scan: the final state is the initial one.
    if (a.final_state) {
      const size_t bytes = (size_t)(a.Bsz * a.H * a.P * a.N) * sizeof(float);
      cudaError_t e = a.h0 ? cudaMemcpyAsync(a.final_state, a.h0, bytes, cudaMemcpyDeviceToDevice, stream)
                           : cudaMemsetAsync(a.final_state, 0, bytes, stream);
      if (e != cudaSuccess) return BDSCAN_ERR_CUDA;
    }
    return BDSCAN_OK;
  }
  cudaError_t e = tc ? bdscan::launch_tc(a, stream) : bdscan::launch_seq(a, stream);
  if (e != cudaSuccess) {
    if (bdscan::opt_verbose()) std::fprintf(stderr, "libbdscan: launch failed: %s\n", cudaGetErrorString(e));
    return BDSCAN_ERR_CUDA;
  }
  return BDSCAN_OK;
}

}  // namespace

extern "C" {

size_t bdscan_workspace_size(const bdscan_shape_t *shape, int op) {
  if (check_shape(shape) != BDSCAN_OK) return 0;
  if (op == BDSCAN_OP_CONV_BLOCK_STEP) {
    // the step's workspace, then the convolved x, B, C of both directions (the
    // two-call path writes them there)
    if (shape->seqlen != shape->block_len) return 0;
    return align256(bdscan_workspace_size(shape, BDSCAN_OP_BLOCK_STEP)) + 2 * conv_scratch_bytes(shape);
  }
  if (op == BDSCAN_OP_ALLBLOCK_BACKWARD)
    return bdscan::kWsHeader + bdscan::bwd_workspace_bytes(shape->batch, shape->seqlen, shape->nheads, shape->dstate);
  if (op != BDSCAN_OP_PREFIX && op != BDSCAN_OP_BLOCK_STEP && op != BDSCAN_OP_ALLBLOCK) return 0;
  // The tensor-core path keeps C B^T of every (direction, batch, block, group)
  // in the workspace; shapes it cannot take need only the status word.
  if (bdscan::tc_shape_ok(shape->headdim, shape->dstate, shape->block_len, shape->in_dtype == BDSCAN_BF16))
    return bdscan::kWsHeader +
           bdscan::tc_workspace_bytes(shape->batch, shape->seqlen, shape->ngroups, shape->nheads,
                                      op == BDSCAN_OP_ALLBLOCK);
  return kStatusBytes;
}

int bdscan_kernel_launches(const bdscan_shape_t *shape, int op) {
  if (check_shape(shape) != BDSCAN_OK) return -1;
  if (op == BDSCAN_OP_GATED_RMSNORM) return (shape->batch == 0 || shape->seqlen == 0) ? 0 : 1;
  if (op == BDSCAN_OP_CONV_PREFIX || op == BDSCAN_OP_CONV_ALLBLOCK)
    return (shape->batch == 0 || shape->seqlen == 0) ? 0 : 1;
  if (op == BDSCAN_OP_BLOCK_STEP || op == BDSCAN_OP_CONV_BLOCK_STEP) {
    if (shape->seqlen != shape->block_len) return -1;
    if (shape->batch == 0 || shape->seqlen == 0) return 0;
    // tensor-core path: one launch for a small-batch step without state_out
    // (C B^T in the scan kernel), else pre-pass + scan; the convolution of
    // BDSCAN_OP_CONV_BLOCK_STEP adds its own kernel
    const int conv = op == BDSCAN_OP_CONV_BLOCK_STEP ? 1 : 0;
    if (bdscan::tc_shape_ok(shape->headdim, shape->dstate, shape->block_len, shape->in_dtype == BDSCAN_BF16) &&
        !bdscan::opt_force_generic()) {
      bdscan::ScanArgs a = base_args(shape);
      a.mode = bdscan::Mode::Step;
      a.has_cr = true;
      return (bdscan::tc_one_launch_step(a) ? 1 : 2) + conv;
    }
    return 1 + conv;
  }
  if (op == BDSCAN_OP_ALLBLOCK_BACKWARD) {
    // backward kernel + a dB/dC and a dA/dD reduction per present direction
    // (2 or 4 directions; counted here for all four)
    if (shape->batch == 0 || shape->seqlen == 0) return 0;
    return 1 + 2 * 4;
  }
  if (op != BDSCAN_OP_PREFIX && op != BDSCAN_OP_BLOCK_STEP && op != BDSCAN_OP_ALLBLOCK) return -1;
  if (op == BDSCAN_OP_BLOCK_STEP && shape->seqlen != shape->block_len) return -1;
  if (shape->batch == 0 || shape->seqlen == 0) return 0;
  // tensor-core path: C B^T pre-pass + scan, plus an aggregate pass and a
  // segment combine when sequences are cut into segments; generic path: one kernel
  if (bdscan::tc_shape_ok(shape->headdim, shape->dstate, shape->block_len, shape->in_dtype == BDSCAN_BF16))
    return bdscan::tc_plan_segments(shape->batch, shape->nheads, shape->seqlen / shape->block_len,
                                    op == BDSCAN_OP_ALLBLOCK) > 1
               ? 4
               : 2;
  return 1;
}

int bdscan_prefix(const bdscan_shape_t *shape, const bdscan_dir_t *fwd, const bdscan_dir_t *rev,
                  const float *h0, void *y, float *block_states, float *final_state, void *ws,
                  size_t ws_bytes, void *cuda_stream) {
  NvtxScope nvtx("bdscan_prefix");
  int rc = check_shape(shape);
  if (rc) return rc;
  const Sizes z = sizes_of(shape);
  std::vector<Range> ins, outs;
  if ((rc = check_dir(fwd, z, ins))) return rc;
  if (rev && (rc = check_dir(rev, z, ins))) return rc;
  if (!y && z.y) return BDSCAN_ERR_INVALID_ARG;
  const void *ptrs[] = {h0, y, block_states, final_state};
  for (const void *p : ptrs)
    if (p && !aligned16(p)) return BDSCAN_ERR_MISALIGNED;
  if (h0) ins.push_back(range_of(h0, z.state));
  outs.push_back(range_of(y, z.y));
  if (block_states) outs.push_back(range_of(block_states, z.states));
  if (final_state) outs.push_back(range_of(final_state, z.state));
  if ((rc = check_outputs(ins, outs))) return rc;
  if ((rc = check_ws(ws, ws_bytes, bdscan_workspace_size(shape, BDSCAN_OP_PREFIX)))) return rc;
  ScanArgs a = base_args(shape);
  a.mode = Mode::Prefix;
  a.cf = to_args(fwd);
  a.cr = to_args(rev);
  a.has_cr = rev != nullptr;
  a.h0 = h0;
  a.y_clean = y;
  a.states = block_states;
  a.final_state = final_state;
  a.ws = ws;
  a.ws_bytes = ws_bytes;
  return launch(a, static_cast<cudaStream_t>(cuda_stream));
}

int bdscan_block_step(const bdscan_shape_t *shape, const bdscan_dir_t *fwd,
                      const bdscan_dir_t *rev, const float *state_in, void *y, float *state_out,
                      void *ws, size_t ws_bytes, void *cuda_stream) {
  NvtxScope nvtx("bdscan_block_step");
  int rc = check_shape(shape);
  if (rc) return rc;
  if (shape->seqlen != shape->block_len) return BDSCAN_ERR_UNSUPPORTED_SHAPE;
  const Sizes z = sizes_of(shape);
  std::vector<Range> ins, outs;
  if ((rc = check_dir(fwd, z, ins))) return rc;
  if (rev && (rc = check_dir(rev, z, ins))) return rc;
  if ((!y && z.y) || (!state_in && z.state)) return BDSCAN_ERR_INVALID_ARG;
  const void *ptrs[] = {state_in, y, state_out};
  for (const void *p : ptrs)
    if (p && !aligned16(p)) return BDSCAN_ERR_MISALIGNED;
  // state_out may be exactly state_in (in-place commit) but must not partially
  // overlap it; an in-place state must not alias any other input.
  const Range rin = range_of(state_in, z.state);
  if (state_out == state_in) {
    for (const Range &r : ins)
      if (overlaps(rin, r)) return BDSCAN_ERR_INVALID_ARG;
  }
  ins.push_back(rin);
  outs.push_back(range_of(y, z.y));
  if (state_out && state_out != state_in) outs.push_back(range_of(state_out, z.state));
  if ((rc = check_outputs(ins, outs))) return rc;
  if ((rc = check_ws(ws, ws_bytes, bdscan_workspace_size(shape, BDSCAN_OP_BLOCK_STEP)))) return rc;
  ScanArgs a = base_args(shape);
  a.mode = Mode::Step;
  a.cf = to_args(fwd);
  a.cr = to_args(rev);
  a.has_cr = rev != nullptr;
  a.h0 = state_in;
  a.y_clean = y;
  a.final_state = state_out;
  a.ws = ws;
  a.ws_bytes = ws_bytes;
  return launch(a, static_cast<cudaStream_t>(cuda_stream));
}

int bdscan_allblock(const bdscan_shape_t *shape, const bdscan_dir_t *clean_fwd,
                    const bdscan_dir_t *clean_rev, const bdscan_dir_t *noisy_fwd,
                    const bdscan_dir_t *noisy_rev, const float *h0, void *y_clean, void *y_noisy,
                    float *block_states, void *ws, size_t ws_bytes, void *cuda_stream) {
  NvtxScope nvtx("bdscan_allblock");
  int rc = check_shape(shape);
  if (rc) return rc;
  const Sizes z = sizes_of(shape);
  std::vector<Range> ins, outs;
  if ((rc = check_dir(clean_fwd, z, ins))) return rc;
  if (clean_rev && (rc = check_dir(clean_rev, z, ins))) return rc;
  if ((rc = check_dir(noisy_fwd, z, ins))) return rc;
  if (noisy_rev && (rc = check_dir(noisy_rev, z, ins))) return rc;
  if ((!y_noisy && z.y) || (!block_states && z.states)) return BDSCAN_ERR_INVALID_ARG;
  const void *ptrs[] = {h0, y_clean, y_noisy, block_states};
  for (const void *p : ptrs)
    if (p && !aligned16(p)) return BDSCAN_ERR_MISALIGNED;
  if (h0) ins.push_back(range_of(h0, z.state));
  if (y_clean) outs.push_back(range_of(y_clean, z.y));
  outs.push_back(range_of(y_noisy, z.y));
  outs.push_back(range_of(block_states, z.states));
  if ((rc = check_outputs(ins, outs))) return rc;
  if ((rc = check_ws(ws, ws_bytes, bdscan_workspace_size(shape, BDSCAN_OP_ALLBLOCK)))) return rc;
  ScanArgs a = base_args(shape);
  a.mode = Mode::AllBlock;
  a.cf = to_args(clean_fwd);
  a.cr = to_args(clean_rev);
  a.nf = to_args(noisy_fwd);
  a.nr = to_args(noisy_rev);
  a.has_cr = clean_rev != nullptr;
  a.has_nr = noisy_rev != nullptr;
  a.h0 = h0;
  a.y_clean = y_clean;
  a.y_noisy = y_noisy;
  a.states = block_states;
  a.ws = ws;
  a.ws_bytes = ws_bytes;
  return launch(a, static_cast<cudaStream_t>(cuda_stream));
}

int bdscan_allblock_backward(const bdscan_shape_t *shape, const bdscan_dir_t *clean_fwd,
                             const bdscan_dir_t *clean_rev, const bdscan_dir_t *noisy_fwd,
                             const bdscan_dir_t *noisy_rev, const float *h0, const float *block_states,
                             const void *dy_clean, const void *dy_noisy, const float *dstates,
                             const bdscan_grad_t *g_clean_fwd, const bdscan_grad_t *g_clean_rev,
                             const bdscan_grad_t *g_noisy_fwd, const bdscan_grad_t *g_noisy_rev,
                             float *dh0, void *ws, size_t ws_bytes, void *cuda_stream) {
  NvtxScope nvtx("bdscan_allblock_backward");
  int rc = check_shape(shape);
  if (rc) return rc;
  const Sizes z = sizes_of(shape);
  // the backward's shared-memory plan: 16-byte rows (block_len and d_state
  // multiples of 4) that fit one CTA
  if (shape->block_len % 4 || shape->dstate % 4 ||
      bdscan::bwd_smem_bytes(shape->headdim, shape->dstate, shape->block_len) > 227u * 1024u)
    return BDSCAN_ERR_UNSUPPORTED_SHAPE;
  const bdscan_dir_t *dirs[4] = {clean_fwd, clean_rev, noisy_fwd, noisy_rev};
  const bdscan_grad_t *grads[4] = {g_clean_fwd, g_clean_rev, g_noisy_fwd, g_noisy_rev};
  if (!clean_fwd || !noisy_fwd) return BDSCAN_ERR_INVALID_ARG;
  std::vector<Range> ins, outs;
  const size_t f32 = 4, B = (size_t)shape->batch, L = (size_t)shape->seqlen, H = (size_t)shape->nheads,
               P = (size_t)shape->headdim, N = (size_t)shape->dstate, G = (size_t)shape->ngroups;
  for (int i = 0; i < 4; ++i) {
    if (!dirs[i]) continue;
    if ((rc = check_dir(dirs[i], z, ins))) return rc;
    if (dirs[i]->z) return BDSCAN_ERR_UNSUPPORTED_SHAPE;  // gated backward is not provided
    const bdscan_grad_t *g = grads[i];
    if (!g || (z.x && (!g->dx || !g->ddt || !g->dB || !g->dC)) || !g->dA || !g->dD) return BDSCAN_ERR_INVALID_ARG;
    const void *gp[] = {g->dx, g->ddt, g->dB, g->dC, g->dA, g->dD};
    for (const void *q : gp)
      if (q && !aligned16(q)) return BDSCAN_ERR_MISALIGNED;
    outs.push_back(range_of(g->dx, B * L * H * P * f32));
    outs.push_back(range_of(g->ddt, B * L * H * f32));
    outs.push_back(range_of(g->dB, B * L * G * N * f32));
    outs.push_back(range_of(g->dC, B * L * G * N * f32));
    outs.push_back(range_of(g->dA, H * f32));
    outs.push_back(range_of(g->dD, H * f32));
  }
  if ((!block_states && z.states) || (!dy_noisy && z.y)) return BDSCAN_ERR_INVALID_ARG;
  const void *ptrs[] = {h0, block_states, dy_clean, dy_noisy, dstates, dh0};
  for (const void *q : ptrs)
    if (q && !aligned16(q)) return BDSCAN_ERR_MISALIGNED;
  if (h0) ins.push_back(range_of(h0, z.state));
  ins.push_back(range_of(block_states, z.states));
  if (dy_clean) ins.push_back(range_of(dy_clean, z.y));
  ins.push_back(range_of(dy_noisy, z.y));
  if (dstates) ins.push_back(range_of(dstates, z.states));
  if (dh0) outs.push_back(range_of(dh0, z.state));
  if ((rc = check_outputs(ins, outs))) return rc;
  if ((rc = check_ws(ws, ws_bytes, bdscan_workspace_size(shape, BDSCAN_OP_ALLBLOCK_BACKWARD)))) return rc;
  cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
  if (cudaMemsetAsync(ws, 0, sizeof(int), stream) != cudaSuccess) return BDSCAN_ERR_CUDA;
  if (shape->batch == 0) return BDSCAN_OK;
  if (shape->seqlen == 0) {
    // nothing scanned: all gradients are zero, dh0 = dstates has no blocks
    for (int i = 0; i < 4; ++i)
      if (dirs[i] && (cudaMemsetAsync(grads[i]->dA, 0, H * f32, stream) != cudaSuccess ||
                      cudaMemsetAsync(grads[i]->dD, 0, H * f32, stream) != cudaSuccess))
        return BDSCAN_ERR_CUDA;
    if (dh0 && cudaMemsetAsync(dh0, 0, z.state, stream) != cudaSuccess) return BDSCAN_ERR_CUDA;
    return BDSCAN_OK;
  }
  bdscan::BwdArgs a{};
  a.Bsz = shape->batch; a.L = shape->seqlen; a.H = shape->nheads; a.P = shape->headdim;
  a.N = shape->dstate; a.G = shape->ngroups; a.T = shape->block_len;
  a.in_bf16 = shape->in_dtype == BDSCAN_BF16;
  a.dy_bf16 = shape->out_dtype == BDSCAN_BF16;
  for (int i = 0; i < 4; ++i) {
    a.dir[i] = to_args(dirs[i]);
    if (dirs[i]) {
      const bdscan_grad_t *g = grads[i];
      a.grad[i] = bdscan::GradArgs{g->dx, g->ddt, g->dB, g->dC, g->dA, g->dD};
    }
  }
  a.h0 = h0;
  a.states = block_states;
  a.dstates = dstates;
  a.dy_clean = dy_clean;
  a.dy_noisy = dy_noisy;
  a.dh0 = dh0;
  a.ws = static_cast<uint8_t *>(ws) + bdscan::kWsHeader;
  cudaError_t e = bdscan::launch_bwd(a, stream);
  if (e != cudaSuccess) {
    if (bdscan::opt_verbose()) std::fprintf(stderr, "libbdscan: launch failed: %s\n", cudaGetErrorString(e));
    return BDSCAN_ERR_CUDA;
  }
  return BDSCAN_OK;
}

int bdscan_check_status(const void *ws, void *cuda_stream) {
  if (!ws) return BDSCAN_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  int host = 0;
  if (cudaMemcpyAsync(&host, ws, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return BDSCAN_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return BDSCAN_ERR_CUDA;
  if (host != 0) {
    if (cudaMemsetAsync(const_cast<void *>(ws), 0, sizeof(int), st) != cudaSuccess)
      return BDSCAN_ERR_CUDA;
  }
  return host;
}

const char *bdscan_status_string(int status) {
  switch (status) {
    case BDSCAN_OK: return "ok";
    case BDSCAN_ERR_INVALID_ARG: return "invalid argument (null pointer, bad enum or overlapping buffers)";
    case BDSCAN_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case BDSCAN_ERR_MISALIGNED: return "pointer not 16-byte aligned";
    case BDSCAN_ERR_WORKSPACE: return "workspace missing or too small";
    case BDSCAN_ERR_CUDA: return "CUDA launch or runtime error";
    case BDSCAN_ERR_TIMEOUT: return "bounded device-side wait timed out";
    case BDSCAN_ERR_SCRATCH_LIMIT:
      return "shape needs more scratch than the no-alloc entry point's built-in buffer holds";
    default: return "unknown status";
  }
}

int bdscan_version(void) { return 100; }

long long bdscan_set_option(int option, long long value) {
  auto &o = bdscan::options();
  switch (option) {
    case BDSCAN_OPT_WAIT_TIMEOUT_NS:
      if (value < 0) return BDSCAN_ERR_INVALID_ARG;
      return (long long)o.wait_timeout_ns.exchange((unsigned long long)value);
    case BDSCAN_OPT_FORCE_GENERIC:
      if (value != 0 && value != 1) return BDSCAN_ERR_INVALID_ARG;
      return o.force_generic.exchange((int)value);
    case BDSCAN_OPT_VERBOSE:
      if (value != 0 && value != 1) return BDSCAN_ERR_INVALID_ARG;
      return o.verbose.exchange((int)value);
    case BDSCAN_OPT_CB_PREPASS:
      if (value != 0 && value != 1) return BDSCAN_ERR_INVALID_ARG;
      return o.cb_prepass.exchange((int)value);
    default:
      return BDSCAN_ERR_INVALID_ARG;
  }
}

long long bdscan_get_option(int option) {
  switch (option) {
    case BDSCAN_OPT_WAIT_TIMEOUT_NS: return (long long)bdscan::opt_wait_timeout_ns();
    case BDSCAN_OPT_FORCE_GENERIC: return bdscan::opt_force_generic() ? 1 : 0;
    case BDSCAN_OPT_VERBOSE: return bdscan::opt_verbose() ? 1 : 0;
    case BDSCAN_OPT_CB_PREPASS: return bdscan::opt_cb_prepass() ? 1 : 0;
    default: return BDSCAN_ERR_INVALID_ARG;
  }
}

}  // extern "C"

// ---------------------------------------------------------------- no-alloc step
// Scratch of bdscan_block_step_noalloc: a static device buffer (every GPU that
// loads the library holds it until exit).  Host code must not pass the symbol
// itself to a kernel -- on the host it is only a stand-in -- but the device
// address that cudaGetSymbolAddress returns for the current device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[BDSCAN_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
struct ScratchAddr {
  void *ctx;  // the context the address was looked up in
  void *ptr;
};
ScratchAddr g_noalloc[kMaxDevices] = {};

// The driver's cuCtxGetCurrent, through the runtime's entry-point query (the
// library links only the runtime).
using CtxGetCurrentFn = int (*)(void **);
CtxGetCurrentFn ctx_get_current_fn() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  return fn;
}

// Device address of the scratch buffer on the current device, looked up once per
// device and context (with that device current): a device reset or a new primary
// context reloads the module, and the address is looked up again in the new
// context.  nullptr if a lookup fails.
void *noalloc_scratch_ptr() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  CtxGetCurrentFn get = ctx_get_current_fn();
  void *ctx = nullptr;
  if (!get || get(&ctx) != 0) return nullptr;
  if (!ctx) {
    // no context bound to this thread yet: the symbol lookup makes the
    // device's primary context current
    void *ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || get(&ctx) != 0 || !ctx) return nullptr;
  }
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  ScratchAddr &e = g_noalloc[dev];
  if (!e.ptr || e.ctx != ctx) {
    void *ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess) return nullptr;
    e.ctx = ctx;
    e.ptr = ptr;
  }
  return e.ptr;
}

}  // namespace

extern "C" {

void *bdscan_noalloc_scratch(void) { return noalloc_scratch_ptr(); }

int bdscan_block_step_noalloc(const bdscan_shape_t *shape, const bdscan_dir_t *fwd,
                              const bdscan_dir_t *rev, const float *state_in, void *y,
                              float *state_out, void *cuda_stream) {
  const size_t need = bdscan_workspace_size(shape, BDSCAN_OP_BLOCK_STEP);
  if (need == 0) {
    const int rc = check_shape(shape);
    return rc ? rc : BDSCAN_ERR_INVALID_ARG;
  }
  if (need > BDSCAN_NOALLOC_SCRATCH_BYTES) return BDSCAN_ERR_SCRATCH_LIMIT;
  void *ws = noalloc_scratch_ptr();
  if (!ws) return BDSCAN_ERR_CUDA;
  // The call clears the status word itself; the C B^T tiles are fully rewritten
  // before they are read, so nothing else needs to start at zero.
  return bdscan_block_step(shape, fwd, rev, state_in, y, state_out, ws, BDSCAN_NOALLOC_SCRATCH_BYTES,
                           cuda_stream);
}

}  // extern "C"

// ---- short convolution in front of the scan --------------------------------
namespace {

struct ConvSizes {
  size_t x, bc, w, bias, state;
  int64_t Cx;
};

ConvSizes conv_sizes(const bdscan_shape_t *s, int width) {
  const size_t in = s->in_dtype == BDSCAN_BF16 ? 2 : 4;
  const size_t B = (size_t)s->batch, L = (size_t)s->seqlen, H = (size_t)s->nheads,
               P = (size_t)s->headdim, N = (size_t)s->dstate, G = (size_t)s->ngroups;
  ConvSizes z;
  z.Cx = (int64_t)(H * P + 2 * G * N);
  z.x = B * L * H * P * in;
  z.bc = B * L * G * N * in;
  z.w = (size_t)z.Cx * (size_t)width * 4;
  z.bias = (size_t)z.Cx * 4;
  z.state = B * (size_t)(width - 1) * (size_t)z.Cx * in;
  return z;
}

int check_conv_shape(const bdscan_shape_t *shape, int width) {
  int rc = check_shape(shape);
  if (rc) return rc;
  if (width < 1 || width > 4) return BDSCAN_ERR_UNSUPPORTED_SHAPE;
  // B and C rows must be whole 4-channel vectors
  if ((shape->ngroups * shape->dstate) % 4) return BDSCAN_ERR_UNSUPPORTED_SHAPE;
  return BDSCAN_OK;
}

// Validates one direction of the convolution; appends its ranges.
int check_conv_dir(const bdscan_conv_t *d, const ConvSizes &z, std::vector<Range> &ins,
                   std::vector<Range> &outs) {
  if (!d || !d->weight) return BDSCAN_ERR_INVALID_ARG;
  if (z.x && (!d->x || !d->B || !d->C || !d->x_out || !d->B_out || !d->C_out)) return BDSCAN_ERR_INVALID_ARG;
  const void *ptrs[] = {d->x, d->B, d->C, d->weight, d->bias, d->x_out, d->B_out, d->C_out};
  for (const void *p : ptrs)
    if (p && !aligned16(p)) return BDSCAN_ERR_MISALIGNED;
  ins.push_back(range_of(d->x, z.x));
  ins.push_back(range_of(d->B, z.bc));
  ins.push_back(range_of(d->C, z.bc));
  ins.push_back(range_of(d->weight, z.w));
  if (d->bias) ins.push_back(range_of(d->bias, z.bias));
  outs.push_back(range_of(d->x_out, z.x));
  outs.push_back(range_of(d->B_out, z.bc));
  outs.push_back(range_of(d->C_out, z.bc));
  return BDSCAN_OK;
}

bdscan::ConvDirArgs to_conv_args(const bdscan_conv_t *d) {
  bdscan::ConvDirArgs a{};
  if (d) {
    a.x = d->x; a.B = d->B; a.C = d->C; a.weight = d->weight; a.bias = d->bias;
    a.x_out = d->x_out; a.B_out = d->B_out; a.C_out = d->C_out;
  }
  return a;
}

bdscan::ConvArgs conv_base(const bdscan_shape_t *s, int width, int silu) {
  bdscan::ConvArgs a{};
  a.Bsz = s->batch; a.L = s->seqlen; a.H = s->nheads; a.P = s->headdim; a.N = s->dstate;
  a.G = s->ngroups; a.T = s->block_len; a.W = width;
  a.in_bf16 = s->in_dtype == BDSCAN_BF16;
  a.silu = silu != 0;
  return a;
}

int conv_launch(const bdscan::ConvArgs &a, const ConvSizes &z, cudaStream_t stream) {
  if (a.Bsz == 0) return BDSCAN_OK;
  if (a.L == 0) {
    // nothing to convolve: the new conv state is the old one (or zeros)
    if (a.state_out && a.state_out != a.state_in && z.state) {
      cudaError_t e = a.state_in ? cudaMemcpyAsync(a.state_out, a.state_in, z.state, cudaMemcpyDeviceToDevice, stream)
                                 : cudaMemsetAsync(a.state_out, 0, z.state, stream);
      if (e != cudaSuccess) return BDSCAN_ERR_CUDA;
    }
    return BDSCAN_OK;
  }
  cudaError_t e = bdscan::launch_conv(a, stream);
  if (e != cudaSuccess) {
    if (bdscan::opt_verbose()) std::fprintf(stderr, "libbdscan: conv launch failed: %s\n", cudaGetErrorString(e));
    return BDSCAN_ERR_CUDA;
  }
  return BDSCAN_OK;
}

}  // namespace

extern "C" {

int bdscan_conv_prefix(const bdscan_shape_t *shape, int width, int silu, const bdscan_conv_t *fwd,
                       const bdscan_conv_t *rev, const void *conv_state_in, void *conv_state_out,
                       void *cuda_stream) {
  NvtxScope nvtx("bdscan_conv_prefix");
  int rc = check_conv_shape(shape, width);
  if (rc) return rc;
  const ConvSizes z = conv_sizes(shape, width);
  std::vector<Range> ins, outs;
  if ((rc = check_conv_dir(fwd, z, ins, outs))) return rc;
  if (rev && (rc = check_conv_dir(rev, z, ins, outs))) return rc;
  if ((conv_state_in && !aligned16(conv_state_in)) || (conv_state_out && !aligned16(conv_state_out)))
    return BDSCAN_ERR_MISALIGNED;
  const Range rin = range_of(conv_state_in, z.state);
  if (conv_state_out && conv_state_out == conv_state_in) {
    // in place: each thread reads its state rows before it writes them, which
    // needs the whole sequence in one tile
    if (shape->seqlen > 32) return BDSCAN_ERR_INVALID_ARG;
    for (const Range &r : ins)
      if (overlaps(rin, r)) return BDSCAN_ERR_INVALID_ARG;
  }
  if (conv_state_in) ins.push_back(rin);
  if (conv_state_out && conv_state_out != conv_state_in) outs.push_back(range_of(conv_state_out, z.state));
  if ((rc = check_outputs(ins, outs))) return rc;
  bdscan::ConvArgs a = conv_base(shape, width, silu);
  a.dir[0] = to_conv_args(fwd);
  a.dir[1] = to_conv_args(rev);
  a.state_in = conv_state_in;
  a.state_out = conv_state_out;
  return conv_launch(a, z, static_cast<cudaStream_t>(cuda_stream));
}

int bdscan_conv_allblock(const bdscan_shape_t *shape, int width, int silu,
                         const bdscan_conv_t *clean_fwd, const bdscan_conv_t *clean_rev,
                         const bdscan_conv_t *noisy_fwd, const bdscan_conv_t *noisy_rev,
                         const void *conv_state_in, void *cuda_stream) {
  NvtxScope nvtx("bdscan_conv_allblock");
  int rc = check_conv_shape(shape, width);
  if (rc) return rc;
  const ConvSizes z = conv_sizes(shape, width);
  std::vector<Range> ins, outs;
  if ((rc = check_conv_dir(clean_fwd, z, ins, outs))) return rc;
  if (clean_rev && (rc = check_conv_dir(clean_rev, z, ins, outs))) return rc;
  if ((rc = check_conv_dir(noisy_fwd, z, ins, outs))) return rc;
  if (noisy_rev && (rc = check_conv_dir(noisy_rev, z, ins, outs))) return rc;
  if (conv_state_in && !aligned16(conv_state_in)) return BDSCAN_ERR_MISALIGNED;
  if (conv_state_in) ins.push_back(range_of(conv_state_in, z.state));
  if ((rc = check_outputs(ins, outs))) return rc;
  bdscan::ConvArgs a = conv_base(shape, width, silu);
  a.dir[0] = to_conv_args(clean_fwd);
  a.dir[1] = to_conv_args(clean_rev);
  a.dir[2] = to_conv_args(noisy_fwd);
  a.dir[3] = to_conv_args(noisy_rev);
  a.state_in = conv_state_in;
  return conv_launch(a, z, static_cast<cudaStream_t>(cuda_stream));
}

int bdscan_conv_block_step(const bdscan_shape_t *shape, int width, int silu, const bdscan_conv_t *conv_fwd,
                           const bdscan_conv_t *conv_rev, const void *conv_state_in, const bdscan_dir_t *fwd,
                           const bdscan_dir_t *rev, const float *state_in, void *y, void *ws, size_t ws_bytes,
                           void *cuda_stream) {
  NvtxScope nvtx("bdscan_conv_block_step");
  int rc = check_conv_shape(shape, width);
  if (rc) return rc;
  if (shape->seqlen != shape->block_len) return BDSCAN_ERR_UNSUPPORTED_SHAPE;
  if (!conv_fwd || !conv_rev || !fwd || !rev) return BDSCAN_ERR_INVALID_ARG;
  const ConvSizes cz = conv_sizes(shape, width);
  const Sizes z = sizes_of(shape);
  std::vector<Range> ins, outs;
  // convolution inputs (its outputs are not used by this call)
  for (const bdscan_conv_t *d : {conv_fwd, conv_rev}) {
    if (!d->weight) return BDSCAN_ERR_INVALID_ARG;
    if (cz.x && (!d->x || !d->B || !d->C)) return BDSCAN_ERR_INVALID_ARG;
    const void *ptrs[] = {d->x, d->B, d->C, d->weight, d->bias};
    for (const void *p : ptrs)
      if (p && !aligned16(p)) return BDSCAN_ERR_MISALIGNED;
    ins.push_back(range_of(d->x, cz.x));
    ins.push_back(range_of(d->B, cz.bc));
    ins.push_back(range_of(d->C, cz.bc));
    ins.push_back(range_of(d->weight, cz.w));
    if (d->bias) ins.push_back(range_of(d->bias, cz.bias));
  }
  // scan directions: dt, A, D, z (their x, B, C are not used)
  for (const bdscan_dir_t *d : {fwd, rev}) {
    if (!d->A || !d->D || (z.dt && !d->dt)) return BDSCAN_ERR_INVALID_ARG;
    const void *ptrs[] = {d->dt, d->z, d->A, d->D};
    for (const void *p : ptrs)
      if (p && !aligned16(p)) return BDSCAN_ERR_MISALIGNED;
    ins.push_back(range_of(d->dt, z.dt));
    if (d->z) ins.push_back(range_of(d->z, z.x));
    ins.push_back(range_of(d->A, z.ad));
    ins.push_back(range_of(d->D, z.ad));
  }
  if ((!y && z.y) || (!state_in && z.state)) return BDSCAN_ERR_INVALID_ARG;
  const void *ptrs[] = {conv_state_in, state_in, y};
  for (const void *p : ptrs)
    if (p && !aligned16(p)) return BDSCAN_ERR_MISALIGNED;
  if (conv_state_in) ins.push_back(range_of(conv_state_in, cz.state));
  ins.push_back(range_of(state_in, z.state));
  outs.push_back(range_of(y, z.y));
  if ((rc = check_outputs(ins, outs))) return rc;
  if ((rc = check_ws(ws, ws_bytes, bdscan_workspace_size(shape, BDSCAN_OP_CONV_BLOCK_STEP)))) return rc;
  // the convolved inputs live in the workspace past the step's own part
  const size_t step_ws = align256(bdscan_workspace_size(shape, BDSCAN_OP_BLOCK_STEP));
  const size_t in = shape->in_dtype == BDSCAN_BF16 ? 2 : 4;
  const size_t BL = (size_t)shape->batch * (size_t)shape->seqlen;
  const size_t xb = align256(BL * (size_t)(shape->nheads * shape->headdim) * in);
  const size_t bcb = align256(BL * (size_t)(shape->ngroups * shape->dstate) * in);
  uint8_t *scratch = static_cast<uint8_t *>(ws) + step_ws;
  bdscan::ConvArgs ca = conv_base(shape, width, silu);
  bdscan::ScanArgs a = base_args(shape);
  a.mode = bdscan::Mode::Step;
  a.has_cr = true;
  a.h0 = state_in;
  a.y_clean = y;
  a.ws = ws;
  a.ws_bytes = step_ws;
  const bdscan_conv_t *cd[2] = {conv_fwd, conv_rev};
  const bdscan_dir_t *sd[2] = {fwd, rev};
  for (int d = 0; d < 2; ++d) {
    uint8_t *base = scratch + d * (xb + 2 * bcb);
    ca.dir[d] = to_conv_args(cd[d]);
    ca.dir[d].x_out = base;
    ca.dir[d].B_out = base + xb;
    ca.dir[d].C_out = base + xb + bcb;
    bdscan::DirArgs &da = d == 0 ? a.cf : a.cr;
    da = to_args(sd[d]);
    da.x = ca.dir[d].x_out;
    da.B = ca.dir[d].B_out;
    da.C = ca.dir[d].C_out;
  }
  ca.state_in = conv_state_in;
  ca.state_out = nullptr;
  // The convolution into the workspace, then the step (the step's kernel is a
  // programmatic dependent of the convolution's: its prologue overlaps it).
  // Convolving inside the one-launch step kernel was measured slower: every
  // (sequence, head) CTA would recompute its group's B and C convolution.
  const cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
  if ((rc = conv_launch(ca, cz, stream))) return rc;
  return launch(a, stream);
}

}  // extern "C"

// ---- gated RMSNorm of the summed output ----------------------------------------
extern "C" {

int bdscan_gated_rmsnorm(const bdscan_shape_t *shape, const void *y, const void *z, const float *weight,
                         int64_t groups, float eps, void *out, void *cuda_stream) {
  NvtxScope nvtx("bdscan_gated_rmsnorm");
  int rc = check_shape(shape);
  if (rc) return rc;
  const int64_t C = shape->nheads * shape->headdim;
  if (groups < 1 || !(eps >= 0.0f) || eps > 3.0e38f) return BDSCAN_ERR_INVALID_ARG;
  if (C % groups || (C / groups) % 4 || bdscan::norm_smem_bytes(C, groups) > 227u * 1024u)
    return BDSCAN_ERR_UNSUPPORTED_SHAPE;
  const size_t rows = (size_t)shape->batch * (size_t)shape->seqlen;
  if (rows > (size_t)INT32_MAX) return BDSCAN_ERR_UNSUPPORTED_SHAPE;  // one CTA per row
  const size_t ysz = rows * (size_t)C * (shape->out_dtype == BDSCAN_BF16 ? 2 : 4);
  const size_t zsz = rows * (size_t)C * (shape->in_dtype == BDSCAN_BF16 ? 2 : 4);
  const size_t osz = rows * (size_t)C * 2;
  if (!weight || (rows && (!y || !out))) return BDSCAN_ERR_INVALID_ARG;
  const void *ptrs[] = {y, z, weight, out};
  for (const void *p : ptrs)
    if (p && !aligned16(p)) return BDSCAN_ERR_MISALIGNED;
  const Range ro = range_of(out, osz);
  // in place (out == y) only when y is bf16: each row is read whole before it is written
  const bool in_place = out == y && shape->out_dtype == BDSCAN_BF16;
  if (!in_place && overlaps(ro, range_of(y, ysz))) return BDSCAN_ERR_INVALID_ARG;
  if (z && overlaps(ro, range_of(z, zsz))) return BDSCAN_ERR_INVALID_ARG;
  if (overlaps(ro, range_of(weight, (size_t)C * 4))) return BDSCAN_ERR_INVALID_ARG;
  bdscan::NormArgs a{};
  a.Bsz = shape->batch; a.L = shape->seqlen; a.C = C; a.groups = groups; a.eps = eps;
  a.y = y; a.z = z; a.weight = weight; a.out = out;
  a.y_bf16 = shape->out_dtype == BDSCAN_BF16;
  a.z_bf16 = shape->in_dtype == BDSCAN_BF16;
  cudaError_t e = bdscan::launch_norm(a, static_cast<cudaStream_t>(cuda_stream));
  if (e != cudaSuccess) {
    if (bdscan::opt_verbose()) std::fprintf(stderr, "libbdscan: norm launch failed: %s\n", cudaGetErrorString(e));
    return BDSCAN_ERR_CUDA;
  }
  return BDSCAN_OK;
}

}  // extern "C"
