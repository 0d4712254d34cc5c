// scan_tc.cu -- tensor-core block-diffusion scan for sm_100a
// (bf16 inputs, headdim P = 64, d_state N = 128, block T = 32; gated or not).
//
// Chunked (state-space-duality) form, one 32-token block at a time, of the
// recurrence of "Training Hybrid Block Diffusion Language Models with Partial
// Bidirectionality", eq. (1), with cum_t = sum_{u<=t in block} dt_u A and
// rcum_t = sum_{u>=t in block} dt_u A:
//
//   CB^T[s][t] = B_s . C_t                    per (b, group, block, direction)
//   M[t][s]    = CB[t][s] dt_s exp(cum_t - cum_s),   s <= t   (forward)
//              = CB[t][s] dt_s exp(rcum_t - rcum_s), s >= t   (block-local
//                reverse, eq. (12))
//   Y_diag     = M X                          (intra-block term)
//   Y_off      = C h_{k-1}^T                  (continuation from the boundary
//                state, eq. (11))
//   S          = (w o X)^T B,   w_t = dt_t exp(cum_31 - cum_t)
//   h_k        = exp(cum_31) h_{k-1} + S      (boundary state, eq. (10))
//   y_t        = exp(cum_t) Y_off + Y_diag,fwd + Y_diag,rev + D_f x_f + D_r x_r
//                (sum of the two directions, eq. (13))
// The all-block pass (eq. (14)) adds the noisy stream: its forward part starts
// from the same h_{k-1} (the clean boundary state before block k), its
// reverse part is block-local.
//
// Kernels:
//   bd_cb_kernel  C B^T of every (direction, batch, block, group) -- shared by
//                 all heads of a group -- with one M=128 tcgen05 MMA chain per
//                 four blocks, into the workspace (bf16, 2 KB per block; the
//                 masked-decay matrix built from it is rounded to bf16 anyway).
//   bd_tc_kernel  persistent, one CTA per SM: each CTA walks its share of the
//                 work items -- (b, h) sequences, or segments of them -- block
//                 by block with the fp32 state on chip, the pipeline running
//                 on across item boundaries.  Warp roles (512 threads; warp w
//                 runs on SM sub-partition w mod 4):
//     warp 0      TMA producer: x, B, C and C B^T tiles of block k into a
//                 3-slot ring (two blocks of lookahead)
//     warp 1      TMEM allocator and single-thread tcgen05.mma issuer
//     warps 2,3,6,7  operands: per-step decay tables, (w o X) (bf16 hi + lo)
//     warps 4,5   idle (they keep the operand warps off the MMA issuer's
//                 sub-partition)
//     warps 8-11  state chain: thread n keeps column n of the fp32 state,
//                 h_k = exp(cum_31) h_{k-1} + S; boundary-state stores (one
//                 128-byte line per warp instruction); h operand (bf16 hi + lo)
//     warps 12-15 epilogue: thread (p, stream) forms y[t][p] = exp(cum_t) Y_off
//                 + Y_diag for the block's 32 tokens and stores them.  Two
//                 blocks ahead, the same warps build the masked-decay matrices
//                 M with each direction's D added to the diagonal (so D x is
//                 part of Y_diag), stored bf16, next to a diagonal matrix of
//                 that diagonal's bf16 remainders: one N = 64 MMA per 16
//                 tokens gives both, summed by the epilogue.  With a gate
//                 (y_dir * silu(z_dir) before the sum) each direction keeps its
//                 own Y_diag accumulator and the epilogue loads z; that
//                 epilogue lives only in the gated instance of the kernel.
//   S, Y and M are double-buffered (Y single-buffered with a gate: its five
//   accumulators fill the TMEM); the h operand is single-buffered.
//   bd_agg_kernel and bd_seg_combine_kernel  (segmented plans: few long
//                 sequences cut into segments) each segment's state from a
//                 zero start as one contraction over its tokens, then the
//                 chain of segment states; the scan kernel then starts each
//                 segment from its true initial state.
// Every wait is bounded; on a timeout the CTA raises BDSCAN_ERR_TIMEOUT in the
// workspace status word, drains its own copies and MMAs, frees TMEM and exits.
//
// Precision: C, B and x are bf16 (exact).  fp32 operands (w o X and the state
// h) are split into bf16 hi + lo parts and fed as two MMAs (~16 mantissa
// bits); M is rounded once to bf16 (it multiplies exact x and only forms the
// intra-block term).  All accumulation is fp32 in TMEM.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "bdscan_internal.h"
#include "sm100.cuh"

namespace bdscan {
namespace {

using namespace sm100;

constexpr int kT = 32, kP = 64, kN = 128;
// stacking slots of the four directions
// (the MMAs and the masked-decay buffers rely on: stream = slot & 1, reverse = slot >= 2)
constexpr int kCF = 0, kNF = 1, kCR = 2, kNR = 3;
static_assert(kCR == (kCF | 2) && kNR == (kNF | 2), "direction slots");
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kStatusTimeout = -6;

constexpr uint32_t kTile = 4096;  // 32 rows x 128 bytes

// ------------------------------------------------------------------ C B^T kernel
constexpr int kCbThreads = 128;
constexpr uint32_t kCbOffBlo = 0, kCbOffBhi = 4 * kTile, kCbOffClo = 8 * kTile, kCbOffChi = 12 * kTile;
constexpr uint32_t kCbOffBar = 16 * kTile;
constexpr uint32_t kCbSmem = kCbOffBar + 64 + 1024;

struct CbParams {
  CUtensorMap tb[4];
  CUtensorMap tc[4];
  int slot[4];  // blockIdx.z -> the direction's C B^T tile set (see cb_set)
  int Bsz, K, G;
  __nv_bfloat16 *cb;  // [4][B][K][G][32 s][32 t]
  int *item_counters;  // the scan passes' work-item counters, zeroed here
  int *status;
  unsigned long long timeout_ns;
};

__device__ __forceinline__ uint32_t pack2(uint32_t lo_bits, uint32_t hi_bits) {
  __nv_bfloat162 v = __floats2bfloat162_rn(__uint_as_float(lo_bits), __uint_as_float(hi_bits));
  return *reinterpret_cast<uint32_t *>(&v);
}

__global__ void __launch_bounds__(kCbThreads) bd_cb_kernel(const __grid_constant__ CbParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t *sm = smem_raw + (base - raw);
  uint64_t *bars = reinterpret_cast<uint64_t *>(sm + kCbOffBar);
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(sm + kCbOffBar + 16);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + kCbOffBar + 20);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int z = blockIdx.z, slot = p.slot[z];
  const int b = blockIdx.y / p.G, g = blockIdx.y % p.G;
  const int k0 = 4 * blockIdx.x;
  const int nvalid = min(4, p.K - k0);
  // Launched as a programmatic dependent of whatever kernel precedes it on the
  // stream (e.g. the short convolution that writes B and C): wait for it before
  // touching memory, then clear the status word and the work counters.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0) {
    if (threadIdx.x < 2) p.item_counters[threadIdx.x] = 0;
    if (threadIdx.x == 2) *p.status = 0;
  }
  // The scan kernel that follows may start now: it reads x, B and C before
  // its own wait, which is safe because every CTA of this grid triggers only
  // after the wait above, i.e. after all earlier kernels have completed.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (threadIdx.x == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(&bars[0], nvalid * 4 * kTile);
    for (int j = 0; j < nvalid; ++j) {
      const int t0 = (k0 + j) * kT;
      tma_load_4d(sm + kCbOffBlo + j * kTile, &p.tb[z], &bars[0], 0, g, t0, b);
      tma_load_4d(sm + kCbOffBhi + j * kTile, &p.tb[z], &bars[0], 64, g, t0, b);
      tma_load_4d(sm + kCbOffClo + j * kTile, &p.tc[z], &bars[0], 0, g, t0, b);
      tma_load_4d(sm + kCbOffChi + j * kTile, &p.tc[z], &bars[0], 64, g, t0, b);
    }
    if (mbar_wait(&bars[0], 0, p.timeout_ns, nullptr)) {
      tc_fence_after();
      const uint32_t id = idesc_bf16(128, 128, 0, 0);
      for (int ks = 0; ks < 8; ++ks) {
        const uint32_t off = (ks & 3) * 32;
        const uint64_t a = sdesc(base + (ks < 4 ? kCbOffBlo : kCbOffBhi) + off, 16, 1024, kLayoutSw128);
        const uint64_t bb = sdesc(base + (ks < 4 ? kCbOffClo : kCbOffChi) + off, 16, 1024, kLayoutSw128);
        umma_bf16(tmem, a, bb, id, ks > 0);
      }
    } else {
      *abort_flag = 1;
      atomicCAS(p.status, 0, kStatusTimeout);
      // the loads of this CTA must land before its shared memory is released
      (void)mbar_wait(&bars[0], 0, 1000000000ull, nullptr);
    }
    umma_commit(&bars[1]);
  }
  bool ok = mbar_wait(&bars[1], 0, p.timeout_ns, abort_flag);
  // one outcome for the whole warp: the TMEM load below is a warp-wide instruction
  ok = __all_sync(0xffffffffu, ok && !*abort_flag);
  if (ok) {
    tc_fence_after();
    uint32_t r[32];
    tmem_ld_32x32b_x32(tmem_addr(tmem, 32 * warp, 32 * warp), r);
    tmem_ld_wait();
    if (warp < nvalid) {
      const int64_t idx = ((static_cast<int64_t>(slot) * p.Bsz + b) * p.K + k0 + warp) * p.G + g;
      uint4 *dst = reinterpret_cast<uint4 *>(p.cb + idx * 1024 + lane * 32);
#pragma unroll
      for (int i = 0; i < 4; ++i)
        dst[i] = make_uint4(pack2(r[8 * i], r[8 * i + 1]), pack2(r[8 * i + 2], r[8 * i + 3]),
                            pack2(r[8 * i + 4], r[8 * i + 5]), pack2(r[8 * i + 6], r[8 * i + 7]));
    }
  } else if (lane == 0) {
    atomicCAS(p.status, 0, kStatusTimeout);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, 128);
  }
}

// ------------------------------------------------------------------ main kernel
constexpr int kThreads = 512;

// shared memory map (bytes from a 1024-aligned base)
//   TMA ring: 144 KB, three 48 KB slots or five 28 KB slots per instance (the
//   tile offsets inside a slot are Lay's, below the mode enum): x tiles [32 t]
//   [64 p] bf16 (SW128), B_cf [32 s][n 0..63] then [32 s][n 64..127] (SW128), C
//   rows x n 0..63 and x n 64..127 (SW128), C B^T tiles [32 s][32 t] bf16
//   (SW64), 2 KB each; step j uses slot j mod (slots)
constexpr int kSlots = 3;
constexpr uint32_t kSlot = 12 * kTile;        // 48 KB per slot of the three-slot layout
constexpr uint32_t kOffXw = kSlots * kSlot;   // hi [32 t][64 p], lo [32 t][64 p] (bf16, SW128)
constexpr uint32_t kOffH = kOffXw + 2 * kTile;  // {hi, lo} x [128 n][64 p] bf16 (SW128)
constexpr uint32_t kOffMh = kOffH + 8 * kTile;  // 2 buffers x 4 dirs x [64 t'][32 s] interleaved
constexpr uint32_t kMhDir = 4096;               // one direction: [M^T | diag(remainder)]
constexpr uint32_t kMhBuf = 4 * kMhDir;
// per-step tables, a ring of kTab steps (slot j mod kTab)
constexpr int kTab = 8;
constexpr uint32_t kOffCum = kOffMh + 2 * kMhBuf;    // [kTab][4 dirs][32] f32: cumulative decay (log2)
constexpr uint32_t kOffDt = kOffCum + kTab * 512;    // [kTab][4][32] f32: dt
constexpr uint32_t kOffDtab = kOffDt + kTab * 512;  // [kTab][4] f32: D of the step's head
constexpr uint32_t kOffFtab = kOffDtab + kTab * 16;  // [kTab] s32: 1 + item parity at an item's first step,
                                                     // 0 at its other steps, -1 past the CTA's last step
constexpr uint32_t kOffBar = kOffFtab + 128;
constexpr int kNumBars = 56;
constexpr int kMaxSlots = 5;  // ring slots of the compact layout (see Lay)
constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;  // TMEM base, abort flag
constexpr int kItemRing = 16;
constexpr uint32_t kOffItemQ = kOffMisc + 64;             // int4[kItemRing]: published work items
constexpr uint32_t kSmemBytes = kOffItemQ + 16 * kItemRing + 1024;
static_assert(kSmemBytes <= 232448, "shared memory budget");

// intra-block operand of one direction (B of its Y_diag MMAs): [64 t'][32 s],
// interleaved MN-major (t' contiguous), t'-groups 128 B apart, s-groups 1024 B
// apart.  t' < 32: the masked-decay matrix M^T[s][t] with D on the diagonal
// (bf16); t' = 32 + s: that diagonal's bf16 remainder; zero elsewhere.  One
// N = 64 MMA per 16 tokens thus yields Y_diag in its first 32 columns and the
// remainder's X contribution in the next 32.
constexpr uint32_t kMhSbo = 128, kMhLbo = 1024;

enum : int {
  bFull0 = 0, bEmpty0 = bFull0 + kMaxSlots, bAux0 = bEmpty0 + kMaxSlots, bAux7 = bAux0 + kTab - 1, bXwFull0, bXwFull1, bSFull0,
  bSFull1,
  bSEmpty0, bSEmpty1, bMhFull0, bMhFull1, bHFull, bHCons, bYFull0, bYFull1, bYEmpty0, bYEmpty1, bDrain,
  bCbFull,
  bItem0, bCount = bItem0 + kItemRing
};
static_assert(bCount <= kNumBars, "barrier array");

// TMEM columns: S^T[2] (M=128 x 64), Y^T[2] = {Y_off^T (M=64 x 64), clean
// [Y_diag^T | remainder] (M=64 x 64), noisy [Y_diag^T | remainder] (M=64 x 64)}.
// With a gate the two directions of a stream are gated separately, so each
// direction keeps its own [Y_diag^T | remainder]: one Y buffer of
// {Y_off^T, clean fwd, noisy fwd, clean rev, noisy rev} (320 columns).
constexpr uint32_t kColS0 = 0, kColY0 = 128, kColYBuf = 192, kColRevGated = 128;
// C B^T accumulator of the fused-C B^T instance (M = 64 rows [s_cf; s_cr], N = 64
// columns [t_cf | t_cr]): the second staging buffer of the initial state, which
// a CTA that takes a single one-block item never uses
constexpr uint32_t kColCb = kColS0 + 64;
constexpr uint32_t kTmemCols = 512;

// Division of n (0 <= n < 2^31) by a divisor d fixed per launch (1 <= d < 2^31)
// as a multiply and a shift (round-up reciprocal): with s = ceil(log2 d) and
// m = ceil(2^(31+s) / d), floor(n m / 2^(31+s)) = floor(n / d) for every such
// n, because the error m d - 2^(31+s) is below d <= 2^s.  A work item's
// coordinates come from three such divisions; five integer divisions (a long
// dependent instruction sequence each) delayed the first load by about 0.6 us.
struct DivU {
  unsigned long long m;
  int sh;
  int pad;
};
inline DivU make_divu(int d) {
  int s = 0;
  while ((1ll << s) < d) ++s;
  const unsigned long long num = 1ull << (31 + s);
  return DivU{(num + static_cast<unsigned long long>(d) - 1) / static_cast<unsigned long long>(d), 31 + s, 0};
}
__device__ __forceinline__ int divu(int n, const DivU &v) {
  return static_cast<int>((static_cast<unsigned long long>(n) * v.m) >> v.sh);
}

struct TcParams {
  CUtensorMap tx[4];
  CUtensorMap tbcf;
  CUtensorMap tccf;
  CUtensorMap tcnf;
  CUtensorMap tcb;
  CUtensorMap tbcr, tccr;  // B and C of the clean reverse direction (kModeCbFused)
  const __nv_bfloat16 *dt[4];
  const float *A[4];
  const float *D[4];
  const __nv_bfloat16 *z[4];  // gate of each direction, or null
  int active[4];
  int gated;                   // some direction has a gate: single Y buffer, per-direction Y_diag
  int cbfused;                 // C B^T computed in the scan kernel (kModeCbFused)
  int Bsz, L, H, G, K;
  int nseg, seg_blocks;  // each (b, h) sequence is walked as nseg segments of seg_blocks blocks
  int items;             // Bsz * H * nseg work items, handed out one at a time
  DivU dv_nseg, dv_h, dv_hpg;  // division by nseg, H and H / G
  int *item_counter;     // next unclaimed work item (zeroed by the C B^T kernel)
  int need_s;            // the state after a block is used (outputs, next block); if not
                         // (one-block items, no state outputs), S, w o X and the state update are skipped
  int allblock;
  int out_bf16;
  const float *seg_init;  // [B][H][nseg][P][N] initial state of every segment (nseg > 1)
  float *seg_local;       // [B][H][nseg][P][N] aggregate kernel: end state from a zero start
  float *seg_decay;       // [B][H][nseg] aggregate kernel: total decay (log2 units)
  const float *h0;
  float *states;
  float *final_state;
  void *y_clean;
  void *y_noisy;
  int *status;
  unsigned long long timeout_ns;
  unsigned long long drain_ns;
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&v);
}
__device__ __forceinline__ float bf16_lo_f(uint32_t v) { return __uint_as_float(v << 16); }
// v * sigmoid(v) with the hardware exponential and divide
__device__ __forceinline__ float silu_approx(float v) { return __fdividef(v, 1.0f + ex2_approx(-v * 1.4426950408889634f)); }
__device__ __forceinline__ float bf16_hi_f(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// silu(z) of 16 gate values z[base + i stride] (1 where there is no gate).
// The 16 loads are issued before any of them is used, so that their latencies
// overlap (a load consumed at once would wait for it before the next is issued).
__device__ __forceinline__ void gates16(const __nv_bfloat16 *z, int64_t base, int64_t stride, float (&g)[16]) {
  if (!z) {
#pragma unroll
    for (int i = 0; i < 16; ++i) g[i] = 1.f;
    return;
  }
  const unsigned short *z16 = reinterpret_cast<const unsigned short *>(z) + base;
  unsigned short r[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) r[i] = z16[i * stride];
#pragma unroll
  for (int i = 0; i < 16; ++i) g[i] = silu_approx(__uint_as_float(static_cast<uint32_t>(r[i]) << 16));
}

// C B^T tile set of direction slot i in the workspace: the all-block pass keeps
// four (one per direction), prefix and block step two (the clean forward and
// reverse directions, slots 0 and 2).
__host__ __device__ __forceinline__ int cb_set(int allblock, int i) { return allblock ? i : (i >> 1); }
__host__ __device__ __forceinline__ int cb_sets(bool allblock) { return allblock ? 4 : 2; }

// Element i of a 4-entry kernel-parameter array without dynamic indexing (which
// would copy the array to local memory).
template <class T>
__device__ __forceinline__ T pick4(const T (&a)[4], int i) {
  return i == 0 ? a[0] : i == 1 ? a[1] : i == 2 ? a[2] : a[3];
}

__device__ __forceinline__ float lds_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ void sts_f32(uint32_t addr, float v) {
  asm volatile("st.shared.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}
__device__ __forceinline__ unsigned short lds_u16(uint32_t addr) {
  unsigned short v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ void sts_u16(uint32_t addr, unsigned short v) {
  asm volatile("st.shared.u16 [%0], %1;" ::"r"(addr), "h"(v) : "memory");
}
__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d)
               : "memory");
}
__device__ __forceinline__ void ld_shared_v4(uint32_t addr, uint32_t &a, uint32_t &b, uint32_t &c,
                                             uint32_t &d) {
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(a), "=r"(b), "=r"(c), "=r"(d)
               : "r"(addr)
               : "memory");
}
__device__ __forceinline__ void ld_shared_v4f(uint32_t addr, float (&v)[4]) {
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3])
               : "r"(addr)
               : "memory");
}

// v ~= hi + lo, both bf16; stores one 16-byte chunk of each.
__device__ __forceinline__ void store_split8(uint32_t addr_hi, uint32_t addr_lo, const float *v) {
  uint32_t hi[4], lo[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    hi[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
    lo[i] = pack_bf16x2(v[2 * i] - bf16_lo_f(hi[i]), v[2 * i + 1] - bf16_hi_f(hi[i]));
  }
  st_shared_v4(addr_hi, hi[0], hi[1], hi[2], hi[3]);
  st_shared_v4(addr_lo, lo[0], lo[1], lo[2], lo[3]);
}

// The CTA's barrier array and control block, by shared-memory address (one
// register each).  Control block: +0 TMEM base, +4 abort flag, +8 wait limit
// (ns, u64), +16 status word pointer (u64).
struct Ctl {
  uint32_t bar;   // barrier 0
  uint32_t misc;  // control block
};
__device__ __forceinline__ uint32_t bar_at(const Ctl &c, int i) { return c.bar + 8u * static_cast<uint32_t>(i); }

__device__ __forceinline__ uint64_t lds_u64(uint32_t addr) {
  uint64_t v;
  asm volatile("ld.shared.u64 %0, [%1];" : "=l"(v) : "r"(addr) : "memory");
  return v;
}

__device__ __noinline__ void raise_timeout_s(uint32_t misc) {
  asm volatile("st.volatile.shared.u32 [%0], %1;" ::"r"(misc + 4), "r"(1u) : "memory");
  atomicCAS(reinterpret_cast<int *>(lds_u64(misc + 16)), 0, kStatusTimeout);
}
__device__ __forceinline__ void raise_timeout(const Ctl &c) { raise_timeout_s(c.misc); }
__device__ __forceinline__ bool aborted(const Ctl &c) { return ld_volatile_shared_u32(c.misc + 4) != 0; }

// Bounded wait.  The first test is inline; the sleeping retry loop with its
// time limit and abort check is out of line, so that the many wait sites do
// not each carry it through the instruction cache.
__device__ __noinline__ bool bwait_slow(uint32_t b, uint32_t parity, uint32_t misc) {
  return mbar_wait_s(b, parity, lds_u64(misc + 8), misc + 4);
}
__device__ __forceinline__ bool bwait(const Ctl &c, int bar, uint32_t parity) {
  const uint32_t b = bar_at(c, bar);
  if (mbar_try_wait_s(b, parity)) return true;
  return bwait_slow(b, parity, c.misc);
}

__device__ __forceinline__ bool wait1(const Ctl &c, int bar, uint32_t parity) {
  if (bwait(c, bar, parity)) return true;
  raise_timeout(c);
  return false;
}

// Whole-warp bounded wait with a warp-uniform outcome.
__device__ __forceinline__ bool waitw(const Ctl &c, int bar, uint32_t parity) {
  bool ok = bwait(c, bar, parity);
  ok = __all_sync(0xffffffffu, ok);
  if (!ok && (threadIdx.x & 31) == 0) raise_timeout(c);
  __syncwarp();
  return ok;
}

__device__ __forceinline__ void arrive_lane0(const Ctl &c, int bar) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive_s(bar_at(c, bar));
}

// parity of the completion of a double-buffered barrier that block k uses
__device__ __forceinline__ uint32_t par2(int k) { return (static_cast<uint32_t>(k) >> 1) & 1u; }
// Y accumulators of step j: buffer, parity of its "full" phase, and the step
// whose read must precede this step's writes (double-buffered, or single-
// buffered with a gate)
__device__ __forceinline__ int ybuf(int gated, int j) { return gated ? 0 : (j & 1); }
__device__ __forceinline__ uint32_t ypar(int gated, int j) { return gated ? (static_cast<uint32_t>(j) & 1u) : par2(j); }
__device__ __forceinline__ int yprev(int gated, int j) { return gated ? j - 1 : j - 2; }
// TMA ring: slot and parity of block k


// ---------------------------------------------------------------- work items
// A work item is one (batch row b, head h, segment seg) sequence of nk blocks
// starting at block k0.  The CTAs claim items one at a time from a global
// counter (SMs that run faster take more), in order, so that the items in
// flight share their B, C tiles in L2.  The producer claims them, one item
// ahead of its own progress, and publishes them in a ring in shared memory;
// every role runs the same sequence of steps j = 0, 1, ... (one block of one
// item each); ring slots, double buffers and barrier phases follow j, so the
// pipeline runs on across item boundaries.
struct Item {
  int b, h, g, seg, k0, nk;
};

__device__ __forceinline__ Item item_unpack(const TcParams &p, int b, int h, int g, int seg) {
  Item r;
  r.b = b;
  r.h = h;
  r.g = g;
  r.seg = seg;
  r.k0 = seg * p.seg_blocks;
  r.nk = min(p.K - r.k0, p.seg_blocks);
  return r;
}

__device__ __forceinline__ Item item_at(const TcParams &p, int it) {
  Item r;
  const int bh = divu(it, p.dv_nseg);
  r.seg = it - bh * p.nseg;
  r.b = divu(bh, p.dv_h);
  r.h = bh - r.b * p.H;
  r.g = divu(r.h, p.dv_hpg);
  r.k0 = r.seg * p.seg_blocks;
  r.nk = min(p.K - r.k0, p.seg_blocks);
  return r;
}

// barrier ring of the per-step tables: phase parity of step j
__device__ __forceinline__ uint32_t part(int j) { return (static_cast<uint32_t>(j) / kTab) & 1u; }

// Kernel instances: the call's mode is a template parameter (bits kModeAll,
// kModeNeedS, kModeCbFused), so each instance carries only the code its mode
// runs.  (The aggregate pass of segmented plans is a kernel of its own.)
enum : int { kModeAll = 2, kModeNeedS = 4, kModeCbFused = 8 };

// Ring-slot layout of an instance.  The all-block pass and the fused-C B^T
// step keep three 48 KB slots (x of four directions, B_cf, the C tiles of two
// streams, four C B^T tiles; or B and C of both clean directions); the
// one-stream scan and step instances use five 28 KB slots in the same space
// (x of the two clean directions, B_cf, C_cf, two C B^T tiles), so that the
// producer runs further ahead of the masked-decay build, which waits for the
// tiles of the step two ahead.
template <int kM>
struct Lay {
  static constexpr bool kCompact = (kM & (kModeAll | kModeCbFused)) == 0;
  static constexpr int kN = kCompact ? 5 : 3;
  static constexpr uint32_t kBytes = kCompact ? 7 * kTile : 12 * kTile;
  static constexpr uint32_t kBcf = kCompact ? 2 * kTile : 4 * kTile;  // B_cf, n 0..63 then 64..127
  static constexpr uint32_t kClo = kCompact ? 4 * kTile : 6 * kTile;  // C rows x n 0..63
  static constexpr uint32_t kChi = kCompact ? 5 * kTile : 8 * kTile;  // C rows x n 64..127
  static constexpr uint32_t kCbBase = kCompact ? 6 * kTile : 10 * kTile;
  // x tile of direction slot i, C B^T tile of direction slot i
  __host__ __device__ static constexpr uint32_t x(int i) {
    return static_cast<uint32_t>(kCompact ? (i >> 1) : i) * kTile;
  }
  __host__ __device__ static constexpr uint32_t cb(int i) {
    return kCbBase + static_cast<uint32_t>(kCompact ? (i >> 1) : i) * 2048u;
  }
  __device__ static int slot(int j) { return j % kN; }
  __device__ static uint32_t par(int j) { return static_cast<uint32_t>(j / kN) & 1u; }
};
static_assert(5 * 7 * kTile <= kSlots * kSlot, "compact ring within the ring's space");
// kModeCbFused (one-block items without a state chain, no more items than
// SMs: the batch-1 denoising step): no C B^T pre-pass; each step loads B and C
// of both directions and computes its own C B^T tiles (one M = 64 MMA chain
// over [B_cf; B_cr] x [C_cf; C_cr]), so a layer's step is one launch.

__device__ __forceinline__ int lds_s32(uint32_t addr) {
  int v;
  asm volatile("ld.shared.s32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ void sts_s32(uint32_t addr, int v) {
  asm volatile("st.shared.s32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

__device__ __forceinline__ void wait_prior_grid() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// Fire-and-forget fetch of a line into this SM's L1 (the next block's gates:
// their loads then wait for L1, not for HBM).
__device__ __forceinline__ void prefetch_l1(const void *ptr) {
  asm volatile("prefetch.global.L1 [%0];" ::"l"(ptr));
}

// Claim the next work item (-1: none left).  With no more items than CTAs,
// CTA c takes item c and nothing else (no counter, no wait for the pre-pass);
// otherwise items come from the global counter the pre-pass zeroed.
__device__ __forceinline__ int claim_item(const TcParams &p, int nth, bool &waited) {
  if (p.items <= static_cast<int>(gridDim.x)) return nth == 0 ? static_cast<int>(blockIdx.x) : -1;
  if (!waited) {
    wait_prior_grid();
    waited = true;
  }
  const int it = atomicAdd(p.item_counter, 1);
  return it < p.items ? it : -1;
}
// Publish item `it` (-1: none) as this CTA's m-th, as its coordinates
// {b, h, g, seg} (the barrier arrival releases the write).
__device__ __forceinline__ void publish_item(const Ctl &c, uint32_t base, int m, int it, const Item &I) {
  const int e = m & (kItemRing - 1);
  const uint32_t a = base + kOffItemQ + 16 * e;
  if (it >= 0) {
    asm volatile("st.shared.v4.s32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(I.b), "r"(I.h), "r"(I.g), "r"(I.seg)
                 : "memory");
  } else {
    sts_s32(a, -1);
  }
  mbar_arrive_s(bar_at(c, bItem0 + e));
}
// Ring entry m (already published) as an item; false: none.
__device__ __forceinline__ bool item_read(const TcParams &p, uint32_t base, int m, Item &I) {
  const uint32_t a = base + kOffItemQ + 16 * (m & (kItemRing - 1));
  int b, h, g, seg;
  asm volatile("ld.shared.v4.s32 {%0, %1, %2, %3}, [%4];" : "=r"(b), "=r"(h), "=r"(g), "=r"(seg) : "r"(a) : "memory");
  if (b < 0) return false;
  I = item_unpack(p, b, h, g, seg);
  return true;
}
// This CTA's m-th item: 1 (in I), 0 (no more) or -1 (the wait timed out).
__device__ __forceinline__ int item_one(const TcParams &p, const Ctl &c, uint32_t base, int m, Item &I) {
  if (!wait1(c, bItem0 + (m & (kItemRing - 1)), static_cast<uint32_t>(m / kItemRing) & 1u)) return -1;
  return item_read(p, base, m, I) ? 1 : 0;
}
__device__ __forceinline__ int item_warp(const TcParams &p, const Ctl &c, uint32_t base, int m, Item &I) {
  if (!waitw(c, bItem0 + (m & (kItemRing - 1)), static_cast<uint32_t>(m / kItemRing) & 1u)) return -1;
  return item_read(p, base, m, I) ? 1 : 0;
}

// ---------------------------------------------------------------- producer
template <int kM>
__device__ void producer(const TcParams &p, const Ctl &c, uint32_t base) {
  constexpr bool kAll = kM & kModeAll, kCbF = kM & kModeCbFused;
  const int nact = p.active[0] + p.active[1] + p.active[2] + p.active[3];
  // x of each active direction, C B^T tiles, B of the clean forward direction
  // (only when S is formed), C of the clean (and noisy) forward direction;
  // with the C B^T tiles computed here: x of both directions, B and C of both
  const uint32_t bytes = kCbF ? 10 * kTile : nact * (kTile + 2048) + (2 + (kAll ? 4 : 2)) * kTile;
#pragma unroll
  for (int i = 0; i < 4; ++i)
    if (p.active[i]) tma_prefetch_desc(&p.tx[i]);
  tma_prefetch_desc(&p.tbcf);
  tma_prefetch_desc(&p.tccf);
  if (kAll) tma_prefetch_desc(&p.tcnf);
  if (kCbF) {
    tma_prefetch_desc(&p.tbcr);
    tma_prefetch_desc(&p.tccr);
  } else {
    tma_prefetch_desc(&p.tcb);
  }
  using Ly = Lay<kM>;
  int last[Ly::kN];
#pragma unroll
  for (int s = 0; s < Ly::kN; ++s) last[s] = -1;
  int j = 0;
  bool ok = true;
  // items m and m + 1 are published when item m starts (nothing after a -1);
  // claiming further ahead would hold items back from CTAs that run dry at
  // the end of the pass
  bool waited = kCbF;  // past the wait for the preceding grid (done by every thread in that instance)
  int nclaim = 0;
  // each claimed item is decomposed once, when it is published
  int cur = claim_item(p, nclaim++, waited), nxt = -1;
  Item Icur{}, Inxt{};
  if (cur >= 0) Icur = item_at(p, cur);
  publish_item(c, base, 0, cur, Icur);
  if (cur >= 0) {
    nxt = claim_item(p, nclaim++, waited);
    if (nxt >= 0) Inxt = item_at(p, nxt);
    publish_item(c, base, 1, nxt, Inxt);
  }
  for (int m = 0; ok && cur >= 0; ++m) {
    const Item I = Icur;
    for (int kk = 0; kk < I.nk; ++kk, ++j) {
      const int k = I.k0 + kk;  // block index in the sequence
      const int r = Ly::slot(j);
      if (!wait1(c, bEmpty0 + r, Ly::par(j) ^ 1)) {
        ok = false;
        break;
      }
      const uint32_t full = bar_at(c, bFull0 + r);
      mbar_arrive_expect_tx_s(full, bytes);
      const uint32_t st = base + r * Ly::kBytes;
      const int t0 = k * kT;
      if constexpr (kCbF) {
        // x_cf, x_cr; [B_cf; B_cr] as the A operand of C B^T (n 0..63 at kBcf,
        // n 64..127 at kCbBase, 64 rows each); [C_cf; C_cr] at kClo / kChi
        tma_load_4d_s(st + Ly::x(kCF), &p.tx[kCF], full, 0, I.h, t0, I.b);
        tma_load_4d_s(st + Ly::x(kCR), &p.tx[kCR], full, 0, I.h, t0, I.b);
        tma_load_4d_s(st + Ly::kBcf, &p.tbcf, full, 0, I.g, t0, I.b);
        tma_load_4d_s(st + Ly::kBcf + kTile, &p.tbcr, full, 0, I.g, t0, I.b);
        tma_load_4d_s(st + Ly::kCbBase, &p.tbcf, full, 64, I.g, t0, I.b);
        tma_load_4d_s(st + Ly::kCbBase + kTile, &p.tbcr, full, 64, I.g, t0, I.b);
        tma_load_4d_s(st + Ly::kClo, &p.tccf, full, 0, I.g, t0, I.b);
        tma_load_4d_s(st + Ly::kClo + kTile, &p.tccr, full, 0, I.g, t0, I.b);
        tma_load_4d_s(st + Ly::kChi, &p.tccf, full, 64, I.g, t0, I.b);
        tma_load_4d_s(st + Ly::kChi + kTile, &p.tccr, full, 64, I.g, t0, I.b);
      } else {
#pragma unroll
        for (int i = 0; i < 4; ++i)
          if (p.active[i]) tma_load_4d_s(st + Ly::x(i), &p.tx[i], full, 0, I.h, t0, I.b);
        tma_load_4d_s(st + Ly::kBcf, &p.tbcf, full, 0, I.g, t0, I.b);
        tma_load_4d_s(st + Ly::kBcf + kTile, &p.tbcf, full, 64, I.g, t0, I.b);
        tma_load_4d_s(st + Ly::kClo, &p.tccf, full, 0, I.g, t0, I.b);
        tma_load_4d_s(st + Ly::kChi, &p.tccf, full, 64, I.g, t0, I.b);
        if (kAll) {
          tma_load_4d_s(st + Ly::kClo + kTile, &p.tcnf, full, 0, I.g, t0, I.b);
          tma_load_4d_s(st + Ly::kChi + kTile, &p.tcnf, full, 64, I.g, t0, I.b);
        }
        // C B^T tiles: written by the pre-pass this kernel may overlap
        if (!waited) {
          wait_prior_grid();
          waited = true;
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          if (!p.active[i]) continue;
          const int idx = ((cb_set(kAll, i) * p.Bsz + I.b) * p.K + k) * p.G + I.g;
          tma_load_3d_s(st + Ly::cb(i), &p.tcb, full, 0, 0, idx);
        }
      }
#pragma unroll
      for (int s = 0; s < Ly::kN; ++s)
        if (s == r) last[s] = j;
    }
    cur = nxt;
    Icur = Inxt;
    nxt = -1;
    if (ok && cur >= 0) {
      nxt = claim_item(p, nclaim++, waited);
      if (nxt >= 0) Inxt = item_at(p, nxt);
      publish_item(c, base, m + 2, nxt, Inxt);
    }
  }
  // no copy into this CTA's shared memory may still be in flight at exit
#pragma unroll
  for (int s = 0; s < Ly::kN; ++s)
    if (last[s] >= 0) (void)mbar_wait_s(bar_at(c, bFull0 + s), Ly::par(last[s]), p.drain_ns, 0);
}

// ---------------------------------------------------------------- MMA issuer
// Issue order per step: S; Y_off (then commit "h consumed" so the state group
// may overwrite the h operand at once); Y_diag and the D x products.
// Descriptors are built once; per step only their start addresses move.
template <int kM, bool kGated>
__device__ void mma_issuer(const TcParams &p, const Ctl &c, uint32_t base, uint32_t tmem) {
  constexpr bool kAll = kM & kModeAll, kNeedS = kM & kModeNeedS, kCbF = kM & kModeCbFused;
  const uint32_t id_s = idesc_bf16(128, 64, 1, 1);  // S^T[n][p] = B^T (w o X)
  // Y_off^T[p][t] = h C^T over the stacked [C_cf; C_nf] rows (only C_cf without a noisy stream)
  const uint32_t id_yo = kAll ? idesc_bf16(64, 64, 1, 0) : idesc_bf16(64, 32, 1, 0);
  const uint32_t id_yd = idesc_bf16(64, 64, 1, 1);  // [Y_diag^T | remainder][p][t'] = X^T [M^T | diag]
  // descriptor of each operand at its first tile; moving an operand by b bytes adds b >> 4
  using Ly = Lay<kM>;
  const D64 dBcf = split64(sdesc(base + Ly::kBcf, kTile, 1024, kLayoutSw128));
  const D64 dXw = split64(sdesc(base + kOffXw, 0, 1024, kLayoutSw128));
  const D64 dH = split64(sdesc(base + kOffH, 0, 1024, kLayoutSw128));
  const D64 dC = split64(sdesc(base + Ly::kClo, 16, 1024, kLayoutSw128));
  const D64 dX = split64(sdesc(base + Ly::x(0), 0, 1024, kLayoutSw128));
  const D64 dM = split64(sdesc(base + kOffMh, kMhLbo, kMhSbo, kLayoutNone));
  // fused C B^T: [B_cf; B_cr] K-major (64 rows s; n 0..63 at kBcf, 64..127 at kCbBase)
  const D64 dBk = split64(sdesc(base + Ly::kBcf, 16, 1024, kLayoutSw128));
  const uint32_t id_cb = idesc_bf16(64, 64, 0, 0);
#define BD_OFF(bytes) (static_cast<uint32_t>((bytes) >> 4))
  int j = 0;
  bool ok = true;
  for (int m = 0; ok; ++m) {
    Item I;
    if (item_one(p, c, base, m, I) <= 0) break;
    const int nk = I.nk;
    for (int kk = 0; kk < nk; ++kk, ++j) {
      ok = false;
      const int r = Ly::slot(j), i2 = j & 1;
      const uint32_t so = BD_OFF(static_cast<uint32_t>(r) * Ly::kBytes);  // this step's ring slot
      if (!wait1(c, bFull0 + r, Ly::par(j))) break;
      if constexpr (kCbF) {
        // ---- [C B^T]: rows s of [B_cf; B_cr] against columns t of [C_cf; C_cr];
        //      the two diagonal 32 x 32 blocks are the directions' tiles.  The
        //      accumulator is free: its previous reader arrived on MhFull of the
        //      previous step, which this warp waited for before that step's Y_diag.
        tc_fence_after();
#pragma unroll 1
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t ko = BD_OFF((ks & 3) * 32);
          umma_bf16(tmem + kColCb, dBk + so + ko + (ks < 4 ? 0u : BD_OFF(Ly::kCbBase - Ly::kBcf)),
                    dC + so + ko + (ks < 4 ? 0u : BD_OFF(Ly::kChi - Ly::kClo)), id_cb, ks > 0);
        }
        umma_commit_s(bar_at(c, bCbFull));
      }
      // ---- S^T = B_cf^T (w o X): A MN-major (n; halves 4 KB apart), B MN-major (p)
      if (kNeedS) {
        if (!wait1(c, bXwFull0 + i2, par2(j))) break;
        if (j >= 2 && !wait1(c, bSEmpty0 + i2, par2(j - 2))) break;
        tc_fence_after();
        const uint32_t colS = tmem + kColS0 + 64 * i2;
        const D64 dxw = dXw;
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) {
          umma_bf16(colS, dBcf + so + BD_OFF(ks * 2048), dxw + BD_OFF(ks * 2048), id_s, ks > 0);
          umma_bf16(colS, dBcf + so + BD_OFF(ks * 2048), dxw + BD_OFF(kTile + ks * 2048), id_s, 1);
        }
        umma_commit_s(bar_at(c, bSFull0 + i2));
      }
      // ---- Y_off^T = h [C_cf; C_nf]^T, h = the state before this block
      if (!wait1(c, bHFull, j & 1)) break;
      const int yb = ybuf(kGated, j), jp = yprev(kGated, j);
      // Double-buffered Y with the masked-decay operands built two steps ahead
      // (ungated, C B^T from the pre-pass): each epilogue warp frees Y of step
      // j - 2 before it builds the operands of step j, so their completion
      // implies the buffer is free -- one wait instead of two.
      constexpr bool kMhFirst = !kGated && !kCbF;
      if constexpr (kMhFirst) {
        if (!wait1(c, bMhFull0 + i2, par2(j))) break;
      } else {
        if (jp >= 0 && !wait1(c, bYEmpty0 + yb, ypar(kGated, jp))) break;
      }
      tc_fence_after();
      const uint32_t colY = tmem + kColY0 + kColYBuf * yb;
#pragma unroll 1
      for (int ks = 0; ks < 8; ++ks) {
        const D64 bc = dC + so + BD_OFF((ks < 4 ? 0u : Ly::kChi - Ly::kClo) + (ks & 3) * 32);
        umma_bf16(colY, dH + BD_OFF(ks * 2048), bc, id_yo, ks > 0);
        umma_bf16(colY, dH + BD_OFF(4 * kTile + ks * 2048), bc, id_yo, 1);
      }
      umma_commit_s(bar_at(c, bHCons));  // the h operand may now be overwritten
      // ---- Y_diag^T of each stream = X_fwd^T M_fwd^T + X_rev^T M_rev^T (M
      //      with D on its diagonal), and in the next 32 columns the same
      //      products with the diagonal's bf16 remainders
      if (!kMhFirst && !wait1(c, bMhFull0 + i2, par2(j))) break;
      tc_fence_after();
      const uint32_t mo = BD_OFF(static_cast<uint32_t>(i2) * kMhBuf);
#pragma unroll
      for (int i = 0; i < 4; ++i) {  // the forward direction of a stream (i < 2) is always active
        if (!p.active[i]) continue;
        // ungated: a stream's directions share one accumulator; gated: each its own
        const bool own = kGated && i >= 2;
        const uint32_t col = colY + 64 + ((i & 1) ? 64 : 0) + (own ? kColRevGated : 0);
#pragma unroll
        for (int ks = 0; ks < 2; ++ks)
          umma_bf16(col, dX + so + BD_OFF(Ly::x(i) + ks * 2048), dM + mo + BD_OFF(i * kMhDir + ks * 2048), id_yd,
                    ((i >= 2 && !own) || ks > 0) ? 1u : 0u);
      }
      umma_commit_s(bar_at(c, bYFull0 + yb));
      umma_commit_s(bar_at(c, bEmpty0 + r));
      ok = true;
    }
  }
#undef BD_OFF
  umma_commit_s(bar_at(c, bDrain));
  (void)mbar_wait_s(bar_at(c, bDrain), 0, p.drain_ns, 0);
}

// The intra-block operand of direction slot q for step jm (see kMhSbo): the
// masked-decay matrix M^T[s][t] of the block with the direction's D added to
// its diagonal, stored bf16, and that diagonal's bf16 remainders; one warp,
// row s = lane.  Reads the step's C B^T tile (ring slot) and decay tables.
__device__ __forceinline__ void build_masked_decay(uint32_t base, uint32_t cbrow, int q, int lane, int jm, bool act,
                                                   bool rev) {
  const int ct = jm % kTab;
  if (act) {
    const uint32_t cq = base + kOffCum + (ct * 4 + q) * 128;
    const float cs = lds_f32(cq + lane * 4);
    const float ds = lds_f32(base + kOffDt + (ct * 4 + q) * 128 + lane * 4);
    const uint32_t mrow = base + kOffMh + (jm & 1) * kMhBuf + q * kMhDir;
    // this direction's D joins the diagonal of M (D x is part of X^T M^T):
    // M[s][s] + D is stored as bf16 hi in M and its bf16 remainder lo on the
    // diagonal of the block's 16 x 16 correction tile of chunk s / 16
    const float Dq = lds_f32(base + kOffDtab + (ct * 4 + q) * 4);
    // off the diagonal in the loop (no divergent branch), the diagonal below
#pragma unroll 1
    for (int jj = 0; jj < 4; ++jj) {
      uint32_t r[4];
      ld_shared_v4(cbrow + sw64_chunk(lane, jj), r[0], r[1], r[2], r[3]);  // C B^T[s = lane][8 jj ..]
      float cj[8];
      ld_shared_v4f(cq + 32 * jj, *reinterpret_cast<float(*)[4]>(&cj[0]));
      ld_shared_v4f(cq + 32 * jj + 16, *reinterpret_cast<float(*)[4]>(&cj[4]));
      float mv[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int t = 8 * jj + i;
        const bool valid = rev ? (t <= lane) : (t >= lane);
        const float e = ex2_approx(cj[i] - cs);
        const float cb = (i & 1) ? bf16_hi_f(r[i >> 1]) : bf16_lo_f(r[i >> 1]);
        mv[i] = valid ? cb * ds * e : 0.f;
      }
      st_shared_v4(mrow + inter_mn_off(8 * jj, lane, kMhSbo, kMhLbo), pack_bf16x2(mv[0], mv[1]),
                   pack_bf16x2(mv[2], mv[3]), pack_bf16x2(mv[4], mv[5]), pack_bf16x2(mv[6], mv[7]));
    }
    {
      // M[s][s] + D (the decay factor is exactly 1 there) as bf16, its remainder
      // on the diagonal of the correction half
      const float cb = __uint_as_float(static_cast<uint32_t>(lds_u16(cbrow + sw64_chunk(lane, lane >> 3) +
                                                                     2u * static_cast<uint32_t>(lane & 7)))
                                       << 16);
      const float v = cb * ds + Dq;
      const __nv_bfloat16 hi = __float2bfloat16_rn(v);
      sts_u16(mrow + inter_mn_off(lane, lane, kMhSbo, kMhLbo), __bfloat16_as_ushort(hi));
      sts_u16(mrow + inter_mn_off(32 + lane, lane, kMhSbo, kMhLbo),
              __bfloat16_as_ushort(__float2bfloat16_rn(v - __bfloat162float(hi))));
    }
  }
}

// The same matrices split over the four epilogue warps for one-block items
// of one stream (fused-C B^T and pre-pass step instances): warp q builds rows s = 16 (q & 1) + (lane & 15) of direction slot
// kCF (q < 2) or kCR (q >= 2); lanes 0..15 the columns t = 0..15, lanes 16..31
// t = 16..31.  cbv holds C B^T[s][t] of the thread's 16 columns.
__device__ __forceinline__ void build_rows16(uint32_t base, int q, int lane, int jm, const float (&cbv)[16]) {
  const int ct = jm % kTab;
  const bool rev = q >= 2;
  const int dq = rev ? kCR : kCF;
  const int s = 16 * (q & 1) + (lane & 15);
  const int th = lane & 16;
  const uint32_t cq = base + kOffCum + (ct * 4 + dq) * 128;
  const float cs = lds_f32(cq + s * 4);
  const float ds = lds_f32(base + kOffDt + (ct * 4 + dq) * 128 + s * 4);
  const float Dq = lds_f32(base + kOffDtab + (ct * 4 + dq) * 4);
  const uint32_t mrow = base + kOffMh + (jm & 1) * kMhBuf + dq * kMhDir;
  float cj[16];
#pragma unroll
  for (int u = 0; u < 4; ++u) ld_shared_v4f(cq + th * 4 + 16 * u, *reinterpret_cast<float(*)[4]>(&cj[4 * u]));
  // M^T[s][t] = C B^T[s][t] dt_s exp(cum_t - cum_s) inside the direction's
  // causal half, and M[s][s] + D on the diagonal (the decay factor is 1 there)
  float mv[16], dv = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int t = th + i;
    const float cb = cbv[i] * ds;
    const bool valid = rev ? (t <= s) : (t >= s);
    float v = cb * ex2_approx(cj[i] - cs);
    if (t == s) {
      v = cb + Dq;
      dv = v;
    }
    mv[i] = valid ? v : 0.f;
  }
#pragma unroll
  for (int h2 = 0; h2 < 2; ++h2)
    st_shared_v4(mrow + inter_mn_off(th + 8 * h2, s, kMhSbo, kMhLbo), pack_bf16x2(mv[8 * h2], mv[8 * h2 + 1]),
                 pack_bf16x2(mv[8 * h2 + 2], mv[8 * h2 + 3]), pack_bf16x2(mv[8 * h2 + 4], mv[8 * h2 + 5]),
                 pack_bf16x2(mv[8 * h2 + 6], mv[8 * h2 + 7]));
  // the diagonal's bf16 remainder, from the lane whose columns hold t = s
  if ((lane >> 4) == (q & 1))
    sts_u16(mrow + inter_mn_off(32 + s, s, kMhSbo, kMhLbo),
            __bfloat16_as_ushort(__float2bfloat16_rn(dv - __bfloat162float(__float2bfloat16_rn(dv)))));
}

// From the step's bf16 C B^T tile in its ring slot (pre-pass instances).
__device__ __forceinline__ void build_masked_decay_split(uint32_t base, uint32_t cbrow, int q, int lane, int jm) {
  const int s = 16 * (q & 1) + (lane & 15);
  const int th = lane & 16;
  uint32_t r[8];
  ld_shared_v4(cbrow + sw64_chunk(s, th >> 3), r[0], r[1], r[2], r[3]);
  ld_shared_v4(cbrow + sw64_chunk(s, (th >> 3) + 1), r[4], r[5], r[6], r[7]);
  float cbv[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) cbv[i] = (i & 1) ? bf16_hi_f(r[i >> 1]) : bf16_lo_f(r[i >> 1]);
  build_rows16(base, q, lane, jm, cbv);
}

// From the fp32 C B^T accumulator in TMEM (fused-C B^T instance; M = 64
// layout: rows 16 q' .. 16 q' + 15 in TMEM lanes 32 q' .. 32 q' + 15, so warp q
// reads exactly its rows).  Warp-wide: every lane of every epilogue warp calls it.
__device__ __forceinline__ void build_masked_decay_tm(uint32_t base, uint32_t tmem, int q, int lane, int jm) {
  uint32_t r[16];
  tmem_ld_16x32bx2_x16i<16>(tmem_addr(tmem, 32 * q, kColCb + (q >= 2 ? 32 : 0)), r);
  tmem_ld_wait();
  float cbv[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) cbv[i] = __uint_as_float(r[i]);
  build_rows16(base, q, lane, jm, cbv);
}

// ---------------------------------------------------------------- operand group
// warps 2, 3, 6, 7 (direction slots q = 0..3, whose decays each computes).
// Per step: the per-step tables (cumulative decays, dt, exp(cum) of the
// forward directions, D of the step's head, item-start flag) and w o X.
// The masked-decay matrices are built by the epilogue warps.
template <int kM>
__device__ void operand_group(const TcParams &p, const Ctl &c, uint32_t base) {
  constexpr bool kNeedS = kM & kModeNeedS;
  const int lane = threadIdx.x & 31;
  const int wq = threadIdx.x >> 5;
  const int q = wq < 4 ? wq - 2 : wq - 4;
  const int gt = q * 32 + (threadIdx.x & 31);  // 0..127
  const bool act = pick4(p.active, q) != 0;
  const uint32_t cum = base + kOffCum, dts = base + kOffDt;
  const int64_t H = p.H, L = p.L;
  const bool rev = q >= 2;
  const float *Ap = pick4(p.A, q);
  const __nv_bfloat16 *dtp = pick4(p.dt, q);
  // D of direction gt >> 4 (one writer per direction into the D table)
  const float *Dp = gt < 64 ? pick4(p.D, gt >> 4) : nullptr;
  const bool dact = gt < 64 && (gt & 15) == 0 && pick4(p.active, gt >> 4) != 0;
  // A failed (timed-out) wait ends the group at once.
  Item I;
  if (item_warp(p, c, base, 0, I) <= 0) return;
  // Global loads two steps ahead (their latency is microseconds under the
  // kernel's own traffic): a cursor walks the steps, through the items the
  // producer publishes, and fills a two-deep register queue with dt of this
  // lane's token, A (log2 units) and D of the step's head.
  int cm = 0, ckk = 0;
  bool cv = true;  // the cursor is on an item
  Item CI = I;
  // (kept as loaded -- dt as its bf16 bits -- and converted at use: an
  // arithmetic use here would wait for the load)
  uint32_t qdt[2];
  float qa[2], qd[2];
  auto cursor_load = [&](int e) {
    qdt[e] = 0u;
    qa[e] = 0.f;
    qd[e] = 0.f;
    if (!cv) return;
    if (act) {
      qdt[e] = reinterpret_cast<const unsigned short *>(
          dtp)[(static_cast<int64_t>(CI.b) * L + (CI.k0 + ckk) * kT + lane) * H + CI.h];
      qa[e] = Ap[CI.h];
    }
    if (dact) qd[e] = Dp[CI.h];
  };
  auto cursor_next = [&]() -> bool {  // false: a wait timed out
    if (!cv) return true;
    if (++ckk < CI.nk) return true;
    ++cm;
    ckk = 0;
    const int r = item_warp(p, c, base, cm, CI);
    if (r < 0) return false;
    cv = r > 0;
    return true;
  };
  cursor_load(0);
  if (!cursor_next()) return;
  cursor_load(1);
  if (!cursor_next()) return;
  int j = 0;
  for (int m = 0;; ++m) {
    bool has_next = false;
    Item In = I;
    for (int kk = 0; kk < I.nk; ++kk, ++j) {
      const int ct = j % kTab;
      const uint32_t st = base + Lay<kM>::slot(j) * Lay<kM>::kBytes;
      const float dt_cur = __uint_as_float(qdt[0] << 16), A2 = qa[0] * kLog2e, Dv = qd[0];
      qdt[0] = qdt[1];
      qa[0] = qa[1];
      qd[0] = qd[1];
      cursor_load(1);
      if (!cursor_next()) return;
      if (kk + 1 == I.nk) {  // the next item
        const int r = item_warp(p, c, base, m + 1, In);
        if (r < 0) return;
        has_next = r > 0;
      }
      // ---- decays of this warp's direction (log2 units): prefix sum over
      //      the block; the reverse direction's suffix sum is total - prefix + own
      const float v0 = dt_cur * A2;
      if (act) {
        float v = v0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const float u = __shfl_up_sync(0xffffffffu, v, o);
          if (lane >= o) v += u;
        }
        if (rev) v = __shfl_sync(0xffffffffu, v, 31) - v + v0;
        sts_f32(cum + ((ct * 4 + q) * 32 + lane) * 4, v);
        sts_f32(dts + ((ct * 4 + q) * 32 + lane) * 4, dt_cur);
      }
      if (dact) sts_f32(base + kOffDtab + (ct * 4 + (gt >> 4)) * 4, Dv);
      if (gt == 0) sts_s32(base + kOffFtab + ct * 4, kk == 0 ? 1 + (m & 1) : 0);
      arrive_lane0(c, bAux0 + ct);
      if (!waitw(c, bAux0 + ct, part(j))) return;
      if (!waitw(c, bFull0 + Lay<kM>::slot(j), Lay<kM>::par(j))) return;
      // ---- (w o X) of the clean forward direction, bf16 hi + lo
      if (kNeedS) {
        const uint32_t xw = base + kOffXw;
        // the S MMA of the previous step has read the w o X buffer
        if (j >= 1 && !waitw(c, bSFull0 + ((j - 1) & 1), par2(j - 1))) return;
        const uint32_t cf = cum + (ct * 4 + kCF) * 128, df = dts + (ct * 4 + kCF) * 128;
        const float c31 = lds_f32(cf + 31 * 4);
#pragma unroll
        for (int rep = 0; rep < 2; ++rep) {
          const int i = gt + 128 * rep;
          const int t = i >> 3, ch = i & 7;
          const uint32_t off = sw128_chunk(t, ch);
          uint32_t r0, r1, r2, r3;
          ld_shared_v4(st + Lay<kM>::x(kCF) + off, r0, r1, r2, r3);
          const float w = lds_f32(df + t * 4) * ex2_approx(c31 - lds_f32(cf + t * 4));
          float vv[8] = {bf16_lo_f(r0) * w, bf16_hi_f(r0) * w, bf16_lo_f(r1) * w, bf16_hi_f(r1) * w,
                         bf16_lo_f(r2) * w, bf16_hi_f(r2) * w, bf16_lo_f(r3) * w, bf16_hi_f(r3) * w};
          store_split8(xw + off, xw + kTile + off, vv);
        }
        fence_proxy_async_smem();
        arrive_lane0(c, bXwFull0 + (j & 1));
      }
      arrive_lane0(c, bEmpty0 + Lay<kM>::slot(j));
    }
    if (!has_next) break;
    I = In;
  }
  // past the last step: tell the epilogue's look-ahead that there is no more
  const int ct = j % kTab;
  if (gt == 0) sts_s32(base + kOffFtab + ct * 4, -1);
  arrive_lane0(c, bAux0 + ct);
}

// ---------------------------------------------------------------- state group
// One-block items whose state after the block is not used (no S chain): the
// group only turns each item's initial state into the h operand of Y_off.
// The fp32 state of item m + 1 is loaded while item m is converted, staged in
// TMEM (the unused S accumulator columns, two buffers of 64 columns: lane n,
// column p), so that the load latency overlaps the pipeline instead of
// adding to every item.
__device__ void state_group_staged(const TcParams &p, const Ctl &c, uint32_t base, uint32_t tmem) {
  const int lane = threadIdx.x & 31;
  const int q = (threadIdx.x >> 5) & 3;
  const int n = 32 * q + lane;
  const int64_t H = p.H;
  const int64_t PN = kP * kN;
  float hreg[kP];
  auto load_h = [&](const Item &I) {
    const float *src = p.h0 ? p.h0 + (static_cast<int64_t>(I.b) * H + I.h) * PN + n : nullptr;
#pragma unroll
    for (int pp = 0; pp < kP; ++pp) hreg[pp] = src ? src[pp * kN] : 0.f;
  };
  auto stage = [&](int e) {  // hreg -> TMEM buffer e
    const uint32_t ta = tmem_addr(tmem, 32 * q, kColS0 + 64 * e);
#pragma unroll
    for (int cq = 0; cq < 4; ++cq) {
      uint32_t r[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) r[i] = __float_as_uint(hreg[16 * cq + i]);
      tmem_st_32x32b_x16(ta + 16 * cq, r);
    }
    tmem_st_wait();
  };
  // h operand rows of this thread: row n, the eight 16-byte chunks of its 64 p
  // in the 128-byte swizzle (row address made opaque so that the chunk
  // addresses are formed at the stores)
  auto h_row = [&]() {
    uint32_t row = base + kOffH + 128u * static_cast<uint32_t>(n);
    asm volatile("" : "+r"(row));
    return row;
  };
  Item I;
  if (item_warp(p, c, base, 0, I) <= 0) return;
  load_h(I);
  if (p.items <= static_cast<int>(gridDim.x)) {
    // a single item per CTA: the state goes straight from registers to the operand
    const uint32_t row = h_row(), sw = (row >> 7) & 7u;
#pragma unroll
    for (int cc = 0; cc < 8; ++cc) {
      const uint32_t a = row + ((static_cast<uint32_t>(cc) ^ sw) << 4);
      store_split8(a, a + 4 * kTile, hreg + 8 * cc);
    }
    fence_proxy_async_smem();
    arrive_lane0(c, bHFull);
    return;
  }
  // The loads of item m + 2 are issued as soon as item m + 1 is staged, so
  // they are in flight through a whole item (the h operand hand-over of item
  // m + 1 included) before item m + 2 is staged.
  stage(0);
  for (int m = 0;; ++m) {
    const int rn = item_warp(p, c, base, m + 1, I);
    if (rn < 0) return;
    if (rn > 0) load_h(I);  // in flight while item m is converted
    // Y_off of the previous item has read the h operand
    if (m >= 1 && !waitw(c, bHCons, (m - 1) & 1)) return;
    {
      const uint32_t row = h_row(), sw = (row >> 7) & 7u;
      const uint32_t ta = tmem_addr(tmem, 32 * q, kColS0 + 64 * (m & 1));
#pragma unroll
      for (int cq = 0; cq < 4; ++cq) {
        uint32_t r[16];
        tmem_ld_32x32b_x16(ta + 16 * cq, r);
        tmem_ld_wait();
        float v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          const uint32_t a = row + ((static_cast<uint32_t>(2 * cq + h2) ^ sw) << 4);
          store_split8(a, a + 4 * kTile, v + 8 * h2);
        }
      }
    }
    fence_proxy_async_smem();
    arrive_lane0(c, bHFull);
    if (rn == 0) return;
    stage((m + 1) & 1);
  }
}

// warps 8..11: thread owns column n = 32 q + lane of the state, h^T[n][0..63].
// A failed (timed-out) wait ends the group at once: nothing else is stored.
template <int kM>
__device__ void state_group(const TcParams &p, const Ctl &c, uint32_t base, uint32_t tmem) {
  constexpr bool kNeedS = kM & kModeNeedS;
  const int lane = threadIdx.x & 31;
  const int q = (threadIdx.x >> 5) & 3;
  const int n = 32 * q + lane;
  const uint32_t cum = base + kOffCum;
  if constexpr (!kNeedS) {
    state_group_staged(p, c, base, tmem);
    return;
  }
  const int64_t H = p.H;
  const int64_t PN = kP * kN;
  float hreg[kP];
  // h operand of Y_off^T (A, MN-major): {hi, lo} x [128 n rows][64 p] (SW128)
  auto write_h = [&]() {
    // (row address made opaque so that the eight chunk addresses are formed
    // here rather than held in registers across the block loop)
    uint32_t row = base + kOffH + 128u * static_cast<uint32_t>(n);
    asm volatile("" : "+r"(row));
    const uint32_t sw = (row >> 7) & 7u;
#pragma unroll
    for (int cc = 0; cc < 8; ++cc) {
      const uint32_t a = row + ((static_cast<uint32_t>(cc) ^ sw) << 4);
      store_split8(a, a + 4 * kTile, hreg + 8 * cc);
    }
    fence_proxy_async_smem();
    arrive_lane0(c, bHFull);
  };
  // Each item: load its initial state, then per block kk: write the h
  // operand of the state entering the block, store the state after block
  // kk - 1, and advance the state with S of block kk; a last pass (kk == nk)
  // stores the state after the item's last block (boundary, final or segment
  // state).  Each store sequence and the operand write appear once in code.
  int j = 0;
  for (int m = 0;; ++m) {
    int nk;
    float *sdst;  // boundary states of this item's blocks, [B][K][H][P][N]
    {
      Item I;
      if (item_warp(p, c, base, m, I) <= 0) return;
      nk = I.nk;
      const int64_t bh = static_cast<int64_t>(I.b) * H + I.h;
      sdst = p.states ? p.states + ((static_cast<int64_t>(I.b) * p.K + I.k0) * H + I.h) * PN + n : nullptr;
      // initial state of this item: h0 (first segment) or the chained state
      // the aggregate and combine kernels left in the workspace (later segments)
      const float *src = I.seg == 0 ? (p.h0 ? p.h0 + bh * PN + n : nullptr)
                                    : p.seg_init + (bh * p.nseg + I.seg) * PN + n;
      if (src && I.seg > 0) wait_prior_grid();  // segment states: written by the combine kernel
#pragma unroll
      for (int pp = 0; pp < kP; ++pp) hreg[pp] = src ? src[pp * kN] : 0.f;
    }
    for (int kk = 0;; ++kk) {
      if (kk < nk) {
        // Y_off of the previous step has read the h operand; the state
        // entering this block replaces it
        if (j >= 1 && !waitw(c, bHCons, (j - 1) & 1)) return;
        write_h();
      }
      if (kk >= 1) {
#pragma unroll 1
        for (int d = 0; d < 2; ++d) {
          float *dst = sdst;
          if (d == 1) {  // after the item's last block: the final state
            dst = nullptr;
            if (kk == nk && !aborted(c)) {
              Item E;  // (re-read from the ring: its entry is not reused before every role moved on)
              (void)item_read(p, base, m, E);
              const int64_t ebh = static_cast<int64_t>(E.b) * H + E.h;
              if (p.final_state && E.k0 + E.nk == p.K) dst = p.final_state + ebh * PN + n;
            }
          }
          if (dst) {  // each warp instruction stores one contiguous 128-byte row segment
#pragma unroll
            for (int pp = 0; pp < kP; ++pp) dst[pp * kN] = hreg[pp];
          }
        }
        if (sdst) sdst += static_cast<int64_t>(p.H) * PN;
      }
      if (kk == nk) break;
      const int i2 = j & 1, ct = j % kTab;
      if (!waitw(c, bAux0 + ct, part(j))) return;
      const float c31 = lds_f32(cum + ((ct * 4 + kCF) * 32 + 31) * 4);
      const float atot = ex2_approx(c31);
      if (!waitw(c, bSFull0 + i2, par2(j))) return;
      tc_fence_after();
      {
        const uint32_t ta = tmem_addr(tmem, 32 * q, kColS0 + 64 * i2);
#pragma unroll
        for (int cq = 0; cq < 4; ++cq) {
          uint32_t sv[16];
          tmem_ld_32x32b_x16(ta + 16 * cq, sv);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i) hreg[16 * cq + i] = fmaf(atot, hreg[16 * cq + i], __uint_as_float(sv[i]));
        }
      }
      tc_fence_before();
      arrive_lane0(c, bSEmpty0 + i2);
      ++j;
    }
  }
}

// bf16 outputs of one thread (32 tokens of column p), out of line in the
// instances with a state chain (their epilogue loop runs faster without the
// inline copy; the one-block-item instance measured the other way).
__device__ __noinline__ void store_y_bf16(__nv_bfloat16 *dst, int64_t tstride, const uint32_t (&yo)[32]) {
#pragma unroll
  for (int t = 0; t < 32; ++t) dst[t * tstride] = __float2bfloat16_rn(__uint_as_float(yo[t]));
}

// ---------------------------------------------------------------- epilogue
// warps 12..15: thread owns column p = 16 q + (lane & 15) of the clean
// (lane < 16) or noisy (lane >= 16) stream's outputs y[t][p], t = 0..31
// (all-block pass; with a single stream, lanes < 16 own tokens 0..15 and
// lanes >= 16 tokens 16..31 of the clean stream's column p):
// y = exp(cum_t) Y_off + Y_diag (Y_diag already holds both directions' D x).
// After the outputs of step j the group builds, two steps ahead, the
// masked-decay matrices of step j + 2 with D on the diagonal (warp q:
// direction slot q, row s = lane of M^T) and the diagonal's bf16 remainders.
template <int kM, bool kGated>
__device__ void epilogue_group(const TcParams &p, const Ctl &c, uint32_t base, uint32_t tmem) {
  constexpr bool kAll = kM & kModeAll, kNeedS = kM & kModeNeedS, kCbF = kM & kModeCbFused;
  const int lane = threadIdx.x & 31;
  const int q = (threadIdx.x >> 5) & 3;
  const int pcol = 16 * q + (lane & 15);
  const bool noisy = lane >= 16;
  const int fs = noisy ? kNF : kCF;
  void *yout = noisy ? p.y_noisy : p.y_clean;
  const bool mine = (noisy ? kAll : true) && yout != nullptr;
  const uint32_t cumt = base + kOffCum;
  const int64_t H = p.H, L = p.L;
  const bool act = pick4(p.active, q) != 0;
  const bool rev = q >= 2;
  int mla = 0;        // next step whose masked-decay matrices this group builds
  bool mend = false;  // past the CTA's last step
  // A failed (timed-out) wait ends the group at once.
  auto build_m = [&]() -> bool {
    if (mend) return true;
    const int jm = mla;
    const int ct = jm % kTab;
    if (!waitw(c, bAux0 + ct, part(jm))) return false;
    const int f = lds_s32(base + kOffFtab + ct * 4);
    if (f < 0) {
      mend = true;
      return true;
    }
    if constexpr (kCbF) {
      if (!waitw(c, bCbFull, static_cast<uint32_t>(jm) & 1u)) return false;  // C B^T in TMEM
      tc_fence_after();
      build_masked_decay_tm(base, tmem, q, lane, jm);
      tc_fence_before();  // the accumulator's next writer waits for this warp's arrival
    } else {
      using Ly = Lay<kM>;
      if (!waitw(c, bFull0 + Ly::slot(jm), Ly::par(jm))) return false;  // C B^T tiles
      const uint32_t sl = base + static_cast<uint32_t>(Ly::slot(jm)) * Ly::kBytes;
      // one-block items without a state chain: the four-warp split (the
      // epilogue is that pipeline's co-bottleneck); otherwise one warp per
      // direction, which keeps warp 13 (the MMA issuer's sub-partition) idle
      // in the issue-bound state-chain instances
      if constexpr (kAll || kNeedS)
        build_masked_decay(base, sl + Ly::cb(q), q, lane, jm, act, rev);
      else if (q < 2 || p.active[kCR])
        build_masked_decay_split(base, sl + Ly::cb(q >= 2 ? kCR : kCF), q, lane, jm);
    }
    fence_proxy_async_smem();
    arrive_lane0(c, bMhFull0 + (jm & 1));
    ++mla;
    return true;
  };
  if (!build_m() || !build_m()) return;  // steps 0 and 1
  int j = 0;
  for (int m = 0;; ++m) {
    Item I;
    if (item_warp(p, c, base, m, I) <= 0) return;
    for (int kk = 0; kk < I.nk; ++kk, ++j) {
      const int k = I.k0 + kk;  // block index in the sequence
      const int yb = ybuf(kGated, j), ct = j % kTab;
      if (!waitw(c, bAux0 + ct, part(j))) return;
      if (!waitw(c, bYFull0 + yb, ypar(kGated, j))) return;
      tc_fence_after();
      if constexpr (!kAll) {
        // one stream: lanes 0..15 take tokens 0..15 of column p, lanes 16..31
        // tokens 16..31 (16x32bx2 loads, the second half 16 columns on)
        const int th = lane & 16;
        uint32_t yo[16], yd[16];
        const uint32_t ta = tmem_addr(tmem, 32 * q, kColY0 + kColYBuf * yb);
        tmem_ld_16x32bx2_x16i<16>(ta, yo);       // Y_off
        tmem_ld_16x32bx2_x16i<16>(ta + 64, yd);  // Y_diag
        tmem_ld_wait();
        const uint32_t eq = cumt + (ct * 4 + kCF) * 128 + 4 * th;
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          float c4[4];
          ld_shared_v4f(eq + 16 * jj, c4);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            yo[4 * jj + i] = __float_as_uint(
                fmaf(ex2_approx(c4[i]), __uint_as_float(yo[4 * jj + i]), __uint_as_float(yd[4 * jj + i])));
        }
        tmem_ld_16x32bx2_x16i<16>(ta + 96, yd);  // the diagonal remainders
        tmem_ld_wait();
#pragma unroll
        for (int t = 0; t < 16; ++t) yo[t] = __float_as_uint(__uint_as_float(yo[t]) + __uint_as_float(yd[t]));
        // gated: the reverse direction's own [Y_diag | remainder] (warp-uniform condition)
        const bool rev_act = kGated && p.active[kCR];
        if (rev_act) {
          tmem_ld_16x32bx2_x16i<16>(ta + 64 + kColRevGated, yd);
          uint32_t r16[16];
          tmem_ld_16x32bx2_x16i<16>(ta + 96 + kColRevGated, r16);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i) yd[i] = __float_as_uint(__uint_as_float(yd[i]) + __uint_as_float(r16[i]));
        }
        // the Y buffer may be reused from here on
        tc_fence_before();
        arrive_lane0(c, bYEmpty0 + yb);
        const int64_t tstride = H * kP;
        const int64_t yi = ((static_cast<int64_t>(I.b) * L + k * kT + th) * H + I.h) * kP + pcol;
        if (kGated) {
          const __nv_bfloat16 *zf = p.z[kCF], *zr = rev_act ? p.z[kCR] : nullptr;
          float gf[16], gr[16];
          gates16(zf, yi, tstride, gf);
          gates16(zr, yi, tstride, gr);
#pragma unroll
          for (int t = 0; t < 16; ++t) {
            float v = __uint_as_float(yo[t]) * gf[t];
            if (rev_act) v = fmaf(__uint_as_float(yd[t]), gr[t], v);
            yo[t] = __float_as_uint(v);
          }
        }
        if (p.y_clean) {
          if (p.out_bf16) {
            __nv_bfloat16 *dst = reinterpret_cast<__nv_bfloat16 *>(p.y_clean) + yi;
#pragma unroll
            for (int t = 0; t < 16; ++t) dst[t * tstride] = __float2bfloat16_rn(__uint_as_float(yo[t]));
          } else {
            float *dst = reinterpret_cast<float *>(p.y_clean) + yi;
#pragma unroll
            for (int t = 0; t < 16; ++t) dst[t * tstride] = __uint_as_float(yo[t]);
          }
        }
      } else {
        uint32_t yo[32], yd[32];
        const uint32_t ta = tmem_addr(tmem, 32 * q, kColY0 + kColYBuf * yb);
        tmem_ld_16x32bx2_x32<32>(ta, yo);       // Y_off: clean columns 0.., noisy 32..
        tmem_ld_16x32bx2_x32<64>(ta + 64, yd);  // Y_diag: clean 64.., noisy 128..
        tmem_ld_wait();
        const uint32_t eq = cumt + (ct * 4 + fs) * 128;
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          float c4[4];
          ld_shared_v4f(eq + 16 * jj, c4);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            yo[4 * jj + i] = __float_as_uint(
                fmaf(ex2_approx(c4[i]), __uint_as_float(yo[4 * jj + i]), __uint_as_float(yd[4 * jj + i])));
        }
        tmem_ld_16x32bx2_x32<64>(ta + 96, yd);  // the diagonal remainders: clean 96.., noisy 160..
        tmem_ld_wait();
#pragma unroll
        for (int t = 0; t < 32; ++t) yo[t] = __float_as_uint(__uint_as_float(yo[t]) + __uint_as_float(yd[t]));
        // gated: yo is the forward direction's output; the reverse direction's
        // own [Y_diag | remainder] goes to yd.  The TMEM loads are warp-wide
        // (.sync.aligned), so they run whenever either stream has a reverse
        // direction (uniform across the warp); a lane uses them only if its own
        // stream has one.
        const bool rev_act = kGated && pick4(p.active, fs | 2);
        if (kGated && (p.active[kCR] || p.active[kNR])) {
          tmem_ld_16x32bx2_x32<64>(ta + 64 + kColRevGated, yd);
          tmem_ld_wait();
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            uint32_t r16[16];
            tmem_ld_16x32bx2_x16i<64>(ta + 96 + kColRevGated + 16 * hh, r16);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i)
              yd[16 * hh + i] = __float_as_uint(__uint_as_float(yd[16 * hh + i]) + __uint_as_float(r16[i]));
          }
        }
        // the Y buffer may be reused from here on
        tc_fence_before();
        arrive_lane0(c, bYEmpty0 + yb);
        if (kGated && mine) {
          // y = y_fwd silu(z_fwd) + y_rev silu(z_rev) (a direction without z is not gated)
          const int64_t zi = ((static_cast<int64_t>(I.b) * L + k * kT) * H + I.h) * kP + pcol;
          const __nv_bfloat16 *zf = pick4(p.z, fs), *zr = rev_act ? pick4(p.z, fs | 2) : nullptr;
#pragma unroll
          for (int t0 = 0; t0 < 32; t0 += 16) {
            float gf[16], gr[16];
            gates16(zf, zi + t0 * H * kP, H * kP, gf);
            gates16(zr, zi + t0 * H * kP, H * kP, gr);
#pragma unroll
            for (int t = 0; t < 16; ++t) {
              float v = __uint_as_float(yo[t0 + t]) * gf[t];
              if (rev_act) v = fmaf(__uint_as_float(yd[t0 + t]), gr[t], v);
              yo[t0 + t] = __float_as_uint(v);
            }
          }
          if (kk + 1 < I.nk) {  // the next block's gates
            const int64_t zn = zi + static_cast<int64_t>(kT) * H * kP;
#pragma unroll
            for (int t = 0; t < 32; ++t) {
              if (zf) prefetch_l1(zf + zn + t * H * kP);
              if (zr) prefetch_l1(zr + zn + t * H * kP);
            }
          }
        }
        if (mine) {
          const int64_t yi = ((static_cast<int64_t>(I.b) * L + k * kT) * H + I.h) * kP + pcol;
          const int64_t tstride = H * kP;
          if (p.out_bf16) {
            __nv_bfloat16 *dst = reinterpret_cast<__nv_bfloat16 *>(yout) + yi;
            if constexpr (kNeedS) {
              store_y_bf16(dst, tstride, yo);
            } else {
#pragma unroll
              for (int t = 0; t < 32; ++t) dst[t * tstride] = __float2bfloat16_rn(__uint_as_float(yo[t]));
            }
          } else {
            float *dst = reinterpret_cast<float *>(yout) + yi;
#pragma unroll
            for (int t = 0; t < 32; ++t) dst[t * tstride] = __uint_as_float(yo[t]);
          }
        }
      }
      if (!build_m()) return;  // step j + 2
    }
  }
}

// Instantiated without and with a gate: the gated epilogue (per-direction
// accumulators, z loads) is compiled only into the gated kernel, so that it adds
// nothing to the instruction footprint of the ungated one.
template <int kM, bool kGated>
__global__ void __launch_bounds__(kThreads, 1) bd_tc_kernel(const __grid_constant__ TcParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t *sm = smem_raw + (base - raw);
  const int warp = threadIdx.x >> 5;

  uint64_t *bars = reinterpret_cast<uint64_t *>(sm + kOffBar);
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(sm + kOffMisc);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + kOffMisc + 4);
  // the next kernel on the stream may be scheduled now; it waits for this
  // grid's completion before it reads anything (its CTAs take SMs as ours exit)
  if (threadIdx.x == 0) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (threadIdx.x == 0) {
    // arrival counts: full = producer (plus TMA bytes); empty = MMA commit + 4
    // operand warps; commits of the MMA warp count 1; the rest 4 warps each
    for (int i = 0; i < bCount; ++i) {
      uint32_t cnt = 4;
      if ((i >= bFull0 && i < bFull0 + kMaxSlots) || i == bSFull0 || i == bSFull1 || i == bYFull0 ||
          i == bYFull1 || i == bHCons || i == bDrain || i == bCbFull || i >= bItem0)
        cnt = 1;
      else if (i >= bEmpty0 && i < bEmpty0 + kMaxSlots)
        cnt = 5;
      mbar_init(&bars[i], cnt);
    }
    *abort_flag = 0;
    *reinterpret_cast<unsigned long long *>(sm + kOffMisc + 8) = p.timeout_ns;
    *reinterpret_cast<int **>(sm + kOffMisc + 16) = p.status;
    fence_mbar_init();
  }
  // Clear the intra-block operands: of their remainder halves only the
  // diagonals are ever written.
  {
    const uint4 zero = make_uint4(0, 0, 0, 0);
    for (uint32_t o = threadIdx.x * 16; o < 2 * kMhBuf; o += kThreads * 16)
      *reinterpret_cast<uint4 *>(sm + kOffMh + o) = zero;
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  Ctl c{smem_u32(bars), base + kOffMisc};
  if constexpr ((kM & kModeCbFused) != 0) {
    // No pre-pass precedes this instance: every thread waits for the previous
    // kernel on the stream before its first read, and one thread clears the
    // status word (a CTA can raise it only after a wait that ran out its limit).
    // The tensor maps are kernel parameters, not the previous kernel's output:
    // their fetch overlaps the wait.
    if (threadIdx.x == 0) {
      tma_prefetch_desc(&p.tx[kCF]);
      tma_prefetch_desc(&p.tx[kCR]);
      tma_prefetch_desc(&p.tbcf);
      tma_prefetch_desc(&p.tbcr);
      tma_prefetch_desc(&p.tccf);
      tma_prefetch_desc(&p.tccr);
    }
    wait_prior_grid();
    if (blockIdx.x == 0 && threadIdx.x == 0) *p.status = 0;
  }
  // Launched as a programmatic dependent of the previous kernel on the stream
  // (the C B^T pre-pass, or the segment combine): the threads that read what it
  // wrote -- the producer (work counter, C B^T tiles) and the state warps
  // (segment initial states) -- wait for its completion (griddepcontrol.wait)
  // just before those reads; everything else overlaps its tail.  The
  // fused-C B^T instance waited above, before any role starts.

  if (warp == 0) {
    if ((threadIdx.x & 31) == 0) producer<kM>(p, c, base);
  } else if (warp == 1) {
    if ((threadIdx.x & 31) == 0) mma_issuer<kM, kGated>(p, c, base, tmem);
  } else if (warp == 2 || warp == 3 || warp == 6 || warp == 7) {
    operand_group<kM>(p, c, base);
  } else if (warp == 4 || warp == 5) {
    // idle: keeps the operand warps off the MMA issuer's SM sub-partition
  } else if (warp < 12) {
    state_group<kM>(p, c, base, tmem);
  } else {
    epilogue_group<kM, kGated>(p, c, base, tmem);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------------ aggregate pass
// Each segment's forward state from a zero start and its total decay, the
// input of the segment combine.  Unrolling [BDLM-PR] eq. (1) over a segment,
//   S_seg = sum_t w_t x_t B_t^T,   w_t = dt_t exp(sum_{u > t in seg} dt_u A),
// one dense contraction per segment, S^T[n][p] = B^T (w o X) over the
// segment's tokens, with no per-block state chain.  It is taken 128 tokens
// (four blocks) per pipeline step, from the segment's last step to its first,
// so that the weights relative to the segment's end are known step by step
// (a running sum of the later steps' decays).  w o X is split into bf16
// hi + lo (two MMAs per 16 tokens); S^T accumulates in TMEM (lane n, 64
// columns p), two buffers so that a segment's readout overlaps the next
// segment's MMAs.  Warps: 0 the TMA producer (x and B tiles, a three-step
// ring), 1 the MMA issuer and TMEM owner, 2..9 the operands (warps 2 + w and
// 6 + w build block w of a step, columns p 0..31 and 32..63) and, at a
// segment's end, the readout (TMEM lanes 32 (warp % 4) .., the same halves of
// the columns).  Work items (b, h, segment) go round-robin: item
// blockIdx.x + m gridDim.x.
namespace agg {
constexpr int kBlocks = 4;                          // blocks per pipeline step
constexpr int kStages = 3;                          // TMA ring depth
constexpr uint32_t kStB = kBlocks * kTile;          // B tiles within a stage (x tiles first)
constexpr uint32_t kStage = 3 * kBlocks * kTile;    // x: one tile per block; B: two per block
constexpr uint32_t kXwBuf = 2 * kBlocks * kTile;    // w o X {hi, lo} per block
constexpr uint32_t kOffXw = kStages * kStage;       // two w o X buffers
constexpr uint32_t kOffBar = kOffXw + 2 * kXwBuf;
enum : int {
  bFull = 0,
  bEmpty = bFull + kStages,
  bXwFull = bEmpty + kStages,
  bXwEmpty = bXwFull + 2,
  bSFull = bXwEmpty + 2,
  bSEmpty = bSFull + 2,
  bDrain = bSEmpty + 2,
  bCount
};
constexpr uint32_t kOffMisc = kOffBar + 8 * bCount;  // control block (layout of Ctl)
constexpr uint32_t kSmem = kOffMisc + 32 + 1024;     // + alignment of the base to 1 KB
constexpr int kThreadsAgg = 320;  // producer, issuer, eight operand warps
constexpr uint32_t kCols = 128;  // two S^T buffers of 64 columns
static_assert(kSmem <= 227 * 1024, "aggregate kernel shared memory");

struct Seg {
  int b, h, g, seg, k0, nk;
};
// This CTA's m-th item; false past the last.
__device__ __forceinline__ bool item(const TcParams &p, int m, Seg &I) {
  const int it = static_cast<int>(blockIdx.x) + m * static_cast<int>(gridDim.x);
  if (it >= p.items) return false;
  const int bh = it / p.nseg;
  I.seg = it - bh * p.nseg;
  I.b = bh / p.H;
  I.h = bh - I.b * p.H;
  I.g = I.h / (p.H / p.G);
  I.k0 = I.seg * p.seg_blocks;
  I.nk = min(p.K - I.k0, p.seg_blocks);
  return true;
}
__device__ __forceinline__ int steps(const Seg &I) { return (I.nk + kBlocks - 1) / kBlocks; }
// Step ci of an item (0: its last four blocks): first block kb, nb blocks.
__device__ __forceinline__ void step_blocks(const Seg &I, int ci, int &kb, int &nb) {
  const int hi = I.k0 + I.nk - kBlocks * ci;
  kb = max(I.k0, hi - kBlocks);
  nb = hi - kb;
}
__device__ __forceinline__ uint32_t doff(uint32_t bytes) { return bytes >> 4; }

__device__ void producer(const TcParams &p, const Ctl &c, uint32_t base) {
  tma_prefetch_desc(&p.tx[kCF]);
  tma_prefetch_desc(&p.tbcf);
  int last[kStages] = {-1, -1, -1};
  int j = 0;
  Seg I;
  for (int m = 0; item(p, m, I); ++m) {
    const int nc = steps(I);
    for (int ci = 0; ci < nc; ++ci, ++j) {
      const int s = j % kStages;
      const uint32_t par = static_cast<uint32_t>(j / kStages) & 1u;
      if (!wait1(c, bEmpty + s, par ^ 1u)) goto drain;
      int kb, nb;
      step_blocks(I, ci, kb, nb);
      const uint32_t full = bar_at(c, bFull + s);
      mbar_arrive_expect_tx_s(full, static_cast<uint32_t>(nb) * 3u * kTile);
      const uint32_t st = base + static_cast<uint32_t>(s) * kStage;
      for (int bi = 0; bi < nb; ++bi) {
        const int t0 = (kb + bi) * kT;
        tma_load_4d_s(st + bi * kTile, &p.tx[kCF], full, 0, I.h, t0, I.b);
        tma_load_4d_s(st + kStB + bi * 2 * kTile, &p.tbcf, full, 0, I.g, t0, I.b);
        tma_load_4d_s(st + kStB + bi * 2 * kTile + kTile, &p.tbcf, full, 64, I.g, t0, I.b);
      }
#pragma unroll
      for (int r = 0; r < kStages; ++r)
        if (r == s) last[r] = j;
    }
  }
drain:
  // no copy into this CTA's shared memory may still be in flight at exit
#pragma unroll
  for (int s = 0; s < kStages; ++s)
    if (last[s] >= 0)
      (void)mbar_wait_s(bar_at(c, bFull + s), static_cast<uint32_t>(last[s] / kStages) & 1u, p.drain_ns, 0);
}

// ---- MMA issuer
__device__ void issuer(const TcParams &p, const Ctl &c, uint32_t base, uint32_t tmem) {
  const uint32_t id_s = idesc_bf16(128, 64, 1, 1);  // S^T[n][p] = B^T (w o X): both MN-major
  const D64 dB = split64(sdesc(base + kStB, kTile, 1024, kLayoutSw128));  // n 0..63, 64..127 one tile apart
  const D64 dXw = split64(sdesc(base + kOffXw, 0, 1024, kLayoutSw128));
  int j = 0;
  Seg I;
  for (int m = 0; item(p, m, I); ++m) {
    const int nc = steps(I), sb = m & 1;
    const uint32_t colS = tmem + 64u * static_cast<uint32_t>(sb);
    // the readout of item m - 2 has emptied this accumulator
    if (!wait1(c, bSEmpty + sb, (static_cast<uint32_t>(m >> 1) & 1u) ^ 1u)) break;
    bool ok = true;
    for (int ci = 0; ci < nc; ++ci, ++j) {
      const int s = j % kStages, xb = j & 1;
      if (!wait1(c, bFull + s, static_cast<uint32_t>(j / kStages) & 1u) ||
          !wait1(c, bXwFull + xb, static_cast<uint32_t>(j >> 1) & 1u)) {
        ok = false;
        break;
      }
      tc_fence_after();
      int kb, nb;
      step_blocks(I, ci, kb, nb);
      const uint32_t so = doff(static_cast<uint32_t>(s) * kStage), xo = doff(static_cast<uint32_t>(xb) * kXwBuf);
#pragma unroll 1
      for (int bi = 0; bi < nb; ++bi) {
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) {
          const uint32_t ob = doff(static_cast<uint32_t>(bi) * 2u * kTile + static_cast<uint32_t>(ks) * 2048u);
          umma_bf16(colS, dB + so + ob, dXw + xo + ob, id_s, (ci > 0 || bi > 0 || ks > 0) ? 1u : 0u);
          umma_bf16(colS, dB + so + ob, dXw + xo + ob + doff(kTile), id_s, 1u);
        }
      }
      umma_commit_s(bar_at(c, bEmpty + s));
      umma_commit_s(bar_at(c, bXwEmpty + xb));
      if (ci + 1 == nc) umma_commit_s(bar_at(c, bSFull + sb));
    }
    if (!ok) break;
  }
  // every MMA issued has completed before TMEM is released
  umma_commit_s(bar_at(c, bDrain));
  (void)mbar_wait_s(bar_at(c, bDrain), 0, p.drain_ns, 0);
}

// ---- operand warps 2..9 (w = (warp - 2) % 4 builds block w of each step,
// half = (warp - 2) / 4 its columns p 32 half .. 32 half + 31)
// Every lane loads dt of its token in all four blocks of a step (two steps
// ahead), so that each warp forms the four blocks' decay sums itself and
// the group needs no exchange: per step, with v_k = dt A (log2 units) of
// block k, the warp's own suffix sums give sum_{u > t} over its block, the
// later blocks' totals and the running sum of the later steps the rest.
// A step's loads stay in their registers, as loaded, until that step is
// processed: the steps go in pairs with one register set each, so nothing
// reads (or converts) a load's destination before its latency has passed.
struct Raw {
  unsigned short dt[kBlocks];  // bf16 bits of dt of this lane's token in each block
  float A;
};

__device__ void operands(const TcParams &p, const Ctl &c, uint32_t base, uint32_t tmem) {
  const int lane = threadIdx.x & 31, w = ((threadIdx.x >> 5) - 2) & 3, half = ((threadIdx.x >> 5) - 2) >> 2;
  const int q = (threadIdx.x >> 5) & 3;  // TMEM lane quadrant of this warp
  const int64_t H = p.H, L = p.L, PN = kP * kN;
  const unsigned short *dtp = reinterpret_cast<const unsigned short *>(p.dt[kCF]);
  const float *Ap = p.A[kCF];
  // cursor over (item, step) of the loads
  int cm = 0, cci = 0;
  Seg CI;
  bool cv = item(p, 0, CI);
  auto load = [&](Raw &r) {
    r.A = 0.f;
#pragma unroll
    for (int k = 0; k < kBlocks; ++k) r.dt[k] = 0;
    if (!cv) return;
    int kb, nb;
    step_blocks(CI, cci, kb, nb);
    r.A = Ap[CI.h];
    const unsigned short *src = dtp + (static_cast<int64_t>(CI.b) * L + static_cast<int64_t>(kb) * kT + lane) * H + CI.h;
#pragma unroll
    for (int k = 0; k < kBlocks; ++k)
      if (k < nb) r.dt[k] = src[static_cast<int64_t>(k) * kT * H];
    if (++cci == steps(CI)) {
      cci = 0;
      cv = item(p, ++cm, CI);
    }
  };
  int j = 0, m = 0, ci = 0;
  Seg I;
  bool have = item(p, 0, I);
  float later_steps = 0.f;  // decay (log2) of the item's steps after this one
  // one step of item m; after its last step, the item's readout. false: a
  // wait ran out
  auto process = [&](const Raw &r) -> bool {
    const int s = j % kStages, xb = j & 1;
    const float A2 = r.A * kLog2e;
    // decays: totals of the four blocks (every lane) and this warp's block's
    // inclusive suffix sums
    float tot[kBlocks], own = 0.f, dt_own = 0.f;
#pragma unroll
    for (int k = 0; k < kBlocks; ++k) {
      const float dtk = __uint_as_float(static_cast<uint32_t>(r.dt[k]) << 16);
      const float v = dtk * A2;
      float rr = v;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) rr += __shfl_xor_sync(0xffffffffu, rr, o);
      tot[k] = rr;
      if (k == w) {
        own = v;
        dt_own = dtk;
      }
    }
    float suf = own;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float u = __shfl_down_sync(0xffffffffu, suf, o);
      if (lane + o < 32) suf += u;
    }
    float later = later_steps + (suf - own);
#pragma unroll
    for (int k = 0; k < kBlocks; ++k)
      if (k > w) later += tot[k];
    const float wt = dt_own * ex2_approx(later);
    later_steps += (tot[0] + tot[1]) + (tot[2] + tot[3]);
    // x of this step has landed; the MMAs of step j - 2 have read this buffer
    if (!waitw(c, bFull + s, static_cast<uint32_t>(j / kStages) & 1u)) return false;
    if (!waitw(c, bXwEmpty + xb, (static_cast<uint32_t>(j >> 1) & 1u) ^ 1u)) return false;
    int kb, nb;
    step_blocks(I, ci, kb, nb);
    if (w < nb) {
      // row `lane` of block w: this half's 32 values of x, scaled by w_t, as bf16 hi + lo
      const uint32_t xs = base + static_cast<uint32_t>(s) * kStage + static_cast<uint32_t>(w) * kTile;
      const uint32_t xh = base + kOffXw + static_cast<uint32_t>(xb) * kXwBuf + static_cast<uint32_t>(w) * 2u * kTile;
#pragma unroll 2
      for (int ch = 4 * half; ch < 4 * half + 4; ++ch) {
        const uint32_t off = sw128_chunk(static_cast<uint32_t>(lane), static_cast<uint32_t>(ch));
        uint32_t r0, r1, r2, r3;
        ld_shared_v4(xs + off, r0, r1, r2, r3);
        float vv[8] = {bf16_lo_f(r0) * wt, bf16_hi_f(r0) * wt, bf16_lo_f(r1) * wt, bf16_hi_f(r1) * wt,
                       bf16_lo_f(r2) * wt, bf16_hi_f(r2) * wt, bf16_lo_f(r3) * wt, bf16_hi_f(r3) * wt};
        store_split8(xh + off, xh + kTile + off, vv);
      }
      fence_proxy_async_smem();
    }
    arrive_lane0(c, bXwFull + xb);
    ++j;
    if (++ci < steps(I)) return true;
    // ---- readout: S^T (lane n = 32 q + lane, columns p) and the decay
    const int sb = m & 1;
    if (!waitw(c, bSFull + sb, static_cast<uint32_t>(m >> 1) & 1u)) return false;
    tc_fence_after();
    const int64_t ebhs = (static_cast<int64_t>(I.b) * p.H + I.h) * p.nseg + I.seg;
    float *dst = p.seg_local + ebhs * PN + 32 * q + lane;
    const uint32_t ta = tmem_addr(tmem, 32u * static_cast<uint32_t>(q), 64u * static_cast<uint32_t>(sb));
#pragma unroll 1
    for (int cq = 2 * half; cq < 2 * half + 2; ++cq) {
      uint32_t sv[16];
      tmem_ld_32x32b_x16(ta + 16u * static_cast<uint32_t>(cq), sv);
      tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < 16; ++i) dst[(16 * cq + i) * kN] = __uint_as_float(sv[i]);
    }
    if (threadIdx.x == 64) p.seg_decay[ebhs] = later_steps;
    tc_fence_before();
    arrive_lane0(c, bSEmpty + sb);
    ++m;
    ci = 0;
    later_steps = 0.f;
    have = item(p, m, I);
    return true;
  };
  Raw ra, rb;
  load(ra);
  load(rb);
  while (have) {
    if (!process(ra)) return;
    load(ra);
    if (!have) break;
    if (!process(rb)) return;
    load(rb);
  }
}
}  // namespace agg

__global__ void __launch_bounds__(agg::kThreadsAgg, 1) bd_agg_kernel(const __grid_constant__ TcParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t *sm = smem_raw + (base - raw);
  const int warp = threadIdx.x >> 5;
  uint64_t *bars = reinterpret_cast<uint64_t *>(sm + agg::kOffBar);
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(sm + agg::kOffMisc);
  if (threadIdx.x == 0) {
    // full: producer + TMA bytes; empty, xw-empty, S-full, drain: one MMA
    // commit; xw-full, S-empty: the eight operand warps
    for (int i = 0; i < agg::bCount; ++i)
      mbar_init(&bars[i], (i >= agg::bXwFull && i < agg::bXwFull + 2) || (i >= agg::bSEmpty && i < agg::bSEmpty + 2) ? 8u : 1u);
    *reinterpret_cast<volatile int *>(sm + agg::kOffMisc + 4) = 0;
    *reinterpret_cast<unsigned long long *>(sm + agg::kOffMisc + 8) = p.timeout_ns;
    *reinterpret_cast<int **>(sm + agg::kOffMisc + 16) = p.status;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, agg::kCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const Ctl c{smem_u32(bars), base + agg::kOffMisc};
  // Launched as a programmatic dependent of the C B^T pre-pass, whose CTAs
  // trigger only after every earlier kernel on the stream has completed: the
  // inputs are ready; the pre-pass's own output is not read here.
  if (warp == 0) {
    if ((threadIdx.x & 31) == 0) agg::producer(p, c, base);
  } else if (warp == 1) {
    if ((threadIdx.x & 31) == 0) agg::issuer(p, c, base, tmem);
  } else {
    agg::operands(p, c, base, tmem);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // this grid completes after the pre-pass, as a plain launch would
  wait_prior_grid();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, agg::kCols);
  }
}

// ------------------------------------------------------------------ segment combine
// Chains the segments of every (b, h) sequence: H_0 = h0 (or 0) and
// H_{j+1} = exp(decay_j) H_j + local_j, where local_j is segment j's end state
// from a zero start and decay_j its total decay (the aggregate pass leaves
// both).  One thread per state element.
__global__ void __launch_bounds__(256) bd_seg_combine_kernel(const float *h0, const float *local,
                                                             const float *decay, float *init, int nseg) {
  const int64_t PN = kP * kN;
  const int64_t bh = blockIdx.x;
  const int64_t e = static_cast<int64_t>(blockIdx.y) * 256 + threadIdx.x;
  float hc = h0 ? h0[bh * PN + e] : 0.f;
  for (int j = 0; j < nseg; ++j) {
    const int64_t bj = bh * nseg + j;
    init[bj * PN + e] = hc;
    hc = fmaf(ex2_approx(decay[bj]), hc, local[bj * PN + e]);
  }
}

// ------------------------------------------------------------------ host side
constexpr size_t kCounterOffset = 256;  // bytes into the workspace header
static_assert(kCounterOffset + 2 * sizeof(int) <= kWsHeader, "workspace header");
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// bf16 [d3][d2][d1][d0] (d0 innermost), box (64, 1, 32, 1), 128-byte swizzle.
bool make_map_bf16(CUtensorMap *m, const void *ptr, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t d3) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {d0, d1, d2, d3};
  cuuint64_t strides[3] = {d0 * 2, d0 * d1 * 2, d0 * d1 * d2 * 2};
  cuuint32_t box[4] = {64, 1, 32, 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(ptr), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}


// bf16 C B^T tiles [n][32][32], box (32, 32, 1), 64-byte swizzle.
bool make_map_cb(CUtensorMap *m, const void *ptr, uint64_t ntiles) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {32, 32, ntiles};
  cuuint64_t strides[2] = {32 * 2, 32 * 32 * 2};
  cuuint32_t box[3] = {32, 32, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int kM, bool kGated>
cudaError_t launch_instance(const cudaLaunchConfig_t &cfg, const TcParams &p) {
  cudaError_t e = cudaFuncSetAttribute(bd_tc_kernel<kM, kGated>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kSmemBytes));
  if (e != cudaSuccess) return e;
  return cudaLaunchKernelEx(&cfg, bd_tc_kernel<kM, kGated>, p);
}

// The scan kernel as a programmatic dependent launch (its prologue may overlap
// the previous kernel in the stream; it waits for that kernel before reading),
// in the instance of the call's mode: the all-block pass, a scan with a state
// chain (per-block or final state), or one-block items without one (with the
// C B^T tiles from the pre-pass or computed in the kernel); each with or
// without a gate.
cudaError_t launch_scan(unsigned grid, cudaStream_t stream, const TcParams &p) {
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e;
  if (p.allblock)
    e = p.gated ? launch_instance<kModeAll | kModeNeedS, true>(cfg, p)
                : launch_instance<kModeAll | kModeNeedS, false>(cfg, p);
  else if (p.need_s)
    e = p.gated ? launch_instance<kModeNeedS, true>(cfg, p) : launch_instance<kModeNeedS, false>(cfg, p);
  else if (p.cbfused)
    e = p.gated ? launch_instance<kModeCbFused, true>(cfg, p) : launch_instance<kModeCbFused, false>(cfg, p);
  else
    e = p.gated ? launch_instance<0, true>(cfg, p) : launch_instance<0, false>(cfg, p);
  return e != cudaSuccess ? e : cudaGetLastError();
}

// The aggregate pass as a programmatic dependent of the C B^T pre-pass (its
// prologue overlaps the pre-pass's tail), one CTA per SM at most.
cudaError_t launch_agg(unsigned grid, cudaStream_t stream, const TcParams &p) {
  cudaError_t e = cudaFuncSetAttribute(bd_agg_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(agg::kSmem));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(agg::kThreadsAgg);
  cfg.dynamicSmemBytes = agg::kSmem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, bd_agg_kernel, p);
  return e != cudaSuccess ? e : cudaGetLastError();
}

bool device_is_sm100() {
  static int cached = -1;
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  if (cached < 0) {
    int dev = 0, major = 0, minor = 0;
    cached = 0;
    if (cudaGetDevice(&dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) == cudaSuccess)
      cached = (major == 10 && minor == 0) ? 1 : 0;
  }
  return cached == 1;
}

}  // namespace

bool tc_shape_ok(int64_t P, int64_t N, int64_t T, bool in_bf16) {
  return in_bf16 && P == kP && N == kN && T == kT;
}

// Number of segments each (b, h) sequence is cut into.  Segments let few long
// sequences (prefill at batch 1) fill the machine, at the price of an
// aggregate pass over the clean forward stream (each segment's state from
// zero), a segment combine and per-item start-up.  The plan minimises a cost
// in units of one main-pass block step: the main pass's makespan (items run
// in waves of one per SM; a wave lasts its longest segment), the aggregate
// pass's (the same waves at kAggCost of a main step), the combine's chain
// and the two extra launches; one segment when that is cheapest.
int tc_plan_segments(int64_t Bsz, int64_t H, int64_t K, bool allblock) {
  constexpr int64_t kSms = 148;
  const double kAggCost = allblock ? 0.13 : 0.2;  // aggregate / main pass time per block, measured
  const int64_t chains = Bsz * H;
  if (K < 8 || chains <= 0) return 1;
  int64_t best = 1;
  double best_cost = static_cast<double>((chains + kSms - 1) / kSms) * static_cast<double>(K);
  for (int64_t s = 2; s <= K / 4; ++s) {
    const int64_t seg_blocks = (K + s - 1) / s;
    const int64_t nseg = (K + seg_blocks - 1) / seg_blocks;
    const int64_t waves = (chains * nseg + kSms - 1) / kSms;
    const double cost = static_cast<double>(waves) * (static_cast<double>(seg_blocks) * (1.0 + kAggCost) + 2.0) +
                        0.5 * static_cast<double>(nseg) + 4.0;
    if (cost < best_cost - 1e-9) {
      best_cost = cost;
      best = nseg;
    }
  }
  return static_cast<int>(best);
}

static size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// C B^T tiles (bf16 [32][32] per direction, b, block, group), then for a
// segmented plan the segments' local end states, their initial states and
// their decays.
size_t tc_workspace_bytes(int64_t Bsz, int64_t L, int64_t G, int64_t H, bool allblock) {
  const int64_t K = L / kT;
  size_t bytes = align256(static_cast<size_t>(cb_sets(allblock)) * Bsz * K * G * 2048);
  const int nseg = tc_plan_segments(Bsz, H, K, allblock);
  if (nseg > 1) {
    const size_t states = static_cast<size_t>(Bsz) * H * nseg * kP * kN * sizeof(float);
    bytes += 2 * align256(states) + align256(static_cast<size_t>(Bsz) * H * nseg * sizeof(float));
  }
  return bytes;
}

bool tc_supported(const ScanArgs &a) {
  if (!tc_shape_ok(a.P, a.N, a.T, a.in_bf16)) return false;
  if (a.Bsz <= 0 || a.L <= 0) return false;
  if (a.Bsz * a.H > 0x7fffffffLL || a.L > 0x7fffffffLL || 4 * a.Bsz * (a.L / kT) * a.G > 0x7fffffffLL)
    return false;
  if (a.ws_bytes < kWsHeader + tc_workspace_bytes(a.Bsz, a.L, a.G, a.H, a.mode == Mode::AllBlock)) return false;
  if (opt_force_generic()) return false;
  return device_is_sm100();
}

// One-block items without a state chain, both clean directions, no more
// items than SMs (small-batch denoising steps): the scan kernel computes the
// C B^T tiles itself and the call is one launch.
bool tc_one_launch_step(const ScanArgs &a) {
  if (a.mode == Mode::AllBlock || !a.has_cr || a.L != kT || a.states || a.final_state || opt_cb_prepass())
    return false;
  int dev = 0, nsm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return false;
  return a.Bsz * a.H <= nsm && tc_plan_segments(a.Bsz, a.H, 1, false) == 1;
}

cudaError_t launch_tc(const ScanArgs &a, cudaStream_t stream) {
  const bool all = a.mode == Mode::AllBlock;
  const DirArgs *ds[4] = {&a.cf, all ? &a.nf : nullptr, a.has_cr ? &a.cr : nullptr,
                          (all && a.has_nr) ? &a.nr : nullptr};
  __nv_bfloat16 *cbws = reinterpret_cast<__nv_bfloat16 *>(static_cast<uint8_t *>(a.ws) + kWsHeader);
  const unsigned long long timeout = opt_wait_timeout_ns();
  const int K = static_cast<int>(a.L / kT);
  int dev = 0, nsm = 0;
  cudaError_t e;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess ||
      (e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return e;
  const bool cbfused = tc_one_launch_step(a);

  // ---- C B^T of every active direction
  CbParams cp;
  std::memset(&cp, 0, sizeof(cp));
  int nz = 0;
  for (int i = 0; i < 4; ++i) {
    if (!ds[i]) continue;
    if (!make_map_bf16(&cp.tb[nz], ds[i]->B, kN, a.G, a.L, a.Bsz) ||
        !make_map_bf16(&cp.tc[nz], ds[i]->C, kN, a.G, a.L, a.Bsz))
      return cudaErrorInvalidValue;
    cp.slot[nz++] = cb_set(all, i);
  }
  cp.Bsz = static_cast<int>(a.Bsz);
  cp.K = K;
  cp.G = static_cast<int>(a.G);
  cp.cb = cbws;
  // work-item counters ([1]: the scan kernel's), in the workspace header next
  // to the status word; the pre-pass zeroes both
  int *counters = reinterpret_cast<int *>(static_cast<uint8_t *>(a.ws) + kCounterOffset);
  cp.item_counters = counters;
  cp.status = a.status;
  cp.timeout_ns = timeout;
  if ((e = cudaFuncSetAttribute(bd_cb_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(kCbSmem))) != cudaSuccess)
    return e;
  dim3 cgrid((K + 3) / 4, static_cast<unsigned>(a.Bsz * a.G), nz);
  if (!cbfused) {
    // programmatic dependent launch: its CTAs may be scheduled while the
    // previous kernel finishes; they wait for it before touching memory
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = cgrid;
    cfg.blockDim = dim3(kCbThreads);
    cfg.dynamicSmemBytes = kCbSmem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if ((e = cudaLaunchKernelEx(&cfg, bd_cb_kernel, cp)) != cudaSuccess) return e;
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }

  // ---- the scan
  TcParams p;
  std::memset(&p, 0, sizeof(p));
  for (int i = 0; i < 4; ++i) {
    p.active[i] = ds[i] != nullptr;
    if (!ds[i]) continue;
    if (!make_map_bf16(&p.tx[i], ds[i]->x, kP, a.H, a.L, a.Bsz)) return cudaErrorInvalidValue;
    p.dt[i] = reinterpret_cast<const __nv_bfloat16 *>(ds[i]->dt);
    p.z[i] = reinterpret_cast<const __nv_bfloat16 *>(ds[i]->z);
    if (ds[i]->z) p.gated = 1;
    p.A[i] = ds[i]->A;
    p.D[i] = ds[i]->D;
  }
  if (!make_map_bf16(&p.tbcf, a.cf.B, kN, a.G, a.L, a.Bsz) ||
      !make_map_bf16(&p.tccf, a.cf.C, kN, a.G, a.L, a.Bsz) ||
      !make_map_cb(&p.tcb, cbws, static_cast<uint64_t>(cb_sets(all)) * a.Bsz * K * a.G))
    return cudaErrorInvalidValue;
  if (all && !make_map_bf16(&p.tcnf, a.nf.C, kN, a.G, a.L, a.Bsz)) return cudaErrorInvalidValue;
  if (cbfused && (!make_map_bf16(&p.tbcr, a.cr.B, kN, a.G, a.L, a.Bsz) ||
                  !make_map_bf16(&p.tccr, a.cr.C, kN, a.G, a.L, a.Bsz)))
    return cudaErrorInvalidValue;
  p.cbfused = cbfused ? 1 : 0;
  p.Bsz = static_cast<int>(a.Bsz);
  p.L = static_cast<int>(a.L);
  p.H = static_cast<int>(a.H);
  p.G = static_cast<int>(a.G);
  p.K = K;
  const int nseg = tc_plan_segments(a.Bsz, a.H, K, all);
  p.nseg = nseg;
  p.seg_blocks = (K + nseg - 1) / nseg;
  p.items = static_cast<int>(a.Bsz * a.H * nseg);
  p.dv_nseg = make_divu(nseg);
  p.dv_h = make_divu(static_cast<int>(a.H));
  p.dv_hpg = make_divu(static_cast<int>(a.H / a.G));
  p.item_counter = counters + 1;
  p.allblock = all ? 1 : 0;
  p.need_s = (a.states || a.final_state || p.seg_blocks > 1 || nseg > 1) ? 1 : 0;
  p.out_bf16 = a.out_bf16 ? 1 : 0;
  p.h0 = a.h0;
  p.states = a.states;
  p.final_state = a.final_state;
  p.y_clean = a.y_clean;
  p.y_noisy = all ? a.y_noisy : nullptr;
  p.status = a.status;
  p.timeout_ns = timeout;
  p.drain_ns = 1000000000ull;
  // persistent CTAs, one per SM, each walking its share of the work items
  const unsigned grid = static_cast<unsigned>(p.items < nsm ? p.items : nsm);
  if (nseg > 1) {
    // aggregate kernel (clean forward state of every segment from zero, items
    // round-robin over the CTAs), then the chain of segment states
    uint8_t *wsb = static_cast<uint8_t *>(a.ws) + kWsHeader;
    const size_t cb_bytes = align256(static_cast<size_t>(cb_sets(all)) * a.Bsz * K * a.G * 2048);
    const size_t st_bytes = align256(static_cast<size_t>(a.Bsz) * a.H * nseg * kP * kN * sizeof(float));
    float *seg_local = reinterpret_cast<float *>(wsb + cb_bytes);
    float *seg_init = reinterpret_cast<float *>(wsb + cb_bytes + st_bytes);
    float *seg_decay = reinterpret_cast<float *>(wsb + cb_bytes + 2 * st_bytes);
    TcParams q = p;
    q.need_s = 1;
    q.allblock = 0;
    for (int i = 1; i < 4; ++i) q.active[i] = 0;
    q.states = nullptr;
    q.final_state = nullptr;
    q.y_clean = q.y_noisy = nullptr;
    q.seg_local = seg_local;
    q.item_counter = nullptr;
    q.seg_decay = seg_decay;
    if ((e = launch_agg(grid, stream, q)) != cudaSuccess) return e;
    bd_seg_combine_kernel<<<dim3(static_cast<unsigned>(a.Bsz * a.H), (kP * kN) / 256), 256, 0, stream>>>(
        a.h0, seg_local, seg_decay, seg_init, nseg);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    p.seg_init = seg_init;
  }
  return launch_scan(grid, stream, p);
}

}  // namespace bdscan
