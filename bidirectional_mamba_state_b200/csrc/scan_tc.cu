// scan_tc.cu -- tensor-core block-diffusion scan for sm_100a
// (bf16 inputs, headdim P = 64, d_state N = 128, block T = 32, no gate).
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
// Two kernels:
//   bd_cb_kernel  C B^T of every (direction, batch, block, group) -- shared by
//                 all heads of a group -- with one M=128 tcgen05 MMA chain per
//                 four blocks, into the workspace (fp32, 4 KB per block).
//   bd_tc_kernel  one CTA per (b, h) walks its blocks in order with the fp32
//                 state on chip.  Warp roles (448 threads, one CTA per SM):
//     warp 0      TMA producer: x, B, C and C B^T tiles of block k, 2 stages
//     warp 1      TMEM allocator and single-thread tcgen05.mma issuer
//     warps 2-5   operands: decays, (w o X) (bf16 hi + lo), masked-decay M
//     warps 6-9   state chain: h_k = exp(cum_31) h_{k-1} + S, boundary-state
//                 stores, h operand (bf16 hi + lo) for the next block
//     warps 10-13 epilogue: y = exp(cum) Y_off + Y_diag + D x, stores
//   S, Y, the h operand and M are double-buffered, so the only serial
//   dependency between blocks is the state recurrence itself.
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
constexpr int kCF = 0, kNF = 1, kCR = 2, kNR = 3;
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
  int slot[4];  // blockIdx.z -> stacking slot
  int Bsz, K, G;
  float *cb;    // [4][B][K][G][32 s][32 t]
  int *status;
  unsigned long long timeout_ns;
};

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
  ok = __all_sync(0xffffffffu, ok) && !*abort_flag;
  if (ok) {
    tc_fence_after();
    uint32_t r[32];
    tmem_ld_32x32b_x32(tmem_addr(tmem, 32 * warp, 32 * warp), r);
    tmem_ld_wait();
    if (warp < nvalid) {
      const int64_t idx = ((static_cast<int64_t>(slot) * p.Bsz + b) * p.K + k0 + warp) * p.G + g;
      float4 *dst = reinterpret_cast<float4 *>(p.cb + idx * 1024 + lane * 32);
#pragma unroll
      for (int i = 0; i < 8; ++i)
        dst[i] = make_float4(__uint_as_float(r[4 * i]), __uint_as_float(r[4 * i + 1]),
                             __uint_as_float(r[4 * i + 2]), __uint_as_float(r[4 * i + 3]));
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
constexpr int kThreads = 448;

// shared memory map (bytes from a 1024-aligned base)
constexpr uint32_t kOffX = 0;                 // 4 slots x [32 t][64 p] bf16, SW128
constexpr uint32_t kOffBcf = 4 * kTile;       // clean-forward B: [32 s][n 0..63], [32 s][n 64..127]
constexpr uint32_t kOffClo = 6 * kTile;       // [C_cf; C_nf] rows x n 0..63
constexpr uint32_t kOffChi = 8 * kTile;       // [C_cf; C_nf] rows x n 64..127
constexpr uint32_t kOffCB = 10 * kTile;       // 4 slots x [32 s][32 t] fp32, SW128
constexpr uint32_t kStage = 14 * kTile;       // 56 KB per stage
constexpr uint32_t kOffXw = 2 * kStage;       // hi [32 t][64 p], lo [32 t][64 p] (bf16, SW128)
constexpr uint32_t kOffH = kOffXw + 2 * kTile;  // 2 buffers x {hi, lo} x {n 0..63, n 64..127} x [64 p][128 B]
constexpr uint32_t kHBuf = 8 * kTile;           // per buffer: hi at +0, lo at +4 tiles; n-half at +2 tiles
constexpr uint32_t kOffMh = kOffH + 2 * kHBuf;  // 2 buffers x {fwd, rev} x [64 t][64 s] interleaved
constexpr uint32_t kMhBuf = 4 * kTile;
constexpr uint32_t kOffCum = kOffMh + 2 * kMhBuf;  // [2][4][32] f32, log2 units
constexpr uint32_t kOffDt = kOffCum + 1024;        // [2][4][32] f32
constexpr uint32_t kOffBar = kOffDt + 1024;
constexpr int kNumBars = 24;
constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;
constexpr uint32_t kSmemBytes = kOffMisc + 64 + 1024;
static_assert(kSmemBytes <= 232448, "shared memory budget");

// masked-decay operand: [64 t][64 s] (block diagonal: first/second direction
// of the pair), interleaved MN-major (t contiguous): t-groups 128 B apart,
// s-groups 1024 B apart.
constexpr uint32_t kMhSbo = 128, kMhLbo = 1024;

enum : int {
  bFull0 = 0, bFull1, bEmpty0, bEmpty1, bAux0, bAux1, bXwFull, bSFull0, bSFull1, bSEmpty0, bSEmpty1,
  bMhFull0, bMhFull1, bHFull0, bHFull1, bYFull0, bYFull1, bYEmpty0, bYEmpty1, bDrain
};

// TMEM columns: S[2] (M=64 x 128), Y[2] = {Y_off (M=64 x 64), Y_diag (M=64 x 64)}
constexpr uint32_t kColS0 = 0, kColY0 = 256;
constexpr uint32_t kTmemCols = 512;

struct TcParams {
  CUtensorMap tx[4];
  CUtensorMap tbcf;
  CUtensorMap tccf;
  CUtensorMap tcnf;
  CUtensorMap tcb;
  const __nv_bfloat16 *dt[4];
  const float *A[4];
  const float *D[4];
  int active[4];
  int Bsz, L, H, G, K;
  int allblock;
  int out_bf16;
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
__device__ __forceinline__ float bf16_hi_f(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

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

struct Ctl {
  uint64_t *bar;
  volatile int *abort;
  int *status;
  unsigned long long timeout_ns;
};

__device__ __noinline__ void raise_timeout(const Ctl &c) {
  *c.abort = 1;
  atomicCAS(c.status, 0, kStatusTimeout);
}

__device__ __forceinline__ bool wait1(const Ctl &c, int bar, uint32_t parity) {
  if (mbar_wait(&c.bar[bar], parity, c.timeout_ns, c.abort)) return true;
  raise_timeout(c);
  return false;
}

// Whole-warp bounded wait with a warp-uniform outcome.
__device__ __forceinline__ bool waitw(const Ctl &c, int bar, uint32_t parity) {
  bool ok = mbar_wait(&c.bar[bar], parity, c.timeout_ns, c.abort);
  ok = __all_sync(0xffffffffu, ok);
  if (!ok && (threadIdx.x & 31) == 0) raise_timeout(c);
  __syncwarp();
  return ok;
}

__device__ __forceinline__ void arrive_lane0(const Ctl &c, int bar) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(&c.bar[bar]);
}

// parity of the completion of a double-buffered barrier that block k uses
__device__ __forceinline__ uint32_t par2(int k) { return (static_cast<uint32_t>(k) >> 1) & 1u; }

// ---------------------------------------------------------------- producer
__device__ void producer(const TcParams &p, const Ctl &c, uint8_t *sm, int b, int h, int g) {
  uint32_t bytes = 2 * kTile + (p.allblock ? 4 : 2) * kTile;
  for (int i = 0; i < 4; ++i)
    if (p.active[i]) bytes += 2 * kTile;
  tma_prefetch_desc(&p.tbcf);
  tma_prefetch_desc(&p.tccf);
  tma_prefetch_desc(&p.tcb);
  int last_k[2] = {-1, -1};
  for (int k = 0; k < p.K; ++k) {
    const int s = k & 1;
    if (!wait1(c, bEmpty0 + s, par2(k) ^ 1)) break;
    uint64_t *full = &c.bar[bFull0 + s];
    mbar_arrive_expect_tx(full, bytes);
    uint8_t *st = sm + s * kStage;
    const int t0 = k * kT;
    for (int i = 0; i < 4; ++i) {
      if (!p.active[i]) continue;
      tma_load_4d(st + kOffX + i * kTile, &p.tx[i], full, 0, h, t0, b);
      const int idx = ((i * p.Bsz + b) * p.K + k) * p.G + g;
      tma_load_3d(st + kOffCB + i * kTile, &p.tcb, full, 0, 0, idx);
    }
    tma_load_4d(st + kOffBcf, &p.tbcf, full, 0, g, t0, b);
    tma_load_4d(st + kOffBcf + kTile, &p.tbcf, full, 64, g, t0, b);
    tma_load_4d(st + kOffClo, &p.tccf, full, 0, g, t0, b);
    tma_load_4d(st + kOffChi, &p.tccf, full, 64, g, t0, b);
    if (p.allblock) {
      tma_load_4d(st + kOffClo + kTile, &p.tcnf, full, 0, g, t0, b);
      tma_load_4d(st + kOffChi + kTile, &p.tcnf, full, 64, g, t0, b);
    }
    last_k[s] = k;
  }
  // no copy into this CTA's shared memory may still be in flight at exit
  for (int s = 0; s < 2; ++s)
    if (last_k[s] >= 0) (void)mbar_wait(&c.bar[bFull0 + s], par2(last_k[s]), p.drain_ns, nullptr);
}

// ---------------------------------------------------------------- MMA issuer
__device__ void mma_issuer(const TcParams &p, const Ctl &c, uint32_t base, uint32_t tmem) {
  const uint32_t id_s = idesc_bf16(64, 128, 1, 1);  // S[p][n] = (w o X)^T B
  const uint32_t id_yo = idesc_bf16(64, 64, 0, 0);  // Y_off[t][p] = C h^T
  const uint32_t id_yd = idesc_bf16(64, 64, 1, 1);  // Y_diag[t][p] = M X
  const bool any_rev = p.active[kCR] || p.active[kNR];
  for (int k = 0; k < p.K; ++k) {
    const int s = k & 1, i2 = k & 1;
    const uint32_t st = base + s * kStage;
    if (!wait1(c, bFull0 + s, par2(k))) break;
    // ---- S(k) = (w o X)^T B_cf: A MN-major (p), B MN-major (n; halves 4 KB apart)
    if (!wait1(c, bXwFull, k & 1)) break;
    if (k >= 2 && !wait1(c, bSEmpty0 + i2, par2(k - 2))) break;
    tc_fence_after();
    const uint32_t colS = kColS0 + 128 * i2;
    for (int ks = 0; ks < 2; ++ks) {
      const uint64_t ah = sdesc(base + kOffXw + ks * 2048, 0, 1024, kLayoutSw128);
      const uint64_t al = sdesc(base + kOffXw + kTile + ks * 2048, 0, 1024, kLayoutSw128);
      const uint64_t bb = sdesc(st + kOffBcf + ks * 2048, kTile, 1024, kLayoutSw128);
      umma_bf16(tmem + colS, ah, bb, id_s, ks > 0);
      umma_bf16(tmem + colS, al, bb, id_s, 1);
    }
    umma_commit(&c.bar[bSFull0 + i2]);
    // ---- Y(k): Y_off = [C_cf; C_nf] h_{k-1}^T, Y_diag = M_fwd X_fwd + M_rev X_rev
    if (!wait1(c, bMhFull0 + i2, par2(k))) break;
    if (!wait1(c, bHFull0 + ((k + 1) & 1), par2(k))) break;  // h_{k-1} lives in buffer (k-1) & 1
    if (k >= 2 && !wait1(c, bYEmpty0 + i2, par2(k - 2))) break;
    tc_fence_after();
    const uint32_t colY = kColY0 + 128 * i2;
    const uint32_t hb = base + kOffH + ((k + 1) & 1) * kHBuf;
    for (int ks = 0; ks < 8; ++ks) {
      const uint32_t koff = (ks < 4 ? 0 : 2 * kTile) + (ks & 3) * 32;
      const uint64_t a = sdesc(st + (ks < 4 ? kOffClo : kOffChi) + (ks & 3) * 32, 16, 1024, kLayoutSw128);
      const uint64_t bh = sdesc(hb + koff, 16, 1024, kLayoutSw128);
      const uint64_t bl = sdesc(hb + 4 * kTile + koff, 16, 1024, kLayoutSw128);
      umma_bf16(tmem + colY, a, bh, id_yo, ks > 0);
      umma_bf16(tmem + colY, a, bl, id_yo, 1);
    }
    const uint32_t mb = base + kOffMh + i2 * kMhBuf;
    for (int ks = 0; ks < 4; ++ks) {
      const uint64_t a = sdesc(mb + ks * 2048, kMhLbo, kMhSbo, kLayoutNone);
      const uint64_t bb = sdesc(st + kOffX + ks * 2048, 0, 1024, kLayoutSw128);
      umma_bf16(tmem + colY + 64, a, bb, id_yd, ks > 0);
    }
    if (any_rev) {
      for (int ks = 0; ks < 4; ++ks) {
        const uint64_t a = sdesc(mb + 2 * kTile + ks * 2048, kMhLbo, kMhSbo, kLayoutNone);
        const uint64_t bb = sdesc(st + kOffX + 2 * kTile + ks * 2048, 0, 1024, kLayoutSw128);
        umma_bf16(tmem + colY + 64, a, bb, id_yd, 1);
      }
    }
    umma_commit(&c.bar[bYFull0 + i2]);
    umma_commit(&c.bar[bEmpty0 + s]);
  }
  umma_commit(&c.bar[bDrain]);
  (void)mbar_wait(&c.bar[bDrain], 0, p.drain_ns, nullptr);
}

// ---------------------------------------------------------------- operand group
// warps 2..5; q = warp & 3 is the direction slot whose decays and M it builds.
__device__ void operand_group(const TcParams &p, const Ctl &c, uint8_t *sm, uint32_t base, int b, int h) {
  const int lane = threadIdx.x & 31;
  const int q = (threadIdx.x >> 5) & 3;
  const int gt = threadIdx.x - 64;  // 0..127
  const bool act = p.active[q] != 0;
  const bool rev = q >= 2;
  float *cum = reinterpret_cast<float *>(sm + kOffCum);
  float *dts = reinterpret_cast<float *>(sm + kOffDt);
  const int64_t H = p.H, L = p.L;
  const float A2 = act ? p.A[q][h] * kLog2e : 0.f;
  const __nv_bfloat16 *dtp = p.dt[q];
  auto load_dt = [&](int k) -> float {
    if (!act || k >= p.K) return 0.f;
    return __bfloat162float(dtp[(static_cast<int64_t>(b) * L + k * kT + lane) * H + h]);
  };
  float dt_next = load_dt(0);
  // position of this direction's block in the stacked [64 t][64 s] operand
  const uint32_t mset = rev ? 2 * kTile : 0;
  const uint32_t d0 = (q & 1) ? 32 : 0;
  for (int k = 0; k < p.K; ++k) {
    const int s = k & 1, i2 = k & 1;
    const float dt_cur = dt_next;
    dt_next = load_dt(k + 1);
    if (!waitw(c, bFull0 + s, par2(k))) break;
    if (act) {
      float v = dt_cur * A2;
      if (!rev) {
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const float u = __shfl_up_sync(0xffffffffu, v, o);
          if (lane >= o) v += u;
        }
      } else {
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const float u = __shfl_down_sync(0xffffffffu, v, o);
          if (lane + o < 32) v += u;
        }
      }
      cum[(s * 4 + q) * 32 + lane] = v;
      dts[(s * 4 + q) * 32 + lane] = dt_cur;
    }
    arrive_lane0(c, bAux0 + s);
    if (!waitw(c, bAux0 + s, par2(k))) break;
    // ---- (w o X) of the clean forward direction, bf16 hi + lo
    if (k >= 1 && !waitw(c, bSFull0 + ((k + 1) & 1), par2(k - 1))) break;
    {
      const float *cf = cum + (s * 4 + kCF) * 32;
      const float *df = dts + (s * 4 + kCF) * 32;
      const float c31 = cf[31];
#pragma unroll
      for (int rep = 0; rep < 2; ++rep) {
        const int i = gt + 128 * rep;
        const int t = i >> 3, ch = i & 7;
        const uint32_t off = sw128_chunk(t, ch);
        uint32_t r0, r1, r2, r3;
        ld_shared_v4(base + s * kStage + kOffX + off, r0, r1, r2, r3);
        const float w = df[t] * exp2f(c31 - cf[t]);
        float v[8] = {bf16_lo_f(r0) * w, bf16_hi_f(r0) * w, bf16_lo_f(r1) * w, bf16_hi_f(r1) * w,
                      bf16_lo_f(r2) * w, bf16_hi_f(r2) * w, bf16_lo_f(r3) * w, bf16_hi_f(r3) * w};
        store_split8(base + kOffXw + off, base + kOffXw + kTile + off, v);
      }
      fence_proxy_async_smem();
      arrive_lane0(c, bXwFull);
    }
    // ---- masked-decay matrix, row s = lane of M^T for this direction
    if (k >= 2 && !waitw(c, bYFull0 + i2, par2(k - 2))) break;
    if (act) {
      const uint32_t cbrow = base + s * kStage + kOffCB + q * kTile + lane * 128;
      float cbv[32];
#pragma unroll
      for (int ch = 0; ch < 8; ++ch) {
        uint32_t r0, r1, r2, r3;
        ld_shared_v4(cbrow + ((ch ^ (lane & 7)) << 4), r0, r1, r2, r3);
        cbv[4 * ch] = __uint_as_float(r0);
        cbv[4 * ch + 1] = __uint_as_float(r1);
        cbv[4 * ch + 2] = __uint_as_float(r2);
        cbv[4 * ch + 3] = __uint_as_float(r3);
      }
      const float *cq = cum + (s * 4 + q) * 32;
      const float cs = cq[lane];
      const float ds = dts[(s * 4 + q) * 32 + lane];
      const uint32_t mrow = base + kOffMh + i2 * kMhBuf + mset;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float m[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int t = 8 * j + i;
          const bool valid = rev ? (t <= lane) : (t >= lane);
          const float e = exp2f(cq[t] - cs);
          m[i] = valid ? cbv[t] * ds * e : 0.f;
        }
        st_shared_v4(mrow + inter_mn_off(d0 + 8 * j, d0 + lane, kMhSbo, kMhLbo), pack_bf16x2(m[0], m[1]),
                     pack_bf16x2(m[2], m[3]), pack_bf16x2(m[4], m[5]), pack_bf16x2(m[6], m[7]));
      }
    }
    fence_proxy_async_smem();
    arrive_lane0(c, bMhFull0 + i2);
    arrive_lane0(c, bEmpty0 + s);
  }
}

// ---------------------------------------------------------------- state group
// warps 6..9: thread owns h[p][n0 .. n0+63], p = 16 q + (lane & 15), n0 = 64 (lane >> 4).
__device__ void state_group(const TcParams &p, const Ctl &c, uint8_t *sm, uint32_t base, uint32_t tmem,
                            int b, int h) {
  const int lane = threadIdx.x & 31;
  const int q = (threadIdx.x >> 5) & 3;
  const int prow = 16 * q + (lane & 15);
  const int half = lane >> 4;
  const int n0 = 64 * half;
  const float *cum = reinterpret_cast<const float *>(sm + kOffCum);
  const int64_t H = p.H;
  const int64_t PN = kP * kN;
  float hreg[64];
  {
    const float *src = p.h0 ? p.h0 + (static_cast<int64_t>(b) * H + h) * PN + prow * kN + n0 : nullptr;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float4 v = src ? reinterpret_cast<const float4 *>(src)[i] : make_float4(0.f, 0.f, 0.f, 0.f);
      hreg[4 * i] = v.x;
      hreg[4 * i + 1] = v.y;
      hreg[4 * i + 2] = v.z;
      hreg[4 * i + 3] = v.w;
    }
  }
  // h operand of Y_off (K-major, SW128): buffer hbuf holds {hi: n 0..63, n 64..127;
  // lo: n 0..63, n 64..127}, each [64 p rows][128 B].
  auto write_h = [&](int hbuf) {
    const uint32_t hb = base + kOffH + hbuf * kHBuf + half * 2 * kTile;
#pragma unroll
    for (int cc = 0; cc < 8; ++cc) {
      const uint32_t off = sw128_chunk(prow, cc);
      store_split8(hb + off, hb + 4 * kTile + off, hreg + 8 * cc);
    }
    fence_proxy_async_smem();
    arrive_lane0(c, bHFull0 + hbuf);
  };
  write_h(1);  // h_{-1} lives in buffer 1
  for (int k = 0; k < p.K; ++k) {
    const int s = k & 1, i2 = k & 1;
    if (!waitw(c, bAux0 + s, par2(k))) break;
    const float atot = exp2f(cum[(s * 4 + kCF) * 32 + 31]);
    if (!waitw(c, bSFull0 + i2, par2(k))) break;
    tc_fence_after();
    {
      uint32_t sv[32];
      const uint32_t ta = tmem_addr(tmem, 32 * q, kColS0 + 128 * i2);
      tmem_ld_16x32bx2_x32<64>(ta, sv);
      tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < 32; ++i) hreg[i] = fmaf(atot, hreg[i], __uint_as_float(sv[i]));
      tmem_ld_16x32bx2_x32<64>(ta + 32, sv);
      tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < 32; ++i) hreg[32 + i] = fmaf(atot, hreg[32 + i], __uint_as_float(sv[i]));
    }
    tc_fence_before();
    arrive_lane0(c, bSEmpty0 + i2);
    arrive_lane0(c, bEmpty0 + s);
    if (p.states) {
      float4 *dst = reinterpret_cast<float4 *>(p.states + ((static_cast<int64_t>(b) * p.K + k) * H + h) * PN +
                                               prow * kN + n0);
#pragma unroll
      for (int i = 0; i < 16; ++i)
        dst[i] = make_float4(hreg[4 * i], hreg[4 * i + 1], hreg[4 * i + 2], hreg[4 * i + 3]);
    }
    // buffer k & 1 held h_{k-2}; Y(k-1) has read it once y_full(k-1) completes
    if (k >= 1 && !waitw(c, bYFull0 + ((k + 1) & 1), par2(k - 1))) break;
    write_h(k & 1);
  }
  if (p.final_state && !*c.abort) {
    float4 *dst =
        reinterpret_cast<float4 *>(p.final_state + (static_cast<int64_t>(b) * H + h) * PN + prow * kN + n0);
#pragma unroll
    for (int i = 0; i < 16; ++i)
      dst[i] = make_float4(hreg[4 * i], hreg[4 * i + 1], hreg[4 * i + 2], hreg[4 * i + 3]);
  }
}

// ---------------------------------------------------------------- epilogue
// warps 10..13: accumulator row r = 16 q + (lane & 15) is token t = r & 31 of the
// clean (r < 32) or noisy (r >= 32) stream; columns p0 .. p0+31, p0 = 32 (lane >> 4).
__device__ void epilogue_group(const TcParams &p, const Ctl &c, uint8_t *sm, uint32_t base, uint32_t tmem,
                               int b, int h) {
  const int lane = threadIdx.x & 31;
  const int q = (threadIdx.x >> 5) & 3;
  const int row = 16 * q + (lane & 15);
  const int t = row & 31;
  const bool noisy = row >= 32;
  const int p0 = 32 * (lane >> 4);
  const float *cum = reinterpret_cast<const float *>(sm + kOffCum);
  const int fs = noisy ? kNF : kCF, rs = noisy ? kNR : kCR;
  void *yout = noisy ? p.y_noisy : p.y_clean;
  const bool mine = (noisy ? p.allblock != 0 : true) && yout != nullptr;
  const bool has_rev = p.active[rs] != 0;
  const float Df = p.active[fs] ? p.D[fs][h] : 0.f;
  const float Dr = has_rev ? p.D[rs][h] : 0.f;
  const int64_t H = p.H, L = p.L;
  for (int k = 0; k < p.K; ++k) {
    const int s = k & 1, i2 = k & 1;
    if (!waitw(c, bFull0 + s, par2(k))) break;
    if (!waitw(c, bAux0 + s, par2(k))) break;
    if (!waitw(c, bYFull0 + i2, par2(k))) break;
    tc_fence_after();
    uint32_t yo[32], yd[32];
    const uint32_t ta = tmem_addr(tmem, 32 * q, kColY0 + 128 * i2);
    tmem_ld_16x32bx2_x32<32>(ta, yo);
    tmem_ld_16x32bx2_x32<32>(ta + 64, yd);
    tmem_ld_wait();
    tc_fence_before();
    arrive_lane0(c, bYEmpty0 + i2);
    if (mine) {
      const float e = exp2f(cum[(s * 4 + fs) * 32 + t]);
      const uint32_t xf = base + s * kStage + kOffX + fs * kTile;
      const uint32_t xr = base + s * kStage + kOffX + rs * kTile;
      float y[32];
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        const uint32_t ch = (p0 >> 3) + cc;
        uint32_t f[4], r[4] = {0, 0, 0, 0};
        ld_shared_v4(xf + sw128_chunk(t, ch), f[0], f[1], f[2], f[3]);
        if (has_rev) ld_shared_v4(xr + sw128_chunk(t, ch), r[0], r[1], r[2], r[3]);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int j = 8 * cc + 2 * i;
          float v0 = fmaf(e, __uint_as_float(yo[j]), __uint_as_float(yd[j]));
          float v1 = fmaf(e, __uint_as_float(yo[j + 1]), __uint_as_float(yd[j + 1]));
          v0 = fmaf(Df, bf16_lo_f(f[i]), v0);
          v1 = fmaf(Df, bf16_hi_f(f[i]), v1);
          v0 = fmaf(Dr, bf16_lo_f(r[i]), v0);
          v1 = fmaf(Dr, bf16_hi_f(r[i]), v1);
          y[j] = v0;
          y[j + 1] = v1;
        }
      }
      const int64_t yi = ((static_cast<int64_t>(b) * L + k * kT + t) * H + h) * kP + p0;
      if (p.out_bf16) {
        uint4 *dst = reinterpret_cast<uint4 *>(reinterpret_cast<__nv_bfloat16 *>(yout) + yi);
#pragma unroll
        for (int i = 0; i < 4; ++i)
          dst[i] = make_uint4(pack_bf16x2(y[8 * i], y[8 * i + 1]), pack_bf16x2(y[8 * i + 2], y[8 * i + 3]),
                              pack_bf16x2(y[8 * i + 4], y[8 * i + 5]), pack_bf16x2(y[8 * i + 6], y[8 * i + 7]));
      } else {
        float4 *dst = reinterpret_cast<float4 *>(reinterpret_cast<float *>(yout) + yi);
#pragma unroll
        for (int i = 0; i < 8; ++i) dst[i] = make_float4(y[4 * i], y[4 * i + 1], y[4 * i + 2], y[4 * i + 3]);
      }
    }
    arrive_lane0(c, bEmpty0 + s);
  }
}

__global__ void __launch_bounds__(kThreads, 1) bd_tc_kernel(const __grid_constant__ TcParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t *sm = smem_raw + (base - raw);
  const int warp = threadIdx.x >> 5;
  const int bh = blockIdx.x;
  const int b = bh / p.H, h = bh % p.H;
  const int g = h / (p.H / p.G);

  uint64_t *bars = reinterpret_cast<uint64_t *>(sm + kOffBar);
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(sm + kOffMisc);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + kOffMisc + 4);
  if (threadIdx.x == 0) {
    const uint32_t counts[bDrain + 1] = {1, 1, 13, 13, 4, 4, 4, 1, 1, 4, 4, 4, 4, 4, 4, 1, 1, 4, 4, 1};
    for (int i = 0; i <= bDrain; ++i) mbar_init(&bars[i], counts[i]);
    *abort_flag = 0;
    fence_mbar_init();
  }
  // Tiles that are never loaded are read by MMAs next to zero operands: clear
  // them (and both masked-decay buffers, whose off-diagonal blocks stay zero) so
  // that no uninitialised NaN/Inf bit pattern can reach an output.
  {
    const uint4 zero = make_uint4(0, 0, 0, 0);
    for (int i = 0; i < 4; ++i) {
      if (p.active[i]) continue;
      for (int s = 0; s < 2; ++s)
        for (uint32_t o = threadIdx.x * 16; o < kTile; o += kThreads * 16)
          *reinterpret_cast<uint4 *>(sm + s * kStage + kOffX + i * kTile + o) = zero;
    }
    if (!p.allblock)
      for (int s = 0; s < 2; ++s)
        for (uint32_t o = threadIdx.x * 16; o < kTile; o += kThreads * 16) {
          *reinterpret_cast<uint4 *>(sm + s * kStage + kOffClo + kTile + o) = zero;
          *reinterpret_cast<uint4 *>(sm + s * kStage + kOffChi + kTile + o) = zero;
        }
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
  Ctl c{bars, abort_flag, p.status, p.timeout_ns};

  if (warp == 0) {
    if ((threadIdx.x & 31) == 0) producer(p, c, sm, b, h, g);
  } else if (warp == 1) {
    if ((threadIdx.x & 31) == 0) mma_issuer(p, c, base, tmem);
  } else if (warp < 6) {
    operand_group(p, c, sm, base, b, h);
  } else if (warp < 10) {
    state_group(p, c, sm, base, tmem, b, h);
  } else {
    epilogue_group(p, c, sm, base, tmem, b, h);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------------ host side
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

// fp32 C B^T tiles [n][32][32], box (32, 32, 1), 128-byte swizzle.
bool make_map_cb(CUtensorMap *m, const void *ptr, uint64_t ntiles) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {32, 32, ntiles};
  cuuint64_t strides[2] = {32 * 4, 32 * 32 * 4};
  cuuint32_t box[3] = {32, 32, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void *>(ptr), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
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

unsigned long long env_ns(const char *name, unsigned long long dflt) {
  const char *v = std::getenv(name);
  if (!v || !*v) return dflt;
  return std::strtoull(v, nullptr, 10);
}

}  // namespace

bool tc_shape_ok(int64_t P, int64_t N, int64_t T, bool in_bf16) {
  return in_bf16 && P == kP && N == kN && T == kT;
}

size_t tc_workspace_bytes(int64_t Bsz, int64_t L, int64_t G) {
  return static_cast<size_t>(4) * Bsz * (L / kT) * G * kTile;
}

bool tc_supported(const ScanArgs &a) {
  if (!tc_shape_ok(a.P, a.N, a.T, a.in_bf16)) return false;
  if (a.Bsz <= 0 || a.L <= 0) return false;
  const DirArgs *ds[4] = {&a.cf, &a.nf, &a.cr, &a.nr};
  for (const DirArgs *d : ds)
    if (d->z) return false;
  if (a.Bsz * a.H > 0x7fffffffLL || a.L > 0x7fffffffLL || 4 * a.Bsz * (a.L / kT) * a.G > 0x7fffffffLL)
    return false;
  if (a.ws_bytes < kWsHeader + tc_workspace_bytes(a.Bsz, a.L, a.G)) return false;
  const char *force = std::getenv("BDSCAN_FORCE_GENERIC");
  if (force && force[0] == '1') return false;
  return device_is_sm100();
}

cudaError_t launch_tc(const ScanArgs &a, cudaStream_t stream) {
  const bool all = a.mode == Mode::AllBlock;
  const DirArgs *ds[4] = {&a.cf, all ? &a.nf : nullptr, a.has_cr ? &a.cr : nullptr,
                          (all && a.has_nr) ? &a.nr : nullptr};
  float *cbws = reinterpret_cast<float *>(static_cast<uint8_t *>(a.ws) + kWsHeader);
  const unsigned long long timeout = env_ns("BDSCAN_WAIT_TIMEOUT_NS", 2000000000ull);
  const int K = static_cast<int>(a.L / kT);

  // ---- C B^T of every active direction
  CbParams cp;
  std::memset(&cp, 0, sizeof(cp));
  int nz = 0;
  for (int i = 0; i < 4; ++i) {
    if (!ds[i]) continue;
    if (!make_map_bf16(&cp.tb[nz], ds[i]->B, kN, a.G, a.L, a.Bsz) ||
        !make_map_bf16(&cp.tc[nz], ds[i]->C, kN, a.G, a.L, a.Bsz))
      return cudaErrorInvalidValue;
    cp.slot[nz++] = i;
  }
  cp.Bsz = static_cast<int>(a.Bsz);
  cp.K = K;
  cp.G = static_cast<int>(a.G);
  cp.cb = cbws;
  cp.status = a.status;
  cp.timeout_ns = timeout;
  cudaError_t e = cudaFuncSetAttribute(bd_cb_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kCbSmem));
  if (e != cudaSuccess) return e;
  dim3 cgrid((K + 3) / 4, static_cast<unsigned>(a.Bsz * a.G), nz);
  bd_cb_kernel<<<cgrid, kCbThreads, kCbSmem, stream>>>(cp);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;

  // ---- the scan
  TcParams p;
  std::memset(&p, 0, sizeof(p));
  for (int i = 0; i < 4; ++i) {
    p.active[i] = ds[i] != nullptr;
    if (!ds[i]) continue;
    if (!make_map_bf16(&p.tx[i], ds[i]->x, kP, a.H, a.L, a.Bsz)) return cudaErrorInvalidValue;
    p.dt[i] = reinterpret_cast<const __nv_bfloat16 *>(ds[i]->dt);
    p.A[i] = ds[i]->A;
    p.D[i] = ds[i]->D;
  }
  if (!make_map_bf16(&p.tbcf, a.cf.B, kN, a.G, a.L, a.Bsz) ||
      !make_map_bf16(&p.tccf, a.cf.C, kN, a.G, a.L, a.Bsz) ||
      !make_map_cb(&p.tcb, cbws, static_cast<uint64_t>(4) * a.Bsz * K * a.G))
    return cudaErrorInvalidValue;
  if (all && !make_map_bf16(&p.tcnf, a.nf.C, kN, a.G, a.L, a.Bsz)) return cudaErrorInvalidValue;
  p.Bsz = static_cast<int>(a.Bsz);
  p.L = static_cast<int>(a.L);
  p.H = static_cast<int>(a.H);
  p.G = static_cast<int>(a.G);
  p.K = K;
  p.allblock = all ? 1 : 0;
  p.out_bf16 = a.out_bf16 ? 1 : 0;
  p.h0 = a.h0;
  p.states = a.states;
  p.final_state = a.final_state;
  p.y_clean = a.y_clean;
  p.y_noisy = all ? a.y_noisy : nullptr;
  p.status = a.status;
  p.timeout_ns = timeout;
  p.drain_ns = 1000000000ull;
  e = cudaFuncSetAttribute(bd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(kSmemBytes));
  if (e != cudaSuccess) return e;
  bd_tc_kernel<<<static_cast<unsigned>(a.Bsz * a.H), kThreads, kSmemBytes, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace bdscan
