// scan_tc.cu -- fused tensor-core block-diffusion scan for sm_100a
// (bf16 inputs, headdim P = 64, d_state N = 128, block T = 32, no gate).
//
// What one CTA computes: one (batch row b, head h) sequence, walking its
// 32-token blocks k = 0 .. K-1 in order and keeping the fp32 forward state on
// chip.  Per block, in the chunked (state-space-duality) form of the
// recurrence of "Training Hybrid Block Diffusion Language Models with Partial
// Bidirectionality", eq. (1), with cum_t = sum_{u<=t in block} dt_u A:
//
//   CB^T[s][t] = B_s . C_t                    (tensor cores, all directions)
//   M[t][s]    = CB[t][s] dt_s exp(cum_t - cum_s), s <= t      (forward)
//              = CB[t][s] dt_s exp(rcum_t - rcum_s), s >= t    (reverse,
//                rcum_t = sum_{u>=t in block} dt_u A; eq. (12))
//   Y_diag^T   = X^T M^T                       (tensor cores)
//   Y_off^T    = h_{k-1} C^T                   (tensor cores; eq. (11): the
//                forward continuation from the boundary state)
//   S^T        = B^T (w o X),  w_t = dt_t exp(cum_31 - cum_t)
//   h_k        = exp(cum_31) h_{k-1} + S       (boundary state, eq. (10))
//   y          = exp(cum_t) Y_off + Y_diag,fwd + Y_diag,rev + D_f x_f + D_r x_r
//                (eq. (13): forward plus block-local reverse)
// The all-block pass (eq. (14)) adds the noisy stream: its forward part starts
// from the same h_{k-1} (the clean boundary state before block k), its
// reverse part is block-local.
//
// Warp roles (320 threads, one CTA per SM):
//   warp 0     TMA producer: x, B, C tiles of block k into a 2-stage ring
//   warp 1     TMEM allocator and single-thread tcgen05.mma issuer
//   warps 2-5  "state" group: decays, (w o X) operand, masked-decay matrices,
//              fp32 state update h_k, boundary-state stores, h operand
//   warps 6-9  epilogue: y = exp(cum) Y_off + Y_diag + D x, stores
// Every wait is bounded; on a timeout the CTA raises BDSCAN_ERR_TIMEOUT in the
// workspace status word, drains its own copies and MMAs, frees TMEM and exits.
//
// Operand precision: C, B and x are bf16 (exact).  fp32 operands (w o X, the
// state h) are split into bf16 hi + lo parts and fed as two MMAs, so the
// state and off-diagonal products keep ~16 mantissa bits; the masked-decay
// matrix M is rounded once to bf16 (it multiplies exact x values and only
// contributes the intra-block term).  Accumulation is fp32 in TMEM.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <cstdlib>
#include <mutex>

#include "bdscan_internal.h"
#include "sm100.cuh"

namespace bdscan {
namespace {

using namespace sm100;

constexpr int kT = 32, kP = 64, kN = 128;
constexpr int kThreads = 320;
// stacking slots of the four directions
constexpr int kCF = 0, kNF = 1, kCR = 2, kNR = 3;

// ---- shared memory map (bytes from a 1024-aligned base)
constexpr uint32_t kTile = 4096;              // 32 rows x 128 B
constexpr uint32_t kOffX = 0;                 // 4 slots x [32 t][64 p] bf16, SW128
constexpr uint32_t kOffBlo = 4 * kTile;       // 4 slots x [32 s][n 0..63]
constexpr uint32_t kOffBhi = 8 * kTile;       // 4 slots x [32 s][n 64..127]
constexpr uint32_t kOffClo = 12 * kTile;
constexpr uint32_t kOffChi = 16 * kTile;
constexpr uint32_t kStage = 20 * kTile;       // 80 KB per stage
constexpr uint32_t kOffXwHi = 2 * kStage;     // [32 t][64 p] bf16, SW128
constexpr uint32_t kOffXwLo = kOffXwHi + kTile;
constexpr uint32_t kOffHHi = kOffXwLo + kTile;  // [128 n][64 p] bf16, SW128
constexpr uint32_t kOffHLo = kOffHHi + 4 * kTile;
constexpr uint32_t kOffMh = kOffHLo + 4 * kTile;  // 4 slots x 2 KB, interleaved MN-major
constexpr uint32_t kOffCum = kOffMh + 4 * 2048;   // [2][4][32] f32 (log2 units)
constexpr uint32_t kOffDt = kOffCum + 1024;       // [2][4][32] f32
constexpr uint32_t kOffBar = kOffDt + 1024;
constexpr int kNumBars = 16;
constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;  // tmem base, abort flag
constexpr uint32_t kSmemBytes = kOffMisc + 64 + 1024;  // + alignment slack

// barrier indices
enum : int {
  bFull0 = 0, bFull1, bEmpty0, bEmpty1, bCbFull, bMhFull, bXwFull, bSFull, bSEmpty,
  bHFull, bYFull, bYEmpty, bAux0, bAux1, bDrain
};

// ---- TMEM columns (512 allocated)
constexpr uint32_t kColS = 0;     // S^T: M=128 (n) x 64 (p)
constexpr uint32_t kColCB = 128;  // CB^T: M=128 (slot, s) x 128 (slot, t)
constexpr uint32_t kColY = 256;   // Y_off^T: M=64 (p) x 64 (t clean | t noisy)
constexpr uint32_t kColYC = 320;  // Y_diag^T clean: M=64 x 32
constexpr uint32_t kColYN = 352;  // Y_diag^T noisy: M=64 x 32
constexpr uint32_t kTmemCols = 512;

// MH (masked-decay matrix, B operand of Y_diag): interleaved MN-major, N = t,
// K = s; core matrices 8 (s) x 16 B (8 t); t-groups 128 B apart, s-groups 512 B.
constexpr uint32_t kMhSbo = 128, kMhLbo = 512;

constexpr float kLog2e = 1.4426950408889634f;

struct TcParams {
  CUtensorMap tx[4];
  CUtensorMap tb[4];
  CUtensorMap tc[4];
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

// Split 8 fp32 values into bf16 hi and lo parts (v ~= hi + lo) and store each
// as one 16-byte chunk.
__device__ __forceinline__ void store_split8(uint32_t addr_hi, uint32_t addr_lo, const float (&v)[8]) {
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
  atomicCAS(c.status, 0, -6 /* BDSCAN_ERR_TIMEOUT */);
}

// Single-thread bounded wait.
__device__ __forceinline__ bool wait1(const Ctl &c, int bar, uint32_t parity) {
  if (mbar_wait(&c.bar[bar], parity, c.timeout_ns, c.abort)) return true;
  raise_timeout(c);
  return false;
}

// Whole-warp bounded wait; the outcome is made warp-uniform.
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

// ------------------------------------------------------------------ roles
__device__ void producer(const TcParams &p, const Ctl &c, uint32_t base, int b, int h, int g) {
  int nact = 0;
  for (int i = 0; i < 4; ++i) nact += p.active[i];
  const uint32_t bytes = nact * 5 * kTile;
  uint8_t *gen = reinterpret_cast<uint8_t *>(__cvta_shared_to_generic(base));
  int last_k[2] = {-1, -1};
  for (int i = 0; i < 4; ++i)
    if (p.active[i]) {
      tma_prefetch_desc(&p.tx[i]);
      tma_prefetch_desc(&p.tb[i]);
      tma_prefetch_desc(&p.tc[i]);
    }
  for (int k = 0; k < p.K; ++k) {
    const int s = k & 1;
    const uint32_t ps = (k >> 1) & 1;
    if (!wait1(c, bEmpty0 + s, ps ^ 1)) break;
    mbar_arrive_expect_tx(&c.bar[bFull0 + s], bytes);
    uint8_t *st = gen + s * kStage;
    const int t0 = k * kT;
    for (int i = 0; i < 4; ++i) {
      if (!p.active[i]) continue;
      tma_load_4d(st + kOffX + i * kTile, &p.tx[i], &c.bar[bFull0 + s], 0, h, t0, b);
      tma_load_4d(st + kOffBlo + i * kTile, &p.tb[i], &c.bar[bFull0 + s], 0, g, t0, b);
      tma_load_4d(st + kOffBhi + i * kTile, &p.tb[i], &c.bar[bFull0 + s], 64, g, t0, b);
      tma_load_4d(st + kOffClo + i * kTile, &p.tc[i], &c.bar[bFull0 + s], 0, g, t0, b);
      tma_load_4d(st + kOffChi + i * kTile, &p.tc[i], &c.bar[bFull0 + s], 64, g, t0, b);
    }
    last_k[s] = k;
  }
  // Make sure no copy into this CTA's shared memory is still in flight.
  for (int s = 0; s < 2; ++s)
    if (last_k[s] >= 0) (void)mbar_wait(&c.bar[bFull0 + s], (last_k[s] >> 1) & 1, p.drain_ns, nullptr);
}

__device__ void mma_issuer(const TcParams &p, const Ctl &c, uint32_t base, uint32_t tmem) {
  const uint32_t id_cb = idesc_bf16(128, 128, 0, 0);
  const uint32_t id_s = idesc_bf16(128, 64, 1, 1);
  const uint32_t id_yo = idesc_bf16(64, p.allblock ? 64 : 32, 1, 0);
  const uint32_t id_yd = idesc_bf16(64, 32, 1, 1);
  for (int k = 0; k < p.K; ++k) {
    const int s = k & 1;
    const uint32_t ps = (k >> 1) & 1;
    const uint32_t st = base + s * kStage;
    if (!wait1(c, bFull0 + s, ps)) break;
    // ---- CB^T for all stacked directions: A = B rows (K-major), B = C rows
    if (k > 0 && !wait1(c, bMhFull, (k - 1) & 1)) break;
    tc_fence_after();
    for (int ks = 0; ks < 8; ++ks) {
      const uint32_t off = (ks & 3) * 32;
      const uint64_t a = sdesc(st + (ks < 4 ? kOffBlo : kOffBhi) + off, 16, 1024, kLayoutSw128);
      const uint64_t bb = sdesc(st + (ks < 4 ? kOffClo : kOffChi) + off, 16, 1024, kLayoutSw128);
      umma_bf16(tmem + kColCB, a, bb, id_cb, ks > 0);
    }
    umma_commit(&c.bar[bCbFull]);
    // ---- S^T = B_cf^T (w o X): A MN-major (n; halves 16 KB apart), B MN-major (p)
    if (!wait1(c, bXwFull, k & 1)) break;
    if (k > 0 && !wait1(c, bSEmpty, (k - 1) & 1)) break;
    tc_fence_after();
    for (int ks = 0; ks < 2; ++ks) {
      const uint64_t a = sdesc(st + kOffBlo + ks * 2048, kOffBhi - kOffBlo, 1024, kLayoutSw128);
      const uint64_t bh = sdesc(base + kOffXwHi + ks * 2048, 0, 1024, kLayoutSw128);
      const uint64_t bl = sdesc(base + kOffXwLo + ks * 2048, 0, 1024, kLayoutSw128);
      umma_bf16(tmem + kColS, a, bh, id_s, ks > 0);
      umma_bf16(tmem + kColS, a, bl, id_s, 1);
    }
    umma_commit(&c.bar[bSFull]);
    // ---- Y_off^T = h_{k-1} C^T and Y_diag^T = X^T M^T
    if (!wait1(c, bMhFull, k & 1)) break;
    if (!wait1(c, bHFull, k & 1)) break;
    if (k > 0 && !wait1(c, bYEmpty, (k - 1) & 1)) break;
    tc_fence_after();
    for (int ks = 0; ks < 8; ++ks) {
      const uint64_t ah = sdesc(base + kOffHHi + ks * 2048, 0, 1024, kLayoutSw128);
      const uint64_t al = sdesc(base + kOffHLo + ks * 2048, 0, 1024, kLayoutSw128);
      const uint64_t bc = sdesc(st + (ks < 4 ? kOffClo : kOffChi) + (ks & 3) * 32, 16, 1024, kLayoutSw128);
      umma_bf16(tmem + kColY, ah, bc, id_yo, ks > 0);
      umma_bf16(tmem + kColY, al, bc, id_yo, 1);
    }
    for (int str = 0; str < (p.allblock ? 2 : 1); ++str) {
      const uint32_t col = str ? kColYN : kColYC;
      const int fs = str ? kNF : kCF, rs = str ? kNR : kCR;
      for (int ks = 0; ks < 2; ++ks) {
        const uint64_t a = sdesc(st + kOffX + fs * kTile + ks * 2048, 0, 1024, kLayoutSw128);
        const uint64_t m = sdesc(base + kOffMh + fs * 2048 + ks * 2 * kMhLbo, kMhLbo, kMhSbo, kLayoutNone);
        umma_bf16(tmem + col, a, m, id_yd, ks > 0);
      }
      if (p.active[rs]) {
        for (int ks = 0; ks < 2; ++ks) {
          const uint64_t a = sdesc(st + kOffX + rs * kTile + ks * 2048, 0, 1024, kLayoutSw128);
          const uint64_t m = sdesc(base + kOffMh + rs * 2048 + ks * 2 * kMhLbo, kMhLbo, kMhSbo, kLayoutNone);
          umma_bf16(tmem + col, a, m, id_yd, 1);
        }
      }
    }
    umma_commit(&c.bar[bYFull]);
    umma_commit(&c.bar[bEmpty0 + s]);
  }
  // Drain: every MMA issued above has completed before TMEM is released.
  umma_commit(&c.bar[bDrain]);
  (void)mbar_wait(&c.bar[bDrain], 0, p.drain_ns, nullptr);
}

// warps 2..5: q = warp & 3 is both the TMEM lane quarter and the stacking slot.
__device__ void state_group(const TcParams &p, const Ctl &c, uint8_t *sm, uint32_t base, uint32_t tmem,
                            int b, int h) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q = warp & 3;
  const int gt = threadIdx.x - 64;  // 0..127
  const int n = 32 * q + lane;      // state row owned by this thread (h^T[n][:])
  const bool act = p.active[q] != 0;
  const bool rev = q >= 2;
  float *cum = reinterpret_cast<float *>(sm + kOffCum);  // [2][4][32]
  float *dts = reinterpret_cast<float *>(sm + kOffDt);
  const int64_t H = p.H, L = p.L;
  const int64_t PN = kP * kN;

  // ---- initial state h_{-1}
  float hreg[kP];
  const float *h0 = p.h0 ? p.h0 + (static_cast<int64_t>(b) * H + h) * PN : nullptr;
#pragma unroll
  for (int pp = 0; pp < kP; ++pp) hreg[pp] = h0 ? h0[pp * kN + n] : 0.f;
  auto write_h = [&]() {
#pragma unroll
    for (int cch = 0; cch < 8; ++cch) {
      float v[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = hreg[8 * cch + i];
      store_split8(base + kOffHHi + sw128_chunk(n, cch), base + kOffHLo + sw128_chunk(n, cch), v);
    }
    fence_proxy_async_smem();
    arrive_lane0(c, bHFull);
  };
  write_h();

  const __nv_bfloat16 *dtp = act ? p.dt[q] : nullptr;
  auto load_dt = [&](int k) -> float {
    if (!act || k >= p.K) return 0.f;
    return __bfloat162float(dtp[(static_cast<int64_t>(b) * L + k * kT + lane) * H + h]);
  };
  float dt_next = load_dt(0);
  const float A2 = act ? p.A[q][h] * kLog2e : 0.f;

  for (int k = 0; k < p.K; ++k) {
    const int s = k & 1;
    const uint32_t ps = (k >> 1) & 1;
    const float dt_cur = dt_next;
    dt_next = load_dt(k + 1);
    if (!waitw(c, bFull0 + s, ps)) break;
    // ---- decays of this warp's direction (log2 units)
    if (act) {
      const float dA = dt_cur * A2;
      float v = dA;
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
    // all four directions' decays are in shared memory (bounded wait, so an
    // aborting warp can never strand the others)
    arrive_lane0(c, bAux0 + s);
    if (!waitw(c, bAux0 + s, ps)) break;
    // ---- (w o X) for the clean forward direction, split into bf16 hi/lo
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
        ld_shared_v4(base + s * kStage + kOffX + kCF * kTile + off, r0, r1, r2, r3);
        const float w = df[t] * exp2f(c31 - cf[t]);
        float v[8] = {bf16_lo_f(r0) * w, bf16_hi_f(r0) * w, bf16_lo_f(r1) * w, bf16_hi_f(r1) * w,
                      bf16_lo_f(r2) * w, bf16_hi_f(r2) * w, bf16_lo_f(r3) * w, bf16_hi_f(r3) * w};
        store_split8(base + kOffXwHi + off, base + kOffXwLo + off, v);
      }
      fence_proxy_async_smem();
      arrive_lane0(c, bXwFull);
      arrive_lane0(c, bEmpty0 + s);
    }
    // ---- masked-decay matrix M^T row s = lane for this warp's direction
    if (!waitw(c, bCbFull, k & 1)) break;
    tc_fence_after();
    {
      uint32_t cb[32];
      tmem_ld_32x32b_x32(tmem_addr(tmem, 32 * q, kColCB + 32 * q), cb);
      tmem_ld_wait();
      if (act) {
        const float *cq = cum + (s * 4 + q) * 32;
        const float cs = cq[lane];
        const float ds = dts[(s * 4 + q) * 32 + lane];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          float m[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int t = 8 * j + i;
            const bool valid = rev ? (t <= lane) : (t >= lane);
            const float e = exp2f(cq[t] - cs);
            m[i] = valid ? __uint_as_float(cb[t]) * ds * e : 0.f;
          }
          const uint32_t addr = base + kOffMh + q * 2048 + inter_mn_off(8 * j, lane, kMhSbo, kMhLbo);
          st_shared_v4(addr, pack_bf16x2(m[0], m[1]), pack_bf16x2(m[2], m[3]), pack_bf16x2(m[4], m[5]),
                       pack_bf16x2(m[6], m[7]));
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      arrive_lane0(c, bMhFull);
    }
    // ---- state update h_k = exp(cum_31) h_{k-1} + S
    if (!waitw(c, bSFull, k & 1)) break;
    tc_fence_after();
    {
      uint32_t sv[32];
      const float atot = exp2f(cum[(s * 4 + kCF) * 32 + 31]);
      tmem_ld_32x32b_x32(tmem_addr(tmem, 32 * q, kColS), sv);
      tmem_ld_wait();
#pragma unroll
      for (int pp = 0; pp < 32; ++pp) hreg[pp] = fmaf(atot, hreg[pp], __uint_as_float(sv[pp]));
      tmem_ld_32x32b_x32(tmem_addr(tmem, 32 * q, kColS + 32), sv);
      tmem_ld_wait();
#pragma unroll
      for (int pp = 0; pp < 32; ++pp) hreg[32 + pp] = fmaf(atot, hreg[32 + pp], __uint_as_float(sv[pp]));
      tc_fence_before();
      arrive_lane0(c, bSEmpty);
      if (p.states) {
        float *dst = p.states + ((static_cast<int64_t>(b) * p.K + k) * H + h) * PN + n;
#pragma unroll
        for (int pp = 0; pp < kP; ++pp) dst[pp * kN] = hreg[pp];
      }
    }
    // h operand of the next block: only after Y_off(k) has consumed h_{k-1}
    if (!waitw(c, bYFull, k & 1)) break;
    write_h();
  }
  if (p.final_state && !*c.abort) {
    float *dst = p.final_state + (static_cast<int64_t>(b) * H + h) * PN + n;
#pragma unroll
    for (int pp = 0; pp < kP; ++pp) dst[pp * kN] = hreg[pp];
  }
}

// warps 6..9: rows p = 16 q + (lane & 15), tokens t = 16 (lane >> 4) + r.
__device__ void epilogue_group(const TcParams &p, const Ctl &c, uint8_t *sm, uint32_t base, uint32_t tmem,
                               int b, int h) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q = warp & 3;
  const int prow = 16 * q + (lane & 15);
  const int tb = 16 * (lane >> 4);
  const float *cum = reinterpret_cast<const float *>(sm + kOffCum);
  const int64_t H = p.H, L = p.L;
  for (int k = 0; k < p.K; ++k) {
    const int s = k & 1;
    const uint32_t ps = (k >> 1) & 1;
    if (!waitw(c, bFull0 + s, ps)) break;
    if (!waitw(c, bAux0 + s, ps)) break;
    if (!waitw(c, bYFull, k & 1)) break;
    tc_fence_after();
    uint32_t yo[16], yon[16], yd[16], ydn[16];
    const uint32_t lq = 32 * q;
    tmem_ld_16x32bx2_x16(tmem_addr(tmem, lq, kColY), yo);
    tmem_ld_16x32bx2_x16(tmem_addr(tmem, lq, kColYC), yd);
    if (p.allblock) {
      tmem_ld_16x32bx2_x16(tmem_addr(tmem, lq, kColY + 32), yon);
      tmem_ld_16x32bx2_x16(tmem_addr(tmem, lq, kColYN), ydn);
    }
    tmem_ld_wait();
    tc_fence_before();
    arrive_lane0(c, bYEmpty);
    const uint32_t st = base + s * kStage;
    for (int str = 0; str < (p.allblock ? 2 : 1); ++str) {
      void *yout = str ? p.y_noisy : p.y_clean;
      if (!yout) continue;
      const int fs = str ? kNF : kCF, rs = str ? kNR : kCR;
      const float *cq = cum + (s * 4 + fs) * 32;
      const float Df = p.D[fs][h], Dr = p.active[rs] ? p.D[rs][h] : 0.f;
      const uint32_t *o = str ? yon : yo;
      const uint32_t *d = str ? ydn : yd;
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        const int t = tb + r;
        const uint32_t xo = sw128_off(t, prow);
        const __nv_bfloat16 *xf =
            reinterpret_cast<const __nv_bfloat16 *>(sm + (st - base) + kOffX + fs * kTile + xo);
        float y = fmaf(exp2f(cq[t]), __uint_as_float(o[r]), __uint_as_float(d[r]));
        y = fmaf(Df, __bfloat162float(*xf), y);
        if (p.active[rs]) {
          const __nv_bfloat16 *xr =
              reinterpret_cast<const __nv_bfloat16 *>(sm + (st - base) + kOffX + rs * kTile + xo);
          y = fmaf(Dr, __bfloat162float(*xr), y);
        }
        const int64_t yi = ((static_cast<int64_t>(b) * L + k * kT + t) * H + h) * kP + prow;
        if (p.out_bf16)
          reinterpret_cast<__nv_bfloat16 *>(yout)[yi] = __float2bfloat16_rn(y);
        else
          reinterpret_cast<float *>(yout)[yi] = y;
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
    mbar_init(&bars[bFull0], 1);
    mbar_init(&bars[bFull1], 1);
    mbar_init(&bars[bEmpty0], 9);
    mbar_init(&bars[bEmpty1], 9);
    mbar_init(&bars[bCbFull], 1);
    mbar_init(&bars[bMhFull], 4);
    mbar_init(&bars[bXwFull], 4);
    mbar_init(&bars[bSFull], 1);
    mbar_init(&bars[bSEmpty], 4);
    mbar_init(&bars[bHFull], 4);
    mbar_init(&bars[bYFull], 1);
    mbar_init(&bars[bYEmpty], 4);
    mbar_init(&bars[bAux0], 4);
    mbar_init(&bars[bAux1], 4);
    mbar_init(&bars[bDrain], 1);
    *abort_flag = 0;
    fence_mbar_init();
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
    if ((threadIdx.x & 31) == 0) producer(p, c, base, b, h, g);
  } else if (warp == 1) {
    if ((threadIdx.x & 31) == 0) mma_issuer(p, c, base, tmem);
  } else if (warp < 6) {
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

// 4-D bf16 tensor map over [d3][d2][d1][d0] (d0 innermost), box (64, 1, 32, 1),
// 128-byte swizzle.
bool make_map(CUtensorMap *m, const void *ptr, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t d3) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {d0, d1, d2, d3};
  cuuint64_t strides[3] = {d0 * 2, d0 * d1 * 2, d0 * d1 * d2 * 2};
  cuuint32_t box[4] = {64, 1, 32, 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(ptr), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
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

bool tc_supported(const ScanArgs &a) {
  if (!a.in_bf16 || a.P != kP || a.N != kN || a.T != kT) return false;
  if (a.Bsz <= 0 || a.L <= 0) return false;
  const DirArgs *ds[4] = {&a.cf, &a.nf, &a.cr, &a.nr};
  for (const DirArgs *d : ds)
    if (d->z) return false;
  if (a.Bsz * a.H > 0x7fffffffLL || a.L > 0x7fffffffLL) return false;
  const char *force = std::getenv("BDSCAN_FORCE_GENERIC");
  if (force && force[0] == '1') return false;
  return device_is_sm100();
}

cudaError_t launch_tc(const ScanArgs &a, cudaStream_t stream) {
  TcParams p;
  memset(&p, 0, sizeof(p));
  const bool all = a.mode == Mode::AllBlock;
  const DirArgs *ds[4] = {&a.cf, all ? &a.nf : nullptr, a.has_cr ? &a.cr : nullptr,
                          (all && a.has_nr) ? &a.nr : nullptr};
  for (int i = 0; i < 4; ++i) {
    p.active[i] = ds[i] != nullptr;
    if (!ds[i]) continue;
    const DirArgs &d = *ds[i];
    if (!make_map(&p.tx[i], d.x, kP, a.H, a.L, a.Bsz) || !make_map(&p.tb[i], d.B, kN, a.G, a.L, a.Bsz) ||
        !make_map(&p.tc[i], d.C, kN, a.G, a.L, a.Bsz))
      return cudaErrorInvalidValue;
    p.dt[i] = reinterpret_cast<const __nv_bfloat16 *>(d.dt);
    p.A[i] = d.A;
    p.D[i] = d.D;
  }
  p.Bsz = static_cast<int>(a.Bsz);
  p.L = static_cast<int>(a.L);
  p.H = static_cast<int>(a.H);
  p.G = static_cast<int>(a.G);
  p.K = static_cast<int>(a.L / kT);
  p.allblock = all ? 1 : 0;
  p.out_bf16 = a.out_bf16 ? 1 : 0;
  p.h0 = a.h0;
  p.states = a.states;
  p.final_state = a.final_state;
  p.y_clean = a.y_clean;
  p.y_noisy = all ? a.y_noisy : nullptr;
  p.status = a.status;
  p.timeout_ns = env_ns("BDSCAN_WAIT_TIMEOUT_NS", 2000000000ull);
  p.drain_ns = 1000000000ull;
  cudaError_t e = cudaFuncSetAttribute(bd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kSmemBytes));
  if (e != cudaSuccess) return e;
  bd_tc_kernel<<<static_cast<unsigned>(a.Bsz * a.H), kThreads, kSmemBytes, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace bdscan
