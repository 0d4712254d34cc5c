// scan_seq.cu -- generic block-diffusion scan: the selective-state recurrence
// run token by token on CUDA cores.
//
// It serves every shape the library accepts (fp32 or bf16 inputs, any
// supported P/N/T, gated or not).  The tensor-core path (scan_tc.cu) takes the
// configurations it is specialised for; this kernel is the general one.
//
// Recurrence ("Training Hybrid Block Diffusion Language Models with Partial
// Bidirectionality", eq. (1), Mamba-2 scalar decay):
//   h_t = exp(dt_t A) h_{t-1} + dt_t x_t B_t^T,   y_t = h_t C_t + D x_t
// forward over the sequence with boundary states (eq. (10)), noisy blocks
// continued from the boundary state before them (eq. (11), all-block form of
// eq. (14)), block-local reverse from a zero state (eq. (12)), sum (eq. (13)).
//
// Work split: one CTA of 128 threads per (b, h, 16-row slice of P).  Warp w
// owns rows 4w..4w+3 of the slice; lane l owns state columns n = l + 32 j.
// The state slice (16 x N fp32) lives in registers for the whole sequence;
// a block's inputs are staged in shared memory 32 tokens at a time, and the
// block's outputs are summed in shared memory (fwd, then rev) before one
// coalesced store.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "bdscan_internal.h"

namespace bdscan {
namespace {

constexpr int kRows = 16;     // P rows per CTA
constexpr int kWarps = 4;     // 4 rows per warp
constexpr int kRowsPerWarp = kRows / kWarps;
constexpr int kStage = 32;    // tokens staged at once

template <bool BF16>
__device__ __forceinline__ float ld_in(const void *p, int64_t i) {
  if constexpr (BF16) {
    return __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(p)[i]);
  } else {
    return reinterpret_cast<const float *>(p)[i];
  }
}

__device__ __forceinline__ float silu(float v) { return v / (1.0f + expf(-v)); }

struct Smem {
  float *x;    // [kStage][kRows]
  float *z;    // [kStage][kRows]
  float *dt;   // [kStage]
  float *Bm;   // [kStage][N]
  float *Cm;   // [kStage][N]
  float *yc;   // [T][kRows]  clean-stream block output
  float *yn;   // [T][kRows]  noisy-stream block output
};

struct Ctx {
  int64_t b, h, g, p0;
  int64_t L, H, P, N, G, T;
};

// Stage tokens [t0, t0 + n) of one direction into shared memory.
template <bool BF16>
__device__ void stage(const DirArgs &d, const Ctx &c, int64_t t0, int n, const Smem &s) {
  const int tid = threadIdx.x;
  for (int i = tid; i < n * kRows; i += blockDim.x) {
    const int tt = i / kRows, r = i % kRows;
    const int64_t xi = ((c.b * c.L + t0 + tt) * c.H + c.h) * c.P + c.p0 + r;
    s.x[tt * kRows + r] = ld_in<BF16>(d.x, xi);
    if (d.z) s.z[tt * kRows + r] = ld_in<BF16>(d.z, xi);
  }
  for (int i = tid; i < n; i += blockDim.x) s.dt[i] = ld_in<BF16>(d.dt, (c.b * c.L + t0 + i) * c.H + c.h);
  for (int i = tid; i < n * c.N; i += blockDim.x) {
    const int tt = i / c.N, nn = i % c.N;
    const int64_t bi = ((c.b * c.L + t0 + tt) * c.G + c.g) * c.N + nn;
    s.Bm[tt * c.N + nn] = ld_in<BF16>(d.B, bi);
    s.Cm[tt * c.N + nn] = ld_in<BF16>(d.C, bi);
  }
}

// Run the recurrence over the n staged tokens, in forward or reverse order,
// on the register state st; write (ACC=false) or add (ACC=true) each token's
// output into yblk[(t_in_block)][row].
template <int NJ, bool ACC>
__device__ void run(const DirArgs &d, const Ctx &c, int n, bool reverse, int tblk0,
                    float (&st)[kRowsPerWarp][NJ], const Smem &s, float *yblk) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float A = d.A[c.h], D = d.D[c.h];
  for (int i = 0; i < n; ++i) {
    const int tt = reverse ? (n - 1 - i) : i;
    const float dt = s.dt[tt];
    const float a = expf(dt * A);
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r) {
      const int row = warp * kRowsPerWarp + r;
      const float xv = s.x[tt * kRows + row];
      const float dtx = dt * xv;
      float acc = 0.f;
#pragma unroll
      for (int j = 0; j < NJ; ++j) {
        const int nn = lane + 32 * j;
        if (nn < c.N) {
          st[r][j] = fmaf(a, st[r][j], dtx * s.Bm[tt * c.N + nn]);
          acc = fmaf(s.Cm[tt * c.N + nn], st[r][j], acc);
        }
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
      if (lane == r) {
        float yv = fmaf(D, xv, acc);
        if (d.z) yv *= silu(s.z[tt * kRows + row]);
        float &dst = yblk[(tblk0 + tt) * kRows + row];
        dst = ACC ? dst + yv : yv;
      }
    }
  }
}

template <int NJ>
__device__ __forceinline__ void zero_state(float (&st)[kRowsPerWarp][NJ]) {
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r)
#pragma unroll
    for (int j = 0; j < NJ; ++j) st[r][j] = 0.f;
}

template <int NJ>
__device__ __forceinline__ void load_state(float (&st)[kRowsPerWarp][NJ], const float *src,
                                           const Ctx &c) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r)
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
      const int nn = lane + 32 * j;
      const int64_t row = c.p0 + warp * kRowsPerWarp + r;
      st[r][j] = (src && nn < c.N) ? src[row * c.N + nn] : 0.f;
    }
}

template <int NJ>
__device__ __forceinline__ void store_state(const float (&st)[kRowsPerWarp][NJ], float *dst,
                                            const Ctx &c) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r)
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
      const int nn = lane + 32 * j;
      const int64_t row = c.p0 + warp * kRowsPerWarp + r;
      if (nn < c.N) dst[row * c.N + nn] = st[r][j];
    }
}

template <bool OUT_BF16>
__device__ void store_y(void *y, const float *yblk, const Ctx &c, int64_t k) {
  for (int i = threadIdx.x; i < c.T * kRows; i += blockDim.x) {
    const int tt = i / kRows, r = i % kRows;
    const int64_t yi = ((c.b * c.L + k * c.T + tt) * c.H + c.h) * c.P + c.p0 + r;
    if constexpr (OUT_BF16)
      reinterpret_cast<__nv_bfloat16 *>(y)[yi] = __float2bfloat16_rn(yblk[i]);
    else
      reinterpret_cast<float *>(y)[yi] = yblk[i];
  }
}

// One block's worth of a direction, staged kStage tokens at a time.
template <int NJ, bool BF16, bool ACC>
__device__ void pass(const DirArgs &d, const Ctx &c, int64_t k, bool reverse,
                     float (&st)[kRowsPerWarp][NJ], const Smem &s, float *yblk) {
  const int ts = c.T < kStage ? (int)c.T : kStage;
  const int nst = (int)(c.T / ts);
  for (int q = 0; q < nst; ++q) {
    const int sub = reverse ? (nst - 1 - q) : q;
    __syncthreads();
    stage<BF16>(d, c, k * c.T + (int64_t)sub * ts, ts, s);
    __syncthreads();
    run<NJ, ACC>(d, c, ts, reverse, sub * ts, st, s, yblk);
  }
}

template <int NJ, bool BF16, bool OUT_BF16>
__global__ void __launch_bounds__(128) bd_seq_kernel(ScanArgs a) {
  extern __shared__ float smem[];
  const int64_t slices = a.P / kRows;
  Ctx c;
  const int64_t bh = blockIdx.x / slices;
  c.p0 = (blockIdx.x % slices) * kRows;
  c.b = bh / a.H;
  c.h = bh % a.H;
  c.L = a.L; c.H = a.H; c.P = a.P; c.N = a.N; c.G = a.G; c.T = a.T;
  c.g = c.h / (a.H / a.G);
  const int ts = a.T < kStage ? (int)a.T : kStage;
  Smem s;
  s.x = smem;
  s.z = s.x + ts * kRows;
  s.dt = s.z + ts * kRows;
  s.Bm = s.dt + kStage;
  s.Cm = s.Bm + ts * a.N;
  s.yc = s.Cm + ts * a.N;
  s.yn = s.yc + a.T * kRows;

  const int64_t K = a.L / a.T;
  const int64_t sH = a.P * a.N;  // one (b, h) state
  float st[kRowsPerWarp][NJ];
  float tmp[kRowsPerWarp][NJ];
  load_state<NJ>(st, a.h0 ? a.h0 + (c.b * a.H + c.h) * sH : nullptr, c);

  for (int64_t k = 0; k < K; ++k) {
    if (a.mode == Mode::AllBlock) {
#pragma unroll
      for (int r = 0; r < kRowsPerWarp; ++r)
#pragma unroll
        for (int j = 0; j < NJ; ++j) tmp[r][j] = st[r][j];
      pass<NJ, BF16, false>(a.nf, c, k, false, tmp, s, s.yn);
    }
    pass<NJ, BF16, false>(a.cf, c, k, false, st, s, s.yc);
    if (a.states) store_state<NJ>(st, a.states + ((c.b * K + k) * a.H + c.h) * sH, c);
    if (a.has_cr) {
      zero_state<NJ>(tmp);
      pass<NJ, BF16, true>(a.cr, c, k, true, tmp, s, s.yc);
    }
    if (a.mode == Mode::AllBlock && a.has_nr) {
      zero_state<NJ>(tmp);
      pass<NJ, BF16, true>(a.nr, c, k, true, tmp, s, s.yn);
    }
    __syncthreads();
    if (a.y_clean) store_y<OUT_BF16>(a.y_clean, s.yc, c, k);
    if (a.mode == Mode::AllBlock) store_y<OUT_BF16>(a.y_noisy, s.yn, c, k);
  }
  if (a.final_state) store_state<NJ>(st, a.final_state + (c.b * a.H + c.h) * sH, c);
}

template <int NJ, bool BF16, bool OUT_BF16>
cudaError_t launch_t(const ScanArgs &a, cudaStream_t stream) {
  const int ts = a.T < kStage ? (int)a.T : kStage;
  const size_t smem = sizeof(float) * (2 * ts * kRows + kStage + 2 * ts * a.N + 2 * a.T * kRows);
  auto kern = bd_seq_kernel<NJ, BF16, OUT_BF16>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int64_t grid = a.Bsz * a.H * (a.P / kRows);
  kern<<<(unsigned)grid, 128, smem, stream>>>(a);
  return cudaGetLastError();
}

template <int NJ>
cudaError_t launch_nj(const ScanArgs &a, cudaStream_t stream) {
  if (a.in_bf16)
    return a.out_bf16 ? launch_t<NJ, true, true>(a, stream) : launch_t<NJ, true, false>(a, stream);
  return a.out_bf16 ? launch_t<NJ, false, true>(a, stream) : launch_t<NJ, false, false>(a, stream);
}

}  // namespace

cudaError_t launch_seq(const ScanArgs &a, cudaStream_t stream) {
  if (a.Bsz == 0 || a.L == 0) return cudaSuccess;
  if (a.N <= 32) return launch_nj<1>(a, stream);
  if (a.N <= 64) return launch_nj<2>(a, stream);
  if (a.N <= 128) return launch_nj<4>(a, stream);
  return launch_nj<8>(a, stream);
}

}  // namespace bdscan
