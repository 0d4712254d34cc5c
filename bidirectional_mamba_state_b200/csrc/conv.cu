// conv.cu -- the short depthwise convolution (+SiLU) that a Mamba-2 layer
// applies to its x, B and C channels before the scan, with the conv state of
// the block-diffusion cache ("Training Hybrid Block Diffusion Language Models
// with Partial Bidirectionality", the paragraph after eq. (14): a Mamba layer's
// cache holds the convolution state beside the scan state).  The forward
// direction is causal over the stream; the reverse direction is anti-causal
// ("Breaking the Bottleneck with DiffuApriel", section 3.2, after eq. (5)) and
// stays inside its block, like the reverse scan (first page, eq. (12)).
//
// Work is HBM-bound (4 flops per byte at most): one pass, every input row read
// once from HBM (the W-1 halo rows a tile shares with its neighbour come from
// L2), every output row written once.  A thread owns one vector of 4
// channels (8 bytes of bf16, 16 of fp32) of one tile of tokens: consecutive
// threads take consecutive vectors of the same token row, so each warp load or
// store is 256 or 512 contiguous bytes.  The taps of the thread's channels, the bias
// and the last W-1 rows stay in registers while the thread walks its tile
// (forward: oldest to newest; reverse: newest to oldest) in batches of 64
// bytes of rows whose loads are all issued before their first use.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>

#include "bdscan_internal.h"

namespace bdscan {
namespace {

constexpr int kConvThreads = 256;

struct ConvJob {
  const void *u[3];     // x, B, C inputs of this direction
  const void *halo[3];  // mode 1: the clean stream's x, B, C (rows before a block)
  void *v[3];           // outputs
  const float *w;        // [Cx][W]
  const float *bias;     // [Cx] or nullptr
  int mode;              // 0 causal over the stream, 1 causal per block from the halo stream,
                         // 2 anti-causal per block
  int tile;              // tokens per thread
  int tiles;             // ceil(L / tile)
  int write_state;       // writes state_out from the last tile (mode 0)
};

struct ConvParams {
  ConvJob job[4];
  const void *state_in;  // [B][W-1][Cx] or nullptr
  void *state_out;       // [B][W-1][Cx] or nullptr
  int64_t L;
  int Bsz, Cx, T;
  int vx, vb, nvec;  // vectors per row of x (H*P / 4) and of B or C (G*N / 4); nvec = vx + 2 vb
  int silu;
};

template <typename E>
struct Vec;

// A vector is 4 channels: 8 bytes of bf16 or 16 bytes of fp32.  (8 bf16
// channels per thread would double the taps, window and bias registers and
// halve the threads an SM can keep loading.)
template <>
struct Vec<__nv_bfloat16> {
  static constexpr int V = 4;
  using Raw = uint2;
  static __device__ __forceinline__ Raw zero() { return make_uint2(0u, 0u); }
  static __device__ __forceinline__ void unpack(const Raw &r, float (&f)[V]) {
    f[0] = __uint_as_float(r.x << 16);
    f[1] = __uint_as_float(r.x & 0xffff0000u);
    f[2] = __uint_as_float(r.y << 16);
    f[3] = __uint_as_float(r.y & 0xffff0000u);
  }
  static __device__ __forceinline__ Raw pack(const float (&f)[V]) {
    const __nv_bfloat162 lo = __floats2bfloat162_rn(f[0], f[1]);
    const __nv_bfloat162 hi = __floats2bfloat162_rn(f[2], f[3]);
    return make_uint2(*reinterpret_cast<const uint32_t *>(&lo), *reinterpret_cast<const uint32_t *>(&hi));
  }
};

template <>
struct Vec<float> {
  static constexpr int V = 4;
  using Raw = uint4;
  static __device__ __forceinline__ Raw zero() { return make_uint4(0u, 0u, 0u, 0u); }
  static __device__ __forceinline__ void unpack(const Raw &r, float (&f)[V]) {
    f[0] = __uint_as_float(r.x);
    f[1] = __uint_as_float(r.y);
    f[2] = __uint_as_float(r.z);
    f[3] = __uint_as_float(r.w);
  }
  static __device__ __forceinline__ Raw pack(const float (&f)[V]) {
    return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                      __float_as_uint(f[3]));
  }
};

// silu(v) = v / (1 + e^-v) with the hardware exponential and reciprocal
// (__expf, __fdividef: a few ulp).  The convolution does only 4 multiply-adds
// per output, so the accurate expf / IEEE division (tens of instructions each)
// would make the kernel instruction-bound instead of HBM-bound.  For v below
// about -88, e^-v overflows to inf and the quotient is -0, the limit of silu.
__device__ __forceinline__ float act(float v, int silu) {
  return silu ? __fdividef(v, 1.0f + __expf(-v)) : v;
}

// NB rows ps[0], ps[step], ... issued back to back (their loads are in flight
// together).
template <class Vt, int NB>
__device__ __forceinline__ void load_rows(typename Vt::Raw (&raw)[NB], const typename Vt::Raw *ps, int64_t step) {
#pragma unroll
  for (int k = 0; k < NB; ++k) raw[k] = __ldg(ps + k * step);
}

// NB consecutive rows (already loaded) of a causal convolution, written to
// pd[0], pd[step], ...: the window (rows before the batch, oldest first) is
// extended by the batch and its last W-1 rows kept.
template <class Vt, int W, int NB>
__device__ __forceinline__ void rows_fwd(const typename Vt::Raw (&raw)[NB], typename Vt::Raw *pd, int64_t step,
                                         const float (&w)[W][Vt::V], const float (&bias)[Vt::V],
                                         float (&win)[W > 1 ? W - 1 : 1][Vt::V], int silu) {
  constexpr int V = Vt::V;
  float uu[W - 1 + NB][V];
#pragma unroll
  for (int m = 0; m < W - 1; ++m)
#pragma unroll
    for (int c = 0; c < V; ++c) uu[m][c] = win[m][c];
#pragma unroll
  for (int k = 0; k < NB; ++k) Vt::unpack(raw[k], uu[W - 1 + k]);
#pragma unroll
  for (int k = 0; k < NB; ++k) {
    float o[V];
#pragma unroll
    for (int c = 0; c < V; ++c) {
      float acc = bias[c];
#pragma unroll
      for (int j = 0; j < W; ++j) acc = fmaf(w[j][c], uu[k + j][c], acc);
      o[c] = act(acc, silu);
    }
    pd[k * step] = Vt::pack(o);
  }
#pragma unroll
  for (int m = 0; m < W - 1; ++m)
#pragma unroll
    for (int c = 0; c < V; ++c) win[m][c] = uu[NB + m][c];
}

// NB consecutive rows (already loaded, ascending) of an anti-causal
// convolution, the window holding the W-1 rows above the batch (nearest first).
template <class Vt, int W, int NB>
__device__ __forceinline__ void rows_rev(const typename Vt::Raw (&raw)[NB], typename Vt::Raw *pd, int64_t step,
                                         const float (&w)[W][Vt::V], const float (&bias)[Vt::V],
                                         float (&win)[W > 1 ? W - 1 : 1][Vt::V], int silu) {
  constexpr int V = Vt::V;
  float uu[NB + W - 1][V];  // ascending tokens: the batch, then the window
#pragma unroll
  for (int k = 0; k < NB; ++k) Vt::unpack(raw[k], uu[k]);
#pragma unroll
  for (int m = 0; m < W - 1; ++m)
#pragma unroll
    for (int c = 0; c < V; ++c) uu[NB + m][c] = win[m][c];
#pragma unroll
  for (int k = 0; k < NB; ++k) {
    float o[V];
#pragma unroll
    for (int c = 0; c < V; ++c) {
      float acc = bias[c];
#pragma unroll
      for (int j = 0; j < W; ++j) acc = fmaf(w[j][c], uu[k + W - 1 - j][c], acc);
      o[c] = act(acc, silu);
    }
    pd[k * step] = Vt::pack(o);
  }
#pragma unroll
  for (int m = 0; m < W - 1; ++m)
#pragma unroll
    for (int c = 0; c < V; ++c) win[m][c] = uu[m][c];
}

template <typename E, int W>
__global__ void __launch_bounds__(kConvThreads, 2) bd_conv_kernel(const __grid_constant__ ConvParams p) {
  using Vt = Vec<E>;
  using Raw = typename Vt::Raw;
  constexpr int V = Vt::V;
  constexpr int WH = W > 1 ? W - 1 : 1;  // window rows (at least one, unused when W == 1)
  constexpr int NBM = sizeof(Raw) == 8 ? 8 : 4;  // rows per batch: 64 bytes of loads in flight
  // Launched as a programmatic dependent of the kernel before it on the stream:
  // wait for that kernel before touching memory, then let the next one (e.g.
  // the scan's pre-pass, which waits for us in turn) be scheduled.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const ConvJob &J = p.job[blockIdx.y];
  const int64_t item = static_cast<int64_t>(blockIdx.x) * kConvThreads + threadIdx.x;
  if (item >= static_cast<int64_t>(p.Bsz) * J.tiles * p.nvec) return;
  const int vec = static_cast<int>(item % p.nvec);
  const int64_t rest = item / p.nvec;
  const int tile = static_cast<int>(rest % J.tiles);
  const int64_t b = rest / J.tiles;

  // the tensor the vector belongs to, its column there and that tensor's row
  // length (in vectors); vec itself is the channel vector in x | B | C order
  const int part = vec < p.vx ? 0 : (vec < p.vx + p.vb ? 1 : 2);
  const int col = part == 0 ? vec : (part == 1 ? vec - p.vx : vec - p.vx - p.vb);
  const int rowv = part == 0 ? p.vx : p.vb;
  const int cvec = vec;
  const Raw *__restrict__ src = static_cast<const Raw *>(J.u[part]);
  const Raw *__restrict__ halo = static_cast<const Raw *>(J.halo[part]);
  Raw *__restrict__ dst = static_cast<Raw *>(J.v[part]);
  const Raw *st_in = static_cast<const Raw *>(p.state_in);
  Raw *st_out = static_cast<Raw *>(p.state_out);
  auto at = [&](int64_t t) { return (b * p.L + t) * rowv + col; };
  const int64_t cxv = p.nvec;  // state row length in vectors
  auto st_at = [&](int r) { return (b * (W - 1) + r) * cxv + cvec; };

  float w[W][V], bias[V];
  {
    const float4 *w4 = reinterpret_cast<const float4 *>(J.w + static_cast<int64_t>(cvec) * V * W);
    float wf[V * W];
#pragma unroll
    for (int i = 0; i < V * W / 4; ++i) {
      const float4 q = __ldg(w4 + i);
      wf[4 * i] = q.x; wf[4 * i + 1] = q.y; wf[4 * i + 2] = q.z; wf[4 * i + 3] = q.w;
    }
#pragma unroll
    for (int c = 0; c < V; ++c)
#pragma unroll
      for (int j = 0; j < W; ++j) w[j][c] = wf[c * W + j];
    if (J.bias) {
      const float4 *b4 = reinterpret_cast<const float4 *>(J.bias + static_cast<int64_t>(cvec) * V);
#pragma unroll
      for (int i = 0; i < V / 4; ++i) {
        const float4 q = __ldg(b4 + i);
        bias[4 * i] = q.x; bias[4 * i + 1] = q.y; bias[4 * i + 2] = q.z; bias[4 * i + 3] = q.w;
      }
    } else {
#pragma unroll
      for (int c = 0; c < V; ++c) bias[c] = 0.f;
    }
  }

  const int64_t t0 = static_cast<int64_t>(tile) * J.tile;
  const Raw zero = Vt::zero();
  float win[WH][V];
  const int64_t step = rowv;  // one token row, in vectors

  if (J.mode != 2) {
    // ---- causal: window = rows t-(W-1) .. t-1, oldest first
    const int64_t t1 = t0 + J.tile < p.L ? t0 + J.tile : p.L;
    const int64_t own_from = J.mode == 1 ? (t0 / p.T) * p.T : 0;
#pragma unroll
    for (int i = 0; i < W - 1; ++i) {
      const int64_t tp = t0 - (W - 1) + i;
      Raw r = zero;
      if (tp >= own_from)
        r = __ldg(src + at(tp));
      else if (tp >= 0)
        r = __ldg(halo + at(tp));
      else if (st_in)
        r = st_in[st_at(static_cast<int>(W - 1 + tp))];
      Vt::unpack(r, win[i]);
    }
    const Raw *ps = src + at(t0);
    Raw *pd = dst + at(t0);
    int64_t n = t1 - t0;
    if (n >= NBM) {
      // the next batch's loads are in flight while this batch is computed
      Raw cur[NBM];
      load_rows<Vt, NBM>(cur, ps, step);
      for (;;) {
        n -= NBM;
        ps += NBM * step;
        Raw nxt[NBM];
        if (n >= NBM) load_rows<Vt, NBM>(nxt, ps, step);
        rows_fwd<Vt, W, NBM>(cur, pd, step, w, bias, win, p.silu);
        pd += NBM * step;
        if (n < NBM) break;
#pragma unroll
        for (int k = 0; k < NBM; ++k) cur[k] = nxt[k];
      }
    }
    if (NBM > 4 && n >= 4) {
      Raw r4[4];
      load_rows<Vt, 4>(r4, ps, step);
      rows_fwd<Vt, W, 4>(r4, pd, step, w, bias, win, p.silu);
      n -= 4; ps += 4 * step; pd += 4 * step;
    }
    for (; n > 0; --n, ps += step, pd += step) {
      Raw r1[1];
      load_rows<Vt, 1>(r1, ps, step);
      rows_fwd<Vt, W, 1>(r1, pd, step, w, bias, win, p.silu);
    }
    // the window now holds the stream's last W-1 rows (exact copies of inputs
    // or of state rows, so packing them back is lossless)
    if (J.write_state && st_out && t1 == p.L) {
#pragma unroll
      for (int r = 0; r < W - 1; ++r) st_out[st_at(r)] = Vt::pack(win[r]);
    }
  } else {
    // ---- anti-causal inside the block: window = rows t+1 .. t+W-1, nearest first
    const int64_t t1 = t0 + J.tile;  // the tile divides the block
    const int64_t bend = (t0 / p.T + 1) * p.T;
#pragma unroll
    for (int i = 0; i < W - 1; ++i) {
      const int64_t tp = t1 + i;
      Vt::unpack(tp < bend ? __ldg(src + at(tp)) : zero, win[i]);
    }
    // walk down from the tile's end: each batch covers the NB rows below ps
    const Raw *ps = src + at(t1);
    Raw *pd = dst + at(t1);
    int64_t n = t1 - t0;
    if (n >= NBM) {
      Raw cur[NBM];
      ps -= NBM * step;
      load_rows<Vt, NBM>(cur, ps, step);
      for (;;) {
        n -= NBM;
        Raw nxt[NBM];
        if (n >= NBM) load_rows<Vt, NBM>(nxt, ps - NBM * step, step);
        pd -= NBM * step;
        rows_rev<Vt, W, NBM>(cur, pd, step, w, bias, win, p.silu);
        if (n < NBM) break;
        ps -= NBM * step;
#pragma unroll
        for (int k = 0; k < NBM; ++k) cur[k] = nxt[k];
      }
    }
    if (NBM > 4 && n >= 4) {
      Raw r4[4];
      ps -= 4 * step; pd -= 4 * step; n -= 4;
      load_rows<Vt, 4>(r4, ps, step);
      rows_rev<Vt, W, 4>(r4, pd, step, w, bias, win, p.silu);
    }
    for (; n > 0; --n) {
      Raw r1[1];
      ps -= step; pd -= step;
      load_rows<Vt, 1>(r1, ps, step);
      rows_rev<Vt, W, 1>(r1, pd, step, w, bias, win, p.silu);
    }
  }
}

// Programmatic dependent launch: the CTAs may be scheduled while the previous
// kernel on the stream finishes (they wait for it in the kernel).
template <typename E, int W>
cudaError_t launch_pdl(const ConvParams &p, dim3 grid, cudaStream_t stream) {
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kConvThreads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, bd_conv_kernel<E, W>, p);
  return e != cudaSuccess ? e : cudaGetLastError();
}

template <typename E>
cudaError_t launch_typed(const ConvParams &p, int W, dim3 grid, cudaStream_t stream) {
  switch (W) {
    case 1: return launch_pdl<E, 1>(p, grid, stream);
    case 2: return launch_pdl<E, 2>(p, grid, stream);
    case 3: return launch_pdl<E, 3>(p, grid, stream);
    default: return launch_pdl<E, 4>(p, grid, stream);
  }
}

// Largest power of two <= want that divides T (a tile never straddles a block).
int block_tile(int64_t T, int want) {
  int t = want;
  while (t > 1 && T % t) t >>= 1;
  return t;
}

}  // namespace

int conv_tile(const ConvArgs &a) {
  // Long tiles amortise the halo rows and the taps; short ones give the small
  // decode-size problems enough threads to fill the GPU and shorten each
  // thread's serial walk (which is what a one-block step waits for).
  const int64_t nvec = (a.H * a.P + 2 * a.G * a.N) / 4;
  int ndir = 0;
  for (int d = 0; d < 4; ++d) ndir += a.dir[d].x != nullptr;
  const int64_t enough = 148 * 2 * kConvThreads;  // two CTAs on every SM
  int t = 32;
  while (t > 4 && a.Bsz * ((a.L + t - 1) / t) * nvec * ndir < enough) t >>= 1;
  return t;
}

cudaError_t launch_conv(const ConvArgs &a, cudaStream_t stream) {
  if (a.Bsz == 0 || a.L == 0) return cudaSuccess;
  const int V = 4;
  ConvParams p{};
  p.L = a.L;
  p.Bsz = static_cast<int>(a.Bsz);
  p.Cx = static_cast<int>(a.H * a.P + 2 * a.G * a.N);
  p.T = static_cast<int>(a.T);
  p.vx = static_cast<int>(a.H * a.P / V);
  p.vb = static_cast<int>(a.G * a.N / V);
  p.nvec = p.vx + 2 * p.vb;
  p.silu = a.silu ? 1 : 0;
  p.state_in = a.state_in;
  p.state_out = a.state_out;
  // in place: one tile per (row, vector) so each thread reads its state rows
  // before it writes them
  const int want = (a.state_out && a.state_out == a.state_in) ? 32 : conv_tile(a);
  int nj = 0;
  int64_t max_items = 0;
  for (int d = 0; d < 4; ++d) {
    const ConvDirArgs &s = a.dir[d];
    if (!s.x) continue;
    ConvJob &j = p.job[nj++];
    const void *in[3] = {s.x, s.B, s.C};
    void *out[3] = {s.x_out, s.B_out, s.C_out};
    const void *halo[3] = {a.dir[0].x, a.dir[0].B, a.dir[0].C};
    for (int k = 0; k < 3; ++k) {
      j.u[k] = in[k];
      j.v[k] = out[k];
      j.halo[k] = halo[k];
    }
    j.w = s.weight;
    j.bias = s.bias;
    const bool reverse = d == 1 || d == 3;
    const bool noisy_fwd = d == 2;
    j.mode = reverse ? 2 : (noisy_fwd ? 1 : 0);
    j.tile = j.mode == 0 ? want : block_tile(a.T, want);
    j.tiles = static_cast<int>((a.L + j.tile - 1) / j.tile);
    j.write_state = d == 0 ? 1 : 0;
    const int64_t items = a.Bsz * j.tiles * p.nvec;
    if (items > max_items) max_items = items;
  }
  if (nj == 0) return cudaSuccess;
  const dim3 grid(static_cast<unsigned>((max_items + kConvThreads - 1) / kConvThreads), nj);
  return a.in_bf16 ? launch_typed<__nv_bfloat16>(p, a.W, grid, stream)
                   : launch_typed<float>(p, a.W, grid, stream);
}

}  // namespace bdscan
