// scan_bwd.cu -- backward pass of the all-block scan: gradients of a loss
// L(y_clean, y_noisy, states) with respect to every input of every direction
// and the initial state.  Through the boundary states the noisy blocks'
// losses reach the clean prefix scan ("Training Hybrid Block Diffusion
// Language Models with Partial Bidirectionality", all-block paragraph after
// eq. (5), eq. (14)).
//
// Per 32-token block, in the processing order i = 0..T-1 of one direction
// (forward: tokens of the block left to right; reverse: right to left), with
// cum_i = sum_{v <= i} dt_v A, Lam_i = exp(cum_i), W_iu = exp(cum_i - cum_u)
// (u <= i), the block maps its start state h_s and inputs to
//   y_i = Lam_i h_s C_i + sum_{u <= i} W_iu dt_u (C_i . B_u) x_u + D x_i
//   h_e = Lam_{T-1} h_s + sum_u W_{T-1,u} dt_u x_u B_u^T
// (eq. (1) unrolled over the block).  Given dy_i and dh_e = dL/dh_e:
//   dx_u = D dy_u + dt_u sum_{i>=u} W_iu (C_i.B_u) dy_i + dt_u W_{T-1,u} dh_e B_u
//   dC_i = Lam_i dy_i^T h_s + sum_{u<=i} W_iu dt_u (dy_i.x_u) B_u
//   dB_u = dt_u sum_{i>=u} W_iu (dy_i.x_u) C_i + dt_u W_{T-1,u} x_u^T dh_e
//   dh_s = Lam_{T-1} dh_e + sum_i Lam_i dy_i C_i^T
//   dL/dcum_i = Lam_i dy_i.(h_s C_i) + sum_{u<=i} W_iu dt_u (C_i.B_u)(dy_i.x_u)
//             - sum_{i'>=i} W_i'i dt_i (C_i'.B_i)(dy_i'.x_i)
//             + [i = T-1] <dh_e, h_e> - dt_i W_{T-1,i} x_i.(dh_e B_i)
//   ddt_v = (explicit dt_v terms) + A sum_{i>=v} dL/dcum_i,
//   dA   += sum_v dt_v sum_{i>=v} dL/dcum_i,   dD += sum_i dy_i . x_i.
// The clean forward stream chains the blocks: dh_e of block k is dL/dstates[k]
// (given) plus dh_s of clean block k+1 plus dh_s of noisy block k+1 (which
// starts from states[k]); dh_s of clean block 0 and of noisy block 0 is dh0.
//
// One CTA of 512 threads per (b, h) walks the forward chain's blocks (clean
// and noisy) from last to first; the reverse directions' blocks, which carry
// nothing, run in CTAs of their own after those, a range of blocks each.  All
// block quantities live in shared memory (with transposed copies where the
// threads run over tokens), the products are register-tiled (TM x 4 per
// thread), fp32 arithmetic on CUDA cores.  dB and dC of a group and dA, dD of
// a head are sums over heads / batch rows (and reverse ranges): each CTA
// writes its own partials to the workspace and a second kernel sums them in a
// fixed order, so the result is deterministic.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <type_traits>

#include "bdscan_internal.h"

namespace bdscan {
namespace {

constexpr int kBwdThreads = 512;
// The reverse directions start every block from a zero state and take no
// end-state gradient, so their blocks depend on nothing carried: they run in
// CTAs of their own, kRevSplit per (b, h), each over a contiguous range of
// blocks, after the (b, h) CTAs of the forward chain.  The short pieces fill
// the SMs that the forward chains' last wave leaves idle.
constexpr int kRevSplit = 8;

struct BwdDir {
  const void *x, *dt, *B, *C;
  const float *A, *D;
  float *dx, *ddt;   // [B][L][H][P], [B][L][H]
  float *pB, *pC;    // partials [B][L][H][N]
  float *pA, *pD;    // partials [B][H]
};

struct BwdParams {
  BwdDir dir[4];     // clean fwd, clean rev, noisy fwd, noisy rev
  int active[4];
  int Bsz, L, H, P, N, G, T, K;
  int in_bf16, dy_bf16;
  int rev_split;         // reverse-direction CTAs per (b, h) (0: the chain CTA runs them)
  const float *h0;       // [B][H][P][N] or null
  const float *states;   // [B][K][H][P][N] (forward output)
  const void *dy_clean;  // [B][L][H][P] or null
  const void *dy_noisy;  // [B][L][H][P]
  const float *dstates;  // [B][K][H][P][N] or null
  float *dh0;            // [B][H][P][N] or null
};

__device__ __forceinline__ float ldv(const void *p, int64_t i, int bf16) {
  return bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(p)[i])
              : reinterpret_cast<const float *>(p)[i];
}

struct BwdSmem {
  float *x, *dy, *Bm, *Cm;  // row-major [T][P], [T][P], [T][N], [T][N]
  float *xt, *dyt;          // transposed [P][T]
  float *Bt, *Ct;           // transposed [N][T]
  float *dt, *cum, *lam, *r;  // [T]; r_u = Lam_{T-1} / Lam_u
  float *S, *expl, *red;    // [T], [T], [kBwdThreads]
  float *WCB, *YX, *G2;     // [T][T]: W o (C B^T), dy x^T, W o (dy x^T)
  float *Q;                 // [T][T + 1]: W o (C B^T) o (dy x^T), padded rows
  float *hsCt, *dhBt;       // [P][T + 1]: (h_s C^T)^T, (dh_e B^T)^T, rows padded so that a
                            // warp reading one column over 32 rows meets 32 banks
  float *hs, *carry;        // [P][N + 4]: rows padded so that rows p, p+1, ... fall into different banks
};

// Eight bf16 values (one 16-byte load) as floats.
__device__ __forceinline__ void unpack8(const uint4 &v, float *o) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    o[2 * i] = __uint_as_float(w[i] << 16);
    o[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

// Sum over the CTA in a fixed order (a shuffle tree per warp, then the warp
// sums in warp order): deterministic, two barriers.
__device__ float block_sum(float v, float *red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float r = 0.f;
#pragma unroll
  for (int w = 0; w < kBwdThreads / 32; ++w) r += red[w];
  __syncthreads();
  return r;
}

// W consecutive floats from an address aligned to W floats (W = 2 or 4)
template <int W>
__device__ __forceinline__ void load_row(const float *p, float *a) {
  if constexpr (W == 4) {
    const float4 v = *reinterpret_cast<const float4 *>(p);
    a[0] = v.x; a[1] = v.y; a[2] = v.z; a[3] = v.w;
  } else if constexpr (W == 2) {
    const float2 v = *reinterpret_cast<const float2 *>(p);
    a[0] = v.x; a[1] = v.y;
  } else {
#pragma unroll
    for (int i = 0; i < W; ++i) a[i] = p[i];
  }
}

// Register-tiled product over shared-memory operands: for every TM x 4 output
// tile (m0.., n0..) of an M x Nn result (TM chosen per product by timing:
// taller tiles need fewer shared-memory loads per FMA but leave threads idle),
//   acc[i][j] = sum_k a1(m0+i, k) B1[k][n0+j]  (+ sum_k a2(m0+i, k) B2[k][n0+j])
// with a(m, k) = A[m am + k ak] (times ks1[k], resp. ms2[m], when given) and
// B rows contiguous in n (16-byte loads).  A threads of a warp share m0, so A
// loads are broadcasts.  epi(m0, n0, acc) consumes the tile.  Threads lo ..
// lo + cnt - 1 take the tiles (two products of a phase run side by side on
// the two halves of the CTA).
template <int TM, class Epi>
__device__ __forceinline__ void sgemm(int lo, int cnt, int M, int Nn, int K1, const float *A1, int am1, int ak1,
                                      const float *ks1, const float *B1, int ldb1, int K2, const float *A2,
                                      int am2, int ak2, const float *ms2, const float *B2, int ldb2, Epi epi) {
  const int nt = Nn >> 2;
  const int tiles = (M / TM) * nt;
  const int me = static_cast<int>(threadIdx.x) - lo;
  if (me < 0 || me >= cnt) return;
  for (int t = me; t < tiles; t += cnt) {
    const int m0 = (t / nt) * TM, n0 = (t % nt) << 2;
    float acc[TM][4];
#pragma unroll
    for (int i = 0; i < TM; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
    // a1(m0.., k) is contiguous in m when am1 = 1 (one vector load per k) and
    // contiguous in k when ak1 = 1 (one 16-byte load per row and four k)
    constexpr int VW = TM >= 4 ? 4 : TM;
    const uintptr_t a_at = reinterpret_cast<uintptr_t>(A1);  // m0 is a multiple of TM
    const int mode = (TM % VW == 0 && VW > 1 && am1 == 1 &&
                      ((a_at | static_cast<uintptr_t>(ak1) * sizeof(float)) & (VW * sizeof(float) - 1)) == 0)
                         ? 1
                     : (ak1 == 1 && (K1 & 3) == 0 &&
                        ((a_at | static_cast<uintptr_t>(am1) * sizeof(float)) & (4 * sizeof(float) - 1)) == 0)
                         ? 2
                         : 0;
    auto k1_loop = [&](auto md) {
      constexpr int kMode = decltype(md)::value;
      if constexpr (kMode == 2) {
        for (int k = 0; k < K1; k += 4) {
          float4 a4[TM];
#pragma unroll
          for (int i = 0; i < TM; ++i) a4[i] = *reinterpret_cast<const float4 *>(A1 + (m0 + i) * am1 + k);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const float4 bv = *reinterpret_cast<const float4 *>(B1 + (k + kk) * ldb1 + n0);
            const float sk = ks1 ? ks1[k + kk] : 1.f;
#pragma unroll
            for (int i = 0; i < TM; ++i) {
              const float ai = (kk == 0 ? a4[i].x : kk == 1 ? a4[i].y : kk == 2 ? a4[i].z : a4[i].w) * sk;
              acc[i][0] = fmaf(ai, bv.x, acc[i][0]);
              acc[i][1] = fmaf(ai, bv.y, acc[i][1]);
              acc[i][2] = fmaf(ai, bv.z, acc[i][2]);
              acc[i][3] = fmaf(ai, bv.w, acc[i][3]);
            }
          }
        }
      } else {
        for (int k = 0; k < K1; ++k) {
          const float4 bv = *reinterpret_cast<const float4 *>(B1 + k * ldb1 + n0);
          const float sk = ks1 ? ks1[k] : 1.f;
          float a[TM];
          if constexpr (kMode == 1) {
#pragma unroll
            for (int i = 0; i < TM; i += VW) load_row<VW>(A1 + m0 + i + k * ak1, a + i);
          } else {
#pragma unroll
            for (int i = 0; i < TM; ++i) a[i] = A1[(m0 + i) * am1 + k * ak1];
          }
#pragma unroll
          for (int i = 0; i < TM; ++i) {
            const float ai = a[i] * sk;
            acc[i][0] = fmaf(ai, bv.x, acc[i][0]);
            acc[i][1] = fmaf(ai, bv.y, acc[i][1]);
            acc[i][2] = fmaf(ai, bv.z, acc[i][2]);
            acc[i][3] = fmaf(ai, bv.w, acc[i][3]);
          }
        }
      }
    };
    if (mode == 1)
      k1_loop(std::integral_constant<int, 1>{});
    else if (mode == 2)
      k1_loop(std::integral_constant<int, 2>{});
    else
      k1_loop(std::integral_constant<int, 0>{});
    if (A2) {
      float sm2[TM];
#pragma unroll
      for (int i = 0; i < TM; ++i) sm2[i] = ms2 ? ms2[m0 + i] : 1.f;
      int k = 0;
      // rows contiguous in k: 16-byte loads, four k at a time
      if (ak2 == 1 && ((reinterpret_cast<uintptr_t>(A2) | static_cast<uintptr_t>(am2) * sizeof(float)) &
                       (4 * sizeof(float) - 1)) == 0) {
        for (; k + 4 <= K2; k += 4) {
          float4 a4[TM];
#pragma unroll
          for (int i = 0; i < TM; ++i) a4[i] = *reinterpret_cast<const float4 *>(A2 + (m0 + i) * am2 + k);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const float4 bv = *reinterpret_cast<const float4 *>(B2 + (k + kk) * ldb2 + n0);
#pragma unroll
            for (int i = 0; i < TM; ++i) {
              const float a = (kk == 0 ? a4[i].x : kk == 1 ? a4[i].y : kk == 2 ? a4[i].z : a4[i].w) * sm2[i];
              acc[i][0] = fmaf(a, bv.x, acc[i][0]);
              acc[i][1] = fmaf(a, bv.y, acc[i][1]);
              acc[i][2] = fmaf(a, bv.z, acc[i][2]);
              acc[i][3] = fmaf(a, bv.w, acc[i][3]);
            }
          }
        }
      }
      for (; k < K2; ++k) {
        const float4 bv = *reinterpret_cast<const float4 *>(B2 + k * ldb2 + n0);
#pragma unroll
        for (int i = 0; i < TM; ++i) {
          const float a = A2[(m0 + i) * am2 + k * ak2] * sm2[i];
          acc[i][0] = fmaf(a, bv.x, acc[i][0]);
          acc[i][1] = fmaf(a, bv.y, acc[i][1]);
          acc[i][2] = fmaf(a, bv.z, acc[i][2]);
          acc[i][3] = fmaf(a, bv.w, acc[i][3]);
        }
      }
    }
    epi(m0, n0, acc);
  }
}

// One block of one direction.  kind: 0 clean fwd (h_s, dh_e = carry, h_e =
// states[k]; carry <- dh_s), 2 noisy fwd (h_s, no dh_e; carry += dh_s),
// 1 / 3 reverse (zero start, no dh_e).  Accumulates this CTA's dA, dD.
__device__ void bwd_block(const BwdParams &p, const BwdSmem &s, int kind, int b, int h, int k, float &accA,
                          float &accD) {
  const BwdDir &d = p.dir[kind];
  const int T = p.T, P = p.P, N = p.N, H = p.H, L = p.L, G = p.G, K = p.K;
  const int NS = N + 4;  // row stride of hs and carry
  const int g = h / (H / G);
  const int tid = threadIdx.x;
  const bool rev = kind == 1 || kind == 3;
  const bool has_hs = !rev && (k > 0 || p.h0 != nullptr);
  const bool has_dhe = kind == 0;
  const void *dy = (kind < 2) ? p.dy_clean : p.dy_noisy;
  const float A = d.A[h], Dh = d.D[h];
  const int64_t PN = static_cast<int64_t>(P) * N;
  auto tok = [&](int i) { return k * T + (rev ? T - 1 - i : i); };
  const float *nul = nullptr;

  // ---- inputs of the block in processing order (row-major and transposed copies);
  //      the loops are unrolled so that each thread has several loads in flight
  //      before their stores wait for them; bf16 rows whose lengths are
  //      multiples of 8 are read 16 bytes at a time
  // (the 16-byte path also forms this thread's part of sum dy . x, the dD term)
  float pd_part = 0.f;
  const bool vec = p.in_bf16 && (P & 7) == 0 && (N & 7) == 0;
  if (vec) {
    const int cx = P >> 3, cn = N >> 3;
    const __nv_bfloat16 *xb = static_cast<const __nv_bfloat16 *>(d.x);
#pragma unroll 2
    for (int e = tid; e < T * cx; e += kBwdThreads) {
      const int i = e / cx, c8 = (e - i * cx) << 3;
      const int64_t xi = ((static_cast<int64_t>(b) * L + tok(i)) * H + h) * P + c8;
      float xv[8], dv[8];
      unpack8(*reinterpret_cast<const uint4 *>(xb + xi), xv);
      if (!dy) {
#pragma unroll
        for (int j = 0; j < 8; ++j) dv[j] = 0.f;
      } else if (p.dy_bf16) {
        unpack8(*reinterpret_cast<const uint4 *>(static_cast<const __nv_bfloat16 *>(dy) + xi), dv);
      } else {
        const float4 *src = reinterpret_cast<const float4 *>(static_cast<const float *>(dy) + xi);
        const float4 v0 = src[0], v1 = src[1];
        dv[0] = v0.x; dv[1] = v0.y; dv[2] = v0.z; dv[3] = v0.w;
        dv[4] = v1.x; dv[5] = v1.y; dv[6] = v1.z; dv[7] = v1.w;
      }
      *reinterpret_cast<float4 *>(s.x + i * P + c8) = make_float4(xv[0], xv[1], xv[2], xv[3]);
      *reinterpret_cast<float4 *>(s.x + i * P + c8 + 4) = make_float4(xv[4], xv[5], xv[6], xv[7]);
      *reinterpret_cast<float4 *>(s.dy + i * P + c8) = make_float4(dv[0], dv[1], dv[2], dv[3]);
      *reinterpret_cast<float4 *>(s.dy + i * P + c8 + 4) = make_float4(dv[4], dv[5], dv[6], dv[7]);
#pragma unroll
      for (int j = 0; j < 8; ++j) pd_part = fmaf(dv[j], xv[j], pd_part);
    }
    const __nv_bfloat16 *Bb = static_cast<const __nv_bfloat16 *>(d.B), *Cb = static_cast<const __nv_bfloat16 *>(d.C);
#pragma unroll 2
    for (int e = tid; e < T * cn; e += kBwdThreads) {
      const int i = e / cn, c8 = (e - i * cn) << 3;
      const int64_t bi = ((static_cast<int64_t>(b) * L + tok(i)) * G + g) * N + c8;
      const uint4 vb = *reinterpret_cast<const uint4 *>(Bb + bi), vc = *reinterpret_cast<const uint4 *>(Cb + bi);
      unpack8(vb, s.Bm + i * N + c8);
      unpack8(vc, s.Cm + i * N + c8);
    }
  } else {
#pragma unroll 4
    for (int e = tid; e < T * P; e += kBwdThreads) {
      const int i = e / P, pp = e % P;
      const int64_t xi = ((static_cast<int64_t>(b) * L + tok(i)) * H + h) * P + pp;
      s.x[e] = ldv(d.x, xi, p.in_bf16);
      s.dy[e] = dy ? ldv(dy, xi, p.dy_bf16) : 0.f;
    }
#pragma unroll 8
    for (int e = tid; e < T * N; e += kBwdThreads) {
      const int i = e / N, n = e % N;
      const int64_t bi = ((static_cast<int64_t>(b) * L + tok(i)) * G + g) * N + n;
      s.Bm[e] = ldv(d.B, bi, p.in_bf16);
      s.Cm[e] = ldv(d.C, bi, p.in_bf16);
    }
  }
  for (int i = tid; i < T; i += kBwdThreads)
    s.dt[i] = ldv(d.dt, (static_cast<int64_t>(b) * L + tok(i)) * H + h, p.in_bf16);
  // (the noisy block starts from the clean stream's state before it, which
  // the clean block of the same k, processed just before, left in place)
  if (has_hs && kind != 2) {
    const float *src = k > 0 ? p.states + ((static_cast<int64_t>(b) * K + (k - 1)) * H + h) * PN
                             : p.h0 + (static_cast<int64_t>(b) * H + h) * PN;
    if ((N & 3) == 0) {
      const int cn4 = N >> 2;
#pragma unroll 4
      for (int e = tid; e < static_cast<int>(PN >> 2); e += kBwdThreads) {
        const int row = e / cn4, c4 = (e - row * cn4) << 2;
        *reinterpret_cast<float4 *>(s.hs + row * NS + c4) = reinterpret_cast<const float4 *>(src)[e];
      }
    } else {
#pragma unroll 8
      for (int64_t e = tid; e < PN; e += kBwdThreads) s.hs[(e / N) * NS + e % N] = src[e];
    }
  }
  // this thread's part of <dh_e, h_e> (the clean forward stream): the end
  // state's loads go out with the inputs', and so do those of the given
  // dL/dstates[k], which completes the carried gradient dh_e in shared memory
  // (below the last block; the last block's was the carry's initial value)
  float he_part = 0.f;
  if (has_dhe) {
    const float *he = p.states + ((static_cast<int64_t>(b) * K + k) * H + h) * PN;
    const float *ds = p.dstates && k + 1 < K ? p.dstates + ((static_cast<int64_t>(b) * K + k) * H + h) * PN : nullptr;
    if ((N & 3) == 0) {
      const int cn4 = N >> 2;
#pragma unroll 4
      for (int e = tid; e < static_cast<int>(PN >> 2); e += kBwdThreads) {
        const int row = e / cn4, c4 = (e - row * cn4) << 2;
        const float4 hv = reinterpret_cast<const float4 *>(he)[e];
        float4 *cp = reinterpret_cast<float4 *>(s.carry + row * NS + c4);
        float4 cv = *cp;
        if (ds) {
          const float4 dv = reinterpret_cast<const float4 *>(ds)[e];
          cv.x += dv.x; cv.y += dv.y; cv.z += dv.z; cv.w += dv.w;
          *cp = cv;
        }
        he_part += hv.x * cv.x + hv.y * cv.y + hv.z * cv.z + hv.w * cv.w;
      }
    } else {
#pragma unroll 8
      for (int64_t e = tid; e < PN; e += kBwdThreads) {
        float &c = s.carry[(e / N) * NS + e % N];
        if (ds) c += ds[e];
        he_part += c * he[e];
      }
    }
  }
  __syncthreads();
  // Transposed copies, skewed: consecutive threads take consecutive columns
  // and rotated rows (i = (j + column) mod T), so that neither the row-major
  // reads nor the transposed writes of a warp fall into one shared-memory bank
  // (with power-of-two sizes the index arithmetic is shifts and masks).
  if (((P & (P - 1)) | (N & (N - 1)) | (T & (T - 1))) == 0) {
    const int lp = __ffs(P) - 1, ln = __ffs(N) - 1;
#pragma unroll 4
    for (int e = tid; e < T * P; e += kBwdThreads) {
      const int pp = e & (P - 1), i = ((e >> lp) + pp) & (T - 1);
      s.xt[pp * T + i] = s.x[i * P + pp];
      s.dyt[pp * T + i] = s.dy[i * P + pp];
    }
#pragma unroll 4
    for (int e = tid; e < T * N; e += kBwdThreads) {
      const int n = e & (N - 1), i = ((e >> ln) + n) & (T - 1);
      s.Bt[n * T + i] = s.Bm[i * N + n];
      s.Ct[n * T + i] = s.Cm[i * N + n];
    }
  } else {
    for (int e = tid; e < T * P; e += kBwdThreads) {
      const int pp = e % P, i = (e / P + pp) % T;
      s.xt[pp * T + i] = s.x[i * P + pp];
      s.dyt[pp * T + i] = s.dy[i * P + pp];
    }
    for (int e = tid; e < T * N; e += kBwdThreads) {
      const int n = e % N, i = (e / N + n) % T;
      s.Bt[n * T + i] = s.Bm[i * N + n];
      s.Ct[n * T + i] = s.Cm[i * N + n];
    }
  }
  // cumulative decays: a warp prefix scan over 32-token chunks (lane order
  // within a chunk, chunks in order), then Lam and r in parallel
  if (tid < 32) {
    float carry = 0.f;
    for (int i0 = 0; i0 < T; i0 += 32) {
      const int i = i0 + tid;
      float v = i < T ? s.dt[i] * A : 0.f;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float u = __shfl_up_sync(0xffffffffu, v, o);
        if (tid >= o) v += u;
      }
      v += carry;
      if (i < T) {
        s.cum[i] = v;
        s.lam[i] = expf(v);
      }
      carry = __shfl_sync(0xffffffffu, v, 31);  // = cum of the chunk's last token (padding adds 0)
    }
    __syncwarp();
    for (int i = tid; i < T; i += 32) s.r[i] = expf(carry - s.cum[i]);
  }
  __syncthreads();

  // ---- Gram matrices C B^T and dy x^T and the products with the start state
  //      and the end-state gradient, side by side on the four quarters of the
  //      CTA (each has a tile per thread of its quarter)
  constexpr int kHalf = kBwdThreads / 2, kQuarter = kBwdThreads / 4;
  sgemm<2>(0, kQuarter, T, T, N, s.Ct, 1, T, nul, s.Bt, T, 0, nullptr, 0, 0, nul, nullptr, 0,
        [&](int m0, int n0, auto &acc) {
          constexpr int R = sizeof(acc) / sizeof(acc[0]);
          for (int i = 0; i < R; ++i)
            *reinterpret_cast<float4 *>(s.WCB + (m0 + i) * T + n0) = make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
        });
  sgemm<2>(kQuarter, kQuarter, T, T, P, s.dyt, 1, T, nul, s.xt, T, 0, nullptr, 0, 0, nul, nullptr, 0,
        [&](int m0, int n0, auto &acc) {
          constexpr int R = sizeof(acc) / sizeof(acc[0]);
          for (int i = 0; i < R; ++i)
            *reinterpret_cast<float4 *>(s.YX + (m0 + i) * T + n0) = make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
        });
  if (has_hs)
    sgemm<4>(2 * kQuarter, kQuarter, P, T, N, s.hs, NS, 1, nul, s.Ct, T, 0, nullptr, 0, 0, nul, nullptr, 0,
          [&](int m0, int n0, auto &acc) {
          constexpr int R = sizeof(acc) / sizeof(acc[0]);
            for (int i = 0; i < R; ++i)
              for (int jj = 0; jj < 4; ++jj) s.hsCt[(m0 + i) * (T + 1) + n0 + jj] = acc[i][jj];
          });
  if (has_dhe)
    sgemm<4>(3 * kQuarter, kQuarter, P, T, N, s.carry, NS, 1, nul, s.Bt, T, 0, nullptr, 0, 0, nul, nullptr, 0,
          [&](int m0, int n0, auto &acc) {
          constexpr int R = sizeof(acc) / sizeof(acc[0]);
            for (int i = 0; i < R; ++i)
              for (int jj = 0; jj < 4; ++jj) s.dhBt[(m0 + i) * (T + 1) + n0 + jj] = acc[i][jj];
          });
  float he_dot = 0.f;
  if (has_dhe) he_dot = block_sum(he_part, s.red);
  __syncthreads();
  // ---- decay-weighted matrices (W_iu = exp(cum_i - cum_u), u <= i)
  for (int e = tid; e < T * T; e += kBwdThreads) {
    const int i = e / T, u = e % T;
    const float w = u <= i ? expf(s.cum[i] - s.cum[u]) : 0.f;
    const float cb = s.WCB[e], yx = s.YX[e];
    s.WCB[e] = w * cb;
    s.G2[e] = w * yx;
    s.Q[i * (T + 1) + u] = w * cb * yx;
  }
  __syncthreads();
  const float lame = s.lam[T - 1];

  // ---- token gradients
  // dx_u = D dy_u + dt_u sum_i WCB[i][u] dy_i (+ dt_u r_u dh_e B_u)
  sgemm<2>(0, kHalf, T, P, T, s.WCB, 1, T, nul, s.dy, P, 0, nullptr, 0, 0, nul, nullptr, 0,
        [&](int m0, int n0, auto &acc) {
          constexpr int R = sizeof(acc) / sizeof(acc[0]);
          for (int i = 0; i < R; ++i) {
            const int u = m0 + i;
            float v[4];
            for (int j = 0; j < 4; ++j) {
              v[j] = Dh * s.dy[u * P + n0 + j] + s.dt[u] * acc[i][j];
              if (has_dhe) v[j] += s.dt[u] * s.r[u] * s.dhBt[(n0 + j) * (T + 1) + u];
            }
            *reinterpret_cast<float4 *>(d.dx + ((static_cast<int64_t>(b) * L + tok(u)) * H + h) * P + n0) =
                make_float4(v[0], v[1], v[2], v[3]);
          }
        });
  // dC_i = sum_u G2[i][u] dt_u B_u (+ Lam_i dy_i^T h_s)
  sgemm<4>(0, kHalf, T, N, T, s.G2, T, 1, s.dt, s.Bm, N, has_hs ? P : 0, has_hs ? s.dy : nullptr, P, 1, s.lam, s.hs, NS,
        [&](int m0, int n0, auto &acc) {
          constexpr int R = sizeof(acc) / sizeof(acc[0]);
          for (int i = 0; i < R; ++i)
            *reinterpret_cast<float4 *>(d.pC + ((static_cast<int64_t>(b) * L + tok(m0 + i)) * H + h) * N + n0) =
                make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
        });
  // dB_u = dt_u (sum_i G2[i][u] C_i (+ r_u x_u^T dh_e))
  sgemm<4>(kHalf, kHalf, T, N, T, s.G2, 1, T, nul, s.Cm, N, has_dhe ? P : 0, has_dhe ? s.x : nullptr, P, 1, s.r, s.carry, NS,
        [&](int m0, int n0, auto &acc) {
          constexpr int R = sizeof(acc) / sizeof(acc[0]);
          for (int i = 0; i < R; ++i) {
            const float du = s.dt[m0 + i];
            *reinterpret_cast<float4 *>(d.pB + ((static_cast<int64_t>(b) * L + tok(m0 + i)) * H + h) * N + n0) =
                make_float4(du * acc[i][0], du * acc[i][1], du * acc[i][2], du * acc[i][3]);
          }
        });
  // dL/dcum and the explicit dt terms (the second half of the CTA, after dB):
  // one warp per token, its lanes over the sums' terms, the lanes' parts
  // added in a fixed shuffle order
  if (tid >= kHalf) {
    const int warp = (tid - kHalf) >> 5, lane = tid & 31;
    for (int i = warp; i < T; i += kHalf / 32) {
      float sa = 0.f, xd = 0.f, num = 0.f, den = 0.f;
      for (int q = lane; q < P; q += 32) {
        if (has_hs) sa += s.dy[i * P + q] * s.hsCt[q * (T + 1) + i];
        if (has_dhe) xd += s.x[i * P + q] * s.dhBt[q * (T + 1) + i];
      }
      for (int u = lane; u <= i; u += 32) num += s.Q[i * (T + 1) + u] * s.dt[u];
      for (int i2 = i + lane; i2 < T; i2 += 32) den += s.Q[i2 * (T + 1) + i];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        sa += __shfl_xor_sync(0xffffffffu, sa, o);
        xd += __shfl_xor_sync(0xffffffffu, xd, o);
        num += __shfl_xor_sync(0xffffffffu, num, o);
        den += __shfl_xor_sync(0xffffffffu, den, o);
      }
      if (lane == 0) {
        float Si = sa * s.lam[i] + num - s.dt[i] * den;
        float ex = den;
        if (has_dhe) {
          Si -= s.dt[i] * s.r[i] * xd;
          ex += s.r[i] * xd;
          if (i == T - 1) Si += he_dot;
        }
        s.S[i] = Si;
        s.expl[i] = ex;
      }
    }
  }
  __syncthreads();
  float pa = 0.f, pd = 0.f;
  // suffix sums of dL/dcum: a warp scan over 32-token chunks from the block's
  // end (lane 0 = the chunk's last token); the dA partial is summed in a fixed
  // shuffle order
  if (tid < 32) {
    float carry = 0.f, pacc = 0.f;
    for (int i1 = T; i1 > 0; i1 -= 32) {
      const int v = i1 - 1 - tid;
      float x = v >= 0 ? s.S[v] : 0.f;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float u = __shfl_up_sync(0xffffffffu, x, o);
        if (tid >= o) x += u;
      }
      x += carry;
      if (v >= 0) {
        d.ddt[(static_cast<int64_t>(b) * L + tok(v)) * H + h] = s.expl[v] + A * x;
        pacc = fmaf(s.dt[v], x, pacc);
      }
      carry = __shfl_sync(0xffffffffu, x, 31);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) pacc += __shfl_xor_sync(0xffffffffu, pacc, o);
    pa = pacc;
  }
  if (vec)
    pd = pd_part;
  else
    for (int e = tid; e < T * P; e += kBwdThreads) pd += s.dy[e] * s.x[e];
  pd = block_sum(pd, s.red);
  if (tid == 0) {
    accA += pa;
    accD += pd;
  }
  // ---- gradient of the start state: dh_s = Lam_e dh_e + sum_i Lam_i dy_i C_i^T
  if (!rev)
    sgemm<4>(0, kBwdThreads, P, N, T, s.dy, 1, P, s.lam, s.Cm, N, 0, nullptr, 0, 0, nul, nullptr, 0,
          [&](int m0, int n0, auto &acc) {
          constexpr int R = sizeof(acc) / sizeof(acc[0]);
            for (int i = 0; i < R; ++i) {
              float4 *cp = reinterpret_cast<float4 *>(s.carry + (m0 + i) * NS + n0);
              float4 c = *cp;
              if (kind == 0) {
                c.x *= lame; c.y *= lame; c.z *= lame; c.w *= lame;
              }
              c.x += acc[i][0]; c.y += acc[i][1]; c.z += acc[i][2]; c.w += acc[i][3];
              *cp = c;
            }
          });
  __syncthreads();
}

__global__ void __launch_bounds__(kBwdThreads) bd_bwd_kernel(const __grid_constant__ BwdParams p) {
  extern __shared__ float sm[];
  const int T = p.T, P = p.P, N = p.N, K = p.K, H = p.H;
  const int64_t PN = static_cast<int64_t>(P) * N;
  BwdSmem s;
  float *q = sm;
  s.x = q; q += T * P;
  s.dy = q; q += T * P;
  s.Bm = q; q += T * N;
  s.Cm = q; q += T * N;
  s.xt = q; q += T * P;
  s.dyt = q; q += T * P;
  s.Bt = q; q += T * N;
  s.Ct = q; q += T * N;
  s.dt = q; q += T;
  s.cum = q; q += T;
  s.lam = q; q += T;
  s.r = q; q += T;
  s.S = q; q += T;
  s.expl = q; q += T;
  s.red = q; q += kBwdThreads;
  s.WCB = q; q += T * T;
  s.YX = q; q += T * T;
  s.G2 = q; q += T * T;
  s.Q = q; q += T * (T + 1);  // (a multiple of 4 floats: the buffers after it stay 16-byte aligned)
  const int PTS = (P * (T + 1) + 3) & ~3;  // padded [P][T + 1], a multiple of 4 floats
  s.hsCt = q; q += PTS;
  s.dhBt = q; q += PTS;
  const int NS = N + 4;  // padded row stride of hs and carry
  s.hs = q; q += static_cast<int64_t>(P) * NS;
  s.carry = q;
  const int BH = p.Bsz * H;
  if (static_cast<int>(blockIdx.x) >= BH) {
    // a piece of the reverse directions: blocks k0 .. k1 - 1 of one (b, h);
    // its dA, dD partials go to row r of the direction's [rev_split][B][H]
    const int idx = static_cast<int>(blockIdx.x) - BH, r = idx / BH, bh = idx % BH;
    const int b = bh / H, h = bh % H;
    const int k0 = r * K / p.rev_split, k1 = (r + 1) * K / p.rev_split;
    float accA[4] = {0.f, 0.f, 0.f, 0.f}, accD[4] = {0.f, 0.f, 0.f, 0.f};
    for (int k = k1 - 1; k >= k0; --k) {
      if (p.active[1]) bwd_block(p, s, 1, b, h, k, accA[1], accD[1]);
      if (p.active[3]) bwd_block(p, s, 3, b, h, k, accA[3], accD[3]);
    }
    if (threadIdx.x == 0)
      for (int di = 1; di < 4; di += 2)
        if (p.active[di]) {
          p.dir[di].pA[static_cast<int64_t>(r) * BH + bh] = accA[di];
          p.dir[di].pD[static_cast<int64_t>(r) * BH + bh] = accD[di];
        }
    return;
  }
  const int b = blockIdx.x / H, h = blockIdx.x % H;
  // carry = dL/dstates[K-1] (given part)
  for (int64_t e = threadIdx.x; e < PN; e += kBwdThreads)
    s.carry[(e / N) * NS + e % N] =
        p.dstates ? p.dstates[((static_cast<int64_t>(b) * K + (K - 1)) * H + h) * PN + e] : 0.f;
  __syncthreads();
  float accA[4] = {0.f, 0.f, 0.f, 0.f}, accD[4] = {0.f, 0.f, 0.f, 0.f};
  for (int k = K - 1; k >= 0; --k) {
    bwd_block(p, s, 0, b, h, k, accA[0], accD[0]);
    bwd_block(p, s, 2, b, h, k, accA[2], accD[2]);
    if (!p.rev_split && p.active[1]) bwd_block(p, s, 1, b, h, k, accA[1], accD[1]);
    if (!p.rev_split && p.active[3]) bwd_block(p, s, 3, b, h, k, accA[3], accD[3]);
    // (dL/dstates[k - 1] joins the carried gradient in the next clean block's loads)
  }
  if (p.dh0)
    for (int64_t e = threadIdx.x; e < PN; e += kBwdThreads)
      p.dh0[(static_cast<int64_t>(b) * H + h) * PN + e] = s.carry[(e / N) * NS + e % N];
  if (threadIdx.x == 0)
    for (int di = 0; di < 4; ++di)
      if (p.active[di] && !(p.rev_split && (di & 1))) {
        p.dir[di].pA[static_cast<int64_t>(b) * H + h] = accA[di];
        p.dir[di].pD[static_cast<int64_t>(b) * H + h] = accD[di];
      }
}

// Fixed-order sums of the partials, all directions in one launch (grid row y =
// the y-th present direction): dB, dC over the heads of a group (16-byte loads
// and stores when N is a multiple of 4 and the outputs are 16-byte aligned),
// and, in the row's first CTA, dA, dD over the batch rows (and reverse ranges).
struct BwdSums {
  const float *pB[4], *pC[4], *pA[4], *pD[4];
  float *dB[4], *dC[4], *dA[4], *dD[4];
  int dir[4];    // direction of grid row y
  int arows[4];  // rows of the dA, dD partials of each direction
  int vec;       // 16-byte path
};

__global__ void bd_bwd_reduce_kernel(const __grid_constant__ BwdSums a, int64_t rows, int H, int G, int N) {
  const int di = a.dir[blockIdx.y];
  if (blockIdx.x == 0)
    for (int h = threadIdx.x; h < H; h += blockDim.x) {
      float sa = 0.f, sd = 0.f;
      for (int b = 0; b < a.arows[di]; ++b) {
        sa += a.pA[di][static_cast<int64_t>(b) * H + h];
        sd += a.pD[di][static_cast<int64_t>(b) * H + h];
      }
      a.dA[di][h] = sa;
      a.dD[di][h] = sd;
    }
  const float *pB = a.pB[di], *pC = a.pC[di];
  const int hpg = H / G;
  const int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (a.vec) {  // e over rows * G * N / 4
    const int n4 = N >> 2;
    if (e >= rows * G * n4) return;
    const int n = static_cast<int>(e % n4) << 2;
    const int g = static_cast<int>((e / n4) % G);
    const int64_t r = e / (static_cast<int64_t>(n4) * G);  // (b, t)
    float4 sb = make_float4(0.f, 0.f, 0.f, 0.f), sc = sb;
    for (int j = 0; j < hpg; ++j) {
      const int64_t o = (r * H + g * hpg + j) * N + n;
      const float4 vb = *reinterpret_cast<const float4 *>(pB + o), vc = *reinterpret_cast<const float4 *>(pC + o);
      sb.x += vb.x; sb.y += vb.y; sb.z += vb.z; sb.w += vb.w;
      sc.x += vc.x; sc.y += vc.y; sc.z += vc.z; sc.w += vc.w;
    }
    reinterpret_cast<float4 *>(a.dB[di])[e] = sb;
    reinterpret_cast<float4 *>(a.dC[di])[e] = sc;
  } else {  // e over rows * G * N
    if (e >= rows * G * N) return;
    const int n = static_cast<int>(e % N);
    const int g = static_cast<int>((e / N) % G);
    const int64_t r = e / (static_cast<int64_t>(N) * G);
    float sb = 0.f, sc = 0.f;
    for (int j = 0; j < hpg; ++j) {
      const int64_t o = (r * H + g * hpg + j) * N + n;
      sb += pB[o];
      sc += pC[o];
    }
    a.dB[di][e] = sb;
    a.dC[di][e] = sc;
  }
}

}  // namespace

size_t bwd_smem_bytes(int64_t P, int64_t N, int64_t T) {
  const int64_t floats = 4 * T * P + 4 * T * N + 6 * T + kBwdThreads + 3 * T * T + T * (T + 1) +
                         2 * ((P * (T + 1) + 3) & ~3) + 2 * P * (N + 4);
  return static_cast<size_t>(floats) * sizeof(float);
}

size_t bwd_workspace_bytes(int64_t Bsz, int64_t L, int64_t H, int64_t N) {
  // per direction: dB, dC partials [B][L][H][N] and dA, dD partials
  // [kRevSplit][B][H] (a forward direction uses the first B x H)
  const size_t per =
      (2 * static_cast<size_t>(Bsz) * L * H * N + 2 * static_cast<size_t>(kRevSplit) * Bsz * H) * sizeof(float);
  return 4 * ((per + 255) & ~static_cast<size_t>(255));
}

cudaError_t launch_bwd(const BwdArgs &a, cudaStream_t stream) {
  BwdParams p;
  std::memset(&p, 0, sizeof(p));
  const int64_t per_floats = 2 * a.Bsz * a.L * a.H * a.N + 2 * kRevSplit * a.Bsz * a.H;
  const size_t per = ((static_cast<size_t>(per_floats) * sizeof(float)) + 255) & ~static_cast<size_t>(255);
  for (int i = 0; i < 4; ++i) {
    p.active[i] = a.dir[i].x != nullptr;
    if (!p.active[i]) continue;
    BwdDir &d = p.dir[i];
    d.x = a.dir[i].x;
    d.dt = a.dir[i].dt;
    d.B = a.dir[i].B;
    d.C = a.dir[i].C;
    d.A = a.dir[i].A;
    d.D = a.dir[i].D;
    d.dx = a.grad[i].dx;
    d.ddt = a.grad[i].ddt;
    float *base = reinterpret_cast<float *>(static_cast<uint8_t *>(a.ws) + i * per);
    d.pB = base;
    d.pC = base + a.Bsz * a.L * a.H * a.N;
    d.pA = base + 2 * a.Bsz * a.L * a.H * a.N;
    d.pD = d.pA + kRevSplit * a.Bsz * a.H;
  }
  p.Bsz = static_cast<int>(a.Bsz);
  p.L = static_cast<int>(a.L);
  p.H = static_cast<int>(a.H);
  p.P = static_cast<int>(a.P);
  p.N = static_cast<int>(a.N);
  p.G = static_cast<int>(a.G);
  p.T = static_cast<int>(a.T);
  p.K = static_cast<int>(a.L / a.T);
  p.in_bf16 = a.in_bf16 ? 1 : 0;
  p.dy_bf16 = a.dy_bf16 ? 1 : 0;
  p.h0 = a.h0;
  p.states = a.states;
  p.dy_clean = a.dy_clean;
  p.dy_noisy = a.dy_noisy;
  p.dstates = a.dstates;
  p.dh0 = a.dh0;
  p.rev_split = (p.active[1] || p.active[3]) ? kRevSplit : 0;
  const size_t smem = bwd_smem_bytes(a.P, a.N, a.T);
  cudaError_t e = cudaFuncSetAttribute(bd_bwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  bd_bwd_kernel<<<static_cast<unsigned>(a.Bsz * a.H * (1 + p.rev_split)), kBwdThreads, smem, stream>>>(p);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const int64_t rows = a.Bsz * a.L;
  BwdSums sums;
  std::memset(&sums, 0, sizeof(sums));
  int ndir = 0;
  bool aligned = (a.N & 3) == 0;
  for (int i = 0; i < 4; ++i) {
    if (!p.active[i]) continue;
    const BwdDir &d = p.dir[i];
    sums.pB[i] = d.pB;
    sums.pC[i] = d.pC;
    sums.pA[i] = d.pA;
    sums.pD[i] = d.pD;
    sums.dB[i] = a.grad[i].dB;
    sums.dC[i] = a.grad[i].dC;
    sums.dA[i] = a.grad[i].dA;
    sums.dD[i] = a.grad[i].dD;
    sums.arows[i] = (i & 1) && p.rev_split ? p.Bsz * p.rev_split : p.Bsz;
    sums.dir[ndir++] = i;
    aligned = aligned && ((reinterpret_cast<uintptr_t>(a.grad[i].dB) | reinterpret_cast<uintptr_t>(a.grad[i].dC)) & 15) == 0;
  }
  sums.vec = aligned ? 1 : 0;
  const int64_t cnt = rows * a.G * (aligned ? a.N / 4 : a.N);
  if (ndir > 0) {
    const dim3 grid(static_cast<unsigned>(std::max<int64_t>(1, (cnt + 255) / 256)), static_cast<unsigned>(ndir));
    bd_bwd_reduce_kernel<<<grid, 256, 0, stream>>>(sums, rows, p.H, p.G, p.N);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace bdscan
