// norm.cu -- the gated RMSNorm of the summed output y = y_fwd + y_rev, with a
// bf16 result ("Breaking the Bottleneck with DiffuApriel", section 3.2 after
// eq. (6): the summed hidden sequence is normalised before the layer's
// projection; read as the Mamba-2 layer's gated RMSNorm, gate before the norm):
//
//   v_c = y_c * silu(z_c)   (v = y without z)
//   per token row and group of gs = C / groups consecutive channels:
//   out_c = bf16( v_c * w_c / sqrt(mean_{c in group} v_c^2 + eps) )
//
// The norm spans all heads of a token while the scan's unit of work is one
// (row, head) sequence, so it runs as its own HBM-bound pass over the scan's
// output: one CTA per token row reads y (and z) once into shared memory as v,
// forms per-vector sums of squares, reduces each group in a fixed order (the
// result is deterministic), and writes the row once in bf16.  In place (out ==
// y, both bf16) is safe: the whole row is in shared memory before any store.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>

#include "bdscan_internal.h"

namespace bdscan {
namespace {

constexpr int kNormThreads = 256;

struct NormParams {
  const void *y, *z;
  const float *w;
  __nv_bfloat16 *out;
  int C, nv, groups, gsv;  // channels, 4-channel vectors per row, groups, vectors per group
  float eps, inv_gs;
};

__device__ __forceinline__ void load4(const float *p, float (&f)[4]) {
  const float4 q = __ldg(reinterpret_cast<const float4 *>(p));
  f[0] = q.x; f[1] = q.y; f[2] = q.z; f[3] = q.w;
}

__device__ __forceinline__ void load4(const __nv_bfloat16 *p, float (&f)[4]) {
  const uint2 q = __ldg(reinterpret_cast<const uint2 *>(p));
  f[0] = __uint_as_float(q.x << 16);
  f[1] = __uint_as_float(q.x & 0xffff0000u);
  f[2] = __uint_as_float(q.y << 16);
  f[3] = __uint_as_float(q.y & 0xffff0000u);
}

// silu with the hardware exponential and reciprocal (a few ulp)
__device__ __forceinline__ float silu_f(float v) { return __fdividef(v, 1.0f + __expf(-v)); }

template <typename TY, typename TZ>
__global__ void __launch_bounds__(kNormThreads) bd_norm_kernel(const __grid_constant__ NormParams p) {
  extern __shared__ float4 smem4[];
  float4 *vrow = smem4;                                           // v of the row, [nv]
  float *part = reinterpret_cast<float *>(smem4 + p.nv);          // sum of squares per vector, [nv]
  float *rstd = part + p.nv;                                      // per group, [groups]
  // programmatic dependent of the kernel before it (the scan that wrote y):
  // wait for it, then let the next kernel be scheduled
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int64_t row = blockIdx.x;
  const TY *y = static_cast<const TY *>(p.y) + row * p.C;
  const TZ *z = p.z ? static_cast<const TZ *>(p.z) + row * p.C : nullptr;

  const int nthr = blockDim.x;
  for (int v = threadIdx.x; v < p.nv; v += nthr) {
    float a[4];
    load4(y + 4 * v, a);
    if (z) {
      float g[4];
      load4(z + 4 * v, g);
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] *= silu_f(g[i]);
    }
    vrow[v] = make_float4(a[0], a[1], a[2], a[3]);
    part[v] = fmaf(a[3], a[3], fmaf(a[2], a[2], fmaf(a[1], a[1], a[0] * a[0])));
  }
  __syncthreads();
  // one warp per group: lanes sum strided vectors, then a fixed shuffle tree
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int g = warp; g < p.groups; g += nthr / 32) {
    float s = 0.f;
    for (int v = g * p.gsv + lane; v < (g + 1) * p.gsv; v += 32) s += part[v];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) rstd[g] = 1.0f / sqrtf(fmaf(s, p.inv_gs, p.eps));
  }
  __syncthreads();
  __nv_bfloat16 *out = p.out + row * p.C;
  for (int v = threadIdx.x; v < p.nv; v += nthr) {
    const float r = rstd[v / p.gsv];
    const float4 a = vrow[v];
    const float4 w = __ldg(reinterpret_cast<const float4 *>(p.w) + v);
    const __nv_bfloat162 lo = __floats2bfloat162_rn(a.x * r * w.x, a.y * r * w.y);
    const __nv_bfloat162 hi = __floats2bfloat162_rn(a.z * r * w.z, a.w * r * w.w);
    *reinterpret_cast<uint2 *>(out + 4 * v) =
        make_uint2(*reinterpret_cast<const uint32_t *>(&lo), *reinterpret_cast<const uint32_t *>(&hi));
  }
}

template <typename TY, typename TZ>
cudaError_t launch_typed(const NormParams &p, int64_t rows, size_t smem, cudaStream_t stream) {
  cudaError_t e = cudaFuncSetAttribute(bd_norm_kernel<TY, TZ>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  // programmatic dependent launch (see the kernel's first lines)
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3(static_cast<unsigned>(rows));
  // about three 4-channel vectors per thread: whole warps, 64 to 256 threads
  const int want = (p.nv + 2) / 3;
  cfg.blockDim = dim3(static_cast<unsigned>(want <= 64 ? 64 : (want <= 128 ? 128 : kNormThreads)));
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, bd_norm_kernel<TY, TZ>, p);
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace

size_t norm_smem_bytes(int64_t C, int64_t groups) {
  return static_cast<size_t>(C) * 4 + static_cast<size_t>(C / 4) * 4 + static_cast<size_t>(groups) * 4;
}

cudaError_t launch_norm(const NormArgs &a, cudaStream_t stream) {
  const int64_t rows = a.Bsz * a.L;
  if (rows == 0) return cudaSuccess;
  NormParams p{};
  p.y = a.y;
  p.z = a.z;
  p.w = a.weight;
  p.out = static_cast<__nv_bfloat16 *>(a.out);
  p.C = static_cast<int>(a.C);
  p.nv = static_cast<int>(a.C / 4);
  p.groups = static_cast<int>(a.groups);
  p.gsv = static_cast<int>(a.C / a.groups / 4);
  p.eps = a.eps;
  p.inv_gs = 1.0f / static_cast<float>(a.C / a.groups);
  const size_t smem = norm_smem_bytes(a.C, a.groups);
  if (a.y_bf16) {
    if (!a.z) return launch_typed<__nv_bfloat16, __nv_bfloat16>(p, rows, smem, stream);
    return a.z_bf16 ? launch_typed<__nv_bfloat16, __nv_bfloat16>(p, rows, smem, stream)
                    : launch_typed<__nv_bfloat16, float>(p, rows, smem, stream);
  }
  if (!a.z) return launch_typed<float, __nv_bfloat16>(p, rows, smem, stream);
  return a.z_bf16 ? launch_typed<float, __nv_bfloat16>(p, rows, smem, stream)
                  : launch_typed<float, float>(p, rows, smem, stream);
}

}  // namespace bdscan
