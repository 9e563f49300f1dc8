// moe_norm.cu - the pre-norm RMSNorm that produces the block's input, with
// zero-centred gains (the Qwen3.5 block: RMSNorm pre-norm directly before the
// router; the stored gain g is centred on zero, so the scale is 1 + g):
//
//   x_norm[t, i] = bf16( x[t, i] * (1 / sqrt(mean_j x[t, j]^2 + eps)) * (1 + g[i]) )
//
// One warp per token; up to d = 4096 the row stays in registers, so x is read
// once.  The arithmetic is double: the square of a bf16 value is
// exact, so the only rounding before the reciprocal square root is in the sum
// of the d squares (fixed order: per lane over its chunks, then a fixed
// shuffle tree), and the result is rounded to bf16
// in a single correctly rounded step.  That step rounds the double to binary32
// with round-to-odd (truncate; force the last bit to 1 when bits were lost),
// then to bf16 to nearest even: with more than two extra bits in the
// intermediate format this equals direct rounding (Boldo and Melquiond,
// "Emulation of FMA and correctly rounded sums: proved algorithms using
// rounding to odd", IEEE Trans. Computers 57(4), 2008).
#include <cuda_bf16.h>

#include "moe_internal.h"
#include "moe_ptx.cuh"

namespace moe {

namespace {

constexpr int kNormThreads = 256;   // 8 tokens per CTA
constexpr int kBatch = 8;           // 16-byte loads in flight per lane

__device__ __forceinline__ __nv_bfloat16 bf16_from_double(double v) {
  float f = __double2float_rz(v);
  if (static_cast<double>(f) != v) f = __uint_as_float(__float_as_uint(f) | 1u);
  return __float2bfloat16_rn(f);
}

__device__ __forceinline__ void widen8(const uint4 v, double (&o)[8]) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h[i]);
    o[2 * i] = f.x;
    o[2 * i + 1] = f.y;
  }
}

__device__ __forceinline__ uint4 norm8(const uint4 xv, const uint4 gv, double rstd) {
  double a[8], g[8];
  widen8(xv, a);
  widen8(gv, g);
  uint4 o;
  __nv_bfloat16* ob = reinterpret_cast<__nv_bfloat16*>(&o);
#pragma unroll
  for (int i = 0; i < 8; ++i) ob[i] = bf16_from_double(__dmul_rn(__dmul_rn(a[i], rstd), 1.0 + g[i]));
  return o;
}

// One warp per token; lane l owns the 16-byte chunks l, l + 32, ... of the
// row and adds their squares in that order, then the lanes' sums meet in a
// fixed shuffle tree.  NC > 0: the row has at most 32 NC chunks, which stay in
// registers (with their gains) between the sum and the scaling, so x is read
// once.  NC == 0: any d; the scaling pass reads the row again, kBatch chunks
// in flight per lane.
template <int NC>
__global__ void __launch_bounds__(kNormThreads)
rmsnorm_kernel(const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ gain, double eps,
               __nv_bfloat16* __restrict__ y, int T, int d) {
  chain_wait();
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (kNormThreads / 32) + (threadIdx.x >> 5);
  if (t >= T) return;
  const int chunks = d >> 3;
  const uint4* xr = reinterpret_cast<const uint4*>(x + static_cast<size_t>(t) * d);
  const uint4* gr = reinterpret_cast<const uint4*>(gain);
  uint4* yr = reinterpret_cast<uint4*>(y + static_cast<size_t>(t) * d);
  double ss = 0.0;
  if constexpr (NC > 0) {
    uint4 v[NC], gv[NC];
#pragma unroll
    for (int i = 0; i < NC; ++i)
      if (lane + 32 * i < chunks) v[i] = __ldg(xr + lane + 32 * i);
#pragma unroll
    for (int i = 0; i < NC; ++i)
      if (lane + 32 * i < chunks) gv[i] = __ldg(gr + lane + 32 * i);
#pragma unroll
    for (int i = 0; i < NC; ++i) {
      if (lane + 32 * i < chunks) {
        double a[8];
        widen8(v[i], a);
#pragma unroll
        for (int j = 0; j < 8; ++j) ss = fma(a[j], a[j], ss);   // a*a is exact: one rounding per term
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const double rstd = 1.0 / sqrt(ss / d + eps);
#pragma unroll
    for (int i = 0; i < NC; ++i)
      if (lane + 32 * i < chunks) yr[lane + 32 * i] = norm8(v[i], gv[i], rstd);
  } else {
    for (int c0 = lane; c0 < chunks; c0 += 32 * kBatch) {
      uint4 v[kBatch];
#pragma unroll
      for (int b = 0; b < kBatch; ++b)
        if (c0 + 32 * b < chunks) v[b] = __ldg(xr + c0 + 32 * b);
#pragma unroll
      for (int b = 0; b < kBatch; ++b) {
        if (c0 + 32 * b < chunks) {
          double a[8];
          widen8(v[b], a);
#pragma unroll
          for (int i = 0; i < 8; ++i) ss = fma(a[i], a[i], ss);   // a*a is exact: one rounding per term
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const double rstd = 1.0 / sqrt(ss / d + eps);
    for (int c0 = lane; c0 < chunks; c0 += 32 * kBatch) {
      uint4 v[kBatch], gv[kBatch];
#pragma unroll
      for (int b = 0; b < kBatch; ++b) {
        if (c0 + 32 * b < chunks) {
          v[b] = __ldg(xr + c0 + 32 * b);
          gv[b] = __ldg(gr + c0 + 32 * b);
        }
      }
#pragma unroll
      for (int b = 0; b < kBatch; ++b)
        if (c0 + 32 * b < chunks) yr[c0 + 32 * b] = norm8(v[b], gv[b], rstd);
    }
  }
}

template <int NC>
int launch_norm(const Plan& p, const void* x, const void* gain, float eps, void* y, cudaStream_t st) {
  return launch_chained(rmsnorm_kernel<NC>, dim3((p.T + kNormThreads / 32 - 1) / (kNormThreads / 32)),
                        dim3(kNormThreads), 0, st,
                        reinterpret_cast<const __nv_bfloat16*>(x), reinterpret_cast<const __nv_bfloat16*>(gain),
                        static_cast<double>(eps), reinterpret_cast<__nv_bfloat16*>(y), p.T, p.d) == cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}

}  // namespace

int launch_rmsnorm(const Plan& p, const void* x, const void* gain, float eps, void* y, cudaStream_t st) {
  const int chunks_per_lane = (p.d / 8 + 31) / 32;
  if (chunks_per_lane <= 2) return launch_norm<2>(p, x, gain, eps, y, st);
  if (chunks_per_lane <= 4) return launch_norm<4>(p, x, gain, eps, y, st);
  if (chunks_per_lane <= 8) return launch_norm<8>(p, x, gain, eps, y, st);
  if (chunks_per_lane <= 16) return launch_norm<16>(p, x, gain, eps, y, st);
  return launch_norm<0>(p, x, gain, eps, y, st);
}

}  // namespace moe
