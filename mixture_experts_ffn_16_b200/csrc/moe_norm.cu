// moe_norm.cu - the pre-norm RMSNorm that produces the block's input, with
// zero-centred gains (the Qwen3.5 block: RMSNorm pre-norm directly before the
// router; the stored gain g is centred on zero, so the scale is 1 + g):
//
//   x_norm[t, i] = bf16( x[t, i] * (1 / sqrt(mean_j x[t, j]^2 + eps)) * (1 + g[i]) )
//
// One warp per token.  The arithmetic is double: the square of a bf16 value is
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

// One warp per token; lane l owns the 16-byte chunks l, l + 32, ... of the row.
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
  double ss = 0.0;
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
  uint4* yr = reinterpret_cast<uint4*>(y + static_cast<size_t>(t) * d);
  for (int c = lane; c < chunks; c += 32) {
    double a[8], g[8];
    widen8(__ldg(xr + c), a);
    widen8(__ldg(gr + c), g);
    uint4 o;
    __nv_bfloat16* ob = reinterpret_cast<__nv_bfloat16*>(&o);
#pragma unroll
    for (int i = 0; i < 8; ++i) ob[i] = bf16_from_double(__dmul_rn(__dmul_rn(a[i], rstd), 1.0 + g[i]));
    yr[c] = o;
  }
}

}  // namespace

int launch_rmsnorm(const Plan& p, const void* x, const void* gain, float eps, void* y, cudaStream_t st) {
  return launch_chained(rmsnorm_kernel, dim3((p.T + kNormThreads / 32 - 1) / (kNormThreads / 32)),
                        dim3(kNormThreads), 0, st,
                        reinterpret_cast<const __nv_bfloat16*>(x), reinterpret_cast<const __nv_bfloat16*>(gain),
                        static_cast<double>(eps), reinterpret_cast<__nv_bfloat16*>(y), p.T, p.d) == cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}

}  // namespace moe
