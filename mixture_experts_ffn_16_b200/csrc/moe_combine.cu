// moe_combine.cu - gate-weighted combine (step a7), the optional per-token
// shared-expert gate, and the bounded-wait self-test kernel.
//
// out[t, :] = sum_{s<S} g[t, s] Y_shared[s, t, :] + sum_{j<k} Y[inv[t, j], :]
// g = 1 (ungated), or sigmoid(W_gate_vec[s] . x[t]) (the Qwen3.5 shared expert).
// The routed rows already carry their combine weight (applied in fp32 by the
// down GEMM before rounding).  Each thread owns 8 consecutive features of one
// token, adds the S + k bf16 rows in that fixed order in fp32 and rounds once,
// so the result is bitwise reproducible and independent of the row layout.
#include <cuda_bf16.h>

#include "moe_internal.h"
#include "moe_ptx.cuh"

namespace moe {

namespace {

constexpr int kCombineThreads = 256;

__device__ __forceinline__ void add8(float (&acc)[8], const uint4 v) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h[i]);
    acc[2 * i] += f.x;
    acc[2 * i + 1] += f.y;
  }
}

// Per-token shared-expert gates g[t, s] = sigmoid(W_gate_vec[s, :] . x[t, :])
// (fp32 dot of bf16 values), one warp per token.
__global__ void __launch_bounds__(256)
shared_gate_kernel(const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ wv, int T, int d, int S,
                   float* __restrict__ g) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (t >= T) return;
  const uint4* xr = reinterpret_cast<const uint4*>(x + static_cast<size_t>(t) * d);
  for (int s = 0; s < S; ++s) {
    const uint4* wr = reinterpret_cast<const uint4*>(wv + static_cast<size_t>(s) * d);
    float acc = 0.0f;
    for (int c = lane; c < (d >> 3); c += 32) {
      const uint4 a = __ldg(xr + c), b = __ldg(wr + c);
      const __nv_bfloat162* ah = reinterpret_cast<const __nv_bfloat162*>(&a);
      const __nv_bfloat162* bh = reinterpret_cast<const __nv_bfloat162*>(&b);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 fa = __bfloat1622float2(ah[i]), fb = __bfloat1622float2(bh[i]);
        acc = fmaf(fa.x, fb.x, acc);
        acc = fmaf(fa.y, fb.y, acc);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) g[static_cast<size_t>(t) * S + s] = 1.0f / (1.0f + expf(-acc));
  }
}

__global__ void __launch_bounds__(kCombineThreads)
combine_kernel(const __nv_bfloat16* __restrict__ Yr, const __nv_bfloat16* __restrict__ Ys,
               const int32_t* __restrict__ inv, const float* __restrict__ sgate, __nv_bfloat16* __restrict__ out,
               int T, int d, int k, int S, int Tp) {
  const int chunks = d >> 3;
  const size_t total = static_cast<size_t>(T) * chunks;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int t = static_cast<int>(i / chunks);
    const int c = static_cast<int>(i - static_cast<size_t>(t) * chunks);
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int s = 0; s < S; ++s) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(
          Ys + (static_cast<size_t>(s) * Tp + t) * d + static_cast<size_t>(c) * 8));
      if (sgate) {
        float sh[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        add8(sh, v);
        const float gs = __ldg(sgate + static_cast<size_t>(t) * S + s);
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = fmaf(gs, sh[i], acc[i]);
      } else {
        add8(acc, v);
      }
    }
    const int32_t* it = inv + static_cast<size_t>(t) * k;
    for (int j = 0; j < k; ++j) {
      const int row = __ldg(it + j);
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(Yr + static_cast<size_t>(row) * d +
                                                           static_cast<size_t>(c) * 8));
      add8(acc, v);
    }
    uint4 o;
    __nv_bfloat162* oh = reinterpret_cast<__nv_bfloat162*>(&o);
#pragma unroll
    for (int q = 0; q < 4; ++q) oh[q] = __floats2bfloat162_rn(acc[2 * q], acc[2 * q + 1]);
    *reinterpret_cast<uint4*>(out + static_cast<size_t>(t) * d + static_cast<size_t>(c) * 8) = o;
  }
}

// Waits on a barrier that nothing completes, for at most timeout_ns, then
// records the timeout.  Used to test the bounded-wait path without a hang.
__global__ void wait_timeout_kernel(uint32_t* err, uint64_t timeout_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    mbar_wait(&bar, 0, &abort_flag, err, timeout_ns);
  }
  __syncthreads();
}

}  // namespace

int launch_combine(const Plan& p, void* out, char* ws, const void* x, const void* shared_gate_vec,
                   cudaStream_t st) {
  const float* sg = nullptr;
  if (shared_gate_vec && p.S > 0) {
    float* g = reinterpret_cast<float*>(ws + p.sgate);
    shared_gate_kernel<<<(p.T + 7) / 8, 256, 0, st>>>(reinterpret_cast<const __nv_bfloat16*>(x),
                                                      reinterpret_cast<const __nv_bfloat16*>(shared_gate_vec),
                                                      p.T, p.d, p.S, g);
    if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
    sg = g;
  }
  const size_t total = static_cast<size_t>(p.T) * (p.d / 8);
  size_t blocks = (total + kCombineThreads - 1) / kCombineThreads;
  if (blocks > 148 * 16) blocks = 148 * 16;
  combine_kernel<<<static_cast<int>(blocks), kCombineThreads, 0, st>>>(
      reinterpret_cast<const __nv_bfloat16*>(ws + p.Yr), reinterpret_cast<const __nv_bfloat16*>(ws + p.Ys),
      reinterpret_cast<const int32_t*>(ws + p.inv), sg, reinterpret_cast<__nv_bfloat16*>(out), p.T, p.d,
      p.k, p.S, p.Tp);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

int launch_wait_timeout(uint32_t* err, uint64_t timeout_ns, cudaStream_t st) {
  wait_timeout_kernel<<<1, 32, 0, st>>>(err, timeout_ns);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe
