// moe_combine.cu - gate-weighted combine (step a7) with the optional per-token
// shared-expert gate fused in, and the bounded-wait self-test kernel.
//
// out[t, :] = sum_{s<S} g[t, s] Y_shared[s, t, :] + sum_{j<k} Y[inv[t, j], :]
// g = 1 (ungated), or sigmoid(W_gate_vec[s] . x[t]) (the Qwen3.5 shared expert).
// The routed rows already carry their combine weight (applied in fp32 by the
// down GEMM before rounding).  One CTA per token: each thread owns 8
// consecutive features per pass, adds the S + k bf16 rows in that fixed order
// with fp32 fused multiply-adds (scale 1 for every row but a gated shared one,
// which makes those adds exact sums) and rounds once, so the result is bitwise
// reproducible and independent of the row layout.  The rows' loads are issued
// eight at a time before their adds so that each thread keeps eight 16-byte
// loads in flight.
#include <cuda_bf16.h>

#include "moe_internal.h"
#include "moe_ptx.cuh"

namespace moe {

namespace {

constexpr int kCombineThreads = 256;
constexpr int kCombineWarps = kCombineThreads / 32;
constexpr int kBatch = 8;

__device__ __forceinline__ void fma8(float (&acc)[8], const float g, const uint4 v) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h[i]);
    acc[2 * i] = fmaf(g, f.x, acc[2 * i]);
    acc[2 * i + 1] = fmaf(g, f.y, acc[2 * i + 1]);
  }
}

__device__ __forceinline__ float dot8(const uint4 a, const uint4 b, float acc) {
  const __nv_bfloat162* ah = reinterpret_cast<const __nv_bfloat162*>(&a);
  const __nv_bfloat162* bh = reinterpret_cast<const __nv_bfloat162*>(&b);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 fa = __bfloat1622float2(ah[i]), fb = __bfloat1622float2(bh[i]);
    acc = fmaf(fa.x, fb.x, acc);
    acc = fmaf(fa.y, fb.y, acc);
  }
  return acc;
}

// grid = T (one CTA per token; the block scheduler balances the load).
// gvec == nullptr: ungated.  Otherwise the gates are also written to g_out[t, s].
__global__ void __launch_bounds__(kCombineThreads)
combine_kernel(const __nv_bfloat16* __restrict__ Yr, const __nv_bfloat16* __restrict__ Ys,
               const int32_t* __restrict__ inv, const __nv_bfloat16* __restrict__ x,
               const __nv_bfloat16* __restrict__ gvec, float* __restrict__ g_out, __nv_bfloat16* __restrict__ out,
               int d, int k, int S, int Tp) {
  __shared__ const __nv_bfloat16* src[kMaxShared + kMaxK];
  __shared__ float scale[kMaxShared + kMaxK];
  __shared__ float red[kMaxShared][kCombineWarps];
  chain_wait();
  const int t = blockIdx.x;
  const int tid = threadIdx.x;
  const int chunks = d >> 3;
  const int n = S + k;

  if (gvec != nullptr) {
    // g[s] = sigmoid(w_s . x_t): per-thread partials over fixed chunks, a
    // fixed shuffle tree per warp, then the warps in order.
    const uint4* xr = reinterpret_cast<const uint4*>(x + static_cast<size_t>(t) * d);
    for (int s = 0; s < S; ++s) {
      const uint4* wr = reinterpret_cast<const uint4*>(gvec + static_cast<size_t>(s) * d);
      float acc = 0.0f;
      for (int c = tid; c < chunks; c += kCombineThreads) acc = dot8(__ldg(xr + c), __ldg(wr + c), acc);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if ((tid & 31) == 0) red[s][tid >> 5] = acc;
    }
  }
  if (tid < n) {
    if (tid < S) {
      src[tid] = Ys + (static_cast<size_t>(tid) * Tp + t) * d;
    } else {
      src[tid] = Yr + static_cast<size_t>(__ldg(inv + static_cast<size_t>(t) * k + (tid - S))) * d;
      scale[tid] = 1.0f;
    }
  }
  __syncthreads();
  if (tid < S) {
    float g = 1.0f;
    if (gvec != nullptr) {
      float z = 0.0f;
      for (int w = 0; w < kCombineWarps; ++w) z += red[tid][w];
      g = 1.0f / (1.0f + expf(-z));
      g_out[static_cast<size_t>(t) * S + tid] = g;
    }
    scale[tid] = g;
  }
  __syncthreads();

  for (int c = tid; c < chunks; c += kCombineThreads) {
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int j0 = 0; j0 < n; j0 += kBatch) {
      uint4 v[kBatch];
#pragma unroll
      for (int q = 0; q < kBatch; ++q)
        if (j0 + q < n) v[q] = __ldg(reinterpret_cast<const uint4*>(src[j0 + q]) + c);
#pragma unroll
      for (int q = 0; q < kBatch; ++q)
        if (j0 + q < n) fma8(acc, scale[j0 + q], v[q]);
    }
    uint4 o;
    __nv_bfloat162* oh = reinterpret_cast<__nv_bfloat162*>(&o);
#pragma unroll
    for (int q = 0; q < 4; ++q) oh[q] = __floats2bfloat162_rn(acc[2 * q], acc[2 * q + 1]);
    reinterpret_cast<uint4*>(out + static_cast<size_t>(t) * d)[c] = o;
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
  const bool gated = shared_gate_vec != nullptr && p.S > 0;
  return launch_chained(combine_kernel, dim3(p.T), dim3(kCombineThreads), 0, st,
                        reinterpret_cast<const __nv_bfloat16*>(ws + p.Yr),
                        reinterpret_cast<const __nv_bfloat16*>(ws + p.Ys),
                        reinterpret_cast<const int32_t*>(ws + p.inv), reinterpret_cast<const __nv_bfloat16*>(x),
                        gated ? reinterpret_cast<const __nv_bfloat16*>(shared_gate_vec) : nullptr,
                        reinterpret_cast<float*>(ws + p.sgate), reinterpret_cast<__nv_bfloat16*>(out), p.d, p.k,
                        p.S, p.Tp) == cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}

int launch_wait_timeout(uint32_t* err, uint64_t timeout_ns, cudaStream_t st) {
  wait_timeout_kernel<<<1, 32, 0, st>>>(err, timeout_ns);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe
