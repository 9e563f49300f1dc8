// moe_route.cu - scoring, top-k selection and combine weights (step a2).
//
// One warp per token reads the token's fp32 logits (written by the router
// GEMM; for small batches as partial sums over slices of d, added here in
// slice order), forms the scores and selection keys in registers, and picks the k
// largest keys by k rounds of a warp-wide arg-max (ties go to the lower expert
// index, matching a stable descending sort); each round reduces the lanes'
// best keys with two warp reductions.
//
//   softmax       : key = logit (same order as the softmax probability);
//                   w_j = exp(l_j - l_max) / (norm ? sum over picks : sum over all E)
//   sigmoid       : s = 1/(1+exp(-l)),            key = s + bias
//   sqrt-softplus : s = sqrt(max(l,0) + log1p(exp(-|l|))), key = s + bias
//                   w_j = s_j (/ sum over picks if norm)
//   then w_j *= route_scale.
// The bias only orders the experts; the weights come from the unbiased scores.
#include <cfloat>
#include <cmath>

#include "moe_internal.h"
#include "moe_ptx.cuh"

namespace moe {

namespace {

constexpr int kWarpsPerBlock = 8;

__device__ __forceinline__ float score_of(float l, int fn) {
  if (fn == MOE_SCORE_SIGMOID) return 1.0f / (1.0f + expf(-l));
  // MOE_SCORE_SQRT_SOFTPLUS
  return sqrtf(fmaxf(l, 0.0f) + log1pf(expf(-fabsf(l))));
}

// Selection keys as order-preserving unsigned integers: a larger float key
// gives a larger code, +0 and -0 the same code.  Every real key, -inf and NaN
// included, maps to a code >= kKeyFloor (NaN ranks with -inf, below every
// other key), and 0 marks an expert already picked, so the k rounds always
// pick k distinct experts in [0, E) whatever the logits hold.
constexpr uint32_t kKeyFloor = 0x007FFFFFu;   // the code of -inf

__device__ __forceinline__ uint32_t key_code(float key) {
  if (key != key) return kKeyFloor;            // NaN
  const uint32_t ub = __float_as_uint(key + 0.0f);
  return (ub & 0x80000000u) ? ~ub : (ub | 0x80000000u);
}

template <int NPL>   // keys per lane: E <= 32 * NPL
__global__ void __launch_bounds__(kWarpsPerBlock * 32)
topk_kernel(const float* __restrict__ logits, int nsplit, const float* __restrict__ bias, int T, int E, int k,
            int score_fn, int norm_topk, float route_scale, int32_t* __restrict__ topk_idx,
            float* __restrict__ topk_w, uint32_t* err) {
  chain_wait();
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5);
  if (t >= T) return;
  // The router GEMM gave up a bounded wait: its logits are incomplete, so no
  // routing is made from them.  Expert -1 with weight 0 marks every token
  // (the permute step flags such routing as invalid).
  if (*reinterpret_cast<volatile uint32_t*>(err) & kDevErrTimeout) {
    if (lane < k) {
      topk_idx[static_cast<size_t>(t) * k + lane] = -1;
      topk_w[static_cast<size_t>(t) * k + lane] = 0.0f;
    }
    return;
  }
  const float* row = logits + static_cast<size_t>(t) * E;
  const size_t slice = static_cast<size_t>(T) * E;
  // logit = the sum of the K slices' partial logits, in slice order; all of
  // this lane's loads of a slice are issued together
  float lv[NPL];
#pragma unroll
  for (int i = 0; i < NPL; ++i) {
    const int e = lane + 32 * i;
    lv[i] = (e < E) ? row[e] : 0.0f;
  }
  for (int s = 1; s < nsplit; ++s) {
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
      const int e = lane + 32 * i;
      if (e < E) lv[i] += row[s * slice + e];
    }
  }
  const bool use_bias = (bias != nullptr) && (score_fn != MOE_SCORE_SOFTMAX);

  uint32_t code[NPL];     // 0: past E, or already picked
  float lmax = -FLT_MAX;
  bool nonfinite = false;
#pragma unroll
  for (int i = 0; i < NPL; ++i) {
    const int e = lane + 32 * i;
    code[i] = 0u;
    if (e < E) {
      const float l = lv[i];
      lmax = fmaxf(lmax, l);
      const float kv = (score_fn == MOE_SCORE_SOFTMAX) ? l : score_of(l, score_fn) + (use_bias ? bias[e] : 0.0f);
      nonfinite |= !isfinite(kv);
      code[i] = key_code(kv);
    }
  }

  // Softmax without renormalisation needs the full denominator.
  float zsum = 0.0f;
  if (score_fn == MOE_SCORE_SOFTMAX) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) lmax = fmaxf(lmax, __shfl_xor_sync(0xffffffffu, lmax, o));
    if (!norm_topk) {
#pragma unroll
      for (int i = 0; i < NPL; ++i)
        if (lane + 32 * i < E) zsum += expf(lv[i] - lmax);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) zsum += __shfl_xor_sync(0xffffffffu, zsum, o);
    }
  }

  int my_idx = 0;    // lane j keeps the j-th pick
  for (int j = 0; j < k; ++j) {
    // this lane's best remaining key (the lower expert index on equal codes)
    uint32_t bc = 0u;
    int bi = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
      if (code[i] > bc) {
        bc = code[i];
        bi = lane + 32 * i;
      }
    }
    // Warp arg-max in two reductions: the largest code, then the lowest
    // expert index among the lanes that hold it.  k <= E leaves at least one
    // unpicked expert, whose code is >= kKeyFloor > 0, so the winner is one.
    const uint32_t cmax = __reduce_max_sync(0xffffffffu, bc);
    bi = static_cast<int>(__reduce_min_sync(0xffffffffu, bc == cmax ? static_cast<uint32_t>(bi) : 0x7fffffffu));
    // Remove the winner (its owner lane), record it in lane j.
#pragma unroll
    for (int i = 0; i < NPL; ++i)
      if (lane + 32 * i == bi) code[i] = 0u;
    if (lane == j) my_idx = bi;
  }

  float s = 0.0f;
  if (lane < k && my_idx >= 0 && my_idx < E) {
    float l = row[my_idx];
    for (int sl = 1; sl < nsplit; ++sl) l += row[sl * slice + my_idx];
    s = (score_fn == MOE_SCORE_SOFTMAX) ? expf(l - lmax) : score_of(l, score_fn);
  }
  float denom;
  if (norm_topk) {
    denom = s;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) denom += __shfl_xor_sync(0xffffffffu, denom, o);
    denom = fmaxf(denom, FLT_MIN);
  } else {
    denom = (score_fn == MOE_SCORE_SOFTMAX) ? zsum : 1.0f;
  }
  const float wv = (s / denom) * route_scale;
  if (lane < k) {
    topk_idx[static_cast<size_t>(t) * k + lane] = my_idx;
    topk_w[static_cast<size_t>(t) * k + lane] = wv;
    nonfinite |= !isfinite(wv);
  }
  // A NaN or infinite key or weight anywhere in this token's row: the routing
  // above is still valid (NaN keys rank lowest), but the caller is told.
  if (__any_sync(0xffffffffu, nonfinite) && lane == 0) atomicOr(err, kDevErrNonFinite);
}

template <int NPL>
int launch_npl(const float* logits, int nsplit, const float* bias, int T, int E, int k, int fn, int norm,
               float scale, int32_t* idx, float* w, uint32_t* err, cudaStream_t st) {
  const int grid = (T + kWarpsPerBlock - 1) / kWarpsPerBlock;
  return launch_chained(topk_kernel<NPL>, dim3(grid), dim3(kWarpsPerBlock * 32), 0, st, logits, nsplit, bias, T, E,
                        k, fn, norm, scale, idx, w, err) == cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}

}  // namespace

int launch_topk(const float* logits, int nsplit, const float* bias, int T, int E, int k, int score_fn,
                int norm_topk, float route_scale, int32_t* topk_idx, float* topk_w, uint32_t* err,
                cudaStream_t st) {
#define MOE_TOPK(NPL) \
  launch_npl<NPL>(logits, nsplit, bias, T, E, k, score_fn, norm_topk, route_scale, topk_idx, topk_w, err, st)
  if (E <= 32) return MOE_TOPK(1);
  if (E <= 64) return MOE_TOPK(2);
  if (E <= 128) return MOE_TOPK(4);
  if (E <= 256) return MOE_TOPK(8);
  if (E <= 512) return MOE_TOPK(16);
  if (E <= 1024) return MOE_TOPK(32);
  return MOE_TOPK(64);
#undef MOE_TOPK
}

}  // namespace moe
