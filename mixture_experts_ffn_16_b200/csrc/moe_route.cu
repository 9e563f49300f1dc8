// moe_route.cu - scoring, top-k selection and combine weights (step a2).
//
// One warp per token reads the token's fp32 logits (written by the router
// GEMM; for small batches as partial sums over slices of d, added here in
// slice order), forms the scores and selection keys in registers, and picks the k
// largest keys by k rounds of a warp-wide arg-max (ties go to the lower expert
// index, matching a stable descending sort); each round reduces the lanes'
// best keys with two warp reductions.  A lane keeps its keys in groups of up
// to 8 with each group's best, so after a round only the winning lane
// rescans one group (instead of every lane rescanning all of its keys).
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

// Group g (slots g*GS .. g*GS + GS - 1) of a lane's codes: drop slot ws (if
// it is in the group) and recompute the group's best code and slot.
template <int NPL, int GS, int g>
__device__ __forceinline__ void rescan_group(uint32_t (&code)[NPL], uint32_t (&gc)[NPL / GS], int (&gs)[NPL / GS],
                                             int ws) {
  if constexpr (g < NPL / GS) {
    gc[g] = 0u;
    gs[g] = 0;
#pragma unroll
    for (int jj = 0; jj < GS; ++jj) {
      if (g * GS + jj == ws) code[g * GS + jj] = 0u;
      if (code[g * GS + jj] > gc[g]) {
        gc[g] = code[g * GS + jj];
        gs[g] = g * GS + jj;
      }
    }
  }
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

  // Groups of GS consecutive slots (slot i = expert lane + 32 i), each with
  // its best code and slot (the lower slot, i.e. the lower expert, on equal
  // codes); the lane's best is the best of its groups in slot order.
  constexpr int GS = NPL < 8 ? NPL : 8;
  constexpr int G = NPL / GS;
  static_assert(G <= 8, "at most 8 groups");
  uint32_t gc[G];
  int gs[G];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    gc[g] = 0u;
    gs[g] = 0;
#pragma unroll
    for (int jj = 0; jj < GS; ++jj) {
      if (code[g * GS + jj] > gc[g]) {
        gc[g] = code[g * GS + jj];
        gs[g] = g * GS + jj;
      }
    }
  }
  uint32_t bc = 0u;   // this lane's best remaining code (0: none left)
  int bs = 0;         // ... and its slot
#pragma unroll
  for (int g = 0; g < G; ++g) {
    if (gc[g] > bc) {
      bc = gc[g];
      bs = gs[g];
    }
  }

  int my_idx = 0;    // lane j keeps the j-th pick
  for (int j = 0; j < k; ++j) {
    // Warp arg-max in two reductions: the largest code, then the lowest
    // expert index among the lanes that hold it.  k <= E leaves at least one
    // unpicked expert, whose code is >= kKeyFloor > 0, so the winner is one.
    const uint32_t cmax = __reduce_max_sync(0xffffffffu, bc);
    const int bi = static_cast<int>(
        __reduce_min_sync(0xffffffffu, bc == cmax ? static_cast<uint32_t>(lane + 32 * bs) : 0x7fffffffu));
    if (lane == j) my_idx = bi;
    // The owner lane removes the winner and rescans the winner's group.
    if ((bi & 31) == lane) {
      const int ws = bi >> 5;
      switch (ws / GS) {   // G <= 8; a switch keeps every index static
        case 0: rescan_group<NPL, GS, 0>(code, gc, gs, ws); break;
        case 1: rescan_group<NPL, GS, 1>(code, gc, gs, ws); break;
        case 2: rescan_group<NPL, GS, 2>(code, gc, gs, ws); break;
        case 3: rescan_group<NPL, GS, 3>(code, gc, gs, ws); break;
        case 4: rescan_group<NPL, GS, 4>(code, gc, gs, ws); break;
        case 5: rescan_group<NPL, GS, 5>(code, gc, gs, ws); break;
        case 6: rescan_group<NPL, GS, 6>(code, gc, gs, ws); break;
        default: rescan_group<NPL, GS, 7>(code, gc, gs, ws); break;
      }
      bc = 0u;
      bs = 0;
#pragma unroll
      for (int g = 0; g < G; ++g) {
        if (gc[g] > bc) {
          bc = gc[g];
          bs = gs[g];
        }
      }
    }
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
