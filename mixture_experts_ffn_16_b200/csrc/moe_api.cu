// moe_api.cu - the C ABI of libmoe.so (declared in include/moe.h): argument
// checks, the workspace plan, TMA tensor maps, and the launch sequence
//   router GEMM -> top-k -> permute (count, scan, scatter) ->
//   gate/up GEMM -> down GEMM -> combine
// on the caller's stream.  No host synchronisation, no device allocation.
#include <cmath>
#include <cstring>

#include "moe_internal.h"
#include "moe_ptx.cuh"

namespace moe {

namespace {

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }
int ceil_div(int a, int b) { return (a + b - 1) / b; }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  // looked up once per process (thread-safe static initialisation); first
  // reached from device_info, after the runtime is up
  static const EncodeTiledFn fn = [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<EncodeTiledFn>(ptr);
    return static_cast<EncodeTiledFn>(nullptr);
  }();
  return fn;
}

// Weight tensor [G, rows, K] bf16 -> tiles of 128 rows x 64 K, 128-byte swizzle.
bool map_weights(CUtensorMap* m, const void* ptr, int K, int rows, int G) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(G)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(K) * 2, static_cast<cuuint64_t>(K) * 2 * rows};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(kTileK), static_cast<cuuint32_t>(kTileRows), 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Block-scaled FP8 weight: codes [G, rows, K] uint8 -> tiles of 128 rows x 64
// codes (unswizzled 64-byte rows); scales [G, K/32, rows] uint8 -> tiles of
// 128 rows x 2 blocks.
bool map_f8_codes(CUtensorMap* m, const void* ptr, int K, int rows, int G) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(G)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(K) * rows};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(kTileK), static_cast<cuuint32_t>(kTileRows), 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(ptr), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool map_f8_scales(CUtensorMap* m, const void* ptr, int K, int rows, int G) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const int nb = K / 32;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(nb), static_cast<cuuint64_t>(G)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(rows) * nb};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(kTileRows), static_cast<cuuint32_t>(kTileK / 32), 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(ptr), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// An expert weight operand: bf16 (s == nullptr), or block-scaled FP8 codes
// (p) with their scales (s).
struct Wt {
  const void* p = nullptr;
  const void* s = nullptr;
  Wt(const void* d = nullptr) : p(d) {}   // NOLINT: bf16 pointers convert implicitly
  Wt(const void* d, const void* sc) : p(d), s(sc) {}
};

bool map_weight_operand(CUtensorMap* a, CUtensorMap* sc, const Wt& w, int K, int rows, int G) {
  if (w.s) return map_f8_codes(a, w.p, K, rows, G) && map_f8_scales(sc, w.s, K, rows, G);
  return map_weights(a, w.p, K, rows, G);
}

// Token-row source [rows, K] bf16, 128-byte swizzle, box of box_rows rows.
bool map_rows(CUtensorMap* m, const void* ptr, int K, int rows, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(kTileK), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            box_rows == 1 ? CU_TENSOR_MAP_L2_PROMOTION_L2_128B : CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// An expert GEMM's output rows [rows, cols] bf16, stored by the epilogue in
// boxes of 32 columns x 16 rows (64-byte row segments, no swizzle).
bool map_out(CUtensorMap* m, const void* ptr, int cols, int rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
  cuuint32_t box[2] = {32, 16};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The four token-row maps of one source: boxes of 16, 32, 64 and 128 rows.
bool map_rows_set(CUtensorMap (&m)[4], const void* ptr, int K, int rows) {
  for (int b = 0; b < 4; ++b)
    if (!map_rows(&m[b], ptr, K, rows, kRowPad << b)) return false;
  return true;
}

void copy_set(CUtensorMap (&dst)[4], const CUtensorMap (&src)[4]) {
  for (int b = 0; b < 4; ++b) dst[b] = src[b];
}

int pick_nmax(double rows_per_expert) {
  int n = 16;
  while (n < 256 && n < rows_per_expert * 1.25) n *= 2;
  return n;
}

int check_ws(const Plan& p, const void* ws, size_t bytes) {
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0 || bytes < p.total) return MOE_ERR_WORKSPACE;
  return MOE_OK;
}

int check_device(DeviceInfo* di) {
  if (device_info(di) != MOE_OK || !di->ok) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

cudaStream_t as_stream(moe_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }

// ---- the steps, after validation ----

// The router GEMM of plan p: partial logits [router_split, T, E] fp32 at
// `logits`, on single CTAs or CTA pairs as the plan chose.
int launch_router_gemm(const Plan& p, const DeviceInfo& di, const void* x, const void* W_router, float* logits,
                       uint32_t* err, cudaStream_t st) {
  GemmParams g;
  std::memset(&g, 0, sizeof g);
  if (!map_weights(&g.mapA[0], W_router, p.d, p.E, 1) || !map_rows_set(g.mapB[0], x, p.d, p.T))
    return MOE_ERR_CUDA;
  g.mapA[1] = g.mapA[2] = g.mapA[3] = g.mapA[0];
  copy_set(g.mapB[1], g.mapB[0]);
  g.num_units_host = p.router_units;
  g.out_r = logits;
  g.err = err;
  g.T = p.T; g.Tp = p.router_Tp; g.E = p.E; g.d = p.d; g.f = p.f; g.fs = p.fs;
  g.nmax = p.nmax_r;
  g.router_nwb = p.router_nwb;
  g.router_split = p.router_split;
  g.router_kbs = p.router_kbs;
  g.timeout_ns = kWaitTimeoutNs;
  g.nbuf = 512 / p.nmax_r < 8 ? 512 / p.nmax_r : 8;   // partial-logit buffers drained in turn
  int stages = 0;
  if (p.router_pair) {
    const size_t smem = gemm_pair_smem_bytes(kModeRouter, p.nmax_r, &stages);
    g.stages = stages;
    const int grid = 2 * p.router_units < di.sms ? 2 * p.router_units : di.sms;
    return launch_gemm_pair(kModeRouter, g, grid, smem, st);
  }
  const size_t smem = gemm_smem_bytes(kModeRouter, p.nmax_r, &stages);
  g.stages = stages;
  const int grid = p.router_units < di.sms ? p.router_units : di.sms;
  return launch_gemm(kModeRouter, g, grid, smem, st);
}

int run_route(const Plan& p, const DeviceInfo& di, const void* x, const void* W_router, const float* bias,
              int score_fn, int norm_topk, float route_scale, int32_t* topk_idx, float* topk_w, char* ws,
              cudaStream_t st) {
  if (cudaMemsetAsync(ws + p.err, 0, sizeof(uint32_t), st) != cudaSuccess) return MOE_ERR_CUDA;
  float* logits = reinterpret_cast<float*>(ws + p.logits);
  uint32_t* err = reinterpret_cast<uint32_t*>(ws + p.err);
  const int rc = launch_router_gemm(p, di, x, W_router, logits, err, st);
  if (rc != MOE_OK) return rc;
  return launch_topk(logits, p.router_split, bias, p.T, p.E, p.k, score_fn, norm_topk, route_scale, topk_idx,
                     topk_w, err, st);
}

int run_gate_up(const Plan& p, const DeviceInfo& di, const void* x, Wt Wg, Wt Wu, Wt Wsg, Wt Wsu, char* ws,
                cudaStream_t st) {
  GemmParams g;
  std::memset(&g, 0, sizeof g);
  const bool f8 = Wg.s != nullptr;
  if (!map_weight_operand(&g.mapA[0], &g.mapS[0], Wg, p.d, p.f, p.E) ||
      !map_weight_operand(&g.mapA[1], &g.mapS[1], Wu, p.d, p.f, p.E) || !map_rows_set(g.mapB[0], x, p.d, p.T) ||
      !map_rows(&g.mapX, x, p.d, p.T, 1))
    return MOE_ERR_CUDA;
  if (p.S > 0) {
    if (!map_weight_operand(&g.mapA[2], &g.mapS[2], Wsg, p.d, p.fs, p.S) ||
        !map_weight_operand(&g.mapA[3], &g.mapS[3], Wsu, p.d, p.fs, p.S))
      return MOE_ERR_CUDA;
  } else {
    g.mapA[2] = g.mapA[0];
    g.mapA[3] = g.mapA[1];
    g.mapS[2] = g.mapS[0];
    g.mapS[3] = g.mapS[1];
  }
  copy_set(g.mapB[1], g.mapB[0]);
  if (!map_out(&g.mapO[0], ws + p.Hr, p.f, p.Rcap)) return MOE_ERR_CUDA;
  if (p.S > 0) {
    if (!map_out(&g.mapO[1], ws + p.Hs, p.fs, p.S * p.Tp)) return MOE_ERR_CUDA;
  } else {
    g.mapO[1] = g.mapO[0];
  }
  g.units = reinterpret_cast<const int4*>(ws + p.units1);
  g.plan_tag_dev = reinterpret_cast<const int*>(ws + p.nunits) + 3;
  g.plan_tag = plan_tag(p);
  g.num_units_dev = reinterpret_cast<const int*>(ws + p.nunits);
  g.perm = reinterpret_cast<const int*>(ws + p.perm);
  g.x = x;
  g.out_r = ws + p.Hr;
  g.out_s = ws + p.Hs;
  g.err = reinterpret_cast<uint32_t*>(ws + p.err);
  g.T = p.T; g.Tp = p.Tp; g.E = p.E; g.d = p.d; g.f = p.f; g.fs = p.fs;
  g.nmax = p.nmax1;
  g.timeout_ns = kWaitTimeoutNs;
  g.weights_evict_first = p.weights_evict_first;
  int stages = 0;
  g.nbuf = (2 * p.nmax1 <= 256) ? 2 : 1;
  if (f8) {
    int raw = 0, tok = 0;
    g.nbuf = (4 * p.nmax1 <= 256) ? 2 : 1;      // accumulators below the widened tiles
    const size_t smem = gemm_f8_smem_bytes(kModeGateUp, p.nmax1, &stages, &tok, &raw);
    g.stages = stages;
    g.tok_stages = tok;
    g.raw_stages = raw;
    return launch_gemm(kModeGateUp, g, di.sms, smem, st, true);
  }
  if (p.pair1) {
    const size_t smem = gemm_pair_smem_bytes(kModeGateUp, p.nmax1, &stages);
    g.stages = stages;
    return launch_gemm_pair(kModeGateUp, g, di.sms, smem, st);
  }
  const size_t smem = gemm_smem_bytes(kModeGateUp, p.nmax1, &stages);
  g.stages = stages;
  return launch_gemm(kModeGateUp, g, di.sms, smem, st);
}

int run_down(const Plan& p, const DeviceInfo& di, Wt Wd, Wt Wsd, char* ws, cudaStream_t st) {
  GemmParams g;
  std::memset(&g, 0, sizeof g);
  const bool f8 = Wd.s != nullptr;
  if (!map_weight_operand(&g.mapA[0], &g.mapS[0], Wd, p.f, p.d, p.E) ||
      !map_rows_set(g.mapB[0], ws + p.Hr, p.f, p.Rcap))
    return MOE_ERR_CUDA;
  if (p.S > 0) {
    if (!map_weight_operand(&g.mapA[2], &g.mapS[2], Wsd, p.fs, p.d, p.S) ||
        !map_rows_set(g.mapB[1], ws + p.Hs, p.fs, p.S * p.Tp))
      return MOE_ERR_CUDA;
  } else {
    g.mapA[2] = g.mapA[0];
    g.mapS[2] = g.mapS[0];
    copy_set(g.mapB[1], g.mapB[0]);
  }
  g.mapA[1] = g.mapA[0];
  g.mapA[3] = g.mapA[2];
  g.mapS[1] = g.mapS[0];
  g.mapS[3] = g.mapS[2];
  if (!map_out(&g.mapO[0], ws + p.Yr, p.d, p.Rcap)) return MOE_ERR_CUDA;
  if (p.S > 0) {
    if (!map_out(&g.mapO[1], ws + p.Ys, p.d, p.S * p.Tp)) return MOE_ERR_CUDA;
  } else {
    g.mapO[1] = g.mapO[0];
  }
  g.units = reinterpret_cast<const int4*>(ws + p.units2);
  g.plan_tag_dev = reinterpret_cast<const int*>(ws + p.nunits) + 3;
  g.plan_tag = plan_tag(p);
  g.num_units_dev = reinterpret_cast<const int*>(ws + p.nunits) + 1;
  g.roww = reinterpret_cast<const float*>(ws + p.roww);
  g.out_r = ws + p.Yr;
  g.out_s = ws + p.Ys;
  g.err = reinterpret_cast<uint32_t*>(ws + p.err);
  g.T = p.T; g.Tp = p.Tp; g.E = p.E; g.d = p.d; g.f = p.f; g.fs = p.fs;
  g.nmax = p.nmax2;
  g.timeout_ns = kWaitTimeoutNs;
  g.weights_evict_first = p.weights_evict_first;
  int stages = 0;
  if (f8) {
    int raw = 0, tok = 0;
    g.nbuf = (4 * p.nmax2 <= 256) ? 2 : 1;      // accumulators below the widened tiles
    const size_t smem = gemm_f8_smem_bytes(kModeDown, p.nmax2, &stages, &tok, &raw);
    g.stages = stages;
    g.tok_stages = tok;
    g.raw_stages = raw;
    return launch_gemm(kModeDown, g, di.sms, smem, st, true);
  }
  if (p.pair2) {
    g.nbuf = (p.nmax2 <= 256) ? 2 : 1;          // one accumulator per CTA
    const size_t smem = gemm_pair_smem_bytes(kModeDown, p.nmax2, &stages);
    g.stages = stages;
    return launch_gemm_pair(kModeDown, g, di.sms, smem, st);
  }
  g.nbuf = (2 * p.nmax2 <= 256) ? 2 : 1;
  const size_t smem = gemm_smem_bytes(kModeDown, p.nmax2, &stages);
  g.stages = stages;
  return launch_gemm(kModeDown, g, di.sms, smem, st);
}

int check_route_args(const void* x, const void* W_router, const float* bias, int score_fn, int norm_topk,
                     float route_scale, const void* topk_idx, const void* topk_w) {
  if (!x || !W_router || !topk_idx || !topk_w) return MOE_ERR_INVALID_ARG;
  if (score_fn < MOE_SCORE_SOFTMAX || score_fn > MOE_SCORE_SQRT_SOFTPLUS) return MOE_ERR_INVALID_ARG;
  if (norm_topk != 0 && norm_topk != 1) return MOE_ERR_INVALID_ARG;
  if (!std::isfinite(route_scale)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(W_router) || !aligned16(topk_idx) || !aligned16(topk_w) ||
      (bias && !aligned16(bias)))
    return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

int check_expert_args(const Plan& p, const void* Wg, const void* Wu, const void* Wd, const void* Wsg,
                      const void* Wsu, const void* Wsd) {
  if (!Wg || !Wu || !Wd) return MOE_ERR_INVALID_ARG;
  if (p.S > 0 && (!Wsg || !Wsu || !Wsd)) return MOE_ERR_INVALID_ARG;
  if (p.S == 0 && (Wsg || Wsu || Wsd)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(Wg) || !aligned16(Wu) || !aligned16(Wd)) return MOE_ERR_UNSUPPORTED;
  if (p.S > 0 && (!aligned16(Wsg) || !aligned16(Wsu) || !aligned16(Wsd))) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

// Steps a3..a7 on a routing already in topk_idx / topk_w.
int experts_impl(const Plan& p, const DeviceInfo& di, const void* x, const int32_t* topk_idx, const float* topk_w,
                 Wt W_gate, Wt W_up, Wt W_down, Wt W_shared_gate, Wt W_shared_up, Wt W_shared_down,
                 const void* W_shared_gate_vec, void* out, char* ws, cudaStream_t st) {
  int rc = launch_permute(p, topk_idx, topk_w, ws, st);
  if (rc == MOE_OK) rc = run_gate_up(p, di, x, W_gate, W_up, W_shared_gate, W_shared_up, ws, st);
  if (rc == MOE_OK) rc = run_down(p, di, W_down, W_shared_down, ws, st);
  if (rc == MOE_OK) rc = launch_combine(p, out, ws, x, W_shared_gate_vec, st);
  return rc;
}

int forward_impl(const Plan& p, const DeviceInfo& di, const void* x, const void* W_router,
                 const float* expert_bias, Wt W_gate, Wt W_up, Wt W_down, Wt W_shared_gate, Wt W_shared_up,
                 Wt W_shared_down, const void* W_shared_gate_vec, int score_fn, int norm_topk, float route_scale, void* out,
                 int32_t* topk_idx, float* topk_w, char* ws, cudaStream_t st) {
  int rc = run_route(p, di, x, W_router, expert_bias, score_fn, norm_topk, route_scale, topk_idx, topk_w, ws, st);
  if (rc == MOE_OK)
    rc = experts_impl(p, di, x, topk_idx, topk_w, W_gate, W_up, W_down, W_shared_gate, W_shared_up, W_shared_down,
                      W_shared_gate_vec, out, ws, st);
  return rc;
}

bool f8_given(const moe_fp8_weight* w) { return w && w->codes && w->scales; }
bool f8_aligned(const moe_fp8_weight* w) { return aligned16(w->codes) && aligned16(w->scales); }

int check_f8_expert_args(const Plan& p, const moe_fp8_weight* Wg, const moe_fp8_weight* Wu,
                         const moe_fp8_weight* Wd, const moe_fp8_weight* Wsg, const moe_fp8_weight* Wsu,
                         const moe_fp8_weight* Wsd) {
  if (!f8_given(Wg) || !f8_given(Wu) || !f8_given(Wd)) return MOE_ERR_INVALID_ARG;
  if (p.S > 0 && (!f8_given(Wsg) || !f8_given(Wsu) || !f8_given(Wsd))) return MOE_ERR_INVALID_ARG;
  if (p.S == 0 && (Wsg || Wsu || Wsd)) return MOE_ERR_INVALID_ARG;
  if (!f8_aligned(Wg) || !f8_aligned(Wu) || !f8_aligned(Wd)) return MOE_ERR_UNSUPPORTED;
  if (p.S > 0 && (!f8_aligned(Wsg) || !f8_aligned(Wsu) || !f8_aligned(Wsd))) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

Wt wt(const moe_fp8_weight* w) { return w ? Wt(w->codes, w->scales) : Wt(); }

int check_gate_vec(const Plan& p, const void* W_shared_gate_vec) {
  if (!W_shared_gate_vec) return MOE_OK;
  if (p.S == 0) return MOE_ERR_INVALID_ARG;
  return aligned16(W_shared_gate_vec) ? MOE_OK : MOE_ERR_UNSUPPORTED;
}

}  // namespace

// SMs of the current device, for the plan's tiling rules; 148 (a B200) when
// no device can be queried (moe_workspace_bytes on a host without a GPU).
static int plan_sms() {
  DeviceInfo di;
  if (device_info(&di) == MOE_OK && di.sms > 0) return di.sms;
  return 148;
}

int make_plan(const moe_shape* s, Plan* p, bool f8) {
  if (!s || !p) return MOE_ERR_INVALID_ARG;
  const int T = s->T, d = s->d_model, E = s->E, k = s->k, f = s->d_ff, S = s->n_shared;
  const int fs = S > 0 ? s->d_ff_shared : 0;
  if (T < 1 || E < 1 || k < 1 || k > E || d < 1 || f < 1 || S < 0) return MOE_ERR_INVALID_ARG;
  if (S > 0 && fs < 1) return MOE_ERR_INVALID_ARG;
  if (E > kMaxE || k > kMaxK || S > kMaxShared) return MOE_ERR_UNSUPPORTED;
  if (d % 64 || f % 64 || (S > 0 && fs % 64)) return MOE_ERR_UNSUPPORTED;
  if (T > (1 << 22) || d > (1 << 16) || f > (1 << 16) || fs > (1 << 16)) return MOE_ERR_UNSUPPORTED;
  if (static_cast<long long>(T) * k + static_cast<long long>(E) * 2 * kRowPad > (1ll << 30)) return MOE_ERR_UNSUPPORTED;
  Plan q;
  std::memset(&q, 0, sizeof q);
  q.T = T; q.d = d; q.E = E; q.k = k; q.f = f; q.S = S; q.fs = fs;
  const int sms = plan_sms();
  const int half_sms = sms / 2;
  const double rows_per_expert = static_cast<double>(T) * k / E;
  q.nmax1 = pick_nmax(rows_per_expert);
  // Experts of 96+ rows on average: both expert GEMMs run on CTA pairs.
  // Gate/up: each CTA loads half of every token tile (runs then come in
  // multiples of 32).  Down: each CTA holds one 256-column accumulator
  // instead of two, so tensor memory takes two buffers and a unit's epilogue
  // overlaps the next unit's MMAs.  Measured faster than single CTAs at 128,
  // 170 and 400 rows per expert; smaller experts keep single CTAs.
  const int pair_bf16 = (q.nmax1 >= 64 && rows_per_expert >= 96.0) ? 1 : 0;
  // FP8 expert weights: single CTAs, token runs of at most 128 (their
  // accumulators share tensor memory with the widened weight tiles).  The
  // workspace layout is the same for both weight formats.
  if (f8 && q.nmax1 > 128) q.nmax1 = 128;
  q.nmax2 = q.nmax1;
  q.pair1 = f8 ? 0 : pair_bf16;
  q.pair2 = f8 ? 0 : pair_bf16;
  q.rowpad = pair_bf16 ? 2 * kRowPad : kRowPad;
  // Experts that fit one token run on average read each weight tile once.
  q.weights_evict_first = rows_per_expert <= 0.75 * q.nmax1 ? 1 : 0;
  q.Tp = ceil_div(T, q.rowpad) * q.rowpad;
  q.Rcap = ceil_div(T * k + E * (q.rowpad - 1), q.rowpad) * q.rowpad;
  q.nb = ceil_div(T, kPermBlock);
  q.nwbE = ceil_div(E, kTileRows);
  const int rows1 = q.pair1 ? 2 * kTileRows : kTileRows;   // weight rows per gate/up unit
  const int ncap = q.nmax1 < 128 ? q.nmax1 : 128;          // unit-list bounds cover both formats
  const int rows2 = 2 * kTileRows;                          // weight rows per down unit
  q.nwb1 = ceil_div(f, rows1);
  q.nwb1s = S > 0 ? ceil_div(fs, rows1) : 0;
  q.nwb2 = ceil_div(d, rows2);
  // Router: runs of up to 128 tokens (their fp32 logit sums live in
  // registers) when that still gives every SM a unit; else runs of 64 or
  // narrower while most SMs stay busy.
  q.nmax_r = 16;
  q.router_pair = 0;
  if (static_cast<long long>(q.nwbE) * ceil_div(q.Tp, 128) >= sms) {
    q.nmax_r = 128;
  } else {
    for (int n = 64; n >= 16; n >>= 1) {
      if (static_cast<long long>(q.nwbE) * ceil_div(q.Tp, n) >= half_sms) {
        q.nmax_r = n;
        break;
      }
    }
  }
  // Too few runs to fill the SMs (decode-sized batches): split K as well, each
  // slice writing its own partial logits, summed in slice order by top-k.
  {
    const int base = q.nwbE * ceil_div(q.Tp, q.nmax_r);
    const int KB = d / kTileK;
    const int Tp32 = ceil_div(T, 2 * kRowPad) * 2 * kRowPad;
    int split = 1;
    if (base < half_sms) {
      split = sms / base;
      if (split > kMaxRouterSplit) split = kMaxRouterSplit;
      if (split > KB) split = KB;
      if (split < 1) split = 1;
    } else {
      // Enough runs for most SMs: the launch is bound by what each SM must
      // load, (units per SM) x (128 + its token rows) x its K slice.  Wider
      // runs re-read W_router less; a CTA pair (256 experts x 256 tokens per
      // unit, each CTA loading 128 of each) halves the bytes per logit
      // again (pairs with 128-token runs measured slower than single CTAs
      // on prefill_softmax); a second K slice spreads the units over more
      // SMs but adds a partial-logit array, written here and read back by
      // top-k.  Another tiling replaces the rule above only when this model
      // calls it clearly cheaper (measured: prefill_softmax routing
      // 32.5 -> 26.4 us with 128-token runs in two slices).
      auto cost = [&](int pr, int n, int sp) {
        const int kbs = ceil_div(KB, sp);
        const int ns = ceil_div(KB, kbs);
        const int slots = pr ? half_sms : sms;
        const long long units = static_cast<long long>(ceil_div(E, pr ? 2 * kTileRows : kTileRows)) *
                                ceil_div(pr ? Tp32 : q.Tp, n) * ns;
        const long long per = (units + slots - 1) / slots;
        const double ingest = static_cast<double>(per) * (kTileRows + (pr ? n / 2 : n)) * kbs * kTileK * 2;
        const double partials = static_cast<double>(ns - 1) * T * E * 4 * 2;
        return ingest / 47e9 + partials / 6.5e12;
      };
      const double c0 = cost(0, q.nmax_r, 1);
      double best = 0.9 * c0;
      int bn = q.nmax_r;
      for (int pr = 0; pr <= 1; ++pr)
        for (int n = pr ? 256 : 32; n <= (pr ? 256 : 128); n <<= 1)
          for (int sp = 1; sp <= 2 && sp <= KB; ++sp) {
            const double c = cost(pr, n, sp);
            if (c < best) {
              best = c;
              bn = n;
              split = sp;
              q.router_pair = pr;
            }
          }
      q.nmax_r = bn;
    }
    q.router_nwb = q.router_pair ? ceil_div(E, 2 * kTileRows) : q.nwbE;
    q.router_Tp = q.router_pair ? Tp32 : q.Tp;
    const int runs = q.router_nwb * ceil_div(q.router_Tp, q.nmax_r);
    q.router_kbs = ceil_div(KB, split);
    q.router_split = ceil_div(KB, q.router_kbs);   // no empty slice
    q.router_units = runs * q.router_split;
  }
  q.shared_units1 = S * q.nwb1s * ceil_div(q.Tp, q.nmax1);
  q.shared_units2 = S * q.nwb2 * ceil_div(q.Tp, q.nmax2);
  const int nwb1cap = ceil_div(f, kTileRows), nwb1scap = S > 0 ? ceil_div(fs, kTileRows) : 0;
  q.U1cap = S * nwb1scap * ceil_div(q.Tp, ncap) + nwb1cap * (q.Rcap / ncap + E);
  q.U2cap = S * q.nwb2 * ceil_div(q.Tp, ncap) + q.nwb2 * (q.Rcap / ncap + E);

  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  };
  q.err = take(16);
  q.nunits = take(16);
  q.logits = take(static_cast<size_t>(q.router_split) * T * E * 4);
  q.blkcnt = take(static_cast<size_t>(q.nb) * E * 4);
  q.counts = take(static_cast<size_t>(E) * 4);
  q.roff = take(static_cast<size_t>(E + 1) * 4);
  q.perm = take(static_cast<size_t>(q.Rcap) * 4);
  q.roww = take(static_cast<size_t>(q.Rcap) * 4);
  q.inv = take(static_cast<size_t>(T) * k * 4);
  q.units1 = take(static_cast<size_t>(q.U1cap) * 16);
  q.units2 = take(static_cast<size_t>(q.U2cap) * 16);
  q.Hr = take(static_cast<size_t>(q.Rcap) * f * 2);
  q.Hs = take(static_cast<size_t>(S) * q.Tp * (fs > 0 ? fs : 0) * 2);
  q.Yr = take(static_cast<size_t>(q.Rcap) * d * 2);
  q.Ys = take(static_cast<size_t>(S) * q.Tp * d * 2);
  q.xstage = take(static_cast<size_t>(T) * d * 2);
  q.ostage = take(static_cast<size_t>(T) * d * 2);
  q.istage = take(static_cast<size_t>(T) * k * 4);
  q.wstage = take(static_cast<size_t>(T) * k * 4);
  q.sgate = take(static_cast<size_t>(T) * (S > 0 ? S : 1) * 4);
  q.total = off;
  *p = q;
  return MOE_OK;
}

std::mutex& host_state_mutex() {
  static std::mutex m;
  return m;
}

int device_info(DeviceInfo* info) {
  static DeviceInfo cache[64];
  static std::atomic<int> have[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MOE_ERR_CUDA;
  if (!have[dev].load(std::memory_order_acquire)) {
    std::lock_guard<std::mutex> lock(host_state_mutex());
    if (have[dev].load(std::memory_order_relaxed)) {
      *info = cache[dev];
      return MOE_OK;
    }
    DeviceInfo d;
    std::memset(&d, 0, sizeof d);
    int major = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.max_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
      return MOE_ERR_CUDA;
    d.ok = (major == 10 && d.max_smem_optin >= 232448 && encode_fn() != nullptr) ? 1 : 0;
    cache[dev] = d;
    have[dev].store(1, std::memory_order_release);
  }
  *info = cache[dev];
  return MOE_OK;
}

}  // namespace moe

using namespace moe;

extern "C" {

int moe_version(void) { return 100; }

const char* moe_status_string(int status) {
  switch (status) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG: invalid argument";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED: unsupported shape, alignment or device";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE: workspace missing, misaligned or too small";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA: CUDA call or kernel launch failed";
    case MOE_ERR_DEVICE_TIMEOUT: return "MOE_ERR_DEVICE_TIMEOUT: a bounded device-side wait ran out";
    case MOE_ERR_SCRATCH_LIMIT:
      return "MOE_ERR_SCRATCH_LIMIT: T * E fp32 logits exceed the 16 MiB built-in scratch of moe_route_noalloc";
    case MOE_ERR_NONFINITE: return "MOE_ERR_NONFINITE: NaN or infinite router logits, selection keys or weights";
    default: return "unknown status";
  }
}

size_t moe_workspace_bytes(const moe_shape* shape) {
  Plan p;
  if (make_plan(shape, &p) != MOE_OK) return 0;
  return p.total;
}

int moe_route(const moe_shape* shape, const void* x, const void* W_router, const float* expert_bias,
              int score_fn, int norm_topk, float route_scale, int32_t* topk_idx, float* topk_w, void* workspace,
              size_t workspace_bytes, moe_stream_t stream) {
  Plan p;
  int rc = make_plan(shape, &p);
  if (rc != MOE_OK) return rc;
  if ((rc = check_route_args(x, W_router, expert_bias, score_fn, norm_topk, route_scale, topk_idx, topk_w)) != MOE_OK)
    return rc;
  if ((rc = check_ws(p, workspace, workspace_bytes)) != MOE_OK) return rc;
  DeviceInfo di;
  if ((rc = check_device(&di)) != MOE_OK) return rc;
  return run_route(p, di, x, W_router, expert_bias, score_fn, norm_topk, route_scale, topk_idx, topk_w,
                   static_cast<char*>(workspace), as_stream(stream));
}

int moe_permute(const moe_shape* shape, const int32_t* topk_idx, const float* topk_w, void* workspace,
                size_t workspace_bytes, moe_stream_t stream) {
  Plan p;
  int rc = make_plan(shape, &p);
  if (rc != MOE_OK) return rc;
  if (!topk_idx || !topk_w) return MOE_ERR_INVALID_ARG;
  if (!aligned16(topk_idx) || !aligned16(topk_w)) return MOE_ERR_UNSUPPORTED;
  if ((rc = check_ws(p, workspace, workspace_bytes)) != MOE_OK) return rc;
  DeviceInfo di;
  if ((rc = check_device(&di)) != MOE_OK) return rc;
  return launch_permute(p, topk_idx, topk_w, static_cast<char*>(workspace), as_stream(stream));
}

int moe_expert_gate_up(const moe_shape* shape, const void* x, const void* W_gate, const void* W_up,
                       const void* W_shared_gate, const void* W_shared_up, void* workspace, size_t workspace_bytes,
                       moe_stream_t stream) {
  Plan p;
  int rc = make_plan(shape, &p);
  if (rc != MOE_OK) return rc;
  if (!x || !W_gate || !W_up) return MOE_ERR_INVALID_ARG;
  if (p.S > 0 && (!W_shared_gate || !W_shared_up)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(W_gate) || !aligned16(W_up) ||
      (p.S > 0 && (!aligned16(W_shared_gate) || !aligned16(W_shared_up))))
    return MOE_ERR_UNSUPPORTED;
  if ((rc = check_ws(p, workspace, workspace_bytes)) != MOE_OK) return rc;
  DeviceInfo di;
  if ((rc = check_device(&di)) != MOE_OK) return rc;
  return run_gate_up(p, di, x, W_gate, W_up, W_shared_gate, W_shared_up, static_cast<char*>(workspace),
                     as_stream(stream));
}

int moe_expert_down(const moe_shape* shape, const void* W_down, const void* W_shared_down, void* workspace,
                    size_t workspace_bytes, moe_stream_t stream) {
  Plan p;
  int rc = make_plan(shape, &p);
  if (rc != MOE_OK) return rc;
  if (!W_down || (p.S > 0 && !W_shared_down)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(W_down) || (p.S > 0 && !aligned16(W_shared_down))) return MOE_ERR_UNSUPPORTED;
  if ((rc = check_ws(p, workspace, workspace_bytes)) != MOE_OK) return rc;
  DeviceInfo di;
  if ((rc = check_device(&di)) != MOE_OK) return rc;
  return run_down(p, di, W_down, W_shared_down, static_cast<char*>(workspace), as_stream(stream));
}

int moe_combine(const moe_shape* shape, const void* x, const void* W_shared_gate_vec, void* out, void* workspace,
                size_t workspace_bytes, moe_stream_t stream) {
  Plan p;
  int rc = make_plan(shape, &p);
  if (rc != MOE_OK) return rc;
  if (!out) return MOE_ERR_INVALID_ARG;
  if (!aligned16(out)) return MOE_ERR_UNSUPPORTED;
  if ((rc = check_gate_vec(p, W_shared_gate_vec)) != MOE_OK) return rc;
  if (W_shared_gate_vec && !x) return MOE_ERR_INVALID_ARG;
  if (W_shared_gate_vec && !aligned16(x)) return MOE_ERR_UNSUPPORTED;
  if ((rc = check_ws(p, workspace, workspace_bytes)) != MOE_OK) return rc;
  DeviceInfo di;
  if ((rc = check_device(&di)) != MOE_OK) return rc;
  return launch_combine(p, out, static_cast<char*>(workspace), x, W_shared_gate_vec, as_stream(stream));
}

int moe_experts_forward(const moe_shape* shape, const void* x, const int32_t* topk_idx, const float* topk_w,
                        const void* W_gate, const void* W_up, const void* W_down, const void* W_shared_gate,
                        const void* W_shared_up, const void* W_shared_down, const void* W_shared_gate_vec, void* out,
                        void* workspace, size_t workspace_bytes, moe_stream_t stream) {
  Plan p;
  int rc = make_plan(shape, &p);
  if (rc != MOE_OK) return rc;
  if (!x || !topk_idx || !topk_w || !out) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(topk_idx) || !aligned16(topk_w) || !aligned16(out)) return MOE_ERR_UNSUPPORTED;
  if ((rc = check_expert_args(p, W_gate, W_up, W_down, W_shared_gate, W_shared_up, W_shared_down)) != MOE_OK)
    return rc;
  if ((rc = check_gate_vec(p, W_shared_gate_vec)) != MOE_OK) return rc;
  if ((rc = check_ws(p, workspace, workspace_bytes)) != MOE_OK) return rc;
  DeviceInfo di;
  if ((rc = check_device(&di)) != MOE_OK) return rc;
  char* ws = static_cast<char*>(workspace);
  cudaStream_t st = as_stream(stream);
  if (cudaMemsetAsync(ws + p.err, 0, sizeof(uint32_t), st) != cudaSuccess) return MOE_ERR_CUDA;
  return experts_impl(p, di, x, topk_idx, topk_w, W_gate, W_up, W_down, W_shared_gate, W_shared_up, W_shared_down,
                      W_shared_gate_vec, out, ws, st);
}

int moe_forward(const moe_shape* shape, const void* x, const void* W_router, const float* expert_bias,
                const void* W_gate, const void* W_up, const void* W_down, const void* W_shared_gate,
                const void* W_shared_up, const void* W_shared_down, const void* W_shared_gate_vec, int score_fn,
                int norm_topk, float route_scale, void* out, int32_t* topk_idx, float* topk_w, void* workspace,
                size_t workspace_bytes, moe_stream_t stream) {
  Plan p;
  int rc = make_plan(shape, &p);
  if (rc != MOE_OK) return rc;
  if ((rc = check_route_args(x, W_router, expert_bias, score_fn, norm_topk, route_scale, topk_idx, topk_w)) != MOE_OK)
    return rc;
  if ((rc = check_expert_args(p, W_gate, W_up, W_down, W_shared_gate, W_shared_up, W_shared_down)) != MOE_OK)
    return rc;
  if (!out) return MOE_ERR_INVALID_ARG;
  if (!aligned16(out)) return MOE_ERR_UNSUPPORTED;
  if ((rc = check_gate_vec(p, W_shared_gate_vec)) != MOE_OK) return rc;
  if ((rc = check_ws(p, workspace, workspace_bytes)) != MOE_OK) return rc;
  DeviceInfo di;
  if ((rc = check_device(&di)) != MOE_OK) return rc;
  return forward_impl(p, di, x, W_router, expert_bias, W_gate, W_up, W_down, W_shared_gate, W_shared_up,
                      W_shared_down, W_shared_gate_vec, score_fn, norm_topk, route_scale, out, topk_idx, topk_w,
                      static_cast<char*>(workspace), as_stream(stream));
}

int moe_forward_host(const moe_shape* shape, const void* x_host, const void* W_router, const float* expert_bias,
                     const void* W_gate, const void* W_up, const void* W_down, const void* W_shared_gate,
                     const void* W_shared_up, const void* W_shared_down, const void* W_shared_gate_vec,
                     int score_fn, int norm_topk, float route_scale, void* out_host, int32_t* topk_idx_host,
                     float* topk_w_host, void* workspace, size_t workspace_bytes, moe_stream_t stream) {
  Plan p;
  int rc = make_plan(shape, &p);
  if (rc != MOE_OK) return rc;
  if (!x_host || !out_host || !topk_idx_host || !topk_w_host) return MOE_ERR_INVALID_ARG;
  char* ws = static_cast<char*>(workspace);
  if ((rc = check_ws(p, workspace, workspace_bytes)) != MOE_OK) return rc;
  void* xd = ws + p.xstage;
  void* od = ws + p.ostage;
  int32_t* id = reinterpret_cast<int32_t*>(ws + p.istage);
  float* wd = reinterpret_cast<float*>(ws + p.wstage);
  if ((rc = check_route_args(xd, W_router, expert_bias, score_fn, norm_topk, route_scale, id, wd)) != MOE_OK)
    return rc;
  if ((rc = check_expert_args(p, W_gate, W_up, W_down, W_shared_gate, W_shared_up, W_shared_down)) != MOE_OK)
    return rc;
  if ((rc = check_gate_vec(p, W_shared_gate_vec)) != MOE_OK) return rc;
  DeviceInfo di;
  if ((rc = check_device(&di)) != MOE_OK) return rc;
  cudaStream_t st = as_stream(stream);
  const size_t xbytes = static_cast<size_t>(p.T) * p.d * 2;
  const size_t tkbytes = static_cast<size_t>(p.T) * p.k * 4;
  if (cudaMemcpyAsync(xd, x_host, xbytes, cudaMemcpyHostToDevice, st) != cudaSuccess) return MOE_ERR_CUDA;
  rc = forward_impl(p, di, xd, W_router, expert_bias, W_gate, W_up, W_down, W_shared_gate, W_shared_up,
                    W_shared_down, W_shared_gate_vec, score_fn, norm_topk, route_scale, od, id, wd, ws, st);
  if (rc != MOE_OK) return rc;
  if (cudaMemcpyAsync(out_host, od, xbytes, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaMemcpyAsync(topk_idx_host, id, tkbytes, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaMemcpyAsync(topk_w_host, wd, tkbytes, cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}

int moe_forward_fp8(const moe_shape* shape, const void* x, const void* W_router, const float* expert_bias,
                    const moe_fp8_weight* W_gate, const moe_fp8_weight* W_up, const moe_fp8_weight* W_down,
                    const moe_fp8_weight* W_shared_gate, const moe_fp8_weight* W_shared_up,
                    const moe_fp8_weight* W_shared_down, const void* W_shared_gate_vec, int score_fn, int norm_topk,
                    float route_scale, void* out, int32_t* topk_idx, float* topk_w, void* workspace,
                    size_t workspace_bytes, moe_stream_t stream) {
  Plan p;
  int rc = make_plan(shape, &p, true);
  if (rc != MOE_OK) return rc;
  if ((rc = check_route_args(x, W_router, expert_bias, score_fn, norm_topk, route_scale, topk_idx, topk_w)) != MOE_OK)
    return rc;
  if ((rc = check_f8_expert_args(p, W_gate, W_up, W_down, W_shared_gate, W_shared_up, W_shared_down)) != MOE_OK)
    return rc;
  if (!out) return MOE_ERR_INVALID_ARG;
  if (!aligned16(out)) return MOE_ERR_UNSUPPORTED;
  if ((rc = check_gate_vec(p, W_shared_gate_vec)) != MOE_OK) return rc;
  if ((rc = check_ws(p, workspace, workspace_bytes)) != MOE_OK) return rc;
  DeviceInfo di;
  if ((rc = check_device(&di)) != MOE_OK) return rc;
  return forward_impl(p, di, x, W_router, expert_bias, wt(W_gate), wt(W_up), wt(W_down), wt(W_shared_gate),
                      wt(W_shared_up), wt(W_shared_down), W_shared_gate_vec, score_fn, norm_topk, route_scale, out,
                      topk_idx, topk_w, static_cast<char*>(workspace), as_stream(stream));
}

int moe_permute_fp8(const moe_shape* shape, const int32_t* topk_idx, const float* topk_w, void* workspace,
                    size_t workspace_bytes, moe_stream_t stream) {
  Plan p;
  int rc = make_plan(shape, &p, true);
  if (rc != MOE_OK) return rc;
  if (!topk_idx || !topk_w) return MOE_ERR_INVALID_ARG;
  if (!aligned16(topk_idx) || !aligned16(topk_w)) return MOE_ERR_UNSUPPORTED;
  if ((rc = check_ws(p, workspace, workspace_bytes)) != MOE_OK) return rc;
  DeviceInfo di;
  if ((rc = check_device(&di)) != MOE_OK) return rc;
  return launch_permute(p, topk_idx, topk_w, static_cast<char*>(workspace), as_stream(stream));
}

int moe_expert_gate_up_fp8(const moe_shape* shape, const void* x, const moe_fp8_weight* W_gate,
                           const moe_fp8_weight* W_up, const moe_fp8_weight* W_shared_gate,
                           const moe_fp8_weight* W_shared_up, void* workspace, size_t workspace_bytes,
                           moe_stream_t stream) {
  Plan p;
  int rc = make_plan(shape, &p, true);
  if (rc != MOE_OK) return rc;
  if (!x || !f8_given(W_gate) || !f8_given(W_up)) return MOE_ERR_INVALID_ARG;
  if (p.S > 0 && (!f8_given(W_shared_gate) || !f8_given(W_shared_up))) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !f8_aligned(W_gate) || !f8_aligned(W_up) ||
      (p.S > 0 && (!f8_aligned(W_shared_gate) || !f8_aligned(W_shared_up))))
    return MOE_ERR_UNSUPPORTED;
  if ((rc = check_ws(p, workspace, workspace_bytes)) != MOE_OK) return rc;
  DeviceInfo di;
  if ((rc = check_device(&di)) != MOE_OK) return rc;
  return run_gate_up(p, di, x, wt(W_gate), wt(W_up), p.S > 0 ? wt(W_shared_gate) : Wt(),
                     p.S > 0 ? wt(W_shared_up) : Wt(), static_cast<char*>(workspace), as_stream(stream));
}

int moe_expert_down_fp8(const moe_shape* shape, const moe_fp8_weight* W_down, const moe_fp8_weight* W_shared_down,
                        void* workspace, size_t workspace_bytes, moe_stream_t stream) {
  Plan p;
  int rc = make_plan(shape, &p, true);
  if (rc != MOE_OK) return rc;
  if (!f8_given(W_down) || (p.S > 0 && !f8_given(W_shared_down))) return MOE_ERR_INVALID_ARG;
  if (!f8_aligned(W_down) || (p.S > 0 && !f8_aligned(W_shared_down))) return MOE_ERR_UNSUPPORTED;
  if ((rc = check_ws(p, workspace, workspace_bytes)) != MOE_OK) return rc;
  DeviceInfo di;
  if ((rc = check_device(&di)) != MOE_OK) return rc;
  return run_down(p, di, wt(W_down), p.S > 0 ? wt(W_shared_down) : Wt(), static_cast<char*>(workspace),
                  as_stream(stream));
}

int moe_rmsnorm(const moe_shape* shape, const void* x, const void* norm_gain, float eps, void* x_norm,
                moe_stream_t stream) {
  Plan p;
  int rc = make_plan(shape, &p);
  if (rc != MOE_OK) return rc;
  if (!x || !norm_gain || !x_norm || !(eps >= 0.0f) || !std::isfinite(eps)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(norm_gain) || !aligned16(x_norm)) return MOE_ERR_UNSUPPORTED;
  DeviceInfo di;
  if ((rc = check_device(&di)) != MOE_OK) return rc;
  return launch_rmsnorm(p, x, norm_gain, eps, x_norm, as_stream(stream));
}

int moe_forward_prenorm(const moe_shape* shape, const void* x, const void* norm_gain, float norm_eps,
                        const void* W_router, const float* expert_bias, const void* W_gate, const void* W_up,
                        const void* W_down, const void* W_shared_gate, const void* W_shared_up,
                        const void* W_shared_down, const void* W_shared_gate_vec, int score_fn, int norm_topk,
                        float route_scale, void* out, int32_t* topk_idx, float* topk_w, void* workspace,
                        size_t workspace_bytes, moe_stream_t stream) {
  Plan p;
  int rc = make_plan(shape, &p);
  if (rc != MOE_OK) return rc;
  if (!norm_gain || !(norm_eps >= 0.0f) || !std::isfinite(norm_eps)) return MOE_ERR_INVALID_ARG;
  if ((rc = check_route_args(x, W_router, expert_bias, score_fn, norm_topk, route_scale, topk_idx, topk_w)) != MOE_OK)
    return rc;
  if (!aligned16(norm_gain)) return MOE_ERR_UNSUPPORTED;
  if ((rc = check_expert_args(p, W_gate, W_up, W_down, W_shared_gate, W_shared_up, W_shared_down)) != MOE_OK)
    return rc;
  if (!out) return MOE_ERR_INVALID_ARG;
  if (!aligned16(out)) return MOE_ERR_UNSUPPORTED;
  if ((rc = check_gate_vec(p, W_shared_gate_vec)) != MOE_OK) return rc;
  if ((rc = check_ws(p, workspace, workspace_bytes)) != MOE_OK) return rc;
  DeviceInfo di;
  if ((rc = check_device(&di)) != MOE_OK) return rc;
  char* ws = static_cast<char*>(workspace);
  cudaStream_t st = as_stream(stream);
  void* xn = ws + p.xstage;
  if ((rc = launch_rmsnorm(p, x, norm_gain, norm_eps, xn, st)) != MOE_OK) return rc;
  // the shared-expert gate reads the block's input, i.e. the normalised rows
  return forward_impl(p, di, xn, W_router, expert_bias, W_gate, W_up, W_down, W_shared_gate, W_shared_up,
                      W_shared_down, W_shared_gate_vec, score_fn, norm_topk, route_scale, out, topk_idx, topk_w, ws,
                      st);
}

int moe_workspace_region(const moe_shape* shape, int region, size_t* offset, size_t* bytes) {
  Plan p;
  if (!offset || !bytes) return MOE_ERR_INVALID_ARG;
  if (make_plan(shape, &p) != MOE_OK) return MOE_ERR_INVALID_ARG;
  const size_t T = p.T, E = p.E, k = p.k, R = p.Rcap, S = p.S, Tp = p.Tp;
  switch (region) {
    case MOE_WS_LOGITS: *offset = p.logits; *bytes = static_cast<size_t>(p.router_split) * T * E * 4; break;
    case MOE_WS_COUNTS: *offset = p.counts; *bytes = E * 4; break;
    case MOE_WS_OFFSETS: *offset = p.roff; *bytes = (E + 1) * 4; break;
    case MOE_WS_PERM: *offset = p.perm; *bytes = R * 4; break;
    case MOE_WS_ROW_W: *offset = p.roww; *bytes = R * 4; break;
    case MOE_WS_INV: *offset = p.inv; *bytes = T * k * 4; break;
    case MOE_WS_H: *offset = p.Hr; *bytes = R * p.f * 2; break;
    case MOE_WS_H_SHARED: *offset = p.Hs; *bytes = S * Tp * p.fs * 2; break;
    case MOE_WS_Y: *offset = p.Yr; *bytes = R * p.d * 2; break;
    case MOE_WS_Y_SHARED: *offset = p.Ys; *bytes = S * Tp * p.d * 2; break;
    case MOE_WS_X_STAGE: *offset = p.xstage; *bytes = T * p.d * 2; break;
    case MOE_WS_WORK_COUNTS: *offset = p.nunits; *bytes = 16; break;
    case MOE_WS_WORK_GATE_UP: *offset = p.units1; *bytes = static_cast<size_t>(p.U1cap) * 16; break;
    case MOE_WS_WORK_DOWN: *offset = p.units2; *bytes = static_cast<size_t>(p.U2cap) * 16; break;
    default: return MOE_ERR_INVALID_ARG;
  }
  return MOE_OK;
}

int moe_device_status(const void* workspace, moe_stream_t stream) {
  if (!workspace) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = as_stream(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return MOE_ERR_CUDA;
  uint32_t word = 0;
  if (cudaMemcpy(&word, workspace, sizeof word, cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
  if (word & kDevErrTimeout) return MOE_ERR_DEVICE_TIMEOUT;
  if (word & (kDevErrBadRouting | kDevErrPlanMismatch)) return MOE_ERR_INVALID_ARG;
  if (word & kDevErrNonFinite) return MOE_ERR_NONFINITE;
  return MOE_OK;
}

int moe_debug_wait_timeout(void* workspace, size_t workspace_bytes, uint64_t timeout_ns, moe_stream_t stream) {
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 || workspace_bytes < 256)
    return MOE_ERR_WORKSPACE;
  DeviceInfo di;
  int rc = check_device(&di);
  if (rc != MOE_OK) return rc;
  if (timeout_ns < 1000000ull) timeout_ns = 1000000ull;
  if (timeout_ns > 1000000000ull) timeout_ns = 1000000000ull;
  if (cudaMemsetAsync(workspace, 0, sizeof(uint32_t), as_stream(stream)) != cudaSuccess) return MOE_ERR_CUDA;
  return launch_wait_timeout(reinterpret_cast<uint32_t*>(workspace), timeout_ns, as_stream(stream));
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Routing for callers that cannot allocate device memory.
//
// moe_route needs a caller-provided workspace for the fp32 logits between the
// router GEMM and the top-k kernel.  Some callers cannot hand one over: an
// inference-engine plugin whose per-call hook may not allocate, or a service
// whose device memory is entirely reserved up front by another allocator.
// moe_route_noalloc runs the same two kernels with that scratch in a
// fixed-size array compiled into this library instead.
namespace moe {
namespace {

constexpr size_t kNoAllocHeaderBytes = 256;                 // device error word, padded
constexpr size_t kNoAllocLogitBytes = size_t(16) << 20;     // fp32 logits: T * E <= 4,194,304
static __device__ __align__(256) unsigned char g_route_scratch[kNoAllocHeaderBytes + kNoAllocLogitBytes];

char* g_route_scratch_dev[64];    // device address of g_route_scratch, per device
std::atomic<int> g_route_scratch_ready[64];

// The host-side name g_route_scratch is not a device address: look up the
// device address once per device (with that device current) and reuse it.
int route_scratch_address(char** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MOE_ERR_CUDA;
  if (!g_route_scratch_ready[dev].load(std::memory_order_acquire)) {
    std::lock_guard<std::mutex> lock(host_state_mutex());
    if (!g_route_scratch_ready[dev].load(std::memory_order_relaxed)) {
      void* ptr = nullptr;
      if (cudaGetSymbolAddress(&ptr, g_route_scratch) != cudaSuccess || ptr == nullptr) return MOE_ERR_CUDA;
      g_route_scratch_dev[dev] = static_cast<char*>(ptr);
      g_route_scratch_ready[dev].store(1, std::memory_order_release);
    }
  }
  *out = g_route_scratch_dev[dev];
  return MOE_OK;
}

}  // namespace
}  // namespace moe

extern "C" int moe_route_noalloc(const moe_shape* shape, const void* x, const void* W_router,
                                 const float* expert_bias, int score_fn, int norm_topk, float route_scale,
                                 int32_t* topk_idx, float* topk_w, moe_stream_t stream) {
  Plan p;
  int rc = make_plan(shape, &p);
  if (rc != MOE_OK) return rc;
  if ((rc = check_route_args(x, W_router, expert_bias, score_fn, norm_topk, route_scale, topk_idx, topk_w)) != MOE_OK)
    return rc;
  const size_t slice_bytes = static_cast<size_t>(p.T) * static_cast<size_t>(p.E) * sizeof(float);
  if (slice_bytes > kNoAllocLogitBytes) return MOE_ERR_SCRATCH_LIMIT;
  if (static_cast<size_t>(p.router_split) * slice_bytes > kNoAllocLogitBytes) {
    // fewer K slices, so that their partial logits fit the scratch
    const int KB = p.d / kTileK;
    const int base = p.router_units / p.router_split;
    const int split = static_cast<int>(kNoAllocLogitBytes / slice_bytes);
    p.router_kbs = ceil_div(KB, split);
    p.router_split = ceil_div(KB, p.router_kbs);
    p.router_units = base * p.router_split;
  }
  DeviceInfo di;
  if ((rc = check_device(&di)) != MOE_OK) return rc;
  char* scratch = nullptr;
  if ((rc = route_scratch_address(&scratch)) != MOE_OK) return rc;
  cudaStream_t st = as_stream(stream);
  uint32_t* err = reinterpret_cast<uint32_t*>(scratch);
  float* logits = reinterpret_cast<float*>(scratch + kNoAllocHeaderBytes);
  // The array keeps the previous call's contents: the error word must start at zero.
  if (cudaMemsetAsync(err, 0, sizeof(uint32_t), st) != cudaSuccess) return MOE_ERR_CUDA;
  if ((rc = launch_router_gemm(p, di, x, W_router, logits, err, st)) != MOE_OK) return rc;
  return launch_topk(logits, p.router_split, expert_bias, p.T, p.E, p.k, score_fn, norm_topk, route_scale, topk_idx,
                     topk_w, err, st);
}
