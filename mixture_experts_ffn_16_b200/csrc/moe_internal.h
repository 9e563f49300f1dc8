// moe_internal.h - host-side plan of one call: workspace carve-up, tiling
// choices and the launchers of each kernel.  Shared by the .cu files of
// libmoe.so only.
#pragma once

#include <atomic>
#include <cstddef>
#include <cstdint>
#include <mutex>
#include <cuda.h>
#include <cuda_runtime.h>

#include "moe.h"

namespace moe {

constexpr int kMaxE = 2048;
constexpr int kMaxK = 32;
constexpr int kMaxRouterSplit = 16;   // K slices of the router GEMM for small batches
constexpr int kMaxShared = 8;
constexpr int kTileRows = 128;     // weight rows per GEMM work unit (MMA M)
constexpr int kTileK = 64;         // bf16 elements per 128-byte swizzled row
constexpr int kRowPad = 16;        // expert segments are padded to this many rows (MMA N step)
constexpr int kPermBlock = 256;    // tokens per block in the permute kernels
constexpr uint64_t kWaitTimeoutNs = 2000000000ull;  // 2 s bound on every device-side wait

// Host-side state kept per device for the life of the process (kernel
// attributes, device queries, the no-alloc scratch address) is filled in
// under this lock, so the entry points may be called from several host
// threads at once.
std::mutex& host_state_mutex();

// Raises `kernel`'s dynamic shared-memory limit on the current device to at
// least `bytes`; `limit` records per device what is set already.  The limit
// only grows, so a launch that needs less is never refused.
template <typename... KArgs>
inline int raise_smem_limit(void (*kernel)(KArgs...), std::atomic<int> (&limit)[64], int bytes) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MOE_ERR_CUDA;
  if (limit[dev].load(std::memory_order_acquire) >= bytes) return MOE_OK;
  std::lock_guard<std::mutex> lock(host_state_mutex());
  if (limit[dev].load(std::memory_order_relaxed) >= bytes) return MOE_OK;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
    return MOE_ERR_CUDA;
  limit[dev].store(bytes, std::memory_order_release);
  return MOE_OK;
}

#ifdef __CUDACC__
// Every kernel of the block is launched with programmatic stream
// serialisation: its CTAs may be scheduled as the previous kernel's CTAs
// exit, before that kernel as a whole has completed, and each kernel runs its
// set-up (barrier initialisation, tensor-memory allocation, descriptor
// prefetch) and then waits in `griddepcontrol.wait` for the previous kernel to
// complete and its writes to be visible before it touches global memory.
// Because every kernel waits before it completes, a kernel's completion
// implies that of all kernels before it in the stream.  No kernel triggers its
// dependents early: measured on the prefill workload, scheduling the next
// kernel's CTAs at the start of the current one cost more (2.5%) than it
// saved, while scheduling them as CTAs exit saves 2%.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_chained(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                                  Args... args) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}
#endif

// Byte offsets of every workspace region, plus the tiling chosen for a shape.
struct Plan {
  // shape
  int T, d, E, k, f, S, fs;
  // derived sizes
  int pair1;       // 1: the gate/up GEMM runs on CTA pairs (cta_group::2)
  int pair2;       // 1: the down GEMM runs on CTA pairs
  int rowpad;      // expert segments (and T) are padded to this many rows: 32 with pairs, else 16
  int weights_evict_first;  // expert weight tiles are read once per call (L2 evict-first)
  int Tp;          // T rounded up to rowpad
  int Rcap;        // routed row capacity: T*k + E*(rowpad-1), rounded to rowpad
  int nb;          // permute blocks: ceil(T / kPermBlock)
  int nmax_r;      // tokens per router work unit
  int router_pair; // 1: the router GEMM runs on CTA pairs (256 experts x nmax_r tokens per unit)
  int router_nwb;  // expert blocks per token run: 128 experts each (256 on CTA pairs)
  int router_Tp;   // T rounded up to the router's row step (32 on CTA pairs: each CTA loads half a run)
  int nmax1;       // rows per gate/up work unit (MMA N max)
  int nmax2;       // rows per down work unit
  int nwbE;        // 128-row blocks of E
  int nwb1;        // weight blocks of f per gate/up unit: 128 rows (256 with pairs)
  int nwb1s;       // the same for fs
  int nwb2;        // weight blocks of d per down unit: 256 rows
  int router_units;
  int router_split;  // router K slices (partial logits summed by the top-k kernel in slice order)
  int router_kbs;    // k-blocks per slice
  int U1cap, U2cap;
  int shared_units1, shared_units2;
  // region offsets (bytes)
  size_t err, nunits, logits, blkcnt, counts, roff, perm, roww, inv, units1, units2;
  size_t Hr, Hs, Yr, Ys, xstage, ostage, istage, wstage, sgate;
  size_t total;
};

// Fills `p` for `s`; returns MOE_OK or MOE_ERR_INVALID_ARG / MOE_ERR_UNSUPPORTED.
int make_plan(const moe_shape* s, Plan* p, bool f8 = false);
// Tag of the work-list layout a plan produces (token-run length, CTA pairs);
// the permute stores it beside the lists and the expert GEMMs check it.
inline int plan_tag(const Plan& p) { return p.nmax1 | (p.pair1 << 12) | (1 << 16); }

// Per-device facts, looked up once per device.
struct DeviceInfo {
  int ok;          // 1 if sm_100 and attributes were read
  int sms;
  int max_smem_optin;
};
int device_info(DeviceInfo* info);

// ---- kernel launchers (each returns MOE_OK or MOE_ERR_CUDA) ----
enum GemmMode { kModeRouter = 0, kModeGateUp = 1, kModeDown = 2 };

struct GemmParams {
  CUtensorMap mapA[4];      // A operands: [0],[1] routed (gate, up | down | router); [2],[3] shared
  CUtensorMap mapB[2][4];   // token-row sources ([0] routed / all tokens, [1] shared), boxes of 16/32/64/128 rows
  CUtensorMap mapO[2];      // expert GEMM outputs ([0] routed rows H_r / Y_r, [1] shared rows), boxes of 32 x 16
  CUtensorMap mapX;         // gate/up on CTA pairs: x rows for 4-row tensor gathers (box of 64 x 1)
  const int4* units;        // work list (gate/up and down)
  const int* num_units_dev; // its length, on the device
  int num_units_host;       // router: number of units
  const int* perm;          // gate/up: token of each routed row
  const float* roww;        // down: combine weight of each routed row
  const void* x;            // gate/up: the tokens [T,d] bf16 (row gather source)
  void* out_r;              // router: logits f32 [T,E]; gate/up: H_r; down: Y_r
  void* out_s;              // gate/up: H_s; down: Y_s
  uint32_t* err;
  int T, Tp, E, d, f, fs;
  int nmax, stages, nbuf, router_nwb;
  int router_split, router_kbs;   // router: K slices per token run, k-blocks per slice
  uint64_t timeout_ns;
  int weights_evict_first;  // 1: each weight tile is read by one unit (experts fit one token run)
  // block-scaled FP8 expert weights: mapA are then the code tensors (uint8,
  // tiles of 128 rows x 64 codes) and mapS their scales ([G, K/32, rows] uint8,
  // tiles of 128 rows x 2 blocks); raw_stages = depth of the landing ring
  CUtensorMap mapS[4];
  int raw_stages, tok_stages;
  const int* plan_tag_dev;  // expert GEMMs: the tag the permute stored
  int plan_tag;             // the tag this launch's plan expects
};

int launch_gemm(int mode, const GemmParams& prm, int grid, size_t smem, cudaStream_t st, bool f8 = false);
size_t gemm_smem_bytes(int mode, int nmax, int* stages);
// FP8 expert GEMMs: MMA stages and landing-ring stages for an nmax
size_t gemm_f8_smem_bytes(int mode, int nmax, int* stages, int* tok_stages, int* raw_stages);
// CTA-pair (cta_group::2) expert GEMMs; grid is rounded down to an even count.
int launch_gemm_pair(int mode, const GemmParams& prm, int grid, size_t smem, cudaStream_t st);
size_t gemm_pair_smem_bytes(int mode, int nmax, int* stages);

// err: the error word of this call.  If the router GEMM recorded a timeout
// there, every token gets expert -1 and weight 0; NaN or infinite keys or
// weights set kDevErrNonFinite.
int launch_topk(const float* logits, int nsplit, const float* bias, int T, int E, int k, int score_fn,
                int norm_topk, float route_scale, int32_t* topk_idx, float* topk_w, uint32_t* err,
                cudaStream_t st);

int launch_permute(const Plan& p, const int32_t* topk_idx, const float* topk_w, char* ws,
                   cudaStream_t st);

int launch_combine(const Plan& p, void* out, char* ws, const void* x, const void* shared_gate_vec,
                   cudaStream_t st);

int launch_wait_timeout(uint32_t* err, uint64_t timeout_ns, cudaStream_t st);

int launch_rmsnorm(const Plan& p, const void* x, const void* gain, float eps, void* y, cudaStream_t st);

}  // namespace moe
