// moe_gemm.cu - the tensor-core GEMMs of the MoE block on sm_100a:
//
//   router  : logits[t, e]   = x[t,:] . W_router[e,:]                      (fp32 out)
//   gate/up : H[r, j]        = SiLU(x[tok(r),:] . Wg[e,j,:]) * (x[tok(r),:] . Wu[e,j,:])
//   down    : Y[r, m]        = w(r) * (H[r,:] . Wd[e,m,:])
//
// One persistent, warp-specialised kernel template serves all three.  A work
// unit is (group g, 128-row block of the weight matrix, a run of n <= nmax
// consecutive rows of the group's row segment); for the router, g is a slice
// of d instead when the plan splits K, each slice writing its own partial
// logits.  A CTA-pair form (cta_group::2, moe_gemm_pair_kernel) serves the
// expert GEMMs of large experts and the router of large batches (256
// experts x 256 tokens per unit).  The GEMM is "swap-AB": the
// 128 weight rows are the MMA's M side and the unit's tokens its N side
// (n a multiple of 16), so an expert with few tokens costs n/16 MMA columns,
// not a padded 128-row tile.
//
//   warp 0      TMA producer: weight tiles by 3-D tiled loads (and, for the
//               router and the down GEMM, the unit's contiguous token rows)
//               into a ring of stages.
//   warp 1      TMEM owner and single-thread tcgen05.mma issuer; fp32
//               accumulators in tensor memory (gate and up side by side for
//               the gate/up GEMM), double-buffered when they fit.
//   epilogue    4 (router; 8 in its pair form) or 8 warps: tcgen05.ld ->
//               fp32 math (SiLU*, weight scale; router: fp32 sums of the
//               drained partial logits) -> bf16 -> transpose through shared
//               memory -> 16-byte stores of whole row segments.
//   gather      gate/up: 4 warps copy the unit's token rows of x (by perm)
//               straight into the swizzled tile (cp.async; CTA pairs: 4-row
//               tensor gathers); no permuted copy of x is ever made.
//   FP8 forms   block-scaled FP8 weights: converter warps widen landed FP8
//               tiles into tensor memory (see moe_gemm_kernel<MODE, true>).
//
// All waits are bounded (see mbar_wait); a block that gives up records the
// timeout in the workspace error word, drains its own copies and MMAs, frees
// its tensor memory and returns.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "moe_internal.h"
#include "moe_ptx.cuh"

namespace moe {

namespace {

constexpr int kGatherWarps = 4;                      // gate/up: warps that gather token rows
constexpr int kGatherThreads = 32 * kGatherWarps;
// Epilogue warps: 4 for the router (one per TMEM lane quarter), 8 for the
// expert GEMMs (two per lane quarter, splitting the columns).
__host__ __device__ constexpr int epi_warps_of(int mode) { return mode == kModeRouter ? 4 : 8; }
// Block-scaled FP8 weights: warps that widen each landed FP8 tile to bf16.
constexpr int kConvWarps = 8;
constexpr int kConvThreads = 32 * kConvWarps;
// FP8 down GEMM: one warp loads the token rows (H) into the token ring.
__host__ __device__ constexpr int threads_of(int mode, bool f8 = false) {
  return 64 + 32 * epi_warps_of(mode) + (mode == kModeGateUp ? kGatherThreads : 0) +
         (f8 ? kConvThreads + (mode == kModeDown ? 32 : 0) : 0);
}
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kATileBytes = kTileRows * 128;   // 128 weight rows x 64 bf16
// CTA-pair kernel: 8 epilogue warps in every mode (router: two per tensor-
// memory lane quarter, each summing half of the run's token columns).
__host__ __device__ constexpr int pair_epi_warps_of(int) { return 8; }
// Token rows: gate/up gathers them with kGatherWarps warps; down and the
// router load them with tiled tensor loads from a second producer warp.
__host__ __device__ constexpr int pair_threads_of(int mode) {
  return 64 + 32 * pair_epi_warps_of(mode) + (mode == kModeGateUp ? kGatherThreads : 32);
}
// Epilogue staging of the CTA-pair kernel: 2 KB per warp, a 16-row transpose
// buffer with 80-byte rows (64 bytes of features + 16 of padding, so the 8
// rows of a transposed matrix store hit distinct banks) and, down, the
// combine weights of the warp's columns.
__host__ __device__ constexpr int pair_epi_bytes_of(int) { return 16384; }
constexpr int kStgRow = 80;
// Epilogue staging of the single-CTA kernel: 2 KB per warp (router: one fp32
// transpose buffer; expert GEMMs: two 1 KB slots that alternate, so a slot
// is refilled while the tensor store of the other is in flight).
__host__ __device__ constexpr int epi_bytes_of(int mode) { return 2048 * epi_warps_of(mode); }
constexpr int kMaxStages = 8;
constexpr int kSmemAlign = 1024;
constexpr int kSmemTail = 768;                       // barriers, TMEM slot, abort flag
constexpr int kMaxTmemBufs = 8;                      // accumulator buffers (router: 8 x 64 columns)
constexpr int kMaxRawStages = 12;                    // FP8: stages of the landed-tile ring
constexpr int kMaxTokStages = 8;                     // FP8: stages of the token ring
constexpr uint32_t kRawTileBytes = kTileRows * kTileK;           // 128 rows x 64 FP8 codes
constexpr uint32_t kScaleTileBytes = kTileRows * (kTileK / 32);  // their scales: [2 blocks][128 rows]
constexpr uint32_t kRawTile = kRawTileBytes + kScaleTileBytes;
// FP8: widened weight tiles live in tensor memory, columns [256, 512): stage s,
// tile a at column 256 + (2 s + a) * 32 (128 rows x 64 bf16 = 32 columns);
// accumulators then use columns [0, 256).
constexpr uint32_t kAColBase = 256;
constexpr int kAStages = 4;
constexpr int kRouterDrainKB = 2;                    // router: k-blocks accumulated in TMEM per drain
constexpr int kRouterMaxN = 128;                     // router: tokens per unit (fp32 sums in registers)

struct Unit {
  int g, wb, row0, n;
};

template <int MODE>
__device__ __forceinline__ Unit get_unit(const GemmParams& p, int u) {
  Unit un;
  if (MODE == kModeRouter) {
    // router: g = the unit's slice of K (split-K when there are few units)
    const int v = u / p.router_split;
    const int chunk = v / p.router_nwb;
    un.g = u - v * p.router_split;
    un.wb = v - chunk * p.router_nwb;
    un.row0 = chunk * p.nmax;
    un.n = min(p.nmax, p.Tp - un.row0);
  } else {
    const int4 v = __ldg(p.units + u);
    un.g = v.x;
    un.wb = v.y;
    un.row0 = v.z;
    un.n = v.w;
  }
  return un;
}

// The it-th work unit of CTA (or CTA pair) p of P: round it covers units
// it*P .. it*P + P - 1, handed out in forward order on even rounds and in
// backward order on odd ones, so that a CTA that got one of the larger
// units of a round (the lists run from large to small units, interleaved)
// gets one of the smaller ones in the next.  Increasing in it for every p,
// so a loop may stop at the first index past the list.
__device__ __forceinline__ int snake_unit(int it, int p, int P) { return it * P + ((it & 1) ? P - 1 - p : p); }

// Bounded wait that ignores the abort flag: used only to drain work this block
// itself put in flight before it leaves.
__device__ __forceinline__ void mbar_wait_drain(uint64_t* bar, uint32_t parity, uint64_t timeout_ns) {
  const uint32_t a = smem_u32(bar);
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(a, parity)) {
    if (global_timer_ns() - t0 > timeout_ns) return;
  }
}

// v[j] for a run-time j in [0, 8), without indexing the array dynamically.
// Two floats to a bf16 pair (each rounded to nearest even), the first in
// the low half.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

__device__ __forceinline__ float pick8(const float (&v)[8], int j) {
  float r = v[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) r = (i == j) ? v[i] : r;
  return r;
}

// ---- FP8 -> bf16 widening (exact) ----
// Integer path (the common case).  An E4M3 code s.eeee.mmm placed at bits
// 15 / 10..7 / 6..4 of a bf16 is the bf16 e4m3(code) * 2^-120, subnormal codes
// included (exponent field 0 is subnormal in both formats, with the same
// mantissa scaling).  Multiplying by the bf16 2^(u-7) then gives
// e4m3(code) * 2^(u-127) exactly whenever that is representable.  Per pair
// of codes: one byte permute, one shift, two logic ops and one packed bf16
// multiply, all on full-rate pipes.  2^(u-7) is a bf16 only for u <= 134;
// larger scale bytes take the conversion-instruction path below.
__device__ __forceinline__ uint32_t e4m3x2_placed(uint32_t y) {   // y: codes in the high bytes of its halves
  return ((y >> 4) & 0x07F007F0u) | (y & 0x80008000u);
}

__device__ __forceinline__ uint32_t bf16x2_mul(uint32_t a, uint32_t b) {
  __nv_bfloat162 r = __hmul2(*reinterpret_cast<const __nv_bfloat162*>(&a), *reinterpret_cast<const __nv_bfloat162*>(&b));
  return *reinterpret_cast<const uint32_t*>(&r);
}

// 16 codes (one 16-byte chunk, lowest address first) -> 16 bf16 in two chunks;
// s2 = the bf16 2^(u-7) in both halves.
__device__ __forceinline__ void fp8x16_to_bf16_int(const uint4 v, uint32_t s2, uint4& lo, uint4& hi) {
  lo.x = bf16x2_mul(e4m3x2_placed(__byte_perm(v.x, 0u, 0x1404)), s2);
  lo.y = bf16x2_mul(e4m3x2_placed(__byte_perm(v.x, 0u, 0x3424)), s2);
  lo.z = bf16x2_mul(e4m3x2_placed(__byte_perm(v.y, 0u, 0x1404)), s2);
  lo.w = bf16x2_mul(e4m3x2_placed(__byte_perm(v.y, 0u, 0x3424)), s2);
  hi.x = bf16x2_mul(e4m3x2_placed(__byte_perm(v.z, 0u, 0x1404)), s2);
  hi.y = bf16x2_mul(e4m3x2_placed(__byte_perm(v.z, 0u, 0x3424)), s2);
  hi.z = bf16x2_mul(e4m3x2_placed(__byte_perm(v.w, 0u, 0x1404)), s2);
  hi.w = bf16x2_mul(e4m3x2_placed(__byte_perm(v.w, 0u, 0x3424)), s2);
}

// Conversion-instruction path, any scale byte: an E4M3 code becomes an fp16
// exactly (hardware conversion), an fp16 becomes an fp32 exactly, the block
// scale 2^(u-127) multiplies exactly, and a value with at most 4 significant
// bits rounds to bf16 exactly.
__device__ __forceinline__ float ue8m0_scale(uint32_t u) {
  return __uint_as_float(u == 0 ? 0x00400000u : (u == 255 ? 0x7FC00000u : u << 23));
}

__device__ __forceinline__ uint32_t fp8x2_to_bf16x2(uint32_t two, float sc) {
  const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(two), __NV_E4M3);
  const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&hr));
  const __nv_bfloat162 b = __floats2bfloat162_rn(f.x * sc, f.y * sc);
  return *reinterpret_cast<const uint32_t*>(&b);
}

__device__ __forceinline__ void fp8x16_to_bf16_cvt(const uint4 v, float sc, uint4& lo, uint4& hi) {
  lo.x = fp8x2_to_bf16x2(v.x & 0xFFFFu, sc);
  lo.y = fp8x2_to_bf16x2(v.x >> 16, sc);
  lo.z = fp8x2_to_bf16x2(v.y & 0xFFFFu, sc);
  lo.w = fp8x2_to_bf16x2(v.y >> 16, sc);
  hi.x = fp8x2_to_bf16x2(v.z & 0xFFFFu, sc);
  hi.y = fp8x2_to_bf16x2(v.z >> 16, sc);
  hi.z = fp8x2_to_bf16x2(v.w & 0xFFFFu, sc);
  hi.w = fp8x2_to_bf16x2(v.w >> 16, sc);
}

// Widens one 32-code block of a landed FP8 tile (its two 16-byte chunks, scale
// byte s) into 16 packed bf16x2 registers, element pairs in K order.
__device__ __forceinline__ void widen_block(const uint4 v0, const uint4 v1, uint32_t s, uint32_t (&o)[16]) {
  uint4 a, b, c, d;
  if (s <= 134u) {
    const uint32_t e = (s + 120u) << 7;    // bf16 bits of 2^(s-7)
    fp8x16_to_bf16_int(v0, e | (e << 16), a, b);
    fp8x16_to_bf16_int(v1, e | (e << 16), c, d);
  } else {
    const float sc = ue8m0_scale(s);
    fp8x16_to_bf16_cvt(v0, sc, a, b);
    fp8x16_to_bf16_cvt(v1, sc, c, d);
  }
  o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w;
  o[4] = b.x; o[5] = b.y; o[6] = b.z; o[7] = b.w;
  o[8] = c.x; o[9] = c.y; o[10] = c.z; o[11] = c.w;
  o[12] = d.x; o[13] = d.y; o[14] = d.z; o[15] = d.w;
}

// SiLU(z) = z * sigmoid(z), with sigmoid(z) = (1 + tanh(z / 2)) / 2: one
// special-function op (tanh.approx) where exp and a reciprocal take two; the
// special-function unit's rate bounds the gate/up epilogue.  tanh.approx has a
// relative error of about 2^-11, so sigmoid's absolute error is at most about
// 2^-12: for z >= 0 that is below the bf16 rounding of h, while for z << 0
// (sigmoid near 0) SiLU's absolute error, about |z| * 2^-12, can exceed the
// relative bf16 rounding of that small value; it stays far inside the
// block's output tolerance (max |err| <= 2e-2 * max |out|).
__device__ __forceinline__ float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float silu_f(float z) { return z * fmaf(0.5f, tanh_approx(0.5f * z), 0.5f); }

// F8: the routed and shared expert weights are block-scaled FP8 (codes plus
// one power-of-two scale per 32 codes along K).  The producer lands code and
// scale tiles in a ring of their own; kConvWarps converter warps widen each
// tile to bf16 into the MMA stage (exact), so the tensor cores and the rest
// of the kernel are those of the bf16 path while HBM moves half the bytes.
template <int MODE, bool F8>
__global__ void __launch_bounds__(threads_of(MODE, F8), 1) moe_gemm_kernel(const __grid_constant__ GemmParams p) {
  static_assert(!F8 || MODE != kModeRouter, "the router weights stay bf16");
  // A tiles (and accumulators) per unit: gate/up: the gate and the up tile of
  // the same 128 rows; down: two consecutive 128-row blocks of W_down (a
  // 256-row unit, so each token row loaded serves 256 outputs); router: one.
  constexpr int NA = (MODE == kModeRouter) ? 1 : 2;
  constexpr int kWbRows = (MODE == kModeDown) ? 2 * kTileRows : kTileRows;   // weight rows per unit
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + (kSmemAlign - 1)) & ~static_cast<uintptr_t>(kSmemAlign - 1));
  const int nmax = p.nmax;
  const int S = p.stages;
  const uint32_t tok_bytes = static_cast<uint32_t>(nmax) * 128u;
  // bf16: each MMA stage holds the weight tiles and the token tile in shared
  // memory.  FP8: the MMA stages (S) hold the widened weight tiles in tensor
  // memory, and shared memory holds two rings - token tiles (TS) and the
  // landed code + scale tiles (R) - so both kinds of load run far ahead.
  const uint32_t stage_bytes = F8 ? 0u : NA * kATileBytes + tok_bytes;
  const int TS = F8 ? p.tok_stages : 0;
  const int R = F8 ? p.raw_stages : 0;
  constexpr uint32_t raw_stage_bytes = NA * kRawTile;
  uint8_t* tokring = smem + static_cast<size_t>(S) * stage_bytes;
  uint8_t* raw = tokring + static_cast<size_t>(TS) * tok_bytes;
  uint8_t* epi = raw + static_cast<size_t>(R) * raw_stage_bytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(epi + epi_bytes_of(MODE));
  uint64_t* empty = full + S;
  uint64_t* tfull = empty + S;
  uint64_t* tempty = tfull + kMaxTmemBufs;
  uint64_t* drain = tempty + kMaxTmemBufs;
  uint64_t* raw_full = drain + 1;
  uint64_t* raw_empty = raw_full + R;
  uint64_t* tok_full = raw_empty + R;
  uint64_t* tok_empty = tok_full + TS;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tok_empty + TS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  // FP8 warps after the epilogue (and gather) warps: down: one token loader,
  // then the converters; gate/up: the converters.
  constexpr int kTokWarp = 2 + epi_warps_of(MODE);
  constexpr int kConvBase =
      2 + epi_warps_of(MODE) + (MODE == kModeGateUp ? kGatherWarps : 0) + (F8 && MODE == kModeDown ? 1 : 0);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      // bf16: the producer's arrival plus (gate/up) one per gathering thread;
      // FP8: one per converter warp
      mbar_init(full + s, F8 ? kConvWarps : 1 + (MODE == kModeGateUp ? kGatherThreads : 0));
      mbar_init(empty + s, 1);
    }
    for (int r = 0; r < R; ++r) {
      mbar_init(raw_full + r, 1);
      mbar_init(raw_empty + r, kConvWarps);
    }
    for (int t = 0; t < TS; ++t) {
      // gate/up: one per gathering thread; down: the token loader's arrival
      mbar_init(tok_full + t, MODE == kModeGateUp ? kGatherThreads : 1);
      mbar_init(tok_empty + t, 1);
    }
    for (int b = 0; b < kMaxTmemBufs; ++b) {
      mbar_init(tfull + b, 1);
      mbar_init(tempty + b, epi_warps_of(MODE));
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    for (int i = 0; i < 2 * NA; ++i) prefetch_tensormap(&p.mapA[i]);
    if (F8)
      for (int i = 0; i < 2 * NA; ++i) prefetch_tensormap(&p.mapS[i]);
    if (MODE != kModeGateUp)
      for (int i = 0; i < 4; ++i) prefetch_tensormap(&p.mapB[0][i]);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  chain_wait();
  int num_units = (MODE == kModeRouter) ? p.num_units_host : *p.num_units_dev;
  if (MODE != kModeRouter && *p.plan_tag_dev != p.plan_tag) {
    // work lists built for the other weight format's plan: do nothing, report it
    if (threadIdx.x == 0 && blockIdx.x == 0) atomicOr(p.err, kDevErrPlanMismatch);
    num_units = 0;
  }

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // router: W_router and x are re-read by every unit -> keep; expert
    // weights that stream through once -> evict first; expert weights that
    // several token runs of one expert share -> keep.
    const uint64_t pol_a = (MODE == kModeRouter || !p.weights_evict_first) ? policy_evict_last()
                                                                           : policy_evict_first();
    const uint64_t pol_b = policy_evict_last();
    // the ring this warp fills: the MMA stages, or (FP8) the landing ring
    uint64_t* pfull = F8 ? raw_full : full;
    uint64_t* pempty = F8 ? raw_empty : empty;
    const int PS = F8 ? R : S;
    int stage = 0;
    uint32_t phase = 0;
    uint32_t issued = 0;
    bool ok = true;
    for (int it = 0, u = snake_unit(0, blockIdx.x, gridDim.x); ok && u < num_units;
         u = snake_unit(++it, blockIdx.x, gridDim.x)) {
      const Unit un = get_unit<MODE>(p, u);
      const bool sh = (MODE != kModeRouter) && un.g >= p.E;
      const int sidx = sh ? un.g - p.E : 0;
      const int K = (MODE == kModeDown) ? (sh ? p.fs : p.f) : p.d;
      const int KB = K / kTileK;
      // router: this unit's k-blocks [kb0, kb1); the expert GEMMs: all of K
      const int kb0 = (MODE == kModeRouter) ? un.g * p.router_kbs : 0;
      const int kb1 = (MODE == kModeRouter) ? min(KB, kb0 + p.router_kbs) : KB;
      const CUtensorMap* mA = &p.mapA[sh ? 2 : 0];
      const CUtensorMap* mB = p.mapB[(MODE == kModeDown && sh) ? 1 : 0];
      const int a_c2 = (MODE == kModeRouter) ? 0 : (sh ? sidx : un.g);
      // Router / down: the unit's rows are contiguous in the source; first row:
      const int brow0 = (MODE == kModeDown && sh) ? sidx * p.Tp + un.row0 : un.row0;
      // Gate/up token rows come from the gather warps, not from TMA.
      const uint32_t tx_bytes =
          NA * kATileBytes + (MODE == kModeGateUp ? 0u : static_cast<uint32_t>(un.n) * 128u);
      int got = 1;
      if (lane == 0) {
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&pempty[stage], phase ^ 1u, abort_flag, p.err, p.timeout_ns)) {
            got = 0;
            break;
          }
          if constexpr (F8) {
            // code tile(s) and their scales into the landing ring; the
            // converter warps widen them into the MMA stage
            const uint32_t rbase = smem_u32(raw + static_cast<size_t>(stage) * raw_stage_bytes);
            const uint32_t fb = smem_u32(&raw_full[stage]);
            const CUtensorMap* mS = &p.mapS[sh ? 2 : 0];
            mbar_arrive_expect_tx(&raw_full[stage], raw_stage_bytes);
#pragma unroll
            for (int a = 0; a < NA; ++a) {
              const int wrow = un.wb * kWbRows + ((MODE == kModeDown) ? a * kTileRows : 0);
              tma_load_3d_hint(rbase + a * kRawTile, (MODE == kModeDown) ? mA : mA + a, fb, kb * kTileK, wrow,
                               a_c2, pol_a);
              tma_load_3d(rbase + a * kRawTile + kRawTileBytes, (MODE == kModeDown) ? mS : mS + a, fb, wrow,
                          kb * (kTileK / 32), a_c2);
            }
          } else {
            const uint32_t sbase = smem_u32(smem + static_cast<size_t>(stage) * stage_bytes);
            const uint32_t fb = smem_u32(&full[stage]);
            mbar_arrive_expect_tx(&full[stage], tx_bytes);
#pragma unroll
            for (int a = 0; a < NA; ++a)
              tma_load_3d_hint(sbase + a * kATileBytes, (MODE == kModeDown) ? mA : mA + a, fb, kb * kTileK,
                               un.wb * kWbRows + ((MODE == kModeDown) ? a * kTileRows : 0), a_c2, pol_a);
            if (MODE != kModeGateUp)
              tma_load_rows<false>(sbase + NA * kATileBytes, mB, fb, kb * kTileK, brow0, un.n, pol_b);
          }
          ++issued;
          if (++stage == PS) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      got = __shfl_sync(0xffffffffu, got, 0);
      if (!got) ok = false;
    }
    // Leave no copy in flight: the last min(PS, issued) stages armed.
    if (lane == 0) {
      const uint32_t outstanding = issued < static_cast<uint32_t>(PS) ? issued : static_cast<uint32_t>(PS);
      for (uint32_t i = 1; i <= outstanding; ++i) {
        const uint32_t I = issued - i;
        mbar_wait_drain(&pfull[I % PS], (I / PS) & 1u, p.timeout_ns);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int tstage = 0;                 // FP8: token ring
      uint32_t tphase = 0;
      uint32_t ucount = 0;
      bool any = false;
      bool ok = true;
      if constexpr (MODE == kModeRouter) {
        // Router: the accumulator is drained every kRouterDrainKB k-blocks
        // into fp32 registers by the epilogue, so no tensor-core accumulation
        // chain is longer than 4 * kRouterDrainKB MMA steps.
        uint32_t dc = 0;
        for (int it = 0, u = snake_unit(0, blockIdx.x, gridDim.x); ok && u < num_units;
             u = snake_unit(++it, blockIdx.x, gridDim.x)) {
          const Unit un = get_unit<MODE>(p, u);
          const int KB = p.d / kTileK;
          const int kb0 = un.g * p.router_kbs;
          const int kb1 = min(KB, kb0 + p.router_kbs);
          const uint32_t idesc = idesc_bf16_f32(kTileRows, un.n);
          uint32_t dcol = tmem_base;
          for (int kb = kb0; kb < kb1; ++kb) {
            const int sub = (kb - kb0) % kRouterDrainKB;
            const int buf = static_cast<int>(dc % static_cast<uint32_t>(p.nbuf));
            if (sub == 0) {
              const uint32_t bpar = (dc / static_cast<uint32_t>(p.nbuf)) & 1u;
              if (!mbar_wait(&tempty[buf], bpar ^ 1u, abort_flag, p.err, p.timeout_ns)) {
                ok = false;
                break;
              }
              tc_fence_after();
              dcol = tmem_base + static_cast<uint32_t>(buf * nmax);
            }
            if (!mbar_wait(&full[stage], phase, abort_flag, p.err, p.timeout_ns)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t sbase = smem_u32(smem + static_cast<size_t>(stage) * stage_bytes);
            const uint64_t adesc = sw128_kmajor_desc(sbase);
            const uint64_t bdesc = sw128_kmajor_desc(sbase + kATileBytes);
#pragma unroll
            for (int ks = 0; ks < kTileK / 16; ++ks)
              tc_mma_bf16(dcol, adesc + 2u * ks, bdesc + 2u * ks, idesc, (sub | ks) != 0 ? 1u : 0u);
            any = true;
            tc_commit(&empty[stage]);
            if (++stage == S) {
              stage = 0;
              phase ^= 1u;
            }
            if (sub == kRouterDrainKB - 1 || kb == kb1 - 1) {
              tc_commit(&tfull[buf]);
              ++dc;
            }
          }
        }
      } else {
        for (int it = 0, u = snake_unit(0, blockIdx.x, gridDim.x); ok && u < num_units;
             u = snake_unit(++it, blockIdx.x, gridDim.x)) {
          const Unit un = get_unit<MODE>(p, u);
          const bool sh = (MODE != kModeRouter) && un.g >= p.E;
          const int K = (MODE == kModeDown) ? (sh ? p.fs : p.f) : p.d;
          const int KB = K / kTileK;
          const int buf = static_cast<int>(ucount % static_cast<uint32_t>(p.nbuf));
          const uint32_t bpar = (ucount / static_cast<uint32_t>(p.nbuf)) & 1u;
          if (!mbar_wait(&tempty[buf], bpar ^ 1u, abort_flag, p.err, p.timeout_ns)) break;
          tc_fence_after();
          const uint32_t idesc = idesc_bf16_f32(kTileRows, un.n);
          const uint32_t dcol = tmem_base + static_cast<uint32_t>(buf * NA * nmax);
          for (int kb = 0; kb < KB; ++kb) {
            if (!mbar_wait(&full[stage], phase, abort_flag, p.err, p.timeout_ns) ||
                (F8 && !mbar_wait(&tok_full[tstage], tphase, abort_flag, p.err, p.timeout_ns))) {
              ok = false;
              break;
            }
            tc_fence_after();
            // Token rows written by cp.async and (FP8) weight tiles written by
            // the converters (generic proxy) are read by the tensor cores
            // (async proxy).
            if (MODE == kModeGateUp || F8) fence_proxy_async_smem();
            const uint32_t sbase = smem_u32(smem + static_cast<size_t>(stage) * stage_bytes);
            const uint64_t bdesc = sw128_kmajor_desc(
                F8 ? smem_u32(tokring + static_cast<size_t>(tstage) * tok_bytes) : sbase + NA * kATileBytes);
            if constexpr (F8) {
              const uint32_t acol = tmem_base + kAColBase + static_cast<uint32_t>(stage * NA * 32);
#pragma unroll
              for (int ks = 0; ks < kTileK / 16; ++ks) {
#pragma unroll
                for (int a = 0; a < NA; ++a)
                  tc_mma_bf16_ta(dcol + static_cast<uint32_t>(a * nmax), acol + static_cast<uint32_t>(a * 32 + ks * 8),
                                 bdesc + 2u * ks, idesc, (kb | ks) != 0 ? 1u : 0u);
              }
            } else {
              uint64_t adesc[NA];
#pragma unroll
              for (int a = 0; a < NA; ++a) adesc[a] = sw128_kmajor_desc(sbase + a * kATileBytes);
#pragma unroll
              for (int ks = 0; ks < kTileK / 16; ++ks) {
#pragma unroll
                for (int a = 0; a < NA; ++a)
                  tc_mma_bf16(dcol + static_cast<uint32_t>(a * nmax), adesc[a] + 2u * ks, bdesc + 2u * ks,
                              idesc, (kb | ks) != 0 ? 1u : 0u);
              }
            }
            any = true;
            tc_commit(&empty[stage]);
            if (++stage == S) {
              stage = 0;
              phase ^= 1u;
            }
            if (F8) {
              tc_commit(&tok_empty[tstage]);
              if (++tstage == TS) {
                tstage = 0;
                tphase ^= 1u;
              }
            }
          }
          if (!ok) break;
          tc_commit(&tfull[buf]);
          ++ucount;
        }
      }
      // Leave no MMA in flight.
      if (any) {
        tc_commit(drain);
        mbar_wait_drain(drain, 0, p.timeout_ns);
      }
    }
    __syncwarp();
  } else if (F8 && warp >= kConvBase) {
    // ------------------------------------------------------------ FP8 -> bf16
    // Warp w may access tensor-memory lanes 32 (w % 4) .. + 31: its lane l
    // widens 32-code block h of weight row r = 32 (w % 4) + l of every landed
    // code tile into the MMA stage's tile in tensor memory; the first four
    // converter warps take h = 0, the next four h = 1.
    const int cq = warp & 3;
    const int crow = 32 * cq + lane;
    const int chalf = (warp - kConvBase) >> 2;
    const uint32_t tlane = static_cast<uint32_t>(32 * cq) << 16;
    int rs = 0, ms = 0;              // landing-ring and MMA-ring positions
    uint32_t rph = 0, mph = 0;
    int pms = -1;                    // MMA stage written but not yet published
    bool ok = true;
    for (int it = 0, u = snake_unit(0, blockIdx.x, gridDim.x); ok && u < num_units;
         u = snake_unit(++it, blockIdx.x, gridDim.x)) {
      const Unit un = get_unit<MODE>(p, u);
      const bool sh = un.g >= p.E;
      const int K = (MODE == kModeDown) ? (sh ? p.fs : p.f) : p.d;
      const int KB = K / kTileK;
      for (int kb = 0; kb < KB; ++kb) {
        int got = 1;
        if (lane == 0)
          got = (mbar_wait(&raw_full[rs], rph, abort_flag, p.err, p.timeout_ns) &&
                 mbar_wait(&empty[ms], mph ^ 1u, abort_flag, p.err, p.timeout_ns))
                    ? 1
                    : 0;
        got = __shfl_sync(0xffffffffu, got, 0);
        if (!got) {
          ok = false;
          break;
        }
        // Codes and scales of both tiles into registers; the landed stage is
        // then free for the producer.
        const uint8_t* rt = raw + static_cast<size_t>(rs) * raw_stage_bytes;
        uint4 cv[NA][2];
        uint32_t sc[NA];
#pragma unroll
        for (int a = 0; a < NA; ++a) {
          const uint8_t* q = rt + a * kRawTile;
          cv[a][0] = *reinterpret_cast<const uint4*>(q + crow * kTileK + 32 * chalf);
          cv[a][1] = *reinterpret_cast<const uint4*>(q + crow * kTileK + 32 * chalf + 16);
          sc[a] = q[kRawTileBytes + chalf * kTileRows + crow];
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&raw_empty[rs]);
        // The previous k-block's tensor-memory stores have had this block's
        // waits and loads to complete in: publish that stage now.
        if (pms >= 0) {
          tmem_st_wait();
          tc_fence_before();           // tensor-memory stores -> the MMA issuer
          __syncwarp();
          if (lane == 0) mbar_arrive(&full[pms]);
        }
#pragma unroll
        for (int a = 0; a < NA; ++a) {
          uint32_t w16[16];
          widen_block(cv[a][0], cv[a][1], sc[a], w16);
          tmem_st_32x32b_x16(tmem_base + tlane + kAColBase + static_cast<uint32_t>((ms * NA + a) * 32 + 16 * chalf),
                             w16);
        }
        pms = ms;
        if (++rs == R) {
          rs = 0;
          rph ^= 1u;
        }
        if (++ms == S) {
          ms = 0;
          mph ^= 1u;
        }
      }
    }
    if (pms >= 0) {
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&full[pms]);
    }
  } else if (F8 && MODE == kModeDown && warp == kTokWarp) {
    // ------------------------------------------------------------ FP8 down: token rows
    // H rows of each k-block into the token ring, up to TS k-blocks ahead.
    if constexpr (F8) if (lane == 0) {
      const uint64_t pol_b = policy_evict_last();
      int ts = 0;
      uint32_t tph = 0, issued = 0;
      bool ok = true;
      for (int it = 0, u = snake_unit(0, blockIdx.x, gridDim.x); ok && u < num_units;
           u = snake_unit(++it, blockIdx.x, gridDim.x)) {
        const Unit un = get_unit<MODE>(p, u);
        const bool sh = un.g >= p.E;
        const int sidx = sh ? un.g - p.E : 0;
        const int KB = (sh ? p.fs : p.f) / kTileK;
        const CUtensorMap* mB = p.mapB[sh ? 1 : 0];
        const int brow0 = sh ? sidx * p.Tp + un.row0 : un.row0;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&tok_empty[ts], tph ^ 1u, abort_flag, p.err, p.timeout_ns)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&tok_full[ts], static_cast<uint32_t>(un.n) * 128u);
          tma_load_rows<false>(smem_u32(tokring + static_cast<size_t>(ts) * tok_bytes), mB, smem_u32(&tok_full[ts]),
                               kb * kTileK, brow0, un.n, pol_b);
          ++issued;
          if (++ts == TS) {
            ts = 0;
            tph ^= 1u;
          }
        }
      }
      // leave no copy in flight
      const uint32_t outstanding = issued < static_cast<uint32_t>(TS) ? issued : static_cast<uint32_t>(TS);
      for (uint32_t i = 1; i <= outstanding; ++i) {
        const uint32_t I = issued - i;
        mbar_wait_drain(&tok_full[I % TS], (I / TS) & 1u, p.timeout_ns);
      }
    }
    __syncwarp();
  } else if (MODE == kModeGateUp && warp >= 2 + epi_warps_of(MODE) &&
             warp < 2 + epi_warps_of(MODE) + kGatherWarps) {
    // ------------------------------------------------------------ row gather
    // Thread g copies 16-byte chunk (g & 7) of rows (g >> 3) + 16 i of the
    // token tile, i < n / 16, into the 128-byte-swizzled slot: chunk c of row
    // r lands at r * 128 + ((c ^ (r & 7)) * 16).
    const int g = threadIdx.x - 32 * (2 + epi_warps_of(MODE));
    const int part = g & 7;
    const int r0 = g >> 3;
    const uint64_t pol_x = policy_evict_last();     // x rows are gathered by every weight block
    // the ring the token tiles go to: the MMA stages, or (FP8) the token ring
    uint64_t* gfull = F8 ? tok_full : full;
    uint64_t* gempty = F8 ? tok_empty : empty;
    const int GS = F8 ? TS : S;
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int it = 0, u = snake_unit(0, blockIdx.x, gridDim.x); ok && u < num_units;
         u = snake_unit(++it, blockIdx.x, gridDim.x)) {
      const Unit un = get_unit<MODE>(p, u);
      const bool sh = un.g >= p.E;
      const int nr = un.n >> 4;                    // rows of this thread
      int tok[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int r = un.row0 + r0 + 16 * i;
        // clamped: a row never reads outside x, even for an invalid routing
        tok[i] = (i < nr) ? min(max(sh ? r : __ldg(p.perm + r), 0), p.T - 1) : 0;
      }
      const int KB = p.d / kTileK;
      for (int kb = 0; kb < KB; ++kb) {
        int got = 1;
        if (lane == 0) got = mbar_wait(&gempty[stage], phase ^ 1u, abort_flag, p.err, p.timeout_ns) ? 1 : 0;
        got = __shfl_sync(0xffffffffu, got, 0);
        if (!got) {
          ok = false;
          break;
        }
        const uint32_t bbase = F8 ? smem_u32(tokring + static_cast<size_t>(stage) * tok_bytes)
                                  : smem_u32(smem + static_cast<size_t>(stage) * stage_bytes) + NA * kATileBytes;
        const __nv_bfloat16* src0 = reinterpret_cast<const __nv_bfloat16*>(p.x) + kb * kTileK + part * 8;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          if (i < nr) {
            const int r = r0 + 16 * i;
            cp_async_16(bbase + r * 128 + ((part ^ (r & 7)) << 4), src0 + static_cast<size_t>(tok[i]) * p.d,
                        pol_x);
          }
        }
        cp_async_mbar_arrive_noinc(&gfull[stage]);
        if (++stage == GS) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    cp_async_wait_all();
  } else if (warp >= 2 && warp < 2 + epi_warps_of(MODE)) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;                       // TMEM lane quarter this warp may read
    uint8_t* stg = epi + (warp - 2) * 2048;
    if constexpr (MODE == kModeRouter) {
      // Router: sum the drained partial logits in fp32 registers, then write
      // logits[t, e] (thread = expert row, column = token).
      uint32_t dc = 0;
      bool ok = true;
      for (int it = 0, u = snake_unit(0, blockIdx.x, gridDim.x); ok && u < num_units;
           u = snake_unit(++it, blockIdx.x, gridDim.x)) {
        const Unit un = get_unit<MODE>(p, u);
        const int KB = p.d / kTileK;
        const int kb0 = un.g * p.router_kbs;
        const int nkb = min(KB, kb0 + p.router_kbs) - kb0;
        const int nd = (nkb + kRouterDrainKB - 1) / kRouterDrainKB;
        float* const lbase = reinterpret_cast<float*>(p.out_r) + static_cast<size_t>(un.g) * p.T * p.E;
        const int feat0 = un.wb * kTileRows + 32 * q;
        const bool live = feat0 < p.E;
        float acc[kRouterMaxN];
#pragma unroll
        for (int j = 0; j < kRouterMaxN; ++j) acc[j] = 0.0f;
        for (int i = 0; i < nd; ++i) {
          const int buf = static_cast<int>(dc % static_cast<uint32_t>(p.nbuf));
          const uint32_t bpar = (dc / static_cast<uint32_t>(p.nbuf)) & 1u;
          int got = 1;
          if (lane == 0) got = mbar_wait(&tfull[buf], bpar, abort_flag, p.err, p.timeout_ns) ? 1 : 0;
          got = __shfl_sync(0xffffffffu, got, 0);
          if (!got) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (live) {
            const uint32_t tb =
                tmem_base + (static_cast<uint32_t>(32 * q) << 16) + static_cast<uint32_t>(buf * nmax);
            // 64 columns per round trip: 4 loads in flight, then add.
#pragma unroll
            for (int g = 0; g < kRouterMaxN / 64; ++g) {
              if (64 * g < un.n) {
                uint32_t v[4][16];
#pragma unroll
                for (int c = 0; c < 4; ++c)
                  if (64 * g + 16 * c < un.n) tmem_ld_32x32b_x16(tb + static_cast<uint32_t>(64 * g + 16 * c), v[c]);
                tmem_ld_wait();
#pragma unroll
                for (int c = 0; c < 4; ++c)
                  if (64 * g + 16 * c < un.n)
#pragma unroll
                    for (int j = 0; j < 16; ++j) acc[64 * g + 16 * c + j] += __uint_as_float(v[c][j]);
              }
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tempty[buf]);
          ++dc;
        }
        if (!ok || !live) continue;
        float* sf = reinterpret_cast<float*>(stg);
#pragma unroll
        for (int c = 0; c < kRouterMaxN / 16; ++c) {
          if (16 * c < un.n) {
#pragma unroll
            for (int i = 0; i < 16; ++i) sf[i * 32 + lane] = acc[16 * c + i];
            __syncwarp();
#pragma unroll
            for (int rep = 0; rep < 4; ++rep) {
              const int cc = lane + 32 * rep;
              const int tok = cc >> 3, part = cc & 7;
              const int t = un.row0 + 16 * c + tok;
              const int e = feat0 + part * 4;
              if (t < p.T) {
                float* dst = lbase + static_cast<size_t>(t) * p.E + e;
                const float4 vv = *reinterpret_cast<const float4*>(sf + tok * 32 + part * 4);
                if ((p.E & 3) == 0 && e + 3 < p.E) {
                  *reinterpret_cast<float4*>(dst) = vv;
                } else {
                  if (e + 0 < p.E) dst[0] = vv.x;
                  if (e + 1 < p.E) dst[1] = vv.y;
                  if (e + 2 < p.E) dst[2] = vv.z;
                  if (e + 3 < p.E) dst[3] = vv.w;
                }
              }
            }
            __syncwarp();
          }
        }
      }
    } else {
      uint32_t ucount = 0;
      uint32_t ech = 0;                 // chunks stored by this warp (staging slot = ech & 1)
      for (int it = 0, u = snake_unit(0, blockIdx.x, gridDim.x); u < num_units;
           u = snake_unit(++it, blockIdx.x, gridDim.x)) {
        const Unit un = get_unit<MODE>(p, u);
        const bool sh = (MODE != kModeRouter) && un.g >= p.E;
        const int sidx = sh ? un.g - p.E : 0;
        const int buf = static_cast<int>(ucount % static_cast<uint32_t>(p.nbuf));
        const uint32_t bpar = (ucount / static_cast<uint32_t>(p.nbuf)) & 1u;
        // down: combine weights of the unit's rows, fetched before the wait
        // (lane l of register j holds the weight of column 32 j + l)
        float wreg[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int c = 32 * j + lane;
          wreg[j] = (MODE == kModeDown && !sh && c < un.n) ? __ldg(p.roww + un.row0 + c) : 1.0f;
        }
        int got = 1;
        if (lane == 0) got = mbar_wait(&tfull[buf], bpar, abort_flag, p.err, p.timeout_ns) ? 1 : 0;
        got = __shfl_sync(0xffffffffu, got, 0);
        if (!got) break;
        tc_fence_after();
        // gate/up: warps (q, half) take column blocks half*16, half*16 + 32, ...
        // of both accumulators; down: warps (q, h) take every column of
        // accumulator h (weight rows wb*256 + h*128 ...).
        const int half = (MODE == kModeGateUp) ? ((warp - 2) >> 2) : 0;
        const int h = (MODE == kModeDown) ? ((warp - 2) >> 2) : 0;
        const uint32_t tbase = tmem_base + (static_cast<uint32_t>(32 * q) << 16) +
                               static_cast<uint32_t>(buf * NA * nmax + h * nmax);
        const int feat0 = un.wb * kWbRows + h * kTileRows + 32 * q;   // first weight row of this warp
        const int wrows = (MODE == kModeGateUp) ? (sh ? p.fs : p.f) : p.d;
        if (feat0 < wrows) {
          const size_t rbase = (sh ? static_cast<size_t>(sidx) * p.Tp : 0) + static_cast<size_t>(un.row0);
          // 16 columns: fp32 math, bf16, transposed into a staging slot as
          // 16 rows x 32 features (64-byte rows), which one tensor store
          // writes to rows rbase + c .. + 15, features feat0 .. + 31.
          const CUtensorMap* omap = &p.mapO[sh ? 1 : 0];
          auto emit = [&](const uint32_t (&A)[16], const uint32_t (&B)[16], int c, float wsel) {
            uint8_t* slot = stg + (ech & 1u) * 1024u;
            if (lane == 0) bulk_wait_group_read<1>();   // the store from this slot two chunks ago has read it
            __syncwarp();
            __nv_bfloat16* sb = reinterpret_cast<__nv_bfloat16*>(slot);
            if (MODE == kModeGateUp) {
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const float g = __uint_as_float(A[i]);
                const float v = __uint_as_float(B[i]);
                sb[i * 32 + lane] = __float2bfloat16_rn(silu_f(g) * v);
              }
            } else {
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const float w = __shfl_sync(0xffffffffu, wsel, (c + i) & 31);
                sb[i * 32 + lane] = __float2bfloat16_rn(__uint_as_float(A[i]) * w);
              }
            }
            fence_proxy_async_smem();                     // these writes -> the tensor store's reads
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(omap, smem_u32(slot), feat0, static_cast<int>(rbase) + c);
              bulk_commit_group();
            }
            ++ech;
          };
          // Two register sets: the TMEM load of the next 16 columns is in
          // flight while the current ones are converted and stored.  This
          // warp takes column blocks half*16, half*16 + 32, ...
          constexpr int kStep = (MODE == kModeGateUp) ? 32 : 16;
          uint32_t a0[16], b0[16], a1[16], b1[16];
          int c0 = 16 * half;
          if (c0 < un.n) {
            tmem_ld_32x32b_x16(tbase + static_cast<uint32_t>(c0), a0);
            if (MODE == kModeGateUp) tmem_ld_32x32b_x16(tbase + static_cast<uint32_t>(nmax + c0), b0);
          }
          while (c0 < un.n) {
            tmem_ld_wait();
            const int c1 = c0 + kStep;
            if (c1 < un.n) {
              tmem_ld_32x32b_x16(tbase + static_cast<uint32_t>(c1), a1);
              if (MODE == kModeGateUp) tmem_ld_32x32b_x16(tbase + static_cast<uint32_t>(nmax + c1), b1);
            }
            emit(a0, b0, c0, MODE == kModeDown ? pick8(wreg, c0 >> 5) : 1.0f);
            if (c1 >= un.n) break;
            tmem_ld_wait();
            const int c2 = c1 + kStep;
            if (c2 < un.n) {
              tmem_ld_32x32b_x16(tbase + static_cast<uint32_t>(c2), a0);
              if (MODE == kModeGateUp) tmem_ld_32x32b_x16(tbase + static_cast<uint32_t>(nmax + c2), b0);
            }
            emit(a1, b1, c1, MODE == kModeDown ? pick8(wreg, c1 >> 5) : 1.0f);
            c0 = c2;
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[buf]);
        ++ucount;
      }
      if (lane == 0) bulk_wait_group_all();        // every output row written before the block leaves
    }
    }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}


// ===========================================================================
// CTA-pair version of the expert GEMMs (tcgen05 cta_group::2).
//
// A cluster of two CTAs (on the two SMs of a TPC) works on one pair-unit
// {group g, weight block wb, first row row0, n tokens}.  Every MMA has M = 256:
// CTA r supplies weight rows [.. + r*128, +128) and token rows
// [r*n/2, (r+1)*n/2) of the tile, and receives its 128 rows of every output
// column in its own tensor memory.  Each CTA therefore loads half of the token
// tile that a single CTA would: the token bytes that stream into the SMs are
// halved for the same weight bytes.
//   gate/up : wb = 256-row block of f; A tiles per CTA: gate rows, up rows.
//   down    : wb = 256-row block of d; A tile per CTA: its 128 rows (one
//             256-column accumulator per CTA, so tensor memory holds two
//             buffers and the epilogue of one unit overlaps the next's MMAs).
//   router  : wb = 256-expert block of E, g = the unit's slice of d; A tile
//             per CTA: its 128 rows of W_router, B its half of the run's
//             token rows of x.  Each CTA thus loads 128 + 128 rows per k-block
//             for 128 x 256 logits where a single CTA loads 128 + 128 for
//             128 x 128.  The accumulator is drained every kRouterDrainKB
//             k-blocks through two buffers of 256 columns by 8 epilogue warps
//             (128 fp32 sums each).
// The leader CTA (rank 0) issues the MMAs; loads of both CTAs complete on the
// leader's stage barrier (cta_group::2 tensor loads and, gate/up, 4-row
// tensor gathers of the token rows; no multicast); the leader's commits
// arrive on the barrier at the same offset in both CTAs.  A stage completes
// on two arrivals, those of the two CTAs' weight producers, each expecting
// its CTA's weight and token bytes; the token rows come from the gather
// warps (gate/up) or a second producer warp (down, router), which do not
// arrive.  Work units are handed to the pairs in snake order (snake_unit).  The gathers move a
// 128-byte row piece per row where cp.async moves 16 bytes per request: with
// 16-byte requests the gather's request rate bounded the pair gate/up
// (measured: 7.2 -> 6.3 ms at T = 16384, d = 7168, E = 896, k = 22).  A
// single CTA gathers twice the rows per stage, and there tensor gathers were
// slower than cp.async (the tensor unit also carries the weight tiles).
template <int MODE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(pair_threads_of(MODE), 1)
    moe_gemm_pair_kernel(const __grid_constant__ GemmParams p) {
  // gate/up: gate and up tile of this CTA's 128 rows; down and router: one
  // 128-row tile.
  constexpr int NA = (MODE == kModeGateUp) ? 2 : 1;
  constexpr int EW = pair_epi_warps_of(MODE);
  constexpr int kWbRows = 2 * kTileRows;   // weight rows per pair-unit (128 per CTA)
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + (kSmemAlign - 1)) & ~static_cast<uintptr_t>(kSmemAlign - 1));
  const int nmax = p.nmax;
  const int S = p.stages;
  const uint32_t stage_bytes = NA * kATileBytes + static_cast<uint32_t>(nmax / 2) * 128u;
  uint8_t* epi = smem + static_cast<size_t>(S) * stage_bytes;
  constexpr int kEpiBytes = pair_epi_bytes_of(MODE);
  uint64_t* full = reinterpret_cast<uint64_t*>(epi + kEpiBytes);
  uint64_t* empty = full + S;
  uint64_t* tfull = empty + S;
  uint64_t* tempty = tfull + kMaxTmemBufs;
  uint64_t* drain = tempty + kMaxTmemBufs;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      // leader: the weight producers' expect-tx arrivals of both CTAs; each
      // also counts the bytes its CTA's token rows bring (gathered by the
      // gather warps, or loaded by the token producer)
      mbar_init(full + s, 2);
      mbar_init(empty + s, 1);
    }
    for (int b = 0; b < kMaxTmemBufs; ++b) {
      mbar_init(tfull + b, 1);
      mbar_init(tempty + b, 2 * EW);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    for (int i = 0; i < 4; ++i) prefetch_tensormap(&p.mapA[i]);
    if (MODE == kModeGateUp) prefetch_tensormap(&p.mapX);
    if (MODE != kModeGateUp)
      for (int i = 0; i < 4; ++i) prefetch_tensormap(&p.mapB[0][i]);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();                                    // peer barriers are initialised
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  chain_wait();
  int num_units = (MODE == kModeRouter) ? p.num_units_host : *p.num_units_dev;
  if (MODE != kModeRouter && *p.plan_tag_dev != p.plan_tag) {
    if (threadIdx.x == 0 && blockIdx.x == 0) atomicOr(p.err, kDevErrPlanMismatch);
    num_units = 0;
  }
  const uint32_t full_leader = mapa_shared(smem_u32(full), 0);     // + 8 * stage
  const uint32_t tempty_leader = mapa_shared(smem_u32(tempty), 0); // + 8 * buf

  if (warp == 0) {
    // ------------------------------------------------------------ weight loads
    // router: W_router is re-read by every token run -> keep
    const uint64_t pol_a =
        (MODE != kModeRouter && p.weights_evict_first) ? policy_evict_first() : policy_evict_last();
    int stage = 0;
    uint32_t phase = 0;
    uint32_t issued = 0;
    bool ok = true;
    for (int it = 0, u = snake_unit(0, pair, npairs); ok && u < num_units; u = snake_unit(++it, pair, npairs)) {
      const Unit un = get_unit<MODE>(p, u);
      const bool sh = (MODE != kModeRouter) && un.g >= p.E;
      const int sidx = sh ? un.g - p.E : 0;
      const int K = (MODE == kModeDown) ? (sh ? p.fs : p.f) : p.d;
      const int KB = K / kTileK;
      // router: this unit's k-blocks [kb0, kb1) (its slice of d); the expert GEMMs: all of K
      const int kb0 = (MODE == kModeRouter) ? un.g * p.router_kbs : 0;
      const int kb1 = (MODE == kModeRouter) ? min(KB, kb0 + p.router_kbs) : KB;
      const CUtensorMap* mA = &p.mapA[sh ? 2 : 0];
      const int a_c2 = (MODE == kModeRouter) ? 0 : (sh ? sidx : un.g);
      // this CTA's token rows (half of the run) land on the same stage barrier
      // without arriving on it; their bytes are expected here
      const uint32_t tx_bytes = NA * kATileBytes + static_cast<uint32_t>(un.n >> 1) * 128u;
      const int wrow = un.wb * kWbRows + static_cast<int>(rank) * kTileRows;
      if constexpr (NA == 1) {
        // one weight tile per stage: lane 0 alone
        int got = 1;
        if (lane == 0) {
          for (int kb = kb0; kb < kb1; ++kb) {
            if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, p.err, p.timeout_ns)) {
              got = 0;
              break;
            }
            const uint32_t fb = full_leader + 8u * stage;
            mbar_arrive_expect_tx_cluster(fb, tx_bytes);
            tma_load_3d_pair_hint(smem_u32(smem + static_cast<size_t>(stage) * stage_bytes), mA, fb, kb * kTileK,
                                  wrow, a_c2, pol_a);
            ++issued;
            if (++stage == S) {
              stage = 0;
              phase ^= 1u;
            }
          }
        }
        got = __shfl_sync(0xffffffffu, got, 0);
        if (!got) ok = false;
      } else {
        // gate and up tile: lane 0 arms the stage, lanes 0 and 1 load one
        // tile each (measured faster than one lane loading both)
        for (int kb = kb0; kb < kb1; ++kb) {
          int got = 1;
          if (lane == 0) {
            if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, p.err, p.timeout_ns))
              got = 0;
            else
              mbar_arrive_expect_tx_cluster(full_leader + 8u * stage, tx_bytes);
          }
          got = __shfl_sync(0xffffffffu, got, 0);
          if (!got) {
            ok = false;
            break;
          }
          if (lane < NA)
            tma_load_3d_pair_hint(smem_u32(smem + static_cast<size_t>(stage) * stage_bytes) + lane * kATileBytes,
                                  mA + lane, full_leader + 8u * stage, kb * kTileK, wrow, a_c2, pol_a);
          ++issued;
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    }
    // The leader's stage barriers count both CTAs' bytes: drain the last ones.
    if (lane == 0 && rank == 0) {
      const uint32_t outstanding = issued < static_cast<uint32_t>(S) ? issued : static_cast<uint32_t>(S);
      for (uint32_t i = 1; i <= outstanding; ++i) {
        const uint32_t I = issued - i;
        mbar_wait_drain(&full[I % S], (I / S) & 1u, p.timeout_ns);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ---------------------------------------------------------- MMA issuer (leader)
      int stage = 0;
      uint32_t phase = 0;
      uint32_t ucount = 0;
      bool any = false;
      bool ok = true;
      if constexpr (MODE == kModeRouter) {
        // Router: M = 256 experts (128 per CTA), N = the run's tokens; the
        // accumulator is drained every kRouterDrainKB k-blocks into fp32
        // registers by both CTAs' epilogues (as in the single-CTA router),
        // through nbuf buffers of nmax columns.
        uint32_t dc = 0;
        for (int it = 0, u = snake_unit(0, pair, npairs); ok && u < num_units; u = snake_unit(++it, pair, npairs)) {
          const Unit un = get_unit<MODE>(p, u);
          const int KB = p.d / kTileK;
          const int kb0 = un.g * p.router_kbs;
          const int kb1 = min(KB, kb0 + p.router_kbs);
          const uint32_t idesc = idesc_bf16_f32(2 * kTileRows, un.n);
          uint32_t dcol = tmem_base;
          int buf = 0;
          for (int kb = kb0; kb < kb1; ++kb) {
            const int sub = (kb - kb0) % kRouterDrainKB;
            if (sub == 0) {
              buf = static_cast<int>(dc % static_cast<uint32_t>(p.nbuf));
              const uint32_t bpar = (dc / static_cast<uint32_t>(p.nbuf)) & 1u;
              if (!mbar_wait(&tempty[buf], bpar ^ 1u, abort_flag, p.err, p.timeout_ns)) {
                ok = false;
                break;
              }
              tc_fence_after();
              dcol = tmem_base + static_cast<uint32_t>(buf * nmax);
            }
            if (!mbar_wait(&full[stage], phase, abort_flag, p.err, p.timeout_ns)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t sbase = smem_u32(smem + static_cast<size_t>(stage) * stage_bytes);
            const uint64_t adesc = sw128_kmajor_desc(sbase);
            const uint64_t bdesc = sw128_kmajor_desc(sbase + kATileBytes);
#pragma unroll
            for (int ks = 0; ks < kTileK / 16; ++ks)
              tc_mma_bf16_pair(dcol, adesc + 2u * ks, bdesc + 2u * ks, idesc, (sub | ks) != 0 ? 1u : 0u);
            any = true;
            tc_commit_pair(&empty[stage], 0x3);
            if (++stage == S) {
              stage = 0;
              phase ^= 1u;
            }
            if (sub == kRouterDrainKB - 1 || kb == kb1 - 1) {
              tc_commit_pair(&tfull[buf], 0x3);
              ++dc;
            }
          }
        }
      }
      for (int it = 0, u = snake_unit(0, pair, npairs); MODE != kModeRouter && ok && u < num_units;
           u = snake_unit(++it, pair, npairs)) {
        const Unit un = get_unit<MODE>(p, u);
        const bool sh = un.g >= p.E;
        const int K = (MODE == kModeDown) ? (sh ? p.fs : p.f) : p.d;
        const int KB = K / kTileK;
        const int buf = static_cast<int>(ucount % static_cast<uint32_t>(p.nbuf));
        const uint32_t bpar = (ucount / static_cast<uint32_t>(p.nbuf)) & 1u;
        if (!mbar_wait(&tempty[buf], bpar ^ 1u, abort_flag, p.err, p.timeout_ns)) break;
        tc_fence_after();
        const uint32_t idesc = idesc_bf16_f32(2 * kTileRows, un.n);
        const uint32_t dcol = tmem_base + static_cast<uint32_t>(buf * NA * nmax);
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag, p.err, p.timeout_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sbase = smem_u32(smem + static_cast<size_t>(stage) * stage_bytes);
          const uint64_t bdesc = sw128_kmajor_desc(sbase + NA * kATileBytes);
          uint64_t adesc[NA];
#pragma unroll
          for (int a = 0; a < NA; ++a) adesc[a] = sw128_kmajor_desc(sbase + a * kATileBytes);
#pragma unroll
          for (int ks = 0; ks < kTileK / 16; ++ks) {
#pragma unroll
            for (int a = 0; a < NA; ++a)
              tc_mma_bf16_pair(dcol + static_cast<uint32_t>(a * nmax), adesc[a] + 2u * ks, bdesc + 2u * ks, idesc,
                               (kb | ks) != 0 ? 1u : 0u);
          }
          any = true;
          tc_commit_pair(&empty[stage], 0x3);
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit_pair(&tfull[buf], 0x3);
        ++ucount;
      }
      if (any) {
        tc_commit_pair(drain, 0x1);
        mbar_wait_drain(drain, 0, p.timeout_ns);
      }
    }
    __syncwarp();
  } else if (MODE != kModeGateUp && warp == 2 + EW) {
    // ------------------------------------------------------------ token-row loads (down, router)
    // A second producer: this CTA's half of each unit's token rows (H rows,
    // or x rows for the router), counted on the leader's stage barrier beside
    // the weight tiles, so that the two operands' loads are issued in
    // parallel.  It does not arrive: the weight producer's arrival expects
    // these bytes too (they may land first; the transaction count then runs
    // below zero until it).  The weight producer of rank 0 drains the stages
    // at the end (a stage completes only when all of its bytes have landed).
    const uint64_t pol_b = policy_evict_last();
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int it = 0, u = snake_unit(0, pair, npairs); ok && u < num_units; u = snake_unit(++it, pair, npairs)) {
      const Unit un = get_unit<MODE>(p, u);
      const bool sh = (MODE != kModeRouter) && un.g >= p.E;
      const int sidx = sh ? un.g - p.E : 0;
      const int K = (MODE == kModeDown) ? (sh ? p.fs : p.f) : p.d;
      const int KB = K / kTileK;
      const int kb0 = (MODE == kModeRouter) ? un.g * p.router_kbs : 0;
      const int kb1 = (MODE == kModeRouter) ? min(KB, kb0 + p.router_kbs) : KB;
      const CUtensorMap* mB = p.mapB[sh ? 1 : 0];
      const int half = un.n >> 1;
      const int brow0 = (sh ? sidx * p.Tp : 0) + un.row0 + static_cast<int>(rank) * half;
      int got = 1;
      if (lane == 0) {
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, p.err, p.timeout_ns)) {
            got = 0;
            break;
          }
          const uint32_t sbase = smem_u32(smem + static_cast<size_t>(stage) * stage_bytes);
          tma_load_rows<true>(sbase + NA * kATileBytes, mB, full_leader + 8u * stage, kb * kTileK, brow0, half,
                              pol_b);
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      got = __shfl_sync(0xffffffffu, got, 0);
      if (!got) ok = false;
    }
  } else if (MODE == kModeGateUp && warp >= 2 + EW) {
    // ------------------------------------------------------------ row gather (this CTA's half)
    // Gather warp gw lands rows [32 gw, 32 gw + 32) of this CTA's half of
    // the token tile with 4-row tensor gathers (one 128-byte row piece each,
    // swizzled by the map like a tiled load), one per lane, counted on the
    // leader's stage barrier; this CTA's weight producer expects their bytes
    // (a gather may land before that arrival: the barrier's transaction
    // count then runs below zero until it, and the phase cannot complete
    // while the arrival is pending).
    const int gw = warp - (2 + EW);
    const uint64_t pol_x = policy_evict_last();
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int it = 0, u = snake_unit(0, pair, npairs); ok && u < num_units; u = snake_unit(++it, pair, npairs)) {
      const Unit un = get_unit<MODE>(p, u);
      const bool sh = un.g >= p.E;
      const int half = un.n >> 1;
      const int nr = min(max(half - 32 * gw, 0), 32);             // a multiple of 16
      const int rb = un.row0 + static_cast<int>(rank) * half + 32 * gw;
      // clamped: a row never reads outside x, even for an invalid routing
      const int my = (lane < nr) ? min(max(sh ? rb + lane : __ldg(p.perm + rb + lane), 0), p.T - 1) : 0;
      // lane j < nr / 4 gathers rows 4 j .. 4 j + 3 of the warp's 32
      const int t0 = __shfl_sync(0xffffffffu, my, (4 * lane) & 31);
      const int t1 = __shfl_sync(0xffffffffu, my, (4 * lane + 1) & 31);
      const int t2 = __shfl_sync(0xffffffffu, my, (4 * lane + 2) & 31);
      const int t3 = __shfl_sync(0xffffffffu, my, (4 * lane + 3) & 31);
      const int KB = p.d / kTileK;
      for (int kb = 0; kb < KB; ++kb) {
        int got = 1;
        // the stage is free once its previous MMAs are done; the weight
        // producer's arrival expects these bytes (before or after they land)
        if (lane == 0 && !mbar_wait(&empty[stage], phase ^ 1u, abort_flag, p.err, p.timeout_ns)) got = 0;
        got = __shfl_sync(0xffffffffu, got, 0);
        if (!got) {
          ok = false;
          break;
        }
        if (sh) {
          // a shared expert reads its token rows in order: one tiled load of
          // this CTA's half of the run (rows past T read as zeros; their
          // outputs are never combined)
          if (gw == 0 && lane == 0)
            tma_load_rows<true>(smem_u32(smem + static_cast<size_t>(stage) * stage_bytes) + NA * kATileBytes,
                                p.mapB[0], full_leader + 8u * stage, kb * kTileK,
                                un.row0 + static_cast<int>(rank) * half, half, pol_x);
        } else if (4 * lane < nr) {
          // the gathers are issued by several lanes at once
          const uint32_t dst = smem_u32(smem + static_cast<size_t>(stage) * stage_bytes) + NA * kATileBytes +
                               static_cast<uint32_t>(32 * gw + 4 * lane) * 128u;
          tma_gather4_pair(dst, &p.mapX, full_leader + 8u * stage, kb * kTileK, t0, t1, t2, t3, pol_x);
        }
        if (++stage == S) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
  } else if (warp >= 2 && warp < 2 + EW) {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int q = warp & 3;
    uint8_t* stg = epi + (warp - 2) * (kEpiBytes / EW);
    if constexpr (MODE == kModeRouter) {
      // Router: warp (q, half) sums experts 32 q .. + 31 of this CTA's 128
      // (thread = expert row) over one half of the run's token columns in
      // fp32 registers, one drained partial accumulator at a time, then
      // writes logits[t, e] through a transpose in its staging buffer.
      const int half = (warp - 2) >> 2;
      uint32_t dc = 0;
      bool ok = true;
      for (int it = 0, u = snake_unit(0, pair, npairs); ok && u < num_units; u = snake_unit(++it, pair, npairs)) {
        const Unit un = get_unit<MODE>(p, u);
        const int KB = p.d / kTileK;
        const int kb0 = un.g * p.router_kbs;
        const int nkb = min(KB, kb0 + p.router_kbs) - kb0;
        const int nd = (nkb + kRouterDrainKB - 1) / kRouterDrainKB;
        float* const lbase = reinterpret_cast<float*>(p.out_r) + static_cast<size_t>(un.g) * p.T * p.E;
        const int feat0 = un.wb * kWbRows + static_cast<int>(rank) * kTileRows + 32 * q;
        const bool live = feat0 < p.E;
        const int ncol = un.n >> 1;     // this warp's token columns [c0, c0 + ncol): a multiple of 16, <= 128
        const int c0 = half * ncol;
        float acc[128];
#pragma unroll
        for (int j = 0; j < 128; ++j) acc[j] = 0.0f;
        for (int i = 0; i < nd; ++i) {
          const int buf = static_cast<int>(dc % static_cast<uint32_t>(p.nbuf));
          const uint32_t bpar = (dc / static_cast<uint32_t>(p.nbuf)) & 1u;
          int got = 1;
          if (lane == 0) got = mbar_wait(&tfull[buf], bpar, abort_flag, p.err, p.timeout_ns) ? 1 : 0;
          got = __shfl_sync(0xffffffffu, got, 0);
          if (!got) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (live) {
            const uint32_t tb = tmem_base + (static_cast<uint32_t>(32 * q) << 16) +
                                static_cast<uint32_t>(buf * nmax + c0);
            // 16 columns per round trip (the 128 sums leave room for one load)
#pragma unroll
            for (int g = 0; g < 8; ++g) {
              if (16 * g < ncol) {
                uint32_t v[16];
                tmem_ld_32x32b_x16(tb + static_cast<uint32_t>(16 * g), v);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 16; ++j) acc[16 * g + j] += __uint_as_float(v[j]);
              }
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(tempty_leader + 8u * buf);
          ++dc;
        }
        if (!ok || !live) continue;
        float* sf = reinterpret_cast<float*>(stg);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          if (16 * c < ncol) {
#pragma unroll
            for (int i = 0; i < 16; ++i) sf[i * 32 + lane] = acc[16 * c + i];
            __syncwarp();
#pragma unroll
            for (int rep = 0; rep < 4; ++rep) {
              const int cc = lane + 32 * rep;
              const int tok = cc >> 3, part = cc & 7;
              const int t = un.row0 + c0 + 16 * c + tok;
              const int e = feat0 + part * 4;
              if (t < p.T) {
                float* dst = lbase + static_cast<size_t>(t) * p.E + e;
                const float4 vv = *reinterpret_cast<const float4*>(sf + tok * 32 + part * 4);
                if ((p.E & 3) == 0 && e + 3 < p.E) {
                  *reinterpret_cast<float4*>(dst) = vv;
                } else {
                  if (e + 0 < p.E) dst[0] = vv.x;
                  if (e + 1 < p.E) dst[1] = vv.y;
                  if (e + 2 < p.E) dst[2] = vv.z;
                  if (e + 3 < p.E) dst[3] = vv.w;
                }
              }
            }
            __syncwarp();
          }
        }
      }
    } else {
    uint32_t ucount = 0;
    for (int it = 0, u = snake_unit(0, pair, npairs); u < num_units; u = snake_unit(++it, pair, npairs)) {
      const Unit un = get_unit<MODE>(p, u);
      const bool sh = un.g >= p.E;
      const int sidx = sh ? un.g - p.E : 0;
      const int buf = static_cast<int>(ucount % static_cast<uint32_t>(p.nbuf));
      const uint32_t bpar = (ucount / static_cast<uint32_t>(p.nbuf)) & 1u;
      const int half = (warp - 2) >> 2;                                   // column blocks half*16 + 32 i
      if constexpr (MODE == kModeDown) {
        // Warp (q, half): features 32 q .. + 31 of this CTA's 128 rows, token
        // columns 16 half + 32 i .. + 15 (i < 8).  Each 16-column block is
        // read from tensor memory as two 16-lane fragments, scaled by the
        // combine weights in fp32, packed to bf16 pairs and written
        // transposed (token rows, 64 bytes of features each) by stmatrix,
        // then stored to global memory as 16-byte row pieces.  The weights
        // sit in shared memory in block order: wsm[16 i + j] = weight of
        // column 16 half + 32 i + j.
        float* wsm = reinterpret_cast<float*>(stg + 16 * kStgRow);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int idx = 32 * j + lane;
          const int c = 16 * half + 32 * (idx >> 4) + (idx & 15);
          wsm[idx] = (!sh && c < un.n) ? __ldg(p.roww + un.row0 + c) : 1.0f;
        }
        __syncwarp();
        int got = 1;
        if (lane == 0) got = mbar_wait(&tfull[buf], bpar, abort_flag, p.err, p.timeout_ns) ? 1 : 0;
        got = __shfl_sync(0xffffffffu, got, 0);
        if (!got) break;
        tc_fence_after();
        const uint32_t tbase =
            tmem_base + (static_cast<uint32_t>(32 * q) << 16) + static_cast<uint32_t>(buf * nmax);
        const int feat0 = un.wb * kWbRows + static_cast<int>(rank) * kTileRows + 32 * q;
        if (feat0 < p.d) {
          __nv_bfloat16* outp = reinterpret_cast<__nv_bfloat16*>(sh ? p.out_s : p.out_r);
          const size_t rbase = (sh ? static_cast<size_t>(sidx) * p.Tp : 0) + static_cast<size_t>(un.row0);
          const uint32_t sbase = smem_u32(stg);
          const int tq = lane & 3;
          const int mi = lane >> 3, mj = lane & 7;     // this thread's stmatrix row: matrix mi, row mj
          uint32_t va[2][8], vb[2][8];
          auto load = [&](uint32_t (&v)[2][8], int c) {
            tmem_ld_16x256b_x2(tbase + static_cast<uint32_t>(c), v[0]);
            tmem_ld_16x256b_x2(tbase + (16u << 16) + static_cast<uint32_t>(c), v[1]);
          };
          auto emit = [&](const uint32_t (&v)[2][8], int i) {
            const int c = 16 * half + 32 * i;
            const float2 w0 = *reinterpret_cast<const float2*>(wsm + 16 * i + 2 * tq);
            const float2 w1 = *reinterpret_cast<const float2*>(wsm + 16 * i + 8 + 2 * tq);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              // matrices: 0 = features 16h + 0..7 x tokens 0..7, 1 = features
              // 16h + 8..15 x tokens 0..7, 2 and 3 = the same for tokens 8..15
              const uint32_t m0 = pack_bf16x2(__uint_as_float(v[h][0]) * w0.x, __uint_as_float(v[h][1]) * w0.y);
              const uint32_t m1 = pack_bf16x2(__uint_as_float(v[h][2]) * w0.x, __uint_as_float(v[h][3]) * w0.y);
              const uint32_t m2 = pack_bf16x2(__uint_as_float(v[h][4]) * w1.x, __uint_as_float(v[h][5]) * w1.y);
              const uint32_t m3 = pack_bf16x2(__uint_as_float(v[h][6]) * w1.x, __uint_as_float(v[h][7]) * w1.y);
              stmatrix_x4_trans(sbase + static_cast<uint32_t>((8 * (mi >> 1) + mj) * kStgRow +
                                                              (16 * h + 8 * (mi & 1)) * 2),
                                m0, m1, m2, m3);
            }
            __syncwarp();
#pragma unroll
            for (int rep = 0; rep < 2; ++rep) {
              const int cc = lane + 32 * rep;
              const int tok = cc >> 2, part = cc & 3;
              const uint4 o = *reinterpret_cast<const uint4*>(stg + tok * kStgRow + part * 16);
              *reinterpret_cast<uint4*>(outp + (rbase + c + tok) * p.d + feat0 + part * 8) = o;
            }
            __syncwarp();
          };
          // two fragment sets: the next block's loads are in flight while the
          // current one is converted and stored
          if (16 * half < un.n) load(va, 16 * half);
#pragma unroll
          for (int i = 0; i < 8; i += 2) {
            if (16 * half + 32 * i >= un.n) break;
            tmem_ld_wait();
            if (16 * half + 32 * (i + 1) < un.n) load(vb, 16 * half + 32 * (i + 1));
            emit(va, i);
            if (16 * half + 32 * (i + 1) >= un.n) break;
            tmem_ld_wait();
            if (i + 2 < 8 && 16 * half + 32 * (i + 2) < un.n) load(va, 16 * half + 32 * (i + 2));
            emit(vb, i + 1);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(tempty_leader + 8u * buf);
        ++ucount;
        continue;
      }
      // gate/up: H = SiLU(gate) * up for features 32 q .. + 31 of this CTA's
      // 128 rows and the same token columns as down, through the same
      // fragment loads and transposed stmatrix stores.
      int got = 1;
      if (lane == 0) got = mbar_wait(&tfull[buf], bpar, abort_flag, p.err, p.timeout_ns) ? 1 : 0;
      got = __shfl_sync(0xffffffffu, got, 0);
      if (!got) break;
      tc_fence_after();
      const uint32_t tbase =
          tmem_base + (static_cast<uint32_t>(32 * q) << 16) + static_cast<uint32_t>(buf * NA * nmax);
      const int feat0 = un.wb * kWbRows + static_cast<int>(rank) * kTileRows + 32 * q;
      const int ld = sh ? p.fs : p.f;
      if (feat0 < ld) {
        __nv_bfloat16* outp = reinterpret_cast<__nv_bfloat16*>(sh ? p.out_s : p.out_r);
        const size_t rbase = (sh ? static_cast<size_t>(sidx) * p.Tp : 0) + static_cast<size_t>(un.row0);
        const uint32_t sbase = smem_u32(stg);
        const int mi = lane >> 3, mj = lane & 7;
        uint32_t ga[2][8], ua[2][8], gb[2][8], ub[2][8];
        auto load = [&](uint32_t (&g)[2][8], uint32_t (&v)[2][8], int c) {
          tmem_ld_16x256b_x2(tbase + static_cast<uint32_t>(c), g[0]);
          tmem_ld_16x256b_x2(tbase + (16u << 16) + static_cast<uint32_t>(c), g[1]);
          tmem_ld_16x256b_x2(tbase + static_cast<uint32_t>(nmax + c), v[0]);
          tmem_ld_16x256b_x2(tbase + (16u << 16) + static_cast<uint32_t>(nmax + c), v[1]);
        };
        auto emit = [&](const uint32_t (&g)[2][8], const uint32_t (&v)[2][8], int i) {
          const int c = 16 * half + 32 * i;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint32_t m[4];
#pragma unroll
            for (int k = 0; k < 4; ++k)
              m[k] = pack_bf16x2(silu_f(__uint_as_float(g[h][2 * k])) * __uint_as_float(v[h][2 * k]),
                                 silu_f(__uint_as_float(g[h][2 * k + 1])) * __uint_as_float(v[h][2 * k + 1]));
            stmatrix_x4_trans(
                sbase + static_cast<uint32_t>((8 * (mi >> 1) + mj) * kStgRow + (16 * h + 8 * (mi & 1)) * 2), m[0],
                m[1], m[2], m[3]);
          }
          __syncwarp();
#pragma unroll
          for (int rep = 0; rep < 2; ++rep) {
            const int cc = lane + 32 * rep;
            const int tok = cc >> 2, part = cc & 3;
            const uint4 o = *reinterpret_cast<const uint4*>(stg + tok * kStgRow + part * 16);
            *reinterpret_cast<uint4*>(outp + (rbase + c + tok) * ld + feat0 + part * 8) = o;
          }
          __syncwarp();
        };
        if (16 * half < un.n) load(ga, ua, 16 * half);
#pragma unroll
        for (int i = 0; i < 8; i += 2) {
          if (16 * half + 32 * i >= un.n) break;
          tmem_ld_wait();
          if (16 * half + 32 * (i + 1) < un.n) load(gb, ub, 16 * half + 32 * (i + 1));
          emit(ga, ua, i);
          if (16 * half + 32 * (i + 1) >= un.n) break;
          tmem_ld_wait();
          if (i + 2 < 8 && 16 * half + 32 * (i + 2) < un.n) load(ga, ua, 16 * half + 32 * (i + 2));
          emit(gb, ub, i + 1);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tempty_leader + 8u * buf);
      ++ucount;
    }
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();                                    // no CTA leaves while its peer may still touch it
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

}  // namespace

size_t gemm_smem_bytes(int mode, int nmax, int* stages) {
  const int NA = (mode == kModeRouter) ? 1 : 2;
  const size_t stage_bytes = NA * static_cast<size_t>(kATileBytes) + static_cast<size_t>(nmax) * 128;
  const size_t fixed = kSmemAlign + epi_bytes_of(mode) + kSmemTail;
  const size_t budget = 232448;   // sm_100 opt-in maximum per block
  int s = static_cast<int>((budget - fixed) / stage_bytes);
  if (s > kMaxStages) s = kMaxStages;
  if (stages) *stages = s;
  return fixed + static_cast<size_t>(s) * stage_bytes;
}

size_t gemm_pair_smem_bytes(int mode, int nmax, int* stages) {
  const int NA = (mode == kModeGateUp) ? 2 : 1;
  const size_t stage_bytes = NA * static_cast<size_t>(kATileBytes) + static_cast<size_t>(nmax / 2) * 128;
  const size_t fixed = kSmemAlign + pair_epi_bytes_of(mode) + kSmemTail;
  const size_t budget = 232448;
  int s = static_cast<int>((budget - fixed) / stage_bytes);
  if (s > kMaxStages) s = kMaxStages;
  if (stages) *stages = s;
  return fixed + static_cast<size_t>(s) * stage_bytes;
}

template <int MODE>
static int launch_pair_mode(const GemmParams& prm, int grid, size_t smem, cudaStream_t st) {
  static std::atomic<int> limit[64];
  const int rc = raise_smem_limit(moe_gemm_pair_kernel<MODE>, limit, static_cast<int>(smem));
  if (rc != MOE_OK) return rc;
  return launch_chained(moe_gemm_pair_kernel<MODE>, dim3(grid), dim3(pair_threads_of(MODE)), smem, st, prm) ==
                 cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}

int launch_gemm_pair(int mode, const GemmParams& prm, int grid, size_t smem, cudaStream_t st) {
  grid &= ~1;
  if (grid < 2) return MOE_ERR_UNSUPPORTED;
  switch (mode) {
    case kModeRouter: return launch_pair_mode<kModeRouter>(prm, grid, smem, st);
    case kModeGateUp: return launch_pair_mode<kModeGateUp>(prm, grid, smem, st);
    case kModeDown: return launch_pair_mode<kModeDown>(prm, grid, smem, st);
    default: return MOE_ERR_INVALID_ARG;
  }
}

size_t gemm_f8_smem_bytes(int mode, int nmax, int* stages, int* tok_stages, int* raw_stages) {
  const int NA = 2;   // gate/up and down both stage two weight tiles
  const size_t stage_bytes = 0;   // widened tiles live in tensor memory
  const size_t tok_bytes = static_cast<size_t>(nmax) * 128;
  const size_t raw_stage = NA * static_cast<size_t>(kRawTile);
  const size_t fixed = kSmemAlign + epi_bytes_of(mode) + kSmemTail;
  const size_t budget = 232448;
  const int s = kAStages;
  int ts = static_cast<int>(65536 / tok_bytes);   // 64 KB of token tiles
  if (ts < 2) ts = 2;
  if (ts > kMaxTokStages) ts = kMaxTokStages;
  int r = static_cast<int>((budget - fixed - s * stage_bytes - ts * tok_bytes) / raw_stage);
  if (r > kMaxRawStages) r = kMaxRawStages;
  if (stages) *stages = s;
  if (tok_stages) *tok_stages = ts;
  if (raw_stages) *raw_stages = r;
  return fixed + s * stage_bytes + ts * tok_bytes + static_cast<size_t>(r) * raw_stage;
}

template <int MODE, bool F8>
static int launch_mode(const GemmParams& prm, int grid, size_t smem, cudaStream_t st) {
  static std::atomic<int> limit[64];
  const int rc = raise_smem_limit(moe_gemm_kernel<MODE, F8>, limit, static_cast<int>(smem));
  if (rc != MOE_OK) return rc;
  return launch_chained(moe_gemm_kernel<MODE, F8>, dim3(grid), dim3(threads_of(MODE, F8)), smem, st, prm) ==
                 cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}

int launch_gemm(int mode, const GemmParams& prm, int grid, size_t smem, cudaStream_t st, bool f8) {
  if (grid < 1) return MOE_OK;
  if (f8) {
    // the accumulators must fit below the widened tiles' columns
    if (prm.raw_stages < 2 || prm.raw_stages > kMaxRawStages || prm.stages != kAStages || prm.tok_stages < 2 ||
        prm.tok_stages > kMaxTokStages || prm.nmax > 128 || 2 * prm.nmax * prm.nbuf > static_cast<int>(kAColBase))
      return MOE_ERR_INVALID_ARG;
    switch (mode) {
      case kModeGateUp: return launch_mode<kModeGateUp, true>(prm, grid, smem, st);
      case kModeDown: return launch_mode<kModeDown, true>(prm, grid, smem, st);
      default: return MOE_ERR_INVALID_ARG;
    }
  }
  switch (mode) {
    case kModeRouter: return launch_mode<kModeRouter, false>(prm, grid, smem, st);
    case kModeGateUp: return launch_mode<kModeGateUp, false>(prm, grid, smem, st);
    case kModeDown: return launch_mode<kModeDown, false>(prm, grid, smem, st);
    default: return MOE_ERR_INVALID_ARG;
  }
}

}  // namespace moe
