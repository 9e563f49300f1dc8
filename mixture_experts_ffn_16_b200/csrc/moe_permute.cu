// moe_permute.cu - token -> expert dispatch (step a3), entirely on the device.
//
//   count   : per block of 256 tokens, a bit mask per (warp, expert) of the
//             lanes whose token picked the expert; popcounts give the block's
//             per-expert histogram.
//   scan    : one block: per expert, exclusive prefix over blocks (-> each
//             block's offset inside the expert's segment) and the expert's
//             count; then an exclusive scan over experts of the padded segment
//             sizes (rows stay in expert order), a rank of every expert by
//             padded rows, exclusive scans of the GEMM work-unit counts in
//             list order (largest, smallest, 2nd largest, ...); writes the
//             work lists and fills the padding rows.
//   scatter : recomputes the masks (each of the ceil(k/2) CTAs of a block
//             places two slots of its tokens); a (token, slot) pair's row is
//             segment start + block offset + popcount of the lower lanes of
//             the lower warps and of its own warp: rows inside an expert are in
//             ascending token order, so the layout is deterministic.
//
// Row space: expert e owns rows [roff[e], roff[e] + pad(count[e])) with
// pad() rounding up to 16 rows (32 when the expert GEMMs run on CTA pairs); padding
// rows point at token 0 with weight 0.  Work units are int4
// {group, weight block, first row, rows (a multiple of the padding)}; shared
// experts are groups E..E+S-1 over rows 0..pad(T) of their own row space and
// come first in each list.
#include "moe_internal.h"
#include "moe_ptx.cuh"

namespace moe {

namespace {

constexpr int kWarps = kPermBlock / 32;
constexpr int kScanThreads = 1024;
constexpr int kScatterSlots = 2;   // (token, slot) pairs per scatter thread

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm volatile("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Fills masks[w*E + e] for this block; flags invalid routing.
__device__ void build_masks(const int32_t* __restrict__ topk_idx, int T, int E, int k,
                            uint32_t* masks, uint32_t* err) {
  for (int i = threadIdx.x; i < kWarps * E; i += blockDim.x) masks[i] = 0u;
  __syncthreads();
  const int t = blockIdx.x * kPermBlock + threadIdx.x;
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (t < T) {
    bool bad = false;
    for (int j = 0; j < k; ++j) {
      const int e = topk_idx[static_cast<size_t>(t) * k + j];
      if (e < 0 || e >= E) {
        bad = true;
        continue;
      }
      const uint32_t old = atomicOr(&masks[w * E + e], 1u << lane);
      if (old & (1u << lane)) bad = true;   // the same expert twice in one token
    }
    if (bad) atomicOr(err, kDevErrBadRouting);
  }
  __syncthreads();
}

__global__ void __launch_bounds__(kPermBlock)
permute_count_kernel(const int32_t* __restrict__ topk_idx, int T, int E, int k,
                     int32_t* __restrict__ blkcnt, uint32_t* err) {
  extern __shared__ uint32_t masks[];
  chain_wait();
  build_masks(topk_idx, T, E, k, masks, err);
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int c = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) c += __popc(masks[w * E + e]);
    blkcnt[static_cast<size_t>(blockIdx.x) * E + e] = c;
  }
}

// Exclusive block-wide scan of three ints per thread (kScanThreads threads):
// shuffles inside each warp, then one warp scans the 32 warp totals.
__device__ int3 block_exclusive_scan3(int3 v, int3* total) {
  __shared__ int3 wsum[kScanThreads / 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int3 inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int x = __shfl_up_sync(0xffffffffu, inc.x, o);
    const int y = __shfl_up_sync(0xffffffffu, inc.y, o);
    const int z = __shfl_up_sync(0xffffffffu, inc.z, o);
    if (lane >= o) {
      inc.x += x;
      inc.y += y;
      inc.z += z;
    }
  }
  if (lane == 31) wsum[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    int3 w = wsum[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int x = __shfl_up_sync(0xffffffffu, w.x, o);
      const int y = __shfl_up_sync(0xffffffffu, w.y, o);
      const int z = __shfl_up_sync(0xffffffffu, w.z, o);
      if (lane >= o) {
        w.x += x;
        w.y += y;
        w.z += z;
      }
    }
    wsum[lane] = w;                              // inclusive over warps
  }
  __syncthreads();
  const int3 base = warp > 0 ? wsum[warp - 1] : make_int3(0, 0, 0);
  *total = wsum[kScanThreads / 32 - 1];
  __syncthreads();   // wsum may be reused by the next call
  return make_int3(base.x + inc.x - v.x, base.y + inc.y - v.y, base.z + inc.z - v.z);
}

struct ScanArgs {
  int32_t* blkcnt;   // [nb, E] in: counts, out: exclusive offsets over blocks
  int32_t* counts;   // [E]
  int32_t* roff;     // [E+1]
  int32_t* perm;     // [Rcap]
  float* roww;       // [Rcap]
  int4* units1;
  int4* units2;
  int32_t* nunits;   // [4]: gate/up units, down units, padded routed rows, 0
  int nb, E, T, Tp, rowpad;
  int nmax1, nmax2, nwb1, nwb1s, nwb2, S;
  int shared_units1, shared_units2;
  int plan_tag;
};

__global__ void __launch_bounds__(kScanThreads) permute_scan_kernel(ScanArgs a) {
  // Padded rows of every expert, then (by rank) its unit counts and their
  // exclusive offsets, in the work lists' interleaved size order.
  __shared__ __align__(16) int s_key[kMaxE];
  __shared__ int s_u1[kMaxE], s_u2[kMaxE];
  chain_wait();
  // Experts per thread, contiguous: one up to E = 1024, else two.
  constexpr int kPer = (kMaxE + kScanThreads - 1) / kScanThreads;
  const int per = a.E > kScanThreads ? kPer : 1;
  int cnt[kPer], pad[kPer], u1[kPer], u2[kPer], rank[kPer];
  int sp = 0;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int e = (i < per) ? threadIdx.x * per + i : a.E;
    int c = 0;
    if (e < a.E) {
      // Column e of the block histogram: exclusive prefix over blocks.  The
      // loads of a batch are issued before any store so they overlap.
      int32_t* col = a.blkcnt + e;
      for (int b0 = 0; b0 < a.nb; b0 += 16) {
        int v[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] = (b0 + j < a.nb) ? col[static_cast<size_t>(b0 + j) * a.E] : 0;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          if (b0 + j < a.nb) col[static_cast<size_t>(b0 + j) * a.E] = c;
          c += v[j];
        }
      }
      a.counts[e] = c;
    }
    cnt[i] = c;
    pad[i] = (c + a.rowpad - 1) / a.rowpad * a.rowpad;
    u1[i] = (pad[i] + a.nmax1 - 1) / a.nmax1 * a.nwb1;
    u2[i] = (pad[i] + a.nmax2 - 1) / a.nmax2 * a.nwb2;
    if (e < a.E) s_key[e] = pad[i];
    sp += pad[i];
  }
  int3 tot;
  const int3 ex = block_exclusive_scan3(make_int3(sp, 0, 0), &tot);
  const int tot_rows = tot.x;
  // Position of each expert in the work lists: experts ranked by padded rows
  // (more first, then the lower expert index: a strict order, ranks 0..E-1),
  // then interleaved from both ends of that ranking - largest, smallest, 2nd
  // largest, 2nd smallest, ...  Large experts' units keep the tensor cores
  // busy while small experts' units, which stream their weights once for few
  // tokens, run beside them instead of all together at the end.  Rows keep
  // the expert order.
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int e = (i < per) ? threadIdx.x * per + i : a.E;
    rank[i] = 0;
    if (e < a.E) {
      int r = 0;
      const int key = pad[i];
      const int E4 = a.E & ~3;
      for (int e2 = 0; e2 < E4; e2 += 4) {
        const int4 k4 = *reinterpret_cast<const int4*>(s_key + e2);
        r += (k4.x > key || (k4.x == key && e2 < e)) + (k4.y > key || (k4.y == key && e2 + 1 < e)) +
             (k4.z > key || (k4.z == key && e2 + 2 < e)) + (k4.w > key || (k4.w == key && e2 + 3 < e));
      }
      for (int e2 = E4; e2 < a.E; ++e2) r += (s_key[e2] > key || (s_key[e2] == key && e2 < e));
      // list position: largest, smallest, 2nd largest, 2nd smallest, ...
      r = (r < (a.E + 1) / 2) ? 2 * r : 2 * (a.E - 1 - r) + 1;
      rank[i] = r;
      s_u1[r] = u1[i];
      s_u2[r] = u2[i];
    }
  }
  __syncthreads();
  // Unit offsets in rank order (thread i owns ranks i*per ..).
  int r1[kPer], r2[kPer];
  int s1 = 0, s2 = 0;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int r = (i < per) ? threadIdx.x * per + i : a.E;
    r1[i] = r < a.E ? s_u1[r] : 0;
    r2[i] = r < a.E ? s_u2[r] : 0;
    s1 += r1[i];
    s2 += r2[i];
  }
  int3 utot;
  const int3 uex = block_exclusive_scan3(make_int3(0, s1, s2), &utot);
  const int tot1 = utot.y, tot2 = utot.z;
  __syncthreads();   // every s_u1 / s_u2 read above is done
  {
    int o1 = uex.y, o2 = uex.z;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int r = (i < per) ? threadIdx.x * per + i : a.E;
      if (r < a.E) {
        s_u1[r] = o1;
        s_u2[r] = o2;
      }
      o1 += r1[i];
      o2 += r2[i];
    }
  }
  __syncthreads();
  int ro = ex.x;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int e = (i < per) ? threadIdx.x * per + i : a.E;
    if (e < a.E) {
      a.roff[e] = ro;
      // padding rows of this expert's segment
      for (int r = cnt[i]; r < pad[i]; ++r) {
        a.perm[ro + r] = 0;
        a.roww[ro + r] = 0.0f;
      }
      const int o1 = a.shared_units1 + s_u1[rank[i]];
      const int o2 = a.shared_units2 + s_u2[rank[i]];
      // gate/up units: (e, wb, chunk), chunks inner so that consecutive units share a weight tile
      const int nch1 = (pad[i] + a.nmax1 - 1) / a.nmax1;
      for (int wb = 0; wb < a.nwb1; ++wb)
        for (int c = 0; c < nch1; ++c)
          a.units1[o1 + wb * nch1 + c] = make_int4(e, wb, ro + c * a.nmax1, min(a.nmax1, pad[i] - c * a.nmax1));
      const int nch2 = (pad[i] + a.nmax2 - 1) / a.nmax2;
      for (int wb = 0; wb < a.nwb2; ++wb)
        for (int c = 0; c < nch2; ++c)
          a.units2[o2 + wb * nch2 + c] = make_int4(e, wb, ro + c * a.nmax2, min(a.nmax2, pad[i] - c * a.nmax2));
    }
    ro += pad[i];
  }
  // Shared-expert units (first in each list).
  const int nch1s = (a.Tp + a.nmax1 - 1) / a.nmax1;
  const int nch2s = (a.Tp + a.nmax2 - 1) / a.nmax2;
  for (int i = threadIdx.x; i < a.shared_units1; i += blockDim.x) {
    const int c = i % nch1s, rest = i / nch1s;
    const int wb = rest % a.nwb1s, s = rest / a.nwb1s;
    a.units1[i] = make_int4(a.E + s, wb, c * a.nmax1, min(a.nmax1, a.Tp - c * a.nmax1));
  }
  for (int i = threadIdx.x; i < a.shared_units2; i += blockDim.x) {
    const int c = i % nch2s, rest = i / nch2s;
    const int wb = rest % a.nwb2, s = rest / a.nwb2;
    a.units2[i] = make_int4(a.E + s, wb, c * a.nmax2, min(a.nmax2, a.Tp - c * a.nmax2));
  }
  if (threadIdx.x == 0) {
    a.roff[a.E] = tot_rows;
    a.nunits[0] = a.shared_units1 + tot1;
    a.nunits[1] = a.shared_units2 + tot2;
    a.nunits[2] = tot_rows;
    a.nunits[3] = a.plan_tag;   // which work-list layout this is (checked by the expert GEMMs)
  }
}

__global__ void __launch_bounds__(kPermBlock)
permute_scatter_kernel(const int32_t* __restrict__ topk_idx, const float* __restrict__ topk_w, int T,
                       int E, int k, const int32_t* __restrict__ blkoff, const int32_t* __restrict__ roff,
                       int32_t* __restrict__ perm, float* __restrict__ roww, int32_t* __restrict__ inv,
                       uint32_t* err) {
  extern __shared__ uint32_t masks[];
  chain_wait();
  build_masks(topk_idx, T, E, k, masks, err);
  const int t = blockIdx.x * kPermBlock + threadIdx.x;
  if (t >= T) return;
  const int w = threadIdx.x >> 5;
  const uint32_t lt = lanemask_lt();
  // CTAs (x, y) share block x's masks; CTA y places slots [y s, y s + s).
  const int j0 = blockIdx.y * kScatterSlots;
  const int j1 = min(k, j0 + kScatterSlots);
  for (int j = j0; j < j1; ++j) {
    const size_t tj = static_cast<size_t>(t) * k + j;
    const int e = topk_idx[tj];
    if (e < 0 || e >= E) {
      inv[tj] = roff[0];   // invalid routing was flagged; keep the index in range
      continue;
    }
    int rank = __popc(masks[w * E + e] & lt);
    for (int v = 0; v < w; ++v) rank += __popc(masks[v * E + e]);
    const int row = roff[e] + blkoff[static_cast<size_t>(blockIdx.x) * E + e] + rank;
    perm[row] = t;
    roww[row] = topk_w[tj];
    inv[tj] = row;
  }
}

}  // namespace

int launch_permute(const Plan& p, const int32_t* topk_idx, const float* topk_w, char* ws,
                   cudaStream_t st) {
  int32_t* blkcnt = reinterpret_cast<int32_t*>(ws + p.blkcnt);
  uint32_t* err = reinterpret_cast<uint32_t*>(ws + p.err);
  const size_t msmem = static_cast<size_t>(kWarps) * p.E * sizeof(uint32_t);
  {
    // set once per device to the largest E's mask array
    static std::atomic<int> count_limit[64], scatter_limit[64];
    const int mx = kWarps * kMaxE * static_cast<int>(sizeof(uint32_t));
    int rc = raise_smem_limit(permute_count_kernel, count_limit, mx);
    if (rc == MOE_OK) rc = raise_smem_limit(permute_scatter_kernel, scatter_limit, mx);
    if (rc != MOE_OK) return rc;
  }
  if (launch_chained(permute_count_kernel, dim3(p.nb), dim3(kPermBlock), msmem, st, topk_idx, p.T, p.E, p.k, blkcnt,
                     err) != cudaSuccess)
    return MOE_ERR_CUDA;

  ScanArgs a;
  a.blkcnt = blkcnt;
  a.counts = reinterpret_cast<int32_t*>(ws + p.counts);
  a.roff = reinterpret_cast<int32_t*>(ws + p.roff);
  a.perm = reinterpret_cast<int32_t*>(ws + p.perm);
  a.roww = reinterpret_cast<float*>(ws + p.roww);
  a.units1 = reinterpret_cast<int4*>(ws + p.units1);
  a.units2 = reinterpret_cast<int4*>(ws + p.units2);
  a.nunits = reinterpret_cast<int32_t*>(ws + p.nunits);
  a.nb = p.nb;
  a.E = p.E;
  a.T = p.T;
  a.Tp = p.Tp;
  a.rowpad = p.rowpad;
  a.nmax1 = p.nmax1;
  a.nmax2 = p.nmax2;
  a.nwb1 = p.nwb1;
  a.nwb1s = p.nwb1s;
  a.nwb2 = p.nwb2;
  a.S = p.S;
  a.shared_units1 = p.shared_units1;
  a.shared_units2 = p.shared_units2;
  a.plan_tag = plan_tag(p);
  if (launch_chained(permute_scan_kernel, dim3(1), dim3(kScanThreads), 0, st, a) != cudaSuccess) return MOE_ERR_CUDA;

  return launch_chained(permute_scatter_kernel, dim3(p.nb, (p.k + kScatterSlots - 1) / kScatterSlots),
                        dim3(kPermBlock), msmem, st, topk_idx, topk_w, p.T, p.E,
                        p.k, blkcnt, a.roff, a.perm, a.roww, reinterpret_cast<int32_t*>(ws + p.inv),
                        err) == cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}

}  // namespace moe
