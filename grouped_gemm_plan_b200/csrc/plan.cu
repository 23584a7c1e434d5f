// plan.cu -- routing plan: per-expert histogram, exclusive scan, stable scatter.
//
// The FrontReorder stage of the PTO MegaMoE article ("MegaMoE 融合算子七阶段")
// and the per-problem size arrays a grouped GEMM takes ("Grouped GEMM 为什么适合
// MoE", section "Grouped GEMM 到底解决什么问题"), computed as a counting sort:
//   counts[e]  = #{i : ids[i] = e}
//   offsets    = exclusive prefix sum of counts (E+1 entries)
//   perm[s]    = i for the slots s of expert e, in ascending i (stable)
//
// One launch.  The R routed rows are cut into chunks, one CTA per chunk.  Every
// CTA reads the whole id array (R int32, served from L2) to build the total
// histogram and the histogram of the rows before its chunk -- warp-aggregated
// with __match_any_sync so that a popular expert costs one shared atomic per
// warp, not one per lane.  A block scan turns the totals into offsets.  Then the
// CTA ranks its own rows: warp w owns a contiguous segment of the chunk, counts
// it per expert, the per-warp counts are scanned in warp order, and a second
// pass over the segment gives every row its slot = offsets[e] + rows of e before
// the chunk + rows of e in earlier warps + rows of e earlier in this warp.
// Stability holds by construction: slots grow with i.
#include "common.cuh"

namespace moe {

constexpr int PLAN_THREADS = 512;
constexpr int PLAN_WARPS = PLAN_THREADS / 32;
constexpr int PLAN_UNROLL = 4;

__global__ void __launch_bounds__(PLAN_THREADS)
    plan_kernel(const int32_t* __restrict__ ids, const float* __restrict__ w, int32_t R,
                int32_t E, int32_t seg, int32_t* __restrict__ counts,
                int32_t* __restrict__ offsets, int32_t* __restrict__ perm,
                int32_t* __restrict__ inv, float* __restrict__ w_sorted, int32_t* status) {
  extern __shared__ int32_t plan_smem[];
  int32_t* tot = plan_smem;           // [E] totals, later exclusive offsets
  int32_t* before = plan_smem + E;    // [E] rows of e before this chunk
  int32_t* wbase = plan_smem + 2 * E; // [PLAN_WARPS][E] per-warp counts, later bases
  __shared__ int32_t s_bad;
  __shared__ int32_t s_warp_sum[PLAN_WARPS];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int32_t chunk = PLAN_WARPS * seg;
  const int32_t c0 = blockIdx.x * chunk;
  const int32_t c1 = min(c0 + chunk, R);

  for (int e = tid; e < E; e += PLAN_THREADS) {
    tot[e] = 0;
    before[e] = 0;
  }
  for (int j = tid; j < PLAN_WARPS * E; j += PLAN_THREADS) wbase[j] = 0;
  if (tid == 0) s_bad = 0;
  __syncthreads();

  // ---- pass over all rows: totals and rows before this chunk
  for (int32_t base = 0; base < R; base += PLAN_THREADS * PLAN_UNROLL) {
    int32_t ev[PLAN_UNROLL];
#pragma unroll
    for (int u = 0; u < PLAN_UNROLL; ++u) {
      const int32_t i = base + u * PLAN_THREADS + tid;
      ev[u] = i < R ? __ldg(ids + i) : -1;
    }
#pragma unroll
    for (int u = 0; u < PLAN_UNROLL; ++u) {
      const int32_t i = base + u * PLAN_THREADS + tid;
      const int32_t e = ev[u];
      const bool valid = i < R;
      const bool good = valid && e >= 0 && e < E;
      if (valid && !good) s_bad = 1;
      const int32_t key = good ? (e * 2 + (i < c0 ? 1 : 0)) : -1;
      const unsigned peers = __match_any_sync(0xffffffffu, key);
      if (good && lane == __ffs(peers) - 1) {
        const int n = __popc(peers);
        atomicAdd(&tot[e], n);
        if (i < c0) atomicAdd(&before[e], n);
      }
    }
  }
  __syncthreads();

  if (s_bad) {
    // Defined failure: identity permutation, empty experts, status recorded.
    for (int32_t i = c0 + tid; i < c1; i += PLAN_THREADS) {
      perm[i] = i;
      if (inv != nullptr) inv[i] = i;
      if (w_sorted != nullptr) w_sorted[i] = w[i];
    }
    if (blockIdx.x == 0) {
      for (int e = tid; e < E; e += PLAN_THREADS) counts[e] = 0;
      for (int e = tid; e <= E; e += PLAN_THREADS) offsets[e] = 0;
      if (tid == 0) set_status(status, MOE_ERR_BAD_EXPERT_ID);
    }
    return;
  }

  // ---- exclusive scan of the totals (E <= 4 * PLAN_THREADS)
  {
    const int per = (E + PLAN_THREADS - 1) / PLAN_THREADS;
    int32_t loc[4];
    int32_t sum = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int e = tid * per + j;
      loc[j] = (j < per && e < E) ? tot[e] : 0;
      sum += loc[j];
    }
    int32_t incl = sum;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int32_t v = __shfl_up_sync(0xffffffffu, incl, d);
      if (lane >= d) incl += v;
    }
    if (lane == 31) s_warp_sum[warp] = incl;
    __syncthreads();
    int32_t run = incl - sum;
    for (int j = 0; j < warp; ++j) run += s_warp_sum[j];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int e = tid * per + j;
      if (j < per && e < E) {
        if (blockIdx.x == 0) {
          counts[e] = loc[j];
          offsets[e] = run;
        }
        tot[e] = run;
        run += loc[j];
      }
    }
    if (blockIdx.x == 0 && tid == 0) offsets[E] = R;
  }

  // ---- per-warp counts of this chunk
  const int32_t r0 = c0 + warp * seg;
  const int32_t r1 = min(r0 + seg, c1);
  int32_t* mybase = wbase + warp * E;
  for (int32_t b = r0; b < r1; b += 32) {
    const int32_t i = b + lane;
    const bool v = i < r1;
    const int32_t e = v ? __ldg(ids + i) : -1;
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    if (v && lane == __ffs(peers) - 1) mybase[e] += __popc(peers);
  }
  __syncthreads();  // also orders the scan's writes of tot[] before the reads below

  for (int e = tid; e < E; e += PLAN_THREADS) {
    int32_t run = tot[e] + before[e];
    for (int wi = 0; wi < PLAN_WARPS; ++wi) {
      const int32_t c = wbase[wi * E + e];
      wbase[wi * E + e] = run;
      run += c;
    }
  }
  __syncthreads();

  // ---- stable scatter of this warp's segment
  for (int32_t b = r0; b < r1; b += 32) {
    const int32_t i = b + lane;
    const bool v = i < r1;
    const int32_t e = v ? __ldg(ids + i) : -1;
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    if (v) {
      const int32_t slot = mybase[e] + __popc(peers & ((1u << lane) - 1u));
      perm[slot] = i;
      if (inv != nullptr) inv[i] = slot;
      if (w_sorted != nullptr) w_sorted[slot] = __ldg(w + i);
    }
    __syncwarp();
    if (v && lane == __ffs(peers) - 1) mybase[e] += __popc(peers);
    __syncwarp();
  }
}

// Host launcher (no validation here; the C ABI layer validates).
cudaError_t launch_plan(const int32_t* ids, const float* w, int32_t R, int32_t E, int32_t* counts,
                        int32_t* offsets, int32_t* perm, int32_t* inv, float* w_sorted,
                        int32_t* status, int num_sms, cudaStream_t stream) {
  const size_t smem = sizeof(int32_t) * (size_t)(2 + PLAN_WARPS) * (size_t)E;
  static int attr_done_mask = 0;  // one bit per device ordinal (< 31)
  int dev = 0;
  cudaError_t aerr = cudaGetDevice(&dev);
  if (aerr != cudaSuccess) return aerr;
  if (dev >= 31 || !(attr_done_mask & (1 << dev))) {
    aerr = cudaFuncSetAttribute(plan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)(sizeof(int32_t) * (2 + PLAN_WARPS) * MOE_MAX_EXPERTS));
    if (aerr != cudaSuccess) return aerr;
    if (dev < 31) attr_done_mask |= (1 << dev);
  }
  if (R == 0) {
    // Only counts/offsets to write: one CTA with no rows.
    plan_kernel<<<1, PLAN_THREADS, smem, stream>>>(ids, w, 0, E, 32, counts, offsets, perm, inv,
                                                   w_sorted, status);
    return cudaGetLastError();
  }
  int32_t per_cta = (R + num_sms - 1) / num_sms;
  int32_t seg = (per_cta + PLAN_WARPS - 1) / PLAN_WARPS;
  seg = ((seg + 31) / 32) * 32;
  if (seg < 32) seg = 32;
  const int32_t chunk = seg * PLAN_WARPS;
  const int32_t grid = (R + chunk - 1) / chunk;
  plan_kernel<<<grid, PLAN_THREADS, smem, stream>>>(ids, w, R, E, seg, counts, offsets, perm, inv,
                                                    w_sorted, status);
  return cudaGetLastError();
}

}  // namespace moe
