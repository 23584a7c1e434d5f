// plan.cu -- routing plan: per-expert histogram, exclusive scan, stable scatter.
//
// The FrontReorder stage of the PTO MegaMoE article ("MegaMoE 融合算子七阶段")
// and the per-problem size arrays a grouped GEMM takes ("Grouped GEMM 为什么适合
// MoE", section "Grouped GEMM 到底解决什么问题"), computed as a counting sort:
//   counts[e]  = #{i : ids[i] = e}
//   offsets    = exclusive prefix sum of counts (E+1 entries)
//   perm[s]    = i for the slots s of expert e, in ascending i (stable)
//
// Two launches when the rows span several chunks (one CTA per chunk), one when
// they fit a single chunk:
//   plan_hist_kernel   each CTA histograms its own chunk (warp-aggregated with
//                      __match_any_sync, so a popular expert costs one shared
//                      atomic per warp) and writes it, plus its count of invalid
//                      ids, to a per-chunk row of the workspace scratch;
//   plan_kernel        each CTA sums the chunk rows into the totals and the rows
//                      of each expert in earlier chunks, scans the totals into
//                      offsets, then ranks its own rows: warp w owns a contiguous
//                      segment of the chunk, counts it per expert, the per-warp
//                      counts are scanned in warp order, and a second pass gives
//                      every row its slot = offsets[e] + rows of e in earlier
//                      chunks + rows of e in earlier warps + rows of e earlier in
//                      this warp.  Stability holds by construction: slots grow
//                      with i.
#include "common.cuh"

namespace moe {

constexpr int PLAN_THREADS = 512;
constexpr int PLAN_WARPS = PLAN_THREADS / 32;
constexpr int PLAN_UNROLL = 4;
constexpr int PLAN_MAX_CHUNKS = 256;   // rows of the per-chunk histogram scratch

// Row c of `hist` (E + 1 ints): rows of each expert in chunk c, then the number
// of ids outside [0, E) in it.
__global__ void __launch_bounds__(PLAN_THREADS)
    plan_hist_kernel(const int32_t* __restrict__ ids, int32_t R, int32_t E, int32_t seg,
                     int32_t* __restrict__ hist) {
  extern __shared__ int32_t hist_smem[];  // [E]
  __shared__ int32_t s_bad;
  const int tid = threadIdx.x, lane = tid & 31;
  const int32_t chunk = PLAN_WARPS * seg;
  const int32_t c0 = blockIdx.x * chunk;
  const int32_t c1 = min(c0 + chunk, R);
  griddep_launch_dependents();
  for (int e = tid; e < E; e += PLAN_THREADS) hist_smem[e] = 0;
  if (tid == 0) s_bad = 0;
  griddep_wait();
  __syncthreads();
  for (int32_t base = c0; base < c1; base += PLAN_THREADS) {
    const int32_t i = base + tid;
    const int32_t e = i < c1 ? __ldg(ids + i) : -1;
    const bool good = i < c1 && e >= 0 && e < E;
    if (i < c1 && !good) atomicAdd(&s_bad, 1);
    const unsigned peers = __match_any_sync(0xffffffffu, good ? e : -1);
    if (good && lane == __ffs(peers) - 1) atomicAdd(&hist_smem[e], __popc(peers));
  }
  __syncthreads();
  int32_t* row = hist + static_cast<int64_t>(blockIdx.x) * (E + 1);
  for (int e = tid; e < E; e += PLAN_THREADS) row[e] = hist_smem[e];
  if (tid == 0) row[E] = s_bad;
}

__global__ void __launch_bounds__(PLAN_THREADS)
    plan_kernel(const int32_t* __restrict__ ids, const float* __restrict__ w, int32_t R,
                int32_t E, int32_t seg, const int32_t* __restrict__ hist, int32_t nchunks,
                int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                int32_t* __restrict__ perm, int32_t* __restrict__ inv,
                float* __restrict__ w_sorted, int32_t* status) {
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

  griddep_launch_dependents();
  for (int e = tid; e < E; e += PLAN_THREADS) {
    tot[e] = 0;
    before[e] = 0;
  }
  for (int j = tid; j < PLAN_WARPS * E; j += PLAN_THREADS) wbase[j] = 0;
  if (tid == 0) s_bad = 0;
  griddep_wait();
  __syncthreads();

  if (hist != nullptr) {
    // ---- totals and rows before this chunk, from the per-chunk histograms
    for (int32_t idx = tid; idx < nchunks * E; idx += PLAN_THREADS) {
      const int32_t c = idx / E, e = idx - c * E;
      const int32_t v = hist[static_cast<int64_t>(c) * (E + 1) + e];
      if (v != 0) {
        atomicAdd(&tot[e], v);
        if (c < static_cast<int32_t>(blockIdx.x)) atomicAdd(&before[e], v);
      }
    }
    for (int32_t c = tid; c < nchunks; c += PLAN_THREADS)
      if (hist[static_cast<int64_t>(c) * (E + 1) + E] != 0) s_bad = 1;
  } else {
    // ---- a single chunk: histogram of all rows here
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
        const unsigned peers = __match_any_sync(0xffffffffu, good ? e : -1);
        if (good && lane == __ffs(peers) - 1) atomicAdd(&tot[e], __popc(peers));
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

// Rows each warp of the plan kernel owns for R routed rows (a multiple of 32):
// the rows are cut into at most min(#SMs, 256) chunks of 16 warps.
int32_t plan_warp_rows(int32_t R, int num_sms) {
  const int max_chunks = num_sms < PLAN_MAX_CHUNKS ? num_sms : PLAN_MAX_CHUNKS;
  const int32_t per_cta = (R + max_chunks - 1) / max_chunks;
  int32_t seg = (per_cta + PLAN_WARPS - 1) / PLAN_WARPS;
  seg = ((seg + 31) / 32) * 32;
  return seg < 32 ? 32 : seg;
}

// The scan-and-scatter kernel over `nchunks` chunks of 16 * seg rows, from the
// per-chunk histograms `hist` (nullptr: one chunk that counts its own rows).
cudaError_t launch_plan_chunks(const int32_t* ids, const float* w, int32_t R, int32_t E, int32_t seg,
                               const int32_t* hist, int32_t nchunks, int32_t* counts,
                               int32_t* offsets, int32_t* perm, int32_t* inv, float* w_sorted,
                               int32_t* status, cudaStream_t stream) {
  static PerDeviceOnce once;
  const cudaError_t aerr = once.run([] {
    return cudaFuncSetAttribute(plan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)(sizeof(int32_t) * (2 + PLAN_WARPS) * MOE_MAX_EXPERTS));
  });
  if (aerr != cudaSuccess) return aerr;
  const size_t smem = sizeof(int32_t) * (size_t)(2 + PLAN_WARPS) * (size_t)E;
  const int32_t grid = hist == nullptr ? 1 : nchunks;
  return launch_pdl(plan_kernel, dim3(grid), dim3(PLAN_THREADS), smem, stream, 1, ids, w, R, E, seg,
                    hist, hist == nullptr ? 1 : nchunks, counts, offsets, perm, inv, w_sorted,
                    status);
}

// Host launcher (no validation here; the C ABI layer validates).  `scratch`
// holds the per-chunk histograms (256 x (E + 1) ints).
cudaError_t launch_plan(const int32_t* ids, const float* w, int32_t R, int32_t E, int32_t* counts,
                        int32_t* offsets, int32_t* perm, int32_t* inv, float* w_sorted,
                        int32_t* status, int32_t* scratch, int num_sms, cudaStream_t stream) {
  if (R == 0)  // only counts/offsets to write: one CTA with no rows
    return launch_plan_chunks(ids, w, 0, E, 32, nullptr, 0, counts, offsets, perm, inv, w_sorted,
                              status, stream);
  const int32_t seg = plan_warp_rows(R, num_sms);
  const int32_t chunk = seg * PLAN_WARPS;
  const int32_t grid = (R + chunk - 1) / chunk;
  if (grid == 1)
    return launch_plan_chunks(ids, w, R, E, seg, nullptr, 1, counts, offsets, perm, inv, w_sorted,
                              status, stream);
  cudaError_t err = launch_pdl(plan_hist_kernel, dim3(grid), dim3(PLAN_THREADS), sizeof(int32_t) * E,
                               stream, 1, ids, R, E, seg, scratch);
  if (err != cudaSuccess) return err;
  return launch_plan_chunks(ids, w, R, E, seg, scratch, grid, counts, offsets, perm, inv, w_sorted,
                            status, stream);
}

}  // namespace moe
