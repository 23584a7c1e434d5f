// route.cu -- the router in front of the layer: top-k expert selection and the
// softmax of the chosen logits.
//
// The grouped GEMM article's introduction has the router hand each token to some
// experts; the pages define nothing further, so this follows the plainest
// reading (the one the layer's gate weights are drawn with): a token goes to the
// topk experts with the largest logits, largest first, ties to the lower expert
// index, and w[t, k] = softmax over those topk logits.
//
// One warp per token.  Lane l holds the logits of experts l, l + 32, ...; each of
// the topk rounds is a warp arg-max over the experts not yet chosen (value, then
// lower index), so the selection compares the given fp32 values exactly.  Lane k
// keeps the k-th chosen logit; the softmax is a warp max and sum in fp32.
#include <cfloat>

#include "common.cuh"

namespace moe {

namespace {
constexpr int RT_THREADS = 256;
constexpr int32_t RT_NONE = 0x7fffffff;

// (v, e) beats (bv, be): a larger value, or an equal value at a lower index; any
// candidate beats "none".
__device__ __forceinline__ bool beats(float v, int32_t e, float bv, int32_t be) {
  if (e == RT_NONE) return false;
  if (be == RT_NONE) return true;
  return v > bv || (v == bv && e < be);
}
}  // namespace

// Routes token t with the calling warp: lane k < topk ends up with the k-th chosen
// expert (*id) and its gate weight (*wt).  Lane l holds the logits of experts
// l, l + 32, ...; each of the topk rounds is a warp arg-max over the experts not
// yet chosen (value, then lower index); the softmax is a warp max and sum in fp32.
template <int PER_LANE>
__device__ __forceinline__ void route_token(const float* __restrict__ logits, int32_t t, int32_t E,
                                            int32_t topk, int lane, int32_t* id, float* wt) {
  const float* row = logits + static_cast<int64_t>(t) * E;
  float v[PER_LANE];
#pragma unroll
  for (int j = 0; j < PER_LANE; ++j) {
    const int32_t e = lane + 32 * j;
    v[j] = e < E ? __ldg(row + e) : -FLT_MAX;
  }
  uint32_t taken = 0;  // bit j: expert lane + 32 j already chosen
  float mine = 0.0f;   // lane k keeps the k-th chosen logit
  int32_t my_id = 0;
  for (int32_t k = 0; k < topk; ++k) {
    float bv = -FLT_MAX;
    int32_t be = RT_NONE;
#pragma unroll
    for (int j = 0; j < PER_LANE; ++j) {
      const int32_t e = lane + 32 * j;
      if (e < E && !(taken & (1u << j)) && beats(v[j], e, bv, be)) {
        bv = v[j];
        be = e;
      }
    }
#pragma unroll
    for (int d = 16; d >= 1; d >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, d);
      const int32_t oe = __shfl_xor_sync(0xffffffffu, be, d);
      if (beats(ov, oe, bv, be)) {
        bv = ov;
        be = oe;
      }
    }
    if (be != RT_NONE && (be & 31) == lane) taken |= 1u << (be >> 5);
    if (lane == k) {
      mine = bv;
      my_id = be;
    }
  }
  // softmax over the chosen logits (lane 0 holds the largest)
  const float mx = __shfl_sync(0xffffffffu, mine, 0);
  const float ex = lane < topk ? expf(mine - mx) : 0.0f;
  float sum = ex;
#pragma unroll
  for (int d = 16; d >= 1; d >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, d);
  *id = my_id;
  *wt = ex / sum;
}

template <int PER_LANE>
__global__ void __launch_bounds__(RT_THREADS)
    route_kernel(const float* __restrict__ logits, int32_t M, int32_t E, int32_t topk,
                 int32_t* __restrict__ ids, float* __restrict__ w) {
  griddep_launch_dependents();
  griddep_wait();
  const int lane = threadIdx.x & 31;
  const int32_t nwarps = static_cast<int32_t>((gridDim.x * RT_THREADS) >> 5);
  for (int32_t t = static_cast<int32_t>((blockIdx.x * RT_THREADS + threadIdx.x) >> 5); t < M;
       t += nwarps) {
    int32_t id;
    float wt;
    route_token<PER_LANE>(logits, t, E, topk, lane, &id, &wt);
    if (lane < topk) {
      ids[static_cast<int64_t>(t) * topk + lane] = id;
      w[static_cast<int64_t>(t) * topk + lane] = wt;
    }
  }
}

// The router fused with the first pass of the plan: one warp per token (as
// route_kernel) writes the token's ids and gate weights and counts each of its
// routed rows i = t*topk + k into the histogram row of the plan chunk that holds i
// (i / chunk_rows), with global atomics on the zeroed chunk histograms.  The
// histograms then feed the plan's scan-and-scatter kernel exactly as the plan's
// own histogram pass would.
template <int PER_LANE>
__global__ void __launch_bounds__(RT_THREADS)
    route_hist_kernel(const float* __restrict__ logits, int32_t M, int32_t E, int32_t topk,
                      int32_t chunk_rows, int32_t* __restrict__ ids, float* __restrict__ w,
                      int32_t* __restrict__ hist) {
  griddep_launch_dependents();
  griddep_wait();
  const int lane = threadIdx.x & 31;
  const int32_t nwarps = static_cast<int32_t>((gridDim.x * RT_THREADS) >> 5);
  for (int32_t t = static_cast<int32_t>((blockIdx.x * RT_THREADS + threadIdx.x) >> 5); t < M;
       t += nwarps) {
    int32_t id;
    float wt;
    route_token<PER_LANE>(logits, t, E, topk, lane, &id, &wt);
    if (lane < topk) {
      const int64_t i = static_cast<int64_t>(t) * topk + lane;
      ids[i] = id;
      w[i] = wt;
      atomicAdd(hist + (i / chunk_rows) * (E + 1) + id, 1);
    }
  }
}

cudaError_t launch_route(const float* logits, int64_t M, int32_t E, int32_t topk, int32_t* ids,
                         float* w, int num_sms, cudaStream_t stream) {
  if (M == 0) return cudaSuccess;
  const int64_t want = (M + (RT_THREADS / 32) - 1) / (RT_THREADS / 32);
  const int64_t cap = static_cast<int64_t>(num_sms) * 8;
  const dim3 grid(static_cast<unsigned>(want < cap ? want : cap));
  const int32_t m = static_cast<int32_t>(M);
  const int per_lane = (E + 31) / 32;
  if (per_lane <= 1) return launch_pdl(route_kernel<1>, grid, dim3(RT_THREADS), 0, stream, 1, logits, m, E, topk, ids, w);
  if (per_lane <= 2) return launch_pdl(route_kernel<2>, grid, dim3(RT_THREADS), 0, stream, 1, logits, m, E, topk, ids, w);
  if (per_lane <= 4) return launch_pdl(route_kernel<4>, grid, dim3(RT_THREADS), 0, stream, 1, logits, m, E, topk, ids, w);
  if (per_lane <= 8) return launch_pdl(route_kernel<8>, grid, dim3(RT_THREADS), 0, stream, 1, logits, m, E, topk, ids, w);
  if (per_lane <= 16) return launch_pdl(route_kernel<16>, grid, dim3(RT_THREADS), 0, stream, 1, logits, m, E, topk, ids, w);
  return launch_pdl(route_kernel<32>, grid, dim3(RT_THREADS), 0, stream, 1, logits, m, E, topk, ids, w);
}

}  // namespace moe

namespace moe {

cudaError_t launch_plan_chunks(const int32_t* ids, const float* w, int32_t R, int32_t E, int32_t seg,
                               const int32_t* hist, int32_t nchunks, int32_t* counts,
                               int32_t* offsets, int32_t* perm, int32_t* inv, float* w_sorted,
                               int32_t* status, cudaStream_t stream);
int32_t plan_warp_rows(int32_t R, int num_sms);

// Router + plan: the chunk histograms zeroed, route_hist_kernel, then the plan's
// scan-and-scatter kernel on the chunk histograms.  `scratch` holds the per-chunk
// histograms (256 x (E + 1) int32).
cudaError_t launch_route_plan(const float* logits, int64_t M, int32_t E, int32_t topk, int32_t* ids,
                              float* w, int32_t* counts, int32_t* offsets, int32_t* perm,
                              int32_t* inv, float* w_sorted, int32_t* status, int32_t* scratch,
                              int num_sms, cudaStream_t stream) {
  const int32_t R = static_cast<int32_t>(M * topk);
  if (M == 0)
    return launch_plan_chunks(ids, w, 0, E, 32, nullptr, 0, counts, offsets, perm, inv, w_sorted,
                              status, stream);
  const int32_t seg = plan_warp_rows(R, num_sms);   // rows per plan warp
  const int32_t chunk_rows = 16 * seg;
  const int32_t nchunks = (R + chunk_rows - 1) / chunk_rows;
  cudaError_t err = cudaMemsetAsync(scratch, 0, sizeof(int32_t) * static_cast<size_t>(nchunks) *
                                                    static_cast<size_t>(E + 1), stream);
  if (err != cudaSuccess) return err;
  const int64_t want = (M + (RT_THREADS / 32) - 1) / (RT_THREADS / 32);
  const int64_t cap = static_cast<int64_t>(num_sms) * 8;
  const dim3 grid(static_cast<unsigned>(want < cap ? want : cap)), block(RT_THREADS);
  const int32_t m = static_cast<int32_t>(M);
  const int per_lane = (E + 31) / 32;
  if (per_lane <= 1) err = launch_pdl(route_hist_kernel<1>, grid, block, 0, stream, 1, logits, m, E, topk, chunk_rows, ids, w, scratch);
  else if (per_lane <= 2) err = launch_pdl(route_hist_kernel<2>, grid, block, 0, stream, 1, logits, m, E, topk, chunk_rows, ids, w, scratch);
  else if (per_lane <= 4) err = launch_pdl(route_hist_kernel<4>, grid, block, 0, stream, 1, logits, m, E, topk, chunk_rows, ids, w, scratch);
  else if (per_lane <= 8) err = launch_pdl(route_hist_kernel<8>, grid, block, 0, stream, 1, logits, m, E, topk, chunk_rows, ids, w, scratch);
  else if (per_lane <= 16) err = launch_pdl(route_hist_kernel<16>, grid, block, 0, stream, 1, logits, m, E, topk, chunk_rows, ids, w, scratch);
  else err = launch_pdl(route_hist_kernel<32>, grid, block, 0, stream, 1, logits, m, E, topk, chunk_rows, ids, w, scratch);
  if (err != cudaSuccess) return err;
  return launch_plan_chunks(ids, w, R, E, seg, scratch, nchunks, counts, offsets, perm, inv, w_sorted,
                            status, stream);
}

}  // namespace moe
