// permute.cu -- dispatch (gather into expert order) and combine (top-k reduction
// back to token order).  Both are HBM-bound copies of bf16 rows; neither has a
// contraction, so they stay off the tensor cores.
//
// Dispatch is the permute of the PTO MegaMoE article ("MegaMoE 融合算子七阶段":
// Dispatch) and COMET's layer-0 token dispatch (COMET review, section 3.2).
// Combine is the top-k weighted accumulation ("MoE dispatch/combine 为什么慢":
// topK 加权累加) plus Unpermute.
//
// Layout of the work: a work item is one 512-byte step of one output row, done by
// one warp; each lane moves a 16-byte vector (8 bf16), so every access is a full,
// coalesced 128-byte line, and even a batch of a few rows spreads over all SMs.
// Grids are a multiple of the SM count with 8 warps per CTA; items are walked
// grid-stride.  Combine reads the top-k source vectors of a step before it
// accumulates, so up to topk loads per lane are in flight; the sum runs in fp32
// registers in ascending k, one bf16 cast at the end.
#include "common.cuh"

namespace moe {

constexpr int PM_THREADS = 256;

// Work item = (row s, step group q): lane l of the warp copies 16-byte vectors
// (q*DU + u)*32 + l of the row, u < DU, all DU loads issued before the stores.
// Splitting rows into 2 KB groups keeps every SM busy even when there are only a
// few rows (small batches) and keeps DU loads in flight per lane.
constexpr int DU = 4;

__global__ void __launch_bounds__(PM_THREADS)
    dispatch_kernel(const uint4* __restrict__ x, const int32_t* __restrict__ perm, int32_t R,
                    int32_t topk, int32_t vpr, uint4* __restrict__ xp, int32_t* status) {
  griddep_launch_dependents();
  griddep_wait();
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * PM_THREADS) >> 5;
  const int32_t groups = (vpr + 32 * DU - 1) / (32 * DU);
  const int64_t items = static_cast<int64_t>(R) * groups;
  for (int64_t it = (static_cast<int64_t>(blockIdx.x) * PM_THREADS + threadIdx.x) >> 5; it < items;
       it += nwarps) {
    const int32_t s = static_cast<int32_t>(it / groups);
    const int32_t c0 = static_cast<int32_t>(it - static_cast<int64_t>(s) * groups) * (32 * DU) + lane;
    const int32_t i = __ldg(perm + s);
    uint4* dst = xp + static_cast<int64_t>(s) * vpr;
    if (i < 0 || i >= R) {
      if (lane == 0) set_status(status, MOE_ERR_BAD_INDEX);
#pragma unroll
      for (int u = 0; u < DU; ++u)
        if (c0 + 32 * u < vpr) dst[c0 + 32 * u] = make_uint4(0, 0, 0, 0);
      continue;
    }
    const uint4* src = x + static_cast<int64_t>(i / topk) * vpr;
    uint4 v[DU];
#pragma unroll
    for (int u = 0; u < DU; ++u)
      if (c0 + 32 * u < vpr) v[u] = __ldg(src + c0 + 32 * u);
#pragma unroll
    for (int u = 0; u < DU; ++u)
      if (c0 + 32 * u < vpr) dst[c0 + 32 * u] = v[u];
  }
}

// The same copy walked in token order: work item = (token t, step group q); the
// warp loads its vectors of x[t] once and stores them to all topk slots
// inv[t*topk + k] of the token.  Every x row is read exactly once (in slot order
// the topk reads of a row come at different times and a large x is partly read
// from DRAM again); the written bytes are the same.
__global__ void __launch_bounds__(PM_THREADS)
    dispatch_tokens_kernel(const uint4* __restrict__ x, const int32_t* __restrict__ inv, int32_t M,
                           int32_t topk, int32_t vpr, uint4* __restrict__ xp, int32_t* status) {
  griddep_launch_dependents();
  griddep_wait();
  const int lane = threadIdx.x & 31;
  const int32_t R = M * topk;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * PM_THREADS) >> 5;
  const int32_t groups = (vpr + 32 * DU - 1) / (32 * DU);
  const int64_t items = static_cast<int64_t>(M) * groups;
  for (int64_t it = (static_cast<int64_t>(blockIdx.x) * PM_THREADS + threadIdx.x) >> 5; it < items;
       it += nwarps) {
    const int32_t t = static_cast<int32_t>(it / groups);
    const int32_t c0 = static_cast<int32_t>(it - static_cast<int64_t>(t) * groups) * (32 * DU) + lane;
    const uint4* src = x + static_cast<int64_t>(t) * vpr;
    uint4 v[DU];
#pragma unroll
    for (int u = 0; u < DU; ++u)
      if (c0 + 32 * u < vpr) v[u] = __ldg(src + c0 + 32 * u);
    for (int32_t k = 0; k < topk; ++k) {
      const int32_t s = __ldg(inv + static_cast<int64_t>(t) * topk + k);
      if (s < 0 || s >= R) {
        if (lane == 0) set_status(status, MOE_ERR_BAD_INDEX);
        continue;
      }
      uint4* dst = xp + static_cast<int64_t>(s) * vpr;
#pragma unroll
      for (int u = 0; u < DU; ++u)
        if (c0 + 32 * u < vpr) dst[c0 + 32 * u] = v[u];
    }
  }
}

__device__ __forceinline__ void acc_bf16x8(float (&acc)[8], const uint4 v, float wk) {
  const float2 p0 = unpack_bf16x2(v.x), p1 = unpack_bf16x2(v.y), p2 = unpack_bf16x2(v.z),
               p3 = unpack_bf16x2(v.w);
  acc[0] = fmaf(wk, p0.x, acc[0]);
  acc[1] = fmaf(wk, p0.y, acc[1]);
  acc[2] = fmaf(wk, p1.x, acc[2]);
  acc[3] = fmaf(wk, p1.y, acc[3]);
  acc[4] = fmaf(wk, p2.x, acc[4]);
  acc[5] = fmaf(wk, p2.y, acc[5]);
  acc[6] = fmaf(wk, p3.x, acc[6]);
  acc[7] = fmaf(wk, p3.y, acc[7]);
}

// Eight consecutive elements of a row, widened to fp32: one 16-byte load of bf16,
// or two 16-byte loads of fp32.
template <bool F32>
struct Vec8;
template <>
struct Vec8<false> {
  uint4 u;
  __device__ __forceinline__ void load(const void* row, int32_t c) {
    u = __ldg(reinterpret_cast<const uint4*>(row) + c);
  }
  __device__ __forceinline__ void zero() { u = make_uint4(0, 0, 0, 0); }
  __device__ __forceinline__ void fma_into(float (&acc)[8], float wk) const { acc_bf16x8(acc, u, wk); }
};
template <>
struct Vec8<true> {
  float4 a, b;
  __device__ __forceinline__ void load(const void* row, int32_t c) {
    const float4* p = reinterpret_cast<const float4*>(row) + 2 * c;
    a = __ldg(p);
    b = __ldg(p + 1);
  }
  __device__ __forceinline__ void zero() { a = b = make_float4(0.f, 0.f, 0.f, 0.f); }
  __device__ __forceinline__ void fma_into(float (&acc)[8], float wk) const {
    acc[0] = fmaf(wk, a.x, acc[0]);
    acc[1] = fmaf(wk, a.y, acc[1]);
    acc[2] = fmaf(wk, a.z, acc[2]);
    acc[3] = fmaf(wk, a.w, acc[3]);
    acc[4] = fmaf(wk, b.x, acc[4]);
    acc[5] = fmaf(wk, b.y, acc[5]);
    acc[6] = fmaf(wk, b.z, acc[6]);
    acc[7] = fmaf(wk, b.w, acc[7]);
  }
};

// Optional epilogue of the combine (the grouped GEMM article's "Fused GemmAdd":
// the accumulated fp32 result and an fp32 add are combined before the one cast):
// out[t] = bf16(alpha * acc + beta * add[t]); add is read only when beta != 0.
struct CombineAdd {
  const uint4* add;  // bf16 [M, H] (may be the layer's x, or out itself)
  float alpha, beta;
};

// out[t] = bf16(sum_k w[t,k] * y[row(t,k)]), row(t,k) = inv ? inv[t*topk+k] : t*topk+k,
// or with an added tensor bf16(alpha * sum + beta * add[t]).
// y is bf16 or fp32 [R, H]; vpr = H / 8 groups of eight elements per row.  Each
// output vector is written by the lane that read its add vector, so add may
// alias out.
template <int KMAX, bool F32, bool ADD>
__global__ void __launch_bounds__(PM_THREADS)
    combine_kernel(const uint8_t* __restrict__ y, const int32_t* __restrict__ inv,
                   const float* __restrict__ w, int32_t M, int32_t R, int32_t topk,
                   int32_t vpr, uint4* out, int32_t* status, CombineAdd ga) {
  griddep_launch_dependents();
  griddep_wait();
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * PM_THREADS) >> 5;
  const int64_t row_bytes = static_cast<int64_t>(vpr) * (F32 ? 32 : 16);
  constexpr int CU = KMAX <= 8 ? 2 : 1;  // steps per work item: CU * topk loads in flight
  const int32_t groups = (vpr + 32 * CU - 1) / (32 * CU);
  const int64_t items = static_cast<int64_t>(M) * groups;
  // Work item = (token t, step group q): lane l handles groups of eight elements
  // (q*CU + u)*32 + l, u < CU.
  for (int64_t it = (static_cast<int64_t>(blockIdx.x) * PM_THREADS + threadIdx.x) >> 5; it < items;
       it += nwarps) {
    const int32_t t = static_cast<int32_t>(it / groups);
    const int32_t cbase = static_cast<int32_t>(it - static_cast<int64_t>(t) * groups) * (32 * CU) + lane;
    int32_t my_row = 0;
    float my_w = 1.0f;
    if (lane < topk) {
      const int32_t i = t * topk + lane;
      my_row = inv != nullptr ? __ldg(inv + i) : i;
      if (w != nullptr) my_w = __ldg(w + i);
      if (my_row < 0 || my_row >= R) {
        set_status(status, MOE_ERR_BAD_INDEX);
        my_row = -1;
      }
    }
    int32_t rows[KMAX];
    float wk[KMAX];
#pragma unroll
    for (int k = 0; k < KMAX; ++k) {
      rows[k] = __shfl_sync(0xffffffffu, my_row, k);
      wk[k] = __shfl_sync(0xffffffffu, my_w, k);
    }
    constexpr int KC = KMAX < 8 ? KMAX : 8;  // top-k rows loaded per batch
    float acc[CU][8];
#pragma unroll
    for (int u = 0; u < CU; ++u)
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[u][e] = 0.f;
#pragma unroll
    for (int k0 = 0; k0 < KMAX; k0 += KC) {
      Vec8<F32> v[CU][KC];
#pragma unroll
      for (int u = 0; u < CU; ++u) {
        const int32_t c = cbase + 32 * u;
#pragma unroll
        for (int kk = 0; kk < KC; ++kk) {
          const int k = k0 + kk;
          if (c < vpr && k < topk && rows[k] >= 0)
            v[u][kk].load(y + static_cast<int64_t>(rows[k]) * row_bytes, c);
          else
            v[u][kk].zero();
        }
      }
#pragma unroll
      for (int u = 0; u < CU; ++u)
#pragma unroll
        for (int kk = 0; kk < KC; ++kk)
          if (k0 + kk < topk) v[u][kk].fma_into(acc[u], wk[k0 + kk]);
    }
#pragma unroll
    for (int u = 0; u < CU; ++u) {
      const int32_t c = cbase + 32 * u;
      if (c >= vpr) continue;
      if (ADD) {
        if (ga.beta != 0.0f) {
          const uint4 a = ga.add[static_cast<int64_t>(t) * vpr + c];
          const float2 a0 = unpack_bf16x2(a.x), a1 = unpack_bf16x2(a.y), a2 = unpack_bf16x2(a.z),
                       a3 = unpack_bf16x2(a.w);
          const float av[8] = {a0.x, a0.y, a1.x, a1.y, a2.x, a2.y, a3.x, a3.y};
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[u][e] = fmaf(ga.beta, av[e], ga.alpha * acc[u][e]);
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[u][e] *= ga.alpha;
        }
      }
      uint4 o;
      o.x = pack_bf16x2(acc[u][0], acc[u][1]);
      o.y = pack_bf16x2(acc[u][2], acc[u][3]);
      o.z = pack_bf16x2(acc[u][4], acc[u][5]);
      o.w = pack_bf16x2(acc[u][6], acc[u][7]);
      out[static_cast<int64_t>(t) * vpr + c] = o;
    }
  }
}

// Grid for `items` warp-sized work items: up to 8 CTAs of 8 warps per SM.
static int grid_for_items(int64_t items, int num_sms) {
  const int64_t per_cta = PM_THREADS / 32;
  const int64_t want = (items + per_cta - 1) / per_cta;
  const int64_t cap = static_cast<int64_t>(num_sms) * 8;
  return static_cast<int>(want < cap ? (want > 0 ? want : 1) : cap);
}

cudaError_t launch_dispatch(const void* x, const int32_t* perm, int64_t M, int64_t H, int32_t topk,
                            void* xp, int32_t* status, int num_sms, cudaStream_t stream) {
  const int64_t R = M * topk;
  if (R == 0) return cudaSuccess;
  const int64_t groups = (H / 8 + 32 * DU - 1) / (32 * DU);
  return launch_pdl(dispatch_kernel, dim3(grid_for_items(R * groups, num_sms)), dim3(PM_THREADS), 0,
                    stream, 1, reinterpret_cast<const uint4*>(x), perm, static_cast<int32_t>(R), topk,
                    static_cast<int32_t>(H / 8), reinterpret_cast<uint4*>(xp), status);
}

cudaError_t launch_dispatch_tokens(const void* x, const int32_t* inv, int64_t M, int64_t H,
                                   int32_t topk, void* xp, int32_t* status, int num_sms,
                                   cudaStream_t stream) {
  if (M == 0) return cudaSuccess;
  const int64_t groups = (H / 8 + 32 * DU - 1) / (32 * DU);
  return launch_pdl(dispatch_tokens_kernel, dim3(grid_for_items(M * groups, num_sms)),
                    dim3(PM_THREADS), 0, stream, 1, reinterpret_cast<const uint4*>(x), inv,
                    static_cast<int32_t>(M), topk, static_cast<int32_t>(H / 8),
                    reinterpret_cast<uint4*>(xp), status);
}

template <bool F32, bool ADD>
static cudaError_t launch_combine_t(int grid, cudaStream_t stream, const uint8_t* y, const int32_t* inv,
                                    const float* w, int32_t m, int32_t R, int32_t topk, int32_t vpr,
                                    uint4* ov, int32_t* status, CombineAdd ga) {
  const dim3 g(grid), b(PM_THREADS);
  if (topk <= 2)
    return launch_pdl(combine_kernel<2, F32, ADD>, g, b, 0, stream, 1, y, inv, w, m, R, topk, vpr, ov, status, ga);
  if (topk <= 4)
    return launch_pdl(combine_kernel<4, F32, ADD>, g, b, 0, stream, 1, y, inv, w, m, R, topk, vpr, ov, status, ga);
  if (topk <= 8)
    return launch_pdl(combine_kernel<8, F32, ADD>, g, b, 0, stream, 1, y, inv, w, m, R, topk, vpr, ov, status, ga);
  if (topk <= 16)
    return launch_pdl(combine_kernel<16, F32, ADD>, g, b, 0, stream, 1, y, inv, w, m, R, topk, vpr, ov, status, ga);
  return launch_pdl(combine_kernel<32, F32, ADD>, g, b, 0, stream, 1, y, inv, w, m, R, topk, vpr, ov, status, ga);
}

// alpha == 1 and beta == 0: the plain combine (add unused, may be nullptr).
cudaError_t launch_combine_add(const void* y, bool y_f32, const int32_t* inv, const float* w,
                               const void* add, float alpha, float beta, int64_t M, int64_t H,
                               int32_t topk, void* out, int32_t* status, int num_sms,
                               cudaStream_t stream) {
  if (M == 0) return cudaSuccess;
  const int grid = grid_for_items(M * ((H / 8 + 31) / 32), num_sms);
  const int32_t R = static_cast<int32_t>(M * topk);
  const int32_t vpr = static_cast<int32_t>(H / 8);
  const uint8_t* yb = reinterpret_cast<const uint8_t*>(y);
  uint4* ov = reinterpret_cast<uint4*>(out);
  const int32_t m = static_cast<int32_t>(M);
  const CombineAdd ga{reinterpret_cast<const uint4*>(add), alpha, beta};
  if (alpha != 1.0f || beta != 0.0f)
    return y_f32 ? launch_combine_t<true, true>(grid, stream, yb, inv, w, m, R, topk, vpr, ov, status, ga)
                 : launch_combine_t<false, true>(grid, stream, yb, inv, w, m, R, topk, vpr, ov, status, ga);
  return y_f32 ? launch_combine_t<true, false>(grid, stream, yb, inv, w, m, R, topk, vpr, ov, status, ga)
               : launch_combine_t<false, false>(grid, stream, yb, inv, w, m, R, topk, vpr, ov, status, ga);
}

cudaError_t launch_combine(const void* y, bool y_f32, const int32_t* inv, const float* w,
                           int64_t M, int64_t H, int32_t topk, void* out, int32_t* status,
                           int num_sms, cudaStream_t stream) {
  return launch_combine_add(y, y_f32, inv, w, nullptr, 1.0f, 0.0f, M, H, topk, out, status, num_sms,
                            stream);
}

}  // namespace moe
