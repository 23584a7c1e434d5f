// fp8.cu -- the down projection in FP8 (E4M3): quantisers and an FP8 grouped GEMM.
//
// The PTO MegaMoE article (section "MegaMoE 融合算子七阶段") has SwiGLU consume each
// GMM1 segment and quantise it at once, so that GMM2 runs on quantised
// activations.  Here, on sm_100a:
//   * weights:     W2 [E, F, H] bf16 -> W2q [E, H, F] E4M3 (K = F contiguous, the
//                  tcgen05 K-major layout) with one fp32 scale per (expert, output
//                  column): scale = max_k |W2[e, k, n]| / 448.  Done once, offline.
//   * activations: h [R, F] bf16 (the SwiGLU epilogue's output) -> hq [R, F] E4M3
//                  with one fp32 scale per row: scale = max_j |h[s, j]| / 448, the
//                  largest element of every row landing on +-448.
//   * GEMM2:       tcgen05.mma kind::f8f6f4 (E4M3 x E4M3, fp32 accumulate in TMEM);
//                  the epilogue multiplies by row scale x column scale x gate weight
//                  and scatters fp32 rows to token order, as the bf16 GEMM2 does.
// Quantised value: q = nearest E4M3 to (v / scale) in fp32, ties to even,
// saturating at 448 (the hardware conversion cvt.rn.satfinite via cuda_fp8.h).
#include <cuda_fp8.h>

#include <cstdlib>

#include "common.cuh"
#include "epilogue.cuh"
#include "pair.cuh"

namespace moe {

namespace {

constexpr float kE4M3Max = 448.0f;

__device__ __forceinline__ uint8_t to_e4m3(float v) {
  return static_cast<uint8_t>(__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3));
}

__device__ __forceinline__ float scale_of(float amax) {
  return amax > 0.0f ? __fdiv_rn(amax, kE4M3Max) : 1.0f;
}

// Eight bf16 (one uint4) divided by `sc` and encoded -> eight bytes.
__device__ __forceinline__ uint2 quant8(uint4 v, float sc) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t o[2] = {0u, 0u};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float lo = __uint_as_float(w[i] << 16), hi = __uint_as_float(w[i] & 0xffff0000u);
    const uint32_t b = static_cast<uint32_t>(to_e4m3(__fdiv_rn(lo, sc))) |
                       (static_cast<uint32_t>(to_e4m3(__fdiv_rn(hi, sc))) << 8);
    o[i >> 1] |= b << (16 * (i & 1));
  }
  return make_uint2(o[0], o[1]);
}

__device__ __forceinline__ float amax8(uint4 v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  float m = 0.0f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    m = fmaxf(m, fabsf(__uint_as_float(w[i] << 16)));
    m = fmaxf(m, fabsf(__uint_as_float(w[i] & 0xffff0000u)));
  }
  return m;
}

constexpr int QR_THREADS = 256;

}  // namespace

// ---------------------------------------------------------------- row quantiser
// One CTA per row (grid-stride): the row's 16-byte vectors stay in registers
// (VPT per thread) between the max and the encoding, so h is read once.
template <int VPT>
__global__ void __launch_bounds__(QR_THREADS)
    quantize_rows_kernel(const uint4* __restrict__ A, int32_t R, int32_t K, uint2* __restrict__ q,
                         float* __restrict__ scale) {
  griddep_wait();
  __shared__ float s_red[QR_THREADS / 32];
  const int32_t vpr = K / 8;
  for (int32_t r = blockIdx.x; r < R; r += gridDim.x) {
    const uint4* row = A + static_cast<int64_t>(r) * vpr;
    uint4 v[VPT];
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const int32_t c = threadIdx.x + i * QR_THREADS;
      v[i] = c < vpr ? __ldg(row + c) : make_uint4(0, 0, 0, 0);
      m = fmaxf(m, amax8(v[i]));
    }
#pragma unroll
    for (int d = 16; d >= 1; d >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, d));
    if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = m;
    __syncthreads();
    m = s_red[0];
#pragma unroll
    for (int w = 1; w < QR_THREADS / 32; ++w) m = fmaxf(m, s_red[w]);
    const float sc = scale_of(m);
    if (threadIdx.x == 0) scale[r] = sc;
    uint2* qrow = q + static_cast<int64_t>(r) * vpr;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const int32_t c = threadIdx.x + i * QR_THREADS;
      if (c < vpr) qrow[c] = quant8(v[i], sc);
    }
    __syncthreads();  // s_red is reused by the next row
  }
  griddep_launch_dependents();
}

cudaError_t launch_quantize_rows(const void* A, int64_t R, int64_t K, void* q, float* scale,
                                 int num_sms, cudaStream_t stream) {
  if (R == 0) return cudaSuccess;
  const int64_t vpr = K / 8;
  const int64_t want = R;
  const int64_t cap = static_cast<int64_t>(num_sms) * 8;
  const dim3 grid(static_cast<unsigned>(want < cap ? want : cap));
  const int32_t r = static_cast<int32_t>(R), k = static_cast<int32_t>(K);
  const uint4* a = static_cast<const uint4*>(A);
  uint2* qq = static_cast<uint2*>(q);
  if (vpr <= QR_THREADS) return launch_pdl(quantize_rows_kernel<1>, grid, dim3(QR_THREADS), 0, stream, 1, a, r, k, qq, scale);
  if (vpr <= 2 * QR_THREADS) return launch_pdl(quantize_rows_kernel<2>, grid, dim3(QR_THREADS), 0, stream, 1, a, r, k, qq, scale);
  if (vpr <= 4 * QR_THREADS) return launch_pdl(quantize_rows_kernel<4>, grid, dim3(QR_THREADS), 0, stream, 1, a, r, k, qq, scale);
  if (vpr <= 8 * QR_THREADS) return launch_pdl(quantize_rows_kernel<8>, grid, dim3(QR_THREADS), 0, stream, 1, a, r, k, qq, scale);
  return launch_pdl(quantize_rows_kernel<16>, grid, dim3(QR_THREADS), 0, stream, 1, a, r, k, qq, scale);
}

// ---------------------------------------------------------------- weight quantiser
// Pass 1: per (expert, column) maximum over K (thread per column, rows walked in
// order, coalesced across the warp).
__global__ void __launch_bounds__(256)
    col_amax_kernel(const __nv_bfloat16* __restrict__ W, int32_t K, int32_t N,
                    float* __restrict__ scale) {
  const int32_t e = blockIdx.y;
  const int32_t n = blockIdx.x * 256 + threadIdx.x;
  if (n >= N) return;
  const __nv_bfloat16* col = W + static_cast<int64_t>(e) * K * N + n;
  float m = 0.0f;
  for (int32_t k = 0; k < K; ++k) m = fmaxf(m, fabsf(__bfloat162float(col[static_cast<int64_t>(k) * N])));
  scale[static_cast<int64_t>(e) * N + n] = scale_of(m);
}

// Pass 2: 64 x 64 tiles, transposed through shared memory: read along N, write
// along K.
__global__ void __launch_bounds__(256)
    quantize_cols_kernel(const __nv_bfloat16* __restrict__ W, int32_t K, int32_t N,
                         const float* __restrict__ scale, uint8_t* __restrict__ qT) {
  __shared__ float tile[64][65];
  const int32_t e = blockIdx.z;
  const int32_t k0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
  const __nv_bfloat16* We = W + static_cast<int64_t>(e) * K * N;
  for (int i = threadIdx.x; i < 64 * 64; i += 256) {
    const int32_t kk = i / 64, nn = i % 64;
    const int32_t k = k0 + kk, n = n0 + nn;
    tile[kk][nn] = (k < K && n < N) ? __bfloat162float(We[static_cast<int64_t>(k) * N + n]) : 0.0f;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < 64 * 64; i += 256) {
    const int32_t nn = i / 64, kk = i % 64;
    const int32_t k = k0 + kk, n = n0 + nn;
    if (k < K && n < N) {
      const float sc = __ldg(scale + static_cast<int64_t>(e) * N + n);
      qT[(static_cast<int64_t>(e) * N + n) * K + k] = to_e4m3(__fdiv_rn(tile[kk][nn], sc));
    }
  }
}

cudaError_t launch_quantize_cols(const void* W, int32_t E, int64_t K, int64_t N, void* qT,
                                 float* scale, cudaStream_t stream) {
  if (E == 0 || K == 0 || N == 0) return cudaSuccess;
  const __nv_bfloat16* w = static_cast<const __nv_bfloat16*>(W);
  const int32_t k = static_cast<int32_t>(K), n = static_cast<int32_t>(N);
  col_amax_kernel<<<dim3(static_cast<unsigned>((N + 255) / 256), static_cast<unsigned>(E)), 256, 0,
                    stream>>>(w, k, n, scale);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  quantize_cols_kernel<<<dim3(static_cast<unsigned>((N + 63) / 64), static_cast<unsigned>((K + 63) / 64),
                              static_cast<unsigned>(E)),
                         256, 0, stream>>>(w, k, n, scale, static_cast<uint8_t*>(qT));
  return cudaGetLastError();
}

// ---------------------------------------------------------------- FP8 grouped GEMM
// Same persistent warp-specialised structure as the bf16 grouped GEMM
// (grouped_gemm.cu): warp 0 TMA, warp 1 TMEM + MMA, warps 2..5 epilogue; 128 x 256
// tiles, experts' rows cut into 128-row tiles, n-tile outer, m-tile inner.  A stage
// holds 128 of K: A 128 rows x 128 bytes, B 256 rows (N) x 128 bytes, both
// K-major with the 128-byte swizzle; four MMAs of K = 32 per stage.

namespace {
constexpr int Q_BM = 128;
constexpr int Q_BN = 256;
constexpr int Q_BK = 128;  // elements = bytes
constexpr int Q_STAGES = 4;
constexpr int Q_THREADS = 192;
constexpr int Q_A_BYTES = Q_BM * Q_BK;
constexpr int Q_B_BYTES = Q_BN * Q_BK;
constexpr int Q_STAGE_BYTES = Q_A_BYTES + Q_B_BYTES;
constexpr int Q_TMEM_COLS = 512;
constexpr int Q_DYN_SMEM = Q_STAGES * Q_STAGE_BYTES + 4 * EPI_STAGE_BYTES_PER_WARP + 1024;
// instruction descriptor, kind::f8f6f4: D fp32, A and B E4M3, both K-major
constexpr uint32_t Q_IDESC = (1u << 4) | (0u << 7) | (0u << 10) | (0u << 15) | (0u << 16) |
                             (static_cast<uint32_t>(Q_BN >> 3) << 17) |
                             (static_cast<uint32_t>(Q_BM >> 4) << 24);

__device__ __forceinline__ void umma_e4m3(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(0u), "r"(0u), "r"(0u), "r"(0u)
      : "memory");
}

struct QArgs {
  const int32_t* offsets;
  int32_t E, R, K, N;
  int32_t n_tiles_n;
  const float* a_scale;  // [R]
  const float* b_scale;  // [E, N]
  const float* w_sorted; // [R] or nullptr (1)
  const int32_t* perm;   // [R] or nullptr (row s -> row s)
  float* C;              // fp32 [R, N]
  int32_t* status;
  uint64_t timeout_ns;
};

struct QTile {
  int32_t e, row0, rows, ni;
};

__device__ __forceinline__ QTile qdecode(int32_t t, const int32_t* s_tstart, const int32_t* s_off,
                                         int32_t E) {
  int32_t lo = 0, hi = E;
  while (hi - lo > 1) {
    const int32_t mid = (lo + hi) >> 1;
    if (s_tstart[mid] <= t) lo = mid; else hi = mid;
  }
  const int32_t e = lo;
  const int32_t mt = (s_off[e + 1] - s_off[e] + Q_BM - 1) / Q_BM;
  const int32_t local = t - s_tstart[e];
  QTile c;
  c.e = e;
  c.ni = local / mt;
  const int32_t mi = local - c.ni * mt;
  c.row0 = s_off[e] + mi * Q_BM;
  c.rows = min(Q_BM, s_off[e + 1] - c.row0);
  return c;
}
}  // namespace

// One accumulator row of a 128 x 256 (or pair-half) tile: acc * (gate weight x row
// scale) * column scale, written in fp32 to row perm[s] (or s), columns col0 ...
__device__ __forceinline__ void fp8_scatter_epilogue(const QArgs& args, uint32_t t_row, int32_t e,
                                                     int32_t s, bool row_ok, int32_t col0,
                                                     uint4* stage_buf, int lane) {
  float rs = 0.0f;
  float* dst = nullptr;
  if (row_ok) {
    int32_t dest = s;
    float w = 1.0f;
    if (args.perm != nullptr) dest = __ldg(args.perm + s);
    if (args.w_sorted != nullptr) w = __ldg(args.w_sorted + s);
    rs = w * __ldg(args.a_scale + s);
    if (dest < 0 || dest >= args.R)
      set_status(args.status, MOE_ERR_BAD_INDEX);
    else
      dst = args.C + static_cast<int64_t>(dest) * args.N + col0;
  }
  const float* bs = args.b_scale + static_cast<int64_t>(e) * args.N + col0;
  const int32_t n_left = args.N - col0;
#pragma unroll 1
  for (int c = 0; c < 8; ++c) {  // 32 fp32 columns = 128 bytes per segment
    float v[32];
    uint4 seg[8];
    tmem_ld32(t_row + c * 32, v);
    tmem_ld_wait();
    const bool in = c * 32 < n_left;
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = v[i] * rs * (in ? __ldg(bs + c * 32 + i) : 0.0f);
#pragma unroll
    for (int i = 0; i < 8; ++i)
      seg[i] = make_uint4(__float_as_uint(v[4 * i]), __float_as_uint(v[4 * i + 1]),
                          __float_as_uint(v[4 * i + 2]), __float_as_uint(v[4 * i + 3]));
    uint8_t* d = (dst != nullptr && in) ? reinterpret_cast<uint8_t*>(dst + c * 32) : nullptr;
    warp_store_rows128(seg, d, stage_buf, lane);
  }
}

__global__ void __launch_bounds__(Q_THREADS, 1)
    grouped_gemm_e4m3_kernel(const __grid_constant__ CUtensorMap tmA,
                             const __grid_constant__ CUtensorMap tmB, const QArgs args) {
  extern __shared__ uint8_t q_dyn_smem[];
  __shared__ __align__(8) uint64_t full_bar[Q_STAGES];
  __shared__ __align__(8) uint64_t empty_bar[Q_STAGES];
  __shared__ __align__(8) uint64_t tfull_bar[2];
  __shared__ __align__(8) uint64_t tempty_bar[2];
  __shared__ __align__(8) uint64_t drain_bar;
  __shared__ uint32_t s_tmem_base;
  __shared__ volatile int32_t s_abort;
  __shared__ int32_t s_off[MOE_MAX_EXPERTS + 1];
  __shared__ int32_t s_tstart[MOE_MAX_EXPERTS + 1];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int32_t E = args.E;
  uint8_t* ring = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(q_dyn_smem) + 1023) & ~static_cast<uintptr_t>(1023));

  if (tid == 0) {
    for (int s = 0; s < Q_STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull_bar[b], 1);
      mbar_init(&tempty_bar[b], 128);
    }
    mbar_init(&drain_bar, 1);
    s_abort = 0;
    fence_barrier_init();
    fence_proxy_async_shared();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(&s_tmem_base, Q_TMEM_COLS);
    tmem_relinquish();
  }
  griddep_wait();
  for (int e = tid; e <= E; e += Q_THREADS) s_off[e] = args.offsets[e];
  __syncthreads();
  if (warp == 0) {
    int32_t bad = 0;
    for (int e = lane; e < E; e += 32)
      if (s_off[e] < 0 || s_off[e + 1] < s_off[e] || s_off[e + 1] > args.R) bad = 1;
    bad = __any_sync(0xffffffffu, bad);
    int32_t run = 0;
    for (int base = 0; base < E; base += 32) {
      const int e = base + lane;
      int32_t tiles = 0;
      if (e < E && !bad) tiles = ((s_off[e + 1] - s_off[e] + Q_BM - 1) / Q_BM) * args.n_tiles_n;
      int32_t incl = tiles;
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const int32_t v = __shfl_up_sync(0xffffffffu, incl, d);
        if (lane >= d) incl += v;
      }
      if (e < E) s_tstart[e] = run + incl - tiles;
      run += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) {
      s_tstart[E] = run;
      if (bad && blockIdx.x == 0) set_status(args.status, MOE_ERR_BAD_INDEX);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const uint32_t tmem_base = s_tmem_base;
  const int32_t T = s_tstart[E];
  const int32_t KB = (args.K + Q_BK - 1) / Q_BK;  // a short last k-block reads zeros

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ TMA producer
    uint32_t stage = 0, phase = 0, issued = 0;
    for (int32_t t = blockIdx.x; t < T && !s_abort; t += gridDim.x) {
      if (t + static_cast<int32_t>(gridDim.x) >= T) griddep_launch_dependents();
      const QTile tc = qdecode(t, s_tstart, s_off, E);
      for (int32_t kb = 0; kb < KB; ++kb) {
        if (!mbar_wait_bounded(&empty_bar[stage], phase ^ 1u, args.timeout_ns, &s_abort)) {
          set_status(args.status, MOE_ERR_TIMEOUT);
          s_abort = 1;
          break;
        }
        uint8_t* sa = ring + stage * Q_STAGE_BYTES;
        mbar_arrive_expect_tx(&full_bar[stage], Q_STAGE_BYTES);
        tma_load_2d(sa, &tmA, &full_bar[stage], kb * Q_BK, tc.row0);
        tma_load_3d(sa + Q_A_BYTES, &tmB, &full_bar[stage], kb * Q_BK, tc.ni * Q_BN, tc.e);
        ++issued;
        if (++stage == Q_STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    if (s_abort) {
      uint32_t st = stage, ph = phase;
      for (uint32_t q = 0; q < Q_STAGES && q < issued; ++q) {
        if (st == 0) {
          st = Q_STAGES - 1;
          ph ^= 1u;
        } else {
          --st;
        }
        mbar_wait_bounded(&full_bar[st], ph, args.timeout_ns, nullptr);
      }
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    uint32_t stage = 0, phase = 0, j = 0;
    bool issued_any = false;
    for (int32_t t = blockIdx.x; t < T && !s_abort; t += gridDim.x, ++j) {
      const uint32_t b = j & 1u, tph = (j >> 1) & 1u;
      if (!mbar_wait_bounded(&tempty_bar[b], tph ^ 1u, args.timeout_ns, &s_abort)) {
        set_status(args.status, MOE_ERR_TIMEOUT);
        s_abort = 1;
        break;
      }
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + b * Q_BN;
      for (int32_t kb = 0; kb < KB; ++kb) {
        if (!mbar_wait_bounded(&full_bar[stage], phase, args.timeout_ns, &s_abort)) {
          set_status(args.status, MOE_ERR_TIMEOUT);
          s_abort = 1;
          break;
        }
        tc_fence_after();
        const uint32_t a_addr = smem_u32(ring + stage * Q_STAGE_BYTES);
        const uint32_t b_addr = a_addr + Q_A_BYTES;
#pragma unroll
        for (int kk = 0; kk < Q_BK / 32; ++kk) {  // 32 elements = 32 bytes per MMA
          const uint64_t adesc = smem_desc_sw128(a_addr + kk * 32, 16, 1024);
          const uint64_t bdesc = smem_desc_sw128(b_addr + kk * 32, 16, 1024);
          umma_e4m3(d_tmem, adesc, bdesc, Q_IDESC, (kb | kk) != 0 ? 1u : 0u);
        }
        issued_any = true;
        umma_commit(&empty_bar[stage]);
        if (++stage == Q_STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (s_abort) break;
      umma_commit(&tfull_bar[b]);
    }
    if (s_abort && issued_any) {
      umma_commit(&drain_bar);
      mbar_wait_bounded(&drain_bar, 0, args.timeout_ns, nullptr);
    }
  } else if (warp >= 2) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const int r = q * 32 + lane;
    uint4* stage_buf = reinterpret_cast<uint4*>(ring + Q_STAGES * Q_STAGE_BYTES +
                                                (warp - 2) * EPI_STAGE_BYTES_PER_WARP);
    uint32_t j = 0;
    for (int32_t t = blockIdx.x; t < T && !s_abort; t += gridDim.x, ++j) {
      const QTile tc = qdecode(t, s_tstart, s_off, E);
      const uint32_t b = j & 1u, tph = (j >> 1) & 1u;
      int32_t okw = 1;
      if (lane == 0) okw = mbar_wait_bounded(&tfull_bar[b], tph, args.timeout_ns, &s_abort) ? 1 : 0;
      okw = __shfl_sync(0xffffffffu, okw, 0);
      if (!okw) {
        if (lane == 0) {
          set_status(args.status, MOE_ERR_TIMEOUT);
          s_abort = 1;
        }
        break;
      }
      __syncwarp();
      tc_fence_after();
      const uint32_t t_row = tmem_base + b * Q_BN + (static_cast<uint32_t>(q * 32) << 16);
      const bool row_ok = r < tc.rows;
      const int32_t s = tc.row0 + r;
      fp8_scatter_epilogue(args, t_row, tc.e, s, row_ok, tc.ni * Q_BN, stage_buf, lane);
      tc_fence_before();
      mbar_arrive(&tempty_bar[b]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, Q_TMEM_COLS);
  }
}


// ---------------------------------------------------------------- FP8 GEMM on CTA pairs
// The CTA-pair structure of grouped_gemm_2sm.cu with E4M3 operands: a cluster of
// two CTAs shares one 256-row m-tile; each CTA loads its 128 rows of A and 128
// rows (columns of the output) of the K-major B, the leader issues
// tcgen05.mma.cta_group::2.kind::f8f6f4 with M = 256, N = 256, K = 32 and commits
// to both CTAs' barriers.  A stage holds 256 of K (two 128-byte swizzle spans for
// A and for B, 64 KB per CTA; three stages): eight MMAs per barrier round trip.
namespace {
constexpr int QP_BM = 256;
constexpr int QP_BN = 256;
constexpr int QP_BK = 256;
constexpr int QP_STAGES = 3;
constexpr int QP_THREADS = 192;
constexpr int QP_BOX_BYTES = 128 * 128;             // 128 rows x 128 bytes of K
constexpr int QP_A_BYTES = (QP_BK / 128) * QP_BOX_BYTES;
constexpr int QP_B_BYTES = (QP_BK / 128) * QP_BOX_BYTES;
constexpr int QP_STAGE_BYTES = QP_A_BYTES + QP_B_BYTES;
constexpr int QP_TMEM_COLS = 512;
constexpr int QP_DYN_SMEM = QP_STAGES * QP_STAGE_BYTES + 4 * EPI_STAGE_BYTES_PER_WARP + 1024;
constexpr uint32_t QP_IDESC = (1u << 4) | (static_cast<uint32_t>(QP_BN >> 3) << 17) |
                              (static_cast<uint32_t>(QP_BM >> 4) << 24);

__device__ __forceinline__ QTile qdecode2(int32_t t, const int32_t* s_tstart, const int32_t* s_off,
                                          int32_t E) {
  int32_t lo = 0, hi = E;
  while (hi - lo > 1) {
    const int32_t mid = (lo + hi) >> 1;
    if (s_tstart[mid] <= t) lo = mid; else hi = mid;
  }
  const int32_t e = lo;
  const int32_t mt = (s_off[e + 1] - s_off[e] + QP_BM - 1) / QP_BM;
  const int32_t local = t - s_tstart[e];
  QTile c;
  c.e = e;
  c.ni = local / mt;
  const int32_t mi = local - c.ni * mt;
  c.row0 = s_off[e] + mi * QP_BM;
  c.rows = min(QP_BM, s_off[e + 1] - c.row0);
  return c;
}
}  // namespace

__global__ void __launch_bounds__(QP_THREADS, 1)
    grouped_gemm_e4m3_2sm_kernel(const __grid_constant__ CUtensorMap tmA,
                                 const __grid_constant__ CUtensorMap tmB, const QArgs args) {
  extern __shared__ uint8_t qp_dyn_smem[];
  __shared__ __align__(8) uint64_t full_bar[QP_STAGES];
  __shared__ __align__(8) uint64_t empty_bar[QP_STAGES];
  __shared__ __align__(8) uint64_t tfull_bar[2];
  __shared__ __align__(8) uint64_t tempty_bar[2];
  __shared__ __align__(8) uint64_t drain_bar;
  __shared__ uint32_t s_tmem_base;
  __shared__ volatile int32_t s_abort;
  __shared__ int32_t s_off[MOE_MAX_EXPERTS + 1];
  __shared__ int32_t s_tstart[MOE_MAX_EXPERTS + 1];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int32_t E = args.E;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const int32_t pair = static_cast<int32_t>(blockIdx.x) >> 1;
  const int32_t npairs = static_cast<int32_t>(gridDim.x) >> 1;
  uint8_t* ring = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(qp_dyn_smem) + 1023) & ~static_cast<uintptr_t>(1023));

  if (tid == 0) {
    for (int s = 0; s < QP_STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull_bar[b], 1);
      mbar_init(&tempty_bar[b], 8);  // 4 epilogue warps in each CTA of the pair
    }
    mbar_init(&drain_bar, 1);
    s_abort = 0;
    fence_barrier_init();
    fence_proxy_async_shared();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc2(&s_tmem_base, QP_TMEM_COLS);
    tmem_relinquish2();
  }
  griddep_wait();
  for (int e = tid; e <= E; e += QP_THREADS) s_off[e] = args.offsets[e];
  __syncthreads();
  if (warp == 0) {
    int32_t bad = 0;
    for (int e = lane; e < E; e += 32)
      if (s_off[e] < 0 || s_off[e + 1] < s_off[e] || s_off[e + 1] > args.R) bad = 1;
    bad = __any_sync(0xffffffffu, bad);
    int32_t run = 0;
    for (int base = 0; base < E; base += 32) {
      const int e = base + lane;
      int32_t tiles = 0;
      if (e < E && !bad) tiles = ((s_off[e + 1] - s_off[e] + QP_BM - 1) / QP_BM) * args.n_tiles_n;
      int32_t incl = tiles;
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const int32_t v = __shfl_up_sync(0xffffffffu, incl, d);
        if (lane >= d) incl += v;
      }
      if (e < E) s_tstart[e] = run + incl - tiles;
      run += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) {
      s_tstart[E] = run;
      if (bad && blockIdx.x == 0) set_status(args.status, MOE_ERR_BAD_INDEX);
    }
  }
  // barriers of both CTAs initialised and TMEM allocated before anyone signals
  tc_fence_before();
  cluster_sync();
  tc_fence_after();

  const uint32_t tmem_base = s_tmem_base;
  const int32_t T = s_tstart[E];
  const int32_t KB = (args.K + QP_BK - 1) / QP_BK;  // a short last k-block reads zeros

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    uint32_t stage = 0, phase = 0;
    bool issued_any = false;
    for (int32_t t = pair; t < T && !s_abort; t += npairs) {
      if (t + npairs >= T) griddep_launch_dependents();
      const QTile tc = qdecode2(t, s_tstart, s_off, E);
      const int32_t arow = tc.row0 + 128 * static_cast<int32_t>(rank);
      const int32_t brow = tc.ni * QP_BN + 128 * static_cast<int32_t>(rank);
      for (int32_t kb = 0; kb < KB; ++kb) {
        if (!mbar_wait_bounded(&empty_bar[stage], phase ^ 1u, args.timeout_ns, &s_abort)) {
          set_status(args.status, MOE_ERR_TIMEOUT);
          s_abort = 1;
          break;
        }
        const uint32_t fb = peer_addr(smem_u32(&full_bar[stage]), 0);
        if (leader) {
          asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(
                           smem_u32(&full_bar[stage])),
                       "r"(2 * QP_STAGE_BYTES)
                       : "memory");
        }
        uint8_t* sa = ring + stage * QP_STAGE_BYTES;
        uint8_t* sb = sa + QP_A_BYTES;
#pragma unroll
        for (int c = 0; c < QP_BK / 128; ++c) {
          tma2_load_2d(sa + c * QP_BOX_BYTES, &tmA, fb, kb * QP_BK + 128 * c, arow);
          tma2_load_3d(sb + c * QP_BOX_BYTES, &tmB, fb, kb * QP_BK + 128 * c, brow, tc.e);
        }
        issued_any = true;
        if (++stage == QP_STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    if (s_abort && issued_any) {
      // Loads in flight complete on the leader's barrier; give them time to land.
      const uint64_t t0 = globaltimer_ns();
      while (globaltimer_ns() - t0 < 2000000ull) __nanosleep(1000);
    }
  } else if (warp == 1 && lane == 0 && leader) {
    // ------------------------------------------------------------ MMA issuer (leader)
    uint32_t stage = 0, phase = 0, j = 0;
    bool issued_any = false;
    for (int32_t t = pair; t < T && !s_abort; t += npairs, ++j) {
      const uint32_t b = j & 1u, tph = (j >> 1) & 1u;
      if (!mbar_wait_cluster(&tempty_bar[b], tph ^ 1u, args.timeout_ns, &s_abort)) {
        set_status(args.status, MOE_ERR_TIMEOUT);
        s_abort = 1;
        break;
      }
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + b * QP_BN;
      for (int32_t kb = 0; kb < KB; ++kb) {
        if (!mbar_wait_bounded(&full_bar[stage], phase, args.timeout_ns, &s_abort)) {
          set_status(args.status, MOE_ERR_TIMEOUT);
          s_abort = 1;
          break;
        }
        tc_fence_after();
        const uint32_t a_addr = smem_u32(ring + stage * QP_STAGE_BYTES);
        const uint32_t b_addr = a_addr + QP_A_BYTES;
#pragma unroll
        for (int kk = 0; kk < QP_BK / 32; ++kk) {  // K = 32 bytes per MMA
          const uint32_t off = (kk >> 2) * QP_BOX_BYTES + (kk & 3) * 32;
          const uint64_t adesc = smem_desc_sw128(a_addr + off, 16, 1024);
          const uint64_t bdesc = smem_desc_sw128(b_addr + off, 16, 1024);
          umma2_e4m3(d_tmem, adesc, bdesc, QP_IDESC, (kb | kk) != 0 ? 1u : 0u);
        }
        issued_any = true;
        const uint32_t eb = smem_u32(&empty_bar[stage]);
        umma2_commit(eb);
        umma2_commit(peer_addr(eb, 1));
        if (++stage == QP_STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (s_abort) break;
      const uint32_t fb = smem_u32(&tfull_bar[b]);
      umma2_commit(fb);
      umma2_commit(peer_addr(fb, 1));
    }
    if (s_abort && issued_any) {
      umma2_commit(smem_u32(&drain_bar));
      mbar_wait_bounded(&drain_bar, 0, args.timeout_ns, nullptr);
    }
  } else if (warp >= 2) {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int q = warp & 3;
    const int r = 128 * static_cast<int>(rank) + q * 32 + lane;  // row of the pair's tile
    uint4* stage_buf = reinterpret_cast<uint4*>(ring + QP_STAGES * QP_STAGE_BYTES +
                                                (warp - 2) * EPI_STAGE_BYTES_PER_WARP);
    const uint32_t te_leader0 = peer_addr(smem_u32(&tempty_bar[0]), 0);
    const uint32_t te_leader1 = peer_addr(smem_u32(&tempty_bar[1]), 0);
    uint32_t j = 0;
    for (int32_t t = pair; t < T && !s_abort; t += npairs, ++j) {
      const QTile tc = qdecode2(t, s_tstart, s_off, E);
      const uint32_t b = j & 1u, tph = (j >> 1) & 1u;
      int32_t okw = 1;
      if (lane == 0) okw = mbar_wait_bounded(&tfull_bar[b], tph, args.timeout_ns, &s_abort) ? 1 : 0;
      okw = __shfl_sync(0xffffffffu, okw, 0);
      if (!okw) {
        if (lane == 0) {
          set_status(args.status, MOE_ERR_TIMEOUT);
          s_abort = 1;
        }
        break;
      }
      __syncwarp();
      tc_fence_after();
      const uint32_t t_row = tmem_base + b * QP_BN + (static_cast<uint32_t>(q * 32) << 16);
      fp8_scatter_epilogue(args, t_row, tc.e, tc.row0 + r, r < tc.rows, tc.ni * QP_BN, stage_buf,
                           lane);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(b == 0 ? te_leader0 : te_leader1);
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the peer no longer touches this CTA's barriers or TMEM
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc2(tmem_base, QP_TMEM_COLS);
  }
}

// ---------------------------------------------------------------- host side

static bool enc_u8(CUtensorMap* m, int rank, const void* base, const cuuint64_t* dims,
                   const cuuint64_t* strides, const cuuint32_t* box) {
  const TensorMapEncodeFn enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, rank, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The pair kernel when experts average at least 1024 rows (as for the bf16
// GEMMs); MOE_GEMM_PAIR=0/1 forces one kernel.
static bool use_pair_e4m3(int64_t R, int32_t E) {
  const char* v = getenv("MOE_GEMM_PAIR");
  if (v != nullptr && v[0] == '0') return false;
  if (v != nullptr && v[0] == '1') return true;
  return E > 0 && R >= 1024 * static_cast<int64_t>(E);
}

// C [R, N] fp32 (row perm[s] if perm is given) = w_sorted[s] * a_scale[s] *
// b_scale[e, n] * (Aq[s, :] . BqT[e, n, :]).  Returns 0 ok, 1 tensor map, 2 CUDA.
int launch_grouped_gemm_e4m3(const void* Aq, const float* a_scale, const void* BqT,
                             const float* b_scale, const int32_t* offsets, int32_t E, int64_t R,
                             int64_t K, int64_t N, const float* w_sorted, const int32_t* perm,
                             float* C, int32_t* status, uint64_t timeout_ns, int num_sms,
                             cudaStream_t stream) {
  if (R == 0) return 0;
  CUtensorMap tmA, tmB;
  const cuuint64_t adims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(R)};
  const cuuint64_t astr[1] = {static_cast<cuuint64_t>(K)};
  const cuuint32_t abox[2] = {Q_BK, Q_BM};
  const cuuint64_t bdims[3] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(N),
                               static_cast<cuuint64_t>(E)};
  const cuuint64_t bstr[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(K * N)};
  const cuuint32_t bbox[3] = {Q_BK, Q_BN, 1};
  if (!enc_u8(&tmA, 2, Aq, adims, astr, abox) || !enc_u8(&tmB, 3, BqT, bdims, bstr, bbox)) return 1;
  QArgs a;
  a.offsets = offsets;
  a.E = E;
  a.R = static_cast<int32_t>(R);
  a.K = static_cast<int32_t>(K);
  a.N = static_cast<int32_t>(N);
  a.n_tiles_n = static_cast<int32_t>((N + Q_BN - 1) / Q_BN);
  a.a_scale = a_scale;
  a.b_scale = b_scale;
  a.w_sorted = w_sorted;
  a.perm = perm;
  a.C = C;
  a.status = status;
  a.timeout_ns = timeout_ns;
  static PerDeviceOnce once;
  const cudaError_t aerr = once.run([] {
    cudaError_t e = cudaFuncSetAttribute(grouped_gemm_e4m3_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, Q_DYN_SMEM);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(grouped_gemm_e4m3_2sm_kernel,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, QP_DYN_SMEM);
    return e;
  });
  if (aerr != cudaSuccess) return 2;
  if (num_sms >= 2 && use_pair_e4m3(R, E)) {
    // boxes of 128 rows: both CTAs of a pair load their own half of A and of B
    CUtensorMap pA, pB;
    const cuuint32_t pabox[2] = {128, 128};
    const cuuint32_t pbbox[3] = {128, 128, 1};
    if (!enc_u8(&pA, 2, Aq, adims, astr, pabox) || !enc_u8(&pB, 3, BqT, bdims, bstr, pbbox)) return 1;
    const int64_t ptiles = (R / QP_BM + (E < R ? E : R)) * a.n_tiles_n;
    int64_t pairs = num_sms / 2;
    if (ptiles < pairs) pairs = ptiles;
    if (pairs < 1) pairs = 1;
    const cudaError_t perr = launch_pdl(grouped_gemm_e4m3_2sm_kernel, dim3(static_cast<unsigned>(2 * pairs)),
                                        dim3(QP_THREADS), QP_DYN_SMEM, stream, 2, pA, pB, a);
    return perr == cudaSuccess ? 0 : 2;
  }
  const int64_t tiles_max = (R / Q_BM + (E < R ? E : R)) * a.n_tiles_n;
  const int grid = static_cast<int>(tiles_max < num_sms ? tiles_max : num_sms);
  const cudaError_t err = launch_pdl(grouped_gemm_e4m3_kernel, dim3(grid), dim3(Q_THREADS),
                                     Q_DYN_SMEM, stream, 1, tmA, tmB, a);
  return err == cudaSuccess ? 0 : 2;
}

}  // namespace moe
