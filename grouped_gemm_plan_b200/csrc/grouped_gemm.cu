// grouped_gemm.cu -- persistent grouped GEMM for sm_100a: TMA -> shared memory ring
// -> tcgen05.mma into TMEM -> fused epilogue.
//
// What it computes ("Grouped GEMM 为什么适合 MoE", section "Grouped GEMM 到底解决什么
// 问题"): C_e = A_e x B_e for every expert e, where A_e is the row segment
// [offsets[e], offsets[e+1]) of the expert-ordered activations and B_e = B[e].
// The same section describes the scheduling this kernel uses: a fixed set of
// CTAs (one per SM, persistent) walks one list of (expert, m-tile, n-tile) work
// units; section "1. Tiling" cuts each expert's rows into uniform 128-row tiles,
// so a busy expert becomes many tiles and an idle one none.  Section "2.
// Double-buffer pipeline" is the shared-memory ring (4 stages of 48 KB, refilled
// by TMA while the tensor cores consume) plus the two TMEM accumulators that let
// the epilogue of tile j overlap the main loop of tile j+1.  Section "Fused
// GemmAdd" is the epilogue: fp32 arithmetic on the accumulator, one cast to bf16.
//
// Roles inside a CTA of 192 threads:
//   warp 0       one thread issues TMA loads (A tile 128x64, B tile 64x256)
//   warp 1       allocates TMEM (512 columns); one thread issues tcgen05.mma
//   warps 2..5   epilogue: tcgen05.ld (one TMEM lane = one output row per thread),
//                fp32 math, bf16 stores (fp32 stores for the gate-weighted scatter,
//                whose rows are summed once more by the combine)
//
// Tile order: expert by expert; inside an expert, n-tile outer, m-tile inner, so
// the CTAs running at the same time share one B column block (read from HBM
// once) and re-read the expert's A rows from L2 (COMET review, section 4.1.2:
// layer 1 runs column-wise so that the first columns finish first).
//
// Layouts in shared memory (128-byte swizzle, as TMA writes them):
//   A: 128 rows x 128 bytes (64 bf16 of K), K-major.  tcgen05 descriptor:
//      SBO = 1024 B (8-row group stride); 16-element K steps advance the start
//      address by 32 B inside the swizzle atom.
//   B: four 64(K) x 64(N) boxes, 8 KB each, N-major (the weights are row-major
//      [K, N], N contiguous).  Descriptor: LBO = 8192 B (next 64-column group),
//      SBO = 1024 B (next 8 K-rows); 16-row K steps advance by 2048 B.
#include <cstdlib>

#include "common.cuh"
#include "epilogue.cuh"

namespace moe {

constexpr int G_BM = 128;
constexpr int G_BN = 256;
constexpr int G_BK = 64;
constexpr int G_STAGES = 4;
constexpr int G_THREADS = 192;
constexpr int G_EPI_THREADS = 128;
constexpr int G_A_BYTES = G_BM * G_BK * 2;        // 16 KB
constexpr int G_B_BOX_BYTES = G_BK * 64 * 2;      // 8 KB
constexpr int G_B_BYTES = 4 * G_B_BOX_BYTES;      // 32 KB
constexpr int G_STAGE_BYTES = G_A_BYTES + G_B_BYTES;
constexpr int G_TMEM_COLS = 512;                  // two 128 x 256 fp32 accumulators
// ring + one 4 KB epilogue staging buffer per epilogue warp + alignment slack
constexpr int G_DYN_SMEM = G_STAGES * G_STAGE_BYTES + 4 * EPI_STAGE_BYTES_PER_WARP + 1024;
constexpr uint32_t G_IDESC = idesc_bf16_f32(G_BM, G_BN, /*b_mn_major=*/true);

struct GemmArgs {
  const int32_t* offsets;
  int32_t E;
  int32_t R;
  int32_t K;
  int32_t n_out;      // columns of C written by one row (F for SWIGLU)
  int32_t n_tiles_n;  // n-tiles per m-tile
  int32_t up_col;     // SWIGLU: first up column of B (= F)
  const float* w_sorted;
  const int32_t* perm;
  __nv_bfloat16* C;   // bf16 output (STORE, SWIGLU)
  float* Cf;          // fp32 output (WEIGHT_SCATTER)
  int64_t ldc;
  int32_t* status;
  uint64_t timeout_ns;
};

struct TileCoord {
  int32_t e, row0, rows, ni;
};

// Tile t -> (expert, first row, valid rows, n-tile), using the per-expert tile
// starts in shared memory.
__device__ __forceinline__ TileCoord decode_tile(int32_t t, const int32_t* s_tstart,
                                                 const int32_t* s_off, int32_t E,
                                                 int32_t n_tiles_n) {
  int32_t lo = 0, hi = E;
  while (hi - lo > 1) {
    const int32_t mid = (lo + hi) >> 1;
    if (s_tstart[mid] <= t) lo = mid; else hi = mid;
  }
  const int32_t e = lo;
  const int32_t cnt = s_off[e + 1] - s_off[e];
  const int32_t mt = (cnt + G_BM - 1) / G_BM;
  const int32_t local = t - s_tstart[e];
  const int32_t ni = local / mt;
  const int32_t mi = local - ni * mt;
  TileCoord c;
  c.e = e;
  c.row0 = s_off[e] + mi * G_BM;
  c.rows = min(G_BM, s_off[e + 1] - c.row0);
  c.ni = ni;
  (void)n_tiles_n;
  return c;
}

template <int EPI>
__global__ void __launch_bounds__(G_THREADS, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmB, const GemmArgs args) {
  extern __shared__ uint8_t g_dyn_smem[];
  __shared__ __align__(8) uint64_t full_bar[G_STAGES];
  __shared__ __align__(8) uint64_t empty_bar[G_STAGES];
  __shared__ __align__(8) uint64_t tfull_bar[2];
  __shared__ __align__(8) uint64_t tempty_bar[2];
  __shared__ __align__(8) uint64_t drain_bar;
  __shared__ uint32_t s_tmem_base;
  __shared__ volatile int32_t s_abort;
  __shared__ int32_t s_off[MOE_MAX_EXPERTS + 1];
  __shared__ int32_t s_tstart[MOE_MAX_EXPERTS + 1];

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int32_t E = args.E;

  // 1024-byte aligned ring (the 128-byte swizzle pattern repeats every 1024 B).
  uint8_t* ring = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(g_dyn_smem) + 1023) & ~static_cast<uintptr_t>(1023));

  if (tid == 0) {
    for (int s = 0; s < G_STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull_bar[b], 1);
      mbar_init(&tempty_bar[b], G_EPI_THREADS);
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
    tmem_alloc(&s_tmem_base, G_TMEM_COLS);
    tmem_relinquish();
  }
  griddep_wait();  // offsets and A are written by the kernels before this one
  for (int e = tid; e <= E; e += G_THREADS) s_off[e] = args.offsets[e];
  __syncthreads();

  // Per-expert tile starts (warp 0); offsets are checked before any use.
  if (warp == 0) {
    int32_t bad = 0;
    for (int e = lane; e < E; e += 32)
      if (s_off[e] < 0 || s_off[e + 1] < s_off[e] || s_off[e + 1] > args.R) bad = 1;
    bad = __any_sync(0xffffffffu, bad);
    int32_t run = 0;
    for (int base = 0; base < E; base += 32) {
      const int e = base + lane;
      int32_t tiles = 0;
      if (e < E && !bad) tiles = ((s_off[e + 1] - s_off[e] + G_BM - 1) / G_BM) * args.n_tiles_n;
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
  const int32_t KB = args.K / G_BK;

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ TMA producer
    uint32_t stage = 0, phase = 0;
    uint32_t issued = 0;
    for (int32_t t = blockIdx.x; t < T && !s_abort; t += gridDim.x) {
      // the next kernel may be scheduled once every CTA is on its last tile
      if (t + static_cast<int32_t>(gridDim.x) >= T) griddep_launch_dependents();
      const TileCoord tc = decode_tile(t, s_tstart, s_off, E, args.n_tiles_n);
      for (int32_t kb = 0; kb < KB; ++kb) {
        if (!mbar_wait_bounded(&empty_bar[stage], phase ^ 1u, args.timeout_ns, &s_abort)) {
          set_status(args.status, MOE_ERR_TIMEOUT);
          s_abort = 1;
          break;
        }
        uint8_t* sa = ring + stage * G_STAGE_BYTES;
        uint8_t* sb = sa + G_A_BYTES;
        mbar_arrive_expect_tx(&full_bar[stage], G_STAGE_BYTES);
        tma_load_2d(sa, &tmA, &full_bar[stage], kb * G_BK, tc.row0);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          int32_t n;
          if (EPI == MOE_EPI_SWIGLU)
            n = (j < 2) ? tc.ni * 128 + 64 * j : args.up_col + tc.ni * 128 + 64 * (j - 2);
          else
            n = tc.ni * G_BN + 64 * j;
          tma_load_3d(sb + j * G_B_BOX_BYTES, &tmB, &full_bar[stage], n, kb * G_BK, tc.e);
        }
        ++issued;
        if (++stage == G_STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    if (s_abort) {
      // Let every load still in flight land before the CTA's memory goes away.
      uint32_t st = stage, ph = phase;
      for (uint32_t q = 0; q < G_STAGES && q < issued; ++q) {
        if (st == 0) {
          st = G_STAGES - 1;
          ph ^= 1u;
        } else {
          --st;
        }
        mbar_wait_bounded(&full_bar[st], ph, args.timeout_ns, nullptr);
      }
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    uint32_t stage = 0, phase = 0;
    uint32_t j = 0;
    bool issued_any = false;
    for (int32_t t = blockIdx.x; t < T && !s_abort; t += gridDim.x, ++j) {
      const uint32_t b = j & 1u;
      const uint32_t tph = (j >> 1) & 1u;
      if (!mbar_wait_bounded(&tempty_bar[b], tph ^ 1u, args.timeout_ns, &s_abort)) {
        set_status(args.status, MOE_ERR_TIMEOUT);
        s_abort = 1;
        break;
      }
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + b * G_BN;
      for (int32_t kb = 0; kb < KB; ++kb) {
        if (!mbar_wait_bounded(&full_bar[stage], phase, args.timeout_ns, &s_abort)) {
          set_status(args.status, MOE_ERR_TIMEOUT);
          s_abort = 1;
          break;
        }
        tc_fence_after();
        const uint32_t a_addr = smem_u32(ring + stage * G_STAGE_BYTES);
        const uint32_t b_addr = a_addr + G_A_BYTES;
#pragma unroll
        for (int kk = 0; kk < G_BK / 16; ++kk) {
          const uint64_t adesc = smem_desc_sw128(a_addr + kk * 32, 16, 1024);
          const uint64_t bdesc = smem_desc_sw128(b_addr + kk * 2048, 8192, 1024);
          umma_bf16(d_tmem, adesc, bdesc, G_IDESC, (kb | kk) != 0 ? 1u : 0u);
        }
        issued_any = true;
        umma_commit(&empty_bar[stage]);
        if (++stage == G_STAGES) {
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
    const int q = warp & 3;                  // TMEM sub-partition of this warp
    const int r = q * 32 + lane;             // row of the tile this thread owns
    uint4* stage_buf = reinterpret_cast<uint4*>(ring + G_STAGES * G_STAGE_BYTES +
                                                (warp - 2) * EPI_STAGE_BYTES_PER_WARP);
    uint32_t j = 0;
    for (int32_t t = blockIdx.x; t < T && !s_abort; t += gridDim.x, ++j) {
      const TileCoord tc = decode_tile(t, s_tstart, s_off, E, args.n_tiles_n);
      const uint32_t b = j & 1u;
      const uint32_t tph = (j >> 1) & 1u;
      // one lane waits, the warp follows its verdict
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
      const uint32_t t_row = tmem_base + b * G_BN + (static_cast<uint32_t>(q * 32) << 16);
      const bool row_ok = r < tc.rows;
      const int32_t s = tc.row0 + r;
      if (EPI == MOE_EPI_SWIGLU) {
        const int32_t col0 = tc.ni * 128;
        uint8_t* dst = row_ok ? reinterpret_cast<uint8_t*>(args.C + static_cast<int64_t>(s) * args.ldc + col0)
                              : nullptr;
        epilogue_tile<MOE_EPI_SWIGLU>(t_row, dst, args.n_out - col0, 1.0f, stage_buf, lane);
      } else if (EPI == MOE_EPI_STORE) {
        const int32_t col0 = tc.ni * G_BN;
        uint8_t* dst = row_ok ? reinterpret_cast<uint8_t*>(args.C + static_cast<int64_t>(s) * args.ldc + col0)
                              : nullptr;
        epilogue_tile<MOE_EPI_STORE>(t_row, dst, args.n_out - col0, 1.0f, stage_buf, lane);
      } else {
        const int32_t col0 = tc.ni * G_BN;
        float scale = 1.0f;
        uint8_t* dst = nullptr;
        if (row_ok) {
          const int32_t dest = __ldg(args.perm + s);
          scale = __ldg(args.w_sorted + s);
          if (dest < 0 || dest >= args.R)
            set_status(args.status, MOE_ERR_BAD_INDEX);
          else
            dst = reinterpret_cast<uint8_t*>(args.Cf + static_cast<int64_t>(dest) * args.ldc + col0);
        }
        epilogue_tile<MOE_EPI_WEIGHT_SCATTER>(t_row, dst, args.n_out - col0, scale, stage_buf, lane);
      }
      tc_fence_before();
      mbar_arrive(&tempty_bar[b]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, G_TMEM_COLS);
  }
}

// ---------------------------------------------------------------- host side

// 2D bf16 map over a row-major [rows, cols] matrix, box 64 cols x box_rows rows.
static bool encode_2d(CUtensorMap* m, const void* base, int64_t rows, int64_t cols,
                      int box_rows) {
  const TensorMapEncodeFn enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
  cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3D bf16 map over row-major [E, K, N] weights, box 64 (N) x 64 (K) x 1.
static bool encode_3d(CUtensorMap* m, const void* base, int64_t E, int64_t K, int64_t N) {
  const TensorMapEncodeFn enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(K),
                        static_cast<cuuint64_t>(E)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(N) * 2, static_cast<cuuint64_t>(K * N) * 2};
  cuuint32_t box[3] = {64, 64, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int EPI>
static cudaError_t set_gemm_attr_once() {
  static PerDeviceOnce once;
  return once.run([] {
    return cudaFuncSetAttribute(grouped_gemm_kernel<EPI>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, G_DYN_SMEM);
  });
}

int launch_grouped_gemm_2sm(const void* A, const void* B, const int32_t* offsets, int32_t E,
                            int64_t R, int64_t K, int64_t N, int epi, const float* w_sorted,
                            const int32_t* perm, void* C, int32_t* status, uint64_t timeout_ns,
                            int num_sms, cudaStream_t stream);

// Which kernel runs a grouped GEMM: the CTA-pair kernel (grouped_gemm_2sm.cu),
// which moves a third fewer bytes into each SM per MMA, takes its tiles from the
// device tile queue and pads short experts only to 128 rows, on every shape; this
// single-CTA kernel (128-row tiles, static tile walk) when MOE_GEMM_PAIR=0 forces
// it (comparisons; the tests run both), or on a device with a single SM.
static bool use_pair_kernel(int64_t R, int32_t E) {
  const char* v = getenv("MOE_GEMM_PAIR");
  if (v != nullptr && v[0] == '0') return false;
  return R > 0 && E > 0;
}

static int launch_grouped_gemm_1sm(const void* A, const void* B, const int32_t* offsets, int32_t E,
                                   int64_t R, int64_t K, int64_t N, int epi, const float* w_sorted,
                                   const int32_t* perm, void* C, int32_t* status,
                                   uint64_t timeout_ns, int num_sms, cudaStream_t stream);

// Returns 0 on success, 1 if a tensor map could not be encoded, 2 on a CUDA error.
int launch_grouped_gemm(const void* A, const void* B, const int32_t* offsets, int32_t E,
                        int64_t R, int64_t K, int64_t N, int epi, const float* w_sorted,
                        const int32_t* perm, void* C, int32_t* status, uint64_t timeout_ns,
                        int num_sms, cudaStream_t stream) {
  if (num_sms >= 2 && use_pair_kernel(R, E))
    return launch_grouped_gemm_2sm(A, B, offsets, E, R, K, N, epi, w_sorted, perm, C, status,
                                   timeout_ns, num_sms, stream);
  return launch_grouped_gemm_1sm(A, B, offsets, E, R, K, N, epi, w_sorted, perm, C, status,
                                 timeout_ns, num_sms, stream);
}

static int launch_grouped_gemm_1sm(const void* A, const void* B, const int32_t* offsets, int32_t E,
                                   int64_t R, int64_t K, int64_t N, int epi, const float* w_sorted,
                                   const int32_t* perm, void* C, int32_t* status,
                                   uint64_t timeout_ns, int num_sms, cudaStream_t stream) {
  if (R == 0) return 0;
  CUtensorMap tmA, tmB;
  if (!encode_2d(&tmA, A, R, K, G_BM)) return 1;
  if (!encode_3d(&tmB, B, E, K, N)) return 1;
  GemmArgs a;
  a.offsets = offsets;
  a.E = E;
  a.R = static_cast<int32_t>(R);
  a.K = static_cast<int32_t>(K);
  a.w_sorted = w_sorted;
  a.perm = perm;
  a.C = reinterpret_cast<__nv_bfloat16*>(C);
  a.Cf = reinterpret_cast<float*>(C);
  a.status = status;
  a.timeout_ns = timeout_ns;
  if (epi == MOE_EPI_SWIGLU) {
    a.n_out = static_cast<int32_t>(N / 2);
    a.up_col = static_cast<int32_t>(N / 2);
    a.n_tiles_n = static_cast<int32_t>((N / 2 + 127) / 128);
    a.ldc = N / 2;
  } else {
    a.n_out = static_cast<int32_t>(N);
    a.up_col = 0;
    a.n_tiles_n = static_cast<int32_t>((N + G_BN - 1) / G_BN);
    a.ldc = N;
  }
  const int64_t m_tiles_max = R / G_BM + (E < R ? E : R);
  const int64_t tiles_max = m_tiles_max * a.n_tiles_n;
  const int grid = static_cast<int>(tiles_max < num_sms ? tiles_max : num_sms);
  cudaError_t err;
  switch (epi) {
    case MOE_EPI_SWIGLU:
      err = set_gemm_attr_once<MOE_EPI_SWIGLU>();
      if (err != cudaSuccess) return 2;
      err = launch_pdl(grouped_gemm_kernel<MOE_EPI_SWIGLU>, dim3(grid), dim3(G_THREADS), G_DYN_SMEM,
                       stream, 1, tmA, tmB, a);
      break;
    case MOE_EPI_WEIGHT_SCATTER:
      err = set_gemm_attr_once<MOE_EPI_WEIGHT_SCATTER>();
      if (err != cudaSuccess) return 2;
      err = launch_pdl(grouped_gemm_kernel<MOE_EPI_WEIGHT_SCATTER>, dim3(grid), dim3(G_THREADS),
                       G_DYN_SMEM, stream, 1, tmA, tmB, a);
      break;
    default:
      err = set_gemm_attr_once<MOE_EPI_STORE>();
      if (err != cudaSuccess) return 2;
      err = launch_pdl(grouped_gemm_kernel<MOE_EPI_STORE>, dim3(grid), dim3(G_THREADS), G_DYN_SMEM,
                       stream, 1, tmA, tmB, a);
      break;
  }
  return err == cudaSuccess ? 0 : 2;
}

}  // namespace moe
