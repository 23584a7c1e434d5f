// grouped_gemm_2sm.cu -- the grouped GEMM on CTA pairs: tcgen05.mma.cta_group::2
// with a 256 x 256 tile per pair of SMs.
//
// Same computation and tile order as grouped_gemm.cu ("Grouped GEMM 为什么适合
// MoE", sections "Grouped GEMM 到底解决什么问题", "1. Tiling", "2. Double-buffer
// pipeline", "Fused GemmAdd"); the difference is how a tile is fed.  A cluster of
// two CTAs on neighbouring SMs shares one 256-row m-tile: each CTA loads its own
// 128 rows of A and one half (128 columns) of B, and the leader CTA issues one
// M = 256, N = 256 MMA that reads A and B from both CTAs' shared memory and
// writes each CTA's 128 rows of the accumulator into that CTA's TMEM.  Per SM
// that halves the B bytes fetched for the same work (32 KB per 64 of K instead
// of 48 KB).  A stage holds 128 of K (eight MMAs per barrier round trip, three
// 64 KB stages), since the pair's barrier hand-offs cross SMs and cost more per
// round trip than the single-CTA kernel's.
//
// Protocol (leader = cluster rank 0, peer = rank 1):
//   full[s]    leader's barrier; the leader arrives with the byte count of both
//              CTAs' loads; both CTAs' TMA loads complete their bytes on it
//   empty[s]   in each CTA; the leader's MMA thread commits to both
//   tfull[b]   in each CTA; the leader commits to both after a tile's last MMA
//   tempty[b]  leader's barrier; one arrival per epilogue warp of both CTAs
// Peer addresses come from mapa.  No load is multicast.
#include "common.cuh"
#include "epilogue.cuh"
#include "pair.cuh"

namespace moe {

namespace {

constexpr int P_BM = 256;                 // rows per CTA pair
constexpr int P_BN = 256;
constexpr int P_BK = 128;                 // K per stage: 8 MMAs per barrier round trip
constexpr int P_STAGES = 3;
constexpr int P_THREADS = 192;
constexpr int P_A_BOX_BYTES = 128 * 64 * 2;     // 128 rows x 64 K (one 128-byte swizzle span)
constexpr int P_A_BYTES = (P_BK / 64) * P_A_BOX_BYTES;  // this CTA's 128 rows
constexpr int P_B_BOX_BYTES = P_BK * 64 * 2;    // 64 columns x P_BK rows of K
constexpr int P_B_BYTES = 2 * P_B_BOX_BYTES;    // this CTA's 128 columns
constexpr int P_STAGE_BYTES = P_A_BYTES + P_B_BYTES;
constexpr int P_TMEM_COLS = 512;
constexpr int P_DYN_SMEM = P_STAGES * P_STAGE_BYTES + 4 * EPI_STAGE_BYTES_PER_WARP + 1024;
constexpr uint32_t P_IDESC = idesc_bf16_f32(256, P_BN, true);

struct Gemm2Args {
  const int32_t* offsets;
  int32_t E, R, K;
  int32_t n_out, n_tiles_n, up_col;
  const float* w_sorted;
  const int32_t* perm;
  __nv_bfloat16* C;
  float* Cf;
  int64_t ldc;
  int32_t* status;
  uint64_t timeout_ns;
};

struct PTile {
  int32_t e, row0, rows, ni;
};

__device__ __forceinline__ PTile decode2(int32_t t, const int32_t* s_tstart, const int32_t* s_off,
                                         int32_t E) {
  int32_t lo = 0, hi = E;
  while (hi - lo > 1) {
    const int32_t mid = (lo + hi) >> 1;
    if (s_tstart[mid] <= t) lo = mid; else hi = mid;
  }
  const int32_t e = lo;
  const int32_t mt = (s_off[e + 1] - s_off[e] + P_BM - 1) / P_BM;
  const int32_t local = t - s_tstart[e];
  PTile c;
  c.e = e;
  c.ni = local / mt;
  const int32_t mi = local - c.ni * mt;
  c.row0 = s_off[e] + mi * P_BM;
  c.rows = min(P_BM, s_off[e + 1] - c.row0);
  return c;
}

}  // namespace

template <int EPI>
__global__ void __launch_bounds__(P_THREADS, 1)
    grouped_gemm_2sm_kernel(const __grid_constant__ CUtensorMap tmA,
                            const __grid_constant__ CUtensorMap tmB, const Gemm2Args args) {
  extern __shared__ uint8_t p_dyn_smem[];
  __shared__ __align__(8) uint64_t full_bar[P_STAGES];
  __shared__ __align__(8) uint64_t empty_bar[P_STAGES];
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
      (reinterpret_cast<uintptr_t>(p_dyn_smem) + 1023) & ~static_cast<uintptr_t>(1023));

  if (tid == 0) {
    for (int s = 0; s < P_STAGES; ++s) {
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
    tmem_alloc2(&s_tmem_base, P_TMEM_COLS);
    tmem_relinquish2();
  }
  griddep_wait();  // offsets and A are written by the kernels before this one
  for (int e = tid; e <= E; e += P_THREADS) s_off[e] = args.offsets[e];
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
      if (e < E && !bad) tiles = ((s_off[e + 1] - s_off[e] + P_BM - 1) / P_BM) * args.n_tiles_n;
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
  const int32_t KB = (args.K + P_BK - 1) / P_BK;  // a short last k-block reads zeros

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    uint32_t stage = 0, phase = 0;
    bool issued_any = false;
    for (int32_t t = pair; t < T && !s_abort; t += npairs) {
      // the next kernel may be scheduled once every CTA is on its last tile
      if (t + npairs >= T) griddep_launch_dependents();
      const PTile tc = decode2(t, s_tstart, s_off, E);
      const int32_t arow = tc.row0 + 128 * static_cast<int32_t>(rank);
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
                       "r"(2 * P_STAGE_BYTES)
                       : "memory");
        }
        uint8_t* sa = ring + stage * P_STAGE_BYTES;
        uint8_t* sb = sa + P_A_BYTES;
#pragma unroll
        for (int c = 0; c < P_BK / 64; ++c)
          tma2_load_2d(sa + c * P_A_BOX_BYTES, &tmA, fb, kb * P_BK + 64 * c, arow);
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          int32_t n;
          if (EPI == MOE_EPI_SWIGLU)  // leader: gate columns, peer: up columns
            n = (rank == 0 ? 0 : args.up_col) + tc.ni * 128 + 64 * j;
          else
            n = tc.ni * P_BN + 128 * static_cast<int32_t>(rank) + 64 * j;
          tma2_load_3d(sb + j * P_B_BOX_BYTES, &tmB, fb, n, kb * P_BK, tc.e);
        }
        issued_any = true;
        if (++stage == P_STAGES) {
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
      const uint32_t d_tmem = tmem_base + b * P_BN;
      for (int32_t kb = 0; kb < KB; ++kb) {
        if (!mbar_wait_bounded(&full_bar[stage], phase, args.timeout_ns, &s_abort)) {
          set_status(args.status, MOE_ERR_TIMEOUT);
          s_abort = 1;
          break;
        }
        tc_fence_after();
        const uint32_t a_addr = smem_u32(ring + stage * P_STAGE_BYTES);
        const uint32_t b_addr = a_addr + P_A_BYTES;
#pragma unroll
        for (int kk = 0; kk < P_BK / 16; ++kk) {
          const uint64_t adesc = smem_desc_sw128(a_addr + (kk >> 2) * P_A_BOX_BYTES + (kk & 3) * 32, 16, 1024);
          const uint64_t bdesc = smem_desc_sw128(b_addr + kk * 2048, P_B_BOX_BYTES, 1024);
          umma2_bf16(d_tmem, adesc, bdesc, P_IDESC, (kb | kk) != 0 ? 1u : 0u);
        }
        issued_any = true;
        const uint32_t eb = smem_u32(&empty_bar[stage]);
        umma2_commit(eb);
        umma2_commit(peer_addr(eb, 1));
        if (++stage == P_STAGES) {
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
    const int rr = q * 32 + lane;                          // row of this CTA's half
    const int r = 128 * static_cast<int>(rank) + rr;        // row of the pair's tile
    uint4* stage_buf = reinterpret_cast<uint4*>(ring + P_STAGES * P_STAGE_BYTES +
                                                (warp - 2) * EPI_STAGE_BYTES_PER_WARP);
    const uint32_t te_leader0 = peer_addr(smem_u32(&tempty_bar[0]), 0);
    const uint32_t te_leader1 = peer_addr(smem_u32(&tempty_bar[1]), 0);
    uint32_t j = 0;
    for (int32_t t = pair; t < T && !s_abort; t += npairs, ++j) {
      const PTile tc = decode2(t, s_tstart, s_off, E);
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
      const uint32_t t_row = tmem_base + b * P_BN + (static_cast<uint32_t>(q * 32) << 16);
      const bool row_ok = r < tc.rows;
      const int32_t s = tc.row0 + r;
      if (EPI == MOE_EPI_SWIGLU) {
        const int32_t col0 = tc.ni * 128;
        uint8_t* dst = row_ok ? reinterpret_cast<uint8_t*>(args.C + static_cast<int64_t>(s) * args.ldc + col0)
                              : nullptr;
        epilogue_tile<MOE_EPI_SWIGLU>(t_row, dst, args.n_out - col0, 1.0f, stage_buf, lane);
      } else if (EPI == MOE_EPI_STORE) {
        const int32_t col0 = tc.ni * P_BN;
        uint8_t* dst = row_ok ? reinterpret_cast<uint8_t*>(args.C + static_cast<int64_t>(s) * args.ldc + col0)
                              : nullptr;
        epilogue_tile<MOE_EPI_STORE>(t_row, dst, args.n_out - col0, 1.0f, stage_buf, lane);
      } else {
        const int32_t col0 = tc.ni * P_BN;
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
    tmem_dealloc2(tmem_base, P_TMEM_COLS);
  }
}

// ---------------------------------------------------------------- host side

static bool enc2(CUtensorMap* m, int rank, const void* base, const cuuint64_t* dims,
                 const cuuint64_t* strides, const cuuint32_t* box) {
  const TensorMapEncodeFn enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int EPI>
static cudaError_t launch2_t(int grid, const CUtensorMap& a, const CUtensorMap& b,
                             const Gemm2Args& args, cudaStream_t stream) {
  static PerDeviceOnce once;
  const cudaError_t err = once.run([] {
    cudaError_t e = cudaFuncSetAttribute(grouped_gemm_2sm_kernel<EPI>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, P_DYN_SMEM);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(grouped_gemm_2sm_kernel<EPI>,
                               cudaFuncAttributeNonPortableClusterSizeAllowed, 0);
    return e;
  });
  if (err != cudaSuccess) return err;
  return launch_pdl(grouped_gemm_2sm_kernel<EPI>, dim3(static_cast<unsigned>(grid)), dim3(P_THREADS),
                    P_DYN_SMEM, stream, 2, a, b, args);
}

// Same contract as launch_grouped_gemm (0 ok, 1 tensor map, 2 CUDA error).
int launch_grouped_gemm_2sm(const void* A, const void* B, const int32_t* offsets, int32_t E,
                            int64_t R, int64_t K, int64_t N, int epi, const float* w_sorted,
                            const int32_t* perm, void* C, int32_t* status, uint64_t timeout_ns,
                            int num_sms, cudaStream_t stream) {
  if (R == 0) return 0;
  CUtensorMap tmA, tmB;
  const cuuint64_t adims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(R)};
  const cuuint64_t astr[1] = {static_cast<cuuint64_t>(K) * 2};
  const cuuint32_t abox[2] = {64, 128};
  const cuuint64_t bdims[3] = {static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(K),
                               static_cast<cuuint64_t>(E)};
  const cuuint64_t bstr[2] = {static_cast<cuuint64_t>(N) * 2, static_cast<cuuint64_t>(K * N) * 2};
  const cuuint32_t bbox[3] = {64, P_BK, 1};
  if (!enc2(&tmA, 2, A, adims, astr, abox) || !enc2(&tmB, 3, B, bdims, bstr, bbox)) return 1;
  Gemm2Args a;
  a.offsets = offsets;
  a.E = E;
  a.R = static_cast<int32_t>(R);
  a.K = static_cast<int32_t>(K);
  a.w_sorted = w_sorted;
  a.perm = perm;
  a.C = static_cast<__nv_bfloat16*>(C);
  a.Cf = static_cast<float*>(C);
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
    a.n_tiles_n = static_cast<int32_t>((N + P_BN - 1) / P_BN);
    a.ldc = N;
  }
  const int64_t tiles_max = (R / P_BM + (E < R ? E : R)) * a.n_tiles_n;
  int64_t pairs = num_sms / 2;
  if (tiles_max < pairs) pairs = tiles_max;
  if (pairs < 1) pairs = 1;
  const int grid = static_cast<int>(2 * pairs);
  cudaError_t err;
  if (epi == MOE_EPI_SWIGLU)
    err = launch2_t<MOE_EPI_SWIGLU>(grid, tmA, tmB, a, stream);
  else if (epi == MOE_EPI_WEIGHT_SCATTER)
    err = launch2_t<MOE_EPI_WEIGHT_SCATTER>(grid, tmA, tmB, a, stream);
  else
    err = launch2_t<MOE_EPI_STORE>(grid, tmA, tmB, a, stream);
  return err == cudaSuccess ? 0 : 2;
}

}  // namespace moe
