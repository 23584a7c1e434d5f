// mx.cu -- the down projection with block-scaled E4M3 operands (MX): quantisers,
// the scale-factor packing, and the grouped GEMM on tcgen05
// kind::mxf8f6f4.block_scale.
//
// The PTO MegaMoE article (section "MegaMoE 融合算子七阶段") has SwiGLU quantise
// each GMM1 segment as it consumes it, so that GMM2 runs on quantised
// activations.  A per-row scale needs the whole row before the first value can be
// encoded; a scale per block of 32 values along K needs only the block, so the
// GEMM1 epilogue can quantise the h values it holds (grouped_gemm_2sm.cu,
// EPI_SWIGLU_MX) and no pass over h follows.  The block scales do not factor out
// of the dot product; the tensor core applies them (one E8M0 scale per 32 K for
// every row of A and every column of B, read from TMEM).
//
// Format: blocks of 32 consecutive values along K share the scale 2^e, e the
// smallest integer with amax <= 448 * 2^e (clamped to [-127, 127], -127 for an
// all-zero block), stored as the byte e + 127; elements are q = E4M3(v * 2^-e),
// nearest, ties to even.
//
// Scale-factor groups.  The MMA reads the scales of 128 rows (or columns) and
// 4 K blocks (128 of K) from 4 TMEM columns, copied there from a 512-byte group
// in shared memory by tcgen05.cp (32x128b, replicated to the four lane quarters):
// row i + 32 j of the 128, K block b of the 4, at byte 16 i + 4 j + b.  In global
// memory the groups are stored in the order the GEMM loads them:
//   A (h):  [m-tile gm][128-row half][k-group g][512 B], m-tiles of 256 rows
//           counted over the experts in order (expert e's m-tile mi is
//           gm = sum over e' < e of ceil(rows_e' / 256), plus mi);
//   B (W2): [expert][256-column tile][k-group g][128-column half][512 B];
// with kg_pad = 2 * ceil(K / 256) groups (whole stages of 256 K).
#include <cuda_fp8.h>

#include "common.cuh"
#include "epilogue.cuh"
#include "pair.cuh"

namespace moe {

// ---------------------------------------------------------------- quantisers

// W [E, K, N] bf16 -> BqT [E, N, K] codes (K contiguous), sf [E, N, K / 32] row-major.
// One thread per (expert, column, K block): 32 reads down the column (coalesced
// across the warp's columns), one 32-byte code row and one scale byte.
__global__ void __launch_bounds__(256)
    quantize_weights_mx_kernel(const __nv_bfloat16* __restrict__ W, int32_t E, int32_t K, int32_t N,
                               uint8_t* __restrict__ BqT, uint8_t* __restrict__ sf) {
  const int32_t KB = K / 32;
  const int64_t total = static_cast<int64_t>(E) * KB * N;
  for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int32_t n = static_cast<int32_t>(idx % N);
    const int64_t rest = idx / N;
    const int32_t kb = static_cast<int32_t>(rest % KB);
    const int32_t e = static_cast<int32_t>(rest / KB);
    const __nv_bfloat16* col = W + (static_cast<int64_t>(e) * K + 32 * kb) * N + n;
    float v[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __bfloat162float(col[static_cast<int64_t>(i) * N]);
    uint4 lo, hi;
    const uint32_t code = mx_block32(v, lo, hi);
    const int64_t row = static_cast<int64_t>(e) * N + n;
    uint4* dst = reinterpret_cast<uint4*>(BqT + row * K + 32 * kb);
    dst[0] = lo;
    dst[1] = hi;
    sf[row * KB + kb] = static_cast<uint8_t>(code);
  }
}

// A [R, K] bf16 -> Aq [R, K] codes, sf [R, K / 32]: one thread per (row, K block).
__global__ void __launch_bounds__(256)
    quantize_rows_mx_kernel(const uint4* __restrict__ A, int32_t R, int32_t K, uint4* __restrict__ Aq,
                            uint8_t* __restrict__ sf) {
  const int32_t KB = K / 32;
  const int64_t total = static_cast<int64_t>(R) * KB;
  for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint4* src = A + idx * 4;   // 32 bf16 = 4 x 16 bytes; blocks are consecutive
    float v[32];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint4 w = __ldg(src + c);
      const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        v[8 * c + 2 * i] = __uint_as_float(u[i] << 16);
        v[8 * c + 2 * i + 1] = __uint_as_float(u[i] & 0xffff0000u);
      }
    }
    uint4 lo, hi;
    const uint32_t code = mx_block32(v, lo, hi);
    Aq[idx * 2] = lo;
    Aq[idx * 2 + 1] = hi;
    sf[idx] = static_cast<uint8_t>(code);
  }
}

// ---------------------------------------------------------------- scale-factor packing

// Row-major A scales [R, K / 32] -> groups.  Every 32-bit word of a group is one
// row's 4 blocks; a thread per word, grid-stride over (row, k-group) with the
// k-group fastest, so the reads of a warp are contiguous.  Each CTA first finds
// every expert's first m-tile (a scan of ceil(rows_e / 256)).  Words of K blocks
// past K / 32 are zero; rows past an expert's end and pad groups are not written
// (the GEMM reads them only for rows it does not store and K steps it does not
// issue).  Offsets inconsistent with R record MOE_ERR_BAD_INDEX and write nothing.
__global__ void __launch_bounds__(256)
    pack_sfa_kernel(const uint8_t* __restrict__ sf, const int32_t* __restrict__ offsets, int32_t E,
                    int32_t R, int32_t KB, int32_t kg_pad, uint8_t* __restrict__ groups,
                    int32_t* status) {
  __shared__ int32_t s_off[MOE_MAX_EXPERTS + 1];
  __shared__ int32_t s_m0[MOE_MAX_EXPERTS + 1];
  __shared__ int32_t s_bad;
  for (int e = threadIdx.x; e <= E; e += blockDim.x) s_off[e] = offsets[e];
  __syncthreads();
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    int32_t bad = 0, run = 0;
    for (int base = 0; base < E; base += 32) {
      const int e = base + lane;
      int32_t m = 0;
      if (e < E) {
        const int32_t lo = s_off[e], hi = s_off[e + 1];
        if (lo < 0 || hi < lo || hi > R) bad = 1;
        else m = (hi - lo + 255) / 256;
      }
      int32_t incl = m;
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const int32_t v = __shfl_up_sync(0xffffffffu, incl, d);
        if (lane >= d) incl += v;
      }
      if (e < E) s_m0[e] = run + incl - m;
      run += __shfl_sync(0xffffffffu, incl, 31);
    }
    bad = __any_sync(0xffffffffu, bad);
    if (lane == 0) {
      s_bad = bad;
      if (bad && blockIdx.x == 0) set_status(status, MOE_ERR_BAD_INDEX);
    }
  }
  __syncthreads();
  if (s_bad) return;
  const int32_t KG = (KB + 3) / 4;
  const int64_t total = static_cast<int64_t>(s_off[E] - s_off[0]) * KG;
  for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int32_t row = s_off[0] + static_cast<int32_t>(idx / KG), g = static_cast<int32_t>(idx % KG);
    int32_t lo = 0, hi = E;                     // expert of the row: s_off[lo] <= row < s_off[lo + 1]
    while (hi - lo > 1) {
      const int32_t mid = (lo + hi) >> 1;
      if (s_off[mid] <= row) lo = mid; else hi = mid;
    }
    const uint8_t* src = sf + static_cast<int64_t>(row) * KB + 4 * g;
    uint32_t w = 0;
#pragma unroll
    for (int b = 0; b < 4; ++b)
      if (4 * g + b < KB) w |= static_cast<uint32_t>(src[b]) << (8 * b);
    const int32_t local = row - s_off[lo];
    const int32_t gm = s_m0[lo] + local / 256, rr = local % 256, ri = rr & 127;
    uint8_t* dst = groups + (static_cast<int64_t>(gm * 2 + (rr >> 7)) * kg_pad + g) * 512 +
                   16 * (ri & 31) + 4 * (ri >> 5);
    *reinterpret_cast<uint32_t*>(dst) = w;
  }
}

// Row-major B scales [E, N, K / 32] -> groups [E][ceil(N / 256)][kg_pad][2][512]
// (256-column tile, k-group, 128-column half); columns past N and K blocks past
// K / 32 (pad groups included) are zero.
__global__ void __launch_bounds__(256)
    pack_sfb_kernel(const uint8_t* __restrict__ sf, int32_t E, int32_t N, int32_t KB, int32_t kg_pad,
                    uint8_t* __restrict__ groups) {
  const int32_t NT = (N + 255) / 256;
  const int64_t words = static_cast<int64_t>(E) * NT * kg_pad * 2 * 128;
  for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < words;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int32_t o = static_cast<int32_t>(idx & 127);           // word in the group
    const int32_t half = static_cast<int32_t>((idx >> 7) & 1);
    const int64_t grp = idx >> 8;
    const int32_t g = static_cast<int32_t>(grp % kg_pad);
    const int64_t en = grp / kg_pad;
    const int32_t nt = static_cast<int32_t>(en % NT), e = static_cast<int32_t>(en / NT);
    // word 4 i + j: column i + 32 j of the half
    const int32_t n = nt * 256 + half * 128 + (o >> 2) + 32 * (o & 3);
    uint32_t w = 0;
    if (n < N) {
      const uint8_t* src = sf + (static_cast<int64_t>(e) * N + n) * KB + 4 * g;
#pragma unroll
      for (int b = 0; b < 4; ++b)
        if (4 * g + b < KB) w |= static_cast<uint32_t>(src[b]) << (8 * b);
    }
    reinterpret_cast<uint32_t*>(groups)[idx] = w;
  }
}

// ---------------------------------------------------------------- MX grouped GEMM on CTA pairs
// Cluster of two CTAs per 256 x 256 output tile (tcgen05.mma.cta_group::2, M = 256,
// N = 256): each CTA loads its 128 rows of A and 128 columns of the K-major B; a
// stage holds 256 of K (two 128-byte swizzle spans of each), the scale groups of
// A (this CTA's 128 rows) and of B (all 256 columns) for its two k-groups; the
// leader's MMA thread copies the groups to the stage's TMEM columns and issues
// eight MMAs (K = 32 each).  Epilogue: acc * gate weight, fp32 rows scattered to
// token order (as the bf16 down projection).  Tiles are walked with a static
// stride, expert by expert, in groups of 8 m-tiles with the n-tile outer inside a
// group.
//
// TMEM (512 columns): two 256-column accumulators cannot sit side by side with
// the scale columns, so they overlap: accumulator 0 in columns [0, 256),
// accumulator 1 in [184, 440), scale slots (24 columns per stage: A groups at +0
// and +4, B groups at +8 (two 128-column blocks, +4 apart) and +16) in [440, 512).
// A tile's MMAs may start once the tile before it (in the other accumulator) has
// had its shared 72 columns read out: the epilogue loads those first (columns
// [160, 256) of accumulator 0, [0, 96) of accumulator 1), signals, then stores.
// Measured alternatives, all slower on B200 (the down projection of the Phi-3.5,
// Qwen2 and Mixtral shapes): N = 128 tiles (no overlap needed, but 0.34 of the
// fp8 peak on Phi-3.5 with plain E4M3 MMAs too: 1.5x the bytes per MMA); M = 128
// tiles for short experts' tails as in the bf16 GEMMs (slower on Qwen2 despite
// the smaller padding: an M = 128 tile loads the same B bytes for half the MMA
// work); six stages of 128 K instead of three of 256 K (6-13 % slower: twice the
// barrier round trips and scale copies per K); copying two stages' scales at once
// (5 % slower).
namespace {
constexpr int X_BM = 256;
constexpr int X_BN = 256;
constexpr int X_BK = 256;                          // bytes (= elements) of K per stage
constexpr int X_STAGES = 3;
constexpr int X_THREADS = 192;
constexpr int X_BOX = 128 * 128;                   // 128 rows x 128 bytes of K
constexpr int X_A_BYTES = 2 * X_BOX;
constexpr int X_B_BYTES = 2 * X_BOX;
constexpr int X_SFA_BYTES = 2 * 512;               // two k-groups, this CTA's 128 rows
constexpr int X_SFB_BYTES = 4 * 512;               // two k-groups x two 128-column blocks
constexpr int X_STAGE_BYTES = X_A_BYTES + X_B_BYTES + X_SFA_BYTES + X_SFB_BYTES;
constexpr int X_TMEM_COLS = 512;
constexpr uint32_t X_ACC1_COL = 184;               // accumulator 1: columns [184, 440)
constexpr uint32_t X_SF_COL = X_ACC1_COL + X_BN;   // stage s: columns 440 + 24 s + [0, 24)
constexpr int X_OVL_SEGS = 3;                      // 32-column segments holding the overlap
constexpr int X_DYN_SMEM = X_STAGES * X_STAGE_BYTES + 4 * EPI_STAGE_BYTES_PER_WARP + 1024;
constexpr int32_t kGroupMX = 8;
// E4M3 A and B, K-major, fp32 accumulate, E8M0 scales (bit 23), N >> 3, M >> 4
constexpr uint32_t X_IDESC = (1u << 23) | (static_cast<uint32_t>(X_BN >> 3) << 17) |
                             (static_cast<uint32_t>(X_BM >> 4) << 24);
static_assert(X_STAGE_BYTES % 1024 == 0, "stages keep the 1024-byte swizzle alignment");
static_assert(X_SF_COL + 24 * X_STAGES == X_TMEM_COLS, "scale columns fill the end of TMEM");
static_assert(32 * X_OVL_SEGS >= static_cast<int>(X_BN - X_ACC1_COL) &&
              X_BN - 32 * X_OVL_SEGS <= static_cast<int>(X_ACC1_COL),
              "the first-read segments cover the overlap of both accumulators");

struct MxArgs {
  const int32_t* offsets;
  int32_t E, R, K, N, n_tiles_n, kg_pad;
  const float* w_sorted;
  const int32_t* perm;
  float* C;
  int64_t ldc;
  int32_t* status;
  uint64_t timeout_ns;
};

struct XTile {
  int32_t e, row0, rows, ni, gm;
};

__device__ __forceinline__ XTile xdecode(int32_t t, const int32_t* s_tstart, const int32_t* s_off,
                                         int32_t E, int32_t n_tiles_n) {
  int32_t lo = 0, hi = E;
  while (hi - lo > 1) {
    const int32_t mid = (lo + hi) >> 1;
    if (s_tstart[mid] <= t) lo = mid; else hi = mid;
  }
  const int32_t e = lo;
  const int32_t mt = (s_off[e + 1] - s_off[e] + X_BM - 1) / X_BM;
  int32_t local = t - s_tstart[e];
  const int32_t gsz = mt < kGroupMX ? mt : kGroupMX;
  const int32_t g = local / (gsz * n_tiles_n);
  local -= g * gsz * n_tiles_n;
  const int32_t g_rows = min(gsz, mt - g * gsz);
  XTile c;
  c.e = e;
  c.ni = local / g_rows;
  const int32_t mi = g * gsz + (local - c.ni * g_rows);
  c.row0 = s_off[e] + mi * X_BM;
  c.rows = min(X_BM, s_off[e + 1] - c.row0);
  c.gm = s_tstart[e] / n_tiles_n + mi;
  return c;
}

// One 32-column fp32 segment of this thread's row, times `scale`, through the
// warp's staging buffer to dst (nullptr: not written).  Warp-collective.
// Arrival on the leader's accumulator barriers: relaxed, since the MMA side needs
// only the TMEM reads to be done (tcgen05.wait::ld precedes the arrival), not this
// warp's global stores, which a release arrival would wait for (measured: 14 %
// of the down projection's time on the Qwen2 shape, 2 % on Phi-3.5).
__device__ __forceinline__ void mbar_arrive_cluster_relaxed(uint32_t bar) {
  asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void store_seg32(const float (&v)[32], float scale, uint8_t* dst,
                                            uint4* buf, int lane) {
  uint4 seg[8];
#pragma unroll
  for (int q = 0; q < 8; ++q)
    seg[q] = make_uint4(__float_as_uint(v[4 * q] * scale), __float_as_uint(v[4 * q + 1] * scale),
                        __float_as_uint(v[4 * q + 2] * scale), __float_as_uint(v[4 * q + 3] * scale));
  warp_store_rows128(seg, dst, buf, lane);
}
}  // namespace

__global__ void __launch_bounds__(X_THREADS, 1)
    grouped_gemm_mx_2sm_kernel(const __grid_constant__ CUtensorMap tmA,
                               const __grid_constant__ CUtensorMap tmB,
                               const __grid_constant__ CUtensorMap tmSA,
                               const __grid_constant__ CUtensorMap tmSB, const MxArgs args) {
  extern __shared__ uint8_t x_dyn_smem[];
  __shared__ __align__(8) uint64_t full_bar[X_STAGES];
  __shared__ __align__(8) uint64_t empty_bar[X_STAGES];
  __shared__ __align__(8) uint64_t tfull_bar[2];
  __shared__ __align__(8) uint64_t tempty_bar[2];
  __shared__ __align__(8) uint64_t ovl_bar[2];
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
      (reinterpret_cast<uintptr_t>(x_dyn_smem) + 1023) & ~static_cast<uintptr_t>(1023));

  if (tid == 0) {
    for (int s = 0; s < X_STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull_bar[b], 1);
      mbar_init(&tempty_bar[b], 8);  // 4 epilogue warps in each CTA of the pair
      mbar_init(&ovl_bar[b], 8);
    }
    mbar_init(&drain_bar, 1);
    s_abort = 0;
    fence_barrier_init();
    fence_proxy_async_shared();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmSA);
    tma_prefetch_desc(&tmSB);
  }
  if (warp == 1) {
    tmem_alloc2(&s_tmem_base, X_TMEM_COLS);
    tmem_relinquish2();
  }
  griddep_wait();  // offsets, A and its scales are written by the kernels before this one
  for (int e = tid; e <= E; e += X_THREADS) s_off[e] = args.offsets[e];
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
      if (e < E && !bad) tiles = ((s_off[e + 1] - s_off[e] + X_BM - 1) / X_BM) * args.n_tiles_n;
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
  const int32_t KB = (args.K + X_BK - 1) / X_BK;   // a short last stage reads zeros
  const int32_t ksteps = args.K / 32;              // MMAs per tile (K is a multiple of 32)

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    uint32_t stage = 0, phase = 0;
    bool issued_any = false;
    for (int32_t t = pair; t < T && !s_abort; t += npairs) {
      if (t + npairs >= T) griddep_launch_dependents();
      const XTile tc = xdecode(t, s_tstart, s_off, E, args.n_tiles_n);
      const int32_t arow = tc.row0 + 128 * static_cast<int32_t>(rank);
      const int32_t brow = tc.ni * X_BN + 128 * static_cast<int32_t>(rank);
      // scale groups as rows of 128 bytes: 4 rows a group
      const int32_t sfa_row = (tc.gm * 2 + static_cast<int32_t>(rank)) * args.kg_pad * 4;
      const int32_t sfb_row = (tc.e * args.n_tiles_n + tc.ni) * args.kg_pad * 8;
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
                       "r"(2 * X_STAGE_BYTES)
                       : "memory");
        }
        uint8_t* sa = ring + stage * X_STAGE_BYTES;
        uint8_t* sb = sa + X_A_BYTES;
        uint8_t* ssfa = sb + X_B_BYTES;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          tma2_load_2d(sa + c * X_BOX, &tmA, fb, kb * X_BK + 128 * c, arow);
          tma2_load_3d(sb + c * X_BOX, &tmB, fb, kb * X_BK + 128 * c, brow, tc.e);
        }
        tma2_load_2d(ssfa, &tmSA, fb, 0, sfa_row + 8 * kb);
        tma2_load_2d(ssfa + X_SFA_BYTES, &tmSB, fb, 0, sfb_row + 16 * kb);
        issued_any = true;
        if (++stage == X_STAGES) {
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
      // this accumulator drained (tile j - 2) ...
      if (!mbar_wait_cluster(&tempty_bar[b], tph ^ 1u, args.timeout_ns, &s_abort)) {
        set_status(args.status, MOE_ERR_TIMEOUT);
        s_abort = 1;
        break;
      }
      // ... and the columns it shares with the other one read out (tile j - 1)
      if (j > 0 && !mbar_wait_cluster(&ovl_bar[b ^ 1u], ((j - 1) >> 1) & 1u, args.timeout_ns,
                                      &s_abort)) {
        set_status(args.status, MOE_ERR_TIMEOUT);
        s_abort = 1;
        break;
      }
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + (b ? X_ACC1_COL : 0u);
      for (int32_t kb = 0; kb < KB; ++kb) {
        if (!mbar_wait_bounded(&full_bar[stage], phase, args.timeout_ns, &s_abort)) {
          set_status(args.status, MOE_ERR_TIMEOUT);
          s_abort = 1;
          break;
        }
        tc_fence_after();
        const uint32_t a_addr = smem_u32(ring + stage * X_STAGE_BYTES);
        const uint32_t b_addr = a_addr + X_A_BYTES;
        const uint32_t sfa_addr = b_addr + X_B_BYTES;
        const uint32_t sfb_addr = sfa_addr + X_SFA_BYTES;
        // this stage's scale groups -> its own TMEM columns (the stage's previous
        // MMAs finished before its data could be reloaded); the copies run before
        // the MMAs that read them
        const uint32_t sf_col = tmem_base + X_SF_COL + 24u * stage;
#pragma unroll
        for (int g = 0; g < 2; ++g) {
          utccp2_sf(sf_col + 4 * g, smem_desc_plain(sfa_addr + 512 * g));
          utccp2_sf(sf_col + 8 + 8 * g, smem_desc_plain(sfb_addr + 1024 * g));
          utccp2_sf(sf_col + 12 + 8 * g, smem_desc_plain(sfb_addr + 1024 * g + 512));
        }
        const int32_t nk = min(8, ksteps - 8 * kb);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          if (kk < nk) {
            const uint32_t off = (kk >> 2) * X_BOX + (kk & 3) * 32;
            const uint64_t adesc = smem_desc_sw128(a_addr + off, 16, 1024);
            const uint64_t bdesc = smem_desc_sw128(b_addr + off, 16, 1024);
            const uint32_t id = static_cast<uint32_t>(kk & 3);
            const uint32_t sfa = (sf_col + 4 * (kk >> 2)) | (id << 30);
            const uint32_t sfb = (sf_col + 8 + 8 * (kk >> 2)) | (id << 30);
            umma2_mx(d_tmem, adesc, bdesc, X_IDESC | (id << 29) | (id << 4), sfa, sfb,
                     (kb | kk) != 0 ? 1u : 0u);
          }
        }
        issued_any = true;
        const uint32_t eb = smem_u32(&empty_bar[stage]);
        umma2_commit(eb);
        umma2_commit(peer_addr(eb, 1));
        if (++stage == X_STAGES) {
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
    uint4* stage_buf = reinterpret_cast<uint4*>(ring + X_STAGES * X_STAGE_BYTES +
                                                (warp - 2) * EPI_STAGE_BYTES_PER_WARP);
    const uint32_t te_leader0 = peer_addr(smem_u32(&tempty_bar[0]), 0);
    const uint32_t te_leader1 = peer_addr(smem_u32(&tempty_bar[1]), 0);
    const uint32_t ov_leader0 = peer_addr(smem_u32(&ovl_bar[0]), 0);
    const uint32_t ov_leader1 = peer_addr(smem_u32(&ovl_bar[1]), 0);
    uint32_t j = 0;
    for (int32_t t = pair; t < T && !s_abort; t += npairs, ++j) {
      const XTile tc = xdecode(t, s_tstart, s_off, E, args.n_tiles_n);
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
      const uint32_t t_row = tmem_base + (b ? X_ACC1_COL : 0u) + (static_cast<uint32_t>(q * 32) << 16);
      // segments (32 columns) that hold the shared columns: the last three of
      // accumulator 0, the first three of accumulator 1
      const int ov0 = b ? 0 : 8 - X_OVL_SEGS;
      float ov[X_OVL_SEGS][32];
#pragma unroll
      for (int c = 0; c < X_OVL_SEGS; ++c) tmem_ld32(t_row + 32 * (ov0 + c), ov[c]);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster_relaxed(b ? ov_leader1 : ov_leader0);
      const int32_t col0 = tc.ni * X_BN;
      const int32_t n_left = args.N - col0;
      float scale = 1.0f;
      uint8_t* dst = nullptr;
      if (r < tc.rows) {
        const int32_t s = tc.row0 + r;
        const int32_t dest = args.perm != nullptr ? __ldg(args.perm + s) : s;
        if (args.w_sorted != nullptr) scale = __ldg(args.w_sorted + s);
        if (dest < 0 || dest >= args.R)
          set_status(args.status, MOE_ERR_BAD_INDEX);
        else
          dst = reinterpret_cast<uint8_t*>(args.C + static_cast<int64_t>(dest) * args.ldc + col0);
      }
#pragma unroll
      for (int c = 0; c < X_OVL_SEGS; ++c) {
        const int sg = ov0 + c;
        store_seg32(ov[c], scale, (dst != nullptr && 32 * sg < n_left) ? dst + 128 * sg : nullptr,
                    stage_buf, lane);
      }
      const int rest0 = b ? X_OVL_SEGS : 0;        // the other five segments
#pragma unroll 1
      for (int c = 0; c < 8 - X_OVL_SEGS; ++c) {
        const int sg = rest0 + c;
        float v[32];
        tmem_ld32(t_row + 32 * sg, v);
        tmem_ld_wait();
        store_seg32(v, scale, (dst != nullptr && 32 * sg < n_left) ? dst + 128 * sg : nullptr,
                    stage_buf, lane);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster_relaxed(b ? te_leader1 : te_leader0);
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the peer no longer touches this CTA's barriers or TMEM
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc2(tmem_base, X_TMEM_COLS);
  }
}

// ---------------------------------------------------------------- host side

int32_t mx_kg_pad(int64_t K) { return static_cast<int32_t>(2 * ((K + X_BK - 1) / X_BK)); }

// Bytes of the A scale groups for R rows in E experts (an upper bound on the
// m-tiles: sum of ceil(rows_e / 256) <= R / 256 + E) and of the B groups.
size_t mx_sfa_bytes(int64_t R, int32_t E, int64_t K) {
  const int64_t mtiles = R / X_BM + (E < R ? E : R);
  return static_cast<size_t>(mtiles) * 2 * static_cast<size_t>(mx_kg_pad(K)) * 512;
}
size_t mx_sfb_bytes(int32_t E, int64_t N, int64_t K) {
  return static_cast<size_t>(E) * static_cast<size_t>((N + 255) / 256) *
         static_cast<size_t>(mx_kg_pad(K)) * 2 * 512;
}

static int grid_for(int64_t work, int per_block, int num_sms) {
  const int64_t want = (work + per_block - 1) / per_block;
  const int64_t cap = static_cast<int64_t>(num_sms) * 8;
  return static_cast<int>(want < 1 ? 1 : (want < cap ? want : cap));
}

cudaError_t launch_quantize_weights_mx(const void* W, int32_t E, int64_t K, int64_t N, void* BqT,
                                       uint8_t* sf, int num_sms, cudaStream_t stream) {
  const int64_t work = static_cast<int64_t>(E) * (K / 32) * N;
  if (work == 0) return cudaSuccess;
  quantize_weights_mx_kernel<<<grid_for(work, 256, num_sms), 256, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(W), E, static_cast<int32_t>(K), static_cast<int32_t>(N),
      static_cast<uint8_t*>(BqT), sf);
  return cudaGetLastError();
}

cudaError_t launch_quantize_rows_mx(const void* A, int64_t R, int64_t K, void* Aq, uint8_t* sf,
                                    int num_sms, cudaStream_t stream) {
  const int64_t work = R * (K / 32);
  if (work == 0) return cudaSuccess;
  quantize_rows_mx_kernel<<<grid_for(work, 256, num_sms), 256, 0, stream>>>(
      static_cast<const uint4*>(A), static_cast<int32_t>(R), static_cast<int32_t>(K),
      static_cast<uint4*>(Aq), sf);
  return cudaGetLastError();
}

cudaError_t launch_pack_sfa(const uint8_t* sf, const int32_t* offsets, int32_t E, int64_t R,
                            int64_t K, uint8_t* groups, int32_t* status, int num_sms,
                            cudaStream_t stream) {
  const int64_t words = R * ((K / 32 + 3) / 4);
  pack_sfa_kernel<<<grid_for(words, 256, num_sms), 256, 0, stream>>>(
      sf, offsets, E, static_cast<int32_t>(R), static_cast<int32_t>(K / 32), mx_kg_pad(K), groups,
      status);
  return cudaGetLastError();
}

cudaError_t launch_pack_sfb(const uint8_t* sf, int32_t E, int64_t N, int64_t K, uint8_t* groups,
                            int num_sms, cudaStream_t stream) {
  const int64_t words = static_cast<int64_t>(E) * ((N + 255) / 256) * mx_kg_pad(K) * 2 * 128;
  pack_sfb_kernel<<<grid_for(words, 256, num_sms), 256, 0, stream>>>(
      sf, E, static_cast<int32_t>(N), static_cast<int32_t>(K / 32), mx_kg_pad(K), groups);
  return cudaGetLastError();
}

static bool enc_mx(CUtensorMap* m, int rank, const void* base, const cuuint64_t* dims,
                   const cuuint64_t* strides, const cuuint32_t* box, bool swizzle) {
  const TensorMapEncodeFn enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, rank, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// C [R, N] fp32 (row perm[s] if perm is given) = w_sorted[s] * sum over K blocks of
// 2^(sa - 127) 2^(sb - 127) (Aq block . BqT block), with the scales in groups
// (sfa_groups for R rows / E experts, sfb_groups for E x N).  K a multiple of 32.
// Returns 0 ok, 1 tensor map, 2 CUDA.
int launch_grouped_gemm_mx(const void* Aq, const uint8_t* sfa_groups, const void* BqT,
                           const uint8_t* sfb_groups, const int32_t* offsets, int32_t E, int64_t R,
                           int64_t K, int64_t N, const float* w_sorted, const int32_t* perm,
                           float* C, int32_t* status, uint64_t timeout_ns, int num_sms,
                           cudaStream_t stream) {
  if (R == 0) return 0;
  const int32_t kg_pad = mx_kg_pad(K);
  const int64_t n_tiles_n = (N + X_BN - 1) / X_BN;
  CUtensorMap tmA, tmB, tmSA, tmSB;
  const cuuint64_t adims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(R)};
  const cuuint64_t astr[1] = {static_cast<cuuint64_t>(K)};
  const cuuint32_t abox[2] = {128, 128};
  const cuuint64_t bdims[3] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(N),
                               static_cast<cuuint64_t>(E)};
  const cuuint64_t bstr[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(K * N)};
  const cuuint32_t bbox[3] = {128, 128, 1};
  // scale groups as rows of 128 bytes: a stage loads two groups of A (8 rows) and
  // four of B (16 rows)
  const cuuint64_t sadims[2] = {128, static_cast<cuuint64_t>(mx_sfa_bytes(R, E, K) / 128)};
  const cuuint64_t sbdims[2] = {128, static_cast<cuuint64_t>(mx_sfb_bytes(E, N, K) / 128)};
  const cuuint64_t sstr[1] = {128};
  const cuuint32_t sabox[2] = {128, 8};
  const cuuint32_t sbbox[2] = {128, 16};
  if (!enc_mx(&tmA, 2, Aq, adims, astr, abox, true) || !enc_mx(&tmB, 3, BqT, bdims, bstr, bbox, true) ||
      !enc_mx(&tmSA, 2, sfa_groups, sadims, sstr, sabox, false) ||
      !enc_mx(&tmSB, 2, sfb_groups, sbdims, sstr, sbbox, false))
    return 1;
  MxArgs a;
  a.offsets = offsets;
  a.E = E;
  a.R = static_cast<int32_t>(R);
  a.K = static_cast<int32_t>(K);
  a.N = static_cast<int32_t>(N);
  a.n_tiles_n = static_cast<int32_t>(n_tiles_n);
  a.kg_pad = kg_pad;
  a.w_sorted = w_sorted;
  a.perm = perm;
  a.C = C;
  a.ldc = N;
  a.status = status;
  a.timeout_ns = timeout_ns;
  static PerDeviceOnce once;
  const cudaError_t aerr = once.run([] {
    return cudaFuncSetAttribute(grouped_gemm_mx_2sm_kernel,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, X_DYN_SMEM);
  });
  if (aerr != cudaSuccess) return 2;
  const int64_t tiles_max = (R / X_BM + (E < R ? E : R)) * n_tiles_n;
  int64_t pairs = num_sms / 2;
  if (tiles_max < pairs) pairs = tiles_max;
  if (pairs < 1) pairs = 1;
  const cudaError_t err = launch_pdl(grouped_gemm_mx_2sm_kernel, dim3(static_cast<unsigned>(2 * pairs)),
                                     dim3(X_THREADS), X_DYN_SMEM, stream, 2, tmA, tmB, tmSA, tmSB, a);
  return err == cudaSuccess ? 0 : 2;
}

}  // namespace moe
