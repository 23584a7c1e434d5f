// grouped_gemm_2sm.cu -- the grouped GEMM on CTA pairs (tcgen05.mma.cta_group::2)
// fed from a device tile queue.
//
// What it computes ("Grouped GEMM 为什么适合 MoE", section "Grouped GEMM 到底解决什么
// 问题"): C_e = A_e x B_e for every expert e, A_e the row segment [offsets[e],
// offsets[e+1]) of the expert-ordered activations, B_e = B[e]; the epilogue as in
// grouped_gemm.cu ("Fused GemmAdd": fp32 math on the accumulator, one cast).
//
// Scheduling (same section: a fixed set of CTAs keeps asking which expert's which
// tile comes next; "什么时候 Grouped GEMM 不一定赚": long tails need finer
// splitting): the grid is one CTA pair per two SMs, persistent.  The work is one
// list of tiles, expert by expert, and inside an expert n-tile outer, m-tile inner
// ("1. Tiling"), so the pairs running at the same time share a B column block.
// The leader CTA of a pair takes the next tile from an atomic ticket counter in
// the workspace (the device tile queue) when its producer starts a tile, and hands
// it to its own MMA and epilogue warps and to the peer CTA through a small ring in
// shared memory.  Tile shapes:
//   - full tiles: 256 rows x 256 accumulator columns (M = 256, N = 256), each CTA
//     loading its 128 rows of A and its half of B;
//   - an expert's last m-tile with at most 128 rows: M = 128 (64 rows per CTA), so
//     a short expert pads to a multiple of 128 rows rather than 256;
//   - when the last partial wave holds at most half as many tiles as there are
//     pairs, its tiles are issued as two N = 128 halves each, so the final wave
//     ends earlier.
// The ticket counter is reset to zero by the last CTA of the grid to finish.  The
// tile a pair computes does not change its arithmetic (no split-K, fixed K order),
// so results are bit-identical whichever pair takes which tile.
//
// Pipeline (per pair): TMA loads of both CTAs complete on the leader's stage
// barrier; the leader's single MMA thread issues eight MMAs (128 of K) per stage
// and commits to both CTAs' barriers; two TMEM accumulators let the epilogue of
// one tile overlap the next tile's main loop ("2. Double-buffer pipeline").
//
// TMEM layout of the accumulator (per CTA, 128 lanes): M = 256: lane l = row
// 128 * rank + l, column n = output column n.  M = 128: the CTA's 64 rows appear
// twice, lanes [0, 64) hold columns [0, 128) and lanes [64, 128) hold columns
// [128, 256), each in TMEM columns [0, 128).
// Peer addresses come from mapa.  No load is multicast.
#include "common.cuh"
#include "epilogue.cuh"
#include "pair.cuh"

namespace moe {

namespace {

constexpr int P_BM = 256;                 // rows of a full pair tile
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
constexpr int P_RING = 8;                 // tile ring entries
// consumers of a ring entry: leader MMA thread, 4 epilogue warps in each CTA, peer producer
constexpr uint32_t P_RING_CONSUMERS = 1 + 4 + 4 + 1;

// Tile variants in the ring
constexpr int32_t V_WHOLE = 0;            // all 256 accumulator columns
constexpr int32_t V_HALF0 = 1;            // accumulator columns [0, 128) of the tile
constexpr int32_t V_HALF1 = 2;            // accumulator columns [128, 256)
constexpr int32_t T_END = -1;

// m-tiles per raster group of the down projection (0: the whole expert): a group's
// activation rows stay in L2 while all of its n-tiles run ("3. L2 cache conflict
// 缓解").  Measured on B200: GEMM2 on the Phi-3.5 shape 0.835 -> 0.844 of the bf16
// peak; L2 eviction-priority hints on the loads (activations kept, weights evicted
// first) made both GEMMs 1-3 % slower and are not used.
constexpr int32_t kGroupM2 = 8;

struct Gemm2Args {
  const int32_t* offsets;
  int32_t E, R, K;
  int32_t n_out, n_tiles_n, up_col;
  const float* w_sorted;
  const int32_t* perm;
  __nv_bfloat16* C;
  float* Cf;
  int64_t ldc;
  // EPI_SWIGLU_MX: E4M3 codes of h [R, ldc] and their scale codes, row-major
  // [R, sf_ld] (sf_ld > 0) or in the 512-byte groups the block-scaled down
  // projection loads (sf_ld = 0; kg_pad groups of 128 columns per 128-row block)
  uint8_t* q;
  uint8_t* sf;
  int32_t sf_ld, kg_pad;
  int32_t* status;
  int32_t* queue;      // [0] ticket counter, [1] CTAs finished (both zero between launches)
  uint64_t timeout_ns;
};

struct PTile {
  int32_t e, row0, rows, ni;
  bool m128;           // M = 128 tile (at most 128 valid rows)
};

// Tile t -> (expert, rows, n-tile).  Inside an expert the tiles run in groups of
// group_m m-tiles (0: one group, the whole expert); inside a group n-tile outer,
// m-tile inner.
__device__ __forceinline__ PTile decode2(int32_t t, const int32_t* s_tstart, const int32_t* s_off,
                                         int32_t E, int32_t n_tiles_n, int32_t group_m) {
  int32_t lo = 0, hi = E;
  while (hi - lo > 1) {
    const int32_t mid = (lo + hi) >> 1;
    if (s_tstart[mid] <= t) lo = mid; else hi = mid;
  }
  const int32_t e = lo;
  const int32_t mt = (s_off[e + 1] - s_off[e] + P_BM - 1) / P_BM;
  int32_t local = t - s_tstart[e];
  const int32_t gm = (group_m > 0 && group_m < mt) ? group_m : mt;
  const int32_t g = local / (gm * n_tiles_n);
  local -= g * gm * n_tiles_n;
  const int32_t g_rows = min(gm, mt - g * gm);  // m-tiles in this group
  PTile c;
  c.e = e;
  c.ni = local / g_rows;
  const int32_t mi = g * gm + (local - c.ni * g_rows);
  c.row0 = s_off[e] + mi * P_BM;
  c.rows = min(P_BM, s_off[e + 1] - c.row0);
  c.m128 = c.rows <= 128;
  return c;
}

// Ticket -> (tile, variant).  Tickets [0, T - L) are whole tiles; tickets
// [T - L, T + L) are the last L tiles, two tickets each: its N halves, or for an
// M = 128 tile the whole tile on the first ticket and nothing (skip, returns
// false) on the second.
__device__ __forceinline__ bool ticket_to_tile(int32_t ticket, int32_t T, int32_t L,
                                               const int32_t* s_tstart, const int32_t* s_off,
                                               int32_t E, int32_t n_tiles_n, int32_t group_m,
                                               int32_t* tile, int32_t* variant) {
  if (ticket < T - L) {
    *tile = ticket;
    *variant = V_WHOLE;
    return true;
  }
  const int32_t u = ticket - (T - L);
  *tile = T - L + (u >> 1);
  const PTile pt = decode2(*tile, s_tstart, s_off, E, n_tiles_n, group_m);
  if (pt.m128) {
    *variant = V_WHOLE;
    return (u & 1) == 0;
  }
  *variant = (u & 1) ? V_HALF1 : V_HALF0;
  return true;
}

__device__ __forceinline__ void st_cluster_u32(uint32_t addr, int32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

}  // namespace

template <int EPI>
__global__ void __launch_bounds__(P_THREADS, 1)
    grouped_gemm_2sm_kernel(const __grid_constant__ CUtensorMap tmA,
                            const __grid_constant__ CUtensorMap tmA64,
                            const __grid_constant__ CUtensorMap tmB, const Gemm2Args args) {
  extern __shared__ uint8_t p_dyn_smem[];
  __shared__ __align__(8) uint64_t full_bar[P_STAGES];
  __shared__ __align__(8) uint64_t empty_bar[P_STAGES];
  __shared__ __align__(8) uint64_t tfull_bar[2];
  __shared__ __align__(8) uint64_t tempty_bar[2];
  __shared__ __align__(8) uint64_t drain_bar;
  __shared__ __align__(8) uint64_t ring_full[P_RING];
  __shared__ __align__(8) uint64_t ring_empty[P_RING];
  __shared__ int32_t s_ring_tile[P_RING];
  __shared__ int32_t s_ring_var[P_RING];
  __shared__ uint32_t s_tmem_base;
  __shared__ volatile int32_t s_abort;
  __shared__ int32_t s_off[MOE_MAX_EXPERTS + 1];
  __shared__ int32_t s_tstart[MOE_MAX_EXPERTS + 1];

  constexpr bool kSwiglu = EPI == MOE_EPI_SWIGLU || EPI == EPI_SWIGLU_MX;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int32_t E = args.E;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
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
    for (int q = 0; q < P_RING; ++q) {
      mbar_init(&ring_full[q], 1);
      mbar_init(&ring_empty[q], P_RING_CONSUMERS);
    }
    mbar_init(&drain_bar, 1);
    s_abort = 0;
    fence_barrier_init();
    fence_proxy_async_shared();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmA64);
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
  // Tiles issued as two tickets: the last partial wave's tiles, when their halves
  // fit one wave (a half tile costs more than half a tile, so splitting a wave that
  // is more than half full would make the end later, not earlier).
  const int32_t r_last = T % npairs;
  const int32_t L = 2 * r_last <= npairs ? r_last : 0;
  const int32_t tickets = T + L;
  const int32_t KB = (args.K + P_BK - 1) / P_BK;  // a short last k-block reads zeros
  const int32_t group_m = EPI == MOE_EPI_WEIGHT_SCATTER ? kGroupM2 : 0;

  // Waits for ring entry j and returns it (tile, variant); T_END when the list is
  // done or the wait ran out (then the abort flag is set).  Releases the entry: a
  // local arrival in the leader CTA, a remote one from the peer.
  auto ring_take = [&](uint32_t j, int32_t* var) -> int32_t {
    const uint32_t slot = j % P_RING, ph = (j / P_RING) & 1u;
    if (!mbar_wait_cluster(&ring_full[slot], ph, args.timeout_ns, &s_abort)) {
      set_status(args.status, MOE_ERR_TIMEOUT);
      s_abort = 1;
      return T_END;
    }
    const int32_t t = s_ring_tile[slot];
    *var = s_ring_var[slot];
    if (leader)
      mbar_arrive(&ring_empty[slot]);
    else
      mbar_arrive_cluster(peer_addr(smem_u32(&ring_empty[slot]), 0));
    return t;
  };

  // Leader only: resolves a ticket into ring entry j (tile and variant, taking more
  // tickets past the empty second tickets of M = 128 tail tiles) and hands it to
  // both CTAs.  Returns false if the wait for the ring slot ran out.
  auto ring_push = [&](uint32_t j, int32_t ticket, int32_t* t_out, int32_t* var_out) -> bool {
    int32_t t = T_END, var = V_WHOLE;
    for (;; ticket = atomicAdd(args.queue, 1)) {
      if (ticket < 0 || ticket >= tickets) {
        t = T_END;
        break;
      }
      if (ticket_to_tile(ticket, T, L, s_tstart, s_off, E, args.n_tiles_n, group_m, &t, &var)) break;
    }
    // this pair's last tile is under way: the next kernel may be scheduled
    if (t == T_END) griddep_launch_dependents();
    const uint32_t slot = j % P_RING, ph = (j / P_RING) & 1u;
    if (!mbar_wait_cluster(&ring_empty[slot], ph ^ 1u, args.timeout_ns, &s_abort)) {
      set_status(args.status, MOE_ERR_TIMEOUT);
      s_abort = 1;
      return false;
    }
    s_ring_tile[slot] = t;
    s_ring_var[slot] = var;
    st_cluster_u32(peer_addr(smem_u32(&s_ring_tile[slot]), 1), t);
    st_cluster_u32(peer_addr(smem_u32(&s_ring_var[slot]), 1), var);
    mbar_arrive_cluster(peer_addr(smem_u32(&ring_full[slot]), 0));
    mbar_arrive_cluster(peer_addr(smem_u32(&ring_full[slot]), 1));
    *t_out = t;
    *var_out = var;
    return true;
  };

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    uint32_t stage = 0, phase = 0;
    bool issued_any = false;
    // The leader hands out tile j + 1 while it issues the last k-blocks of tile j:
    // it takes the ticket four k-blocks before the end (the atomic's round trip to
    // L2 overlaps those loads) and pushes the entry two k-blocks before the end,
    // after that k-block's loads are issued, so neither producer waits for it at
    // the tile boundary.
    int32_t t = T_END, var = V_WHOLE;
    bool pushed = true;
    if (leader) pushed = ring_push(0, atomicAdd(args.queue, 1), &t, &var);
    for (uint32_t j = 0; !s_abort && pushed; ++j) {
      if (!leader) {
        t = ring_take(j, &var);
        if (t == T_END) griddep_launch_dependents();
      }
      if (t == T_END) break;
      const PTile tc = decode2(t, s_tstart, s_off, E, args.n_tiles_n, group_m);
      const bool half = var != V_WHOLE;
      const int32_t h = var == V_HALF1 ? 1 : 0;
      // this CTA's A rows: 128 of a full tile, 64 of an M = 128 tile
      const int32_t arow = tc.row0 + (tc.m128 ? 64 : 128) * static_cast<int32_t>(rank);
      const uint32_t a_bytes = tc.m128 ? P_A_BYTES / 2 : P_A_BYTES;
      const int nbox = half ? 1 : 2;  // B boxes of 64 columns this CTA loads
      const uint32_t cta_bytes = a_bytes + static_cast<uint32_t>(nbox) * P_B_BOX_BYTES;
      const int32_t kb_fetch = KB > 4 ? KB - 4 : 0;
      const int32_t kb_push = KB > 2 ? KB - 2 : 0;
      int32_t next_ticket = 0, next_t = T_END, next_var = V_WHOLE;
      bool next_pushed = false;
      for (int32_t kb = 0; kb < KB; ++kb) {
        if (!mbar_wait_bounded(&empty_bar[stage], phase ^ 1u, args.timeout_ns, &s_abort)) {
          set_status(args.status, MOE_ERR_TIMEOUT);
          s_abort = 1;
          break;
        }
        if (leader && kb == kb_fetch) next_ticket = atomicAdd(args.queue, 1);
        const uint32_t fb = peer_addr(smem_u32(&full_bar[stage]), 0);
        if (leader) {
          asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(
                           smem_u32(&full_bar[stage])),
                       "r"(2 * cta_bytes)
                       : "memory");
        }
        uint8_t* sa = ring + stage * P_STAGE_BYTES;
        uint8_t* sb = sa + P_A_BYTES;
#pragma unroll
        for (int c = 0; c < P_BK / 64; ++c)
          tma2_load_2d(sa + c * P_A_BOX_BYTES, tc.m128 ? &tmA64 : &tmA, fb, kb * P_BK + 64 * c, arow);
        for (int b = 0; b < nbox; ++b) {
          int32_t n;
          if (kSwiglu) {
            const int32_t j0 = tc.ni * 128;
            if (half)            // leader: gate, peer: up, 64 columns of the half
              n = (rank == 0 ? 0 : args.up_col) + j0 + 64 * h;
            else if (tc.m128)    // each CTA: 64 gate columns, then the same 64 up columns
              n = (b == 0 ? 0 : args.up_col) + j0 + 64 * static_cast<int32_t>(rank);
            else                 // leader: 128 gate columns, peer: 128 up columns
              n = (rank == 0 ? 0 : args.up_col) + j0 + 64 * b;
          } else {
            n = half ? tc.ni * P_BN + 128 * h + 64 * static_cast<int32_t>(rank)
                     : tc.ni * P_BN + 128 * static_cast<int32_t>(rank) + 64 * b;
          }
          tma2_load_3d(sb + b * P_B_BOX_BYTES, &tmB, fb, n, kb * P_BK, tc.e);
        }
        issued_any = true;
        if (++stage == P_STAGES) {
          stage = 0;
          phase ^= 1u;
        }
        if (leader && kb == kb_push) {
          next_pushed = ring_push(j + 1, next_ticket, &next_t, &next_var);
          if (!next_pushed) break;
        }
      }
      if (leader) {
        if (!next_pushed) break;   // abort before the next entry was handed out
        t = next_t;
        var = next_var;
      }
    }
    if (s_abort && issued_any) {
      // Loads in flight complete on the leader's barrier; give them time to land.
      const uint64_t t0 = globaltimer_ns();
      while (globaltimer_ns() - t0 < 2000000ull) __nanosleep(1000);
    }
  } else if (warp == 1 && lane == 0 && leader) {
    // ------------------------------------------------------------ MMA issuer (leader)
    uint32_t stage = 0, phase = 0;
    bool issued_any = false;
    for (uint32_t j = 0; !s_abort; ++j) {
      int32_t var = V_WHOLE;
      const int32_t t = ring_take(j, &var);
      if (t == T_END) break;
      const PTile tc = decode2(t, s_tstart, s_off, E, args.n_tiles_n, group_m);
      const uint32_t idesc = var != V_WHOLE ? idesc_bf16_f32(256, 128, true)
                                            : idesc_bf16_f32(tc.m128 ? 128 : 256, P_BN, true);
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
          umma2_bf16(d_tmem, adesc, bdesc, idesc, (kb | kk) != 0 ? 1u : 0u);
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
    const int q = warp & 3;              // TMEM sub-partition of this warp: lanes [32q, 32q + 32)
    uint4* stage_buf = reinterpret_cast<uint4*>(ring + P_STAGES * P_STAGE_BYTES +
                                                (warp - 2) * EPI_STAGE_BYTES_PER_WARP);
    const uint32_t te_leader0 = peer_addr(smem_u32(&tempty_bar[0]), 0);
    const uint32_t te_leader1 = peer_addr(smem_u32(&tempty_bar[1]), 0);
    for (uint32_t j = 0; !s_abort; ++j) {
      int32_t t = 0, var = V_WHOLE;
      if (lane == 0) t = ring_take(j, &var);
      t = __shfl_sync(0xffffffffu, t, 0);
      var = __shfl_sync(0xffffffffu, var, 0);
      if (t == T_END) break;
      const PTile tc = decode2(t, s_tstart, s_off, E, args.n_tiles_n, group_m);
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
      // which rows and output columns this warp's lanes hold
      int32_t r, col0, nseg;
      uint32_t up_off;
      const int32_t h = var == V_HALF1 ? 1 : 0;
      if (tc.m128) {
        r = 64 * static_cast<int32_t>(rank) + 32 * (q & 1) + lane;
        const int32_t nh = q >> 1;       // lanes [64, 128) hold accumulator columns [128, 256)
        if (kSwiglu) {
          col0 = tc.ni * 128 + 64 * nh;
          nseg = 1;
          up_off = 64;
        } else {
          col0 = tc.ni * P_BN + 128 * nh;
          nseg = EPI == MOE_EPI_WEIGHT_SCATTER ? 4 : 2;
          up_off = 0;
        }
      } else {
        r = 128 * static_cast<int32_t>(rank) + 32 * q + lane;
        if (kSwiglu) {
          col0 = tc.ni * 128 + (var != V_WHOLE ? 64 * h : 0);
          nseg = var != V_WHOLE ? 1 : 2;
          up_off = var != V_WHOLE ? 64 : 128;
        } else {
          col0 = tc.ni * P_BN + (var != V_WHOLE ? 128 * h : 0);
          nseg = (EPI == MOE_EPI_WEIGHT_SCATTER ? 8 : 4) / (var != V_WHOLE ? 2 : 1);
          up_off = 0;
        }
      }
      const bool row_ok = r < tc.rows;
      const int32_t s = tc.row0 + r;
      if (EPI == MOE_EPI_WEIGHT_SCATTER) {
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
        epilogue_segments<MOE_EPI_WEIGHT_SCATTER>(t_row, dst, args.n_out - col0, nseg, 0, scale,
                                                  stage_buf, lane);
      } else if (EPI == EPI_SWIGLU_MX) {
        // h columns past F (F an odd multiple of 64: the last column tile is half
        // used) are neither computed nor written
        const int32_t n_left = args.n_out - col0;
        const int ns = n_left >= 64 * nseg ? nseg : (n_left > 0 ? 1 : 0);
        uint8_t* dst = row_ok ? args.q + static_cast<int64_t>(s) * args.ldc + col0 : nullptr;
        const uint32_t codes = ns > 0 ? epilogue_swiglu_mx(t_row, dst, ns, up_off, stage_buf, lane) : 0u;
        if (row_ok) {
          // two scale codes (one 64-column segment) per 16-bit store
          const int32_t kb0 = col0 / 32;
          for (int c = 0; c < ns; ++c) {
            const int32_t kb = kb0 + 2 * c;
            const uint16_t v = static_cast<uint16_t>(codes >> (16 * c));
            uint8_t* p;
            if (args.sf_ld > 0) {
              p = args.sf + static_cast<int64_t>(s) * args.sf_ld + kb;
            } else {
              // group (m-tile gm, 128-row half, 128 columns kb / 4): row i + 32 j of the
              // half and its block b of the group at byte 16 i + 4 j + b
              const int32_t gm = s_tstart[tc.e] / args.n_tiles_n + (tc.row0 - s_off[tc.e]) / P_BM;
              const int32_t ri = r & 127;
              p = args.sf + (static_cast<int64_t>(gm * 2 + (r >> 7)) * args.kg_pad + kb / 4) * 512 +
                  16 * (ri & 31) + 4 * (ri >> 5) + (kb & 3);
            }
            *reinterpret_cast<uint16_t*>(p) = v;
          }
        }
      } else {
        uint8_t* dst = row_ok ? reinterpret_cast<uint8_t*>(args.C + static_cast<int64_t>(s) * args.ldc + col0)
                              : nullptr;
        epilogue_segments<EPI>(t_row, dst, args.n_out - col0, nseg, up_off, 1.0f, stage_buf, lane);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(b == 0 ? te_leader0 : te_leader1);
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the peer no longer touches this CTA's barriers, ring or TMEM
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc2(tmem_base, P_TMEM_COLS);
  }
  if (tid == 0) {
    // the last CTA to finish leaves the queue at zero for the next launch
    __threadfence();
    if (atomicAdd(args.queue + 1, 1) == static_cast<int32_t>(gridDim.x) - 1) {
      atomicExch(args.queue, 0);
      atomicExch(args.queue + 1, 0);
    }
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
static cudaError_t launch2_t(int grid, const CUtensorMap& a, const CUtensorMap& a64,
                             const CUtensorMap& b, const Gemm2Args& args, cudaStream_t stream) {
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
                    P_DYN_SMEM, stream, 2, a, a64, b, args);
}

// Tensor maps, arguments and grid of one launch; false if a tensor map cannot be
// encoded.  `swiglu`: B holds gate | up column halves of N / 2 each.
static bool prepare2(const void* A, const void* B, const int32_t* offsets, int32_t E, int64_t R,
                     int64_t K, int64_t N, bool swiglu, int32_t* status, uint64_t timeout_ns,
                     int num_sms, CUtensorMap* tmA, CUtensorMap* tmA64, CUtensorMap* tmB,
                     Gemm2Args* a, int* grid) {
  const cuuint64_t adims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(R)};
  const cuuint64_t astr[1] = {static_cast<cuuint64_t>(K) * 2};
  const cuuint32_t abox[2] = {64, 128};
  const cuuint32_t abox64[2] = {64, 64};
  const cuuint64_t bdims[3] = {static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(K),
                               static_cast<cuuint64_t>(E)};
  const cuuint64_t bstr[2] = {static_cast<cuuint64_t>(N) * 2, static_cast<cuuint64_t>(K * N) * 2};
  const cuuint32_t bbox[3] = {64, P_BK, 1};
  if (!enc2(tmA, 2, A, adims, astr, abox) || !enc2(tmA64, 2, A, adims, astr, abox64) ||
      !enc2(tmB, 3, B, bdims, bstr, bbox))
    return false;
  *a = Gemm2Args{};
  a->offsets = offsets;
  a->E = E;
  a->R = static_cast<int32_t>(R);
  a->K = static_cast<int32_t>(K);
  a->status = status;
  a->queue = status + 32;
  a->timeout_ns = timeout_ns;
  if (swiglu) {
    a->n_out = static_cast<int32_t>(N / 2);
    a->up_col = static_cast<int32_t>(N / 2);
    a->n_tiles_n = static_cast<int32_t>((N / 2 + 127) / 128);
    a->ldc = N / 2;
  } else {
    a->n_out = static_cast<int32_t>(N);
    a->up_col = 0;
    a->n_tiles_n = static_cast<int32_t>((N + P_BN - 1) / P_BN);
    a->ldc = N;
  }
  const int64_t tiles_max = (R / P_BM + (E < R ? E : R)) * a->n_tiles_n;
  int64_t pairs = num_sms / 2;
  if (2 * tiles_max < pairs) pairs = 2 * tiles_max;   // the last tiles run as two halves
  if (pairs < 1) pairs = 1;
  *grid = static_cast<int>(2 * pairs);
  return true;
}

// Same contract as launch_grouped_gemm (0 ok, 1 tensor map, 2 CUDA error).  `status`
// is the workspace's status word; the tile queue lives at status + 32 (byte 128 of
// the workspace's 256-byte control block).
int launch_grouped_gemm_2sm(const void* A, const void* B, const int32_t* offsets, int32_t E,
                            int64_t R, int64_t K, int64_t N, int epi, const float* w_sorted,
                            const int32_t* perm, void* C, int32_t* status, uint64_t timeout_ns,
                            int num_sms, cudaStream_t stream) {
  if (R == 0) return 0;
  CUtensorMap tmA, tmA64, tmB;
  Gemm2Args a;
  int grid = 0;
  if (!prepare2(A, B, offsets, E, R, K, N, epi == MOE_EPI_SWIGLU, status, timeout_ns, num_sms, &tmA,
                &tmA64, &tmB, &a, &grid))
    return 1;
  a.w_sorted = w_sorted;
  a.perm = perm;
  a.C = static_cast<__nv_bfloat16*>(C);
  a.Cf = static_cast<float*>(C);
  cudaError_t err;
  if (epi == MOE_EPI_SWIGLU)
    err = launch2_t<MOE_EPI_SWIGLU>(grid, tmA, tmA64, tmB, a, stream);
  else if (epi == MOE_EPI_WEIGHT_SCATTER)
    err = launch2_t<MOE_EPI_WEIGHT_SCATTER>(grid, tmA, tmA64, tmB, a, stream);
  else
    err = launch2_t<MOE_EPI_STORE>(grid, tmA, tmA64, tmB, a, stream);
  return err == cudaSuccess ? 0 : 2;
}

// GEMM1 with the SwiGLU + block-scaled E4M3 epilogue: B = W1 [E, K, N2] (gate |
// up), q [R, N2 / 2] codes, sf their scale codes, row-major [R, N2 / 64] when
// sf_row_major, else in the 512-byte groups of the MX down projection (kg_pad
// groups per 128-row block).  Same return contract as launch_grouped_gemm_2sm.
int launch_grouped_gemm_swiglu_mx(const void* A, const void* B, const int32_t* offsets, int32_t E,
                                  int64_t R, int64_t K, int64_t N2, uint8_t* q, uint8_t* sf,
                                  bool sf_row_major, int32_t kg_pad, int32_t* status,
                                  uint64_t timeout_ns, int num_sms, cudaStream_t stream) {
  if (R == 0) return 0;
  CUtensorMap tmA, tmA64, tmB;
  Gemm2Args a;
  int grid = 0;
  if (!prepare2(A, B, offsets, E, R, K, N2, true, status, timeout_ns, num_sms, &tmA, &tmA64, &tmB,
                &a, &grid))
    return 1;
  a.q = q;
  a.sf = sf;
  a.sf_ld = sf_row_major ? static_cast<int32_t>(N2 / 64) : 0;
  a.kg_pad = kg_pad;
  return launch2_t<EPI_SWIGLU_MX>(grid, tmA, tmA64, tmB, a, stream) == cudaSuccess ? 0 : 2;
}

}  // namespace moe
