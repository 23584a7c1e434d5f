// fused_layer.cu -- the whole layer after the plan in ONE persistent kernel:
// dispatch, GEMM1 + SwiGLU, GEMM2 + gate-weight scatter and combine overlap,
// handing off tile by tile through ready flags in global memory.
//
// This is the single-GPU analogue of COMET's thread-block specialisation (COMET
// review, section 4.2.1): the first n_c CTAs are memory CTAs (dispatch, then
// combine) and the rest are GEMM CTAs with the same warp-specialised tcgen05
// pipeline as grouped_gemm.cu in warps 0-5, plus six memory warps (6-11) that do
// the same dispatch and combine work in the GEMM SMs' idle issue slots; the split
// n_c comes from profiled metadata (section 4.2.2).  The hand-offs follow the shared-tensor decomposition of
// section 4.1.1: dispatch -> GEMM1 per m-tile (tokens are independent along M),
// GEMM1 -> GEMM2 per m-tile once every GEMM1 column block of it is written, and
// GEMM2 -> combine per token once all top-k rows of the token are complete (the
// top-k reduction couples rows, so readiness is counted per row and per token).
// The PTO MegaMoE article describes the same idea with expert-level arrival and
// ready flags instead of global barriers ("MegaMoE 融合算子七阶段").
//
// Work order.  Memory warps claim dispatch items (16 rows of one m-tile) with an
// atomic counter in the order GEMM1 consumes them; GEMM CTAs walk one static list: all GEMM1 tiles
// (expert by expert, n-tile outer, m-tile inner) then all GEMM2 tiles.  Every
// wait is on work that comes earlier in that order and all CTAs are co-resident
// (cooperative launch, one CTA per SM), so the smallest unfinished item can
// always proceed.  Every wait is also bounded: it gives up once no tile anywhere
// has completed for `timeout_ns`, records MOE_ERR_TIMEOUT, raises a global abort
// flag and lets every CTA leave cleanly (in-flight TMA loads landed, MMAs
// drained, TMEM freed).
#include "common.cuh"
#include "epilogue.cuh"

namespace moe {

namespace {

constexpr int L_BM = 128;
constexpr int L_BN = 256;
constexpr int L_BK = 64;
constexpr int L_STAGES = 4;
constexpr int L_THREADS = 384;          // 6 GEMM-role warps + 6 memory warps
constexpr int L_FIRST_MEM_WARP = 6;      // in GEMM CTAs, warps 6..11 do memory work
constexpr int L_GROUP_ROWS = 16;         // rows of one dispatch work item
constexpr int L_GROUPS_PER_MT = 128 / L_GROUP_ROWS;
constexpr int L_A_BYTES = L_BM * L_BK * 2;
constexpr int L_B_BOX_BYTES = L_BK * 64 * 2;
constexpr int L_STAGE_BYTES = L_A_BYTES + 4 * L_B_BOX_BYTES;
constexpr int L_TMEM_COLS = 512;
constexpr int L_DYN_SMEM = L_STAGES * L_STAGE_BYTES + 4 * EPI_STAGE_BYTES_PER_WARP + 1024;
constexpr uint32_t L_IDESC = idesc_bf16_f32(L_BM, L_BN, true);

}  // namespace

// Counters and flags of one launch (zeroed by the host before the launch).
struct LayerSync {
  int32_t* abort;          // [1] any CTA gave up
  int32_t* progress;       // [1] completed work items (tiles, dispatched m-tiles, tokens)
  int32_t* dispatch_head;  // [1] next dispatch item (m-tile, group of 16 rows)
  int32_t* combine_head;   // [1] next slot of the ready list to combine
  int32_t* ready_tail;     // [1] next free slot of the ready list
  int32_t* xp_ready;       // [MT] groups of 16 rows of the m-tile written to Xp
  int32_t* h_done;         // [MT] GEMM1 warps that wrote their rows of h (4 per n-tile)
  int32_t* row_done;       // [R] GEMM2 column tiles written for the row
  int32_t* tok_done;       // [M] complete rows of the token
  int32_t* ready_list;     // [M] token + 1 in completion order (0 = not yet)
};

struct LayerArgs {
  const uint4* x;          // [M, H] bf16
  const int32_t* perm;     // [R]
  const float* w_sorted;   // [R]
  const int32_t* offsets;  // [E + 1]
  uint4* xp;               // [R, H] bf16 (written by memory CTAs, read by TMA)
  __nv_bfloat16* h;        // [R, F] bf16
  float* yk;               // [R, H] fp32, token-major
  uint4* out;              // [M, H] bf16
  int32_t M, H, F, E, topk, R;
  int32_t n_c;
  int32_t nt1, nt2;        // n-tiles of GEMM1 (F / 128) and GEMM2 (H / 256)
  int32_t* status;
  LayerSync sync;
  uint64_t timeout_ns;
  int32_t withhold_mtile;  // fault injection (tests): never publish this m-tile; -1 off
};

struct LTile {
  int32_t e, mt, row0, rows, ni;
};

// Tile t of a list with nt n-tiles per m-tile -> (expert, m-tile, rows, n-tile).
// s_ms[e] = first m-tile of expert e; the tiles of expert e are
// [nt * s_ms[e], nt * s_ms[e+1]), n-tile outer, m-tile inner.
__device__ __forceinline__ LTile decode(int32_t t, int32_t nt, const int32_t* s_ms,
                                        const int32_t* s_off, int32_t E) {
  const int32_t q = t / nt;
  int32_t lo = 0, hi = E;
  while (hi - lo > 1) {
    const int32_t mid = (lo + hi) >> 1;
    if (s_ms[mid] <= q) lo = mid; else hi = mid;
  }
  const int32_t e = lo;
  const int32_t mte = s_ms[e + 1] - s_ms[e];
  const int32_t local = t - nt * s_ms[e];
  LTile c;
  c.e = e;
  c.ni = local / mte;
  const int32_t mi = local - c.ni * mte;
  c.mt = s_ms[e] + mi;
  c.row0 = s_off[e] + mi * L_BM;
  c.rows = min(L_BM, s_off[e + 1] - c.row0);
  return c;
}

// Wait until *flag >= target.  Gives up (false) when the global abort flag is
// raised or when the progress counter has not moved for timeout_ns.
__device__ __forceinline__ bool wait_flag(const int32_t* flag, int32_t target, const LayerSync& sy,
                                          uint64_t timeout_ns, uint32_t max_sleep_ns = 128) {
  if (ld_acquire(flag) >= target) return true;
  uint32_t sleep_ns = 32;
  int32_t last = ld_relaxed(sy.progress);
  uint64_t t0 = globaltimer_ns();
  for (;;) {
    if (ld_acquire(flag) >= target) return true;
    if (ld_relaxed(sy.abort) != 0) return false;
    const int32_t p = ld_relaxed(sy.progress);
    const uint64_t now = globaltimer_ns();
    if (p != last) {
      last = p;
      t0 = now;
    } else if (now - t0 > timeout_ns) {
      return false;
    }
    __nanosleep(sleep_ns);
    if (sleep_ns < max_sleep_ns) sleep_ns *= 2;
  }
}

// mbarrier wait with the same progress-aware limit (a GEMM CTA's stages can
// legitimately sit idle while the producer waits for another CTA's tile).
__device__ __forceinline__ bool mbar_wait_layer(uint64_t* bar, uint32_t parity, const LayerSync& sy,
                                                uint64_t timeout_ns, const volatile int32_t* sabort) {
  const uint32_t addr = smem_u32(bar);
  if (mbar_try_wait(addr, parity)) return true;
  int32_t last = ld_relaxed(sy.progress);
  uint64_t t0 = globaltimer_ns();
  for (uint32_t spin = 1;; ++spin) {
    if (mbar_try_wait(addr, parity)) return true;
    if ((spin & 255u) == 0) {
      if (*sabort != 0 || ld_relaxed(sy.abort) != 0) return false;
      const int32_t p = ld_relaxed(sy.progress);
      const uint64_t now = globaltimer_ns();
      if (p != last) {
        last = p;
        t0 = now;
      } else if (now - t0 > timeout_ns) {
        return false;
      }
    }
  }
}

__device__ __forceinline__ void give_up(const LayerArgs& a, volatile int32_t* sabort) {
  set_status(a.status, MOE_ERR_TIMEOUT);
  atomicExch(a.sync.abort, 1);
  *sabort = 1;
}

// Memory work of one warp: first dispatch items (16 rows of one m-tile, in
// GEMM1's order; the warp that completes a group counts it on the m-tile), then
// combine tokens from the ready list as GEMM2 completes them.  Runs in every warp
// of a memory CTA and in warps 6..11 of every GEMM CTA.
__device__ void memory_warp(const LayerArgs& a, const int32_t* s_ms, const int32_t* s_off,
                            int32_t E, int32_t MT, volatile int32_t* s_abort, int lane) {
  const LayerSync& sy = a.sync;
  const int32_t vpr = a.H / 8;  // 16-byte vectors per bf16 row
  // ---- dispatch
  for (;;) {
    int32_t item = 0;
    if (lane == 0) item = ld_relaxed(sy.abort) != 0 ? MT * L_GROUPS_PER_MT : atomicAdd(sy.dispatch_head, 1);
    item = __shfl_sync(0xffffffffu, item, 0);
    const int32_t mt = item / L_GROUPS_PER_MT;
    if (mt >= MT) break;
    const int32_t grp = item - mt * L_GROUPS_PER_MT;
    int32_t lo = 0, hi = E;
    while (hi - lo > 1) {
      const int32_t mid = (lo + hi) >> 1;
      if (s_ms[mid] <= mt) lo = mid; else hi = mid;
    }
    const int32_t row0 = s_off[lo] + (mt - s_ms[lo]) * L_BM;
    const int32_t rows = min(L_BM, s_off[lo + 1] - row0);
    const int32_t r0 = grp * L_GROUP_ROWS;
    if (r0 >= rows) continue;  // the m-tile is short: this group has no rows
    const int32_t r1 = min(r0 + L_GROUP_ROWS, rows);
    for (int32_t r = r0; r < r1; ++r) {
      const int32_t s = row0 + r;
      const int32_t i = __ldg(a.perm + s);
      uint4* dst = a.xp + static_cast<int64_t>(s) * vpr;
      if (i < 0 || i >= a.R) {
        if (lane == 0) set_status(a.status, MOE_ERR_BAD_INDEX);
        for (int32_t c = lane; c < vpr; c += 32) dst[c] = make_uint4(0, 0, 0, 0);
        continue;
      }
      const uint4* src = a.x + static_cast<int64_t>(i / a.topk) * vpr;
      int32_t c = lane;
      for (; c + 96 < vpr; c += 128) {
        const uint4 v0 = __ldg(src + c), v1 = __ldg(src + c + 32), v2 = __ldg(src + c + 64),
                    v3 = __ldg(src + c + 96);
        dst[c] = v0;
        dst[c + 32] = v1;
        dst[c + 64] = v2;
        dst[c + 96] = v3;
      }
      for (; c < vpr; c += 32) dst[c] = __ldg(src + c);
    }
    __syncwarp();
    if (lane == 0 && mt != a.withhold_mtile) {
      __threadfence();
      fence_proxy_async_global();  // the rows are read next by TMA (async proxy)
      red_release_add(sy.xp_ready + mt, 1);
      red_release_add(sy.progress, 1);
    }
  }
  // ---- combine, token by token as tokens complete
  const int32_t steps = (vpr + 31) / 32;
  for (;;) {
    int32_t idx = 0;
    if (lane == 0) idx = atomicAdd(sy.combine_head, 1);
    idx = __shfl_sync(0xffffffffu, idx, 0);
    if (idx >= a.M) break;
    int32_t v = 0;
    if (lane == 0)
      v = wait_flag(sy.ready_list + idx, 1, sy, a.timeout_ns, 2048) ? ld_acquire(sy.ready_list + idx)
                                                                    : 0;
    v = __shfl_sync(0xffffffffu, v, 0);
    if (v <= 0) {
      if (lane == 0 && ld_relaxed(sy.abort) == 0) give_up(a, s_abort);
      break;
    }
    const int32_t t = v - 1;
    const float4* yrow = reinterpret_cast<const float4*>(a.yk) + static_cast<int64_t>(t) * a.topk * (a.H / 4);
    for (int32_t q = 0; q < steps; ++q) {
      const int32_t c = q * 32 + lane;  // group of 8 columns
      if (c >= vpr) break;
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      for (int32_t k = 0; k < a.topk; ++k) {
        const float4* p = yrow + static_cast<int64_t>(k) * (a.H / 4) + 2 * c;
        const float4 u0 = __ldcg(p), u1 = __ldcg(p + 1);
        acc[0] += u0.x; acc[1] += u0.y; acc[2] += u0.z; acc[3] += u0.w;
        acc[4] += u1.x; acc[5] += u1.y; acc[6] += u1.z; acc[7] += u1.w;
      }
      uint4 o;
      o.x = pack_bf16x2(acc[0], acc[1]);
      o.y = pack_bf16x2(acc[2], acc[3]);
      o.z = pack_bf16x2(acc[4], acc[5]);
      o.w = pack_bf16x2(acc[6], acc[7]);
      a.out[static_cast<int64_t>(t) * vpr + c] = o;
    }
    if (lane == 0) red_release_add(sy.progress, 1);
  }
}

__global__ void __launch_bounds__(L_THREADS, 1)
    moe_layer_kernel(const __grid_constant__ CUtensorMap tmXp,
                     const __grid_constant__ CUtensorMap tmW1,
                     const __grid_constant__ CUtensorMap tmH,
                     const __grid_constant__ CUtensorMap tmW2, const LayerArgs a) {
  extern __shared__ uint8_t l_dyn_smem[];
  __shared__ __align__(8) uint64_t full_bar[L_STAGES];
  __shared__ __align__(8) uint64_t empty_bar[L_STAGES];
  __shared__ __align__(8) uint64_t tfull_bar[2];
  __shared__ __align__(8) uint64_t tempty_bar[2];
  __shared__ __align__(8) uint64_t drain_bar;
  __shared__ uint32_t s_tmem_base;
  __shared__ volatile int32_t s_abort;
  __shared__ int32_t s_plan_ok;
  __shared__ int32_t s_off[MOE_MAX_EXPERTS + 1];
  __shared__ int32_t s_ms[MOE_MAX_EXPERTS + 1];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int32_t E = a.E;
  const bool memory_cta = static_cast<int32_t>(blockIdx.x) < a.n_c;
  uint8_t* ring = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(l_dyn_smem) + 1023) & ~static_cast<uintptr_t>(1023));

  if (tid == 0) {
    for (int s = 0; s < L_STAGES; ++s) {
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
  if (!memory_cta && warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmXp);
    tma_prefetch_desc(&tmW1);
    tma_prefetch_desc(&tmH);
    tma_prefetch_desc(&tmW2);
  }
  if (!memory_cta && warp == 1) {
    tmem_alloc(&s_tmem_base, L_TMEM_COLS);
    tmem_relinquish();
  }
  for (int e = tid; e <= E; e += L_THREADS) s_off[e] = a.offsets[e];
  __syncthreads();
  if (warp == 0) {
    // m-tile starts per expert; offsets inconsistent with R (a failed plan) leave
    // every list empty and the kernel does nothing.
    int32_t bad = (s_off[0] != 0 || s_off[E] != a.R) ? 1 : 0;
    for (int e = lane; e < E; e += 32)
      if (s_off[e + 1] < s_off[e]) bad = 1;
    bad = __any_sync(0xffffffffu, bad);
    int32_t run = 0;
    for (int base = 0; base < E; base += 32) {
      const int e = base + lane;
      const int32_t m = (e < E && !bad) ? (s_off[e + 1] - s_off[e] + L_BM - 1) / L_BM : 0;
      int32_t incl = m;
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const int32_t v = __shfl_up_sync(0xffffffffu, incl, d);
        if (lane >= d) incl += v;
      }
      if (e < E) s_ms[e] = run + incl - m;
      run += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) {
      s_ms[E] = run;
      s_plan_ok = bad ? 0 : 1;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const int32_t MT = s_ms[E];
  const LayerSync& sy = a.sync;

  if (memory_cta) {
    // ================================================================ memory CTA
    if (s_plan_ok) memory_warp(a, s_ms, s_off, E, MT, &s_abort, lane);
    return;  // no TMEM, no outstanding async copies
  }

  // ================================================================== GEMM CTA
  const int32_t g = static_cast<int32_t>(blockIdx.x) - a.n_c;
  const int32_t G = static_cast<int32_t>(gridDim.x) - a.n_c;
  const int32_t T1 = MT * a.nt1;
  const int32_t T = T1 + MT * a.nt2;
  const uint32_t tmem_base = s_tmem_base;

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ TMA producer
    uint32_t stage = 0, phase = 0, issued = 0;
    for (int32_t t = g; t < T && !s_abort; t += G) {
      const bool two = t >= T1;
      const LTile tc = two ? decode(t - T1, a.nt2, s_ms, s_off, E) : decode(t, a.nt1, s_ms, s_off, E);
      const bool ok = two ? wait_flag(sy.h_done + tc.mt, 4 * a.nt1, sy, a.timeout_ns)
                          : wait_flag(sy.xp_ready + tc.mt, (tc.rows + L_GROUP_ROWS - 1) / L_GROUP_ROWS,
                                      sy, a.timeout_ns);
      if (!ok) {
        give_up(a, &s_abort);
        break;
      }
      fence_proxy_async_global();  // generic-proxy writes of other CTAs -> TMA reads
      const int32_t KB = (two ? a.F : a.H) / L_BK;
      for (int32_t kb = 0; kb < KB; ++kb) {
        if (!mbar_wait_layer(&empty_bar[stage], phase ^ 1u, sy, a.timeout_ns, &s_abort)) {
          give_up(a, &s_abort);
          break;
        }
        uint8_t* sa = ring + stage * L_STAGE_BYTES;
        uint8_t* sb = sa + L_A_BYTES;
        mbar_arrive_expect_tx(&full_bar[stage], L_STAGE_BYTES);
        if (!two) {
          tma_load_2d(sa, &tmXp, &full_bar[stage], kb * L_BK, tc.row0);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int32_t n = (j < 2) ? tc.ni * 128 + 64 * j : a.F + tc.ni * 128 + 64 * (j - 2);
            tma_load_3d(sb + j * L_B_BOX_BYTES, &tmW1, &full_bar[stage], n, kb * L_BK, tc.e);
          }
        } else {
          tma_load_2d(sa, &tmH, &full_bar[stage], kb * L_BK, tc.row0);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            tma_load_3d(sb + j * L_B_BOX_BYTES, &tmW2, &full_bar[stage], tc.ni * L_BN + 64 * j,
                        kb * L_BK, tc.e);
        }
        ++issued;
        if (++stage == L_STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    if (s_abort) {
      uint32_t st = stage, ph = phase;
      for (uint32_t q = 0; q < L_STAGES && q < issued; ++q) {
        if (st == 0) {
          st = L_STAGES - 1;
          ph ^= 1u;
        } else {
          --st;
        }
        mbar_wait_bounded(&full_bar[st], ph, a.timeout_ns, nullptr);
      }
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    uint32_t stage = 0, phase = 0, j = 0;
    bool issued_any = false;
    for (int32_t t = g; t < T && !s_abort; t += G, ++j) {
      const uint32_t b = j & 1u, tph = (j >> 1) & 1u;
      if (!mbar_wait_layer(&tempty_bar[b], tph ^ 1u, sy, a.timeout_ns, &s_abort)) {
        give_up(a, &s_abort);
        break;
      }
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + b * L_BN;
      const int32_t KB = (t >= T1 ? a.F : a.H) / L_BK;
      for (int32_t kb = 0; kb < KB; ++kb) {
        if (!mbar_wait_layer(&full_bar[stage], phase, sy, a.timeout_ns, &s_abort)) {
          give_up(a, &s_abort);
          break;
        }
        tc_fence_after();
        const uint32_t a_addr = smem_u32(ring + stage * L_STAGE_BYTES);
        const uint32_t b_addr = a_addr + L_A_BYTES;
#pragma unroll
        for (int kk = 0; kk < L_BK / 16; ++kk) {
          const uint64_t adesc = smem_desc_sw128(a_addr + kk * 32, 16, 1024);
          const uint64_t bdesc = smem_desc_sw128(b_addr + kk * 2048, 8192, 1024);
          umma_bf16(d_tmem, adesc, bdesc, L_IDESC, (kb | kk) != 0 ? 1u : 0u);
        }
        issued_any = true;
        umma_commit(&empty_bar[stage]);
        if (++stage == L_STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (s_abort) break;
      umma_commit(&tfull_bar[b]);
    }
    if (s_abort && issued_any) {
      umma_commit(&drain_bar);
      mbar_wait_bounded(&drain_bar, 0, a.timeout_ns, nullptr);
    }
  } else if (warp >= L_FIRST_MEM_WARP) {
    // ------------------------------------------------------------ memory warps
    if (s_plan_ok) memory_warp(a, s_ms, s_off, E, MT, &s_abort, lane);
  } else if (warp >= 2) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const int r = q * 32 + lane;
    uint4* stage_buf = reinterpret_cast<uint4*>(ring + L_STAGES * L_STAGE_BYTES +
                                                (warp - 2) * EPI_STAGE_BYTES_PER_WARP);
    uint32_t j = 0;
    for (int32_t t = g; t < T; t += G, ++j) {
      const bool two = t >= T1;
      const LTile tc = two ? decode(t - T1, a.nt2, s_ms, s_off, E) : decode(t, a.nt1, s_ms, s_off, E);
      const uint32_t b = j & 1u, tph = (j >> 1) & 1u;
      // one lane waits, the warp follows its result (keeps the warp's decision uniform)
      int32_t okw = 1;
      if (lane == 0) okw = mbar_wait_layer(&tfull_bar[b], tph, sy, a.timeout_ns, &s_abort) ? 1 : 0;
      okw = __shfl_sync(0xffffffffu, okw, 0);
      if (!okw) {
        if (lane == 0 && ld_relaxed(sy.abort) == 0) give_up(a, &s_abort);
        break;
      }
      __syncwarp();
      tc_fence_after();
      const uint32_t t_row = tmem_base + b * L_BN + (static_cast<uint32_t>(q * 32) << 16);
      const bool row_ok = r < tc.rows;
      const int32_t s = tc.row0 + r;
      if (!two) {
        const int32_t col0 = tc.ni * 128;
        uint8_t* dst = row_ok ? reinterpret_cast<uint8_t*>(a.h + static_cast<int64_t>(s) * a.F + col0)
                              : nullptr;
        epilogue_tile<MOE_EPI_SWIGLU>(t_row, dst, a.F - col0, 1.0f, stage_buf, lane);
        tc_fence_before();
        mbar_arrive(&tempty_bar[b]);
        // publish this warp's 32 rows of the m-tile's column block
        __syncwarp();
        if (lane == 0) {
          __threadfence();
          fence_proxy_async_global();  // read next by TMA (async proxy)
          red_release_add(sy.h_done + tc.mt, 1);
          if (q == 2) red_release_add(sy.progress, 1);
        }
      } else {
        const int32_t col0 = tc.ni * L_BN;
        float scale = 1.0f;
        int32_t dest = -1;
        if (row_ok) {
          dest = __ldg(a.perm + s);
          scale = __ldg(a.w_sorted + s);
          if (dest < 0 || dest >= a.R) {
            set_status(a.status, MOE_ERR_BAD_INDEX);
            dest = -1;
          }
        }
        uint8_t* dst = dest >= 0 ? reinterpret_cast<uint8_t*>(a.yk + static_cast<int64_t>(dest) * a.H + col0)
                                 : nullptr;
        epilogue_tile<MOE_EPI_WEIGHT_SCATTER>(t_row, dst, a.H - col0, scale, stage_buf, lane);
        tc_fence_before();
        mbar_arrive(&tempty_bar[b]);
        // The warp wrote its rows' segments cooperatively: order them before the
        // per-row completion counts of the lanes that own the rows.
        __syncwarp();
        if (dest >= 0) {
          // row complete once all nt2 column tiles wrote it; token complete once
          // all its topk rows are complete
          __threadfence();
          if (atomicAdd(sy.row_done + s, 1) == a.nt2 - 1) {
            __threadfence();
            const int32_t tok = dest / a.topk;
            if (atomicAdd(sy.tok_done + tok, 1) == a.topk - 1) {
              __threadfence();
              const int32_t pos = atomicAdd(sy.ready_tail, 1);
              st_release(sy.ready_list + pos, tok + 1);
            }
          }
        }
        __syncwarp();
        if (lane == 0 && q == 2) red_release_add(sy.progress, 1);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, L_TMEM_COLS);
  }
}

// ---------------------------------------------------------------- host side

static bool enc2d(CUtensorMap* m, const void* base, int64_t rows, int64_t cols) {
  const TensorMapEncodeFn enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
  cuuint32_t box[2] = {64, static_cast<cuuint32_t>(L_BM)};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static bool enc3d(CUtensorMap* m, const void* base, int64_t E, int64_t K, int64_t N) {
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

// Bytes of the sync area for R rows, M tokens, E experts (all int32, zeroed per launch).
size_t layer_sync_bytes(int64_t M, int64_t R, int32_t E) {
  const int64_t mt_max = R / L_BM + E + 1;
  return size_t(64 + 2 * mt_max + R + 2 * M) * 4;
}

// Returns 0 on success, 1 if a tensor map could not be encoded, 2 on a CUDA error,
// 3 if the grid cannot be co-resident (cooperative launch refused).
int launch_moe_layer(const void* x, const void* W1, const void* W2, const int32_t* perm,
                     const float* w_sorted, const int32_t* offsets, void* xp, void* h, void* yk,
                     void* out, int64_t M, int64_t H, int64_t F, int32_t E, int32_t topk,
                     int32_t n_c, int32_t* status, void* sync_area, uint64_t timeout_ns,
                     int32_t withhold_mtile, int num_sms, cudaStream_t stream) {
  const int64_t R = M * topk;
  if (R == 0) return 0;
  CUtensorMap tmXp, tmW1, tmH, tmW2;
  if (!enc2d(&tmXp, xp, R, H) || !enc3d(&tmW1, W1, E, H, 2 * F) || !enc2d(&tmH, h, R, F) ||
      !enc3d(&tmW2, W2, E, F, H))
    return 1;
  const int64_t mt_max = R / L_BM + E + 1;
  int32_t* base = static_cast<int32_t*>(sync_area);
  LayerArgs a;
  a.x = static_cast<const uint4*>(x);
  a.perm = perm;
  a.w_sorted = w_sorted;
  a.offsets = offsets;
  a.xp = static_cast<uint4*>(xp);
  a.h = static_cast<__nv_bfloat16*>(h);
  a.yk = static_cast<float*>(yk);
  a.out = static_cast<uint4*>(out);
  a.M = static_cast<int32_t>(M);
  a.H = static_cast<int32_t>(H);
  a.F = static_cast<int32_t>(F);
  a.E = E;
  a.topk = topk;
  a.R = static_cast<int32_t>(R);
  a.n_c = n_c;
  a.nt1 = static_cast<int32_t>((F + 127) / 128);
  a.nt2 = static_cast<int32_t>((H + L_BN - 1) / L_BN);
  a.status = status;
  a.sync.abort = base + 0;
  a.sync.progress = base + 1;
  a.sync.dispatch_head = base + 2;
  a.sync.combine_head = base + 3;
  a.sync.ready_tail = base + 4;
  a.sync.xp_ready = base + 64;
  a.sync.h_done = base + 64 + mt_max;
  a.sync.row_done = base + 64 + 2 * mt_max;
  a.sync.tok_done = base + 64 + 2 * mt_max + R;
  a.sync.ready_list = base + 64 + 2 * mt_max + R + M;
  a.timeout_ns = timeout_ns;
  a.withhold_mtile = withhold_mtile;

  cudaError_t err = cudaMemsetAsync(sync_area, 0, layer_sync_bytes(M, R, E), stream);
  if (err != cudaSuccess) return 2;
  static PerDeviceOnce once;
  err = once.run([] {
    return cudaFuncSetAttribute(moe_layer_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                L_DYN_SMEM);
  });
  if (err != cudaSuccess) return 2;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(num_sms));
  cfg.blockDim = dim3(L_THREADS);
  cfg.dynamicSmemBytes = L_DYN_SMEM;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  err = cudaLaunchKernelEx(&cfg, moe_layer_kernel, tmXp, tmW1, tmH, tmW2, a);
  if (err == cudaErrorCooperativeLaunchTooLarge) return 3;
  return err == cudaSuccess ? 0 : 2;
}

}  // namespace moe
