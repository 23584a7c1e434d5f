// nc_table.cu -- the profiled choice of n_c, the number of memory CTAs beside the
// GEMM CTAs in the single-kernel layer (COMET review, section 4.2.2: several
// precompiled partition points, the best one found by offline profiling and
// stored as metadata, looked up at run time).
//
// The entries are measured with bench.py (--n-c sweep, L2 flushed per step) on
// B200; n_c = 0 selects the five-launch sequence.  A shape that matches no entry
// uses the nearest one of the same (H, F, E, topk) by token count, else 0.
#include <cstdint>
#include <cstdlib>

namespace moe {

namespace {
struct NcEntry {
  int64_t H, F;
  int32_t E, topk;
  int64_t M;
  int32_t n_c;
};

// Measured on B200 (ms per layer step).  Two designs were swept: dedicated
// memory CTAs only (n_c = 0 / 2 / 4 / 8 / 16 / 32, first column of each comment),
// and the current kernel, where six memory warps of every GEMM CTA dispatch and
// combine beside the n_c dedicated CTAs (n_c = 0 / 1 / 2 / 4 / 8, "warps:").  The
// memory warps cut the cost of the single kernel from 4x to 1.1-1.2x the
// five-launch sequence, but it still loses on every shape: the GEMM tiles run
// 3-10 % slower beside the polling memory warps and the dispatch must finish
// before the first GEMM1 wave either way.  Every entry selects the sequence.
// clang-format off
const NcEntry kTable[] = {
    // H     F      E   topk  M      n_c
    {256,   512,    8,  2,    256,   0},  // 0.046 / 0.101 / 0.074 / 0.060 / 0.054 / 0.052; warps: 0.051 / 0.073 / 0.072 / 0.073 / 0.073
    {4096,  14336,  8,  2,    4096,  0},  // 2.12 / 9.31 / 5.25 / 3.49 / 2.72 / 2.96; warps: 2.13 / 2.60 / 2.76 / 2.71 / 2.82
    {2048,  1408,   64, 4,    8192,  0},  // 0.69 / 10.2 / 5.26 / 2.77 / 1.52 / 1.05; warps: 0.668 / 0.743 / 0.744 / 0.782 / 0.872
    {4096,  6400,   16, 2,    16384, 0},  // 4.07 / 34.0 / 17.8 / 10.3 / 6.81 / 5.87
    {7168,  4096,   16, 8,    16,    0},  // 0.474 / 0.563 / 0.513 / 0.511 / 0.521 / 0.534
    {7168,  4096,   16, 8,    128,   0},  // 0.472 / 1.21 / 0.805 / 0.659 / 0.591 / 0.568; warps: 0.488 / 0.574 / 0.574 / 0.572 / 0.580
    {7168,  4096,   16, 8,    512,   0},  // 0.803 / 4.25 / 2.42 / 1.62 / 1.38 / 1.22; warps: 0.817 / 0.936 / 0.979 / 0.999 / 1.021
    {7168,  4096,   16, 8,    2048,  0},  // 2.42 / 16.8 / 8.99 / 5.16 / 3.81 / 3.48
};
// clang-format on
}  // namespace

int32_t profiled_n_c(int64_t M, int64_t H, int64_t F, int32_t E, int32_t topk) {
  const NcEntry* best = nullptr;
  int64_t best_d = 0;
  for (const NcEntry& t : kTable) {
    if (t.H != H || t.F != F || t.E != E || t.topk != topk) continue;
    const int64_t d = std::llabs(t.M - M);
    if (best == nullptr || d < best_d) {
      best = &t;
      best_d = d;
    }
  }
  return best != nullptr ? best->n_c : 0;
}

}  // namespace moe
