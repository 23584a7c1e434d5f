// epilogue.cuh -- coalesced row stores for the GEMM epilogues.
//
// After tcgen05.ld every epilogue thread holds a piece of ONE output row (TMEM
// lane = row), so storing straight from registers makes each warp store touch 32
// different rows with 16 bytes each: 32 partial-line transactions per
// instruction.  Instead each warp passes its 32 row segments of 128 bytes
// through a 4 KB shared-memory buffer and writes them back four rows per
// instruction: eight lanes cover one row's 128 contiguous bytes, so every store
// instruction writes four full 128-byte lines.
//
// The buffer is XOR-swizzled in 16-byte units (slot j of row r lives at
// r * 8 + (j ^ (r & 7))), so both the row-wise writes and the column-wise reads
// are free of bank conflicts.
#pragma once

#include <cuda_fp8.h>

#include "common.cuh"

namespace moe {

// Bytes of staging buffer per epilogue warp.
constexpr int EPI_STAGE_BYTES_PER_WARP = 32 * 128;

// `seg` is this thread's 128-byte row segment; `dst` where it goes (nullptr: the
// row is not written).  `buf` is this warp's staging buffer (256 x 16 B).
__device__ __forceinline__ void warp_store_rows128(const uint4 (&seg)[8], uint8_t* dst, uint4* buf,
                                                   int lane) {
  __syncwarp();
#pragma unroll
  for (int j = 0; j < 8; ++j) buf[lane * 8 + (j ^ (lane & 7))] = seg[j];
  __syncwarp();
  const unsigned long long mine = reinterpret_cast<unsigned long long>(dst);
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    const int row = it * 4 + (lane >> 3);
    const int c16 = lane & 7;
    const unsigned long long d = __shfl_sync(0xffffffffu, mine, row);
    const uint4 v = buf[row * 8 + (c16 ^ (row & 7))];
    if (d != 0ull) reinterpret_cast<uint4*>(d)[c16] = v;
  }
}

// The same for 64-byte row segments (slot j of row r at r * 4 + (j ^ ((r >> 1) & 3)):
// conflict-free both ways); four lanes cover one row's 64 bytes, eight rows per
// store instruction.
__device__ __forceinline__ void warp_store_rows64(const uint4* seg, uint8_t* dst, uint4* buf, int lane) {
  __syncwarp();
#pragma unroll
  for (int j = 0; j < 4; ++j) buf[lane * 4 + (j ^ ((lane >> 1) & 3))] = seg[j];
  __syncwarp();
  const unsigned long long mine = reinterpret_cast<unsigned long long>(dst);
#pragma unroll
  for (int it = 0; it < 4; ++it) {
    const int row = it * 8 + (lane >> 2);
    const int c16 = lane & 3;
    const unsigned long long d = __shfl_sync(0xffffffffu, mine, row);
    const uint4 v = buf[row * 4 + (c16 ^ ((row >> 1) & 3))];
    if (d != 0ull) reinterpret_cast<uint4*>(d)[c16] = v;
  }
}

__device__ __forceinline__ void pack8_bf16(const float* v, float scale, uint4& out) {
  out.x = pack_bf16x2(v[0] * scale, v[1] * scale);
  out.y = pack_bf16x2(v[2] * scale, v[3] * scale);
  out.z = pack_bf16x2(v[4] * scale, v[5] * scale);
  out.w = pack_bf16x2(v[6] * scale, v[7] * scale);
}

__device__ __forceinline__ float silu_fast(float g) { return g / (1.0f + __expf(-g)); }

// SwiGLU of 8 gate/up pairs -> 8 bf16.
__device__ __forceinline__ void pack8_swiglu(const float* g, const float* u, uint4& out) {
  out.x = pack_bf16x2(silu_fast(g[0]) * u[0], silu_fast(g[1]) * u[1]);
  out.y = pack_bf16x2(silu_fast(g[2]) * u[2], silu_fast(g[3]) * u[3]);
  out.z = pack_bf16x2(silu_fast(g[4]) * u[4], silu_fast(g[5]) * u[5]);
  out.w = pack_bf16x2(silu_fast(g[6]) * u[6], silu_fast(g[7]) * u[7]);
}

// ---------------------------------------------------------------- block-scaled E4M3 (MX)
// Blocks of 32 consecutive h values of a row share one power-of-two scale 2^e, e
// the smallest integer with amax <= 448 * 2^e (448: the largest E4M3 value),
// stored as the E8M0 code e + 127; the elements are q = E4M3(v * 2^-e), nearest,
// ties to even.  (The PTO MegaMoE article, section "MegaMoE 融合算子七阶段": SwiGLU
// quantises each segment it consumes; the block size and scale format are those of
// the tcgen05 block-scaled MMA.)

// e of a block with largest magnitude `amax` >= 0, clamped to [-127, 127] (-127
// for an all-zero block), from the bits of amax = m * 2^p, m in [1, 2): since
// 448 = 1.75 * 2^8, e = p - 8 when m <= 1.75, else p - 7.  Below 2^-126 (zero or
// subnormal) e would be at most -134, which clamps to -127.
__device__ __forceinline__ int mx_exponent_of(float amax) {
  const uint32_t b = __float_as_uint(amax);
  const int biased = static_cast<int>(b >> 23);
  if (biased == 0) return -127;
  const int e = biased - 127 - 8 + ((b & 0x7FFFFFu) > 0x600000u ? 1 : 0);
  return e < -127 ? -127 : (e > 127 ? 127 : e);
}

__device__ __forceinline__ uint32_t e4m3x4(float a, float b, float c, float d) {
  return static_cast<uint32_t>(__nv_cvt_float_to_fp8(a, __NV_SATFINITE, __NV_E4M3)) |
         (static_cast<uint32_t>(__nv_cvt_float_to_fp8(b, __NV_SATFINITE, __NV_E4M3)) << 8) |
         (static_cast<uint32_t>(__nv_cvt_float_to_fp8(c, __NV_SATFINITE, __NV_E4M3)) << 16) |
         (static_cast<uint32_t>(__nv_cvt_float_to_fp8(d, __NV_SATFINITE, __NV_E4M3)) << 24);
}

// 32 values -> their 32 codes (value i in byte i of lo:hi) and the block's scale
// code e + 127 (returned).  v * 2^-e is exact in fp32 (a power-of-two scaling
// that stays at or below 448), so the only rounding is the E4M3 one.
__device__ __forceinline__ uint32_t mx_block32(const float* v, uint4& lo, uint4& hi) {
  float m = 0.0f;
#pragma unroll
  for (int i = 0; i < 32; ++i) m = fmaxf(m, fabsf(v[i]));
  const int e = mx_exponent_of(m);
  const int es = e > 126 ? 126 : e;
  const float s = __uint_as_float(static_cast<uint32_t>(127 - es) << 23);  // 2^-e
  uint32_t w[8];
#pragma unroll
  for (int k = 0; k < 8; ++k)
    w[k] = e4m3x4(v[4 * k] * s, v[4 * k + 1] * s, v[4 * k + 2] * s, v[4 * k + 3] * s);
  lo = make_uint4(w[0], w[1], w[2], w[3]);
  hi = make_uint4(w[4], w[5], w[6], w[7]);
  return static_cast<uint32_t>(e + 127);
}

// SwiGLU + block-scaled E4M3 of `nseg` (1 or 2) segments of 64 h columns of this
// warp's 32 rows: segment c takes gate columns [64c, 64c + 64) and up columns
// up_off + [64c, 64c + 64) of the accumulator and holds two blocks of 32 h values.
// The 64 * nseg code bytes of a row go to row_dst (nullptr: not written).
// Returns the scale codes of the 2 * nseg blocks, block b in byte b.
// Warp-collective.
__device__ __forceinline__ uint32_t epilogue_swiglu_mx(uint32_t t_row, uint8_t* row_dst, int nseg,
                                                       uint32_t up_off, uint4* buf, int lane) {
  uint4 seg[8];
  uint32_t codes = 0;
#pragma unroll
  for (int c = 0; c < 2; ++c) {
    if (c >= nseg) break;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      float g[32], u[32];
      tmem_ld32(t_row + c * 64 + half * 32, g);
      tmem_ld32(t_row + up_off + c * 64 + half * 32, u);
      tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < 32; ++i) g[i] = silu_fast(g[i]) * u[i];
      const uint32_t code = mx_block32(g, seg[4 * c + 2 * half], seg[4 * c + 2 * half + 1]);
      codes |= code << (8 * (2 * c + half));
    }
  }
  if (nseg == 2)
    warp_store_rows128(seg, row_dst, buf, lane);
  else
    warp_store_rows64(seg, row_dst, buf, lane);
  return codes;
}

// The epilogue of `nseg` 128-byte output segments of this warp's 32 rows:
//   EPI = MOE_EPI_STORE           segment c: bf16 of accumulator cols [64c, 64c + 64)
//         MOE_EPI_SWIGLU          segment c: bf16 silu(gate) * up of gate cols
//                                 [64c, 64c + 64) and up cols up_off + [64c, 64c + 64)
//         MOE_EPI_WEIGHT_SCATTER  segment c: fp32 of accumulator cols [32c, 32c + 32) * scale
// t_row: TMEM address of this warp's lanes, first accumulator column; row_dst: byte
// address of this thread's output row at the warp's first output column (nullptr:
// the row is not written); n_left: output columns from there to the end of the
// row (segments past it are skipped).  Warp-collective.
template <int EPI>
__device__ __forceinline__ void epilogue_segments(uint32_t t_row, uint8_t* row_dst, int32_t n_left,
                                                  int nseg, uint32_t up_off, float scale,
                                                  uint4* buf, int lane) {
#pragma unroll 1
  for (int c = 0; c < nseg; ++c) {
    uint4 seg[8];
    if (EPI == MOE_EPI_SWIGLU) {
      float g[32], u[32];
      tmem_ld32(t_row + c * 64, g);
      tmem_ld32(t_row + up_off + c * 64, u);
      tmem_ld_wait();
#pragma unroll
      for (int q = 0; q < 4; ++q) pack8_swiglu(g + 8 * q, u + 8 * q, seg[q]);
      tmem_ld32(t_row + c * 64 + 32, g);
      tmem_ld32(t_row + up_off + c * 64 + 32, u);
      tmem_ld_wait();
#pragma unroll
      for (int q = 0; q < 4; ++q) pack8_swiglu(g + 8 * q, u + 8 * q, seg[4 + q]);
    } else if (EPI == MOE_EPI_STORE) {
      float v[32];
      tmem_ld32(t_row + c * 64, v);
      tmem_ld_wait();
#pragma unroll
      for (int q = 0; q < 4; ++q) pack8_bf16(v + 8 * q, 1.0f, seg[q]);
      tmem_ld32(t_row + c * 64 + 32, v);
      tmem_ld_wait();
#pragma unroll
      for (int q = 0; q < 4; ++q) pack8_bf16(v + 8 * q, 1.0f, seg[4 + q]);
    } else {
      float v[32];
      tmem_ld32(t_row + c * 32, v);
      tmem_ld_wait();
#pragma unroll
      for (int q = 0; q < 8; ++q)
        seg[q] = make_uint4(__float_as_uint(v[4 * q] * scale), __float_as_uint(v[4 * q + 1] * scale),
                            __float_as_uint(v[4 * q + 2] * scale),
                            __float_as_uint(v[4 * q + 3] * scale));
    }
    const int32_t seg_cols = EPI == MOE_EPI_WEIGHT_SCATTER ? 32 : 64;
    uint8_t* d = (row_dst != nullptr && c * seg_cols < n_left) ? row_dst + c * 128 : nullptr;
    warp_store_rows128(seg, d, buf, lane);
  }
}

// The epilogue of one 128-row accumulator tile (this warp: 32 of the rows).
//   EPI = MOE_EPI_STORE           bf16 C[row, col0 + 0..255]     (4 segments)
//         MOE_EPI_SWIGLU          bf16 C[row, col0 + 0..127] from gate cols
//                                 0..127 and up cols 128..255    (2 segments)
//         MOE_EPI_WEIGHT_SCATTER  fp32 C[dest, col0 + 0..255] * scale (8 segments)
// t_row: TMEM address of this warp's lanes, accumulator column 0.
// row_dst: byte address of this thread's output row at column col0 (nullptr: the
// row is not written); n_left: output columns from col0 to the end of the row
// (segments past it are skipped, n_left is a multiple of 64).
template <int EPI>
__device__ __forceinline__ void epilogue_tile(uint32_t t_row, uint8_t* row_dst, int32_t n_left,
                                              float scale, uint4* buf, int lane) {
  if (EPI == MOE_EPI_SWIGLU) {
#pragma unroll 1
    for (int c = 0; c < 2; ++c) {  // 64 output columns = 128 bytes per segment
      float g[32], u[32];
      uint4 seg[8];
      tmem_ld32(t_row + c * 64, g);
      tmem_ld32(t_row + 128 + c * 64, u);
      tmem_ld_wait();
#pragma unroll
      for (int q = 0; q < 4; ++q) pack8_swiglu(g + 8 * q, u + 8 * q, seg[q]);
      tmem_ld32(t_row + c * 64 + 32, g);
      tmem_ld32(t_row + 128 + c * 64 + 32, u);
      tmem_ld_wait();
#pragma unroll
      for (int q = 0; q < 4; ++q) pack8_swiglu(g + 8 * q, u + 8 * q, seg[4 + q]);
      uint8_t* d = (row_dst != nullptr && c * 64 < n_left) ? row_dst + c * 128 : nullptr;
      warp_store_rows128(seg, d, buf, lane);
    }
  } else if (EPI == MOE_EPI_STORE) {
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {  // 64 bf16 columns per segment
      float v[32];
      uint4 seg[8];
      tmem_ld32(t_row + c * 64, v);
      tmem_ld_wait();
#pragma unroll
      for (int q = 0; q < 4; ++q) pack8_bf16(v + 8 * q, 1.0f, seg[q]);
      tmem_ld32(t_row + c * 64 + 32, v);
      tmem_ld_wait();
#pragma unroll
      for (int q = 0; q < 4; ++q) pack8_bf16(v + 8 * q, 1.0f, seg[4 + q]);
      uint8_t* d = (row_dst != nullptr && c * 64 < n_left) ? row_dst + c * 128 : nullptr;
      warp_store_rows128(seg, d, buf, lane);
    }
  } else {
#pragma unroll 1
    for (int c = 0; c < 8; ++c) {  // 32 fp32 columns per segment
      float v[32];
      uint4 seg[8];
      tmem_ld32(t_row + c * 32, v);
      tmem_ld_wait();
#pragma unroll
      for (int q = 0; q < 8; ++q)
        seg[q] = make_uint4(__float_as_uint(v[4 * q] * scale), __float_as_uint(v[4 * q + 1] * scale),
                            __float_as_uint(v[4 * q + 2] * scale),
                            __float_as_uint(v[4 * q + 3] * scale));
      uint8_t* d = (row_dst != nullptr && c * 32 < n_left) ? row_dst + c * 128 : nullptr;
      warp_store_rows128(seg, d, buf, lane);
    }
  }
}

}  // namespace moe
