// Device helpers: number formats, warp reductions and the warp-resident
// Walsh-Hadamard transform.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "tq_internal.h"

#define TQ_FULL 0xffffffffu

__device__ __forceinline__ float tq_load_elem(const void *p, int64_t i, int dtype) {
  if (dtype == TQ_BF16) {
    const uint16_t b = reinterpret_cast<const uint16_t *>(p)[i];
    return __uint_as_float(static_cast<uint32_t>(b) << 16);
  }
  return reinterpret_cast<const float *>(p)[i];
}

__device__ __forceinline__ float tq_bf16_to_f32(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

__device__ __forceinline__ float tq_half_to_f32(uint16_t h) {
  return __half2float(__ushort_as_half(h));
}

__device__ __forceinline__ uint16_t tq_f32_to_half(float f) {
  return __half_as_ushort(__float2half_rn(f));
}

__device__ __forceinline__ float tq_warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(TQ_FULL, v, o);
  return v;
}

__device__ __forceinline__ float tq_warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(TQ_FULL, v, o));
  return v;
}

// Unnormalised Walsh-Hadamard transform (Sylvester / natural order) of a
// d-vector held by one warp with coordinate i = lane + 32 k in x[k],
// k < NPL = d / 32.  Output y = H_d x.
// FMA = true does each shuffle stage as one fma with a +-1 factor (fewer
// instructions, identical results; the factors take registers).
template <int NPL, bool FMA = false>
__device__ __forceinline__ void tq_warp_wht(float (&x)[NPL], int lane) {
  // strides 1..16: lane bits, exchanged with shuffles
#pragma unroll
  for (int s = 1; s < 32; s <<= 1) {
    const bool upper = lane & s;
    const float sg = upper ? -1.f : 1.f;
#pragma unroll
    for (int k = 0; k < NPL; ++k) {
      const float o = __shfl_xor_sync(TQ_FULL, x[k], s);
      // o - x or x + o: one rounding either way
      x[k] = FMA ? fmaf(sg, x[k], o) : (upper ? (o - x[k]) : (x[k] + o));
    }
  }
  // strides 32, 64, ...: register index bits
#pragma unroll
  for (int s = 1; s < NPL; s <<= 1) {
#pragma unroll
    for (int k = 0; k < NPL; ++k) {
      if (!(k & s)) {
        const float a = x[k], b = x[k + s];
        x[k] = a + b;
        x[k + s] = a - b;
      }
    }
  }
}

// x_i *= D_i for coordinate i = lane + 32 k (dneg bit set <=> D_i = -1).
template <int NPL>
__device__ __forceinline__ void tq_apply_signs(float (&x)[NPL], const uint32_t *dneg, int lane) {
#pragma unroll
  for (int k = 0; k < NPL; ++k) {
    const uint32_t neg = (dneg[k] >> lane) & 1u;
    x[k] = __uint_as_float(__float_as_uint(x[k]) ^ (neg << 31));
  }
}

// Code of u: #{k : u >= t_k} for ascending thresholds t[0 .. 2^STEPS - 2]
// (STEPS <= 4) whose later slots hold +inf (the codec pads them): a
// branch-free binary search of STEPS steps (the count is the same as a
// linear scan's), valid for every codebook of at most STEPS bits.
template <int STEPS = 4>
__device__ __forceinline__ int tq_code(float u, const float *t) {
  static_assert(STEPS >= 1 && STEPS <= 4 && TQ_MAX_LEVELS == 16, "at most 15 thresholds");
  int idx = 0;
#pragma unroll
  for (int s = STEPS - 1; s >= 0; --s) idx += (u >= t[idx + (1 << s) - 1]) ? (1 << s) : 0;
  return idx;
}

// Dense rotation of a warp-held d-vector (coordinate lane + 32 k in x[k]):
// x <- M x with M given through MT[j*d + i] = M[i][j] (so a row j of MT is
// read by the warp as one coalesced line).  scratch: d floats of shared memory
// that belong to this warp.  fp32 products and sums in order j = 0 .. d-1.
template <int NPL>
__device__ __forceinline__ void tq_warp_dense(float (&x)[NPL], const float *__restrict__ MT,
                                              float *scratch, int lane) {
  constexpr int D = NPL * 32;
#pragma unroll
  for (int k = 0; k < NPL; ++k) scratch[lane + 32 * k] = x[k];
  __syncwarp();
  float acc[NPL];
#pragma unroll
  for (int k = 0; k < NPL; ++k) acc[k] = 0.f;
#pragma unroll 4
  for (int j = 0; j < D; ++j) {
    const float xj = scratch[j];
#pragma unroll
    for (int k = 0; k < NPL; ++k) acc[k] = fmaf(__ldg(MT + j * D + lane + 32 * k), xj, acc[k]);
  }
  __syncwarp();
#pragma unroll
  for (int k = 0; k < NPL; ++k) x[k] = acc[k];
}

// Same rotation for R rows held by one warp at once (x[r][k]: coordinate
// lane + 32 k of row r): each line of MT is read once for all R rows and the
// inputs are broadcast four at a time from shared memory.  scratch: R * d
// floats of this warp's shared memory, 16-byte aligned.  Per row the sums run
// in the same order as tq_warp_dense, so the results are identical.
template <int NPL, int R>
__device__ __forceinline__ void tq_warp_dense_rows(float (&x)[R][NPL], const float *__restrict__ MT,
                                                   float *scratch, int lane) {
  constexpr int D = NPL * 32;
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int k = 0; k < NPL; ++k) scratch[r * D + lane + 32 * k] = x[r][k];
  __syncwarp();
  float acc[R][NPL];
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int k = 0; k < NPL; ++k) acc[r][k] = 0.f;
#pragma unroll 1
  for (int j = 0; j < D; j += 4) {
    float m[4][NPL];
#pragma unroll
    for (int jj = 0; jj < 4; ++jj)
#pragma unroll
      for (int k = 0; k < NPL; ++k) m[jj][k] = __ldg(MT + (j + jj) * D + lane + 32 * k);
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const float4 xv = *reinterpret_cast<const float4 *>(scratch + r * D + j);
#pragma unroll
      for (int k = 0; k < NPL; ++k) {
        acc[r][k] = fmaf(m[0][k], xv.x, acc[r][k]);
        acc[r][k] = fmaf(m[1][k], xv.y, acc[r][k]);
        acc[r][k] = fmaf(m[2][k], xv.z, acc[r][k]);
        acc[r][k] = fmaf(m[3][k], xv.w, acc[r][k]);
      }
    }
  }
  __syncwarp();
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int k = 0; k < NPL; ++k) x[r][k] = acc[r][k];
}

