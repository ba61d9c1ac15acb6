// Fused quantize-append kernel: RoPE -> norm -> randomized WHT -> scalar codes
// -> bit planes, plus the QJL residual sketch for keys.
//
// Sources: "TurboESM ..." section 2.A (RoPE, then the rotation); "FibQuant ..."
// section 2.3 (store nu, rotate x/nu, quantize); "Ablazione ..."
// ("Configurazione Sperimentale": randomized Walsh-Hadamard rotation, Beta
// Lloyd-Max codebook, optional 1-bit QJL residual sketch on the key path);
// "Google presenta TurboQuant ..." ("Eliminacion del sesgo": b-1 MSE bits then a
// 1-bit QJL transform of the residual).
//
// Work split: one warp per (batch, head, 32-token group).  Coordinate
// i = lane + 32 k lives in register k of `lane`, so rotate-half RoPE pairs
// (i, i + d/2) are register-local, the transform runs on shuffles, and
// __ballot_sync over the warp produces each 32-coordinate key-plane word
// directly.  Value codes are accumulated per coordinate across the group's
// 32 tokens and stored as column-group words.
#include <cstdlib>

#include "tq_device.cuh"
#include "tq_sm100.cuh"

namespace {

constexpr int QWARPS = 8;
constexpr int QTC_T = 512;   // threads of quantize_tc_kernel: 4 groups x 4 row slices

struct QuantArgs {
  const void *k;
  const void *v;
  int dtype;
  int B, H, T;
  int64_t sb, sh, st;
  const float *rc;
  const float *rs;
  int64_t pos0;
  uint8_t *kcode;
  uint16_t *kscale;
  uint32_t *vcode;
  uint16_t *vnorm;
  int64_t rows_cap;
  int64_t row0;
  uint32_t *status;
  const uint16_t *S;
  const uint16_t *ST;  // S transposed (bf16)
  int64_t g_first;   // first 32-token group touched
  int64_t n_groups;  // groups touched per (b, h)
  TqRowMap map;      // channel map of an outlier-channel split (k == nullptr: none)
  TqBooks books;
};

// Channel map of KV head h (nullptr without a map).
__device__ __forceinline__ const int16_t *head_map(const int16_t *m, int64_t hs, int h) {
  return m != nullptr ? m + h * hs : nullptr;
}

// Load one row (coordinates lane + 32 k), optional RoPE at position pos.
// With a channel map (outlier-channel split), coordinate i is channel cmap[i]
// of a dfull-wide input row, and RoPE pairs channels (c, c + dfull/2) of that
// whole row, as in the unsplit case.
template <int NPL>
__device__ __forceinline__ void load_row(float (&x)[NPL], const void *base, int64_t off,
                                         int dtype, int lane, const float *rc, const float *rs,
                                         int64_t pos, const int16_t *cmap = nullptr,
                                         int dfull = 0) {
  if (cmap != nullptr) {
    const int half = dfull >> 1;
#pragma unroll
    for (int k = 0; k < NPL; ++k) {
      const int c = cmap[lane + 32 * k] & (dfull - 1);   // in bounds for any map
      float v = tq_load_elem(base, off + c, dtype);
      if (rc != nullptr) {
        const bool first = c < half;
        const int f = first ? c : c - half;
        const float w = tq_load_elem(base, off + (first ? c + half : c - half), dtype);
        const float cs = rc[pos * half + f], sn = rs[pos * half + f];
        v = first ? v * cs - w * sn : v * cs + w * sn;
      }
      x[k] = v;
    }
    return;
  }
#pragma unroll
  for (int k = 0; k < NPL; ++k) x[k] = tq_load_elem(base, off + lane + 32 * k, dtype);
  if (rc != nullptr) {
    constexpr int HALF = NPL / 2;  // register offset of coordinate i + d/2
    const int64_t tb = pos * (NPL * 16);
#pragma unroll
    for (int k = 0; k < HALF; ++k) {
      const float c = rc[tb + lane + 32 * k];
      const float s = rs[tb + lane + 32 * k];
      const float a = x[k], b = x[k + HALF];
      x[k] = a * c - b * s;
      x[k + HALF] = b * c + a * s;
    }
  }
}

// Normalise and rotate: returns nu (0 for bad rows), u = H D x / (sqrt(d) nu),
// or u = Pi x / nu with a dense rotation (scratch: this warp's d floats of
// shared memory, used only then).
template <int NPL>
__device__ __forceinline__ float normalize_rotate(float (&x)[NPL], const TqBooks &bk,
                                                  float *scratch, int lane, bool &bad) {
  bool finite = true;
  float ss = 0.f;
#pragma unroll
  for (int k = 0; k < NPL; ++k) {
    finite &= isfinite(x[k]);
    ss += x[k] * x[k];
  }
  bad = __any_sync(TQ_FULL, !finite);
  ss = tq_warp_sum(ss);
  float nu = sqrtf(ss);
  if (!bad && isinf(__half2float(__float2half_rn(nu)))) bad = true;
  if (bad) nu = 0.f;
#pragma unroll
  for (int k = 0; k < NPL; ++k) x[k] = bad ? 0.f : x[k];
  if (bk.pi_t != nullptr) {
    const float inv = nu > 0.f ? 1.0f / nu : 0.f;
    tq_warp_dense<NPL>(x, bk.pi_t, scratch, lane);
#pragma unroll
    for (int k = 0; k < NPL; ++k) x[k] *= inv;
    return nu;
  }
  const float inv = nu > 0.f ? 1.0f / (sqrtf(static_cast<float>(NPL * 32)) * nu) : 0.f;
  tq_apply_signs<NPL>(x, bk.dneg, lane);
  tq_warp_wht<NPL>(x, lane);
#pragma unroll
  for (int k = 0; k < NPL; ++k) x[k] *= inv;
  return nu;
}

// nu of a warp-held row and x <- x / nu (zero for a bad row), as in
// normalize_rotate but without the rotation (applied later to several rows).
template <int NPL>
__device__ __forceinline__ float normalize_only(float (&x)[NPL], int lane, bool &bad) {
  bool finite = true;
  float ss = 0.f;
#pragma unroll
  for (int k = 0; k < NPL; ++k) {
    finite &= isfinite(x[k]);
    ss += x[k] * x[k];
  }
  bad = __any_sync(TQ_FULL, !finite);
  ss = tq_warp_sum(ss);
  float nu = sqrtf(ss);
  if (!bad && isinf(__half2float(__float2half_rn(nu)))) bad = true;
  if (bad) nu = 0.f;
  const float inv = nu > 0.f ? 1.0f / nu : 0.f;
#pragma unroll
  for (int k = 0; k < NPL; ++k) x[k] = bad ? 0.f : x[k] * inv;
  return nu;
}

template <int D>
__global__ void __launch_bounds__(QWARPS * 32) quantize_kernel(QuantArgs a) {
  constexpr int NPL = D / 32;
  extern __shared__ float smem[];
  float *ST = smem;                      // S^T fp32 [D][D]: ST[j*D + i] = S[i][j]
  __shared__ float cks[TQ_MAX_LEVELS], tks[TQ_MAX_LEVELS], tvs[TQ_MAX_LEVELS];
  __shared__ float rbuf[QWARPS][D];

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x < TQ_MAX_LEVELS) {
    cks[threadIdx.x] = a.books.ck[threadIdx.x];
    tks[threadIdx.x] = a.books.tk[threadIdx.x];
    tvs[threadIdx.x] = a.books.tv[threadIdx.x];
  }
  if (a.books.qjl) {
    // stage S^T as fp32: coalesced 16-byte loads of the transposed bf16 copy
    const uint4 *src = reinterpret_cast<const uint4 *>(a.ST);
    for (int e = threadIdx.x; e < D * D / 8; e += blockDim.x) {
      const uint4 v = src[e];
      const float4 lo = make_float4(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xffff0000u),
                                    __uint_as_float(v.y << 16), __uint_as_float(v.y & 0xffff0000u));
      const float4 hi = make_float4(__uint_as_float(v.z << 16), __uint_as_float(v.z & 0xffff0000u),
                                    __uint_as_float(v.w << 16), __uint_as_float(v.w & 0xffff0000u));
      reinterpret_cast<float4 *>(ST)[2 * e] = lo;
      reinterpret_cast<float4 *>(ST)[2 * e + 1] = hi;
    }
  }
  __syncthreads();

  const int planes_k = a.books.mse_bits_k + a.books.qjl;
  const int64_t items = static_cast<int64_t>(a.B) * a.H * a.n_groups;
  for (int64_t it = static_cast<int64_t>(blockIdx.x) * QWARPS + warp; it < items;
       it += static_cast<int64_t>(gridDim.x) * QWARPS) {
    const int64_t g = a.g_first + it % a.n_groups;
    const int64_t bh = it / a.n_groups;
    const int b = static_cast<int>(bh / a.H), h = static_cast<int>(bh % a.H);
    const int64_t r_begin = max(a.row0, g * 32), r_end = min(a.row0 + a.T, g * 32 + 32);
    const int64_t cache_bh = static_cast<int64_t>(b) * a.H + h;

    uint32_t vw[4][NPL];
#pragma unroll
    for (int p = 0; p < 4; ++p)
#pragma unroll
      for (int k = 0; k < NPL; ++k) vw[p][k] = 0u;

    for (int64_t r = r_begin; r < r_end; ++r) {
      const int64_t t = r - a.row0;
      const int64_t in_off = b * a.sb + h * a.sh + t * a.st;
      // ------------------------------------------------------------ keys
      float x[NPL];
      load_row<NPL>(x, a.k, in_off, a.dtype, lane, a.rc, a.rs, a.pos0 + t,
                    head_map(a.map.k, a.map.hstride, h), a.map.dfull);
      bool bad;
      const float nu = normalize_rotate<NPL>(x, a.books, rbuf[warp], lane, bad);
      int idx[NPL];
#pragma unroll
      for (int k = 0; k < NPL; ++k) idx[k] = tq_code(x[k], tks);
      // plane words: lane p*NPL + k stores word k of plane p
      uint32_t myword = 0u;
      for (int p = 0; p < a.books.mse_bits_k; ++p) {
#pragma unroll
        for (int k = 0; k < NPL; ++k) {
          const uint32_t w = __ballot_sync(TQ_FULL, (idx[k] >> p) & 1);
          if (lane == p * NPL + k) myword = w;
        }
      }
      float rho = 0.f;
      if (a.books.qjl) {
        float r2 = 0.f;
#pragma unroll
        for (int k = 0; k < NPL; ++k) {
          const float rr = x[k] - cks[idx[k]];
          rbuf[warp][lane + 32 * k] = rr;
          r2 += rr * rr;
        }
        rho = sqrtf(tq_warp_sum(r2));
        __syncwarp();
        float z[NPL];
#pragma unroll
        for (int k = 0; k < NPL; ++k) z[k] = 0.f;
#pragma unroll 4
        for (int j = 0; j < D; ++j) {
          const float rj = rbuf[warp][j];
#pragma unroll
          for (int k = 0; k < NPL; ++k) z[k] = fmaf(ST[j * D + lane + 32 * k], rj, z[k]);
        }
        __syncwarp();
        const int p = a.books.mse_bits_k;
#pragma unroll
        for (int k = 0; k < NPL; ++k) {
          const uint32_t w = __ballot_sync(TQ_FULL, z[k] >= 0.f);
          if (lane == p * NPL + k) myword = w;
        }
      }
      uint32_t *krow = reinterpret_cast<uint32_t *>(
          a.kcode + (cache_bh * a.rows_cap + r) * planes_k * (D / 8));
      if (lane < planes_k * NPL) krow[lane] = myword;
      if (lane == 0) {
        const uint32_t pair = static_cast<uint32_t>(tq_f32_to_half(nu)) |
                              (static_cast<uint32_t>(tq_f32_to_half(rho)) << 16);
        reinterpret_cast<uint32_t *>(a.kscale)[cache_bh * a.rows_cap + r] = pair;
        if (bad && a.status) atomicAdd(a.status, 1u);
      }
      // ------------------------------------------------------------ values
      load_row<NPL>(x, a.v, in_off, a.dtype, lane, nullptr, nullptr, 0,
                    head_map(a.map.v, a.map.hstride, h), a.map.dfull);
      const float nv = normalize_rotate<NPL>(x, a.books, rbuf[warp], lane, bad);
      const uint32_t bit = 1u << (r & 31);
#pragma unroll
      for (int k = 0; k < NPL; ++k) {
        const int iv = tq_code(x[k], tvs);
#pragma unroll
        for (int p = 0; p < 4; ++p)
          if ((iv >> p) & 1) vw[p][k] |= bit;
      }
      if (lane == 0) {
        a.vnorm[cache_bh * a.rows_cap + r] = tq_f32_to_half(nv);
        if (bad && a.status) atomicAdd(a.status, 1u);
      }
    }
    // store the group's value words (read-modify-write for partial groups)
    const uint32_t nrows = static_cast<uint32_t>(r_end - r_begin);
    const uint32_t mask = nrows == 32 ? TQ_FULL : (((1u << nrows) - 1u) << (r_begin & 31));
    uint32_t *vg = a.vcode + (cache_bh * (a.rows_cap / 32) + g) * a.books.bits_v * D;
    for (int p = 0; p < a.books.bits_v; ++p) {
#pragma unroll
      for (int k = 0; k < NPL; ++k) {
        uint32_t *w = vg + p * D + lane + 32 * k;
        if (mask == TQ_FULL) {
          *w = vw[p][k];
        } else {
          atomicAnd(w, ~mask);
          atomicOr(w, vw[p][k] & mask);
        }
      }
    }
  }
}


// ---------------------------------------------------------------------------
// Small calls (decode appends): one 128-thread block per (b, h, 32-token
// group).  Warp 0 runs the key pipeline of a row and warp 1 the value
// pipeline (same steps as quantize_kernel); the sketch z = S r of the key row
// is spread over the block: thread i computes z_i from row i of S (bf16,
// row-major, read from L2 as 16-byte loads), so no block stages S^T.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(128) quantize_append_kernel(QuantArgs a) {
  constexpr int NPL = D / 32;
  __shared__ float cks[TQ_MAX_LEVELS], tks[TQ_MAX_LEVELS], tvs[TQ_MAX_LEVELS];
  __shared__ __align__(16) float rsm[D];
  __shared__ uint32_t sgw[NPL];
  __shared__ float dsc[2][D];          // dense-rotation scratch of warps 0 and 1
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid < TQ_MAX_LEVELS) {
    cks[tid] = a.books.ck[tid];
    tks[tid] = a.books.tk[tid];
    tvs[tid] = a.books.tv[tid];
  }
  __syncthreads();
  const int planes_k = a.books.mse_bits_k + a.books.qjl;
  // a following decode's query prologue may start now (it waits for this
  // grid before it completes)
  sm100::pdl_trigger();
  // row tid of S (bf16), loaded up front so its latency overlaps the rows'
  uint4 srow[D / 8];
  if (a.books.qjl && tid < D) {
    const uint4 *sp = reinterpret_cast<const uint4 *>(a.S + static_cast<int64_t>(tid) * D);
#pragma unroll
    for (int q = 0; q < D / 8; ++q) srow[q] = sp[q];
  }
  const int64_t it = blockIdx.x;
  const int64_t g = a.g_first + it % a.n_groups;
  const int64_t bh = it / a.n_groups;
  const int b = static_cast<int>(bh / a.H), h = static_cast<int>(bh % a.H);
  const int64_t r_begin = max(a.row0, g * 32), r_end = min(a.row0 + a.T, g * 32 + 32);
  const int64_t cache_bh = static_cast<int64_t>(b) * a.H + h;
  uint32_t vw[4][NPL];
#pragma unroll
  for (int p = 0; p < 4; ++p)
#pragma unroll
    for (int k = 0; k < NPL; ++k) vw[p][k] = 0u;
  // a partial group keeps its other rows: their words are read now, so the
  // load overlaps the rows' pipeline instead of trailing it
  const uint32_t nrows = static_cast<uint32_t>(r_end - r_begin);
  const uint32_t vmask = nrows >= 32 ? TQ_FULL : (((1u << nrows) - 1u) << (r_begin & 31));
  uint32_t *vgw = a.vcode + (cache_bh * (a.rows_cap / 32) + g) * a.books.bits_v * D;
  uint32_t vold[4][NPL];
  if (warp == 1 && vmask != TQ_FULL) {
#pragma unroll
    for (int p = 0; p < 4; ++p)
#pragma unroll
      for (int k = 0; k < NPL; ++k) vold[p][k] = p < a.books.bits_v ? vgw[p * D + lane + 32 * k] : 0u;
  }

  for (int64_t r = r_begin; r < r_end; ++r) {
    const int64_t t = r - a.row0;
    const int64_t in_off = b * a.sb + h * a.sh + t * a.st;
    uint32_t myword = 0u;
    float nu = 0.f, rho = 0.f;
    bool bad = false;
    // dense rotation: warps 0 and 1 normalise their rows, then the whole block
    // forms u = Pi x for both (thread i: row i of Pi, 16-byte loads in flight)
    const bool dense = a.books.pi != nullptr;
    float dnu = 0.f;
    bool dbad = false;
    if (dense) {
      if (warp < 2) {
        float x[NPL];
        load_row<NPL>(x, warp == 0 ? a.k : a.v, in_off, a.dtype, lane, warp == 0 ? a.rc : nullptr,
                      warp == 0 ? a.rs : nullptr, a.pos0 + t,
                      head_map(warp == 0 ? a.map.k : a.map.v, a.map.hstride, h), a.map.dfull);
        dnu = normalize_only<NPL>(x, lane, dbad);
#pragma unroll
        for (int k = 0; k < NPL; ++k) dsc[warp][lane + 32 * k] = x[k];
      }
      __syncthreads();
      float u0 = 0.f, u1 = 0.f;
      if (tid < D) {
        const float4 *row = reinterpret_cast<const float4 *>(a.books.pi + tid * D);
#pragma unroll 8
        for (int c = 0; c < D / 4; ++c) {
          const float4 pv = row[c];
          u0 = fmaf(pv.x, dsc[0][4 * c], u0);
          u0 = fmaf(pv.y, dsc[0][4 * c + 1], u0);
          u0 = fmaf(pv.z, dsc[0][4 * c + 2], u0);
          u0 = fmaf(pv.w, dsc[0][4 * c + 3], u0);
          u1 = fmaf(pv.x, dsc[1][4 * c], u1);
          u1 = fmaf(pv.y, dsc[1][4 * c + 1], u1);
          u1 = fmaf(pv.z, dsc[1][4 * c + 2], u1);
          u1 = fmaf(pv.w, dsc[1][4 * c + 3], u1);
        }
      }
      __syncthreads();
      if (tid < D) {
        dsc[0][tid] = u0;
        dsc[1][tid] = u1;
      }
      __syncthreads();
    }
    if (warp == 0) {
      float x[NPL];
      if (dense) {
#pragma unroll
        for (int k = 0; k < NPL; ++k) x[k] = dsc[0][lane + 32 * k];
        nu = dnu;
        bad = dbad;
      } else {
        load_row<NPL>(x, a.k, in_off, a.dtype, lane, a.rc, a.rs, a.pos0 + t,
                      head_map(a.map.k, a.map.hstride, h), a.map.dfull);
        nu = normalize_rotate<NPL>(x, a.books, dsc[warp], lane, bad);
      }
      int idx[NPL];
#pragma unroll
      for (int k = 0; k < NPL; ++k) idx[k] = tq_code(x[k], tks);
      for (int p = 0; p < a.books.mse_bits_k; ++p) {
#pragma unroll
        for (int k = 0; k < NPL; ++k) {
          const uint32_t w = __ballot_sync(TQ_FULL, (idx[k] >> p) & 1);
          if (lane == p * NPL + k) myword = w;
        }
      }
      if (a.books.qjl) {
        float r2 = 0.f;
#pragma unroll
        for (int k = 0; k < NPL; ++k) {
          const float rr = x[k] - cks[idx[k]];
          rsm[lane + 32 * k] = rr;
          r2 += rr * rr;
        }
        rho = sqrtf(tq_warp_sum(r2));
      }
    } else if (warp == 1) {
      float x[NPL];
      bool vbad;
      float nv;
      if (dense) {
#pragma unroll
        for (int k = 0; k < NPL; ++k) x[k] = dsc[1][lane + 32 * k];
        nv = dnu;
        vbad = dbad;
      } else {
        load_row<NPL>(x, a.v, in_off, a.dtype, lane, nullptr, nullptr, 0,
                      head_map(a.map.v, a.map.hstride, h), a.map.dfull);
        nv = normalize_rotate<NPL>(x, a.books, dsc[warp], lane, vbad);
      }
      const uint32_t bit = 1u << (r & 31);
#pragma unroll
      for (int k = 0; k < NPL; ++k) {
        const int iv = tq_code(x[k], tvs);
#pragma unroll
        for (int p = 0; p < 4; ++p)
          if ((iv >> p) & 1) vw[p][k] |= bit;
      }
      if (lane == 0) {
        a.vnorm[cache_bh * a.rows_cap + r] = tq_f32_to_half(nv);
        if (vbad && a.status) atomicAdd(a.status, 1u);
      }
    }
    __syncthreads();
    if (a.books.qjl && tid < D) {
      // z_tid = sum_j S[tid][j] r_j; whole warps take part (D is a multiple of 32)
      float z = 0.f;
#pragma unroll
      for (int q = 0; q < D / 8; ++q) {
        const uint4 v = srow[q];
        const float4 r0 = reinterpret_cast<const float4 *>(rsm)[2 * q];
        const float4 r1 = reinterpret_cast<const float4 *>(rsm)[2 * q + 1];
        z = fmaf(__uint_as_float(v.x << 16), r0.x, z);
        z = fmaf(__uint_as_float(v.x & 0xffff0000u), r0.y, z);
        z = fmaf(__uint_as_float(v.y << 16), r0.z, z);
        z = fmaf(__uint_as_float(v.y & 0xffff0000u), r0.w, z);
        z = fmaf(__uint_as_float(v.z << 16), r1.x, z);
        z = fmaf(__uint_as_float(v.z & 0xffff0000u), r1.y, z);
        z = fmaf(__uint_as_float(v.w << 16), r1.z, z);
        z = fmaf(__uint_as_float(v.w & 0xffff0000u), r1.w, z);
      }
      const uint32_t w = __ballot_sync(TQ_FULL, z >= 0.f);
      if (lane == 0) sgw[warp] = w;
    }
    __syncthreads();
    if (warp == 0) {
      const int p = a.books.mse_bits_k;
      if (a.books.qjl && lane >= p * NPL && lane < (p + 1) * NPL) myword = sgw[lane - p * NPL];
      uint32_t *krow = reinterpret_cast<uint32_t *>(
          a.kcode + (cache_bh * a.rows_cap + r) * planes_k * (D / 8));
      if (lane < planes_k * NPL) krow[lane] = myword;
      if (lane == 0) {
        const uint32_t pair = static_cast<uint32_t>(tq_f32_to_half(nu)) |
                              (static_cast<uint32_t>(tq_f32_to_half(rho)) << 16);
        reinterpret_cast<uint32_t *>(a.kscale)[cache_bh * a.rows_cap + r] = pair;
        if (bad && a.status) atomicAdd(a.status, 1u);
      }
    }
    __syncthreads();   // rsm and sgw are reused by the next row
  }
  if (warp == 1) {
    // the group's value words (partial groups merge the words read above;
    // this block is the only writer of the group within the call)
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      if (p >= a.books.bits_v) break;
#pragma unroll
      for (int k = 0; k < NPL; ++k)
        vgw[p * D + lane + 32 * k] = vmask == TQ_FULL ? vw[p][k] : ((vold[p][k] & ~vmask) | (vw[p][k] & vmask));
    }
  }
}

// ---------------------------------------------------------------------------
// tcgen05 variant for large calls: the QJL sketch z = S r of a 128-row tile
// is one tensor-core contraction.  Each warp runs the fused per-row pipeline
// above for one 32-token group and writes its residuals, split into bf16
// hi + lo (r = hi + lo + O(2^-18 |r|)), into the shared A tile; one thread
// issues 2d/16 kind::f16 MMAs against S (exactly representable: S is stored
// as bf16) with fp32 accumulation in tensor memory; thread t then reads row
// t of z and writes that key's sign plane.
// Shared layouts (K-major, no swizzle): A byte (m, kb) at
// (kb/16)*2048 + (m/8)*128 + (m%8)*16 + kb%16 for K = 2d elements (hi | lo);
// B = S, byte (i, kb) at (kb/16)*(16d) + (i/8)*128 + (i%8)*16 + kb%16.
// MBK / BV: key MSE bits and value bits the kernel is specialised for (the
// code searches and plane loops then have fixed trip counts); MBK = BV = 4
// takes any codec of at most 4 + 4 bits, with the plane loops bounded by the
// codec's own widths.
template <int D, int MBK, int BV>
__global__ void __launch_bounds__(QTC_T, 1) quantize_tc_kernel(QuantArgs a) {
  constexpr int NPL = D / 32;
  constexpr int KE = 2 * D;                       // K elements (hi | lo)
  constexpr uint32_t A_BYTES = 128u * KE * 2u;
  constexpr uint32_t IDESC = sm100::idesc_bf16(128, D);
  extern __shared__ __align__(128) float smem_tc[];
  uint8_t *As = reinterpret_cast<uint8_t *>(smem_tc);
  uint8_t *Bs = As + A_BYTES;
  __shared__ float cks[TQ_MAX_LEVELS], tks[TQ_MAX_LEVELS], tvs[TQ_MAX_LEVELS];
  __shared__ uint32_t vbuf[4][4][D];   // value column words of the tile's 4 groups
  // dense-rotation scratch: the PF rows of each warp
  __shared__ __align__(16) float dsc[QTC_T / 32][(D == 64 ? 8 : 4) * D];
  __shared__ __align__(8) uint64_t mb;
  __shared__ uint32_t tmem_s;
  __shared__ int abort_s;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid < TQ_MAX_LEVELS) {
    cks[tid] = a.books.ck[tid];
    tks[tid] = a.books.tk[tid];
    tvs[tid] = a.books.tv[tid];
  }
  for (int e = tid; e < D * D; e += QTC_T) {
    const int i = e / D, kb = 2 * (e % D);
    *reinterpret_cast<uint16_t *>(Bs + (kb >> 4) * (D * 16) + (i >> 3) * 128 + (i & 7) * 16 +
                                  (kb & 15)) = a.S[e];
  }
  if (warp == 0) sm100::tmem_alloc(&tmem_s, D);
  if (tid == 0) {
    sm100::mbar_init(&mb, 1);
    abort_s = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  sm100::fence_async_smem();
  sm100::fence_before_sync();
  __syncthreads();
  sm100::fence_after_sync();
  const uint32_t tm = tmem_s;
  const uint32_t a_addr = sm100::smem_addr(As), b_addr = sm100::smem_addr(Bs);
  const int planes_k = a.books.mse_bits_k + 1;
  const int64_t items = static_cast<int64_t>(a.B) * a.H * a.n_groups;
  const int64_t tiles = (items + 3) / 4;
  uint32_t phase = 0;

  // warp w: group grp = w / 4 of the tile, rows 8 (w % 4) .. +7 of that group
  const int grp = warp >> 2, sub8 = warp & 3;
  for (int64_t tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
    for (int e = tid; e < 4 * 4 * D; e += QTC_T) (&vbuf[0][0][0])[e] = 0u;
    const int64_t it = tile * 4 + grp;
    const bool have = it < items;
    int64_t g = 0, cache_bh = 0, r_begin = 0, r_end = 0;
    int b = 0, h = 0;
    if (have) {
      g = a.g_first + it % a.n_groups;
      const int64_t bh = it / a.n_groups;
      b = static_cast<int>(bh / a.H);
      h = static_cast<int>(bh % a.H);
      r_begin = max(a.row0, g * 32);
      r_end = min(a.row0 + a.T, g * 32 + 32);
      cache_bh = static_cast<int64_t>(b) * a.H + h;
    }
    uint32_t vw[4][NPL];
#pragma unroll
    for (int p = 0; p < 4; ++p)
#pragma unroll
      for (int k = 0; k < NPL; ++k) vw[p][k] = 0u;
    const int64_t rb = max(r_begin, g * 32 + 8 * sub8), re = min(r_end, g * 32 + 8 * sub8 + 8);
    __syncthreads();   // vbuf cleared
    // rows are loaded PF at a time (all loads issued before any row is
    // processed) so each warp keeps PF rows of K and V in flight
    constexpr int PF = D == 64 ? 8 : 4;
    for (int64_t r0 = rb; r0 < re; r0 += PF) {
    float xk[PF][NPL], xv[PF][NPL];
#pragma unroll
    for (int i = 0; i < PF; ++i) {
      if (r0 + i < re) {
        const int64_t t = r0 + i - a.row0;
        const int64_t in_off = b * a.sb + h * a.sh + t * a.st;
        load_row<NPL>(xk[i], a.k, in_off, a.dtype, lane, a.rc, a.rs, a.pos0 + t,
                      head_map(a.map.k, a.map.hstride, h), a.map.dfull);
        load_row<NPL>(xv[i], a.v, in_off, a.dtype, lane, nullptr, nullptr, 0,
                      head_map(a.map.v, a.map.hstride, h), a.map.dfull);
      } else {
#pragma unroll
        for (int k = 0; k < NPL; ++k) xk[i][k] = xv[i][k] = 0.f;
      }
    }
    // dense rotation: norms first, then the PF rows of K and of V rotated
    // together (each line of Pi^T read once per PF rows)
    const bool dense = a.books.pi_t != nullptr;
    float nuk[PF], nuv[PF];
    bool badk[PF], badv[PF];
    if (dense) {
#pragma unroll
      for (int i = 0; i < PF; ++i) {
        nuk[i] = normalize_only<NPL>(xk[i], lane, badk[i]);
        nuv[i] = normalize_only<NPL>(xv[i], lane, badv[i]);
      }
      tq_warp_dense_rows<NPL, PF>(xk, a.books.pi_t, dsc[warp], lane);
      tq_warp_dense_rows<NPL, PF>(xv, a.books.pi_t, dsc[warp], lane);
    }
#pragma unroll
    for (int i = 0; i < PF; ++i) {
      const int64_t r = r0 + i;
      if (r >= re) break;
      float x[NPL];
#pragma unroll
      for (int k = 0; k < NPL; ++k) x[k] = xk[i][k];
      bool bad = dense ? badk[i] : false;
      const float nu = dense ? nuk[i] : normalize_rotate<NPL>(x, a.books, dsc[warp], lane, bad);
      int idx[NPL];
#pragma unroll
      for (int k = 0; k < NPL; ++k) idx[k] = tq_code<MBK>(x[k], tks);
      uint32_t myword = 0u;
#pragma unroll
      for (int p = 0; p < MBK; ++p) {
        if (MBK == 4 && p >= a.books.mse_bits_k) break;
#pragma unroll
        for (int k = 0; k < NPL; ++k) {
          const uint32_t w = __ballot_sync(TQ_FULL, (idx[k] >> p) & 1);
          if (lane == p * NPL + k) myword = w;
        }
      }
      const int m = grp * 32 + static_cast<int>(r & 31);
      float r2 = 0.f;
#pragma unroll
      for (int k = 0; k < NPL; ++k) {
        const float rr = x[k] - cks[idx[k]];
        r2 += rr * rr;
        const __nv_bfloat16 hi = __float2bfloat16_rn(rr);
        const __nv_bfloat16 lo = __float2bfloat16_rn(rr - __bfloat162float(hi));
        const int j = lane + 32 * k;
        const int kb_hi = 2 * j, kb_lo = 2 * (D + j);
        const int row_off = (m >> 3) * 128 + (m & 7) * 16;
        *reinterpret_cast<__nv_bfloat16 *>(As + (kb_hi >> 4) * 2048 + row_off + (kb_hi & 15)) = hi;
        *reinterpret_cast<__nv_bfloat16 *>(As + (kb_lo >> 4) * 2048 + row_off + (kb_lo & 15)) = lo;
      }
      const float rho = sqrtf(tq_warp_sum(r2));
      uint32_t *krow = reinterpret_cast<uint32_t *>(
          a.kcode + (cache_bh * a.rows_cap + r) * planes_k * (D / 8));
      if (lane < a.books.mse_bits_k * NPL) krow[lane] = myword;
      if (lane == 0) {
        const uint32_t pair = static_cast<uint32_t>(tq_f32_to_half(nu)) |
                              (static_cast<uint32_t>(tq_f32_to_half(rho)) << 16);
        reinterpret_cast<uint32_t *>(a.kscale)[cache_bh * a.rows_cap + r] = pair;
        if (bad && a.status) atomicAdd(a.status, 1u);
      }
#pragma unroll
      for (int k = 0; k < NPL; ++k) x[k] = xv[i][k];
      if (dense) bad = badv[i];
      const float nv = dense ? nuv[i] : normalize_rotate<NPL>(x, a.books, dsc[warp], lane, bad);
      const uint32_t bit = 1u << (r & 31);
#pragma unroll
      for (int k = 0; k < NPL; ++k) {
        const int iv = tq_code<BV>(x[k], tvs);
#pragma unroll
        for (int p = 0; p < BV; ++p)
          if ((iv >> p) & 1) vw[p][k] |= bit;
      }
      if (lane == 0) {
        a.vnorm[cache_bh * a.rows_cap + r] = tq_f32_to_half(nv);
        if (bad && a.status) atomicAdd(a.status, 1u);
      }
    }
    }
    if (have && rb < re) {
#pragma unroll
      for (int p = 0; p < BV; ++p) {
        if (p >= a.books.bits_v) break;
#pragma unroll
        for (int k = 0; k < NPL; ++k) atomicOr(&vbuf[grp][p][lane + 32 * k], vw[p][k]);
      }
    }
    // ---- the sketch of the whole tile on the tensor cores
    sm100::fence_async_smem();
    sm100::fence_before_sync();
    __syncthreads();
    sm100::fence_after_sync();
    // the group's value words (read-modify-write for partial groups)
    if (have && sub8 == 0) {
      const uint32_t nrows = static_cast<uint32_t>(r_end - r_begin);
      const uint32_t mask = nrows == 32 ? TQ_FULL : (((1u << nrows) - 1u) << (r_begin & 31));
      uint32_t *vg = a.vcode + (cache_bh * (a.rows_cap / 32) + g) * a.books.bits_v * D;
      for (int p = 0; p < a.books.bits_v; ++p) {
#pragma unroll
        for (int k = 0; k < NPL; ++k) {
          uint32_t *w = vg + p * D + lane + 32 * k;
          const uint32_t v = vbuf[grp][p][lane + 32 * k];
          if (mask == TQ_FULL) {
            *w = v;
          } else {
            atomicAnd(w, ~mask);
            atomicOr(w, v & mask);
          }
        }
      }
    }
    if (tid == 0) {
#pragma unroll
      for (int s = 0; s < KE / 16; ++s) {
        const int kk = (16 * s) % D;
        sm100::mma_bf16_ss(tm, sm100::smem_desc(a_addr + s * 2 * 2048, 2048, 128),
                           sm100::smem_desc(b_addr + (kk / 8) * (D * 16), D * 16, 128), IDESC,
                           s > 0);
      }
      sm100::mma_commit(&mb);
    }
    if (!sm100::mbar_wait(&mb, phase)) abort_s = 1;
    phase ^= 1;
    __syncthreads();
    if (abort_s) break;
    sm100::fence_after_sync();
    // warps 0..3 read TMEM lane quarter q = warp: rows of group q of the tile
    if (warp < 4) {
    const int64_t itq = tile * 4 + warp;
    bool row_ok = false;
    int64_t myr = 0, cbq = 0;
    if (itq < items) {
      const int64_t gq = a.g_first + itq % a.n_groups;
      const int64_t bhq = itq / a.n_groups;
      cbq = (bhq / a.H) * a.H + bhq % a.H;
      const int64_t rbq = max(a.row0, gq * 32), req = min(a.row0 + a.T, gq * 32 + 32);
      myr = gq * 32 + lane;
      row_ok = myr >= rbq && myr < req;
    }
    uint32_t sw[NPL];
#pragma unroll
    for (int wd = 0; wd < NPL; ++wd) {
      uint32_t z0[16], z1[16];
      sm100::tmem_ld16(sm100::tmem_lane(tm + 32 * wd, warp), z0);
      sm100::tmem_ld16(sm100::tmem_lane(tm + 32 * wd + 16, warp), z1);
      sm100::wait_ld();
      uint32_t word = 0u;
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        word |= (__uint_as_float(z0[c]) >= 0.f ? 1u : 0u) << c;
        word |= (__uint_as_float(z1[c]) >= 0.f ? 1u : 0u) << (16 + c);
      }
      sw[wd] = word;
    }
    if (row_ok) {
      uint32_t *srow = reinterpret_cast<uint32_t *>(
          a.kcode + (cbq * a.rows_cap + myr) * planes_k * (D / 8) + a.books.mse_bits_k * (D / 8));
#pragma unroll
      for (int wd = 0; wd < NPL; ++wd) srow[wd] = sw[wd];
    }
    }
    sm100::fence_before_sync();
    __syncthreads();
    sm100::fence_after_sync();
  }
  if (abort_s) {
    sm100::mbar_wait(&mb, phase, 1u << 20);
    if (tid == 0 && a.status) atomicOr(a.status, 1u << 31);
  }
  sm100::fence_before_sync();
  __syncthreads();
  sm100::fence_after_sync();
  if (warp == 0) sm100::tmem_dealloc(tm, D);
}

template <int D, int MBK, int BV>
int run_quantize_tc_bits(const QuantArgs &a, cudaStream_t stream) {
  constexpr size_t shm = 128u * 2 * D * 2 + static_cast<size_t>(D) * D * 2;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  static bool done[64] = {};
  if (dev < 64 && !done[dev]) {
    if (cudaFuncSetAttribute(quantize_tc_kernel<D, MBK, BV>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(shm)) != cudaSuccess)
      return tq_check_launch("cudaFuncSetAttribute(quantize_tc)");
    done[dev] = true;
  }
  const int64_t items = static_cast<int64_t>(a.B) * a.H * a.n_groups;
  const int64_t tiles = (items + 3) / 4;
  const int64_t cap = static_cast<int64_t>(sms) * (D == 128 ? 1 : 2);
  const int grid = static_cast<int>(tiles < cap ? tiles : cap);
  quantize_tc_kernel<D, MBK, BV><<<grid, QTC_T, shm, stream>>>(a);
  tq_count_launch(1);
  return tq_check_launch("quantize_tc_kernel");
}

// The Llama- and ESM-2-shaped codecs get their own instantiations; any other
// codec takes the generic one (a (1, 2) instantiation spills at d = 128).
template <int D>
int run_quantize_tc(const QuantArgs &a, cudaStream_t stream) {
  const int mbk = a.books.mse_bits_k, bv = a.books.bits_v;
  if (mbk == 3 && bv == 4) return run_quantize_tc_bits<D, 3, 4>(a, stream);
  if (mbk == 2 && bv == 3) return run_quantize_tc_bits<D, 2, 3>(a, stream);
  return run_quantize_tc_bits<D, 4, 4>(a, stream);
}

template <int D>
int run_quantize_append(const QuantArgs &a, int64_t items, cudaStream_t stream) {
  quantize_append_kernel<D><<<static_cast<unsigned>(items), 128, 0, stream>>>(a);
  tq_count_launch(1);
  return tq_check_launch("quantize_append_kernel");
}

template <int D>
int run_quantize(const QuantArgs &a, cudaStream_t stream) {
  const size_t shm = a.books.qjl ? sizeof(float) * D * D : 0;
  static bool attr_set = false;
  if (!attr_set) {
    if (cudaFuncSetAttribute(quantize_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             sizeof(float) * D * D) != cudaSuccess)
      return tq_check_launch("cudaFuncSetAttribute(quantize)");
    attr_set = true;
  }
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t items = static_cast<int64_t>(a.B) * a.H * a.n_groups;
  const int64_t want = (items + QWARPS - 1) / QWARPS;
  const int grid = static_cast<int>(want < 4LL * sms ? want : 4LL * sms);
  quantize_kernel<D><<<grid, QWARPS * 32, shm, stream>>>(a);
  tq_count_launch(1);
  return tq_check_launch("quantize_kernel");
}

}  // namespace

int launch_quantize(const tq_codec *c, const void *k, const void *v, int dtype, int B, int H,
                    int T, int64_t sb, int64_t sh, int64_t st, const float *rc, const float *rs,
                    int64_t pos0, const tq_cache *cache, int64_t row0, uint32_t *status,
                    cudaStream_t stream, const TqRowMap &map) {
  QuantArgs a;
  a.k = k;
  a.v = v;
  a.dtype = dtype;
  a.B = B;
  a.H = H;
  a.T = T;
  a.sb = sb;
  a.sh = sh;
  a.st = st;
  a.rc = rc;
  a.rs = rs;
  a.pos0 = pos0;
  a.kcode = cache->kcode;
  a.kscale = cache->kscale;
  a.vcode = cache->vcode;
  a.vnorm = cache->vnorm;
  a.rows_cap = cache->rows_cap;
  a.row0 = row0;
  a.status = status;
  a.S = c->S_dev;
  a.ST = c->ST_dev;
  a.g_first = row0 / 32;
  a.n_groups = (row0 + T - 1) / 32 - row0 / 32 + 1;
  a.map = map;
  a.books = c->books;
  if (T == 0) return TQ_OK;
  const int64_t items = static_cast<int64_t>(B) * H * a.n_groups;
  // TQ_QUANT_IMPL=simt keeps the CUDA-core sketch (a complete second
  // implementation, used to cross-check the tensor-core one)
  const char *impl = getenv("TQ_QUANT_IMPL");
  const bool simt = impl && impl[0] == 's';
  if (items >= 256 && !simt && map.k == nullptr && c->books.pi == nullptr) {
    // large bf16 calls: one thread per row, TMA tiles (quantize_tile.cu); a
    // channel map (gathered loads) or a dense rotation takes the warp-per-row
    // kernels below
    const int e = launch_quantize_tile(c, k, v, dtype, B, H, T, sb, sh, st, rc, rs, pos0, cache,
                                       row0, status, stream);
    if (e != TQ_ERR_UNSUPPORTED) return e;
  }
  if (items >= 256 && !simt && map.k == nullptr && c->books.pi != nullptr) {
    // dense rotation: the tile's rotation as a tensor-core product (quantize_rot.cu)
    const int e = launch_quantize_rot(c, k, v, dtype, B, H, T, sb, sh, st, rc, rs, pos0, cache,
                                      row0, status, stream);
    if (e != TQ_ERR_UNSUPPORTED) return e;
  }
  const bool tc = c->qjl_k && items >= 256 && !simt;
  const bool append = items < 256 && !simt;
  switch (c->d) {
    case 64:
      return tc ? run_quantize_tc<64>(a, stream)
                : append ? run_quantize_append<64>(a, items, stream) : run_quantize<64>(a, stream);
    case 128:
      return tc ? run_quantize_tc<128>(a, stream)
                : append ? run_quantize_append<128>(a, items, stream) : run_quantize<128>(a, stream);
    default: return tq_fail(TQ_ERR_UNSUPPORTED, "quantize: head dim not built");
  }
}
