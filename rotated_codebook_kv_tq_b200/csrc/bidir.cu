// Bidirectional attention over the compressed cache, tensor-core tiles.
//
// "TurboESM ..." section 2.A (RoPE first, then the shared rotation, so
// (Pi R_i q)^T (Pi R_j k) = q^T R_i^T R_j k) and section 2.E (attention from the
// compressed cache with online softmax); "Google presenta TurboQuant ...",
// "Eliminacion del sesgo" (the prod estimator).  Query i sits at position i and
// attends to all T keys of its KV head, no mask.
//
// Everything runs in the rotated domain with d' = 2d columns:
//   Q_rot[i] = [ q'_i | q''_i ]                     q' = Pi RoPE(q), q'' = S q'
//   K_rot[j] = [ c[idx_j] | sqrt(pi/2)/d rho_j (2 sigma_j - 1) ]
//   logit_ij = scale nu_j <Q_rot[i], K_rot[j]>,      O_rot = softmax(logit) V_rot,
//   V_rot[j] = nu^v_j c_v[idx^v_j],                  out = Pi^T O_rot.
// A CTA owns 128 queries of one (batch, head) (TMEM lane = query) and walks the
// keys in tiles of 64: S = Q_rot K_rot^T and O_tile = P V_rot each run as six
// bf16 kind::f16 MMA sets (the order <= 2 products of a three-term bf16 split,
// about 2^-26 relative: the logits reach a few hundred on data with outlier
// channels, and a two-term split's 2^-17 would shift them by ~1e-3) with fp32
// accumulators in tensor memory; softmax statistics stay in fp32 registers
// of the query's thread and the output sum accumulates in tensor memory
// (rescaled in place when a row's running maximum moves).
// The tensor core's fp32 accumulation does not round to nearest: every MMA
// that adds into an accumulator can lose up to an ulp of it, and a chain of
// 48 MMAs into one accumulator moves logits of ~200 by ~5e-4.  So S is split
// over five accumulators: the five small split products share one (its
// magnitude is ~2^-8 of the logit), and the leading hi*hi product spreads its
// K steps over four, each a chain of two; they are added in fp32 registers.
#include <math_constants.h>

#include <cstdlib>

#include "tq_device.cuh"
#include "tq_sm100.cuh"

namespace {

constexpr int BQ = 128;   // queries per CTA
constexpr int BK = 64;    // keys per tile
constexpr int PR = 4;     // threads per query row in the tile kernel
constexpr int BT = PR * BQ;

struct BidirArgs {
  const void *q;
  int dtype;
  int B, H, Hkv, Lq, T;
  const uint8_t *kcode;
  const uint16_t *kscale;
  const uint32_t *vcode;
  const uint16_t *vnorm;
  int64_t rows_cap;
  float scale, qjl_coef;
  const float *rc;
  const float *rs;
  const uint16_t *ST;
  float *qrot;      // [B][H][Lq][2d] fp32
  float *out;       // [B][H][Lq][d]
  uint32_t *err;
  uint32_t wait_limit;   // polls per wait before giving up
  TqBooks books;
};

// One warp per query: q' = Pi RoPE(q, i), q'' = S q' (S^T staged in smem).
template <int D>
__global__ void __launch_bounds__(256) bidir_qprep_kernel(BidirArgs a) {
  constexpr int NPL = D / 32;
  extern __shared__ float sts_f[];   // S^T fp32 [D][D]
  __shared__ float qs[8][D];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (a.books.qjl) {
    for (int e = threadIdx.x; e < D * D; e += blockDim.x) sts_f[e] = tq_bf16_to_f32(a.ST[e]);
  }
  __syncthreads();
  const int64_t nq = static_cast<int64_t>(a.B) * a.H * a.Lq;
  for (int64_t qi = static_cast<int64_t>(blockIdx.x) * 8 + warp; qi < nq;
       qi += static_cast<int64_t>(gridDim.x) * 8) {
    const int64_t pos = qi % a.Lq;
    float x[NPL];
#pragma unroll
    for (int k = 0; k < NPL; ++k) x[k] = tq_load_elem(a.q, qi * D + lane + 32 * k, a.dtype);
    if (a.rc != nullptr) {
      constexpr int HALF = NPL / 2;
#pragma unroll
      for (int k = 0; k < HALF; ++k) {
        const float c = a.rc[pos * (D / 2) + lane + 32 * k];
        const float s = a.rs[pos * (D / 2) + lane + 32 * k];
        const float u = x[k], v = x[k + HALF];
        x[k] = u * c - v * s;
        x[k + HALF] = v * c + u * s;
      }
    }
    tq_apply_signs<NPL>(x, a.books.dneg, lane);
    tq_warp_wht<NPL>(x, lane);
    const float inv_sqrt_d = 1.0f / sqrtf(static_cast<float>(D));
    float *dst = a.qrot + qi * 2 * D;
#pragma unroll
    for (int k = 0; k < NPL; ++k) {
      x[k] *= inv_sqrt_d;
      dst[lane + 32 * k] = x[k];
      qs[warp][lane + 32 * k] = x[k];
    }
    __syncwarp();
    float z[NPL];
#pragma unroll
    for (int k = 0; k < NPL; ++k) z[k] = 0.f;
    if (a.books.qjl) {
      for (int j = 0; j < D; ++j) {
        const float qj = qs[warp][j];
#pragma unroll
        for (int k = 0; k < NPL; ++k) z[k] = fmaf(sts_f[j * D + lane + 32 * k], qj, z[k]);
      }
    }
#pragma unroll
    for (int k = 0; k < NPL; ++k) dst[D + lane + 32 * k] = z[k];
    __syncwarp();
  }
}

// byte offset of element (row, k) of a K-major no-swizzle bf16 operand with
// R rows: each 16-byte slice of K (8 elements) holds all R rows
__device__ __forceinline__ int kmaj16(int row, int k, int R) {
  const int kb = 2 * k;
  return (kb >> 4) * (R * 16) + (row >> 3) * 128 + (row & 7) * 16 + (kb & 15);
}

// v = p0 + p1 + p2 in bf16 (each the rounding of what is left): |error| < 2^-26 |v|.
// Eight consecutive K elements (k0 a multiple of 8) of one row as the three
// split planes, each one 16-byte core-matrix row written with one store.
__device__ __forceinline__ void split3_store8(uint8_t *base, uint32_t stride, int off, const float (&v)[8]) {
  uint32_t w[3][4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    uint32_t pp[3][2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const float x = v[2 * e + h];
      const __nv_bfloat16 p0 = __float2bfloat16_rn(x);
      const float r1 = x - __bfloat162float(p0);
      const __nv_bfloat16 p1 = __float2bfloat16_rn(r1);
      const __nv_bfloat16 p2 = __float2bfloat16_rn(r1 - __bfloat162float(p1));
      pp[0][h] = __bfloat16_as_ushort(p0);
      pp[1][h] = __bfloat16_as_ushort(p1);
      pp[2][h] = __bfloat16_as_ushort(p2);
    }
#pragma unroll
    for (int j = 0; j < 3; ++j) w[j][e] = pp[j][0] | (pp[j][1] << 16);
  }
#pragma unroll
  for (int j = 0; j < 3; ++j)
    *reinterpret_cast<uint4 *>(base + j * stride + off) = make_uint4(w[j][0], w[j][1], w[j][2], w[j][3]);
}

// v = p0 + p1 in bf16 (|error| < 2^-17 |v|), planes at base and base + stride.
__device__ __forceinline__ void split2_store8(uint8_t *base, uint32_t stride, int off, const float (&v)[8]) {
  uint32_t w0[4], w1[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    uint32_t p0[2], p1[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const float x = v[2 * e + h];
      const __nv_bfloat16 hi = __float2bfloat16_rn(x);
      const __nv_bfloat16 lo = __float2bfloat16_rn(x - __bfloat162float(hi));
      p0[h] = __bfloat16_as_ushort(hi);
      p1[h] = __bfloat16_as_ushort(lo);
    }
    w0[e] = p0[0] | (p0[1] << 16);
    w1[e] = p1[0] | (p1[1] << 16);
  }
  *reinterpret_cast<uint4 *>(base + off) = make_uint4(w0[0], w0[1], w0[2], w0[3]);
  *reinterpret_cast<uint4 *>(base + stride + off) = make_uint4(w1[0], w1[1], w1[2], w1[3]);
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t s) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(s));
  return d;
}

// bf16 entries i0 and i1 (< 2^nbits <= 16) of a table packed two per word,
// returned as one packed pair (i0 in the low half): byte permutes pick from
// four entries at a time, bits 2 and 3 of the index select between them.
__device__ __forceinline__ uint32_t lut2(const uint32_t *t, uint32_t i0, uint32_t i1, int nbits) {
  const uint32_t sel = (0x22u * (i0 & 3u) + 0x10u) | ((0x22u * (i1 & 3u) + 0x10u) << 8);
  uint32_t r = prmt(t[0], t[1], sel);
  if (nbits > 2) {
    const uint32_t m2 = ((i0 & 4u) ? 0xffffu : 0u) | ((i1 & 4u) ? 0xffff0000u : 0u);
    r = (prmt(t[2], t[3], sel) & m2) | (r & ~m2);
    if (nbits > 3) {
      uint32_t r8 = prmt(t[4], t[5], sel);
      r8 = (prmt(t[6], t[7], sel) & m2) | (r8 & ~m2);
      const uint32_t m3 = ((i0 & 8u) ? 0xffffu : 0u) | ((i1 & 8u) ? 0xffff0000u : 0u);
      r = (r8 & m3) | (r & ~m3);
    }
  }
  return r;
}

// Codes of elements `bit` and `bit + 1` from nb plane words.
__device__ __forceinline__ void code_pair(const uint32_t (&pw)[4], int nb, int bit, uint32_t &i0, uint32_t &i1) {
  i0 = 0u;
  i1 = 0u;
#pragma unroll
  for (int p = 0; p < 4; ++p)
    if (p < nb) {
      const uint32_t x = (pw[p] >> bit) & 3u;
      i0 |= (x & 1u) << p;
      i1 |= (x >> 1) << p;
    }
}

template <int D>
__global__ void __launch_bounds__(BT, 1) bidir_tile_kernel(BidirArgs a) {
  constexpr int DP = 2 * D;                        // rotated-domain width of Q/K
  constexpr uint32_t Q_BYTES = BQ * DP * 2;        // one split plane
  constexpr uint32_t K_BYTES = BK * DP * 2;
  constexpr uint32_t P_BYTES = BQ * BK * 2;
  constexpr uint32_t V_BYTES = D * BK * 2;
  constexpr uint32_t IDESC_S = sm100::idesc_bf16(128, BK);
  constexpr uint32_t IDESC_O = sm100::idesc_bf16(128, D);
  constexpr uint32_t STG = 4608;                   // one stage of compressed rows
  static_assert(BT == PR * BQ && BQ == 2 * BK && D == BK && BK == 64 && (PR == 2 || PR == 4), "thread mapping");
  constexpr int CPT = 16 * BK / BT;   // 8-column chunks of K_rot per thread (16 per key row)
  constexpr int TPT = 8 * D / BT;     // 8-key chunks of V_rot^T per thread (8 per coordinate)
  constexpr int KPT = BK / PR;        // keys (scores) and output columns per thread
  extern __shared__ __align__(128) float smem_b[];
  // each operand is stored as bf16 split planes (three, two for P)
  uint8_t *qs3 = reinterpret_cast<uint8_t *>(smem_b);
  uint8_t *ks3 = qs3 + 3 * Q_BYTES;
  uint8_t *ps3 = ks3 + 3 * K_BYTES;
  uint8_t *vs3 = ps3 + 2 * P_BYTES;
  float *nuk = reinterpret_cast<float *>(vs3 + 3 * V_BYTES);  // [BK]
  // two stages of one key tile's compressed rows, copied a tile ahead:
  // key planes, (nu, rho), the two value groups' words, value norms
  uint8_t *stg0 = reinterpret_cast<uint8_t *>(nuk + BK);
  // the three bf16 split planes of every key and value centroid, two entries
  // per word: K_rot's MSE half and V_rot are table lookups
  __shared__ __align__(16) uint16_t tabk[3][8], tabv[3][16];
  __shared__ float vns[BK];        // value norms of the current key tile
  __shared__ float xmax[PR][BQ];   // the parts' tile maxima of each query row
  __shared__ float lsum_s[PR][BQ];
  __shared__ __align__(8) uint64_t mbS, mbO, fin[4], kvf[2];
  __shared__ uint32_t tmem_s;
  __shared__ int abort_s;

  const int tid = threadIdx.x, warp = tid >> 5;
  const int r = tid & (BQ - 1), hf = tid >> 7;   // query row (TMEM lane), part of its keys / columns
  const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int kvh = h / (a.H / a.Hkv);
  const int64_t bh = static_cast<int64_t>(b) * a.Hkv + kvh;
  const int q0 = qt * BQ;
  const int mbk = a.books.mse_bits_k, planes_k = mbk + a.books.qjl, nbv = a.books.bits_v;
  if (tid < 16) {
#pragma unroll
    for (int w = 0; w < 2; ++w) {
      const float v = w == 0 ? (tid < 8 && tid < (1 << mbk) ? a.books.ck[tid] : 0.f)
                             : (tid < (1 << nbv) ? a.books.cv[tid] : 0.f);
      const __nv_bfloat16 p0 = __float2bfloat16_rn(v);
      const float r1 = v - __bfloat162float(p0);
      const __nv_bfloat16 p1 = __float2bfloat16_rn(r1);
      const __nv_bfloat16 p2 = __float2bfloat16_rn(r1 - __bfloat162float(p1));
      uint16_t *t = w == 0 ? &tabk[0][0] : &tabv[0][0];
      const int ne = w == 0 ? 8 : 16;
      if (w == 1 || tid < 8) {
        t[0 * ne + tid] = __bfloat16_as_ushort(p0);
        t[1 * ne + tid] = __bfloat16_as_ushort(p1);
        t[2 * ne + tid] = __bfloat16_as_ushort(p2);
      }
    }
  }
  if (warp == 0) sm100::tmem_alloc(&tmem_s, 512);
  if (tid == 0) {
    sm100::mbar_init(&mbS, 4);
    sm100::mbar_init(&mbO, 2);
    for (int i = 0; i < 4; ++i) sm100::mbar_init(&fin[i], 1);
    sm100::mbar_init(&kvf[0], 1);
    sm100::mbar_init(&kvf[1], 1);
    abort_s = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  // query tile: row r = query q0 + r (rows past Lq are zero), the DP / PR
  // columns of part hf, read as 16-byte loads all in flight at once
  {
    constexpr int QC = DP / PR;
    const int qi = q0 + r;
    float qv[QC];
    if (qi < a.Lq) {
      const float4 *src = reinterpret_cast<const float4 *>(
          a.qrot + ((static_cast<int64_t>(b) * a.H + h) * a.Lq + qi) * DP + hf * QC);
#pragma unroll
      for (int c = 0; c < QC / 4; ++c) {
        const float4 v = src[c];
        qv[4 * c] = v.x; qv[4 * c + 1] = v.y; qv[4 * c + 2] = v.z; qv[4 * c + 3] = v.w;
      }
    } else {
#pragma unroll
      for (int c = 0; c < QC; ++c) qv[c] = 0.f;
    }
#pragma unroll
    for (int c = 0; c < QC; c += 8) {
      float v8[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) v8[e] = qv[c + e];
      split3_store8(qs3, Q_BYTES, kmaj16(r, hf * QC + c, BQ), v8);
    }
  }
  sm100::fence_async_smem();
  sm100::fence_before_sync();
  __syncthreads();
  sm100::fence_after_sync();
  // columns: three small-product S accumulators, two for the leading hi*hi
  // product, two O accumulators (warps 0-3 issue S, warps 0-1 issue O, each
  // lane 0 into its own accumulators, so the MMAs are issued in parallel and
  // no accumulator takes a chain longer than 16)
  constexpr int NBIG = 2;
  const uint32_t tm = tmem_s;
  const uint32_t tS0 = tm, tSb = tm + BK, tO = tm + 3 * BK, tS1 = tm + 4 * BK, tS2 = tm + 5 * BK,
                 tO2 = tm + 6 * BK;
  const uint32_t a_q = sm100::smem_addr(qs3), a_k = sm100::smem_addr(ks3);
  const uint32_t a_p = sm100::smem_addr(ps3), a_v = sm100::smem_addr(vs3);
  const int lq = warp & 3;    // this warp's TMEM lane quarter

  // stage layout (bytes): key planes [0, 2048), (nu, rho) [2048, 2304),
  // value words [2304, 4352), value norms [4352, 4480)
  auto issue_tile = [&](int jt) {
    const int j0 = jt * BK;
    uint8_t *st = stg0 + (jt & 1) * STG;
    const uint32_t n = static_cast<uint32_t>(min(static_cast<int64_t>(BK), a.rows_cap - j0));
    const uint32_t ng = n / 32;
    const uint32_t bk_ = n * planes_k * (D / 8), bs = n * 4, bv = ng * nbv * D * 4, bn = n * 2;
    sm100::mbar_expect_tx(&kvf[jt & 1], bk_ + bs + bv + bn);
    sm100::bulk_g2s(st, a.kcode + (bh * a.rows_cap + j0) * planes_k * (D / 8), bk_, &kvf[jt & 1]);
    sm100::bulk_g2s(st + 2048, a.kscale + (bh * a.rows_cap + j0) * 2, bs, &kvf[jt & 1]);
    sm100::bulk_g2s(st + 2304, a.vcode + (bh * (a.rows_cap / 32) + j0 / 32) * nbv * D, bv, &kvf[jt & 1]);
    sm100::bulk_g2s(st + 4352, a.vnorm + bh * a.rows_cap + j0, bn, &kvf[jt & 1]);
  };
  const int ntiles = (a.T + BK - 1) / BK;
  // thread 0: the parity of the last copy issued into each stage (-1: none)
  int last_par[2] = {-1, -1};
  auto issue_next = [&](int jt) {
    issue_tile(jt);
    last_par[jt & 1] = (jt >> 1) & 1;
  };
  if (tid == 0) {
    if (ntiles > 0) issue_next(0);
    if (ntiles > 1) issue_next(1);
  }
  // The tile loop is software-pipelined so that each MMA set overlaps the
  // CUDA-core work of the next step:
  //   softmax(j) -> P(j) | issue O(j) | expand K(j+1) while O(j) runs |
  //   issue S(j+1) | wait O(j) | expand V(j+1) while S(j+1) runs | wait S(j+1)
  // Buffers: K_rot (ks3) is rewritten once S(j) has completed, V_rot (vs3)
  // and P (ps3) once O(j) has; the nu_k / nu_v arrays of tile j+1 are
  // written after softmax(j) has read tile j's.  A two-stage ring holds the
  // compressed rows; tile j+2 is copied into the stage of tile j once both of
  // its expansions are done.
  auto expand_k = [&](int jt) {
    const int j0 = jt * BK;
    const uint8_t *st = stg0 + (jt & 1) * STG;
      // ---- key tile: thread (row tid % BK, q = tid / BK) writes CPT of the 16
      // 8-column chunks of one key row (chunk k: half k / 8 (the MSE half
      // c[idx], or the sign half +-coef rho), word (k / 4) % 2, slice k % 4);
      // value tile: thread (coordinate, group, slice) writes TPT 8-key chunks of
      // V_rot^T
      {
        const int row = tid % BK, qk = tid / BK;
        const int half = (qk * CPT) >> 3, w = ((qk * CPT) >> 2) & 1;   // the same for all CPT chunks
        const int j = j0 + row;
        const bool ok = j < a.T;
        const uint32_t *krow = reinterpret_cast<const uint32_t *>(st + row * planes_k * (D / 8));
        const uint32_t sc = ok ? reinterpret_cast<const uint32_t *>(st + 2048)[row] : 0u;
        const float nu = tq_half_to_f32(static_cast<uint16_t>(sc & 0xffffu));
        const float rho = tq_half_to_f32(static_cast<uint16_t>(sc >> 16));
        if (qk == 0) nuk[row] = ok ? nu : 0.f;
        uint32_t pw[4] = {0u, 0u, 0u, 0u};
  #pragma unroll
        for (int p = 0; p < 4; ++p)
          if (p < planes_k) pw[p] = krow[p * (D / 32) + w];
        uint32_t pos[3] = {0u, 0u, 0u};
        uint32_t sgn = 0u;
        if (half == 1) {
          // the sign half is +-qv: its split, negated where the sign bit is 0
          const float qv = a.qjl_coef * rho;
          const __nv_bfloat16 p0 = __float2bfloat16_rn(qv);
          const float r1 = qv - __bfloat162float(p0);
          const __nv_bfloat16 p1 = __float2bfloat16_rn(r1);
          const __nv_bfloat16 p2 = __float2bfloat16_rn(r1 - __bfloat162float(p1));
          const uint32_t u[3] = {__bfloat16_as_ushort(p0), __bfloat16_as_ushort(p1), __bfloat16_as_ushort(p2)};
  #pragma unroll
          for (int p = 0; p < 3; ++p) pos[p] = (ok && a.books.qjl) ? (u[p] | (u[p] << 16)) : 0u;
  #pragma unroll
          for (int p = 0; p < 4; ++p)
            if (p == mbk) sgn = pw[p];
        }
        const uint32_t *tk32 = reinterpret_cast<const uint32_t *>(&tabk[0][0]);
  #pragma unroll
        for (int ci = 0; ci < CPT; ++ci) {
          const int c8 = (qk * CPT + ci) & 3;
          uint32_t o[3][4];
  #pragma unroll
          for (int e2 = 0; e2 < 4; ++e2) {
            const int bit = 8 * c8 + 2 * e2;
            if (half == 0) {
              uint32_t i0, i1;
              code_pair(pw, mbk, bit, i0, i1);
  #pragma unroll
              for (int p = 0; p < 3; ++p) o[p][e2] = ok ? lut2(tk32 + 4 * p, i0, i1, mbk) : 0u;
            } else {
              const uint32_t sb = ~(sgn >> bit);
              const uint32_t neg = ((sb & 1u) << 15) | ((sb & 2u) << 30);
  #pragma unroll
              for (int p = 0; p < 3; ++p) o[p][e2] = pos[p] ^ (pos[p] ? neg : 0u);
            }
          }
          const int off = kmaj16(row, half * D + 32 * w + 8 * c8, BK);
  #pragma unroll
          for (int p = 0; p < 3; ++p)
            *reinterpret_cast<uint4 *>(ks3 + p * K_BYTES + off) = make_uint4(o[p][0], o[p][1], o[p][2], o[p][3]);
        }
      }
  };
  auto expand_v = [&](int jt) {
    const int j0 = jt * BK;
    const uint8_t *st = stg0 + (jt & 1) * STG;
      if (tid < BK)
        vns[tid] = j0 + tid < a.T ? tq_half_to_f32(reinterpret_cast<const uint16_t *>(st + 4352)[tid]) : 0.f;
      {
        // V_rot^T: centroids only (the value norms scale P instead)
        const int coord = tid % D, g = (tid / D) & 1, th = tid / (2 * D);   // th: which TPT slices
        const int jg = j0 + 32 * g;
        uint32_t vw[4] = {0u, 0u, 0u, 0u};
        if (jg < a.T)
          for (int p = 0; p < nbv; ++p)
            vw[p] = reinterpret_cast<const uint32_t *>(st + 2304)[(g * nbv + p) * D + coord];
        const uint32_t *tv32 = reinterpret_cast<const uint32_t *>(&tabv[0][0]);
  #pragma unroll
        for (int t8 = TPT * th; t8 < TPT * th + TPT; ++t8) {
          uint32_t o[3][4];
  #pragma unroll
          for (int e2 = 0; e2 < 4; ++e2) {
            uint32_t i0, i1;
            code_pair(vw, nbv, 8 * t8 + 2 * e2, i0, i1);
  #pragma unroll
            for (int p = 0; p < 3; ++p) o[p][e2] = lut2(tv32 + 8 * p, i0, i1, nbv);
          }
          const int off = kmaj16(coord, 32 * g + 8 * t8, D);
  #pragma unroll
          for (int p = 0; p < 3; ++p)
            *reinterpret_cast<uint4 *>(vs3 + p * V_BYTES + off) = make_uint4(o[p][0], o[p][1], o[p][2], o[p][3]);
        }
      }
  };
  auto issue_s = [&]() {
      // ---- S = Q_rot K_rot^T (M = 128 queries, N = 64 keys, K = 2d): the six
      // split products of order <= 2 (about 2^-26 relative); warp 0 issues
      // a2 b0 + a1 b1, warp 1 a0 b2 + a1 b0, warp 2 a0 b1, warp 3 the K steps
      // of a0 b0 alternating over two accumulators
      if ((tid & 31) == 0 && warp < 4) {
        constexpr uint32_t LA = BQ * 16, LB = BK * 16;
        if (warp < 3) {
          const int pa[5] = {2, 1, 0, 1, 0}, pb[5] = {0, 1, 2, 0, 1};
          const int t0 = 2 * warp, nt = warp == 2 ? 1 : 2;
          const uint32_t d = warp == 0 ? tS0 : warp == 1 ? tS1 : tS2;
          int n = 0;
          for (int t = t0; t < t0 + nt; ++t)
  #pragma unroll
            for (int k = 0; k < DP / 16; ++k, ++n)
              sm100::mma_bf16_ss(d, sm100::smem_desc(a_q + pa[t] * Q_BYTES + k * 2 * LA, LA, 128),
                                 sm100::smem_desc(a_k + pb[t] * K_BYTES + k * 2 * LB, LB, 128), IDESC_S,
                                 n > 0 ? 1u : 0u);
        } else {
  #pragma unroll
          for (int k = 0; k < DP / 16; ++k)
            sm100::mma_bf16_ss(tSb + (k % NBIG) * BK, sm100::smem_desc(a_q + k * 2 * LA, LA, 128),
                               sm100::smem_desc(a_k + k * 2 * LB, LB, 128), IDESC_S, k >= NBIG ? 1u : 0u);
        }
        sm100::mma_commit(&mbS);
      }
  };

  float m = -CUDART_INF_F, l = 0.f;   // l: this half's share of the row sum
  uint32_t sph = 0, oph = 0;           // phases of the S and O commit barriers
  if (ntiles > 0) {
    if (!sm100::mbar_wait(&kvf[0], 0, a.wait_limit)) abort_s = 1;
    expand_k(0);
    expand_v(0);
    sm100::fence_async_smem();
    sm100::fence_before_sync();
    __syncthreads();
    sm100::fence_after_sync();
    if (!abort_s) issue_s();
  }
  // every thread passes every barrier of an iteration and leaves only right
  // after one, so a give-up (abort_s) takes the whole CTA out together
  for (int jt = 0; jt < ntiles; ++jt) {
    const int j0 = jt * BK;
    // S(jt) has completed
    if (!abort_s && !sm100::mbar_wait(&mbS, sph, a.wait_limit)) abort_s = 1;
    sph ^= 1;
    __syncthreads();
    if (abort_s) break;
    // the stage of tile jt is free (both its expansions are done): tile jt + 2
    if (tid == 0 && jt + 2 < ntiles) issue_next(jt + 2);
    sm100::fence_after_sync();
    // this part's KPT scores of row r: the five S accumulators added in fp32
    const int c0 = KPT * hf;
    float sv[KPT];
    {
      // the five accumulators in two rounds of loads in flight together
#pragma unroll
      for (int c = 0; c < KPT; c += 16) {
        uint32_t r0[16], r1[16], r2[16];
        sm100::tmem_ld16(sm100::tmem_lane(tS0 + c0 + c, lq), r0);
        sm100::tmem_ld16(sm100::tmem_lane(tS1 + c0 + c, lq), r1);
        sm100::tmem_ld16(sm100::tmem_lane(tS2 + c0 + c, lq), r2);
        sm100::wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e)
          sv[c + e] = (__uint_as_float(r0[e]) + __uint_as_float(r1[e])) + __uint_as_float(r2[e]);
        sm100::tmem_ld16(sm100::tmem_lane(tSb + c0 + c, lq), r0);
        sm100::tmem_ld16(sm100::tmem_lane(tSb + BK + c0 + c, lq), r1);
        sm100::wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) sv[c + e] += __uint_as_float(r0[e]) + __uint_as_float(r1[e]);
      }
    }
    float tmax = -CUDART_INF_F;
#pragma unroll
    for (int e = 0; e < KPT; ++e) {
      sv[e] = j0 + c0 + e < a.T ? a.scale * nuk[c0 + e] * sv[e] : -CUDART_INF_F;
      tmax = fmaxf(tmax, sv[e]);
    }
    xmax[hf][r] = tmax;
    __syncthreads();
    float tmx = -CUDART_INF_F;
#pragma unroll
    for (int i = 0; i < PR; ++i) tmx = fmaxf(tmx, xmax[i][r]);
    // the reference maximum of the row moves only when a tile exceeds it by
    // more than 8 (so exp(s - m) stays below e^8): the running output is
    // rescaled in tensor memory rarely, not on most tiles
    const float mn = tmx > m + 8.f ? tmx : m;
    const float corr = __expf(m - mn);
    // P nu_v (the value norms of the keys, so V_rot holds centroids only),
    // as a two-term bf16 split: its 2^-17 error reaches the output directly,
    // not through the softmax
    float ps = 0.f;
#pragma unroll
    for (int c = 0; c < KPT; c += 8) {
      float w[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float pe = __expf(sv[c + e] - mn);
        ps += pe;
        w[e] = pe * vns[c0 + c + e];
      }
      split2_store8(ps3, P_BYTES, kmaj16(r, c0 + c, BQ), w);
    }
    l = l * corr + ps;
    m = mn;
    // the running output lives in TMEM: rescale this half's columns of both
    // O accumulators when some row of the warp moved its maximum
    if (jt > 0 && __any_sync(TQ_FULL, corr != 1.f)) {
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int c = 0; c < KPT; c += 8) {
          const uint32_t t = (i ? tO2 : tO) + KPT * hf + c;
          uint32_t rr[8];
          sm100::tmem_ld8(sm100::tmem_lane(t, lq), rr);
          sm100::wait_ld();
#pragma unroll
          for (int e = 0; e < 8; ++e) rr[e] = __float_as_uint(__uint_as_float(rr[e]) * corr);
          sm100::tmem_st8(sm100::tmem_lane(t, lq), rr);
        }
      sm100::wait_st();
    }
    sm100::fence_async_smem();
    sm100::fence_before_sync();
    __syncthreads();
    sm100::fence_after_sync();
    // ---- O_tile = (P nu) V_rot (M = 128 queries, N = d, K = 64 keys): the
    // five products of a two-term P and a three-term V of order <= 2: warp 0
    // issues a1 b0 + a1 b1 + a0 b2 into O, warp 1 a0 b1 + a0 b0 into O2
    if ((tid & 31) == 0 && warp < 2) {
      constexpr uint32_t LA = BQ * 16, LB = D * 16;
      const int pa[5] = {1, 1, 0, 0, 0}, pb[5] = {0, 1, 2, 1, 0};
      const uint32_t d = warp == 0 ? tO : tO2;
      int n = 0;
      for (int t = 3 * warp; t < (warp == 0 ? 3 : 5); ++t)
#pragma unroll
        for (int k = 0; k < BK / 16; ++k, ++n)
          sm100::mma_bf16_ss(d, sm100::smem_desc(a_p + pa[t] * P_BYTES + k * 2 * LA, LA, 128),
                             sm100::smem_desc(a_v + pb[t] * V_BYTES + k * 2 * LB, LB, 128), IDESC_O,
                             (n > 0 || jt > 0) ? 1u : 0u);
      sm100::mma_commit(&mbO);
    }
    if (jt + 1 < ntiles) {
      // K(jt + 1) while O(jt) runs: S(jt) has read K_rot, softmax(jt) nu_k
      if (!abort_s && !sm100::mbar_wait(&kvf[(jt + 1) & 1], ((jt + 1) >> 1) & 1, a.wait_limit)) abort_s = 1;
      expand_k(jt + 1);
      sm100::fence_async_smem();
      sm100::fence_before_sync();
      __syncthreads();
      sm100::fence_after_sync();
      if (abort_s) break;
      issue_s();
    }
    // O(jt) has completed: V_rot, P and nu_v are free
    if (!abort_s && !sm100::mbar_wait(&mbO, oph, a.wait_limit)) abort_s = 1;
    oph ^= 1;
    if (jt + 1 < ntiles) {
      sm100::fence_after_sync();
      expand_v(jt + 1);
      sm100::fence_async_smem();
    } else {
      __syncthreads();
    }
    sm100::fence_after_sync();
  }
  // ---- out = Pi^T O_rot / l = D (H O_rot) / (sqrt(d) l), by the part-0 threads
  lsum_s[hf][r] = l;
  __syncthreads();
  if (hf == 0) {
    float o[D];
#pragma unroll
    for (int c = 0; c < D; c += 16) {
      uint32_t r1[16], r2[16];
      sm100::tmem_ld16(sm100::tmem_lane(tO + c, lq), r1);
      sm100::tmem_ld16(sm100::tmem_lane(tO2 + c, lq), r2);
      sm100::wait_ld();
#pragma unroll
      for (int e = 0; e < 16; ++e) o[c + e] = __uint_as_float(r1[e]) + __uint_as_float(r2[e]);
    }
    if (abort_s && q0 + r < a.Lq) {
      // a bounded wait gave up: this CTA's queries are reported as NaN
      float *dst = a.out + ((static_cast<int64_t>(b) * a.H + h) * a.Lq + q0 + r) * D;
#pragma unroll
      for (int i = 0; i < D; ++i) dst[i] = CUDART_NAN_F;
    } else if (q0 + r < a.Lq) {
#pragma unroll
      for (int s2 = 1; s2 < D; s2 <<= 1)
#pragma unroll
        for (int i = 0; i < D; ++i)
          if (!(i & s2)) {
            const float x = o[i], y = o[i + s2];
            o[i] = x + y;
            o[i + s2] = x - y;
          }
      float lt = 0.f;
#pragma unroll
      for (int i = 0; i < PR; ++i) lt += lsum_s[i][r];
      const float f = 1.0f / (sqrtf(static_cast<float>(D)) * lt);
      float *dst = a.out + ((static_cast<int64_t>(b) * a.H + h) * a.Lq + q0 + r) * D;
#pragma unroll
      for (int i = 0; i < D; ++i) {
        const float sgn = ((a.books.dneg[i >> 5] >> (i & 31)) & 1) ? -1.f : 1.f;
        dst[i] = o[i] * sgn * f;
      }
    }
  }
  // this CTA's copies have landed before its shared memory is released: the
  // last issued tile's phase completes (at once if it was consumed)
  if (tid == 0)
    for (int i = 0; i < 2; ++i)
      if (last_par[i] >= 0) sm100::mbar_wait(&kvf[i], static_cast<uint32_t>(last_par[i]), 1u << 20);
  // every MMA this thread issued has landed before tensor memory is released
  if ((tid & 31) == 0 && warp < 4) {
    sm100::mma_commit(&fin[warp]);
    sm100::mbar_wait(&fin[warp], 0, 1u << 20);
  }
  if (abort_s && tid == 0 && a.err) atomicExch(a.err, 1u);
  sm100::fence_before_sync();
  __syncthreads();
  sm100::fence_after_sync();
  if (warp == 0) sm100::tmem_dealloc(tm, 512);
}

}  // namespace

size_t bidir_workspace_bytes(const tq_codec *c, int B, int H, int Lq) {
  return sizeof(float) * static_cast<size_t>(B) * H * Lq * 2 * c->d;
}

int launch_bidir(const tq_codec *c, const void *q, int dtype, int B, int H, int Hkv, int Lq,
                 const tq_cache *cache, int T, float scale, const float *rc, const float *rs,
                 void *ws, float *out, cudaStream_t stream) {
  if (c->d != 64)
    return tq_fail(TQ_ERR_UNSUPPORTED, "bidirectional attention: built for d = 64 only");
  if (c->mse_bits_k > 3 || c->bits_v > 4)
    return tq_fail(TQ_ERR_UNSUPPORTED, "bidirectional attention: key MSE bits <= 3");
  BidirArgs a;
  a.q = q;
  a.dtype = dtype;
  a.B = B;
  a.H = H;
  a.Hkv = Hkv;
  a.Lq = Lq;
  a.T = T;
  a.kcode = cache->kcode;
  a.kscale = cache->kscale;
  a.vcode = cache->vcode;
  a.vnorm = cache->vnorm;
  a.rows_cap = cache->rows_cap;
  a.scale = scale;
  a.qjl_coef = c->qjl_k ? sqrtf(static_cast<float>(M_PI) / 2.0f) / c->d : 0.f;
  a.rc = rc;
  a.rs = rs;
  a.ST = c->ST_dev;
  a.qrot = static_cast<float *>(ws);
  a.out = out;
  a.err = nullptr;
  a.wait_limit = 1u << 26;
  if (const char *e = getenv("TQ_WAIT_LIMIT")) a.wait_limit = static_cast<uint32_t>(strtoul(e, nullptr, 10));
  a.books = c->books;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  constexpr int D = 64;
  const size_t qshm = c->qjl_k ? sizeof(float) * D * D : 0;
  const int64_t nq = static_cast<int64_t>(B) * H * Lq;
  const int64_t qb = (nq + 7) / 8;
  bidir_qprep_kernel<D><<<static_cast<int>(qb < 8LL * sms ? qb : 8LL * sms), 256, qshm, stream>>>(a);
  if (int e = tq_check_launch("bidir_qprep_kernel")) return e;
  constexpr size_t shm = 3 * (BQ * 2 * D * 2) + 3 * (BK * 2 * D * 2) + 2 * (BQ * BK * 2) +
                         3 * (D * BK * 2) + BK * 4 + 2 * 4608;
  static bool done[64] = {};
  if (dev < 64 && !done[dev]) {
    if (cudaFuncSetAttribute(bidir_tile_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(shm)) != cudaSuccess)
      return tq_check_launch("cudaFuncSetAttribute(bidir_tile)");
    done[dev] = true;
  }
  dim3 grid((Lq + BQ - 1) / BQ, H, B);
  cudaEvent_t ev0, ev1;
  tq_timing_events(&ev0, &ev1);
  if (ev0) cudaEventRecord(ev0, stream);
  bidir_tile_kernel<D><<<grid, BT, shm, stream>>>(a);
  if (int e = tq_check_launch("bidir_tile_kernel")) return e;
  if (ev1) cudaEventRecord(ev1, stream);
  tq_count_launch(2);
  return TQ_OK;
}
