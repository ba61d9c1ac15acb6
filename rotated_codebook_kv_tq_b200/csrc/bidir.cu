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

#include "tq_device.cuh"
#include "tq_sm100.cuh"

namespace {

constexpr int BQ = 128;   // queries per CTA
constexpr int BK = 64;    // keys per tile

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
// Plane j of the split lives at base + j * stride.
__device__ __forceinline__ void split3_store(uint8_t *base, uint32_t stride, int off, float v) {
  const __nv_bfloat16 a = __float2bfloat16_rn(v);
  const float r1 = v - __bfloat162float(a);
  const __nv_bfloat16 b = __float2bfloat16_rn(r1);
  const __nv_bfloat16 c = __float2bfloat16_rn(r1 - __bfloat162float(b));
  *reinterpret_cast<__nv_bfloat16 *>(base + off) = a;
  *reinterpret_cast<__nv_bfloat16 *>(base + stride + off) = b;
  *reinterpret_cast<__nv_bfloat16 *>(base + 2 * stride + off) = c;
}

// Eight consecutive K elements (k0 a multiple of 8) of one row: the three
// split planes are each one 16-byte core-matrix row, stored with one write.
__device__ __forceinline__ void split3_store8(uint8_t *base, uint32_t stride, int off, const float (&v)[8]) {
  uint32_t w0[4], w1[4], w2[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    uint32_t p0[2], p1[2], p2[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const float x = v[2 * e + h];
      const __nv_bfloat16 a = __float2bfloat16_rn(x);
      const float r1 = x - __bfloat162float(a);
      const __nv_bfloat16 b = __float2bfloat16_rn(r1);
      const __nv_bfloat16 c = __float2bfloat16_rn(r1 - __bfloat162float(b));
      p0[h] = __bfloat16_as_ushort(a);
      p1[h] = __bfloat16_as_ushort(b);
      p2[h] = __bfloat16_as_ushort(c);
    }
    w0[e] = p0[0] | (p0[1] << 16);
    w1[e] = p1[0] | (p1[1] << 16);
    w2[e] = p2[0] | (p2[1] << 16);
  }
  *reinterpret_cast<uint4 *>(base + off) = make_uint4(w0[0], w0[1], w0[2], w0[3]);
  *reinterpret_cast<uint4 *>(base + stride + off) = make_uint4(w1[0], w1[1], w1[2], w1[3]);
  *reinterpret_cast<uint4 *>(base + 2 * stride + off) = make_uint4(w2[0], w2[1], w2[2], w2[3]);
}

// The six split products of order <= 2: a0 b0 + a0 b1 + a1 b0 + a0 b2 + a1 b1 + a2 b0
// (about 2^-26 relative).  The five small ones go first into d_small; the
// K steps of a0 b0 go round-robin into `nbig` accumulators d_big + i * dstride
// (nbig = 1 folds everything into d_small, for the P V product).
__device__ __forceinline__ void mma6(uint32_t d_small, uint32_t d_big, uint32_t dstride, int nbig,
                                     uint32_t a, uint32_t astr, uint32_t b, uint32_t bstr,
                                     int ksteps, uint32_t lbo_a, uint32_t lbo_b, uint32_t idesc,
                                     bool acc_first) {
  const int pa[6] = {2, 1, 0, 1, 0, 0}, pb[6] = {0, 1, 2, 0, 1, 0};
  int n = 0;
#pragma unroll
  for (int t = 0; t < 5; ++t)
    for (int s = 0; s < ksteps; ++s, ++n)
      sm100::mma_bf16_ss(d_small, sm100::smem_desc(a + pa[t] * astr + s * 2 * lbo_a, lbo_a, 128),
                         sm100::smem_desc(b + pb[t] * bstr + s * 2 * lbo_b, lbo_b, 128), idesc,
                         (n > 0 || acc_first) ? 1u : 0u);
  for (int s = 0; s < ksteps; ++s) {
    const uint32_t d = nbig > 1 ? d_big + (s % nbig) * dstride : d_small;
    sm100::mma_bf16_ss(d, sm100::smem_desc(a + s * 2 * lbo_a, lbo_a, 128),
                       sm100::smem_desc(b + s * 2 * lbo_b, lbo_b, 128), idesc,
                       nbig > 1 ? (s >= nbig ? 1u : 0u) : 1u);
  }
}

template <int D>
__global__ void __launch_bounds__(BQ, 1) bidir_tile_kernel(BidirArgs a) {
  constexpr int DP = 2 * D;                        // rotated-domain width of Q/K
  constexpr uint32_t Q_BYTES = BQ * DP * 2;        // one of hi / lo
  constexpr uint32_t K_BYTES = BK * DP * 2;
  constexpr uint32_t P_BYTES = BQ * BK * 2;
  constexpr uint32_t V_BYTES = D * BK * 2;
  constexpr uint32_t IDESC_S = sm100::idesc_bf16(128, BK);
  constexpr uint32_t IDESC_O = sm100::idesc_bf16(128, D);
  constexpr int NPL = D / 32;
  extern __shared__ __align__(128) float smem_b[];
  // each operand is stored as three bf16 planes (split3_store)
  uint8_t *qs3 = reinterpret_cast<uint8_t *>(smem_b);
  uint8_t *ks3 = qs3 + 3 * Q_BYTES;
  uint8_t *ps3 = ks3 + 3 * K_BYTES;
  uint8_t *vs3 = ps3 + 3 * P_BYTES;
  float *nuk = reinterpret_cast<float *>(vs3 + 3 * V_BYTES);  // [BK]
  __shared__ float cks[TQ_MAX_LEVELS], cvs[TQ_MAX_LEVELS];
  __shared__ float vns[BK];   // value norms of the current key tile
  __shared__ __align__(8) uint64_t mb;
  __shared__ uint32_t tmem_s;
  __shared__ int abort_s;

  const int tid = threadIdx.x, warp = tid >> 5;
  const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int kvh = h / (a.H / a.Hkv);
  const int64_t bh = static_cast<int64_t>(b) * a.Hkv + kvh;
  const int q0 = qt * BQ;
  const int mbk = a.books.mse_bits_k, planes_k = mbk + a.books.qjl, nbv = a.books.bits_v;
  if (tid < TQ_MAX_LEVELS) {
    cks[tid] = a.books.ck[tid];
    cvs[tid] = a.books.cv[tid];
  }
  if (warp == 0) sm100::tmem_alloc(&tmem_s, 512);
  if (tid == 0) {
    sm100::mbar_init(&mb, 1);
    abort_s = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  // query tile: row tid = query q0 + tid (rows past Lq are zero)
  {
    const int qi = q0 + tid;
    const float *src = a.qrot + ((static_cast<int64_t>(b) * a.H + h) * a.Lq + qi) * DP;
    for (int k = 0; k < DP; ++k) split3_store(qs3, Q_BYTES, kmaj16(tid, k, BQ), qi < a.Lq ? src[k] : 0.f);
  }
  sm100::fence_async_smem();
  sm100::fence_before_sync();
  __syncthreads();
  sm100::fence_after_sync();
  // columns: S small-product accumulator, four hi*hi accumulators, O
  constexpr int NBIG = 4;
  const uint32_t tm = tmem_s, tS = tm, tSb = tm + BK, tO = tm + (1 + NBIG) * BK;
  const uint32_t a_q = sm100::smem_addr(qs3), a_k = sm100::smem_addr(ks3);
  const uint32_t a_p = sm100::smem_addr(ps3), a_v = sm100::smem_addr(vs3);

  float m = -CUDART_INF_F, l = 0.f;
  uint32_t phase = 0;
  for (int j0 = 0; j0 < a.T; j0 += BK) {
    // ---- key tile: thread (row tid % BK, half tid / BK) writes the MSE half
    // (c[idx]) or the sign half (+-coef rho) of one key row; value tile:
    // thread (coordinate tid % D, key group tid / D) writes 32 keys of V_rot^T.
    static_assert(BQ == 2 * BK && BQ == 2 * D && BK == 64, "thread mapping");
    if (tid < BK)
      vns[tid] = j0 + tid < a.T ? tq_half_to_f32(a.vnorm[bh * a.rows_cap + j0 + tid]) : 0.f;
    __syncthreads();
    {
      const int row = tid % BK, half = tid / BK;
      const int j = j0 + row;
      const bool ok = j < a.T;
      const uint8_t *krow = a.kcode + (bh * a.rows_cap + (ok ? j : 0)) * planes_k * (D / 8);
      const uint32_t sc = reinterpret_cast<const uint32_t *>(a.kscale)[bh * a.rows_cap + (ok ? j : 0)];
      const float nu = tq_half_to_f32(static_cast<uint16_t>(sc & 0xffffu));
      const float rho = tq_half_to_f32(static_cast<uint16_t>(sc >> 16));
      if (half == 0) nuk[row] = ok ? nu : 0.f;
      const float qv = a.qjl_coef * rho;
#pragma unroll 1
      for (int w = 0; w < D / 32; ++w) {
        uint32_t pw[4] = {0u, 0u, 0u, 0u};
#pragma unroll
        for (int p = 0; p < 4; ++p)
          if (p < planes_k) pw[p] = reinterpret_cast<const uint32_t *>(krow)[p * (D / 32) + w];
        uint32_t sgn = 0u;
#pragma unroll
        for (int p = 0; p < 4; ++p)
          if (p == mbk) sgn = pw[p];
#pragma unroll
        for (int c8 = 0; c8 < 4; ++c8) {
          float v[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int bit = 8 * c8 + e;
            if (half == 0) {
              int idx = 0;
#pragma unroll
              for (int p = 0; p < 3; ++p)
                if (p < mbk) idx |= ((pw[p] >> bit) & 1) << p;
              v[e] = ok ? cks[idx] : 0.f;
            } else {
              v[e] = (ok && a.books.qjl) ? (((sgn >> bit) & 1) ? qv : -qv) : 0.f;
            }
          }
          split3_store8(ks3, K_BYTES, kmaj16(row, half * D + 32 * w + 8 * c8, BK), v);
        }
      }
    }
    {
      const int coord = tid % D, g = tid / D;
      {
        const int jg = j0 + 32 * g;
        uint32_t vw[4] = {0u, 0u, 0u, 0u};
        if (jg < a.T)
          for (int p = 0; p < nbv; ++p)
            vw[p] = a.vcode[(bh * (a.rows_cap / 32) + jg / 32) * nbv * D + p * D + coord];
#pragma unroll
        for (int t8 = 0; t8 < 4; ++t8) {
          float v[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int t = 8 * t8 + e;
            int idx = 0;
#pragma unroll
            for (int p = 0; p < 4; ++p)
              if (p < nbv) idx |= ((vw[p] >> t) & 1) << p;
            v[e] = jg + t < a.T ? vns[32 * g + t] * cvs[idx] : 0.f;
          }
          split3_store8(vs3, V_BYTES, kmaj16(coord, 32 * g + 8 * t8, D), v);
        }
      }
    }
    sm100::fence_async_smem();
    sm100::fence_before_sync();
    __syncthreads();
    sm100::fence_after_sync();
    // ---- S = Q_rot K_rot^T (M = 128 queries, N = 64 keys, K = 2d)
    if (tid == 0) {
      mma6(tS, tSb, BK, NBIG, a_q, Q_BYTES, a_k, K_BYTES, DP / 16, BQ * 16, BK * 16, IDESC_S, false);
      sm100::mma_commit(&mb);
    }
    if (!sm100::mbar_wait(&mb, phase)) abort_s = 1;
    phase ^= 1;
    __syncthreads();
    if (abort_s) break;
    sm100::fence_after_sync();
    // scores of 16 keys (c .. c+15) of this query row from the five accumulators
    auto scores16 = [&](int c, float (&v)[16]) {
      uint32_t r[16];
      sm100::tmem_ld16(sm100::tmem_lane(tS + c, warp), r);
      sm100::wait_ld();
#pragma unroll
      for (int e = 0; e < 16; ++e) v[e] = __uint_as_float(r[e]);
#pragma unroll
      for (int i = 0; i < NBIG; ++i) {
        sm100::tmem_ld16(sm100::tmem_lane(tSb + i * BK + c, warp), r);
        sm100::wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) v[e] += __uint_as_float(r[e]);
      }
#pragma unroll
      for (int e = 0; e < 16; ++e) v[e] = j0 + c + e < a.T ? a.scale * nuk[c + e] * v[e] : -CUDART_INF_F;
    };
    // pass 1: the tile's maximum; pass 2: probabilities into the P planes
    float tmax = -CUDART_INF_F;
#pragma unroll 1
    for (int c = 0; c < BK; c += 16) {
      float v[16];
      scores16(c, v);
#pragma unroll
      for (int e = 0; e < 16; ++e) tmax = fmaxf(tmax, v[e]);
    }
    const float mn = fmaxf(m, tmax);
    const float corr = __expf(m - mn);
    float ps = 0.f;
#pragma unroll 1
    for (int c = 0; c < BK; c += 16) {
      float v[16];
      scores16(c, v);
#pragma unroll
      for (int h8 = 0; h8 < 2; ++h8) {
        float w[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          w[e] = __expf(v[8 * h8 + e] - mn);
          ps += w[e];
        }
        split3_store8(ps3, P_BYTES, kmaj16(tid, c + 8 * h8, BQ), w);
      }
    }
    l = l * corr + ps;
    m = mn;
    // the running output lives in TMEM (columns tO): rescale a warp's rows
    // when some row's maximum moved, before the P V MMAs add this tile
    if (j0 > 0 && __any_sync(TQ_FULL, corr != 1.f)) {
#pragma unroll
      for (int c = 0; c < D; c += 8) {
        uint32_t r[8];
        sm100::tmem_ld8(sm100::tmem_lane(tO + c, warp), r);
        sm100::wait_ld();
#pragma unroll
        for (int e = 0; e < 8; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * corr);
        sm100::tmem_st8(sm100::tmem_lane(tO + c, warp), r);
      }
      sm100::wait_st();
    }
    sm100::fence_async_smem();
    sm100::fence_before_sync();
    __syncthreads();
    sm100::fence_after_sync();
    // ---- O_tile = P V_rot (M = 128 queries, N = d, K = 64 keys)
    if (tid == 0) {
      mma6(tO, tO, 0, 1, a_p, P_BYTES, a_v, V_BYTES, BK / 16, BQ * 16, D * 16, IDESC_O, j0 > 0);
      sm100::mma_commit(&mb);
    }
    if (!sm100::mbar_wait(&mb, phase)) abort_s = 1;
    phase ^= 1;
    __syncthreads();
    if (abort_s) break;
    sm100::fence_after_sync();
  }
  float o[D];
#pragma unroll
  for (int c = 0; c < D; c += 16) {
    uint32_t r[16];
    sm100::tmem_ld16(sm100::tmem_lane(tO + c, warp), r);
    sm100::wait_ld();
#pragma unroll
    for (int e = 0; e < 16; ++e) o[c + e] = __uint_as_float(r[e]);
  }
  // ---- out = Pi^T O_rot / l = D (H O_rot) / (sqrt(d) l)
  if (!abort_s && q0 + tid < a.Lq) {
#pragma unroll
    for (int s = 1; s < D; s <<= 1)
#pragma unroll
      for (int i = 0; i < D; ++i)
        if (!(i & s)) {
          const float x = o[i], y = o[i + s];
          o[i] = x + y;
          o[i + s] = x - y;
        }
    const float f = 1.0f / (sqrtf(static_cast<float>(D)) * l);
    float *dst = a.out + ((static_cast<int64_t>(b) * a.H + h) * a.Lq + q0 + tid) * D;
#pragma unroll
    for (int i = 0; i < D; ++i) {
      const float sgn = ((a.books.dneg[i >> 5] >> (i & 31)) & 1) ? -1.f : 1.f;
      dst[i] = o[i] * sgn * f;
    }
  }
  if (abort_s) {
    sm100::mbar_wait(&mb, phase, 1u << 20);
    if (tid == 0 && a.err) atomicExch(a.err, 1u);
  }
  sm100::fence_before_sync();
  __syncthreads();
  sm100::fence_after_sync();
  if (warp == 0) sm100::tmem_dealloc(tm, 512);
  (void)NPL;
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
  constexpr size_t shm = 3 * (BQ * 2 * D * 2) + 3 * (BK * 2 * D * 2) + 3 * (BQ * BK * 2) +
                         3 * (D * BK * 2) + BK * 4;
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
  bidir_tile_kernel<D><<<grid, BQ, shm, stream>>>(a);
  if (int e = tq_check_launch("bidir_tile_kernel")) return e;
  if (ev1) cudaEventRecord(ev1, stream);
  tq_count_launch(2);
  return TQ_OK;
}
