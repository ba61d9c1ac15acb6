// Vector-search index and inner-product scan over TurboQuant_prod codes, d = 1536.
//
// "Google presenta TurboQuant ..." (7minutos.es), "Velocidad y eficiencia de
// indexacion": nearest-neighbour search over data-oblivious codes, so building
// the index is one encode pass with no training; "Eliminacion del sesgo
// interno del producto": (b-1) MSE bits plus the 1-bit QJL residual sketch give
// an unbiased inner-product estimate.  "TurboQuant: Jak rozwiazac ..."
// (securhub.pl), "Zaskakujace przyspieszenie baz wektorowych": the same use for
// vector databases.
//
// The rotation for d = 1536 (not a power of two) is Pi = (H_12 kron H_128)
// diag(D) / sqrt(1536): H_128 is the Sylvester matrix, H_12 the Paley type-I
// matrix over GF(11).  A warp holds one row with coordinate
// i = 128 j1 + 32 k + lane in register (j1, k): H_128 runs on shuffles inside
// each 128-block and H_12 mixes the 12 blocks in registers.
//
// Encoding a database row (tq_index_build):
//   ix_encode_kernel   norm, rotation, 3-bit codes -> MSE bit planes, residual
//                      r written as bf16 hi | lo into a scratch matrix [n][2d]
//   ix_gemm_kernel     z = S r for 128 x 256 tiles: tcgen05 kind::f16 MMAs of
//                      [r_hi | r_lo] against [S | S] (S is exactly bf16),
//                      fp32 in tensor memory, sign bits -> the QJL plane.
#include <math_constants.h>

#include <vector>

#include "tq_device.cuh"
#include "tq_sm100.cuh"

namespace {

constexpr int XD = 1536;
constexpr int XNB = 12;          // 128-blocks
constexpr int XW = XD / 32;      // 48 words per plane row

struct IxArgs {
  const float *x;        // [n][XD] fp32
  int64_t n;
  uint8_t *kcode;        // [n][planes][XD/8]
  uint16_t *kscale;      // [n][2]
  uint16_t *rbuf;        // [n][2*XD] bf16 residual hi | lo
  uint32_t h12[XNB];     // row masks of H_12: bit j set <=> entry -1
  uint32_t dneg[XW];
  float ck[TQ_MAX_LEVELS], tk[TQ_MAX_LEVELS];
  int mbk;
  uint32_t *status;
};

// x[j1][k] holds coordinate 128 j1 + 32 k + lane; y = (H_12 kron H_128) x.
__device__ __forceinline__ void rotate1536(float (&x)[XNB][4], const uint32_t (&h12)[XNB],
                                           int lane) {
#pragma unroll
  for (int j1 = 0; j1 < XNB; ++j1) tq_warp_wht<4>(x[j1], lane);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    float t[XNB];
#pragma unroll
    for (int i1 = 0; i1 < XNB; ++i1) {
      float s = 0.f;
#pragma unroll
      for (int j1 = 0; j1 < XNB; ++j1) s += ((h12[i1] >> j1) & 1) ? -x[j1][k] : x[j1][k];
      t[i1] = s;
    }
#pragma unroll
    for (int i1 = 0; i1 < XNB; ++i1) x[i1][k] = t[i1];
  }
}

__global__ void __launch_bounds__(256) ix_encode_kernel(IxArgs a) {
  __shared__ float cks[TQ_MAX_LEVELS], tks[TQ_MAX_LEVELS];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x < TQ_MAX_LEVELS) {
    cks[threadIdx.x] = a.ck[threadIdx.x];
    tks[threadIdx.x] = a.tk[threadIdx.x];
  }
  __syncthreads();
  const int nl = 1 << a.mbk, planes = a.mbk + 1;
  for (int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + warp; row < a.n;
       row += static_cast<int64_t>(gridDim.x) * 8) {
    const float *src = a.x + row * XD;
    float x[XNB][4];
    bool finite = true;
    float ss = 0.f;
#pragma unroll
    for (int j1 = 0; j1 < XNB; ++j1)
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float v = src[128 * j1 + 32 * k + lane];
        finite &= isfinite(v);
        ss += v * v;
        x[j1][k] = v;
      }
    bool bad = __any_sync(TQ_FULL, !finite);
    float nu = sqrtf(tq_warp_sum(ss));
    if (!bad && isinf(__half2float(__float2half_rn(nu)))) bad = true;   // fp16 norm overflow
    if (bad) nu = 0.f;
    const bool zero = bad || !(nu > 0.f);
#pragma unroll
    for (int j1 = 0; j1 < XNB; ++j1)
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint32_t neg = (a.dneg[4 * j1 + k] >> lane) & 1u;
        x[j1][k] = zero ? 0.f : __uint_as_float(__float_as_uint(x[j1][k]) ^ (neg << 31));
      }
    rotate1536(x, a.h12, lane);
    const float inv = zero ? 0.f : 1.0f / (sqrtf(static_cast<float>(XD)) * nu);
    uint32_t mw[4][2];
#pragma unroll
    for (int p = 0; p < 4; ++p) mw[p][0] = mw[p][1] = 0u;
    float r2 = 0.f;
    uint16_t *rrow = a.rbuf + row * 2 * XD;
#pragma unroll
    for (int j1 = 0; j1 < XNB; ++j1)
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float u = x[j1][k] * inv;
        const int idx = tq_code(u, tks, nl - 1);
        const int w = 4 * j1 + k;
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          if (p < a.mbk) {
            const uint32_t word = __ballot_sync(TQ_FULL, (idx >> p) & 1);
            if (lane == (w & 31)) mw[p][w >> 5] = word;
          }
        }
        const float r = u - cks[idx];
        r2 += r * r;
        const __nv_bfloat16 hi = __float2bfloat16_rn(r);
        const __nv_bfloat16 lo = __float2bfloat16_rn(r - __bfloat162float(hi));
        const int i = 128 * j1 + 32 * k + lane;
        rrow[i] = __bfloat16_as_ushort(hi);
        rrow[XD + i] = __bfloat16_as_ushort(lo);
      }
    const float rho = sqrtf(tq_warp_sum(r2));
    uint32_t *krow = reinterpret_cast<uint32_t *>(a.kcode + row * planes * (XD / 8));
    for (int p = 0; p < a.mbk; ++p) {
      krow[p * XW + lane] = mw[p][0];
      if (lane < XW - 32) krow[p * XW + 32 + lane] = mw[p][1];
    }
    if (lane == 0) {
      const uint32_t pair = static_cast<uint32_t>(tq_f32_to_half(nu)) |
                            (static_cast<uint32_t>(tq_f32_to_half(rho)) << 16);
      reinterpret_cast<uint32_t *>(a.kscale)[row] = pair;
      if (bad && a.status) atomicAdd(a.status, 1u);
    }
  }
}

// ---------------------------------------------------------------------------
// C = A B^T on the tensor cores for A [M][KA] and B [N][KB] bf16 row-major
// (K contiguous), KA a multiple of KB: A's K range wraps over B (A = [r_hi |
// r_lo] against B = S gives S r_hi + S r_lo).  Tile 128 x 256, K chunks of 64
// through a 3-stage cp.async ring; fp32 accumulators in 256 TMEM columns.
// MODE 0 writes sign bits (z >= 0) of each row into a bit plane; MODE 1 writes
// the fp32 values.
// ---------------------------------------------------------------------------
struct GemmArgs {
  const uint16_t *A;
  const uint16_t *B;
  int64_t M;
  int N, KA, KB;
  uint8_t *plane;        // MODE 0: bit plane base, row stride plane_stride bytes
  int64_t plane_stride;
  float *out;            // MODE 1: [M][N]
  uint16_t *out_hl;      // MODE 2: [M][2N] bf16 hi | lo of scale * value
  float scale;
  uint32_t *status;
};

constexpr int GM = 128, GN = 256, GK = 64, GST = 3;
constexpr uint32_t GA_BYTES = GM * GK * 2, GB_BYTES = GN * GK * 2;

__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(sm100::smem_addr(dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

template <int MODE>
__global__ void __launch_bounds__(128, 1) ix_gemm_kernel(GemmArgs g) {
  extern __shared__ __align__(128) float gsm[];
  uint8_t *base = reinterpret_cast<uint8_t *>(gsm);
  __shared__ __align__(8) uint64_t mb[GST];
  __shared__ uint32_t tmem_s;
  __shared__ int abort_s;
  const int tid = threadIdx.x, warp = tid >> 5;
  const int64_t m0 = static_cast<int64_t>(blockIdx.x) * GM;
  const int n0 = blockIdx.y * GN;
  if (warp == 0) sm100::tmem_alloc(&tmem_s, 256);
  if (tid == 0) {
    for (int s = 0; s < GST; ++s) sm100::mbar_init(&mb[s], 1);
    abort_s = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  sm100::fence_before_sync();
  __syncthreads();
  sm100::fence_after_sync();
  const uint32_t tm = tmem_s;
  const int nk = g.KA / GK;

  auto load = [&](int kc) {
    uint8_t *As = base + (kc % GST) * (GA_BYTES + GB_BYTES);
    uint8_t *Bs = As + GA_BYTES;
    const int ka = kc * GK, kb = ka % g.KB;
    // A: 128 rows x 8 segments of 16 bytes; rows past M repeat the last row
    for (int e = tid; e < GM * 8; e += 128) {
      const int row = e >> 3, seg = e & 7;
      const int64_t r = m0 + row < g.M ? m0 + row : g.M - 1;
      cp_async16(As + seg * (GM * 16) + (row >> 3) * 128 + (row & 7) * 16, g.A + r * g.KA + ka + seg * 8);
    }
    for (int e = tid; e < GN * 8; e += 128) {
      const int row = e >> 3, seg = e & 7;
      const int r = n0 + row < g.N ? n0 + row : g.N - 1;
      cp_async16(Bs + seg * (GN * 16) + (row >> 3) * 128 + (row & 7) * 16,
                 g.B + static_cast<int64_t>(r) * g.KB + kb + seg * 8);
    }
  };

  for (int kc = 0; kc < GST - 1 && kc < nk; ++kc) {
    load(kc);
    cp_commit();
  }
  uint32_t ph = 0;   // bit s: parity to wait for on mb[s]
  for (int kc = 0; kc < nk; ++kc) {
    // make room: chunk kc + GST - 1 reuses the stage of chunk kc - 1
    const int nxt = kc + GST - 1;
    if (nxt < nk) {
      if (kc >= 1) {
        const int s = (kc - 1) % GST;
        if (!sm100::mbar_wait(&mb[s], (ph >> s) & 1)) abort_s = 1;
        ph ^= 1u << s;
      }
      load(nxt);
    }
    cp_commit();
    cp_wait<GST - 1>();
    sm100::fence_async_smem();
    sm100::fence_before_sync();
    __syncthreads();
    sm100::fence_after_sync();
    if (abort_s) break;
    if (tid == 0) {
      const int s = kc % GST;
      const uint32_t a_addr = sm100::smem_addr(base + s * (GA_BYTES + GB_BYTES));
      const uint32_t b_addr = a_addr + GA_BYTES;
#pragma unroll
      for (int ks = 0; ks < GK / 16; ++ks)
        sm100::mma_bf16_ss(tm, sm100::smem_desc(a_addr + ks * 2 * (GM * 16), GM * 16, 128),
                           sm100::smem_desc(b_addr + ks * 2 * (GN * 16), GN * 16, 128),
                           sm100::idesc_bf16(GM, GN), (kc > 0 || ks > 0) ? 1u : 0u);
      sm100::mma_commit(&mb[s]);
    }
  }
  // drain: the loop waited chunk c's commit iff c + GST < nk
  if (!abort_s)
    for (int c = nk - GST > 0 ? nk - GST : 0; c < nk; ++c) {
      const int s = c % GST;
      if (!sm100::mbar_wait(&mb[s], (ph >> s) & 1)) abort_s = 1;
      ph ^= 1u << s;
    }
  __syncthreads();
  sm100::fence_after_sync();
  if (!abort_s) {
    const int64_t row = m0 + tid;
    for (int c0 = 0; c0 < GN; c0 += 32) {
      uint32_t z0[16], z1[16];
      sm100::tmem_ld16(sm100::tmem_lane(tm + c0, warp), z0);
      sm100::tmem_ld16(sm100::tmem_lane(tm + c0 + 16, warp), z1);
      sm100::wait_ld();
      if (row < g.M && n0 + c0 < g.N) {
        if (MODE == 0) {
          uint32_t word = 0u;
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            word |= (__uint_as_float(z0[c]) >= 0.f ? 1u : 0u) << c;
            word |= (__uint_as_float(z1[c]) >= 0.f ? 1u : 0u) << (16 + c);
          }
          reinterpret_cast<uint32_t *>(g.plane + row * g.plane_stride)[(n0 + c0) >> 5] = word;
        } else if (MODE == 2) {
          uint16_t *o = g.out_hl + row * 2 * g.N + n0 + c0;
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const float v = g.scale * __uint_as_float(c < 16 ? z0[c] : z1[c - 16]);
            const __nv_bfloat16 hi = __float2bfloat16_rn(v);
            const __nv_bfloat16 lo = __float2bfloat16_rn(v - __bfloat162float(hi));
            if (n0 + c0 + c < g.N) {
              o[c] = __bfloat16_as_ushort(hi);
              o[g.N + c] = __bfloat16_as_ushort(lo);
            }
          }
        } else {
          float *o = g.out + row * g.N + n0 + c0;
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            if (n0 + c0 + c < g.N) o[c] = __uint_as_float(z0[c]);
            if (n0 + c0 + 16 + c < g.N) o[16 + c] = __uint_as_float(z1[c]);
          }
        }
      }
    }
  } else if (tid == 0 && g.status) {
    atomicAdd(g.status, 1u << 31);
  }
  sm100::fence_before_sync();
  __syncthreads();
  sm100::fence_after_sync();
  if (warp == 0) sm100::tmem_dealloc(tm, 256);
}

// ---------------------------------------------------------------------------
// Queries: q' = Pi q (fp32 and bf16 hi | lo); q'' = S q' by ix_gemm_kernel<1>.
// ---------------------------------------------------------------------------
struct QrotArgs {
  const float *q;
  int nq;
  float *q1;            // [nq][XD]
  uint16_t *q1hl;       // [nq][2 XD] bf16 hi | lo
  uint32_t h12[XNB];
  uint32_t dneg[XW];
};

__global__ void __launch_bounds__(256) ix_qrot_kernel(QrotArgs a) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int qi = blockIdx.x * 8 + warp;
  if (qi >= a.nq) return;
  float x[XNB][4];
#pragma unroll
  for (int j1 = 0; j1 < XNB; ++j1)
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint32_t neg = (a.dneg[4 * j1 + k] >> lane) & 1u;
      const float v = a.q[static_cast<int64_t>(qi) * XD + 128 * j1 + 32 * k + lane];
      x[j1][k] = __uint_as_float(__float_as_uint(v) ^ (neg << 31));
    }
  rotate1536(x, a.h12, lane);
  const float inv = 1.0f / sqrtf(static_cast<float>(XD));
#pragma unroll
  for (int j1 = 0; j1 < XNB; ++j1)
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int i = 128 * j1 + 32 * k + lane;
      const float v = x[j1][k] * inv;
      a.q1[static_cast<int64_t>(qi) * XD + i] = v;
      const __nv_bfloat16 hi = __float2bfloat16_rn(v);
      const __nv_bfloat16 lo = __float2bfloat16_rn(v - __bfloat162float(hi));
      a.q1hl[static_cast<int64_t>(qi) * 2 * XD + i] = __bfloat16_as_ushort(hi);
      a.q1hl[static_cast<int64_t>(qi) * 2 * XD + XD + i] = __bfloat16_as_ushort(lo);
    }
}

// ---------------------------------------------------------------------------
// Scan: scores s_ij = nu_j (<q'_i, c[idx_j]> + sqrt(pi/2)/d rho_j <q''_i, 2 sigma_j - 1>)
// for 128 queries (TMEM lane = query) against 128-row database tiles, K = 1536
// in chunks of 64.  Database codes are dequantized per chunk into bf16 tiles
// c_hi, c_lo (c = c_hi + c_lo to ~2^-17) and s = +-1 (exact); the queries'
// q', q'' come as bf16 hi | lo.  Two fp32 accumulators:
//   D_m = q'_hi c_hi + q'_hi c_lo + q'_lo c_hi,   D_s = q''_hi s + q''_lo s.
// Each query lane keeps its top-k in registers over the CTA's tile range.
// ---------------------------------------------------------------------------
constexpr int SQ = 128, SR = 128, SK = 64;
constexpr int SKMAX = 16;                       // largest k of the top-k

struct ScanArgs {
  const uint16_t *q1hl;   // [nq][2 XD]
  const uint16_t *q2hl;   // [nq][2 XD]
  const uint8_t *kcode;
  const uint16_t *kscale;
  int64_t n;
  int nq, k;
  int tiles_per_cta;
  float coef;
  float ck[TQ_MAX_LEVELS];
  int mbk;
  float *cand_s;          // [nq][grid.y][k]
  int32_t *cand_i;
  uint32_t *err;
};

__device__ __forceinline__ int kmaj_off(int row, int k, int R) {   // bf16 element offset in bytes
  const int kb = 2 * k;
  return (kb >> 4) * (R * 16) + (row >> 3) * 128 + (row & 7) * 16 + (kb & 15);
}

__global__ void __launch_bounds__(128, 1) ix_scan_kernel(ScanArgs a) {
  constexpr uint32_t QB = SQ * SK * 2;         // one query operand chunk
  constexpr uint32_t RB = SR * SK * 2;         // one database operand chunk
  extern __shared__ __align__(128) float ssm[];
  uint8_t *base = reinterpret_cast<uint8_t *>(ssm);
  uint8_t *q1h = base, *q1l = q1h + QB, *q2h = q1l + QB, *q2l = q2h + QB;
  uint8_t *chi = q2l + QB, *clo = chi + RB, *sgn = clo + RB;
  __shared__ float cks[TQ_MAX_LEVELS];
  __shared__ float nus[SR], rhos[SR];
  __shared__ __align__(8) uint64_t mb;
  __shared__ uint32_t tmem_s;
  __shared__ int abort_s;
  const int tid = threadIdx.x, warp = tid >> 5;
  const int qb = blockIdx.x;
  if (tid < TQ_MAX_LEVELS) cks[tid] = a.ck[tid];
  if (warp == 0) sm100::tmem_alloc(&tmem_s, 256);
  if (tid == 0) {
    sm100::mbar_init(&mb, 1);
    abort_s = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  sm100::fence_before_sync();
  __syncthreads();
  sm100::fence_after_sync();
  const uint32_t tm = tmem_s, tDm = tm, tDs = tm + SR;
  const int planes = a.mbk + 1;
  const int q = qb * SQ + tid;
  float ts[SKMAX];
  int ti[SKMAX];
#pragma unroll
  for (int e = 0; e < SKMAX; ++e) {
    ts[e] = -CUDART_INF_F;
    ti[e] = 0x7fffffff;
  }
  uint32_t ph = 0;
  const int64_t ntiles = (a.n + SR - 1) / SR;
  const int64_t t_begin = static_cast<int64_t>(blockIdx.y) * a.tiles_per_cta;
  const int64_t t_end = t_begin + a.tiles_per_cta < ntiles ? t_begin + a.tiles_per_cta : ntiles;
  const uint32_t idesc = sm100::idesc_bf16(SQ, SR);
  for (int64_t t = t_begin; t < t_end && !abort_s; ++t) {
    const int64_t r0 = t * SR;
    {
      const int64_t r = r0 + tid < a.n ? r0 + tid : a.n - 1;
      const uint32_t sc = reinterpret_cast<const uint32_t *>(a.kscale)[r];
      nus[tid] = r0 + tid < a.n ? tq_half_to_f32(static_cast<uint16_t>(sc & 0xffffu)) : 0.f;
      rhos[tid] = tq_half_to_f32(static_cast<uint16_t>(sc >> 16));
    }
    for (int kc = 0; kc < XD / SK; ++kc) {
      const int k0 = kc * SK;
      // query operand chunks (rows past nq repeat the last query)
      const int qq = q < a.nq ? q : a.nq - 1;
      for (int seg = 0; seg < 8; ++seg) {
        const int off = seg * (SQ * 16) + (tid >> 3) * 128 + (tid & 7) * 16;
        cp_async16(q1h + off, a.q1hl + static_cast<int64_t>(qq) * 2 * XD + k0 + seg * 8);
        cp_async16(q1l + off, a.q1hl + static_cast<int64_t>(qq) * 2 * XD + XD + k0 + seg * 8);
        cp_async16(q2h + off, a.q2hl + static_cast<int64_t>(qq) * 2 * XD + k0 + seg * 8);
        cp_async16(q2l + off, a.q2hl + static_cast<int64_t>(qq) * 2 * XD + XD + k0 + seg * 8);
      }
      cp_commit();
      // database operand: thread tid dequantizes row r0 + tid, coordinates k0 .. k0+63
      {
        const int64_t r = r0 + tid < a.n ? r0 + tid : a.n - 1;
        const uint32_t *kr = reinterpret_cast<const uint32_t *>(a.kcode + r * planes * (XD / 8));
        uint32_t pw[5][2];
#pragma unroll
        for (int p = 0; p < 5; ++p)
#pragma unroll
          for (int w = 0; w < 2; ++w) pw[p][w] = p < planes ? kr[p * XW + (k0 >> 5) + w] : 0u;
#pragma unroll
        for (int w = 0; w < 2; ++w)
#pragma unroll 8
          for (int bit = 0; bit < 32; ++bit) {
            int idx = 0;
#pragma unroll
            for (int p = 0; p < 4; ++p)
              if (p < a.mbk) idx |= ((pw[p][w] >> bit) & 1) << p;
            const float c = cks[idx];
            const __nv_bfloat16 h = __float2bfloat16_rn(c);
            const __nv_bfloat16 l = __float2bfloat16_rn(c - __bfloat162float(h));
            const int off = kmaj_off(tid, 32 * w + bit, SR);
            *reinterpret_cast<__nv_bfloat16 *>(chi + off) = h;
            *reinterpret_cast<__nv_bfloat16 *>(clo + off) = l;
            const bool sb = (pw[planes - 1][w] >> bit) & 1;
            *reinterpret_cast<uint16_t *>(sgn + off) = sb ? 0x3F80u : 0xBF80u;   // +-1 in bf16
          }
      }
      cp_wait<0>();
      sm100::fence_async_smem();
      sm100::fence_before_sync();
      __syncthreads();
      sm100::fence_after_sync();
      if (tid == 0) {
        const uint32_t aq1h = sm100::smem_addr(q1h), aq1l = sm100::smem_addr(q1l);
        const uint32_t aq2h = sm100::smem_addr(q2h), aq2l = sm100::smem_addr(q2l);
        const uint32_t ach = sm100::smem_addr(chi), acl = sm100::smem_addr(clo), asg = sm100::smem_addr(sgn);
#pragma unroll
        for (int ks = 0; ks < SK / 16; ++ks) {
          const uint32_t oq = ks * 2 * (SQ * 16), orr = ks * 2 * (SR * 16);
          const uint32_t first = (kc > 0 || ks > 0) ? 1u : 0u;
          sm100::mma_bf16_ss(tDm, sm100::smem_desc(aq1h + oq, SQ * 16, 128), sm100::smem_desc(ach + orr, SR * 16, 128), idesc, first);
          sm100::mma_bf16_ss(tDm, sm100::smem_desc(aq1h + oq, SQ * 16, 128), sm100::smem_desc(acl + orr, SR * 16, 128), idesc, 1);
          sm100::mma_bf16_ss(tDm, sm100::smem_desc(aq1l + oq, SQ * 16, 128), sm100::smem_desc(ach + orr, SR * 16, 128), idesc, 1);
          sm100::mma_bf16_ss(tDs, sm100::smem_desc(aq2h + oq, SQ * 16, 128), sm100::smem_desc(asg + orr, SR * 16, 128), idesc, first);
          sm100::mma_bf16_ss(tDs, sm100::smem_desc(aq2l + oq, SQ * 16, 128), sm100::smem_desc(asg + orr, SR * 16, 128), idesc, 1);
        }
        sm100::mma_commit(&mb);
      }
      if (!sm100::mbar_wait(&mb, ph)) abort_s = 1;
      ph ^= 1;
      __syncthreads();
      if (abort_s) break;
    }
    if (abort_s) break;
    sm100::fence_after_sync();
    // scores of query `q` against the tile's rows; running top-k
    for (int c0 = 0; c0 < SR; c0 += 16) {
      uint32_t dm[16], ds[16];
      sm100::tmem_ld16(sm100::tmem_lane(tDm + c0, warp), dm);
      sm100::tmem_ld16(sm100::tmem_lane(tDs + c0, warp), ds);
      sm100::wait_ld();
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const int64_t r = r0 + c0 + c;
        if (r >= a.n) continue;
        const float s = nus[c0 + c] * fmaf(a.coef * rhos[c0 + c], __uint_as_float(ds[c]), __uint_as_float(dm[c]));
        if (s > ts[SKMAX - 1]) {
          ts[SKMAX - 1] = s;
          ti[SKMAX - 1] = static_cast<int>(r);
#pragma unroll
          for (int e = SKMAX - 1; e > 0; --e) {
            if (ts[e] > ts[e - 1]) {
              const float fs = ts[e];
              ts[e] = ts[e - 1];
              ts[e - 1] = fs;
              const int fi = ti[e];
              ti[e] = ti[e - 1];
              ti[e - 1] = fi;
            }
          }
        }
      }
    }
    sm100::fence_before_sync();
    __syncthreads();
    sm100::fence_after_sync();
  }
  if (!abort_s && q < a.nq) {
    float *cs = a.cand_s + (static_cast<int64_t>(q) * gridDim.y + blockIdx.y) * a.k;
    int32_t *ci = a.cand_i + (static_cast<int64_t>(q) * gridDim.y + blockIdx.y) * a.k;
#pragma unroll
    for (int e = 0; e < SKMAX; ++e)
      if (e < a.k) {
        cs[e] = ts[e];
        ci[e] = ti[e];
      }
  }
  if (abort_s) {
    sm100::mbar_wait(&mb, ph, 1u << 20);
    if (tid == 0 && a.err) atomicExch(a.err, 1u);
  }
  sm100::fence_before_sync();
  __syncthreads();
  sm100::fence_after_sync();
  if (warp == 0) sm100::tmem_dealloc(tm, 256);
}

// Merge the per-CTA candidate lists of each query: order (-score, index).
__global__ void ix_merge_kernel(const float *cs, const int32_t *ci, int nq, int lists, int k,
                                int32_t *idx, float *score) {
  const int q = blockIdx.x * blockDim.x + threadIdx.x;
  if (q >= nq) return;
  float bs[SKMAX];
  int bi[SKMAX];
  for (int e = 0; e < SKMAX; ++e) {
    bs[e] = -CUDART_INF_F;
    bi[e] = 0x7fffffff;
  }
  const int64_t base = static_cast<int64_t>(q) * lists * k;
  for (int c = 0; c < lists * k; ++c) {
    const float s = cs[base + c];
    const int j = ci[base + c];
    const bool better = s > bs[k - 1] || (s == bs[k - 1] && j < bi[k - 1]);
    if (!better) continue;
    bs[k - 1] = s;
    bi[k - 1] = j;
    for (int e = k - 1; e > 0; --e) {
      const bool up = bs[e] > bs[e - 1] || (bs[e] == bs[e - 1] && bi[e] < bi[e - 1]);
      if (!up) break;
      const float fs = bs[e];
      bs[e] = bs[e - 1];
      bs[e - 1] = fs;
      const int fi = bi[e];
      bi[e] = bi[e - 1];
      bi[e - 1] = fi;
    }
  }
  for (int e = 0; e < k; ++e) {
    idx[static_cast<int64_t>(q) * k + e] = bi[e];
    score[static_cast<int64_t>(q) * k + e] = bs[e];
  }
}

}  // namespace

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
namespace {

constexpr int64_t kIxBatch = 65536;   // rows encoded per residual-scratch batch

// Paley construction I for q = 11: H = I + [[0, 1^T], [-1, Q]] with the
// Jacobsthal matrix Q[i][j] = chi(j - i) of the quadratic character mod 11.
void paley12(uint32_t masks[12]) {
  int chi[11] = {0};
  for (int x = 1; x < 11; ++x) chi[(x * x) % 11] = 1;
  for (int a = 1; a < 11; ++a)
    if (chi[a] != 1) chi[a] = -1;
  int h[12][12];
  for (int i = 0; i < 12; ++i)
    for (int j = 0; j < 12; ++j) h[i][j] = 0;
  for (int j = 1; j < 12; ++j) {
    h[0][j] = 1;
    h[j][0] = -1;
  }
  for (int i = 0; i < 11; ++i)
    for (int j = 0; j < 11; ++j) h[i + 1][j + 1] = chi[((j - i) % 11 + 11) % 11];
  for (int i = 0; i < 12; ++i) h[i][i] += 1;
  for (int i = 0; i < 12; ++i) {
    masks[i] = 0;
    for (int j = 0; j < 12; ++j)
      if (h[i][j] < 0) masks[i] |= 1u << j;
  }
}

int sm_count() {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

template <int MODE>
int run_gemm(const GemmArgs &g, cudaStream_t stream) {
  constexpr int shm = GST * (GA_BYTES + GB_BYTES);
  static bool done[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !done[dev]) {
    if (cudaFuncSetAttribute(ix_gemm_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, shm) !=
        cudaSuccess)
      return tq_check_launch("cudaFuncSetAttribute(ix_gemm)");
    done[dev] = true;
  }
  dim3 grid(static_cast<unsigned>((g.M + GM - 1) / GM), (g.N + GN - 1) / GN);
  ix_gemm_kernel<MODE><<<grid, 128, shm, stream>>>(g);
  tq_count_launch(1);
  return tq_check_launch("ix_gemm_kernel");
}

bool index_codec_ok(const tq_codec *c) { return c->d == XD && c->qjl_k && c->mse_bits_k <= 4; }

int scan_grid_y(int64_t n, int nq) {
  const int64_t tiles = (n + SR - 1) / SR;
  const int qblocks = (nq + SQ - 1) / SQ;
  int64_t gy = sm_count() / qblocks;   // one wave: grid.x * grid.y <= SMs (one CTA per SM)
  if (gy > tiles) gy = tiles;
  return static_cast<int>(gy < 1 ? 1 : gy);
}

}  // namespace

extern "C" {

int tq_index_workspace(const tq_codec *c, int64_t n, size_t *bytes) {
  if (!c || !bytes || n < 1) return tq_fail(TQ_ERR_INVALID_ARG, "index workspace: bad arguments");
  const int64_t rows = n < kIxBatch ? n : kIxBatch;
  *bytes = static_cast<size_t>(rows) * 2 * XD * sizeof(uint16_t);
  return TQ_OK;
}

int tq_index_build(const tq_codec *c, const float *x, int64_t n, uint8_t *kcode, uint16_t *kscale,
                   uint32_t *status, void *workspace, size_t ws_bytes, void *stream) {
  if (!c) return tq_fail(TQ_ERR_INVALID_ARG, "index: NULL codec");
  if (!index_codec_ok(c))
    return tq_fail(TQ_ERR_UNSUPPORTED, "index: needs a d = 1536 codec with QJL keys");
  if (!x || !kcode || !kscale || !workspace || n < 1)
    return tq_fail(TQ_ERR_INVALID_ARG, "index: NULL buffer or n < 1");
  size_t need = 0;
  tq_index_workspace(c, n, &need);
  if (ws_bytes < need) return tq_fail(TQ_ERR_WORKSPACE, "index: workspace too small");
  if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(kcode) |
       reinterpret_cast<uintptr_t>(workspace)) % 16 || reinterpret_cast<uintptr_t>(kscale) % 4)
    return tq_fail(TQ_ERR_ALIGNMENT, "index: x/kcode/workspace need 16-byte, kscale 4-byte alignment");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  IxArgs a;
  a.mbk = c->mse_bits_k;
  paley12(a.h12);
  for (int i = 0; i < XW; ++i) a.dneg[i] = c->books.dneg[i];
  for (int i = 0; i < TQ_MAX_LEVELS; ++i) {
    a.ck[i] = c->books.ck[i];
    a.tk[i] = c->books.tk[i];
  }
  a.status = status;
  const int planes = c->mse_bits_k + 1;
  for (int64_t r0 = 0; r0 < n; r0 += kIxBatch) {
    const int64_t rows = n - r0 < kIxBatch ? n - r0 : kIxBatch;
    a.x = x + r0 * XD;
    a.n = rows;
    a.kcode = kcode + r0 * planes * (XD / 8);
    a.kscale = kscale + r0 * 2;
    a.rbuf = static_cast<uint16_t *>(workspace);
    const int64_t blocks = (rows + 7) / 8;
    ix_encode_kernel<<<static_cast<int>(blocks < 16LL * sm_count() ? blocks : 16LL * sm_count()), 256, 0, st>>>(a);
    tq_count_launch(1);
    if (int e = tq_check_launch("ix_encode_kernel")) return e;
    GemmArgs g;
    g.A = a.rbuf;
    g.B = c->S_dev;
    g.M = rows;
    g.N = XD;
    g.KA = 2 * XD;
    g.KB = XD;
    g.plane = a.kcode + c->mse_bits_k * (XD / 8);
    g.plane_stride = planes * (XD / 8);
    g.out = nullptr;
    g.out_hl = nullptr;
    g.scale = 1.f;
    g.status = status;
    if (int e = run_gemm<0>(g, st)) return e;
  }
  return TQ_OK;
}

int tq_scan_workspace(const tq_codec *c, int64_t n, int nq, int k, size_t *bytes) {
  if (!c || !bytes || n < 1 || nq < 1 || k < 1 || k > SKMAX)
    return tq_fail(TQ_ERR_INVALID_ARG, "scan workspace: bad arguments (1 <= k <= 16)");
  const int gy = scan_grid_y(n, nq);
  size_t b = 0;
  b += static_cast<size_t>(nq) * XD * 4;          // q'
  b += static_cast<size_t>(nq) * 2 * XD * 2;      // q' hi | lo
  b += static_cast<size_t>(nq) * 2 * XD * 2;      // q'' hi | lo
  b += static_cast<size_t>(nq) * gy * k * 8;      // candidates
  *bytes = b + 256;
  return TQ_OK;
}

int tq_scan_topk(const tq_codec *c, const uint8_t *kcode, const uint16_t *kscale, int64_t n,
                 const float *q, int nq, int k, int32_t *idx, float *score, void *workspace,
                 size_t ws_bytes, void *stream) {
  if (!c) return tq_fail(TQ_ERR_INVALID_ARG, "scan: NULL codec");
  if (!index_codec_ok(c))
    return tq_fail(TQ_ERR_UNSUPPORTED, "scan: needs a d = 1536 codec with QJL keys");
  if (!kcode || !kscale || !q || !idx || !score || !workspace || n < 1 || nq < 1 || k < 1 ||
      k > SKMAX || k > n)
    return tq_fail(TQ_ERR_INVALID_ARG, "scan: NULL buffer or bad n / nq / k (1 <= k <= min(16, n))");
  size_t need = 0;
  tq_scan_workspace(c, n, nq, k, &need);
  if (ws_bytes < need) return tq_fail(TQ_ERR_WORKSPACE, "scan: workspace too small");
  if ((reinterpret_cast<uintptr_t>(kcode) | reinterpret_cast<uintptr_t>(q) |
       reinterpret_cast<uintptr_t>(workspace)) % 16 || reinterpret_cast<uintptr_t>(kscale) % 4)
    return tq_fail(TQ_ERR_ALIGNMENT, "scan: kcode/q/workspace need 16-byte, kscale 4-byte alignment");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t *w = static_cast<uint8_t *>(workspace);
  float *q1 = reinterpret_cast<float *>(w);
  uint16_t *q1hl = reinterpret_cast<uint16_t *>(q1 + static_cast<size_t>(nq) * XD);
  uint16_t *q2hl = q1hl + static_cast<size_t>(nq) * 2 * XD;
  float *cand_s = reinterpret_cast<float *>(q2hl + static_cast<size_t>(nq) * 2 * XD);
  const int gy = scan_grid_y(n, nq);
  int32_t *cand_i = reinterpret_cast<int32_t *>(cand_s + static_cast<size_t>(nq) * gy * k);
  QrotArgs qa;
  qa.q = q;
  qa.nq = nq;
  qa.q1 = q1;
  qa.q1hl = q1hl;
  paley12(qa.h12);
  for (int i = 0; i < XW; ++i) qa.dneg[i] = c->books.dneg[i];
  ix_qrot_kernel<<<(nq + 7) / 8, 256, 0, st>>>(qa);
  tq_count_launch(1);
  if (int e = tq_check_launch("ix_qrot_kernel")) return e;
  GemmArgs g;
  g.A = q1hl;
  g.B = c->S_dev;
  g.M = nq;
  g.N = XD;
  g.KA = 2 * XD;
  g.KB = XD;
  g.plane = nullptr;
  g.plane_stride = 0;
  g.out = nullptr;
  g.out_hl = q2hl;
  g.scale = 1.f;
  g.status = nullptr;
  if (int e = run_gemm<2>(g, st)) return e;
  ScanArgs sa;
  sa.q1hl = q1hl;
  sa.q2hl = q2hl;
  sa.kcode = kcode;
  sa.kscale = kscale;
  sa.n = n;
  sa.nq = nq;
  sa.k = k;
  const int64_t tiles = (n + SR - 1) / SR;
  sa.tiles_per_cta = static_cast<int>((tiles + gy - 1) / gy);
  sa.coef = sqrtf(static_cast<float>(M_PI) / 2.0f) / XD;
  for (int i = 0; i < TQ_MAX_LEVELS; ++i) sa.ck[i] = c->books.ck[i];
  sa.mbk = c->mse_bits_k;
  sa.cand_s = cand_s;
  sa.cand_i = cand_i;
  sa.err = nullptr;
  constexpr int shm = 4 * (SQ * SK * 2) + 3 * (SR * SK * 2);
  static bool done[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !done[dev]) {
    if (cudaFuncSetAttribute(ix_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, shm) != cudaSuccess)
      return tq_check_launch("cudaFuncSetAttribute(ix_scan)");
    done[dev] = true;
  }
  dim3 grid((nq + SQ - 1) / SQ, gy);
  cudaEvent_t ev0, ev1;
  tq_timing_events(&ev0, &ev1);
  if (ev0) cudaEventRecord(ev0, st);
  ix_scan_kernel<<<grid, 128, shm, st>>>(sa);
  if (int e = tq_check_launch("ix_scan_kernel")) return e;
  if (ev1) cudaEventRecord(ev1, st);
  ix_merge_kernel<<<(nq + 127) / 128, 128, 0, st>>>(cand_s, cand_i, nq, gy, k, idx, score);
  tq_count_launch(2);
  return tq_check_launch("ix_merge_kernel");
}

}  // extern "C"
