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
//   ix_sketch_kernel   z = S r for 128 x 256 tiles: one warp streams the
//                      [r_hi | r_lo] and S tiles by cp.async.bulk into a
//                      4-stage ring and issues tcgen05 kind::f16 MMAs (S is
//                      exactly bf16), fp32 in tensor memory; four epilogue
//                      warps turn the signs into the QJL plane.
// Scanning (tq_scan_topk):
//   ix_qrot_kernel     q' = Pi q per query
//   ix_gemm_kernel     q'' = S q' (fp32 GEMM on CUDA cores)
//   ix_qpack_kernel    fp16 B operand [2^e q' | 2^e coef q''] in chunk order
//   ix_scan2_kernel    rows dequantized into tensor memory, M128 x N256 MMAs,
//                      per-thread top-k lists
//   ix_merge_kernel    merge of the per-CTA lists into the final top-k
#include <math_constants.h>

#include <cstdlib>
#include <cstring>
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
  uint16_t *rbuf;        // residual hi | lo, tiled for ix_sketch_kernel (rows rounded up to 128)
  uint32_t dneg[XW];
  float ck[TQ_MAX_LEVELS], tk[TQ_MAX_LEVELS];
  int mbk;
  uint32_t *status;
};

// Sign of entry (i, j) of the Paley (type I) Hadamard matrix of order 12
// built from the quadratic residues {1, 3, 4, 5, 9} of GF(11): row 0 is all
// +1, column 0 is -1 below row 0, the diagonal is +1 and entry (i, j) of the
// remaining 11 x 11 core is the Legendre symbol of (j - i) mod 11.  Called
// with constant indices only, so every sign folds at compile time.
__host__ __device__ __forceinline__ constexpr bool h12_neg(int i, int j) {
  return i == 0 || i == j ? false
         : j == 0         ? true
                          : ((0x23Au >> (((j - i) % 11 + 11) % 11)) & 1u) == 0u;
}

// x[j1][k] holds coordinate 128 j1 + 32 k + lane; y = (H_12 kron H_128) x.
__device__ __forceinline__ void rotate1536(float (&x)[XNB][4], int lane) {
#pragma unroll
  for (int j1 = 0; j1 < XNB; ++j1) tq_warp_wht<4, true>(x[j1], lane);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    float t[XNB];
#pragma unroll
    for (int i1 = 0; i1 < XNB; ++i1) {
      float s = h12_neg(i1, 0) ? -x[0][k] : x[0][k];
#pragma unroll
      for (int j1 = 1; j1 < XNB; ++j1) s += h12_neg(i1, j1) ? -x[j1][k] : x[j1][k];
      t[i1] = s;
    }
#pragma unroll
    for (int i1 = 0; i1 < XNB; ++i1) x[i1][k] = t[i1];
  }
}

__global__ void __launch_bounds__(256, 2) ix_encode_kernel(IxArgs a) {
  __shared__ float cks[TQ_MAX_LEVELS], tks[TQ_MAX_LEVELS];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x < TQ_MAX_LEVELS) {
    cks[threadIdx.x] = a.ck[threadIdx.x];
    tks[threadIdx.x] = a.tk[threadIdx.x];
  }
  __syncthreads();
  const int planes = a.mbk + 1;
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
    rotate1536(x, lane);
    const float inv = zero ? 0.f : 1.0f / (sqrtf(static_cast<float>(XD)) * nu);
    uint32_t mw[4][2];
#pragma unroll
    for (int p = 0; p < 4; ++p) mw[p][0] = mw[p][1] = 0u;
    float r2 = 0.f;
    // residual hi | lo in the sketch GEMM's A layout: K-major core-matrix
    // tiles of 128 rows x 64 K elements (16 KB), tile (row / 128, k / 64)
    uint16_t *rtile = a.rbuf + (row >> 7) * (2 * XD / 64) * 8192 + ((row & 127) >> 3) * 64 + (row & 7) * 8;
#pragma unroll
    for (int j1 = 0; j1 < XNB; ++j1)
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float u = x[j1][k] * inv;
        const int idx = tq_code<3>(u, tks);   // index codecs have at most 3 MSE bits
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
        const int kl = XD + i;
        rtile[(i >> 6) * 8192 + ((i & 63) >> 3) * 1024 + (i & 7)] = __bfloat16_as_ushort(hi);
        rtile[(kl >> 6) * 8192 + ((kl & 63) >> 3) * 1024 + (kl & 7)] = __bfloat16_as_ushort(lo);
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
// Index-build sketch: sign(S r) for every residual row as one GEMM on the
// tensor cores, z = [r_hi | r_lo] [S | S]^T (S is exactly bf16).  Both
// operands sit in global memory as K-major core-matrix tiles (A: 128 rows x
// 64 K = 16 KB, written by ix_encode_kernel; B: 256 rows of S x 64 K = 32 KB,
// built with the codec), so one warp streams them into a 4-stage shared ring
// with cp.async.bulk and issues M128 x N256 kind::f16 MMAs into one of two
// fp32 accumulators in TMEM; four epilogue warps turn the other accumulator
// into sign words.  Persistent CTAs walk (m tile, n tile) pairs, m-major, so
// the six n tiles of an m tile run at the same time and share its A tiles in L2.
// ---------------------------------------------------------------------------
constexpr int SKN_T = XD / 256;                 // 6 n tiles
constexpr int SKA_CH = 2 * XD / 64;             // 48 A chunks (hi | lo)
constexpr int SKB_CH = XD / 64;                 // 24 B chunks
constexpr uint32_t SKA_BYTES = 128 * 64 * 2;
constexpr uint32_t SKB_BYTES = 256 * 64 * 2;
constexpr int SKS = 4;                          // ring stages
constexpr int SK_T = 5 * 32;                    // 4 epilogue warps + the MMA warp
constexpr uint32_t SK_SMEM = SKS * (SKA_BYTES + SKB_BYTES);

struct SketchArgs {
  const uint16_t *A;      // residual tiles of this batch
  const uint16_t *B;      // S tiles
  int64_t M;              // rows in the batch
  uint8_t *plane;         // sign plane of row 0 of the batch; row stride plane_stride bytes
  int64_t plane_stride;
  uint32_t *status;
  uint32_t wait_limit;    // polls per wait before giving up
};

__global__ void __launch_bounds__(SK_T, 1) ix_sketch_kernel(SketchArgs g) {
  extern __shared__ __align__(1024) uint8_t skm[];
  __shared__ __align__(8) uint64_t full[SKS], empty[SKS], acc_full[2], acc_free[2], fin;
  __shared__ uint32_t tmem_s;
  __shared__ int abort_s;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (warp == 0) sm100::tmem_alloc(&tmem_s, 512);
  if (tid == 0) {
    for (int s = 0; s < SKS; ++s) {
      sm100::mbar_init(&full[s], 1);
      sm100::mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      sm100::mbar_init(&acc_full[b], 1);
      sm100::mbar_init(&acc_free[b], 4);
    }
    sm100::mbar_init(&fin, 1);
    abort_s = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  sm100::fence_before_sync();
  __syncthreads();
  sm100::fence_after_sync();
  const uint32_t tm = tmem_s;
  const int64_t tiles = (g.M + 127) / 128 * SKN_T;
  const int ntl = tiles > blockIdx.x ? static_cast<int>((tiles - 1 - blockIdx.x) / gridDim.x + 1) : 0;
  const int total = ntl * SKA_CH;
  if (warp == 4) {
    if (lane == 0 && total > 0) {
      // per stage: the parity of its last issued copy (-1: none); whether any
      // MMA was issued (both drained before the CTA releases its memory)
      int lastc[SKS];
      for (int s = 0; s < SKS; ++s) lastc[s] = -1;
      bool mma_issued = false;
      auto copy = [&](int gc) {
        const int tl = gc / SKA_CH, c = gc % SKA_CH, s = gc % SKS;
        lastc[s] = (gc / SKS) & 1;
        const int64_t t = blockIdx.x + static_cast<int64_t>(tl) * gridDim.x;
        const int64_t mt = t / SKN_T;
        const int nt = static_cast<int>(t % SKN_T);
        uint8_t *dst = skm + s * (SKA_BYTES + SKB_BYTES);
        sm100::mbar_expect_tx(&full[s], SKA_BYTES + SKB_BYTES);
        sm100::bulk_g2s(dst, g.A + (mt * SKA_CH + c) * (SKA_BYTES / 2), SKA_BYTES, &full[s]);
        sm100::bulk_g2s(dst + SKA_BYTES, g.B + (static_cast<int64_t>(nt) * SKB_CH + c % SKB_CH) * (SKB_BYTES / 2),
                        SKB_BYTES, &full[s]);
      };
      for (int gc = 0; gc < SKS - 1 && gc < total; ++gc) copy(gc);
      constexpr uint32_t IDESC = sm100::idesc_bf16(128, 256);
      bool ok = true;
      for (int tl = 0; tl < ntl && ok; ++tl) {
        const int ab = tl & 1;
        if (tl >= 2) {
          ok = sm100::mbar_wait(&acc_free[ab], ((tl >> 1) - 1) & 1, g.wait_limit);
          if (!ok) break;
          sm100::fence_after_sync();
        }
        for (int c = 0; c < SKA_CH && ok; ++c) {
          const int gc = tl * SKA_CH + c, s = gc % SKS;
          ok = sm100::mbar_wait(&full[s], (gc / SKS) & 1, g.wait_limit);
          if (!ok) break;
          sm100::fence_after_sync();
          const uint32_t a_addr = sm100::smem_addr(skm + s * (SKA_BYTES + SKB_BYTES));
          const uint32_t b_addr = a_addr + SKA_BYTES;
          mma_issued = true;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            sm100::mma_bf16_ss(tm + ab * 256, sm100::smem_desc(a_addr + kk * 2 * 2048, 2048, 128),
                               sm100::smem_desc(b_addr + kk * 2 * 4096, 4096, 128), IDESC,
                               (c > 0 || kk > 0) ? 1u : 0u);
          sm100::mma_commit(&empty[s]);
          if (c == SKA_CH - 1) sm100::mma_commit(&acc_full[ab]);
          // refill: chunk gc + SKS - 1 reuses the stage of chunk gc - 1
          const int gn = gc + SKS - 1;
          if (gn < total) {
            if (gn >= SKS) {
              ok = sm100::mbar_wait(&empty[gn % SKS], ((gn / SKS) - 1) & 1, g.wait_limit);
              if (!ok) break;
            }
            copy(gn);
          }
        }
      }
      if (!ok) {
        abort_s = 1;
        // this CTA's copies and MMAs land before its shared and tensor
        // memory are released
        for (int s = 0; s < SKS; ++s)
          if (lastc[s] >= 0) sm100::mbar_wait(&full[s], static_cast<uint32_t>(lastc[s]), 1u << 20);
        if (mma_issued) {
          sm100::mma_commit(&fin);
          sm100::mbar_wait(&fin, 0, 1u << 20);
        }
      }
    }
    __syncwarp();
  } else {
    // epilogue warp = TMEM lane quarter: row 32 warp + lane of the m tile
    for (int tl = 0; tl < ntl; ++tl) {
      const int ab = tl & 1;
      if (lane == 0 && !abort_s && !sm100::mbar_wait(&acc_full[ab], (tl >> 1) & 1, g.wait_limit)) abort_s = 1;
      __syncwarp();
      sm100::fence_after_sync();
      const int64_t t = blockIdx.x + static_cast<int64_t>(tl) * gridDim.x;
      const int64_t row = (t / SKN_T) * 128 + 32 * warp + lane;
      const int nt = static_cast<int>(t % SKN_T);
      uint32_t *dst = reinterpret_cast<uint32_t *>(g.plane + row * g.plane_stride) + nt * 8;
#pragma unroll
      for (int cc = 0; cc < 8; ++cc) {
        uint32_t z[32];
        sm100::tmem_ld32(sm100::tmem_lane(tm + ab * 256 + 32 * cc, warp), z);
        sm100::wait_ld();
        uint32_t word = 0u;
#pragma unroll
        for (int e = 0; e < 32; ++e) word |= (__uint_as_float(z[e]) >= 0.f ? 1u : 0u) << e;
        if (row < g.M) dst[cc] = word;
      }
      sm100::fence_before_sync();
      __syncwarp();
      if (lane == 0) sm100::mbar_arrive(&acc_free[ab]);
    }
  }
  if (abort_s && tid == 0 && g.status) atomicOr(g.status, 1u << 31);
  sm100::fence_before_sync();
  __syncthreads();
  sm100::fence_after_sync();
  if (warp == 0) sm100::tmem_dealloc(tm, 512);
}

// ---------------------------------------------------------------------------
// C = A B^T on the tensor cores for A [M][KA] and B [N][KB] bf16 row-major
// (K contiguous), KA a multiple of KB: A's K range wraps over B (A = [r_hi |
// r_lo] against B = S gives S r_hi + S r_lo).  Tile 128 x 256, K chunks of 64
// through a 3-stage cp.async ring; fp32 accumulators in 256 TMEM columns,
// written out as fp32 (the scan's q'' = S q' for a block of queries).
// ---------------------------------------------------------------------------
struct GemmArgs {
  const uint16_t *A;
  const uint16_t *B;
  int64_t M;
  int N, KA, KB;
  float *out;            // [M][N]
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
        float *o = g.out + row * g.N + n0 + c0;
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          if (n0 + c0 + c < g.N) o[c] = __uint_as_float(z0[c]);
          if (n0 + c0 + 16 + c < g.N) o[16 + c] = __uint_as_float(z1[c]);
        }
      }
    }
  } else if (tid == 0 && g.status) {
    atomicOr(g.status, 1u << 31);
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
  rotate1536(x, lane);
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
// as ONE fp16 product per element over K = 2d:
//   A (database row j, in tensor memory)  = [ c[idx_j] | rho_j (2 sigma_j - 1) ]
//   B (query i, in shared memory)         = 2^e_i [ q'_i | sqrt(pi/2)/d q''_i ]
// with K ordered in 48 chunks of 64 = [32 MSE coordinates | the same 32 sign
// coordinates].  A row's codes are dequantized into TMEM by the worker lane
// that owns the row (tcgen05.st), the query chunks stream into shared memory
// by cp.async.bulk, and one warp issues tcgen05.mma kind::f16 (M = 128 rows,
// N = 256 queries) into fp32 accumulators.  Per-element rounding: centroids
// and rho are fp16 (2^-11 relative), queries fp16 after the power-of-two
// scale; the score error is ~1e-5 of |q| for unit data.
// Epilogue: the 128 x 256 scores go through shared memory (two passes of 128
// queries) so each worker thread walks 64 rows of one query and keeps a
// running top-k in registers; a merge kernel combines the per-CTA lists.
// ---------------------------------------------------------------------------
constexpr int QN = 256;                       // queries per CTA (MMA N)
constexpr int RM = 128;                       // database rows per tile (MMA M)
constexpr int XCH = XD / 32;                  // K chunks
constexpr int NAS = 4;                        // pipeline stages (A in TMEM, B in smem)
constexpr uint32_t QCH_BYTES = QN * 64 * 2;   // one query chunk, fp16
constexpr int SCW = 8;                        // worker warps
constexpr int SCT = (SCW + 1) * 32;           // + the MMA warp
constexpr int SBP = RM + 1;                   // padded stride of the score transpose
constexpr int SKMAX = 16;                     // largest k of the top-k
constexpr uint32_t SC_B_OFF = 0;
constexpr uint32_t SC_SB_OFF = NAS * QCH_BYTES;
constexpr uint32_t SC_LUT_OFF = SC_SB_OFF + 128 * SBP * 4;
constexpr uint32_t SC_SMEM = SC_LUT_OFF + 64 * 32 * 4;

// Element offset (16-bit units) of (n, k) in a K-major, no-swizzle operand of QN rows.
__host__ __device__ constexpr uint32_t qop_off(int n, int k) {
  return ((k >> 3) * (QN * 16) + (n >> 3) * 128 + (n & 7) * 16) / 2 + (k & 7);
}

struct QpackArgs {
  const float *q1;      // [nq][XD] q' = Pi q
  const float *q2;      // [nq][XD] q'' = S q'
  int nq;
  float coef;           // sqrt(pi/2) / d
  uint16_t *qop;        // [ceil(nq / QN)][XCH][QN * 64] fp16
  float *qinv;          // [nq] 2^-e
  uint32_t *status;     // the scan's give-up flag, cleared here for this call
};

// One warp per (padded) query: power-of-two scale putting max |B| in
// [2^14, 2^15), then the fp16 operand in chunk order.
__global__ void __launch_bounds__(256) ix_qpack_kernel(QpackArgs a) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (blockIdx.x == 0 && threadIdx.x == 0 && a.status) *a.status = 0u;
  const int q = blockIdx.x * 8 + warp;
  const int nqp = (a.nq + QN - 1) / QN * QN;
  if (q >= nqp) return;
  const bool valid = q < a.nq;
  const float *s1 = a.q1 + static_cast<int64_t>(valid ? q : 0) * XD;
  const float *s2 = a.q2 + static_cast<int64_t>(valid ? q : 0) * XD;
  float mx = 0.f;
  if (valid)
    for (int i = lane; i < XD; i += 32) mx = fmaxf(mx, fmaxf(fabsf(s1[i]), a.coef * fabsf(s2[i])));
  mx = tq_warp_max(mx);
  int e2 = 0;
  if (mx > 0.f) frexpf(mx, &e2);            // mx in [2^(e2-1), 2^e2)
  const float sc = mx > 0.f ? ldexpf(1.f, 15 - e2) : 1.f;
  if (lane == 0 && valid) a.qinv[q] = mx > 0.f ? ldexpf(1.f, e2 - 15) : 1.f;
  uint16_t *dst = a.qop + static_cast<int64_t>(q / QN) * XCH * (QN * 64);
  const int n = q % QN;
  for (int c = 0; c < XCH; ++c) {
    const int coord = 32 * c + lane;
    const float v1 = valid ? s1[coord] * sc : 0.f;
    const float v2 = valid ? a.coef * s2[coord] * sc : 0.f;
    dst[c * (QN * 64) + qop_off(n, lane)] = __half_as_ushort(__float2half_rn(v1));
    dst[c * (QN * 64) + qop_off(n, 32 + lane)] = __half_as_ushort(__float2half_rn(v2));
  }
}

struct Scan2Args {
  const uint8_t *kcode;   // [n][planes][XD / 8]
  const uint16_t *kscale; // [n][2]
  int64_t n;
  const uint16_t *qop;
  const float *qinv;
  int nq;
  int tiles_per_cta;
  int mbk;                // MSE planes (1..3)
  uint32_t lut[64];       // half2 (c[m_even], c[m_odd]); index bits (b0e b0o b1e b1o b2e b2o)
  float *cand_s;          // [nq][lists][k]
  int32_t *cand_i;
  int k;
  uint32_t *err;          // set when a bounded wait gave up (read by the merge)
  uint32_t wait_limit;    // polls per wait before giving up
};

__global__ void __launch_bounds__(SCT, 1) ix_scan2_kernel(Scan2Args a) {
  extern __shared__ __align__(1024) uint8_t ssm[];
  uint8_t *bst = ssm + SC_B_OFF;
  float *sb = reinterpret_cast<float *>(ssm + SC_SB_OFF);
  uint32_t *lut = reinterpret_cast<uint32_t *>(ssm + SC_LUT_OFF);
  __shared__ __align__(8) uint64_t a_full[NAS], b_full[NAS], done[NAS], acc_full, acc_free, fin;
  __shared__ uint32_t tmem_s;
  __shared__ int abort_s;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t wl = a.wait_limit;
  for (int e = tid; e < 64 * 32; e += SCT) lut[e] = a.lut[e >> 5];
  if (warp == 0) sm100::tmem_alloc(&tmem_s, 512);
  if (tid == 0) {
    for (int s = 0; s < NAS; ++s) {
      sm100::mbar_init(&a_full[s], 4);
      sm100::mbar_init(&b_full[s], 1);
      sm100::mbar_init(&done[s], 1);
    }
    sm100::mbar_init(&acc_full, 1);
    sm100::mbar_init(&acc_free, SCW);
    sm100::mbar_init(&fin, 1);
    abort_s = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  sm100::fence_before_sync();
  __syncthreads();
  sm100::fence_after_sync();
  const uint32_t tm = tmem_s;            // D: columns [0, 256); A stages: [256, 256 + 32 NAS)
  const int64_t ntiles = (a.n + RM - 1) / RM;
  const int64_t t_begin = static_cast<int64_t>(blockIdx.y) * a.tiles_per_cta;
  const int64_t t_end = t_begin + a.tiles_per_cta < ntiles ? t_begin + a.tiles_per_cta : ntiles;
  const int nt = t_end > t_begin ? static_cast<int>(t_end - t_begin) : 0;
  const int total = nt * XCH;

  if (warp == SCW) {
    // ---------------- MMA warp: query-chunk copies and the MMAs
    if (lane == 0 && total > 0) {
      const uint16_t *qsrc = a.qop + static_cast<int64_t>(blockIdx.x) * XCH * (QN * 64);
      // per stage: the parity of its last issued copy (-1: none); whether any
      // MMA was issued (both drained before the CTA releases its memory)
      int lastb[NAS];
      for (int s = 0; s < NAS; ++s) lastb[s] = -1;
      bool mma_issued = false;
      auto copy = [&](int g) {
        const int s = g % NAS, c = g % XCH;
        sm100::mbar_expect_tx(&b_full[s], QCH_BYTES);
        sm100::bulk_g2s(bst + s * QCH_BYTES, qsrc + c * (QN * 64), QCH_BYTES, &b_full[s]);
        lastb[s] = (g / NAS) & 1;
      };
      for (int g = 0; g < NAS - 1 && g < total; ++g) copy(g);
      constexpr uint32_t IDESC = sm100::idesc_f16(RM, QN);
      bool ok = true;
      for (int tl = 0; tl < nt && ok; ++tl) {
        if (tl >= 1) {
          ok = sm100::mbar_wait(&acc_free, (tl - 1) & 1, wl);
          if (!ok) break;
          sm100::fence_after_sync();
        }
        for (int c = 0; c < XCH && ok; ++c) {
          const int g = tl * XCH + c, s = g % NAS, u = g / NAS;
          ok = sm100::mbar_wait(&a_full[s], u & 1, wl) && sm100::mbar_wait(&b_full[s], u & 1, wl);
          if (!ok) break;
          sm100::fence_after_sync();
          const uint32_t bb = sm100::smem_addr(bst + s * QCH_BYTES);
          mma_issued = true;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            sm100::mma_f16_ts(tm, tm + 256 + s * 32 + kk * 8,
                              sm100::smem_desc(bb + kk * 2 * (QN * 16), QN * 16, 128), IDESC,
                              (c > 0 || kk > 0) ? 1u : 0u);
          sm100::mma_commit(&done[s]);
          if (c == XCH - 1) sm100::mma_commit(&acc_full);
          // refill: chunk g + NAS - 1 reuses the stage of chunk g - 1
          const int gn = g + NAS - 1;
          if (gn < total) {
            if (gn >= NAS) {
              ok = sm100::mbar_wait(&done[gn % NAS], ((gn / NAS) - 1) & 1, wl);
              if (!ok) break;
            }
            copy(gn);
          }
        }
      }
      if (!ok) {
        abort_s = 1;
        // this CTA's copies and MMAs land before its shared and tensor
        // memory are released
        for (int s = 0; s < NAS; ++s)
          if (lastb[s] >= 0) sm100::mbar_wait(&b_full[s], static_cast<uint32_t>(lastb[s]), 1u << 20);
        if (mma_issued) {
          sm100::mma_commit(&fin);
          sm100::mbar_wait(&fin, 0, 1u << 20);
        }
      }
    }
    __syncwarp();
  } else {
    // ---------------- workers: warp (quarter wq, half h); thread = row 32 wq + lane
    const int wq = warp & 3, h = warp >> 2;
    const int r = 32 * wq + lane;
    const int planes = a.mbk + 1;
    float ts0[SKMAX], ts1[SKMAX];
    int ti0[SKMAX], ti1[SKMAX];
#pragma unroll
    for (int e = 0; e < SKMAX; ++e) {
      ts0[e] = ts1[e] = -CUDART_INF_F;
      ti0[e] = ti1[e] = 0x7fffffff;
    }
    const int qq = tid & 127, rh = tid >> 7;   // top-k role: query qq of a pass, rows 64 rh ..
    const int qbase = blockIdx.x * QN;
    const float qs0 = qbase + qq < a.nq ? a.qinv[qbase + qq] : 0.f;
    const float qs1 = qbase + 128 + qq < a.nq ? a.qinv[qbase + 128 + qq] : 0.f;
    // Waits are bounded; after one gives up (abort_s) every later wait is
    // skipped but the loops keep their fixed trip counts, so all worker warps
    // still meet at every named barrier.
    auto wwait = [&](uint64_t *bar, uint32_t par) {
      if (lane == 0 && !abort_s && !sm100::mbar_wait(bar, par, wl)) abort_s = 1;
      __syncwarp();
    };
    auto insert = [&](float (&ts)[SKMAX], int (&ti)[SKMAX], float v, int idx) {
      if (v > ts[SKMAX - 1]) {
        ts[SKMAX - 1] = v;
        ti[SKMAX - 1] = idx;
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
    };
    for (int tl = 0; tl < nt; ++tl) {
      const int64_t row = (t_begin + tl) * RM + r;
      const bool valid = row < a.n;
      uint32_t sc = 0;
      if (valid) sc = reinterpret_cast<const uint32_t *>(a.kscale)[row];
      const float nu = tq_half_to_f32(static_cast<uint16_t>(sc & 0xffffu));
      const uint32_t rho2 = (sc >> 16) | (sc & 0xffff0000u);     // half2 (rho, rho)
      const uint32_t *kr = reinterpret_cast<const uint32_t *>(a.kcode + (valid ? row : 0) * planes * (XD / 8));
      // chunks of this half: pairs (c, c + 1) with (c / 2) % 2 == h
      for (int c2 = 2 * h; c2 < XCH; c2 += 4) {
        uint2 w[4];
#pragma unroll
        for (int p = 0; p < 4; ++p)
          w[p] = (valid && p < planes) ? *reinterpret_cast<const uint2 *>(kr + p * XW + c2) : make_uint2(0u, 0u);
        // plane order: MSE planes 0 .. mbk-1, then the sign plane (index mbk)
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          const int c = c2 + cc;
          const int g = tl * XCH + c, s = g % NAS, u = g / NAS;
          if (u >= 1) {
            wwait(&done[s], (u - 1) & 1);
            sm100::fence_after_sync();
          }
          const uint32_t p0 = cc ? w[0].y : w[0].x;
          const uint32_t p1 = a.mbk > 1 ? (cc ? w[1].y : w[1].x) : 0u;
          const uint32_t p2 = a.mbk > 2 ? (cc ? w[2].y : w[2].x) : 0u;
          const uint32_t sg = a.mbk == 1 ? (cc ? w[1].y : w[1].x)
                              : a.mbk == 2 ? (cc ? w[2].y : w[2].x)
                                           : (cc ? w[3].y : w[3].x);
          const uint32_t nsg = ~sg;
          uint32_t out[32];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const uint32_t idx = ((p0 >> (2 * j)) & 3u) | (((p1 >> (2 * j)) & 3u) << 2) |
                                 (((p2 >> (2 * j)) & 3u) << 4);
            out[j] = lut[idx * 32 + lane];
            out[16 + j] = rho2 ^ (((nsg >> (2 * j)) & 1u) << 15) ^ (((nsg >> (2 * j + 1)) & 1u) << 31);
          }
          sm100::tmem_st32(sm100::tmem_lane(tm + 256 + s * 32, wq), out);
          sm100::wait_st();
          sm100::fence_before_sync();
          __syncwarp();
          if (lane == 0) sm100::mbar_arrive(&a_full[s]);
        }
      }
      // ---- epilogue of the tile
      wwait(&acc_full, tl & 1);
      sm100::fence_after_sync();
#pragma unroll
      for (int qh = 0; qh < 2; ++qh) {
#pragma unroll
        for (int cc = 0; cc < 64; cc += 32) {
          uint32_t v[32];
          sm100::tmem_ld32(sm100::tmem_lane(tm + 128 * qh + 64 * h + cc, wq), v);
          sm100::wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) sb[(64 * h + cc + e) * SBP + r] = nu * __uint_as_float(v[e]);
        }
        if (qh == 1) {   // this warp has read its part of D
          sm100::fence_before_sync();
          __syncwarp();
          if (lane == 0) sm100::mbar_arrive(&acc_free);
        }
        sm100::named_sync(1, SCW * 32);
        const float qs = qh ? qs1 : qs0;
        const float *srow = sb + qq * SBP + 64 * rh;
        const int64_t r0 = (t_begin + tl) * RM + 64 * rh;
        const int nr = a.n - r0 < 64 ? static_cast<int>(a.n - r0) : 64;
        if (qh == 0) {
          for (int rr = 0; rr < nr; ++rr) insert(ts0, ti0, srow[rr] * qs, static_cast<int>(r0 + rr));
        } else {
          for (int rr = 0; rr < nr; ++rr) insert(ts1, ti1, srow[rr] * qs, static_cast<int>(r0 + rr));
        }
        sm100::named_sync(1, SCW * 32);
      }
    }
    // candidate lists: one per (query, CTA row range, row half)
    const int lists = gridDim.y * 2, list = blockIdx.y * 2 + rh;
    if (!abort_s) {
#pragma unroll
      for (int qh = 0; qh < 2; ++qh) {
        const int q = qbase + 128 * qh + qq;
        if (q < a.nq) {
          float *cs = a.cand_s + (static_cast<int64_t>(q) * lists + list) * a.k;
          int32_t *ci = a.cand_i + (static_cast<int64_t>(q) * lists + list) * a.k;
#pragma unroll
          for (int e = 0; e < SKMAX; ++e)
            if (e < a.k) {
              cs[e] = qh ? ts1[e] : ts0[e];
              ci[e] = qh ? ti1[e] : ti0[e];
            }
        }
      }
    }
  }
  if (abort_s && tid == 0 && a.err) atomicExch(a.err, 1u);
  sm100::fence_before_sync();
  __syncthreads();
  sm100::fence_after_sync();
  if (warp == 0) sm100::tmem_dealloc(tm, 512);
}

// Merge the per-CTA candidate lists of each query: order (-score, index).
__global__ void ix_merge_kernel(const float *cs, const int32_t *ci, int nq, int lists, int k,
                                int32_t *idx, float *score, const uint32_t *err) {
  const int q = blockIdx.x * blockDim.x + threadIdx.x;
  if (q >= nq) return;
  if (err && *err) {
    // a bounded wait of the scan gave up: its candidate lists are incomplete
    for (int e = 0; e < k; ++e) {
      idx[static_cast<int64_t>(q) * k + e] = -1;
      score[static_cast<int64_t>(q) * k + e] = CUDART_NAN_F;
    }
    return;
  }
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

// ---------------------------------------------------------------------------
// LUT-path scan (the comparison path to the tensor-core scan): per query a
// table T[i][m] = q'_i c_m over every coordinate i and code m, and the QJL
// column coef * q''_i, in shared memory; a warp scores one database row at a
// time, lane l taking coordinates 32 w + l, with one table lookup and one
// signed add per coordinate in fp32 (no fp16 rounding of the products).
// Every warp keeps its own top-k; the block merges its 8 lists into one
// candidate list per (query, row block), merged across blocks by
// ix_merge_kernel.
// ---------------------------------------------------------------------------
constexpr int LT = 256;        // threads (8 warps) of ix_lut_kernel
constexpr int LSTR = 9;        // padded table row: 8 codes + 1 (bank spread)
constexpr uint32_t LUT_SMEM = XD * (LSTR + 1) * 4;

struct LutArgs {
  const uint8_t *kcode;   // [n][planes][XD / 8]
  const uint16_t *kscale; // [n][2]
  int64_t n;
  const float *q1;        // [nq][XD]  q' = Pi q
  const float *q2;        // [nq][XD]  q'' = S q'
  int nq;
  float coef;             // sqrt(pi/2) / XD
  int mbk;
  float ck[8];            // key centroids
  int64_t rows_per_block;
  float *cand_s;          // [nq][lists][k]
  int32_t *cand_i;
  int k;
  int lists;
};

// Insert (v, j) into a descending list of k (ties to the lower index).
__device__ __forceinline__ void topk_insert(float *bs, int *bi, int k, float v, int j) {
  const bool better = v > bs[k - 1] || (v == bs[k - 1] && j < bi[k - 1]);
  if (!better) return;
  int e = k - 1;
  while (e > 0 && (v > bs[e - 1] || (v == bs[e - 1] && j < bi[e - 1]))) {
    bs[e] = bs[e - 1];
    bi[e] = bi[e - 1];
    --e;
  }
  bs[e] = v;
  bi[e] = j;
}

__global__ void __launch_bounds__(LT) ix_lut_kernel(LutArgs a) {
  extern __shared__ float lut_smem[];
  float *tq = lut_smem;                  // [XD][LSTR]
  float *sq = lut_smem + XD * LSTR;      // [XD]
  __shared__ float ws[LT / 32][SKMAX];
  __shared__ int wi[LT / 32][SKMAX];
  const int q = blockIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < XD; i += LT) {
    const float v = a.q1[static_cast<int64_t>(q) * XD + i];
#pragma unroll
    for (int m = 0; m < 8; ++m) tq[i * LSTR + m] = v * a.ck[m];
    sq[i] = a.coef * a.q2[static_cast<int64_t>(q) * XD + i];
  }
  __syncthreads();
  float bs[SKMAX];
  int bi[SKMAX];
  for (int e = 0; e < SKMAX; ++e) {
    bs[e] = -CUDART_INF_F;
    bi[e] = 0x7fffffff;
  }
  const int planes = a.mbk + 1;
  const int64_t r_begin = static_cast<int64_t>(blockIdx.y) * a.rows_per_block;
  const int64_t r_end = min(a.n, r_begin + a.rows_per_block);
  for (int64_t row = r_begin + warp; row < r_end; row += LT / 32) {
    const uint32_t *kr = reinterpret_cast<const uint32_t *>(a.kcode + row * planes * (XD / 8));
    float acc = 0.f, sacc = 0.f;
    for (int w = 0; w < XW; ++w) {
      const uint32_t w0 = kr[w];
      const uint32_t w1 = a.mbk > 1 ? kr[XW + w] : 0u;
      const uint32_t w2 = a.mbk > 2 ? kr[2 * XW + w] : 0u;
      const uint32_t wsg = kr[a.mbk * XW + w];
      const int idx = static_cast<int>(((w0 >> lane) & 1u) | (((w1 >> lane) & 1u) << 1) |
                                       (((w2 >> lane) & 1u) << 2));
      const int i = 32 * w + lane;
      acc += tq[i * LSTR + idx];
      const float sv = sq[i];
      sacc += ((wsg >> lane) & 1u) ? sv : -sv;
    }
    acc = tq_warp_sum(acc);
    sacc = tq_warp_sum(sacc);
    const uint32_t sc = reinterpret_cast<const uint32_t *>(a.kscale)[row];
    const float nu = tq_half_to_f32(static_cast<uint16_t>(sc & 0xffffu));
    const float rho = tq_half_to_f32(static_cast<uint16_t>(sc >> 16));
    const float score = nu * fmaf(rho, sacc, acc);
    if (lane == 0) topk_insert(bs, bi, a.k, score, static_cast<int>(row));
  }
  if (lane == 0)
    for (int e = 0; e < a.k; ++e) {
      ws[warp][e] = bs[e];
      wi[warp][e] = bi[e];
    }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < LT / 32; ++w)
      for (int e = 0; e < a.k; ++e) topk_insert(bs, bi, a.k, ws[w][e], wi[w][e]);
    const int64_t base = (static_cast<int64_t>(q) * a.lists + blockIdx.y) * a.k;
    for (int e = 0; e < a.k; ++e) {
      a.cand_s[base + e] = bs[e];
      a.cand_i[base + e] = bi[e];
    }
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
int sm_count() {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

int run_gemm(const GemmArgs &g, cudaStream_t stream) {
  constexpr int shm = GST * (GA_BYTES + GB_BYTES);
  static bool done[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !done[dev]) {
    if (cudaFuncSetAttribute(ix_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, shm) !=
        cudaSuccess)
      return tq_check_launch("cudaFuncSetAttribute(ix_gemm)");
    done[dev] = true;
  }
  dim3 grid(static_cast<unsigned>((g.M + GM - 1) / GM), (g.N + GN - 1) / GN);
  ix_gemm_kernel<<<grid, 128, shm, stream>>>(g);
  tq_count_launch(1);
  return tq_check_launch("ix_gemm_kernel");
}

bool index_codec_ok(const tq_codec *c) { return c->d == XD && c->qjl_k && c->mse_bits_k <= 3; }

uint32_t half_bits(float x) {   // fp32 -> fp16 bit pattern, round to nearest even
  const __half h = __float2half_rn(x);
  uint16_t b;
  memcpy(&b, &h, 2);
  return b;
}

int scan_grid_y(int64_t n, int nq) {
  const int64_t tiles = (n + RM - 1) / RM;
  const int qblocks = (nq + QN - 1) / QN;
  int64_t gy = sm_count() / qblocks;   // one wave: grid.x * grid.y <= SMs (one CTA per SM)
  if (gy > tiles) gy = tiles;
  return static_cast<int>(gy < 1 ? 1 : gy);
}

// Row blocks of the LUT scan: about two CTAs per SM in all, whole queries per CTA.
int lut_blocks(int64_t n, int nq) {
  int64_t b = (2LL * sm_count() + nq - 1) / nq;
  const int64_t max_b = (n + 255) / 256;
  if (b > max_b) b = max_b;
  return static_cast<int>(b < 1 ? 1 : b);
}

// q' = Pi q and q'' = S q' into the scan workspace (both scan paths).
int scan_query_prologue(const tq_codec *c, const float *q, int nq, float *q1, uint16_t *q1hl,
                        float *q2, cudaStream_t st) {
  QrotArgs qa;
  qa.q = q;
  qa.nq = nq;
  qa.q1 = q1;
  qa.q1hl = q1hl;
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
  g.out = q2;
  g.status = nullptr;
  return run_gemm(g, st);
}

}  // namespace

extern "C" {

int tq_index_workspace(const tq_codec *c, int64_t n, size_t *bytes) {
  if (!c || !bytes || n < 1) return tq_fail(TQ_ERR_INVALID_ARG, "index workspace: bad arguments");
  const int64_t rows = n < kIxBatch ? n : kIxBatch;
  *bytes = static_cast<size_t>((rows + 127) / 128 * 128) * 2 * XD * sizeof(uint16_t);   // whole 128-row tiles
  return TQ_OK;
}

int tq_index_build(const tq_codec *c, const float *x, int64_t n, uint8_t *kcode, uint16_t *kscale,
                   uint32_t *status, void *workspace, size_t ws_bytes, void *stream) {
  if (!c) return tq_fail(TQ_ERR_INVALID_ARG, "index: NULL codec");
  if (!index_codec_ok(c))
    return tq_fail(TQ_ERR_UNSUPPORTED, "index: needs a d = 1536 codec with QJL keys and 1..3 MSE bits");
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
    SketchArgs g;
    g.A = a.rbuf;
    g.B = c->S_tile;
    g.M = rows;
    g.plane = a.kcode + c->mse_bits_k * (XD / 8);
    g.plane_stride = planes * (XD / 8);
    g.status = status;
    g.wait_limit = 1u << 26;
    if (const char *e = getenv("TQ_WAIT_LIMIT")) g.wait_limit = static_cast<uint32_t>(strtoul(e, nullptr, 10));
    static bool sk_attr[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !sk_attr[dev]) {
      if (cudaFuncSetAttribute(ix_sketch_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(SK_SMEM)) != cudaSuccess)
        return tq_check_launch("cudaFuncSetAttribute(ix_sketch)");
      sk_attr[dev] = true;
    }
    const int64_t sk_tiles = (rows + 127) / 128 * SKN_T;
    const int sk_grid = static_cast<int>(sk_tiles < sm_count() ? sk_tiles : sm_count());
    ix_sketch_kernel<<<sk_grid, SK_T, SK_SMEM, st>>>(g);
    tq_count_launch(1);
    if (int e = tq_check_launch("ix_sketch_kernel")) return e;
  }
  return TQ_OK;
}

// Scan workspace, 256-byte aligned pieces: q' fp32, q' bf16 hi | lo (GEMM A),
// q'' fp32, the packed fp16 query operand, 2^-e per query, candidate lists.
struct ScanWs {
  size_t q1, q1hl, q2, qop, qinv, cand_s, cand_i, status, total;
};

ScanWs scan_ws(int nq, int k, int gy) {
  auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
  const size_t nqb = (nq + QN - 1) / QN;
  ScanWs w;
  size_t o = 0;
  w.q1 = o;
  o += up(static_cast<size_t>(nq) * XD * 4);
  w.q1hl = o;
  o += up(static_cast<size_t>(nq) * 2 * XD * 2);
  w.q2 = o;
  o += up(static_cast<size_t>(nq) * XD * 4);
  w.qop = o;
  o += up(nqb * XCH * QCH_BYTES);
  w.qinv = o;
  o += up(static_cast<size_t>(nq) * 4);
  const size_t nc = static_cast<size_t>(nq) * (2 * gy) * k;
  w.cand_s = o;
  o += up(nc * 4);
  w.cand_i = o;
  o += up(nc * 4);
  w.status = o;
  o += up(4);
  w.total = o;
  return w;
}

int tq_scan_workspace(const tq_codec *c, int64_t n, int nq, int k, size_t *bytes) {
  if (!c || !bytes || n < 1 || nq < 1 || k < 1 || k > SKMAX)
    return tq_fail(TQ_ERR_INVALID_ARG, "scan workspace: bad arguments (1 <= k <= 16)");
  const int gy = scan_grid_y(n, nq), lb = lut_blocks(n, nq);
  // covers both scan paths: 2 gy candidate lists (tensor cores) or lb (LUT)
  *bytes = scan_ws(nq, k, gy > (lb + 1) / 2 ? gy : (lb + 1) / 2).total;
  return TQ_OK;
}

int tq_scan_topk(const tq_codec *c, const uint8_t *kcode, const uint16_t *kscale, int64_t n,
                 const float *q, int nq, int k, int32_t *idx, float *score, void *workspace,
                 size_t ws_bytes, void *stream) {
  if (!c) return tq_fail(TQ_ERR_INVALID_ARG, "scan: NULL codec");
  if (!index_codec_ok(c))
    return tq_fail(TQ_ERR_UNSUPPORTED, "scan: needs a d = 1536 codec with QJL keys and 1..3 MSE bits");
  if (!kcode || !kscale || !q || !idx || !score || !workspace || n < 1 || nq < 1 || k < 1 ||
      k > SKMAX || k > n)
    return tq_fail(TQ_ERR_INVALID_ARG, "scan: NULL buffer or bad n / nq / k (1 <= k <= min(16, n))");
  if (n > 0x7fffffffLL) return tq_fail(TQ_ERR_INVALID_ARG, "scan: n must fit in int32 indices");
  const int gy = scan_grid_y(n, nq);
  const ScanWs W = scan_ws(nq, k, gy);
  if (ws_bytes < W.total) return tq_fail(TQ_ERR_WORKSPACE, "scan: workspace too small");
  if ((reinterpret_cast<uintptr_t>(kcode) | reinterpret_cast<uintptr_t>(q) |
       reinterpret_cast<uintptr_t>(workspace)) % 16 || reinterpret_cast<uintptr_t>(kscale) % 4)
    return tq_fail(TQ_ERR_ALIGNMENT, "scan: kcode/q/workspace need 16-byte, kscale 4-byte alignment");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t *w = static_cast<uint8_t *>(workspace);
  float *q1 = reinterpret_cast<float *>(w + W.q1);
  uint16_t *q1hl = reinterpret_cast<uint16_t *>(w + W.q1hl);
  float *q2 = reinterpret_cast<float *>(w + W.q2);
  uint16_t *qop = reinterpret_cast<uint16_t *>(w + W.qop);
  float *qinv = reinterpret_cast<float *>(w + W.qinv);
  float *cand_s = reinterpret_cast<float *>(w + W.cand_s);
  int32_t *cand_i = reinterpret_cast<int32_t *>(w + W.cand_i);
  uint32_t *status = reinterpret_cast<uint32_t *>(w + W.status);
  // q' = Pi q (fp32 and bf16 hi | lo), q'' = S q' (fp32) on the tensor cores
  if (int e = scan_query_prologue(c, q, nq, q1, q1hl, q2, st)) return e;
  // fp16 B operand with a power-of-two scale per query
  const float coef = sqrtf(static_cast<float>(M_PI) / 2.0f) / XD;
  QpackArgs pa;
  pa.q1 = q1;
  pa.q2 = q2;
  pa.nq = nq;
  pa.coef = coef;
  pa.qop = qop;
  pa.qinv = qinv;
  pa.status = status;
  const int nqp = (nq + QN - 1) / QN * QN;
  ix_qpack_kernel<<<(nqp + 7) / 8, 256, 0, st>>>(pa);
  tq_count_launch(1);
  if (int e = tq_check_launch("ix_qpack_kernel")) return e;
  // scan
  Scan2Args sa;
  sa.kcode = kcode;
  sa.kscale = kscale;
  sa.n = n;
  sa.qop = qop;
  sa.qinv = qinv;
  sa.nq = nq;
  const int64_t tiles = (n + RM - 1) / RM;
  sa.tiles_per_cta = static_cast<int>((tiles + gy - 1) / gy);
  sa.mbk = c->mse_bits_k;
  for (int e = 0; e < 64; ++e) {
    // index bits (b0 even, b0 odd, b1 even, b1 odd, b2 even, b2 odd)
    const int me = (e & 1) | ((e >> 2) & 1) << 1 | ((e >> 4) & 1) << 2;
    const int mo = ((e >> 1) & 1) | ((e >> 3) & 1) << 1 | ((e >> 5) & 1) << 2;
    const uint32_t lo = half_bits(me < (1 << sa.mbk) ? c->books.ck[me] : 0.f);
    const uint32_t hi = half_bits(mo < (1 << sa.mbk) ? c->books.ck[mo] : 0.f);
    sa.lut[e] = lo | (hi << 16);
  }
  sa.cand_s = cand_s;
  sa.cand_i = cand_i;
  sa.k = k;
  sa.err = status;
  sa.wait_limit = 1u << 26;
  if (const char *e = getenv("TQ_WAIT_LIMIT")) sa.wait_limit = static_cast<uint32_t>(strtoul(e, nullptr, 10));
  static bool done[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !done[dev]) {
    if (cudaFuncSetAttribute(ix_scan2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(SC_SMEM)) != cudaSuccess)
      return tq_check_launch("cudaFuncSetAttribute(ix_scan2)");
    done[dev] = true;
  }
  dim3 grid((nq + QN - 1) / QN, gy);
  cudaEvent_t ev0, ev1;
  tq_timing_events(&ev0, &ev1);
  if (ev0) cudaEventRecord(ev0, st);
  ix_scan2_kernel<<<grid, SCT, SC_SMEM, st>>>(sa);
  if (int e = tq_check_launch("ix_scan2_kernel")) return e;
  if (ev1) cudaEventRecord(ev1, st);
  ix_merge_kernel<<<(nq + 127) / 128, 128, 0, st>>>(cand_s, cand_i, nq, 2 * gy, k, idx, score, status);
  tq_count_launch(2);
  return tq_check_launch("ix_merge_kernel");
}

int tq_scan_topk_lut(const tq_codec *c, const uint8_t *kcode, const uint16_t *kscale, int64_t n,
                     const float *q, int nq, int k, int32_t *idx, float *score, void *workspace,
                     size_t ws_bytes, void *stream) {
  if (!c) return tq_fail(TQ_ERR_INVALID_ARG, "scan (LUT): NULL codec");
  if (!index_codec_ok(c))
    return tq_fail(TQ_ERR_UNSUPPORTED, "scan (LUT): needs a d = 1536 codec with QJL keys and 1..3 MSE bits");
  if (!kcode || !kscale || !q || !idx || !score || !workspace || n < 1 || nq < 1 || k < 1 ||
      k > SKMAX || k > n)
    return tq_fail(TQ_ERR_INVALID_ARG, "scan (LUT): NULL buffer or bad n / nq / k (1 <= k <= min(16, n))");
  if (n > 0x7fffffffLL) return tq_fail(TQ_ERR_INVALID_ARG, "scan (LUT): n must fit in int32 indices");
  size_t need = 0;
  tq_scan_workspace(c, n, nq, k, &need);
  if (ws_bytes < need) return tq_fail(TQ_ERR_WORKSPACE, "scan (LUT): workspace too small");
  if ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(workspace)) % 16 ||
      reinterpret_cast<uintptr_t>(kcode) % 4 || reinterpret_cast<uintptr_t>(kscale) % 4)
    return tq_fail(TQ_ERR_ALIGNMENT, "scan (LUT): q/workspace need 16-byte, kcode/kscale 4-byte alignment");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int lb = lut_blocks(n, nq);
  const int gy = scan_grid_y(n, nq);
  const ScanWs W = scan_ws(nq, k, gy > (lb + 1) / 2 ? gy : (lb + 1) / 2);
  uint8_t *w = static_cast<uint8_t *>(workspace);
  float *q1 = reinterpret_cast<float *>(w + W.q1);
  uint16_t *q1hl = reinterpret_cast<uint16_t *>(w + W.q1hl);
  float *q2 = reinterpret_cast<float *>(w + W.q2);
  if (int e = scan_query_prologue(c, q, nq, q1, q1hl, q2, st)) return e;
  LutArgs la;
  la.kcode = kcode;
  la.kscale = kscale;
  la.n = n;
  la.q1 = q1;
  la.q2 = q2;
  la.nq = nq;
  la.coef = sqrtf(static_cast<float>(M_PI) / 2.0f) / XD;
  la.mbk = c->mse_bits_k;
  for (int m = 0; m < 8; ++m) la.ck[m] = m < (1 << c->mse_bits_k) ? c->books.ck[m] : 0.f;
  la.rows_per_block = (n + lb - 1) / lb;
  la.cand_s = reinterpret_cast<float *>(w + W.cand_s);
  la.cand_i = reinterpret_cast<int32_t *>(w + W.cand_i);
  la.k = k;
  la.lists = lb;
  static bool done[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !done[dev]) {
    if (cudaFuncSetAttribute(ix_lut_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(LUT_SMEM)) != cudaSuccess)
      return tq_check_launch("cudaFuncSetAttribute(ix_lut)");
    done[dev] = true;
  }
  cudaEvent_t ev0, ev1;
  tq_timing_events(&ev0, &ev1);
  if (ev0) cudaEventRecord(ev0, st);
  ix_lut_kernel<<<dim3(nq, lb), LT, LUT_SMEM, st>>>(la);
  if (int e = tq_check_launch("ix_lut_kernel")) return e;
  if (ev1) cudaEventRecord(ev1, st);
  ix_merge_kernel<<<(nq + 127) / 128, 128, 0, st>>>(la.cand_s, la.cand_i, nq, lb, k, idx, score, nullptr);
  tq_count_launch(2);
  return tq_check_launch("ix_merge_kernel");
}

}  // extern "C"
