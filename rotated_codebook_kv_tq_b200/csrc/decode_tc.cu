// Tensor-core split-K decode from the compressed cache (sm_100a, tcgen05).
//
// Same computation as decode.cu ("TurboESM ..." section 2.E: one pass over the
// compressed cache; "Google presenta TurboQuant ...", "Eliminacion del sesgo":
// the prod estimator), restructured so every per-coordinate product runs on
// the 5th-generation tensor cores as exact integer MMAs:
//
// * A symmetric Lloyd-Max codebook is an odd function of its code bits, so
//   c[idx] = sum_S a_S (2 x_S - 1) over odd subsets S of the bit planes, with
//   x_S the XOR of the planes in S (exact; a_S solved on the host).  Every
//   key/value term is therefore a 0/1 plane.
// * A plane word w (32 coordinates or 32 tokens) becomes 8 registers
//   w & (0x01010101 << r), r = 0..7: four u8 MMA elements each, worth
//   x * 2^r.  They are stored straight into tensor memory (tcgen05.st) and fed
//   to tcgen05.mma kind::i8 as the A operand.  The 2^r weight is undone on the
//   B side: B holds 24-bit fixed-point values times 2^(7-r), split into four
//   signed 8-bit limbs, so each int32 accumulator is exact.
// * Keys: M = 128 key rows (TMEM lane = row), N = 4 limbs x G heads, K = terms x d.
//   Values: M = 128 coordinates (TMEM lane = coordinate; the cache's 32-token
//   column groups give each lane its own words), N = 4 limbs x G heads,
//   K = 32 tokens; one accumulator per Walsh term, combined at the end.
// * Persistent CTAs, one per SM, stream (chunk, sub-chunk) units through a
//   double-buffered shared-memory ring filled by cp.async.bulk.  Each CTA has
//   two 4-warp slices over the same 128 TMEM lanes that split the Walsh terms
//   of every expansion, and key tiles are double-buffered in tensor memory so
//   the expansion of tile j+1 overlaps the MMAs of tile j.
//
// Kernels: tc_prep (per (batch, KV head): RoPE, rotation and sketch of the G
// query heads, fixed-point B operand for the keys) and tc_chunk (the split-K
// main loop); the chunk partials are merged by decode.cu's combine kernel.
#include <math_constants.h>

#include <cstdlib>

#include "tq_device.cuh"
#include "tq_sm100.cuh"
#include "tq_tc.h"

namespace {

constexpr int TD = 128;   // head dim of this path
constexpr int TNW = TD / 32;
constexpr int TCT = 128;  // threads of tc_prep: one TMEM lane each
constexpr int CW = 256;   // worker threads of tc_chunk: two slices of 128 TMEM lanes
constexpr int CT = CW + 32;   // + the MMA-issuing warp

// Odd subsets of {0..nb-1} in increasing bit-mask order (the Walsh terms).
__host__ __device__ constexpr int odd_mask(int nb, int t) {
  int seen = 0;
  for (int m = 1; m < (1 << nb); ++m) {
    int pc = 0;
    for (int x = m; x; x >>= 1) pc += x & 1;
    if (pc & 1) {
      if (seen == t) return m;
      ++seen;
    }
  }
  return 0;
}

// Columns used by tc_chunk: key phase (two accumulator pairs in [0, 64), two
// A buffers of 32 columns per key term from 64) or value phase (two A buffers
// of 8 columns per Walsh term, then one accumulator of N columns per term).
__host__ __device__ constexpr int tc_tmem_cols(int G, int MBK, int BV, bool QJL) {
  return (64 + 64 * ((1 << (MBK - 1)) + (QJL ? 1 : 0))) > (2 * (1 << (BV - 1)) * 8 + (1 << (BV - 1)) * tc_n(G))
             ? (64 + 64 * ((1 << (MBK - 1)) + (QJL ? 1 : 0)))
             : (2 * (1 << (BV - 1)) * 8 + (1 << (BV - 1)) * tc_n(G));
}
__host__ __device__ constexpr int tc_tmem_alloc(int G, int MBK, int BV, bool QJL) {
  return tc_tmem_cols(G, MBK, BV, QJL) <= 64    ? 64
         : tc_tmem_cols(G, MBK, BV, QJL) <= 128 ? 128
         : tc_tmem_cols(G, MBK, BV, QJL) <= 256 ? 256
                                                 : 512;
}

// Signed base-256 digits of v (|v| < 2^31): v = L0 + 2^8 L1 + 2^16 L2 + 2^24 L3.
__device__ __forceinline__ int8_t limb_of(int v, int l) {
  int8_t d = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    d = static_cast<int8_t>(v & 0xff);
    if (i == l) break;
    v = (v - d) >> 8;
  }
  return d;
}

// Byte offset of element (n, k) in a K-major, no-swizzle operand of N rows.
__device__ __forceinline__ int kmajor_off(int n, int k, int N) {
  return (k >> 4) * (N * 16) + (n >> 3) * 128 + (n & 7) * 16 + (k & 15);
}

__device__ __forceinline__ float pow2_scale(float maxabs) {
  // largest power of two F with maxabs * F < 2^23 (1 when maxabs == 0)
  if (!(maxabs > 0.f)) return 1.f;
  int e;
  frexpf(maxabs, &e);               // maxabs in [2^(e-1), 2^e)
  return ldexpf(1.f, 23 - e);
}

// ---------------------------------------------------------------------------
// tc_prep: one block (128 threads) per (batch, KV head).
// ---------------------------------------------------------------------------
template <int G, int MBK, bool QJL>
__global__ void __launch_bounds__(TCT) tc_prep_kernel(TcArgs a) {
  constexpr int TK = 1 << (MBK - 1);
  constexpr int N = tc_n(G);
  constexpr int KM = TK * TD;                 // MSE K bytes
  constexpr int KTOT = KM + (QJL ? TD : 0);
  __shared__ float q1s[G][TD], q2s[G][TD];
  __shared__ float red[TCT / 32][2 * G];
  __shared__ double dred[TCT / 32][2 * G];
  __shared__ float Fs[2 * G];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int bh = blockIdx.x;
  const int b = bh / a.Hkv, kvh = bh % a.Hkv;
  const int len = a.seq_lens ? min(max(a.seq_lens[b], 1), a.max_len) : a.max_len;
  const int64_t pos = len - 1;

  if (warp < G) {
    const int64_t hq = static_cast<int64_t>(b) * a.Hq + kvh * G + warp;
    float x[TNW];
#pragma unroll
    for (int k = 0; k < TNW; ++k) x[k] = tq_load_elem(a.q, hq * TD + lane + 32 * k, a.dtype);
    if (a.rc != nullptr) {
      constexpr int HALF = TNW / 2;
#pragma unroll
      for (int k = 0; k < HALF; ++k) {
        const float c = a.rc[pos * (TD / 2) + lane + 32 * k];
        const float s = a.rs[pos * (TD / 2) + lane + 32 * k];
        const float u = x[k], v = x[k + HALF];
        x[k] = u * c - v * s;
        x[k + HALF] = v * c + u * s;
      }
    }
    tq_apply_signs<TNW>(x, a.books.dneg, lane);
    tq_warp_wht<TNW>(x, lane);
    const float inv_sqrt_d = 1.0f / sqrtf(static_cast<float>(TD));
#pragma unroll
    for (int k = 0; k < TNW; ++k) q1s[warp][lane + 32 * k] = x[k] * inv_sqrt_d;
  }
  __syncthreads();
  if (QJL) {
    // q''_i = sum_j S[i][j] q'_j: thread i reads row i of S (bf16) as 16-byte loads
    const uint4 *srow = reinterpret_cast<const uint4 *>(a.S + static_cast<int64_t>(tid) * TD);
    float acc[G];
#pragma unroll
    for (int h = 0; h < G; ++h) acc[h] = 0.f;
#pragma unroll 4
    for (int q = 0; q < TD / 8; ++q) {
      const uint4 v = srow[q];
      const uint32_t wds[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float sv = __uint_as_float((e & 1) ? (wds[e >> 1] & 0xffff0000u) : (wds[e >> 1] << 16));
#pragma unroll
        for (int h = 0; h < G; ++h) acc[h] = fmaf(sv, q1s[h][8 * q + e], acc[h]);
      }
    }
#pragma unroll
    for (int h = 0; h < G; ++h) q2s[h][tid] = acc[h];
  }
  __syncthreads();
  // fixed-point scales: largest |B value| of each head and part
  {
    float m1[G], m2[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      m1[h] = tq_warp_max(fabsf(q1s[h][tid]));
      m2[h] = QJL ? tq_warp_max(fabsf(q2s[h][tid])) : 0.f;
    }
    if (lane == 0)
#pragma unroll
      for (int h = 0; h < G; ++h) {
        red[warp][h] = m1[h];
        red[warp][G + h] = m2[h];
      }
    __syncthreads();
    if (tid < 2 * G) {
      float m = red[0][tid];
      for (int w = 1; w < TCT / 32; ++w) m = fmaxf(m, red[w][tid]);
      Fs[tid] = pow2_scale(2.f * (tid < G ? a.wk_absmax : 1.f) * m);
    }
    __syncthreads();
  }
  // B operand (K-major, no swizzle): MSE part then QJL part.  One item =
  // (head h, K chunk kc): its 16 fixed-point values are computed once and
  // split into the four limb rows n = 4h + l, each stored as one 16-byte
  // write straight to the group's global B region.
  uint8_t *dst = a.bk + static_cast<int64_t>(bh) * a.bk_stride;
  constexpr int NKC = KTOT / 16, NKM = KM / 16;
  for (int it = tid; it < G * NKC; it += TCT) {
    const int h = it % G, kc = it / G;
    const bool mse = kc < NKM;
    const int kb = mse ? kc * 16 : (kc - NKM) * 16;
    uint32_t wv[4][4] = {{0u, 0u, 0u, 0u}, {0u, 0u, 0u, 0u}, {0u, 0u, 0u, 0u}, {0u, 0u, 0u, 0u}};
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const int kk = kb + e;
      const int col = kk >> 2, nb = kk & 3;
      const int ti = col >> 5, w = (col & 31) >> 3, r = col & 7;
      const int i = 32 * w + 8 * nb + r;
      const float val = mse ? 2.f * a.wk[ti] * q1s[h][i] * Fs[h] : 2.f * q2s[h][i] * Fs[G + h];
      int v = __float2int_rn(val) * (1 << (7 - r));
      // signed base-256 digits: v = L0 + 2^8 L1 + 2^16 L2 + 2^24 L3
#pragma unroll
      for (int l = 0; l < 4; ++l) {
        const int8_t d = static_cast<int8_t>(v & 0xff);
        wv[l][e >> 2] |= static_cast<uint32_t>(static_cast<uint8_t>(d)) << (8 * (e & 3));
        v = (v - d) >> 8;
      }
    }
#pragma unroll
    for (int l = 0; l < 4; ++l)
      *reinterpret_cast<uint4 *>(dst + (mse ? 0 : N * KM) + kmajor_off(4 * h + l, kb, N)) =
          make_uint4(wv[l][0], wv[l][1], wv[l][2], wv[l][3]);
  }
  // rows beyond the G heads' limbs (N > 4 G) are zero
  if constexpr (N > 4 * G) {
    for (int it = tid; it < (N - 4 * G) * NKC; it += TCT) {
      const int n = 4 * G + it % (N - 4 * G), kc = it / (N - 4 * G);
      const bool mse = kc < NKM;
      const int kb = mse ? kc * 16 : (kc - NKM) * 16;
      *reinterpret_cast<uint4 *>(dst + (mse ? 0 : N * KM) + kmajor_off(n, kb, N)) = make_uint4(0u, 0u, 0u, 0u);
    }
  }
  // constants: C = sum of the quantized B values / (2F), per head and part
  {
    double c1[G], c2[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      double s1 = 0.0;
#pragma unroll
      for (int ti = 0; ti < TK; ++ti) s1 += __float2int_rn(2.f * a.wk[ti] * q1s[h][tid] * Fs[h]);
      c1[h] = s1;
      c2[h] = QJL ? static_cast<double>(__float2int_rn(2.f * q2s[h][tid] * Fs[G + h])) : 0.0;
    }
#pragma unroll
    for (int h = 0; h < G; ++h) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        c1[h] += __shfl_xor_sync(TQ_FULL, c1[h], o);
        c2[h] += __shfl_xor_sync(TQ_FULL, c2[h], o);
      }
    }
    if (lane == 0)
#pragma unroll
      for (int h = 0; h < G; ++h) {
        dred[warp][h] = c1[h];
        dred[warp][G + h] = c2[h];
      }
  }
  __syncthreads();
  if (tid < G) {
    double s1 = 0.0, s2 = 0.0;
    for (int w = 0; w < TCT / 32; ++w) {
      s1 += dred[w][tid];
      s2 += dred[w][G + tid];
    }
    float *kc = reinterpret_cast<float *>(dst + N * KTOT);
    kc[tid * 4 + 0] = static_cast<float>(s1 / (2.0 * Fs[tid]));
    kc[tid * 4 + 1] = 1.0f / (128.0f * Fs[tid]);
    kc[tid * 4 + 2] = static_cast<float>(s2 / (2.0 * Fs[G + tid]));
    kc[tid * 4 + 3] = 1.0f / (128.0f * Fs[G + tid]);
  }
}

// ---------------------------------------------------------------------------
// tc_chunk: persistent, one CTA (128 threads, one TMEM lane each) per SM.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float comb_limbs(const uint32_t *d) {
  // int32 accumulators of limbs 0..3 -> value (exact digits, fp32 rounding)
  float v = static_cast<float>(static_cast<int>(d[3]));
  v = fmaf(v, 256.f, static_cast<float>(static_cast<int>(d[2])));
  v = fmaf(v, 256.f, static_cast<float>(static_cast<int>(d[1])));
  return fmaf(v, 256.f, static_cast<float>(static_cast<int>(d[0])));
}

struct TcLayout {
  int o_ks, o_vc, o_vn, o_bk, ubytes, o_bv, o_lg, total;
};

__host__ __device__ inline TcLayout tc_layout(int sub, int PK, int BV, int G, int N, int BKC) {
  TcLayout L;
  L.o_ks = sub * PK * 16;
  L.o_vc = L.o_ks + sub * 4;
  L.o_vn = L.o_vc + (sub / 32) * BV * TD * 4;
  L.o_bk = L.o_vn + sub * 2;
  L.ubytes = (L.o_bk + BKC + 127) & ~127;
  L.o_bv = 2 * L.ubytes;
  L.o_lg = L.o_bv + (sub / 32) * N * 32;
  L.total = L.o_lg + sub * G * 4;
  return L;
}

__device__ __forceinline__ int tc_len(const TcArgs &a, int b) {
  return a.seq_lens ? min(max(a.seq_lens[b], 1), a.max_len) : a.max_len;
}

// Move (it, r0) to the next non-empty unit of this CTA; r0 < 0 means "start
// of item".  Returns false when the CTA has no work left.
__device__ __forceinline__ bool tc_next(const TcArgs &a, int &it, int &r0) {
  const int items = a.B * a.Hkv * a.splits;
  while (it < items) {
    const int b = it / (a.Hkv * a.splits), sp = it % a.splits;
    const int c0 = sp * a.chunk, c1 = min(tc_len(a, b), c0 + a.chunk);
    if (r0 < 0) r0 = c0;
    if (r0 < c1) return true;
    it += gridDim.x;
    r0 = -1;
  }
  return false;
}

// tc_chunk: 288 threads = 8 worker warps (two slices of 4) + 1 MMA warp.
// Worker warp w serves TMEM lane quarter w % 4 (rows or coordinates
// 32 (w % 4) .. +31) for slice w / 4; the slices split the Walsh terms of
// every expansion and the rows of the value B-operand build.  A tcgen05.mma
// issue blocks for about as long as the MMA runs, so one lane of the last
// warp does nothing but issue: workers publish each filled tensor-memory
// buffer on an mbarrier (ak_full / av_full) and the MMA warp waits on those;
// workers wait on the MMA commits (mb_k / mb_v) before reusing a buffer.
// Key tiles are double-buffered: tile j+1 is expanded while tile j runs.
template <int G, int MBK, int BV, bool QJL>
__global__ void __launch_bounds__(CT, 1) tc_chunk_kernel(TcArgs a) {
  constexpr int NWW = CW / 32;               // worker warps
  constexpr int TK = 1 << (MBK - 1);
  constexpr int TV = 1 << (BV - 1);
  constexpr int N = tc_n(G);
  constexpr int PK = MBK + (QJL ? 1 : 0);
  constexpr int KM = TK * TD;
  constexpr int KTOT = KM + (QJL ? TD : 0);
  constexpr int BKB = N * KTOT;
  constexpr int BKC = BKB + G * 16;
  constexpr int NKT = TK + (QJL ? 1 : 0);   // key terms: TK Walsh terms + the sign plane
  // Tensor memory: the key phase and the value phase of a unit never overlap
  // in time, so their regions share columns.
  //   key phase:   DK[b] [32 b, 32 b + 2N)   AK[b] [64 + 32 NKT b, 64 + 32 NKT (b + 1))
  //   value phase: AV [0, 16 TV) (two buffers)   DV [16 TV, 16 TV + N TV)
  constexpr int C_DK = 0;
  constexpr int C_AK = 64;
  constexpr int C_AV = 0;
  constexpr int C_DV = 2 * TV * 8;
  constexpr int USED = tc_tmem_cols(G, MBK, BV, QJL);
  constexpr int NCOLS = tc_tmem_alloc(G, MBK, BV, QJL);
  static_assert(USED <= 512, "tensor memory budget");
  static_assert(2 * N <= 32, "key accumulators must fit in 32 columns");
  constexpr uint32_t IDESC = sm100::idesc_i8(128, N);

  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ __align__(8) uint64_t mb_load[2], mb_k[2], mb_v[2], ak_full[2], av_full[2];
  __shared__ uint32_t tmem_s;
  __shared__ float redf[NWW][2 * G + 1];
  __shared__ long long redi[NWW][G];
  __shared__ float part[G][TD];
  __shared__ int abort_s;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int wq = warp & 3;            // TMEM lane quarter
  const int slice = warp >> 2;        // 0 or 1
  const int lt = tid & 127;           // TMEM lane = row (keys) or coordinate (values)
  const int sub = a.sub;
  const TcLayout L = tc_layout(sub, PK, BV, G, N, BKC);
  int8_t *bvs = reinterpret_cast<int8_t *>(smem + L.o_bv);
  float *lg = reinterpret_cast<float *>(smem + L.o_lg);

  if (warp == 0) sm100::tmem_alloc(&tmem_s, NCOLS);
  if (tid == 0) {
    sm100::mbar_init(&mb_load[0], 1);
    sm100::mbar_init(&mb_load[1], 1);
    sm100::mbar_init(&mb_k[0], 1);
    sm100::mbar_init(&mb_k[1], 1);
    sm100::mbar_init(&mb_v[0], 1);
    sm100::mbar_init(&mb_v[1], 1);
    sm100::mbar_init(&ak_full[0], NWW);
    sm100::mbar_init(&ak_full[1], NWW);
    sm100::mbar_init(&av_full[0], NWW);
    sm100::mbar_init(&av_full[1], NWW);
    abort_s = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  sm100::fence_before_sync();
  __syncthreads();
  sm100::fence_after_sync();
  const uint32_t tm = tmem_s;

  if (warp == NWW) {
    // ---------------- MMA warp: walks the same units as the workers
    if (lane == 0) {
      int cit = blockIdx.x, cr0 = -1, u = 0;
      uint32_t akph = 0, avph = 0;
      bool have = tc_next(a, cit, cr0);
      bool ok = true;
      while (have && ok) {
        int nit = cit, nr0 = cr0 + sub;
        const bool nhave = tc_next(a, nit, nr0);
        uint8_t *ub = smem + (u & 1) * L.ubytes;
        const int b = cit / (a.Hkv * a.splits), sp = cit % a.splits;
        const int c0 = sp * a.chunk, c1 = min(tc_len(a, b), c0 + a.chunk);
        const int nvalid = min(sub, c1 - cr0);
        const uint32_t bk_addr = sm100::smem_addr(ub + L.o_bk);
        const int ntile = (nvalid + 127) / 128, ngroups = (nvalid + 31) / 32;
        for (int j = 0; j < ntile && ok; ++j) {
          const int kb = j & 1;
          ok = sm100::mbar_wait(&ak_full[kb], (akph >> kb) & 1);
          akph ^= 1u << kb;
          if (!ok) break;
          sm100::fence_after_sync();
          const uint32_t ak = tm + C_AK + kb * 32 * NKT, dk = tm + C_DK + kb * 32;
#pragma unroll
          for (int s = 0; s < TK * 4; ++s)
            sm100::mma_i8_ts(dk, ak + s * 8, sm100::smem_desc(bk_addr + s * 2 * N * 16, N * 16, 128),
                             IDESC, s > 0);
          if (QJL) {
#pragma unroll
            for (int s = 0; s < 4; ++s)
              sm100::mma_i8_ts(dk + N, ak + TK * 32 + s * 8,
                               sm100::smem_desc(bk_addr + N * KM + s * 2 * N * 16, N * 16, 128),
                               IDESC, s > 0);
          }
          sm100::mma_commit(&mb_k[kb]);
        }
        const uint32_t bv_addr = sm100::smem_addr(bvs);
        for (int g = 0; g < ngroups && ok; ++g) {
          const int ab = g & 1;
          ok = sm100::mbar_wait(&av_full[ab], (avph >> ab) & 1);
          avph ^= 1u << ab;
          if (!ok) break;
          sm100::fence_after_sync();
          const uint64_t bd = sm100::smem_desc(bv_addr + g * N * 32, N * 16, 128);
#pragma unroll
          for (int ti = 0; ti < TV; ++ti)
            sm100::mma_i8_ts(tm + C_DV + ti * N, tm + C_AV + ab * TV * 8 + ti * 8, bd, IDESC, g > 0);
          sm100::mma_commit(&mb_v[ab]);
        }
        cit = nit;
        cr0 = nr0;
        have = nhave;
        ++u;
      }
      // a wait that gave up leaves the workers to time out on the commits
      // they expect and take their own abort path
    }
    __syncwarp();
  } else {
  // ---------------- workers
  // empty chunks (beyond a batch's length) merge with weight zero
  const int items = a.B * a.Hkv * a.splits;
  for (int it = blockIdx.x; it < items; it += gridDim.x) {
    const int b = it / (a.Hkv * a.splits), kvh = (it / a.splits) % a.Hkv, sp = it % a.splits;
    if (sp * a.chunk < tc_len(a, b)) continue;
    if (tid < TD)
      for (int h = 0; h < G; ++h) {
        const int64_t hq = static_cast<int64_t>(b) * a.Hq + kvh * G + h;
        a.po[(hq * a.splits + sp) * TD + tid] = 0.f;
        if (tid == 0) {
          a.pml[(hq * a.splits + sp) * 2] = -CUDART_INF_F;
          a.pml[(hq * a.splits + sp) * 2 + 1] = 0.f;
        }
      }
  }

  auto issue = [&](int buf, int it, int r0) {
    const int b = it / (a.Hkv * a.splits), kvh = (it / a.splits) % a.Hkv;
    const int64_t bh = static_cast<int64_t>(b) * a.Hkv + kvh;
    const int nrow = static_cast<int>(min(static_cast<int64_t>(sub), a.rows_cap - r0));
    uint8_t *u = smem + buf * L.ubytes;
    const uint32_t b_kc = nrow * PK * 16, b_ks = nrow * 4, b_vc = (nrow / 32) * BV * TD * 4,
                   b_vn = nrow * 2, b_bk = (BKC + 15) & ~15;
    sm100::mbar_expect_tx(&mb_load[buf], b_kc + b_ks + b_vc + b_vn + b_bk);
    sm100::bulk_g2s(u, a.kcode + (bh * a.rows_cap + r0) * PK * 16, b_kc, &mb_load[buf]);
    sm100::bulk_g2s(u + L.o_ks, a.kscale + (bh * a.rows_cap + r0) * 2, b_ks, &mb_load[buf]);
    sm100::bulk_g2s(u + L.o_vc, a.vcode + (bh * (a.rows_cap / 32) + r0 / 32) * BV * TD, b_vc,
                    &mb_load[buf]);
    sm100::bulk_g2s(u + L.o_vn, a.vnorm + bh * a.rows_cap + r0, b_vn, &mb_load[buf]);
    sm100::bulk_g2s(u + L.o_bk, a.bk + bh * a.bk_stride, b_bk, &mb_load[buf]);
  };
  // worker-only barrier (named barrier 1 over the 256 worker threads)
  auto wsync = [&]() { sm100::named_sync(1, CW); };
  auto wait_all = [&](uint64_t *bar, uint32_t parity) -> bool {
    if (lane == 0 && !sm100::mbar_wait(bar, parity)) abort_s = 1;
    wsync();
    return abort_s == 0;
  };
  auto sync_tc = [&]() {
    sm100::fence_before_sync();
    wsync();
    sm100::fence_after_sync();
  };
  // this warp's tcgen05.st are complete: publish them to the MMA warp
  auto publish = [&](uint64_t *bar) {
    sm100::fence_before_sync();
    __syncwarp();
    if (lane == 0) sm100::mbar_arrive(bar);
  };

  int cit = blockIdx.x, cr0 = -1;
  bool have = tc_next(a, cit, cr0);
  if (have && tid == 0) issue(0, cit, cr0);
  int inflight = have ? 0 : -1;   // buffer whose bulk copies were issued, not yet waited
  // barrier parities: bit b of kph / vph / lph is the parity to wait for next on buffer b
  uint32_t kph = 0, vph = 0, lph = 0;
  float o[G], m_run[G], l_run[G];
  int u = 0;
  while (have) {
    int nit = cit, nr0 = cr0 + sub;
    const bool nhave = tc_next(a, nit, nr0);
    if (nhave && tid == 0) {
      sm100::fence_async_smem();
      issue((u + 1) & 1, nit, nr0);
    }
    const int buf = u & 1;
    if (!wait_all(&mb_load[buf], (lph >> buf) & 1)) break;
    lph ^= 1u << buf;
    inflight = nhave ? (u + 1) & 1 : -1;
    uint8_t *ub = smem + buf * L.ubytes;

    const int b = cit / (a.Hkv * a.splits), kvh = (cit / a.splits) % a.Hkv, sp = cit % a.splits;
    const int len = tc_len(a, b);
    const int c0 = sp * a.chunk, c1 = min(len, c0 + a.chunk);
    const int nvalid = min(sub, c1 - cr0);
    if (cr0 == c0) {
#pragma unroll
      for (int h = 0; h < G; ++h) {
        o[h] = 0.f;
        m_run[h] = -CUDART_INF_F;
        l_run[h] = 0.f;
      }
    }
    const float *kcst = reinterpret_cast<const float *>(ub + L.o_bk + BKB);
    const uint32_t bk_addr = sm100::smem_addr(ub + L.o_bk);

    // ---------------- keys: logits of the G heads, 128 rows per tile
    // expand tile j's bit planes (this slice's terms) into AK[kb]
    auto expand_keys = [&](int j, int kb) {
      const int rl = j * 128 + lt;
      uint32_t pw[PK][TNW];
      const uint4 *kr = reinterpret_cast<const uint4 *>(ub + rl * PK * 16);
#pragma unroll
      for (int p = 0; p < PK; ++p) {
        const uint4 v = kr[p];
        pw[p][0] = v.x;
        pw[p][1] = v.y;
        pw[p][2] = v.z;
        pw[p][3] = v.w;
      }
      const uint32_t ak = tm + C_AK + kb * 32 * NKT;
#pragma unroll
      for (int t = 0; t < NKT; ++t) {
        if ((t & 1) != slice) continue;
#pragma unroll
        for (int w = 0; w < TNW; ++w) {
          uint32_t x = 0;
          if (t < TK) {
            const int mask = odd_mask(MBK, t);
#pragma unroll
            for (int p = 0; p < MBK; ++p)
              if ((mask >> p) & 1) x ^= pw[p][w];
          } else {
            x = pw[PK - 1][w];
          }
          uint32_t r8[8];
#pragma unroll
          for (int r = 0; r < 8; ++r) r8[r] = x & (0x01010101u << r);
          sm100::tmem_st8(sm100::tmem_lane(ak + t * 32 + w * 8, wq), r8);
        }
      }
      sm100::wait_st();
    };
    float mloc[G];
#pragma unroll
    for (int h = 0; h < G; ++h) mloc[h] = -CUDART_INF_F;
    const int ntile = (nvalid + 127) / 128;
    bool ok = true;
    expand_keys(0, 0);
    publish(&ak_full[0]);
    for (int j = 0; j < ntile; ++j) {
      const int kb = j & 1;
      if (j + 1 < ntile) {
        // AK[kb ^ 1] and DK[kb ^ 1] were released by tile j - 1 (waited, read)
        expand_keys(j + 1, kb ^ 1);
        publish(&ak_full[kb ^ 1]);
      }
      ok = wait_all(&mb_k[kb], (kph >> kb) & 1);
      kph ^= 1u << kb;
      if (!ok) break;
      sm100::fence_after_sync();
      if (slice == 0) {
        const int rl = j * 128 + lt;
        const bool valid = rl < nvalid;
        uint32_t dk[2 * N];
        const uint32_t dka = tm + C_DK + kb * 32;
        if (N == 16) {
          uint32_t t0[16], t1[16];
          sm100::tmem_ld16(sm100::tmem_lane(dka, wq), t0);
          sm100::tmem_ld16(sm100::tmem_lane(dka + 16, wq), t1);
          sm100::wait_ld();
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            dk[c] = t0[c];
            dk[N + c] = t1[c];
          }
        } else {
          uint32_t t0[8], t1[8];
          sm100::tmem_ld8(sm100::tmem_lane(dka, wq), t0);
          sm100::tmem_ld8(sm100::tmem_lane(dka + N, wq), t1);
          sm100::wait_ld();
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            dk[c] = t0[c];
            dk[N + c] = t1[c];
          }
        }
        const uint32_t sc = reinterpret_cast<const uint32_t *>(ub + L.o_ks)[rl];
        const float nu = tq_half_to_f32(static_cast<uint16_t>(sc & 0xffffu));
        const float rho = tq_half_to_f32(static_cast<uint16_t>(sc >> 16));
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float dm = comb_limbs(dk + 4 * h) * kcst[4 * h + 1] - kcst[4 * h + 0];
          float est = dm;
          if (QJL) {
            const float dj = comb_limbs(dk + N + 4 * h) * kcst[4 * h + 3] - kcst[4 * h + 2];
            est = fmaf(a.qjl_coef * rho, dj, dm);
          }
          const float l = valid ? a.scale * nu * est : -CUDART_INF_F;
          lg[rl * G + h] = l;
          mloc[h] = fmaxf(mloc[h], l);
          if (a.logits && valid)
            a.logits[(static_cast<int64_t>(b) * a.Hq + kvh * G + h) * a.max_len + cr0 + rl] = l;
        }
      }
    }
    if (!ok) break;

    // ---------------- softmax statistics of the unit
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float m = tq_warp_max(mloc[h]);
      if (lane == 0) redf[warp][h] = m;
    }
    sync_tc();   // the key epilogue's TMEM reads are complete before any value-phase store
    float mnew[G], corr[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float m = redf[0][h];
#pragma unroll
      for (int w = 1; w < NWW; ++w) m = fmaxf(m, redf[w][h]);
      mnew[h] = fmaxf(m_run[h], m);
      corr[h] = __expf(m_run[h] - mnew[h]);
    }
    const uint16_t *vn = reinterpret_cast<const uint16_t *>(ub + L.o_vn);
    float lsum[G], numax = 0.f;
#pragma unroll
    for (int h = 0; h < G; ++h) lsum[h] = 0.f;
    for (int rl = tid; rl < nvalid; rl += CW) {
      numax = fmaxf(numax, tq_half_to_f32(vn[rl]));
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float p = __expf(lg[rl * G + h] - mnew[h]);
        lg[rl * G + h] = p;
        lsum[h] += p;
      }
    }
    wsync();
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float s = tq_warp_sum(lsum[h]);
      if (lane == 0) redf[warp][h] = s;
    }
    {
      const float m = tq_warp_max(numax);
      if (lane == 0) redf[warp][2 * G] = m;
    }
    wsync();
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float s = 0.f;
#pragma unroll
      for (int w = 0; w < NWW; ++w) s += redf[w][h];
      lsum[h] = s;
    }
    float nmax = redf[0][2 * G];
#pragma unroll
    for (int w = 1; w < NWW; ++w) nmax = fmaxf(nmax, redf[w][2 * G]);
    const float FV = pow2_scale(nmax);
    const float invFV = 1.0f / (128.0f * FV);

    // ---------------- value-side B operand: 24-bit weights p * nu_v, limbs
    const int ngroups = (nvalid + 31) / 32;
    long long wsum[G];
#pragma unroll
    for (int h = 0; h < G; ++h) wsum[h] = 0;
    for (int rl = tid; rl < ngroups * 32; rl += CW) {
      const int g = rl >> 5, jj = rl & 31, r = jj & 7, nb = jj >> 3;
      const int k = 4 * r + nb;
      int8_t *dst = bvs + g * N * 32;
      const float nv = rl < nvalid ? tq_half_to_f32(vn[rl]) : 0.f;
#pragma unroll
      for (int h = 0; h < N / 4; ++h) {
        int W = 0;
        if (h < G && rl < nvalid) W = __float2int_rn(lg[rl * G + h] * nv * FV);
        if (h < G) wsum[h] += W;
        const int v = W * (1 << (7 - r));
#pragma unroll
        for (int l = 0; l < 4; ++l) dst[kmajor_off(4 * h + l, k, N)] = limb_of(v, l);
      }
    }
#pragma unroll
    for (int h = 0; h < G; ++h) {
      long long s = wsum[h];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(TQ_FULL, s, off);
      if (lane == 0) redi[warp][h] = s;
    }
    sm100::fence_async_smem();
    wsync();
    float wtot[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      long long s = 0;
#pragma unroll
      for (int w = 0; w < NWW; ++w) s += redi[w][h];
      wtot[h] = static_cast<float>(s) / FV;
      o[h] *= corr[h];
      l_run[h] = l_run[h] * corr[h] + lsum[h];
      m_run[h] = mnew[h];
    }

    // ---------------- values: rotated-domain sums, 32 tokens per MMA step
    const uint32_t *vc = reinterpret_cast<const uint32_t *>(ub + L.o_vc);
    for (int g = 0; g < ngroups && ok; ++g) {
      const int ab = g & 1;
      if (g >= 2) {  // buffer ab was last fed to the MMAs of group g - 2
        ok = wait_all(&mb_v[ab], (vph >> ab) & 1);
        vph ^= 1u << ab;
        if (!ok) break;
      }
      uint32_t pw[BV];
#pragma unroll
      for (int p = 0; p < BV; ++p) pw[p] = vc[(g * BV + p) * TD + lt];
#pragma unroll
      for (int ti = 0; ti < TV; ++ti) {
        if ((ti & 1) != slice) continue;
        const int mask = odd_mask(BV, ti);
        uint32_t x = 0;
#pragma unroll
        for (int p = 0; p < BV; ++p)
          if ((mask >> p) & 1) x ^= pw[p];
        uint32_t r8[8];
#pragma unroll
        for (int r = 0; r < 8; ++r) r8[r] = x & (0x01010101u << r);
        sm100::tmem_st8(sm100::tmem_lane(tm + C_AV + ab * TV * 8 + ti * 8, wq), r8);
      }
      sm100::wait_st();
      publish(&av_full[ab]);
    }
    // the last one or two groups' MMAs are still outstanding
    for (int g = ngroups > 2 ? ngroups - 2 : 0; g < ngroups && ok; ++g) {
      const int ab = g & 1;
      ok = wait_all(&mb_v[ab], (vph >> ab) & 1);
      vph ^= 1u << ab;
    }
    if (!ok) break;
    sm100::fence_after_sync();
    // each slice folds its Walsh terms for coordinate lt; slice 1 hands its
    // partial sums to slice 0, which keeps the running output
    {
      float acc[G];
#pragma unroll
      for (int h = 0; h < G; ++h) acc[h] = 0.f;
#pragma unroll
      for (int ti = 0; ti < TV; ++ti) {
        if ((ti & 1) != slice) continue;
        uint32_t dv[N];
        if (N == 16) {
          uint32_t t0[16];
          sm100::tmem_ld16(sm100::tmem_lane(tm + C_DV + ti * N, wq), t0);
          sm100::wait_ld();
#pragma unroll
          for (int c = 0; c < 16; ++c) dv[c] = t0[c];
        } else {
          uint32_t t0[8];
          sm100::tmem_ld8(sm100::tmem_lane(tm + C_DV + ti * N, wq), t0);
          sm100::wait_ld();
#pragma unroll
          for (int c = 0; c < 8; ++c) dv[c] = t0[c];
        }
#pragma unroll
        for (int h = 0; h < G; ++h) acc[h] = fmaf(2.f * a.wv[ti], comb_limbs(dv + 4 * h), acc[h]);
      }
      if (slice == 1) {
#pragma unroll
        for (int h = 0; h < G; ++h) part[h][lt] = acc[h];
      }
      wsync();
      if (slice == 0) {
#pragma unroll
        for (int h = 0; h < G; ++h) o[h] += (acc[h] + part[h][lt]) * invFV - a.wv_sum * wtot[h];
      }
    }
    if (cr0 + sub >= c1 && slice == 0) {
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const int64_t hq = static_cast<int64_t>(b) * a.Hq + kvh * G + h;
        a.po[(hq * a.splits + sp) * TD + lt] = o[h];
        if (tid == 0) {
          a.pml[(hq * a.splits + sp) * 2] = m_run[h];
          a.pml[(hq * a.splits + sp) * 2 + 1] = l_run[h];
        }
      }
    }
    sync_tc();
    cit = nit;
    cr0 = nr0;
    have = nhave;
    ++u;
  }
  if (abort_s) {
    // a bounded wait gave up: let this CTA's own outstanding copies and MMAs
    // land (again bounded) before its shared and tensor memory are released
    if (inflight >= 0) sm100::mbar_wait(&mb_load[inflight], (lph >> inflight) & 1, 1u << 20);
    sm100::mbar_wait(&mb_k[0], kph & 1, 1u << 20);
    sm100::mbar_wait(&mb_k[1], (kph >> 1) & 1, 1u << 20);
    sm100::mbar_wait(&mb_v[0], vph & 1, 1u << 20);
    sm100::mbar_wait(&mb_v[1], (vph >> 1) & 1, 1u << 20);
    if (tid == 0 && a.err) atomicExch(a.err, 1u);
  }
  }  // workers
  sm100::fence_before_sync();
  __syncthreads();
  sm100::fence_after_sync();
  if (warp == 0) sm100::tmem_dealloc(tm, NCOLS);
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
struct TcCfg {
  int G, mbk, bv, qjl;
};

constexpr TcCfg kTcConfigs[] = {{4, 3, 4, 1}, {4, 1, 2, 1}, {4, 2, 3, 1}, {2, 3, 4, 1},
                                {2, 1, 2, 1}, {2, 2, 3, 1}, {1, 3, 4, 1}, {1, 1, 2, 1},
                                {1, 2, 3, 1}};

template <int G, int MBK, int BV, bool QJL>
int run_tc(TcArgs &a, cudaStream_t stream) {
  constexpr int TK = 1 << (MBK - 1);
  constexpr int N = tc_n(G);
  constexpr int PK = MBK + (QJL ? 1 : 0);
  constexpr int BKC = N * (TK * TD + (QJL ? TD : 0)) + G * 16;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // CTAs per SM: one by default (largest sub-chunks); TQ_TC_CTAS_PER_SM asks
  // for more, capped by tensor-memory slots, after which the sub-chunk shrinks
  // until that many fit in shared memory (each unit is double-buffered)
  constexpr int NCOLS = tc_tmem_alloc(G, MBK, BV, QJL);
  int per_sm = 1;
  if (const char *e = getenv("TQ_TC_CTAS_PER_SM")) per_sm = atoi(e);
  if (per_sm > 512 / NCOLS) per_sm = 512 / NCOLS;
  if (per_sm > 4) per_sm = 4;
  if (per_sm < 1) per_sm = 1;
  const int budget = per_sm == 1 ? 200 * 1024 : (227 * 1024) / per_sm - 2048;
  int sub = a.chunk;
  while (sub > 128 && tc_layout(sub, PK, BV, G, N, BKC).total > budget) sub -= 128;
  a.sub = sub;
  const int smem = tc_layout(sub, PK, BV, G, N, BKC).total;
  static bool attr_done[64] = {};
  if (dev < 64 && !attr_done[dev]) {
    if (cudaFuncSetAttribute(tc_chunk_kernel<G, MBK, BV, QJL>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, 210 * 1024) != cudaSuccess)
      return tq_check_launch("cudaFuncSetAttribute(tc_chunk)");
    attr_done[dev] = true;
  }
  int occ = 1;
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, tc_chunk_kernel<G, MBK, BV, QJL>, CT, smem);
  if (occ < 1) occ = 1;
  if (occ < per_sm) per_sm = occ;
  tc_prep_kernel<G, MBK, QJL><<<a.B * a.Hkv, TCT, 0, stream>>>(a);
  if (int e = tq_check_launch("tc_prep_kernel")) return e;
  const int items = a.B * a.Hkv * a.splits;
  const int grid = items < sms * per_sm ? items : sms * per_sm;
  cudaEvent_t ev0, ev1;
  tq_timing_events(&ev0, &ev1);
  unsigned ev_flags = cudaEventRecordDefault;
  if (ev0) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    cudaStreamIsCapturing(stream, &cs);
    if (cs == cudaStreamCaptureStatusActive) ev_flags = cudaEventRecordExternal;
    cudaEventRecordWithFlags(ev0, stream, ev_flags);
  }
  tc_chunk_kernel<G, MBK, BV, QJL><<<grid, CT, smem, stream>>>(a);
  if (int e = tq_check_launch("tc_chunk_kernel")) return e;
  if (ev1) cudaEventRecordWithFlags(ev1, stream, ev_flags);
  tq_count_launch(2);
  return TQ_OK;
}

}  // namespace

bool tc_supported(const tq_codec *c, int G) {
  if (c->d != TD) return false;
  for (const TcCfg &k : kTcConfigs)
    if (k.G == G && k.mbk == c->mse_bits_k && k.bv == c->bits_v && k.qjl == c->qjl_k) return true;
  return false;
}

int tc_bk_stride(const tq_codec *c, int G) {
  const int TK = 1 << (c->mse_bits_k - 1);
  const int bytes = tc_n(G) * (TK * TD + (c->qjl_k ? TD : 0)) + G * 16;
  return (bytes + 127) & ~127;
}

int launch_decode_tc(const tq_codec *c, const void *q, int dtype, int B, int Hq, int Hkv,
                     const tq_cache *cache, const int32_t *seq_lens, int max_len, float scale,
                     const float *rc, const float *rs, int splits, float *po, float *pml,
                     uint8_t *bk, float *logits, cudaStream_t stream) {
  TcArgs a;
  a.q = q;
  a.dtype = dtype;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.kcode = cache->kcode;
  a.kscale = cache->kscale;
  a.vcode = cache->vcode;
  a.vnorm = cache->vnorm;
  a.rows_cap = cache->rows_cap;
  a.seq_lens = seq_lens;
  a.max_len = max_len;
  a.scale = scale;
  a.qjl_coef = c->qjl_k ? sqrtf(static_cast<float>(M_PI) / 2.0f) / c->d : 0.f;
  a.rc = rc;
  a.rs = rs;
  a.S = c->S_dev;
  a.ST = c->ST_dev;
  a.splits = splits;
  const int per = (max_len + splits - 1) / splits;
  a.chunk = (per + 127) / 128 * 128;
  a.sub = a.chunk;
  const int G = Hq / Hkv;
  a.bk = bk;
  a.bk_stride = tc_bk_stride(c, G);
  a.po = po;
  a.pml = pml;
  a.logits = logits;
  for (int i = 0; i < 8; ++i) {
    a.wk[i] = c->walsh_k[i];
    a.wv[i] = c->walsh_v[i];
  }
  a.wk_absmax = c->walsh_k_absmax;
  a.wv_sum = c->walsh_v_sum;
  a.err = nullptr;
  a.books = c->books;
  const int key = G * 1000 + c->mse_bits_k * 100 + c->bits_v * 10 + c->qjl_k;
  switch (key) {
    case 4341: return run_tc<4, 3, 4, true>(a, stream);
    case 4121: return run_tc<4, 1, 2, true>(a, stream);
    case 4231: return run_tc<4, 2, 3, true>(a, stream);
    case 2341: return run_tc<2, 3, 4, true>(a, stream);
    case 2121: return run_tc<2, 1, 2, true>(a, stream);
    case 2231: return run_tc<2, 2, 3, true>(a, stream);
    case 1341: return run_tc<1, 3, 4, true>(a, stream);
    case 1121: return run_tc<1, 1, 2, true>(a, stream);
    case 1231: return run_tc<1, 2, 3, true>(a, stream);
    default: return tq_fail(TQ_ERR_UNSUPPORTED, "tensor-core decode: configuration not built");
  }
}
