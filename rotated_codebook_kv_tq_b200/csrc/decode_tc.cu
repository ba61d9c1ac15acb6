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
// * dec_kernel (two CTAs per SM) walks (batch, KV head, split) units of at
//   most 1024 rows phase by phase: key tiles through a ring of tensor-memory
//   term slots, the unit's softmax and value-side B operand, then value
//   groups; bulk copies run ahead of use in shared-memory rings, and two
//   warps issue the MMAs side by side.
//
// Kernels: tc_prep (per (batch, KV head): RoPE, rotation and sketch of the G
// query heads, fixed-point B operand for the keys) and dec_kernel (the split-K
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
// tc_prep: one block (128 threads) per query head: its RoPE, rotation and
// sketch, and its four limb rows of the (batch, KV head) group's B operand.
// ---------------------------------------------------------------------------
template <int G, int MBK, bool QJL>
__global__ void __launch_bounds__(TCT) tc_prep_kernel(TcArgs a) {
  constexpr int TK = 1 << (MBK - 1);
  constexpr int N = tc_n(G);
  constexpr int KM = TK * TD;                 // MSE K bytes
  constexpr int KTOT = KM + (QJL ? TD : 0);
  __shared__ float q1s[TD], q2s[TD];
  __shared__ float red[TCT / 32][2];
  __shared__ double dred[TCT / 32][2];
  __shared__ float Fs[2];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int bh = blockIdx.x / G, h = blockIdx.x % G;   // one block per query head
  const int b = bh / a.Hkv, kvh = bh % a.Hkv;
  const int len = a.seq_lens ? min(max(a.seq_lens[b], 1), a.max_len) : a.max_len;
  const int64_t pos = len - 1;
  sm100::pdl_trigger();   // the main loop may launch and set itself up meanwhile
  if (blockIdx.x == 0 && tid == 0 && a.err) *a.err = 0u;   // this call's give-up flag
  // row tid of S (bf16) is loaded while warp 0 rotates the query
  uint4 srow[QJL ? TD / 8 : 1];
  if (QJL) {
    const uint4 *sp = reinterpret_cast<const uint4 *>(a.S + static_cast<int64_t>(tid) * TD);
#pragma unroll
    for (int q = 0; q < TD / 8; ++q) srow[q] = sp[q];
  }
  if (warp == 0) {
    const int64_t hq = static_cast<int64_t>(b) * a.Hq + kvh * G + h;
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
    for (int k = 0; k < TNW; ++k) q1s[lane + 32 * k] = x[k] * inv_sqrt_d;
  }
  __syncthreads();
  if (QJL) {
    // q''_i = sum_j S[i][j] q'_j for i = tid
    float acc = 0.f;
#pragma unroll
    for (int q = 0; q < TD / 8; ++q) {
      const uint32_t wds[4] = {srow[q].x, srow[q].y, srow[q].z, srow[q].w};
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float sv = __uint_as_float((e & 1) ? (wds[e >> 1] & 0xffff0000u) : (wds[e >> 1] << 16));
        acc = fmaf(sv, q1s[8 * q + e], acc);
      }
    }
    q2s[tid] = acc;
  }
  __syncthreads();
  // fixed-point scales: largest |B value| of each part
  {
    const float m1 = tq_warp_max(fabsf(q1s[tid]));
    const float m2 = QJL ? tq_warp_max(fabsf(q2s[tid])) : 0.f;
    if (lane == 0) {
      red[warp][0] = m1;
      red[warp][1] = m2;
    }
    __syncthreads();
    if (tid < 2) {
      float m = red[0][tid];
      for (int w = 1; w < TCT / 32; ++w) m = fmaxf(m, red[w][tid]);
      Fs[tid] = pow2_scale(2.f * (tid == 0 ? a.wk_absmax : 1.f) * m);
    }
    __syncthreads();
  }
  // B operand (K-major, no swizzle): MSE part then QJL part.  One item = K
  // chunk kc: its 16 fixed-point values of this head are computed once and
  // split into the four limb rows n = 4h + l, each stored as one 16-byte
  // write straight to the group's global B region.
  uint8_t *dst = a.bk + static_cast<int64_t>(bh) * a.bk_stride;
  constexpr int NKC = KTOT / 16, NKM = KM / 16;
  for (int kc = tid; kc < NKC; kc += TCT) {
    const bool mse = kc < NKM;
    const int kb = mse ? kc * 16 : (kc - NKM) * 16;
    uint32_t wv[4][4] = {{0u, 0u, 0u, 0u}, {0u, 0u, 0u, 0u}, {0u, 0u, 0u, 0u}, {0u, 0u, 0u, 0u}};
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const int kk = kb + e;
      const int col = kk >> 2, nb = kk & 3;
      const int ti = col >> 5, w = (col & 31) >> 3, r = col & 7;
      const int i = 32 * w + 8 * nb + r;
      const float val = mse ? 2.f * a.wk[ti] * q1s[i] * Fs[0] : 2.f * q2s[i] * Fs[1];
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
  // rows beyond the G heads' limbs (N > 4 G) are zero (written by head 0's block)
  if constexpr (N > 4 * G) {
    if (h == 0)
      for (int it = tid; it < (N - 4 * G) * NKC; it += TCT) {
        const int n = 4 * G + it % (N - 4 * G), kc = it / (N - 4 * G);
        const bool mse = kc < NKM;
        const int kb = mse ? kc * 16 : (kc - NKM) * 16;
        *reinterpret_cast<uint4 *>(dst + (mse ? 0 : N * KM) + kmajor_off(n, kb, N)) = make_uint4(0u, 0u, 0u, 0u);
      }
  }
  // constants: C = sum of the quantized B values / (2F) of each part
  {
    double s1 = 0.0;
#pragma unroll
    for (int ti = 0; ti < TK; ++ti) s1 += __float2int_rn(2.f * a.wk[ti] * q1s[tid] * Fs[0]);
    double s2 = QJL ? static_cast<double>(__float2int_rn(2.f * q2s[tid] * Fs[1])) : 0.0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      s1 += __shfl_xor_sync(TQ_FULL, s1, o);
      s2 += __shfl_xor_sync(TQ_FULL, s2, o);
    }
    if (lane == 0) {
      dred[warp][0] = s1;
      dred[warp][1] = s2;
    }
  }
  __syncthreads();
  if (tid == 0) {
    double s1 = 0.0, s2 = 0.0;
    for (int w = 0; w < TCT / 32; ++w) {
      s1 += dred[w][0];
      s2 += dred[w][1];
    }
    float *kc = reinterpret_cast<float *>(dst + N * KTOT);
    kc[h * 4 + 0] = static_cast<float>(s1 / (2.0 * Fs[0]));
    kc[h * 4 + 1] = 1.0f / (128.0f * Fs[0]);
    kc[h * 4 + 2] = static_cast<float>(s2 / (2.0 * Fs[1]));
    kc[h * 4 + 3] = 1.0f / (128.0f * Fs[1]);
  }
  // the main loop reads the cache rows the preceding append kernel writes:
  // this grid completes only after that one (which it may have overlapped)
  sm100::pdl_wait();
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

// ---------------------------------------------------------------------------
// dec_kernel: split-K decode main loop.  Two CTAs per SM, each walking its
// (batch, KV head, split) units (at most UMAX rows) phase by phase:
//   K  key tiles of 128 rows: bit planes -> Walsh-term operands in tensor
//      memory (two term slots per warp group) -> kind::i8 MMAs against the
//      fixed-point query (B, shared memory) -> logits of the G heads;
//   S  softmax statistics of the unit and the value-side B operand (24-bit
//      weights p * nu_v as four int8 limbs) for all of its 32-token groups;
//   V  value groups: bit planes -> Walsh-term operands (lane = coordinate) ->
//      MMAs accumulating the rotated-domain sums over the unit;
//   E  fold the value accumulators into the running output of the chunk.
// The two CTAs of an SM overlap each other's S and E phases with streaming.
// Warp roles: warp groups 0 (warps 0-3) and 1 (warps 4-7), one TMEM lane per
// thread, take alternate key tiles (expansion and epilogue) and alternate
// value groups, share S, and group 0 runs E.  Warp 8 + g issues the key MMAs
// of group g's tiles (a tcgen05.mma issue holds its thread for ~45 cycles at
// these N, so the two issue side by side) and the value MMAs of Walsh terms
// of parity g (each term's accumulator has one issuer).  Warp 10 issues every
// bulk copy ahead of use.  Every wait is bounded and warp-uniform; one that
// gives up makes the whole CTA drain its copies and MMAs and set the call's
// status word.
// ---------------------------------------------------------------------------
constexpr int DT = 352;        // 11 warps
constexpr int UMAX = 1024;     // rows per unit
constexpr int KS = 4;          // key tile stages (shared memory)
constexpr int VS = 8;          // value group stages (shared memory)
constexpr int DCOLS = 256;     // tensor memory per CTA

struct DecLayout {
  int ktb, vgb, bkc, o_kt, o_vt, o_bk, o_vn, o_lg, o_bv, total;
};

__host__ __device__ inline DecLayout dec_layout(int PK, int BV, int G, int N, int BKC) {
  DecLayout L;
  L.ktb = (128 * PK * 16 + 128 * 4 + 127) & ~127;
  L.vgb = BV * TD * 4;
  L.bkc = (BKC + 127) & ~127;
  L.o_kt = 0;
  L.o_vt = L.o_kt + KS * L.ktb;
  L.o_bk = L.o_vt + VS * L.vgb;
  L.o_vn = L.o_bk + 2 * L.bkc;
  L.o_lg = L.o_vn + 2 * UMAX * 2;
  L.o_bv = L.o_lg + UMAX * G * 4;
  L.total = L.o_bv + (UMAX / 32) * N * 32;
  return L;
}

// Warp-uniform bounded wait: every lane polls (so every lane acquires the
// phase), the loop ends for all lanes together.  Gives up when the budget
// runs out or another warp has given up.
__device__ __forceinline__ bool dwait(uint64_t *bar, uint32_t parity, uint32_t outer,
                                      volatile int *abort_flag) {
  for (uint32_t it = 0; it < outer; ++it) {
    const bool ok = sm100::mbar_wait(bar, parity, 1u << 8);
    if (__all_sync(TQ_FULL, ok)) return true;
    if (__shfl_sync(TQ_FULL, *abort_flag, 0)) return false;
  }
  *abort_flag = 1;
  return false;
}

// Single-thread bounded wait for the issuing and copying lanes.
__device__ __forceinline__ bool dwait1(uint64_t *bar, uint32_t parity, uint32_t outer,
                                       volatile int *abort_flag) {
  for (uint32_t it = 0; it < outer; ++it) {
    if (sm100::mbar_wait(bar, parity, 1u << 8)) return true;
    if (*abort_flag) return false;
  }
  *abort_flag = 1;
  return false;
}

template <int G, int MBK, int BV, bool QJL>
__global__ void __launch_bounds__(DT, 2) dec_kernel(TcArgs a) {
  constexpr int TK = 1 << (MBK - 1);
  constexpr int TV = 1 << (BV - 1);
  constexpr int N = tc_n(G);
  constexpr int PK = MBK + (QJL ? 1 : 0);
  constexpr int KM = TK * TD;
  constexpr int KTOT = KM + (QJL ? TD : 0);
  constexpr int BKB = N * KTOT;
  constexpr int BKC = BKB + G * 16;
  constexpr int NKT = TK + (QJL ? 1 : 0);
  constexpr int NACC = QJL ? 2 : 1;      // key accumulators per tile: MSE terms, sign plane
  // tensor memory (256 columns): key phase: group g's term slots [64 g, 64 g + 64),
  // D_k[g] [128 + 2 N g, ...); value phase: A_v[g] [8 TV g, ...), D_v [128, 128 + N TV)
  constexpr int C_DK = 128, C_DV = 128;
  static_assert(C_DK + 2 * NACC * N <= DCOLS && C_DV + TV * N <= DCOLS && 2 * TV * 8 <= 128,
                "tensor memory budget");
  constexpr uint32_t IDESC = sm100::idesc_i8(128, N);
  const DecLayout L = dec_layout(PK, BV, G, N, BKC);

  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ __align__(8) uint64_t kf[KS], ke[KS], vf[VS], ve[VS], hdr[2], hdr_free[2];
  __shared__ __align__(8) uint64_t as_full[4], as_empty[4], dk_full[2], dk_empty[2];
  __shared__ __align__(8) uint64_t av_full[2], av_empty[2], bv_full, dv_full, tm_free, sbar, done[2];
  __shared__ uint32_t tmem_s;
  __shared__ volatile int abort_s;
  __shared__ float redf[8][2 * G + 1];
  __shared__ unsigned long long wsum_s[8];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int lt = tid & 127;
  const uint32_t outer = a.wait_limit >> 8;

  if (warp == 0) sm100::tmem_alloc(&tmem_s, DCOLS);
  if (tid == 0) {
    for (int i = 0; i < KS; ++i) { sm100::mbar_init(&kf[i], 1); sm100::mbar_init(&ke[i], 4); }
    for (int i = 0; i < VS; ++i) { sm100::mbar_init(&vf[i], 1); sm100::mbar_init(&ve[i], 4); }
    for (int i = 0; i < 4; ++i) { sm100::mbar_init(&as_full[i], 4); sm100::mbar_init(&as_empty[i], 1); }
    for (int i = 0; i < 2; ++i) {
      sm100::mbar_init(&hdr[i], 1);
      sm100::mbar_init(&hdr_free[i], 8);
      sm100::mbar_init(&dk_full[i], 1);
      sm100::mbar_init(&dk_empty[i], 4);
      sm100::mbar_init(&av_full[i], 4);
      sm100::mbar_init(&av_empty[i], 2);
      sm100::mbar_init(&done[i], 1);
    }
    sm100::mbar_init(&bv_full, 8);
    sm100::mbar_init(&dv_full, 2);
    sm100::mbar_init(&tm_free, 4);
    sm100::mbar_init(&sbar, 8);
    abort_s = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  sm100::fence_before_sync();
  __syncthreads();
  sm100::fence_after_sync();
  const uint32_t tm = tmem_s;
  // the query prologue (and, through it, the append) has completed
  sm100::pdl_wait();
  sm100::pdl_trigger();

  // empty chunks (beyond a batch's length) merge with weight zero
  if (warp < 8) {
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
  }

  if (warp == 10) {
    // ------------------------------------------------------------ copies
    if (lane == 0) {
      int cit = blockIdx.x, cr0 = -1, u = 0;
      uint32_t kt = 0, vg = 0;
      // per stage: 1 + the parity of its last issued copy (0 = never issued)
      uint8_t lk[KS] = {}, lv[VS] = {}, lh[2] = {};
      bool have = tc_next(a, cit, cr0);
      while (have && !abort_s) {
        const int b = cit / (a.Hkv * a.splits), kvh = (cit / a.splits) % a.Hkv, sp = cit % a.splits;
        const int64_t bh = static_cast<int64_t>(b) * a.Hkv + kvh;
        const int c0 = sp * a.chunk, c1 = min(tc_len(a, b), c0 + a.chunk);
        const int nvalid = min(a.sub, c1 - cr0);
        const int ntile = (nvalid + 127) / 128, ngroups = (nvalid + 31) / 32;
        // unit header: this unit's B operand and value norms (buffer u & 1),
        // once unit u - 2 has finished its softmax phase with that buffer
        {
          const int hb = u & 1;
          if (u >= 2 && !dwait1(&hdr_free[hb], ((u >> 1) - 1) & 1, outer, &abort_s)) break;
          const uint32_t nvn = static_cast<uint32_t>(ngroups) * 64;
          sm100::mbar_expect_tx(&hdr[hb], static_cast<uint32_t>((BKC + 15) & ~15) + nvn);
          sm100::bulk_g2s(smem + L.o_bk + hb * L.bkc, a.bk + bh * a.bk_stride, (BKC + 15) & ~15, &hdr[hb]);
          sm100::bulk_g2s(smem + L.o_vn + hb * UMAX * 2, a.vnorm + bh * a.rows_cap + cr0, nvn, &hdr[hb]);
          lh[hb] = static_cast<uint8_t>(1 + ((u >> 1) & 1));
        }
        for (int j = 0; j < ntile && !abort_s; ++j, ++kt) {
          const int s = kt % KS;
          if (kt >= KS && !dwait1(&ke[s], ((kt / KS) - 1) & 1, outer, &abort_s)) break;
          const int64_t row = cr0 + j * 128;
          const uint32_t nrow = static_cast<uint32_t>(min(static_cast<int64_t>(128), a.rows_cap - row));
          uint8_t *st = smem + L.o_kt + s * L.ktb;
          sm100::mbar_expect_tx(&kf[s], nrow * PK * 16 + nrow * 4);
          sm100::bulk_g2s(st, a.kcode + (bh * a.rows_cap + row) * PK * 16, nrow * PK * 16, &kf[s]);
          sm100::bulk_g2s(st + 128 * PK * 16, a.kscale + (bh * a.rows_cap + row) * 2, nrow * 4, &kf[s]);
          lk[s] = static_cast<uint8_t>(1 + ((kt / KS) & 1));
        }
        for (int g = 0; g < ngroups && !abort_s; ++g, ++vg) {
          const int s = vg % VS;
          if (vg >= VS && !dwait1(&ve[s], ((vg / VS) - 1) & 1, outer, &abort_s)) break;
          sm100::mbar_expect_tx(&vf[s], L.vgb);
          sm100::bulk_g2s(smem + L.o_vt + s * L.vgb,
                          a.vcode + (bh * (a.rows_cap / 32) + cr0 / 32 + g) * BV * TD, L.vgb, &vf[s]);
          lv[s] = static_cast<uint8_t>(1 + ((vg / VS) & 1));
        }
        cr0 += a.sub;
        have = tc_next(a, cit, cr0);
        ++u;
      }
      if (abort_s) {
        // this CTA's own copies land before its shared memory is released:
        // each stage's last issued phase completes (at once if consumed)
        for (int i = 0; i < KS; ++i)
          if (lk[i]) sm100::mbar_wait(&kf[i], lk[i] - 1u, 1u << 20);
        for (int i = 0; i < VS; ++i)
          if (lv[i]) sm100::mbar_wait(&vf[i], lv[i] - 1u, 1u << 20);
        for (int i = 0; i < 2; ++i)
          if (lh[i]) sm100::mbar_wait(&hdr[i], lh[i] - 1u, 1u << 20);
      }
    }
    __syncwarp();
  } else if (warp >= 8) {
    // ------------------------------------------------------------ MMA issue
    const int is = warp - 8;           // serves warp group `is`
    if (lane == 0) {
      int cit = blockIdx.x, cr0 = -1, u = 0;
      uint32_t tw = 0, ktw = 0, vu[2] = {0u, 0u};   // terms / tiles of group is; uses of A_v[b]
      bool have = tc_next(a, cit, cr0);
      bool ok = true;
      while (have && ok) {
        const int b = cit / (a.Hkv * a.splits), sp = cit % a.splits;
        const int c0 = sp * a.chunk, c1 = min(tc_len(a, b), c0 + a.chunk);
        const int nvalid = min(a.sub, c1 - cr0);
        const int ntile = (nvalid + 127) / 128, ngroups = (nvalid + 31) / 32;
        const uint32_t bk_addr = sm100::smem_addr(smem + L.o_bk + (u & 1) * L.bkc);
        // the previous unit's value epilogue has read D_v (it overlaps D_k)
        if (u > 0) ok = dwait1(&tm_free, (u - 1) & 1, outer, &abort_s);
        if (ok) ok = dwait1(&hdr[u & 1], (u >> 1) & 1, outer, &abort_s);
        const uint32_t dk = tm + C_DK + is * NACC * N;
        for (int j = is; j < ntile && ok; j += 2, ++ktw) {
          if (ktw >= 1 && !(ok = dwait1(&dk_empty[is], (ktw - 1) & 1, outer, &abort_s))) break;
#pragma unroll
          for (int t = 0; t < NKT; ++t, ++tw) {
            const int slot = 2 * is + (tw & 1);
            if (!(ok = dwait1(&as_full[slot], (tw >> 1) & 1, outer, &abort_s))) break;
            sm100::fence_after_sync();
            const bool sign = QJL && t == TK;
            const uint32_t acc = sign ? dk + N : dk;
            const uint32_t boff = sign ? N * KM : static_cast<uint32_t>(t) * 4 * 2 * N * 16;
#pragma unroll
            for (int s4 = 0; s4 < 4; ++s4)
              sm100::mma_i8_ts(acc, tm + slot * 32 + s4 * 8,
                               sm100::smem_desc(bk_addr + boff + s4 * 2 * N * 16, N * 16, 128), IDESC,
                               ((t == 0 || sign) && s4 == 0) ? 0u : 1u);
            sm100::mma_commit(&as_empty[slot]);
          }
          if (!ok) break;
          sm100::mma_commit(&dk_full[is]);
        }
        if (!ok) break;
        // value groups: the unit's B operand is complete
        ok = dwait1(&bv_full, u & 1, outer, &abort_s);
        const uint32_t bv_addr = sm100::smem_addr(smem + L.o_bv);
        for (int g = 0; g < ngroups && ok; ++g) {
          const int ab = g & 1;
          if (!(ok = dwait1(&av_full[ab], vu[ab] & 1, outer, &abort_s))) break;
          ++vu[ab];
          sm100::fence_after_sync();
          const uint64_t bd = sm100::smem_desc(bv_addr + g * N * 32, N * 16, 128);
          bool any = false;
#pragma unroll
          for (int ti = 0; ti < TV; ++ti) {
            if ((ti & 1) != is) continue;
            sm100::mma_i8_ts(tm + C_DV + ti * N, tm + ab * TV * 8 + ti * 8, bd, IDESC, g > 0);
            any = true;
          }
          if (any) sm100::mma_commit(&av_empty[ab]);
          else sm100::mbar_arrive(&av_empty[ab]);
        }
        if (!ok) break;
        sm100::mma_commit(&dv_full);
        cr0 += a.sub;
        have = tc_next(a, cit, cr0);
        ++u;
      }
      // every MMA of this thread has landed before tensor memory is freed
      sm100::mma_commit(&done[is]);
      sm100::mbar_wait(&done[is], 0, 1u << 20);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ warp groups 0 and 1
    const int wg = warp >> 2;
    const int wq = warp & 3;
    float *lg = reinterpret_cast<float *>(smem + L.o_lg);
    int8_t *bvs = reinterpret_cast<int8_t *>(smem + L.o_bv);
    int cit = blockIdx.x, cr0 = -1, u = 0;
    uint32_t kt = 0, tw = 0, ktw = 0, vg = 0, vu = 0, sp_par = 0;
    float o[G], m_run[G], l_run[G];
#pragma unroll
    for (int h = 0; h < G; ++h) { o[h] = 0.f; m_run[h] = -CUDART_INF_F; l_run[h] = 0.f; }
    bool have = tc_next(a, cit, cr0);
    // all 8 row warps meet (bounded)
    auto sync8 = [&]() -> bool {
      sm100::fence_before_sync();
      __syncwarp();
      if (lane == 0) sm100::mbar_arrive(&sbar);
      const bool r = dwait(&sbar, sp_par, outer, &abort_s);
      sp_par ^= 1u;
      sm100::fence_after_sync();
      return r;
    };
    while (have) {
      const int b = cit / (a.Hkv * a.splits), kvh = (cit / a.splits) % a.Hkv, sp = cit % a.splits;
      const int len = tc_len(a, b);
      const int c0 = sp * a.chunk, c1 = min(len, c0 + a.chunk);
      const int nvalid = min(a.sub, c1 - cr0);
      const int ntile = (nvalid + 127) / 128, ngroups = (nvalid + 31) / 32;
      const float *kcst = reinterpret_cast<const float *>(smem + L.o_bk + (u & 1) * L.bkc + BKB);
      if (cr0 == c0) {
#pragma unroll
        for (int h = 0; h < G; ++h) { o[h] = 0.f; m_run[h] = -CUDART_INF_F; l_run[h] = 0.f; }
      }
      float mloc[G];
#pragma unroll
      for (int h = 0; h < G; ++h) mloc[h] = -CUDART_INF_F;
      bool ok = dwait(&hdr[u & 1], (u >> 1) & 1, outer, &abort_s);   // kcst of this unit
      // ---------------- K phase: this group's tiles (expansion, then epilogue)
      for (int j = wg; j < ntile && ok; j += 2, ++ktw) {
        const uint32_t ktj = kt + j;
        const int s = ktj % KS;
        if (!(ok = dwait(&kf[s], (ktj / KS) & 1, outer, &abort_s))) break;
        const uint8_t *stg = smem + L.o_kt + s * L.ktb;
        const uint4 *kr = reinterpret_cast<const uint4 *>(stg + lt * PK * 16);
        uint32_t pw[PK][TNW];
#pragma unroll
        for (int p = 0; p < PK; ++p) {
          const uint4 v = kr[p];
          pw[p][0] = v.x; pw[p][1] = v.y; pw[p][2] = v.z; pw[p][3] = v.w;
        }
        const uint32_t sc = reinterpret_cast<const uint32_t *>(stg + 128 * PK * 16)[lt];
        __syncwarp();
        if (lane == 0) sm100::mbar_arrive(&ke[s]);
#pragma unroll
        for (int t = 0; t < NKT; ++t, ++tw) {
          const int slot = 2 * wg + (tw & 1);
          if (tw >= 2 && !(ok = dwait(&as_empty[slot], ((tw >> 1) - 1) & 1, outer, &abort_s))) break;
          sm100::fence_after_sync();
          uint32_t r32[32];
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
#pragma unroll
            for (int r = 0; r < 8; ++r) r32[w * 8 + r] = x & (0x01010101u << r);
          }
          sm100::tmem_st32(sm100::tmem_lane(tm + slot * 32, wq), r32);
          sm100::wait_st();
          sm100::fence_before_sync();
          __syncwarp();
          if (lane == 0) sm100::mbar_arrive(&as_full[slot]);
        }
        if (!ok) break;
        // epilogue of this tile
        if (!(ok = dwait(&dk_full[wg], ktw & 1, outer, &abort_s))) break;
        sm100::fence_after_sync();
        const uint32_t dka = tm + C_DK + wg * NACC * N;
        uint32_t dm[N], dq[N];
        if (N == 16) {
          uint32_t t16[16];
          sm100::tmem_ld16(sm100::tmem_lane(dka, wq), t16);
          if (QJL) {
            uint32_t q16[16];
            sm100::tmem_ld16(sm100::tmem_lane(dka + N, wq), q16);
            sm100::wait_ld();
#pragma unroll
            for (int c = 0; c < 16; ++c) dq[c % N] = q16[c];
          } else {
            sm100::wait_ld();
          }
#pragma unroll
          for (int c = 0; c < 16; ++c) dm[c % N] = t16[c];
        } else {
          uint32_t t8[8];
          sm100::tmem_ld8(sm100::tmem_lane(dka, wq), t8);
          if (QJL) {
            uint32_t q8[8];
            sm100::tmem_ld8(sm100::tmem_lane(dka + N, wq), q8);
            sm100::wait_ld();
#pragma unroll
            for (int c = 0; c < 8; ++c) dq[c % N] = q8[c];
          } else {
            sm100::wait_ld();
          }
#pragma unroll
          for (int c = 0; c < 8; ++c) dm[c % N] = t8[c];
        }
        sm100::fence_before_sync();
        __syncwarp();
        if (lane == 0) sm100::mbar_arrive(&dk_empty[wg]);
        const int rl = j * 128 + lt;
        const bool valid = rl < nvalid;
        const float nu = tq_half_to_f32(static_cast<uint16_t>(sc & 0xffffu));
        const float rho = tq_half_to_f32(static_cast<uint16_t>(sc >> 16));
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float dmv = comb_limbs(dm + 4 * h) * kcst[4 * h + 1] - kcst[4 * h + 0];
          float est = dmv;
          if (QJL) {
            const float dj = comb_limbs(dq + 4 * h) * kcst[4 * h + 3] - kcst[4 * h + 2];
            est = fmaf(a.qjl_coef * rho, dj, dmv);
          }
          const float l = valid ? a.scale * nu * est : -CUDART_INF_F;
          lg[rl * G + h] = l;
          mloc[h] = fmaxf(mloc[h], l);
          if (a.logits && valid)
            a.logits[(static_cast<int64_t>(b) * a.Hq + kvh * G + h) * a.max_len + cr0 + rl] = l;
        }
      }
      kt += ntile;
      // ---------------- S phase (8 warps)
      if (ok) {
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float m = tq_warp_max(mloc[h]);
          if (lane == 0) redf[warp][h] = m;
        }
        ok = sync8();
      }
      float mnew[G], corr[G], lsum[G], FV = 1.f, invFV = 1.f;
      if (ok) {
#pragma unroll
        for (int h = 0; h < G; ++h) {
          float m = redf[0][h];
#pragma unroll
          for (int w = 1; w < 8; ++w) m = fmaxf(m, redf[w][h]);
          mnew[h] = fmaxf(m_run[h], m);
          corr[h] = __expf(m_run[h] - mnew[h]);
          lsum[h] = 0.f;
        }
        const uint16_t *vn = reinterpret_cast<const uint16_t *>(smem + L.o_vn + (u & 1) * UMAX * 2);
        float numax = 0.f;
        for (int rl = tid; rl < nvalid; rl += 256) {
          numax = fmaxf(numax, tq_half_to_f32(vn[rl]));
#pragma unroll
          for (int h = 0; h < G; ++h) {
            const float p = __expf(lg[rl * G + h] - mnew[h]);
            lg[rl * G + h] = p;
            lsum[h] += p;
          }
        }
        ok = sync8();   // redf is free again; the weights are in place
        if (ok) {
#pragma unroll
          for (int h = 0; h < G; ++h) {
            const float sm = tq_warp_sum(lsum[h]);
            if (lane == 0) redf[warp][h] = sm;
          }
          const float nm = tq_warp_max(numax);
          if (lane == 0) redf[warp][2 * G] = nm;
          if (tid < 8) wsum_s[tid] = 0ull;
          ok = sync8();
        }
        if (ok) {
#pragma unroll
          for (int h = 0; h < G; ++h) {
            float sm = 0.f;
#pragma unroll
            for (int w = 0; w < 8; ++w) sm += redf[w][h];
            lsum[h] = sm;
          }
          float nmax = redf[0][2 * G];
#pragma unroll
          for (int w = 1; w < 8; ++w) nmax = fmaxf(nmax, redf[w][2 * G]);
          FV = pow2_scale(nmax);
          invFV = 1.0f / (128.0f * FV);
          // value-side B operand: element (n = 4h + l, k) of group g holds limb
          // l of W(token) * 2^(7-r) for token 32g + 8nb + r, k = 4r + nb; one
          // item = (group, r, head) makes the four consecutive k of one limb
          // row and stores them as one 32-bit word; rows n >= 4G are zero
          constexpr int NH = N / 4;
          long long wpart = 0;
          const int h = tid % NH;
          for (int it = tid; it < ngroups * 8 * NH; it += 256) {
            const int r = (it / NH) & 7, g = it / (8 * NH);
            uint32_t word[4] = {0u, 0u, 0u, 0u};
            if (h < G) {
#pragma unroll
              for (int nb = 0; nb < 4; ++nb) {
                const int rl = 32 * g + 8 * nb + r;
                int W = 0;
                if (rl < nvalid) W = __float2int_rn(lg[rl * G + h] * tq_half_to_f32(vn[rl]) * FV);
                wpart += W;
                int v = W * (1 << (7 - r));
#pragma unroll
                for (int l = 0; l < 4; ++l) {
                  const int8_t dgt = static_cast<int8_t>(v & 0xff);
                  word[l] |= static_cast<uint32_t>(static_cast<uint8_t>(dgt)) << (8 * nb);
                  v = (v - dgt) >> 8;
                }
              }
            }
            int8_t *dst = bvs + g * N * 32;
#pragma unroll
            for (int l = 0; l < 4; ++l)
              *reinterpret_cast<uint32_t *>(dst + kmajor_off(4 * h + l, 4 * r, N)) = word[l];
          }
          if (h < G) atomicAdd(&wsum_s[h], static_cast<unsigned long long>(wpart));
          sm100::fence_async_smem();
          ok = sync8();
          if (ok && lane == 0) {
            sm100::mbar_arrive(&bv_full);
            sm100::mbar_arrive(&hdr_free[u & 1]);   // B operand and value norms no longer read
          }
        }
      }
      if (!ok) break;
      float wtot[G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        wtot[h] = static_cast<float>(static_cast<long long>(wsum_s[h])) / FV;
        o[h] *= corr[h];
        l_run[h] = l_run[h] * corr[h] + lsum[h];
        m_run[h] = mnew[h];
      }
      // ---------------- V phase: this group's value groups (lane = coordinate)
      for (int g = wg; g < ngroups && ok; g += 2, ++vu) {
        const uint32_t vgg = vg + g;
        const int s = vgg % VS;
        if (!(ok = dwait(&vf[s], (vgg / VS) & 1, outer, &abort_s))) break;
        const uint32_t *vc = reinterpret_cast<const uint32_t *>(smem + L.o_vt + s * L.vgb);
        uint32_t pw[BV];
#pragma unroll
        for (int p = 0; p < BV; ++p) pw[p] = vc[p * TD + lt];
        __syncwarp();
        if (lane == 0) sm100::mbar_arrive(&ve[s]);
        if (vu >= 1 && !(ok = dwait(&av_empty[wg], (vu - 1) & 1, outer, &abort_s))) break;
        sm100::fence_after_sync();
#pragma unroll
        for (int h4 = 0; h4 < (TV + 3) / 4; ++h4) {
          uint32_t r32[32];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int ti = 4 * h4 + q;
            uint32_t x = 0;
            if (ti < TV) {
              const int mask = odd_mask(BV, ti);
#pragma unroll
              for (int p = 0; p < BV; ++p)
                if ((mask >> p) & 1) x ^= pw[p];
            }
#pragma unroll
            for (int r = 0; r < 8; ++r) r32[q * 8 + r] = x & (0x01010101u << r);
          }
          if (TV >= 4) {
            sm100::tmem_st32(sm100::tmem_lane(tm + wg * TV * 8 + h4 * 32, wq), r32);
          } else {
            uint32_t r8[8];
#pragma unroll
            for (int q = 0; q < TV; ++q) {
#pragma unroll
              for (int r = 0; r < 8; ++r) r8[r] = r32[q * 8 + r];
              sm100::tmem_st8(sm100::tmem_lane(tm + wg * TV * 8 + q * 8, wq), r8);
            }
          }
        }
        sm100::wait_st();
        sm100::fence_before_sync();
        __syncwarp();
        if (lane == 0) sm100::mbar_arrive(&av_full[wg]);
      }
      vg += ngroups;
      // ---------------- E phase: all value MMAs of the unit have landed
      if (ok) ok = dwait(&dv_full, u & 1, outer, &abort_s);
      if (ok && wg == 0) {
        sm100::fence_after_sync();
        float acc[G];
#pragma unroll
        for (int h = 0; h < G; ++h) acc[h] = 0.f;
#pragma unroll
        for (int ti = 0; ti < TV; ++ti) {
          uint32_t dv[N];
          if (N == 16) {
            uint32_t t0[16];
            sm100::tmem_ld16(sm100::tmem_lane(tm + C_DV + ti * N, wq), t0);
            sm100::wait_ld();
#pragma unroll
            for (int c = 0; c < 16; ++c) dv[c % N] = t0[c];
          } else {
            uint32_t t0[8];
            sm100::tmem_ld8(sm100::tmem_lane(tm + C_DV + ti * N, wq), t0);
            sm100::wait_ld();
#pragma unroll
            for (int c = 0; c < 8; ++c) dv[c % N] = t0[c];
          }
#pragma unroll
          for (int h = 0; h < G; ++h) acc[h] = fmaf(2.f * a.wv[ti], comb_limbs(dv + 4 * h), acc[h]);
        }
        sm100::fence_before_sync();
        __syncwarp();
        if (lane == 0) sm100::mbar_arrive(&tm_free);
#pragma unroll
        for (int h = 0; h < G; ++h) o[h] += acc[h] * invFV - a.wv_sum * wtot[h];
        if (cr0 + a.sub >= c1) {
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
      }
      if (!ok) break;
      cr0 += a.sub;
      have = tc_next(a, cit, cr0);
      ++u;
    }
  }
  sm100::fence_before_sync();
  __syncthreads();
  sm100::fence_after_sync();
  if (abort_s && tid == 0 && a.err) atomicExch(a.err, 1u);
  if (warp == 0) sm100::tmem_dealloc(tm, DCOLS);
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
struct TcCfg {
  int G, mbk, bv, qjl;
};

constexpr TcCfg kTcConfigs[] = {{4, 3, 4, 1}, {4, 1, 2, 1}, {4, 2, 3, 1}, {2, 3, 4, 1},
                                {2, 1, 2, 1}, {2, 2, 3, 1}, {1, 3, 4, 1}, {1, 1, 2, 1},
                                {1, 2, 3, 1}, {4, 4, 4, 0}, {4, 2, 2, 0}, {4, 3, 3, 0},
                                {1, 3, 3, 0}};

template <int G, int MBK, int BV, bool QJL>
int run_dec(TcArgs &a, cudaStream_t stream) {
  constexpr int TK = 1 << (MBK - 1);
  constexpr int N = tc_n(G);
  constexpr int PK = MBK + (QJL ? 1 : 0);
  constexpr int BKC = N * (TK * TD + (QJL ? TD : 0)) + G * 16;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  a.sub = a.chunk < UMAX ? a.chunk : UMAX;
  const int smem = dec_layout(PK, BV, G, N, BKC).total;
  static bool attr_done[64] = {};
  if (dev < 64 && !attr_done[dev]) {
    if (cudaFuncSetAttribute(dec_kernel<G, MBK, BV, QJL>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem) != cudaSuccess)
      return tq_check_launch("cudaFuncSetAttribute(dec_kernel)");
    attr_done[dev] = true;
  }
  if (tq_launch_pdl(tc_prep_kernel<G, MBK, QJL>, dim3(a.B * a.Hkv * G), dim3(TCT), 0, stream, a) !=
      cudaSuccess)
    return tq_check_launch("tc_prep_kernel");
  const int items = a.B * a.Hkv * a.splits;
  const int grid = items < 2 * sms ? items : 2 * sms;
  cudaEvent_t ev0, ev1;
  tq_timing_events(&ev0, &ev1);
  unsigned ev_flags = cudaEventRecordDefault;
  if (ev0) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    cudaStreamIsCapturing(stream, &cs);
    if (cs == cudaStreamCaptureStatusActive) ev_flags = cudaEventRecordExternal;
    cudaEventRecordWithFlags(ev0, stream, ev_flags);
  }
  if (tq_launch_pdl(dec_kernel<G, MBK, BV, QJL>, dim3(grid), dim3(DT), smem, stream, a) != cudaSuccess)
    return tq_check_launch("dec_kernel");
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
                     uint8_t *bk, float *logits, uint32_t *err, cudaStream_t stream) {
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
  a.err = err;
  a.wait_limit = 1u << 26;
  if (const char *e = getenv("TQ_WAIT_LIMIT")) a.wait_limit = static_cast<uint32_t>(strtoul(e, nullptr, 10));
  a.books = c->books;
  const int key = G * 1000 + c->mse_bits_k * 100 + c->bits_v * 10 + c->qjl_k;
  switch (key) {
    case 4341: return run_dec<4, 3, 4, true>(a, stream);
    case 4121: return run_dec<4, 1, 2, true>(a, stream);
    case 4231: return run_dec<4, 2, 3, true>(a, stream);
    case 2341: return run_dec<2, 3, 4, true>(a, stream);
    case 2121: return run_dec<2, 1, 2, true>(a, stream);
    case 2231: return run_dec<2, 2, 3, true>(a, stream);
    case 1341: return run_dec<1, 3, 4, true>(a, stream);
    case 1121: return run_dec<1, 1, 2, true>(a, stream);
    case 1231: return run_dec<1, 2, 3, true>(a, stream);
    case 4440: return run_dec<4, 4, 4, false>(a, stream);
    case 4220: return run_dec<4, 2, 2, false>(a, stream);
    case 4330: return run_dec<4, 3, 3, false>(a, stream);
    case 1330: return run_dec<1, 3, 3, false>(a, stream);
    default: return tq_fail(TQ_ERR_UNSUPPORTED, "tensor-core decode: configuration not built");
  }
}
