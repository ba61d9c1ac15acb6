// Tensor-core split-K decode from the compressed cache (sm_100a, tcgen05).
//
// Same computation as decode.cu ("TurboESM ..." section 2.E: one pass over the
// compressed cache; "Google presenta TurboQuant ...", "Eliminacion del sesgo":
// the prod estimator), restructured so every per-coordinate product runs on
// the 5th-generation tensor cores as integer MMAs (kind::i8, int32
// accumulators, A unsigned from tensor memory, B signed from shared memory):
//
// * Operands.  Each 32-element slice of a code (32 coordinates of a key row,
//   or 32 tokens of a value coordinate) becomes 32 A bytes per operand:
//   - 1- and 2-bit codebooks: one operand per code bit.  A symmetric
//     codebook is an odd function of its bits, so with one or two bits
//     c[idx] = sum_p a_p (2 bit_p - 1) exactly (the odd Walsh terms; a_p
//     solved on the host).  Byte j of A word r holds bit 8j + r as 2^r
//     (w & (0x01010101 << r)); the 2^r is undone on the B side (x 2^(7-r)).
//   - 3- and 4-bit codebooks: three operands, the 7-bit digits of the
//     centroid in 21-bit fixed point, V = 2^20 + round(c F) = 2^14 d0 +
//     2^7 d1 + d2.  A byte permute (prmt) looks up four codes at once from
//     the nibble-packed code bits; 16-entry books take both 8-entry halves
//     and keep one per byte.
//   The QJL sign plane is a one-bit operand of its own.
// * B holds the other factor in 24-bit fixed point as four signed 8-bit limbs
//   (N = 4 limbs x G query heads), so every accumulator is exact; the host
//   constants undo the fixed-point scales and offsets.
// * Keys: M = 128 key rows (TMEM lane = row), K = d, one accumulator per
//   operand.  Values: M = 128 coordinates (lane = coordinate; the cache's
//   32-token column groups give each lane its own words), K = 32 tokens.
//
// Kernels: tc_prep (one block per query head: RoPE, rotation and sketch, the
// head's rows of the key-side B operand) and dec_kernel (the split-K main
// loop); the chunk partials are merged by decode.cu's combine kernel.
#include <math_constants.h>

#include <cstdlib>

#include "tq_device.cuh"
#include "tq_sm100.cuh"
#include "tq_tc.h"

namespace {

constexpr int TD = 128;   // head dim of this path
constexpr int TNW = TD / 32;
constexpr int TCT = 128;  // threads of tc_prep

// 3- and 4-bit codebooks use centroid digits, 1- and 2-bit ones bit planes.
__host__ __device__ constexpr bool use_digits(int bits) { return bits >= 3; }
// A operands per 32-element slice.
__host__ __device__ constexpr int n_ops(int bits) { return use_digits(bits) ? 3 : bits; }
constexpr int NDIG = 3;             // centroid digits
constexpr float DIG_W0 = 16384.f;   // their weights: 2^14, 2^7, 1
constexpr float DIG_W1 = 128.f;
constexpr double DIG_OFF = 1048576.0;   // V = 2^20 + round(c F)

// Element of a 32-element slice at byte k (0..31) of an operand chunk.  Bit
// planes: byte j of word r holds element 8j + r.  Digits: byte b of word
// 2j + h holds element 16h + 4b + j.
__host__ __device__ constexpr int elem_of(bool digits, int k) {
  return digits ? 16 * ((k >> 2) & 1) + 4 * (k & 3) + (k >> 3) : 8 * (k & 3) + (k >> 2);
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

// prmt.b32: byte i of the result is byte s[4i+2:4i] of {b, a}; bit 4i+3 set
// replicates that byte's top bit instead.
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t s) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(s));
  return d;
}

// The 8 A words of a bit plane: word r = bit 8j + r of x in byte j, as 2^r.
__device__ __forceinline__ void plane_words(uint32_t x, uint32_t *o) {
#pragma unroll
  for (int r = 0; r < 8; ++r) o[r] = x & (0x01010101u << r);
}

// Code of element 4i + j (bit p from plane word pl[p]) in nibble i.
template <int NB>
__device__ __forceinline__ uint32_t gather_nibbles(const uint32_t *pl, int j) {
  uint32_t n = 0;
#pragma unroll
  for (int p = 0; p < NB; ++p) {
    const uint32_t x = p >= j ? pl[p] << (p - j) : pl[p] >> (j - p);
    n |= x & (0x11111111u << p);
  }
  return n;
}

// Digit words of a 32-element slice: o[k][2j + h], byte b = digit k of the
// centroid of element 16h + 4b + j (tab[k]: entries 0..15, four per word;
// every digit is below 128).
template <int NB>
__device__ __forceinline__ void digit_words(const uint32_t *pl, const uint32_t (&tab)[NDIG][4],
                                            uint32_t (&o)[NDIG][8]) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t nib = gather_nibbles<NB>(pl, j);
    if constexpr (NB <= 3) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint32_t sel = h ? nib >> 16 : nib;
#pragma unroll
        for (int k = 0; k < NDIG; ++k) o[k][2 * j + h] = prmt(tab[k][0], tab[k][1], sel);
      }
    } else {
      // 16 entries: look both halves up with the low three code bits and
      // keep, byte by byte, the half that bit 3 picks.  The mask comes from
      // prmt's sign mode: 0xff where bit 3 is set, else 0x80, whose top bit
      // is harmless since no digit has it.
      const uint32_t s7 = nib & 0x77777777u;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint32_t sel = h ? s7 >> 16 : s7;
        const uint32_t m = prmt(0x80808080u, 0x80808080u, h ? nib >> 16 : nib);
#pragma unroll
        for (int k = 0; k < NDIG; ++k) {
          const uint32_t lo = prmt(tab[k][0], tab[k][1], sel);
          const uint32_t hi = prmt(tab[k][2], tab[k][3], sel);
          o[k][2 * j + h] = (hi & m) | (lo & ~m);
        }
      }
    }
  }
}

// ---------------------------------------------------------------------------
// tc_prep: one block (128 threads) per query head: its RoPE, rotation and
// sketch, and its four limb rows of the (batch, KV head) group's B operand.
// ---------------------------------------------------------------------------
template <int G, int MBK, bool QJL>
__global__ void __launch_bounds__(TCT) tc_prep_kernel(TcArgs a) {
  constexpr bool DIG = use_digits(MBK);
  constexpr int NT = n_ops(MBK);
  constexpr int N = tc_n(G);
  constexpr int KM = NT * TD;                 // MSE K bytes
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
    if (a.books.pi != nullptr) {
#pragma unroll
      for (int k = 0; k < TNW; ++k) q2s[lane + 32 * k] = x[k];   // RoPE'd q for the product below
    } else {
      tq_apply_signs<TNW>(x, a.books.dneg, lane);
      tq_warp_wht<TNW>(x, lane);
      const float scl = 1.0f / sqrtf(static_cast<float>(TD));
#pragma unroll
      for (int k = 0; k < TNW; ++k) q1s[lane + 32 * k] = x[k] * scl;
    }
  }
  __syncthreads();
  if (a.books.pi != nullptr) {
    // dense rotation q' = Pi q: thread i takes row i of Pi (16-byte loads, all
    // in flight at once), sums in order j = 0 .. d-1
    const float4 *row = reinterpret_cast<const float4 *>(a.books.pi + tid * TD);
    float acc = 0.f;
#pragma unroll 8
    for (int c = 0; c < TD / 4; ++c) {
      const float4 p = row[c];
      acc = fmaf(p.x, q2s[4 * c], acc);
      acc = fmaf(p.y, q2s[4 * c + 1], acc);
      acc = fmaf(p.z, q2s[4 * c + 2], acc);
      acc = fmaf(p.w, q2s[4 * c + 3], acc);
    }
    q1s[tid] = acc;
    __syncthreads();
  }
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
      Fs[tid] = pow2_scale(2.f * ((tid == 0 && !DIG) ? a.wk_absmax : 1.f) * m);
    }
    __syncthreads();
  }
  // B operand (K-major, no swizzle): the NT MSE operands, then the sign plane,
  // 128 K bytes each (a digit operand's B is the query itself: the digit
  // weights are applied to its accumulator).  One item = a 16-byte K slice kb: its 16 fixed-point
  // values of this head are computed once and split into the four limb rows
  // n = 4h + l, each stored as one 16-byte write to the group's B region.
  uint8_t *dst = a.bk + static_cast<int64_t>(bh) * a.bk_stride;
  constexpr int NKC = KTOT / 16;
  for (int kc = tid; kc < NKC; kc += TCT) {
    const int kb = kc * 16;
    const int op = kb / TD;                  // operand (NT = the sign plane)
    const int w = (kb % TD) >> 5;            // 32-coordinate chunk
    const bool dig = DIG && op < NT;
    uint32_t wv[4][4] = {{0u, 0u, 0u, 0u}, {0u, 0u, 0u, 0u}, {0u, 0u, 0u, 0u}, {0u, 0u, 0u, 0u}};
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const int k = (kb & 31) + e;
      const int i = 32 * w + elem_of(dig, k);
      int v;
      if (dig)
        v = __float2int_rn(q1s[i] * Fs[0]);
      else if (op < NT)
        v = __float2int_rn(2.f * a.wk[op] * q1s[i] * Fs[0]) * (1 << (7 - (k >> 2)));
      else
        v = __float2int_rn(2.f * q2s[i] * Fs[1]) * (1 << (7 - (k >> 2)));
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
      *reinterpret_cast<uint4 *>(dst + kmajor_off(4 * h + l, kb, N)) =
          make_uint4(wv[l][0], wv[l][1], wv[l][2], wv[l][3]);
  }
  // rows beyond the G heads' limbs (N > 4 G) are zero (written by head 0's block)
  if constexpr (N > 4 * G) {
    if (h == 0)
      for (int it = tid; it < (N - 4 * G) * NKC; it += TCT) {
        const int n = 4 * G + it % (N - 4 * G), kc = it / (N - 4 * G);
        *reinterpret_cast<uint4 *>(dst + kmajor_off(n, kc * 16, N)) = make_uint4(0u, 0u, 0u, 0u);
      }
  }
  // constants: the offset of each part in B units, and its scale
  {
    double s1 = 0.0;
    if (DIG) {
      s1 = __float2int_rn(q1s[tid] * Fs[0]);
    } else {
#pragma unroll
      for (int t = 0; t < NT; ++t) s1 += __float2int_rn(2.f * a.wk[t] * q1s[tid] * Fs[0]);
    }
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
    if (DIG) {
      // sum_j (V_j - 2^20) B_j / (F_c F): the rotated query against the centroids
      kc[h * 4 + 0] = static_cast<float>(DIG_OFF * s1 / (static_cast<double>(Fs[0]) * a.kfc));
      kc[h * 4 + 1] = static_cast<float>(1.0 / (static_cast<double>(Fs[0]) * a.kfc));
    } else {
      // sum_t a_t (2 x_t - 1): the 0/1 planes weigh 2 a_t, minus sum_t a_t
      kc[h * 4 + 0] = static_cast<float>(s1 / (2.0 * Fs[0]));
      kc[h * 4 + 1] = 1.0f / (128.0f * Fs[0]);
    }
    kc[h * 4 + 2] = static_cast<float>(s2 / (2.0 * Fs[1]));
    kc[h * 4 + 3] = 1.0f / (128.0f * Fs[1]);
  }
  // the main loop reads the cache rows the preceding append kernel writes:
  // this grid completes only after that one (which it may have overlapped)
  sm100::pdl_wait();
}

// ---------------------------------------------------------------------------
// dec_kernel helpers
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

// Warp-uniform bounded wait: every lane polls (so every lane acquires the
// phase), the loop ends for all lanes together.  Gives up when the budget
// runs out or another warp has given up.
__device__ __forceinline__ bool dwait(uint64_t *bar, uint32_t parity, uint32_t outer,
                                      volatile int *abort_flag) {
#pragma unroll 1
  for (uint32_t it = 0; it < outer; ++it) {
    const bool ok = sm100::mbar_wait(bar, parity, 1u << 8);
    if (__all_sync(TQ_FULL, ok)) return true;
    if (__shfl_sync(TQ_FULL, *abort_flag, 0)) return false;
  }
  *abort_flag = 1;
  return false;
}

// Single-thread bounded wait for the copying lanes.
__device__ __forceinline__ bool dwait1(uint64_t *bar, uint32_t parity, uint32_t outer,
                                       volatile int *abort_flag) {
#pragma unroll 1
  for (uint32_t it = 0; it < outer; ++it) {
    if (sm100::mbar_wait(bar, parity, 1u << 8)) return true;
    if (*abort_flag) return false;
  }
  *abort_flag = 1;
  return false;
}

// Barrier of the warp group (warps 0-3) that also tells every thread whether
// all of them are still on track; the tensor-memory fences order the group's
// tcgen05 traffic around it.
__device__ __forceinline__ bool wg_sync(bool ok) {
  sm100::fence_before_sync();
  uint32_t bad;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.eq.u32 q, %1, 0;\n\t"
      "bar.red.or.pred p, 1, 128, q;\n\tselp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(bad)
      : "r"(ok ? 1u : 0u)
      : "memory");
  sm100::fence_after_sync();
  return bad == 0u;
}

// x[i] for a runtime i without indexing the register array (x[0] when i is
// out of range).
template <int K>
__device__ __forceinline__ float pick(const float (&x)[K], int i) {
  float v = x[0];
#pragma unroll
  for (int k = 1; k < K; ++k) v = i == k ? x[k] : v;
  return v;
}

// N accumulator columns of this warp's lanes (N = 8 or 16), loads in flight.
template <int N>
__device__ __forceinline__ void tmem_ldn(uint32_t taddr, uint32_t (&r)[16]) {
  if constexpr (N == 16) {
    sm100::tmem_ld16(taddr, r);
  } else {
    uint32_t t[8];
    sm100::tmem_ld8(taddr, t);
#pragma unroll
    for (int c = 0; c < 8; ++c) r[c] = t[c];
  }
}

// ---------------------------------------------------------------------------
// dec_kernel: split-K decode main loop.  Two CTAs per SM, each walking its
// (batch, KV head, split) units (at most UMAX rows) phase by phase:
//   K  key tiles of 128 rows: code planes -> A operands in tensor memory ->
//      MMAs against the fixed-point query (accumulators for two tiles) ->
//      logits, two tiles later;
//   S  softmax statistics of the unit and the value-side B operand (24-bit
//      weights p * nu_v as four int8 limbs) for all of its 32-token groups;
//   V  value batches of four 32-token groups (two batch buffers) -> MMAs
//      accumulating the rotated-domain sums over the unit;
//   E  fold the value accumulators into the running output of the chunk.
// Warps 0-3 (one TMEM lane per thread) expand, issue and fold: after a
// warp-group barrier, lane 0 of warp w issues the MMAs of operand w, so MMAs
// are issued from several threads at once and no other warp sits between
// expansion and issue.  Warp 4 copies unit headers and key tiles, warp 5
// value groups, ahead of use.  Every wait is bounded; a warp that gives up
// makes the group leave at its next barrier, the CTA drain its copies and
// MMAs, and the call's status word report it.
// ---------------------------------------------------------------------------
constexpr int DT = 192;        // 6 warps
constexpr int UMAX = 1024;     // rows per unit
constexpr int KS = 4;          // key tile stages (shared memory)
constexpr int VS = 8;          // value group stages (shared memory)
constexpr int VB = 4;          // value groups per batch
static_assert(VB % 2 == 0, "value groups are expanded in pairs");
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

template <int G, int MBK, int BV, bool QJL>
__global__ void __launch_bounds__(DT, 2) dec_kernel(TcArgs a) {
  constexpr bool KDIG = use_digits(MBK), VDIG = use_digits(BV);
  constexpr int NT = n_ops(MBK);             // key MSE operands
  constexpr int NV = n_ops(BV);              // value operands
  constexpr int NKO = NT + (QJL ? 1 : 0);    // key operands (one accumulator each)
  constexpr int N = tc_n(G);
  constexpr int NH = N / 4;
  constexpr int PK = MBK + (QJL ? 1 : 0);
  constexpr int BKB = N * TD * NKO;
  constexpr int BKC = BKB + G * 16;
  // tensor memory: key phase: the tile's operands [0, KA) (chunk-major MSE
  // operands, then the sign plane), accumulators D_k[tile parity][op] at
  // C_DK + N (NKO parity + op); value phase: batch buffers [VA b, VA (b + 1))
  // (group g at 8 NV g, operand at 8 op), accumulators D_v[op] at C_DV + N op
  constexpr int KA = 32 * NKO;
  constexpr int C_DK = KA;
  constexpr int VA = VB * NV * 8;
  constexpr int C_DV = 2 * VA;
  static_assert(C_DK + 2 * NKO * N <= DCOLS && C_DV + NV * N <= DCOLS, "tensor memory budget");
  constexpr uint32_t IDESC = sm100::idesc_i8(128, N);
  const DecLayout L = dec_layout(PK, BV, G, N, BKC);

  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ __align__(8) uint64_t kf[KS], ke[KS], vf[VS], ve[VS], hdr[2], hdr_free[2];
  __shared__ __align__(8) uint64_t kdone, vdone[2], fin[4];
  __shared__ uint32_t tmem_s;
  __shared__ volatile int abort_s;
  __shared__ float redf[4][G + 1];
  __shared__ float redl[4][4];
  __shared__ long long redw[4][4];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t outer = a.wait_limit >> 8;

  if (warp == 0) sm100::tmem_alloc(&tmem_s, DCOLS);
  if (tid == 0) {
    for (int i = 0; i < KS; ++i) { sm100::mbar_init(&kf[i], 1); sm100::mbar_init(&ke[i], 4); }
    for (int i = 0; i < VS; ++i) { sm100::mbar_init(&vf[i], 1); sm100::mbar_init(&ve[i], 4); }
    for (int i = 0; i < 2; ++i) {
      sm100::mbar_init(&hdr[i], 1);
      sm100::mbar_init(&hdr_free[i], 1);
      sm100::mbar_init(&vdone[i], NV);
    }
    sm100::mbar_init(&kdone, NKO);
    for (int i = 0; i < 4; ++i) sm100::mbar_init(&fin[i], 1);
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

  if (warp == 4) {
    // ------------------------------------------------ unit headers, key tiles
    if (lane == 0) {
      int cit = blockIdx.x, cr0 = -1, u = 0;
      uint32_t kt = 0;
      // per stage: 1 + the parity of its last issued copy (0 = never issued)
      uint8_t lk[KS] = {}, lh[2] = {};
      bool have = tc_next(a, cit, cr0);
      while (have && !abort_s) {
        const int b = cit / (a.Hkv * a.splits), kvh = (cit / a.splits) % a.Hkv, sp = cit % a.splits;
        const int64_t bh = static_cast<int64_t>(b) * a.Hkv + kvh;
        const int c0 = sp * a.chunk, c1 = min(tc_len(a, b), c0 + a.chunk);
        const int nvalid = min(a.sub, c1 - cr0);
        const int ntile = (nvalid + 127) / 128, ngroups = (nvalid + 31) / 32;
        // key tiles; the unit header (B operand, constants and value norms,
        // buffer u & 1, once unit u - 2 has finished its softmax phase with
        // it) follows the first tile, whose data has the longer way to come
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
          if (j == 0) {
            const int hb = u & 1;
            if (u >= 2 && !dwait1(&hdr_free[hb], ((u >> 1) - 1) & 1, outer, &abort_s)) break;
            const uint32_t nvn = static_cast<uint32_t>(ngroups) * 64;
            sm100::mbar_expect_tx(&hdr[hb], static_cast<uint32_t>((BKC + 15) & ~15) + nvn);
            sm100::bulk_g2s(smem + L.o_bk + hb * L.bkc, a.bk + bh * a.bk_stride, (BKC + 15) & ~15, &hdr[hb]);
            sm100::bulk_g2s(smem + L.o_vn + hb * UMAX * 2, a.vnorm + bh * a.rows_cap + cr0, nvn, &hdr[hb]);
            lh[hb] = static_cast<uint8_t>(1 + ((u >> 1) & 1));
          }
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
        for (int i = 0; i < 2; ++i)
          if (lh[i]) sm100::mbar_wait(&hdr[i], lh[i] - 1u, 1u << 20);
      }
    }
    __syncwarp();
  } else if (warp == 5) {
    // ------------------------------------------------------------ value groups
    if (lane == 0) {
      int cit = blockIdx.x, cr0 = -1;
      uint32_t vg = 0;
      uint8_t lv[VS] = {};
      bool have = tc_next(a, cit, cr0);
      while (have && !abort_s) {
        const int b = cit / (a.Hkv * a.splits), kvh = (cit / a.splits) % a.Hkv, sp = cit % a.splits;
        const int64_t bh = static_cast<int64_t>(b) * a.Hkv + kvh;
        const int c0 = sp * a.chunk, c1 = min(tc_len(a, b), c0 + a.chunk);
        const int nvalid = min(a.sub, c1 - cr0);
        const int ngroups = (nvalid + 31) / 32;
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
      }
      if (abort_s)
        for (int i = 0; i < VS; ++i)
          if (lv[i]) sm100::mbar_wait(&vf[i], lv[i] - 1u, 1u << 20);
    }
    __syncwarp();
  } else {
    // --------------------------------------------------------- the warp group
    // empty chunks (beyond a batch's length) merge with weight zero
    {
      const int items = a.B * a.Hkv * a.splits;
      for (int it = blockIdx.x; it < items; it += gridDim.x) {
        const int b = it / (a.Hkv * a.splits), kvh = (it / a.splits) % a.Hkv, sp = it % a.splits;
        if (sp * a.chunk < tc_len(a, b)) continue;
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
    uint32_t ktab[NDIG][4], vtab[NDIG][4];
#pragma unroll
    for (int d = 0; d < NDIG; ++d)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        ktab[d][i] = a.ktab[d][i];
        vtab[d][i] = a.vtab[d][i];
      }
    float *lg = reinterpret_cast<float *>(smem + L.o_lg);
    int8_t *bvs = reinterpret_cast<int8_t *>(smem + L.o_bv);
    const uint32_t bv_addr = sm100::smem_addr(bvs);
    int cit = blockIdx.x, cr0 = -1, u = 0;
    uint32_t kt = 0, vg = 0, vb = 0;
    float o[G], m_run[G], l_run[G];
#pragma unroll
    for (int h = 0; h < G; ++h) { o[h] = 0.f; m_run[h] = -CUDART_INF_F; l_run[h] = 0.f; }
    bool ok = true;
    bool have = tc_next(a, cit, cr0);
    while (have) {
      const int b = cit / (a.Hkv * a.splits), kvh = (cit / a.splits) % a.Hkv, sp = cit % a.splits;
      const int len = tc_len(a, b);
      const int c0 = sp * a.chunk, c1 = min(len, c0 + a.chunk);
      const int nvalid = min(a.sub, c1 - cr0);
      const int ntile = (nvalid + 127) / 128, ngroups = (nvalid + 31) / 32;
      const float *kcst = reinterpret_cast<const float *>(smem + L.o_bk + (u & 1) * L.bkc + BKB);
      const uint32_t bk_addr = sm100::smem_addr(smem + L.o_bk + (u & 1) * L.bkc);
      if (cr0 == c0) {
#pragma unroll
        for (int h = 0; h < G; ++h) { o[h] = 0.f; m_run[h] = -CUDART_INF_F; l_run[h] = 0.f; }
      }
      float mloc[G];
#pragma unroll
      for (int h = 0; h < G; ++h) mloc[h] = -CUDART_INF_F;
      if (ok) ok = dwait(&hdr[u & 1], (u >> 1) & 1, outer, &abort_s);   // B operand, constants
      if (!wg_sync(ok)) break;
      // ---------------- K phase: tile j is expanded once the MMAs of tile j - 1
      // have released the operand buffer; its epilogue runs two tiles later
      // (accumulators double-buffered), so MMAs overlap expansion both ways
      uint32_t sc_hist[2] = {0u, 0u};
      for (int j = 0; j <= ntile + 1; ++j) {
        const uint32_t ti = kt + j;
        const bool expand = j < ntile;
        uint32_t pw[PK][TNW];
        uint32_t sc = 0u;
        if (expand && ok) ok = dwait(&kf[ti % KS], (ti / KS) & 1, outer, &abort_s);
        if (expand && ok) {
          const uint8_t *stg = smem + L.o_kt + (ti % KS) * L.ktb;
          const uint4 *kr = reinterpret_cast<const uint4 *>(stg + tid * PK * 16);
#pragma unroll
          for (int p = 0; p < PK; ++p) {
            const uint4 v = kr[p];
            pw[p][0] = v.x; pw[p][1] = v.y; pw[p][2] = v.z; pw[p][3] = v.w;
          }
          sc = reinterpret_cast<const uint32_t *>(stg + 128 * PK * 16)[tid];
          __syncwarp();
          if (lane == 0) sm100::mbar_arrive(&ke[ti % KS]);
        }
        // epilogue of tile j - 2
        if (j >= 2) {
          if (j - 1 >= ntile && ok) ok = dwait(&kdone, (ti - 2) & 1, outer, &abort_s);
          if (ok) {
            sm100::fence_after_sync();
            uint32_t dacc[NKO][16];
#pragma unroll
            for (int op = 0; op < NKO; ++op)
              tmem_ldn<N>(sm100::tmem_lane(tm + C_DK + (((ti - 2) & 1) * NKO + op) * N, warp), dacc[op]);
            sm100::wait_ld();
            const uint32_t scj = sc_hist[(ti - 2) & 1];
            const int rl = (j - 2) * 128 + tid;
            const bool valid = rl < nvalid;
            const float nu = tq_half_to_f32(static_cast<uint16_t>(scj & 0xffffu));
            const float rho = tq_half_to_f32(static_cast<uint16_t>(scj >> 16));
#pragma unroll
            for (int h = 0; h < G; ++h) {
              float raw;
              if constexpr (KDIG)
                raw = fmaf(DIG_W0, comb_limbs(dacc[0] + 4 * h),
                           fmaf(DIG_W1, comb_limbs(dacc[1] + 4 * h), comb_limbs(dacc[2] + 4 * h)));
              else if constexpr (NT == 2)
                raw = comb_limbs(dacc[0] + 4 * h) + comb_limbs(dacc[1] + 4 * h);
              else
                raw = comb_limbs(dacc[0] + 4 * h);
              const float dmv = raw * kcst[4 * h + 1] - kcst[4 * h + 0];
              float est = dmv;
              if (QJL) {
                const float dj = comb_limbs(dacc[NKO - 1] + 4 * h) * kcst[4 * h + 3] - kcst[4 * h + 2];
                est = fmaf(a.qjl_coef * rho, dj, dmv);
              }
              const float l = valid ? a.scale * nu * est : -CUDART_INF_F;
              lg[rl * G + h] = l;
              mloc[h] = fmaxf(mloc[h], l);
              if (a.logits && valid)
                a.logits[(static_cast<int64_t>(b) * a.Hq + kvh * G + h) * a.max_len + cr0 + rl] = l;
            }
          }
        }
        if (expand) {
          // the MMAs of tile j - 1 have released the operand buffer
          if (j >= 1 && ok) ok = dwait(&kdone, (ti - 1) & 1, outer, &abort_s);
          if (ok) {
            sm100::fence_after_sync();
            const uint32_t abuf = sm100::tmem_lane(tm, warp);
            // operand op, chunk w at columns 32 op + 8 w
#pragma unroll
            for (int w = 0; w < TNW; ++w) {
              if constexpr (KDIG) {
                uint32_t pl[MBK], dw[NDIG][8];
#pragma unroll
                for (int p = 0; p < MBK; ++p) pl[p] = pw[p][w];
                digit_words<MBK>(pl, ktab, dw);
#pragma unroll
                for (int k = 0; k < NDIG; ++k) sm100::tmem_st8(abuf + 32 * k + 8 * w, dw[k]);
              } else {
#pragma unroll
                for (int t = 0; t < NT; ++t) {
                  uint32_t r8[8];
                  plane_words(pw[t][w], r8);
                  sm100::tmem_st8(abuf + 32 * t + 8 * w, r8);
                }
              }
            }
            if (QJL) {
              uint32_t r32[32];
#pragma unroll
              for (int w = 0; w < TNW; ++w) plane_words(pw[PK - 1][w], r32 + 8 * w);
              sm100::tmem_st32(abuf + 32 * NT, r32);
            }
            sm100::wait_st();
          }
          sc_hist[ti & 1] = sc;
        }
        // tile j's operands are stored, D_k[j & 1] has been read: issue
        if (!(ok = wg_sync(ok))) break;
        if (expand && warp < NKO && lane == 0) {
          const uint32_t acc = tm + C_DK + ((ti & 1) * NKO + warp) * N;
#pragma unroll
          for (int w = 0; w < TNW; ++w)
            sm100::mma_i8_ts(acc, tm + 32 * warp + 8 * w,
                             sm100::smem_desc(bk_addr + warp * 128 * N + w * 32 * N, N * 16, 128), IDESC,
                             w > 0 ? 1u : 0u);
          sm100::mma_commit(&kdone);
        }
        __syncwarp();
      }
      if (!ok) break;
      kt += ntile;
      // ---------------- S phase: softmax statistics and the value-side B operand
      const uint16_t *vn = reinterpret_cast<const uint16_t *>(smem + L.o_vn + (u & 1) * UMAX * 2);
      {
        // the unit's largest logit of each head and largest value norm
        float numax = 0.f;
        for (int rl = tid; rl < nvalid; rl += 128) numax = fmaxf(numax, tq_half_to_f32(vn[rl]));
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float m = tq_warp_max(mloc[h]);
          if (lane == 0) redf[warp][h] = m;
        }
        const float nm = tq_warp_max(numax);
        if (lane == 0) redf[warp][G] = nm;
      }
      if (!(ok = wg_sync(ok))) break;
      float mnew[G], corr[G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float m = fmaxf(fmaxf(redf[0][h], redf[1][h]), fmaxf(redf[2][h], redf[3][h]));
        mnew[h] = fmaxf(m_run[h], m);
        corr[h] = __expf(m_run[h] - mnew[h]);
      }
      const float FV = pow2_scale(fmaxf(fmaxf(redf[0][G], redf[1][G]), fmaxf(redf[2][G], redf[3][G])));
      {
        // element (n = 4h + l, k = 4w + b) of group g's B operand holds limb l
        // of W = round(p nu_v FV), p = exp(l - m_new), for the token at byte b
        // of A word w (times 2^(7-w) for bit planes); one item = (group, word,
        // head) makes the 4 bytes of each limb row, stored as one 32-bit word;
        // rows n >= 4G are zero.  Every (token, head) weight is made once, so
        // the softmax sums are taken here too.
        const int h = tid % NH;
        const float mh = pick(mnew, h);
        float lpart = 0.f;
        long long wpart = 0;
        for (int it = tid; it < ngroups * 8 * NH; it += 128) {
          const int w = (it / NH) & 7, g = it / (8 * NH);
          uint32_t word[4] = {0u, 0u, 0u, 0u};
          if (h < G) {
            // v + 0x808080 = sum_l 256^l b_l: limbs l < 3 are b_l - 128 (the
            // byte XOR 0x80), limb 3 is b_3; a 4 x 4 byte transpose gathers
            // limb l of the four tokens into word l
            uint32_t bv[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int rl = 32 * g + elem_of(VDIG, 4 * w + e);
              int W = 0;
              if (rl < nvalid) {
                const float p = __expf(lg[rl * G + h] - mh);
                lpart += p;
                W = __float2int_rn(p * tq_half_to_f32(vn[rl]) * FV);
              }
              wpart += W;
              const int v = VDIG ? W : W * (1 << (7 - w));
              bv[e] = static_cast<uint32_t>(v) + 0x808080u;
            }
            const uint32_t lo01 = prmt(bv[0], bv[1], 0x5140u), hi01 = prmt(bv[0], bv[1], 0x7362u);
            const uint32_t lo23 = prmt(bv[2], bv[3], 0x5140u), hi23 = prmt(bv[2], bv[3], 0x7362u);
            word[0] = prmt(lo01, lo23, 0x5410u) ^ 0x80808080u;
            word[1] = prmt(lo01, lo23, 0x7632u) ^ 0x80808080u;
            word[2] = prmt(hi01, hi23, 0x5410u) ^ 0x80808080u;
            word[3] = prmt(hi01, hi23, 0x7632u);
          }
          int8_t *dst = bvs + g * N * 32;
#pragma unroll
          for (int l = 0; l < 4; ++l)
            *reinterpret_cast<uint32_t *>(dst + kmajor_off(4 * h + l, 4 * w, N)) = word[l];
        }
        // sums over the lanes of this warp that share head h
#pragma unroll
        for (int o = NH; o < 32; o <<= 1) {
          lpart += __shfl_xor_sync(TQ_FULL, lpart, o);
          wpart += __shfl_xor_sync(TQ_FULL, wpart, o);
        }
        if (lane < NH) {
          redl[warp][lane] = lpart;
          redw[warp][lane] = wpart;
        }
      }
      sm100::fence_async_smem();
      if (!(ok = wg_sync(ok))) break;
      if (tid == 0) sm100::mbar_arrive(&hdr_free[u & 1]);   // header no longer read
      float wtot[G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float lsum = redl[0][h] + redl[1][h] + redl[2][h] + redl[3][h];
        wtot[h] = static_cast<float>(redw[0][h] + redw[1][h] + redw[2][h] + redw[3][h]) / FV;
        o[h] *= corr[h];
        l_run[h] = l_run[h] * corr[h] + lsum;
        m_run[h] = mnew[h];
      }
      // ---------------- V phase: batches of VB groups (lane = coordinate)
      const int nbat = (ngroups + VB - 1) / VB;
      for (int bi = 0; bi < nbat; ++bi) {
        const uint32_t vbi = vb + bi;
        const uint32_t abuf = sm100::tmem_lane(tm + (vbi & 1) * VA, warp);
        // the buffer's previous batch (vbi - 2) has been multiplied
        if (vbi >= 2 && ok) ok = dwait(&vdone[vbi & 1], ((vbi >> 1) - 1) & 1, outer, &abort_s);
        if (ok) sm100::fence_after_sync();
        // the batch's groups: every wait first, then the column words of all
        // of them, then the expansion as straight-line code (two groups at
        // a time, so their independent chains interleave).  A group past the
        // unit's end is expanded from whatever its stage holds and never
        // multiplied; only real groups release their stages.
        const int gcount = min(VB, ngroups - bi * VB);
#pragma unroll
        for (int gi = 0; gi < VB; ++gi) {
          const uint32_t vgg = vg + bi * VB + gi;
          if (gi < gcount && ok) ok = dwait(&vf[vgg % VS], (vgg / VS) & 1, outer, &abort_s);
        }
        if (ok) {
          uint32_t pv[VB][BV];
#pragma unroll
          for (int gi = 0; gi < VB; ++gi) {
            const uint32_t *vc =
                reinterpret_cast<const uint32_t *>(smem + L.o_vt + ((vg + bi * VB + gi) % VS) * L.vgb);
#pragma unroll
            for (int p = 0; p < BV; ++p) pv[gi][p] = vc[p * TD + tid];
          }
          __syncwarp();
          if (lane < gcount) sm100::mbar_arrive(&ve[(vg + bi * VB + lane) % VS]);
#pragma unroll
          for (int g2 = 0; g2 < VB; g2 += 2) {
            if constexpr (VDIG) {
              uint32_t dw[2][NDIG][8];
              digit_words<BV>(pv[g2], vtab, dw[0]);
              digit_words<BV>(pv[g2 + 1], vtab, dw[1]);
#pragma unroll
              for (int e = 0; e < 2; ++e)
#pragma unroll
                for (int k = 0; k < NDIG; ++k) sm100::tmem_st8(abuf + (g2 + e) * NV * 8 + 8 * k, dw[e][k]);
            } else {
#pragma unroll
              for (int e = 0; e < 2; ++e)
#pragma unroll
                for (int t = 0; t < NV; ++t) {
                  uint32_t r8[8];
                  plane_words(pv[g2 + e][t], r8);
                  sm100::tmem_st8(abuf + (g2 + e) * NV * 8 + 8 * t, r8);
                }
            }
          }
        }
        sm100::wait_st();
        if (!(ok = wg_sync(ok))) break;
        if (warp < NV && lane == 0) {
          // warp op issues accumulator D_v[op] (its first group starts it)
          const uint32_t acc = tm + C_DV + warp * N;
#pragma unroll
          for (int gi = 0; gi < VB; ++gi) {
            const int g = bi * VB + gi;
            if (g < ngroups)
              sm100::mma_i8_ts(acc, tm + (vbi & 1) * VA + gi * NV * 8 + warp * 8,
                               sm100::smem_desc(bv_addr + g * N * 32, N * 16, 128), IDESC, g > 0 ? 1u : 0u);
          }
          sm100::mma_commit(&vdone[vbi & 1]);
        }
        __syncwarp();
      }
      if (!ok) break;
      vb += nbat;
      vg += ngroups;
      // ---------------- E phase: all value MMAs of the unit have landed
      ok = dwait(&vdone[(vb - 1) & 1], ((vb - 1) >> 1) & 1, outer, &abort_s);
      if (ok) {
        sm100::fence_after_sync();
        uint32_t dv[NV][16];
#pragma unroll
        for (int op = 0; op < NV; ++op) tmem_ldn<N>(sm100::tmem_lane(tm + C_DV + op * N, warp), dv[op]);
        sm100::wait_ld();
        float acc[G];
#pragma unroll
        for (int h = 0; h < G; ++h) {
          acc[h] = 0.f;
#pragma unroll
          for (int op = 0; op < NV; ++op) acc[h] = fmaf(a.vcoef[op], comb_limbs(dv[op] + 4 * h), acc[h]);
        }
        const float ivs = 1.0f / FV;
#pragma unroll
        for (int h = 0; h < G; ++h) o[h] += acc[h] * ivs - a.vbias * wtot[h];
        if (cr0 + a.sub >= c1) {
#pragma unroll
          for (int h = 0; h < G; ++h) {
            const int64_t hq = static_cast<int64_t>(b) * a.Hq + kvh * G + h;
            a.po[(hq * a.splits + sp) * TD + tid] = o[h];
            if (tid == 0) {
              a.pml[(hq * a.splits + sp) * 2] = m_run[h];
              a.pml[(hq * a.splits + sp) * 2 + 1] = l_run[h];
            }
          }
        }
      }
      cr0 += a.sub;
      have = tc_next(a, cit, cr0);
      ++u;
    }
    // every MMA this thread issued has landed before tensor memory is freed
    if (lane == 0) {
      sm100::mma_commit(&fin[warp]);
      sm100::mbar_wait(&fin[warp], 0, 1u << 20);
    }
    __syncwarp();
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
  constexpr int N = tc_n(G);
  constexpr int PK = MBK + (QJL ? 1 : 0);
  constexpr int BKC = N * TD * (n_ops(MBK) + (QJL ? 1 : 0)) + G * 16;
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
  const int bytes = tc_n(G) * TD * (n_ops(c->mse_bits_k) + (c->qjl_k ? 1 : 0)) + G * 16;
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
  for (int i = 0; i < 8; ++i) a.wk[i] = c->walsh_k[i];
  a.wk_absmax = c->walsh_k_absmax;
  for (int d = 0; d < 3; ++d)
    for (int i = 0; i < 4; ++i) {
      a.ktab[d][i] = c->digit_k[d][i];
      a.vtab[d][i] = c->digit_v[d][i];
    }
  a.kfc = c->digit_k_scale;
  if (use_digits(c->bits_v)) {
    // value = sum_tokens W (V - 2^20) / F_c with V = 2^14 d0 + 2^7 d1 + d2
    a.vcoef[0] = 16384.0f / c->digit_v_scale;
    a.vcoef[1] = 128.0f / c->digit_v_scale;
    a.vcoef[2] = 1.0f / c->digit_v_scale;
    a.vbias = 1048576.0f / c->digit_v_scale;
  } else {
    // value = sum_t a_t (2 x_t - 1); the planes' B carries an extra 2^7
    a.vcoef[0] = c->walsh_v[0] / 64.0f;
    a.vcoef[1] = c->walsh_v[1] / 64.0f;
    a.vcoef[2] = 0.f;
    a.vbias = c->walsh_v_sum;
  }
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
