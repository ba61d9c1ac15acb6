// Prefill quantize, one thread per token row (sm_100a).
//
// Same per-row computation as quantize.cu ("TurboESM ..." section 2.A: RoPE,
// then the rotation; "FibQuant ..." section 2.3: store nu, rotate x / nu,
// quantize; "Ablazione ..." "Configurazione Sperimentale": randomized
// Walsh-Hadamard rotation and Beta Lloyd-Max codebooks; "Google presenta
// TurboQuant ..." "Eliminacion del sesgo": b-1 MSE bits plus the 1-bit QJL
// sketch of the residual), laid out for throughput on large calls:
//
// * A tile is 128 consecutive cache rows of one (batch, head), aligned to 128
//   rows, so each warp owns exactly one 32-token value column group.  The
//   K, V and RoPE-table tiles arrive by TMA tensor copies with the 128-byte
//   swizzle, so thread r reads its own row from shared memory without bank
//   conflicts.  Rows outside the call are zero-filled by the copy and skipped
//   on store; the tiles of a unit's missing heads (the last head group of an
//   odd B x H) are not copied and their rows are inactive.
// * Every thread runs its row alone: RoPE, norm, the sign flip D (a packed
//   multiply by +-1), the d-point Walsh-Hadamard transform in registers (no
//   shuffles), codes by compares against the upper half of the symmetric
//   codebook (the middle threshold is 0), and bit planes accumulated one
//   funnel shift per coordinate (the sign of y enters the lower planes once
//   per 32-coordinate word).  Value planes are moved into the 32-token column
//   layout with warp-wide 32 x 32 bit transposes.
// * Keys: the residual of the tile, split into bf16 hi + lo, is stored into
//   tensor memory and sketched against S (exactly bf16) by tcgen05 kind::f16
//   MMAs with fp32 accumulation; each thread reads its row of S r back.
// * One CTA per SM with NTL row-warp groups (four at d = 64, two at d = 128),
//   group g taking the rows of tile g of a unit.  A unit is NTL tiles at the
//   same positions (consecutive heads of the flattened batch x head index)
//   and one kind, keys or values; units are ordered (position tile, head
//   group, kind), and each CTA takes a contiguous range of them, first all of
//   its key units, then its value units, so the SM's instruction cache holds
//   one row path at a time and the load stays balanced to half a unit.
//   Thread 0 issues the copies of the next unit (once a barrier shows every
//   row of the current one in registers) and, for keys, the sketch MMAs of
//   the unit (once a barrier shows every operand stored).  Without a separate
//   copy warp a thread keeps 128 (d = 64) or 255 (d = 128) registers.  The
//   RoPE table tile is reloaded only when the position range changes.
//
// Codes are decided on the scaled transform y = H D x against t_k * sqrt(d) nu
// (the same decision as u = y / (sqrt(d) nu) against t_k, up to fp32
// rounding); the sketch signs are invariant to that positive scale.
#include <cuda.h>

#include <cstdlib>
#include <cstring>

#include "tq_device.cuh"
#include "tq_sm100.cuh"

namespace {

constexpr int QR = 128;         // rows per tile
// tiles per unit: at d = 64 four tiles' sketch accumulators (4 x 128 tensor
// memory columns) and 16 row warps of 128 registers fill an SM; at d = 128 two
__host__ __device__ constexpr int tiles_per_unit(int d) { return d == 64 ? 4 : 2; }
constexpr uint32_t BOX = QR * 128;   // bytes of one swizzled 128-row box

struct TileArgs {
  int B, H, T;
  int64_t row0, pos0, rows_cap;
  int64_t R_first;   // cache row of the first row tile (multiple of 128)
  int64_t nrt;       // row tiles per (batch, head)
  int64_t groups;    // head groups per row tile: ceil(B * H / tiles per unit)
  int64_t nunits;    // 2 * nrt * groups, ordered (row tile, head group, kind)
  uint8_t *kcode;
  uint16_t *kscale;
  uint32_t *vcode;
  uint16_t *vnorm;
  uint32_t *status;
  const uint16_t *S;
  uint32_t wait_outer;   // rounds of 2^14 polls per wait before giving up
  int rope;
  float ck[8];       // key centroid magnitudes c[half + m], m = 0 .. half-1
  float tk[8];       // key thresholds above 0: t[half - 1 + j], j = 1 .. half-1 (tk[j - 1])
  float tv[8];       // value thresholds above 0
  float dsg[128];    // D as +-1 pairs: dsg[2 j] = D_j, dsg[2 j + 1] = D_{j + d/2}, j < d/2
};

// ---------------------------------------------------------------- TMA

__device__ __forceinline__ void tma_4d(void *dst, const CUtensorMap *map, int c0, int c1, int c2,
                                       int c3, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(sm100::smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3),
      "r"(sm100::smem_addr(bar))
      : "memory");
}

__device__ __forceinline__ void tma_2d(void *dst, const CUtensorMap *map, int c0, int c1,
                                       uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3}], [%4];" ::"r"(sm100::smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(sm100::smem_addr(bar))
      : "memory");
}

// 16-byte chunk c of row r in a 128-byte-swizzled box (1024-byte aligned).
__device__ __forceinline__ uint4 swz_ld(const uint8_t *box, int r, int c) {
  return *reinterpret_cast<const uint4 *>(box + r * 128 + ((c ^ (r & 7)) << 4));
}

// Bounded wait that also gives up as soon as another thread has.
__device__ __forceinline__ bool wait_or_abort(uint64_t *bar, uint32_t parity, uint32_t outer,
                                              volatile int *abort_flag) {
  for (uint32_t it = 0; it < outer; ++it) {
    if (sm100::mbar_wait(bar, parity, 1u << 14)) return true;
    if (*abort_flag) return false;
  }
  return false;
}

// Barrier of the CTA that also tells every thread whether all of them are
// still on track (bar.red.or over the give-up flags); the tensor-memory
// fences order tcgen05 traffic around it.
template <int NT>
__device__ __forceinline__ bool cta_all_ok(bool ok) {
  sm100::fence_before_sync();
  uint32_t bad;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.eq.u32 q, %1, 0;\n\t"
      "bar.red.or.pred p, 1, %2, q;\n\tselp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(bad)
      : "r"(ok ? 1u : 0u), "n"(NT)
      : "memory");
  sm100::fence_after_sync();
  return bad == 0u;
}

// Packed fp32 pair arithmetic (sm_100): each half rounds exactly like the
// scalar instruction.
__device__ __forceinline__ void addsub2(float &a0, float &a1, float &b0, float &b1) {
  // (a, b) <- (a + b, a - b) for both halves of the pairs (a0, a1), (b0, b1)
  asm("{\n\t.reg .b64 p, q, s, d;\n\t"
      "mov.b64 p, {%0, %1};\n\tmov.b64 q, {%2, %3};\n\t"
      "add.rn.f32x2 s, p, q;\n\tsub.rn.f32x2 d, p, q;\n\t"
      "mov.b64 {%0, %1}, s;\n\tmov.b64 {%2, %3}, d;\n\t}\n"
      : "+f"(a0), "+f"(a1), "+f"(b0), "+f"(b1));
}

// (a, b) packed into one 64-bit register.
__device__ __forceinline__ uint64_t pk2(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}

// (d0, d1) = (a0, a1) - c
__device__ __forceinline__ void sub2c(float a0, float a1, uint64_t c, float &d0, float &d1) {
  asm("{\n\t.reg .b64 p, d;\n\tmov.b64 p, {%2, %3};\n\tsub.rn.f32x2 d, p, %4;\n\t"
      "mov.b64 {%0, %1}, d;\n\t}\n"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "l"(c));
}

// (d0, d1) = (a0, a1) - (b0, b1)
__device__ __forceinline__ void sub2(float a0, float a1, float b0, float b1, float &d0, float &d1) {
  asm("{\n\t.reg .b64 p, q, d;\n\tmov.b64 p, {%2, %3};\n\tmov.b64 q, {%4, %5};\n\t"
      "sub.rn.f32x2 d, p, q;\n\tmov.b64 {%0, %1}, d;\n\t}\n"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

// (a0, a1) *= c (exact for c = (+-1, +-1))
__device__ __forceinline__ void mul2c(float &a0, float &a1, uint64_t c) {
  asm("{\n\t.reg .b64 p, d;\n\tmov.b64 p, {%0, %1};\n\tmul.rn.f32x2 d, p, %2;\n\t"
      "mov.b64 {%0, %1}, d;\n\t}\n"
      : "+f"(a0), "+f"(a1)
      : "l"(c));
}

// acc += (a0 * a0, a1 * a1)
__device__ __forceinline__ void sq2acc(float a0, float a1, uint64_t &acc) {
  asm("{\n\t.reg .b64 p;\n\tmov.b64 p, {%1, %2};\n\tfma.rn.f32x2 %0, p, p, %0;\n\t}\n"
      : "+l"(acc)
      : "f"(a0), "f"(a1));
}

__device__ __forceinline__ float hsum2(uint64_t v) {
  float a, b;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
  return a + b;
}

// In-register Walsh-Hadamard transform, Sylvester natural order: y = H_D x.
// Stages of stride s < D/2 pair element i with i + D/2 (the same butterfly
// in both halves) and run on packed pairs; the stride-D/2 stage is scalar.
// Same stage order and operations as the plain radix-2 loop.
template <int D>
__device__ __forceinline__ void wht_regs(float (&x)[D]) {
  constexpr int H = D / 2;
#pragma unroll
  for (int s = 1; s < H; s <<= 1) {
#pragma unroll
    for (int i = 0; i < H; ++i) {
      if (!(i & s)) addsub2(x[i], x[i + H], x[i + s], x[i + s + H]);
    }
  }
#pragma unroll
  for (int i = 0; i < H; ++i) {
    const float a = x[i], b = x[i + H];
    x[i] = a + b;
    x[i + H] = a - b;
  }
}

// Sign bits of the code planes of one coordinate: plane p's bit, inverted,
// sits in the top bit of the returned word p (see the thermometer identities
// in the kernel comment).  y: transformed coordinate; th: thresholds above 0
// times the row scale, ascending; NB: code bits.
template <int NB>
__device__ __forceinline__ void plane_msbs(float y, const float *th, uint32_t (&w)[4]) {
  constexpr int NT = (1 << (NB - 1)) - 1;   // thresholds above 0
  const float a = fabsf(y);
  uint32_t s[NT > 0 ? NT : 1];
#pragma unroll
  for (int j = 0; j < NT; ++j) s[j] = __float_as_uint(a - th[j]);
  const uint32_t sy = __float_as_uint(y);
  w[NB - 1] = sy;                       // top bit = [y >= 0]
  if (NB == 2) {
    w[0] = s[0] ^ sy;
  } else if (NB == 3) {
    w[1] = s[1] ^ sy;
    w[0] = s[0] ^ s[1] ^ s[2] ^ sy;
  } else if (NB == 4) {
    w[2] = s[3] ^ sy;
    w[1] = s[1] ^ s[3] ^ s[5] ^ sy;
    w[0] = s[0] ^ s[1] ^ s[2] ^ s[3] ^ s[4] ^ s[5] ^ s[6] ^ sy;
  }
}

// plane_msbs for two coordinates at once, the threshold differences taken as
// packed pairs (th2[j] = (th[j], th[j])).
template <int NB>
__device__ __forceinline__ void plane_msbs2(float y0, float y1, const uint64_t *th2, uint32_t (&w0)[4],
                                            uint32_t (&w1)[4]) {
  constexpr int NT = (1 << (NB - 1)) - 1;   // thresholds above 0
  const float a0 = fabsf(y0), a1 = fabsf(y1);
  uint32_t s0[NT > 0 ? NT : 1], s1[NT > 0 ? NT : 1];
#pragma unroll
  for (int j = 0; j < NT; ++j) {
    float d0, d1;
    sub2c(a0, a1, th2[j], d0, d1);
    s0[j] = __float_as_uint(d0);
    s1[j] = __float_as_uint(d1);
  }
  const uint32_t sy0 = __float_as_uint(y0), sy1 = __float_as_uint(y1);
  w0[NB - 1] = sy0;
  w1[NB - 1] = sy1;
  if (NB == 2) {
    w0[0] = s0[0] ^ sy0;
    w1[0] = s1[0] ^ sy1;
  } else if (NB == 3) {
    w0[1] = s0[1] ^ sy0;
    w0[0] = s0[0] ^ s0[1] ^ s0[2] ^ sy0;
    w1[1] = s1[1] ^ sy1;
    w1[0] = s1[0] ^ s1[1] ^ s1[2] ^ sy1;
  } else if (NB == 4) {
    w0[2] = s0[3] ^ sy0;
    w0[1] = s0[1] ^ s0[3] ^ s0[5] ^ sy0;
    w0[0] = s0[0] ^ s0[1] ^ s0[2] ^ s0[3] ^ s0[4] ^ s0[5] ^ s0[6] ^ sy0;
    w1[2] = s1[3] ^ sy1;
    w1[1] = s1[1] ^ s1[3] ^ s1[5] ^ sy1;
    w1[0] = s1[0] ^ s1[1] ^ s1[2] ^ s1[3] ^ s1[4] ^ s1[5] ^ s1[6] ^ sy1;
  }
}

// The code planes below the top one for two coordinates, without their sign
// term (plane_msbs's thermometer XORs with sy left out): word p's top bit is
// plane p's bit for |y| alone.  a0, a1: |y|; th2: packed thresholds above 0
// times the row scale.
template <int NB>
__device__ __forceinline__ void therm_msbs2(float a0, float a1, const uint64_t *th2, uint32_t (&w0)[4],
                                            uint32_t (&w1)[4]) {
  constexpr int NT = (1 << (NB - 1)) - 1;   // thresholds above 0
  uint32_t s0[NT > 0 ? NT : 1], s1[NT > 0 ? NT : 1];
#pragma unroll
  for (int j = 0; j < NT; ++j) {
    float d0, d1;
    sub2c(a0, a1, th2[j], d0, d1);
    s0[j] = __float_as_uint(d0);
    s1[j] = __float_as_uint(d1);
  }
  if constexpr (NB == 2) {
    w0[0] = s0[0];
    w1[0] = s1[0];
  } else if constexpr (NB == 3) {
    w0[1] = s0[1];
    w0[0] = s0[0] ^ s0[1] ^ s0[2];
    w1[1] = s1[1];
    w1[0] = s1[0] ^ s1[1] ^ s1[2];
  } else if constexpr (NB == 4) {
    w0[2] = s0[3];
    w0[1] = s0[1] ^ s0[3] ^ s0[5];
    w0[0] = s0[0] ^ s0[1] ^ s0[2] ^ s0[3] ^ s0[4] ^ s0[5] ^ s0[6];
    w1[2] = s1[3];
    w1[1] = s1[1] ^ s1[3] ^ s1[5];
    w1[0] = s1[0] ^ s1[1] ^ s1[2] ^ s1[3] ^ s1[4] ^ s1[5] ^ s1[6];
  }
}

// Raw decision bits of coordinates i and i + D/2, accumulated one funnel shift
// per bit (coordinate 32 w + 31 first, so bit e of word w is coordinate
// 32 w + e): acc[t] gathers the sign bits of |y| - th[t] (t < NT, th2[t] =
// (th[t], th[t])), acc[NT] those of y.  planes_of() then forms each code
// plane word from them by the thermometer identities of plane_msbs.
template <int NB, int NW>
__device__ __forceinline__ void raw_bits2(float y0, float y1, const uint64_t *th2,
                                          uint32_t (&acc)[1 << (NB - 1)][NW], int i, int i1) {
  constexpr int NT = (1 << (NB - 1)) - 1;   // thresholds above 0
  const float a0 = fabsf(y0), a1 = fabsf(y1);
#pragma unroll
  for (int t = 0; t < NT; ++t) {
    float d0, d1;
    sub2c(a0, a1, th2[t], d0, d1);
    acc[t][i >> 5] = __funnelshift_l(__float_as_uint(d0), acc[t][i >> 5], 1);
    acc[t][i1 >> 5] = __funnelshift_l(__float_as_uint(d1), acc[t][i1 >> 5], 1);
  }
  acc[NT][i >> 5] = __funnelshift_l(__float_as_uint(y0), acc[NT][i >> 5], 1);
  acc[NT][i1 >> 5] = __funnelshift_l(__float_as_uint(y1), acc[NT][i1 >> 5], 1);
}

template <int NB, int NW>
__device__ __forceinline__ void planes_of(const uint32_t (&r)[1 << (NB - 1)][NW], uint32_t (&pw)[NB][NW]) {
  constexpr int NT = (1 << (NB - 1)) - 1;
#pragma unroll
  for (int w = 0; w < NW; ++w) {
    const uint32_t sy = r[NT][w];
    pw[NB - 1][w] = sy;
    if constexpr (NB == 2) {
      pw[0][w] = r[0][w] ^ sy;
    } else if constexpr (NB == 3) {
      pw[1][w] = r[1][w] ^ sy;
      pw[0][w] = r[0][w] ^ r[1][w] ^ r[2][w] ^ sy;
    } else if constexpr (NB == 4) {
      pw[2][w] = r[3][w] ^ sy;
      pw[1][w] = r[1][w] ^ r[3][w] ^ r[5][w] ^ sy;
      pw[0][w] = r[0][w] ^ r[1][w] ^ r[2][w] ^ r[3][w] ^ r[4][w] ^ r[5][w] ^ r[6][w] ^ sy;
    }
  }
}

// 32 x 32 bit transposes across a warp: on return bit L of lane i's word is
// bit i of lane L's input word.  Stage j (16, 8, 4, 2, 1) swaps j-bit blocks
// between lanes i and i ^ j: the partner's word rotated left by j (lanes
// without bit j) or right by j (lanes with it) brings the wanted block into
// place, and one bitwise select keeps the rest of the lane's own word.
struct WarpTranspose {
  uint32_t keep[5], rot[5];
  __device__ __forceinline__ explicit WarpTranspose(int lane) {
    const uint32_t masks[5] = {0xffff0000u, 0xff00ff00u, 0xf0f0f0f0u, 0xccccccccu, 0xaaaaaaaau};
#pragma unroll
    for (int st = 0; st < 5; ++st) {
      const int j = 16 >> st;
      const bool hi = lane & j;
      keep[st] = hi ? masks[st] : ~masks[st];
      rot[st] = hi ? 32u - j : static_cast<uint32_t>(j);
    }
  }
  __device__ __forceinline__ uint32_t operator()(uint32_t x) const {
#pragma unroll
    for (int st = 0; st < 5; ++st) {
      const uint32_t y = __shfl_xor_sync(TQ_FULL, x, 16 >> st);
      const uint32_t r = __funnelshift_l(y, y, rot[st]);
      x = (x & keep[st]) | (r & ~keep[st]);
    }
    return x;
  }
};

template <int D, int MBK, int BV, bool QJL>
__global__ void __launch_bounds__(128 * tiles_per_unit(D), 1)
    qtile_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                 const __grid_constant__ CUtensorMap tmc, const __grid_constant__ CUtensorMap tms,
                 TileArgs a) {
  constexpr int NBX = D / 64;             // boxes per row (64 bf16 or 32 fp32 table entries)
  constexpr int PK = MBK + (QJL ? 1 : 0);
  constexpr int NW = D / 32;              // words per plane row
  constexpr int HK = 1 << (MBK - 1), HV = 1 << (BV - 1);
  constexpr uint32_t IDESC = sm100::idesc_bf16(128, D);
  constexpr int NTL = tiles_per_unit(D);
  constexpr int QT = 128 * NTL;
  constexpr int TCOLS = 2 * D;            // per tile: A (hi | lo, D/2 columns each) + z (D columns)
  // tensor memory is allocated in powers of two columns
  constexpr int TALLOC = NTL * TCOLS <= 256 ? 256 : 512;
  static_assert(NTL * TCOLS <= 512, "tensor memory budget");
  extern __shared__ uint8_t qsm_raw[];
  uint8_t *qsm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(qsm_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *Xt0 = qsm;                     // the unit's tiles, NBX boxes each
  uint8_t *Ct = Xt0 + NTL * NBX * BOX;
  uint8_t *Snt = Ct + NBX * BOX;
  uint8_t *Bs = Snt + NBX * BOX;
  __shared__ __align__(8) uint64_t full, z_ready;
  __shared__ uint32_t tmem_s;
  __shared__ int abort_s;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t BH = static_cast<int64_t>(a.B) * a.H;
  // this CTA's units [u0, u1): its key units (even u) first, then its value units
  const int64_t u0 = a.nunits * blockIdx.x / gridDim.x;
  const int64_t u1 = a.nunits * (blockIdx.x + 1) / gridDim.x;
  const int64_t k_first = u0 + (u0 & 1), v_first = u0 + 1 - (u0 & 1);
  const int64_t nk = u1 > k_first ? (u1 - k_first + 1) / 2 : 0;
  const int64_t nloc = u1 - u0;
  auto unit_of = [&](int64_t s) { return s < nk ? k_first + 2 * s : v_first + 2 * (s - nk); };

  if (QJL) {
    for (int e = tid; e < D * D; e += QT) {
      const int i = e / D, kb = 2 * (e % D);
      *reinterpret_cast<uint16_t *>(Bs + (kb >> 4) * (D * 16) + (i >> 3) * 128 + (i & 7) * 16 +
                                    (kb & 15)) = a.S[e];
    }
    if (warp == 0) sm100::tmem_alloc(&tmem_s, TALLOC);
  }
  if (tid == 0) {
    sm100::mbar_init(&full, 1);
    sm100::mbar_init(&z_ready, 1);
    abort_s = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  sm100::fence_async_smem();
  sm100::fence_before_sync();
  __syncthreads();
  sm100::fence_after_sync();
  const uint32_t tm = QJL ? tmem_s : 0u;

  // thread 0: the position tile of the RoPE table in shared memory, the
  // last step whose copies were issued and the last sketch commit
  int64_t cur_pt = -1;
  int issued = -1, committed = -1;
  auto issue = [&](int64_t s, int idx) {
    const int64_t u = unit_of(s), q = u >> 1;
    const bool keys = !(u & 1);
    const int64_t pt = q / a.groups, bh0 = (q % a.groups) * NTL;
    const int nt = static_cast<int>(BH - bh0 < NTL ? BH - bh0 : NTL);   // the last group may be short
    const int t0 = static_cast<int>(a.R_first + pt * QR - a.row0);
    const bool table = keys && a.rope && pt != cur_pt;
    sm100::mbar_expect_tx(&full, (nt + (table ? 2 : 0)) * NBX * BOX);
    const CUtensorMap *src = keys ? &tmk : &tmv;
    for (int g = 0; g < nt; ++g) {
      const int64_t bh = bh0 + g;
#pragma unroll
      for (int x = 0; x < NBX; ++x)
        tma_4d(Xt0 + (g * NBX + x) * BOX, src, 64 * x, t0, static_cast<int>(bh % a.H),
               static_cast<int>(bh / a.H), &full);
    }
    if (table) {
      const int p0 = static_cast<int>(a.pos0) + t0;
#pragma unroll
      for (int x = 0; x < NBX; ++x) {
        tma_2d(Ct + x * BOX, &tmc, 32 * x, p0, &full);
        tma_2d(Snt + x * BOX, &tms, 32 * x, p0, &full);
      }
      cur_pt = pt;
    }
    issued = idx;
  };
  if (tid == 0 && nloc > 0) issue(0, 0);
  {
    // ------------------------------------------------ row threads
    const int rl = tid & 127;                 // row of the tile = TMEM lane
    const int wq = warp & 3;
    const int wg = warp >> 2;                 // which tile of the unit
    const uint8_t *Xt = Xt0 + wg * NBX * BOX;
    const uint32_t tmg = tm + wg * TCOLS;
    float thr[8];
    // every thread passes every barrier of a step; a wait that gives up
    // clears ok, and the next barrier makes the whole CTA leave together
    bool ok = true;
    int kz = 0;                               // sketch commits so far
    for (int i = 0; i < nloc; ++i) {
      const int64_t u = unit_of(i), q = u >> 1;
      const bool is_key = !(u & 1);
      const int64_t pt = q / a.groups, bh = (q % a.groups) * NTL + wg;
      const int64_t R = a.R_first + pt * QR + rl;     // cache row
      const int64_t t = R - a.row0;                    // token of the call
      const bool active = t >= 0 && t < a.T && bh < BH;
      if (ok && !wait_or_abort(&full, i & 1, a.wait_outer, &abort_s)) { abort_s = 1; ok = false; }
      // ---- row into registers (+ RoPE for keys); after a give-up the
      // values read are never used
      float x[D];
#pragma unroll
      for (int c = 0; c < D / 8; ++c) {
        const uint4 v = swz_ld(Xt + (c >> 3) * BOX, rl, c & 7);
        const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          x[8 * c + 2 * e] = __uint_as_float(w4[e] << 16);
          x[8 * c + 2 * e + 1] = __uint_as_float(w4[e] & 0xffff0000u);
        }
      }
      if (is_key && a.rope) {
        constexpr int HALF = D / 2;
#pragma unroll
        for (int c = 0; c < HALF / 4; ++c) {
          const uint4 cv = swz_ld(Ct + (c >> 3) * BOX, rl, c & 7);
          const uint4 sv = swz_ld(Snt + (c >> 3) * BOX, rl, c & 7);
          const float cs[4] = {__uint_as_float(cv.x), __uint_as_float(cv.y), __uint_as_float(cv.z),
                               __uint_as_float(cv.w)};
          const float sn[4] = {__uint_as_float(sv.x), __uint_as_float(sv.y), __uint_as_float(sv.z),
                               __uint_as_float(sv.w)};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int j = 4 * c + e;
            const float u = x[j], w = x[j + HALF];
            x[j] = u * cs[e] - w * sn[e];
            x[j + HALF] = w * cs[e] + u * sn[e];
          }
        }
      }
      // every row of the step is in registers: the buffers may be refilled
      if (!(ok = cta_all_ok<QT>(ok))) break;
      if (tid == 0 && i + 1 < nloc) issue(i + 1, i + 1);
      // ---- norm, sign flip, transform
      uint64_t ss2 = 0ull;
#pragma unroll
      for (int j = 0; j < D / 2; ++j) sq2acc(x[j], x[j + D / 2], ss2);
      const float ss = hsum2(ss2);
      float nu = sqrtf(ss);
      bool bad = !(ss <= 3.402823466e38f) || isinf(__half2float(__float2half_rn(nu)));
      if (bad) nu = 0.f;
#pragma unroll
      for (int j = 0; j < D / 2; ++j) mul2c(x[j], x[j + D / 2], pk2(a.dsg[2 * j], a.dsg[2 * j + 1]));
      wht_regs<D>(x);
      if (bad || !(nu > 0.f)) {
#pragma unroll
        for (int j = 0; j < D; ++j) x[j] = 0.f;   // zero row: u = 0 (+0 decides the upper half)
      }
      const float sc = nu > 0.f ? sqrtf(static_cast<float>(D)) * nu : 1.f;
      if (bad && active && a.status) atomicAdd(a.status, 1u);
      if (is_key) {
        // ---------------------------------------------- key row
#pragma unroll
        for (int j = 0; j < HK - 1; ++j) thr[j] = a.tk[j] * sc;
        uint32_t raw[HK][NW];
#pragma unroll
        for (int p = 0; p < HK; ++p)
#pragma unroll
          for (int w = 0; w < NW; ++w) raw[p][w] = 0u;
        uint64_t r2p = 0ull;
        float cks[HK];
#pragma unroll
        for (int m = 0; m < HK; ++m) cks[m] = a.ck[m] * sc;
        uint64_t th2[HK > 1 ? HK - 1 : 1];
#pragma unroll
        for (int j = 0; j < HK - 1; ++j) th2[j] = pk2(thr[j], thr[j]);
        // coordinates j and j + D/2 together (their words take the same bit)
#pragma unroll
        for (int j = D / 2 - 1; j >= 0; --j) {
          constexpr int H2 = D / 2;
          raw_bits2<MBK, NW>(x[j], x[j + H2], th2, raw, j, j + H2);
          if (QJL) {
            // residual (scaled by sc): y - sign(y) c_m = sign(y) (|y| - c_m)
            const float aa0 = fabsf(x[j]), aa1 = fabsf(x[j + H2]);
            float cm0 = cks[0], cm1 = cks[0];
#pragma unroll
            for (int m = 1; m < HK; ++m) {
              cm0 = aa0 >= thr[m - 1] ? cks[m] : cm0;
              cm1 = aa1 >= thr[m - 1] ? cks[m] : cm1;
            }
            float r0, r1;
            sub2c(aa0, aa1, pk2(cm0, cm1), r0, r1);
            sq2acc(r0, r1, r2p);
            x[j] = __uint_as_float(__float_as_uint(r0) ^ (__float_as_uint(x[j]) & 0x80000000u));
            x[j + H2] = __uint_as_float(__float_as_uint(r1) ^ (__float_as_uint(x[j + H2]) & 0x80000000u));
          }
        }
        const float r2 = hsum2(r2p);
        uint32_t pw[MBK][NW];
        planes_of<MBK, NW>(raw, pw);
#pragma unroll
        for (int p = 0; p < MBK; ++p)
#pragma unroll
          for (int w = 0; w < NW; ++w) pw[p][w] = ~pw[p][w];
        float rho = 0.f;
        if (QJL) {
          rho = sqrtf(r2) / sc;
          // tensor memory A: columns [0, D/2) hi, [D/2, D) lo (two bf16 per
          // column, lower K index in the low half); lane = row
#pragma unroll
          for (int c = 0; c < D / 16; ++c) {
            uint32_t h8[8], l8[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const int j = 8 * c + e;
              const __nv_bfloat162 hi = __floats2bfloat162_rn(x[2 * j], x[2 * j + 1]);
              const float2 hf = __bfloat1622float2(hi);
              float l0, l1;
              sub2(x[2 * j], x[2 * j + 1], hf.x, hf.y, l0, l1);
              const __nv_bfloat162 lo = __floats2bfloat162_rn(l0, l1);
              h8[e] = *reinterpret_cast<const uint32_t *>(&hi);
              l8[e] = *reinterpret_cast<const uint32_t *>(&lo);
            }
            sm100::tmem_st8(sm100::tmem_lane(tmg + 8 * c, wq), h8);
            sm100::tmem_st8(sm100::tmem_lane(tmg + D / 2 + 8 * c, wq), l8);
          }
          sm100::wait_st();
        }
        const int64_t crow = bh * a.rows_cap + R;
        if (active) {
          uint8_t *kr = a.kcode + crow * (PK * (D / 8));
#pragma unroll
          for (int p = 0; p < MBK; ++p) {
            if (NW == 2)
              *reinterpret_cast<uint2 *>(kr + p * (D / 8)) = make_uint2(pw[p][0], pw[p][1]);
            else
              *reinterpret_cast<uint4 *>(kr + p * (D / 8)) =
                  make_uint4(pw[p][0], pw[p][1 % NW], pw[p][2 % NW], pw[p][3 % NW]);
          }
          reinterpret_cast<uint32_t *>(a.kscale)[crow] =
              static_cast<uint32_t>(tq_f32_to_half(nu)) | (static_cast<uint32_t>(tq_f32_to_half(rho)) << 16);
        }
        if (QJL) {
          // every tile's operand is stored: thread 0 issues their sketches
          if (!(ok = cta_all_ok<QT>(ok))) break;
          if (tid == 0) {
#pragma unroll
            for (int g = 0; g < NTL; ++g) {
              const uint32_t tg = tm + g * TCOLS;
#pragma unroll
              for (int s = 0; s < D / 16; ++s)
                sm100::mma_f16_ts(tg + D, tg + 8 * s,
                                  sm100::smem_desc(sm100::smem_addr(Bs) + s * 2 * D * 16, D * 16, 128),
                                  IDESC, s > 0);
#pragma unroll
              for (int s = 0; s < D / 16; ++s)
                sm100::mma_f16_ts(tg + D, tg + D / 2 + 8 * s,
                                  sm100::smem_desc(sm100::smem_addr(Bs) + s * 2 * D * 16, D * 16, 128),
                                  IDESC, 1);
            }
            sm100::mma_commit(&z_ready);
            committed = kz;
          }
          if (!wait_or_abort(&z_ready, (kz++) & 1, a.wait_outer, &abort_s)) {
            abort_s = 1;
            ok = false;
            continue;   // the next step's first barrier takes the CTA out
          }
          sm100::fence_after_sync();
          uint32_t sg[NW];
#pragma unroll
          for (int w = 0; w < NW; ++w) {
            uint32_t z[32];
            sm100::tmem_ld32(sm100::tmem_lane(tmg + D + 32 * w, wq), z);
            sm100::wait_ld();
            uint32_t acc = 0u;
#pragma unroll
            for (int e = 31; e >= 0; --e) acc = __funnelshift_l(z[e], acc, 1);
            sg[w] = ~acc;                  // bit e = [z >= 0]
          }
          if (active) {
            uint8_t *kr = a.kcode + crow * (PK * (D / 8)) + MBK * (D / 8);
            if (NW == 2)
              *reinterpret_cast<uint2 *>(kr) = make_uint2(sg[0], sg[1]);
            else
              *reinterpret_cast<uint4 *>(kr) = make_uint4(sg[0], sg[1 % NW], sg[2 % NW], sg[3 % NW]);
          }
        }
      } else {
        // ---------------------------------------------- value row
#pragma unroll
        for (int j = 0; j < HV - 1; ++j) thr[j] = a.tv[j] * sc;
        uint32_t pw[BV][NW];
#pragma unroll
        for (int p = 0; p < BV; ++p)
#pragma unroll
          for (int w = 0; w < NW; ++w) pw[p][w] = 0u;
        uint64_t th2[HV > 1 ? HV - 1 : 1];
#pragma unroll
        for (int j = 0; j < HV - 1; ++j) th2[j] = pk2(thr[j], thr[j]);
        if constexpr (BV < 3) {
#pragma unroll
          for (int j = D / 2 - 1; j >= 0; --j) {
            constexpr int H2 = D / 2;
            uint32_t ms0[4], ms1[4];
            plane_msbs2<BV>(x[j], x[j + H2], th2, ms0, ms1);
#pragma unroll
            for (int p = 0; p < BV; ++p) {
              pw[p][j >> 5] = __funnelshift_l(ms0[p], pw[p][j >> 5], 1);
              pw[p][(j + H2) >> 5] = __funnelshift_l(ms1[p], pw[p][(j + H2) >> 5], 1);
            }
          }
        } else {
          // the planes below the top one without their sign term (the
          // thermometer XORs of plane_msbs with sy left out) and the sign
          // word beside them; the sign goes into the lower planes once per word
          uint32_t syw[NW];
#pragma unroll
          for (int w = 0; w < NW; ++w) syw[w] = 0u;
#pragma unroll
          for (int j = D / 2 - 1; j >= 0; --j) {
            constexpr int H2 = D / 2;
            uint32_t ms0[4], ms1[4];
            therm_msbs2<BV>(fabsf(x[j]), fabsf(x[j + H2]), th2, ms0, ms1);
#pragma unroll
            for (int p = 0; p < BV - 1; ++p) {
              pw[p][j >> 5] = __funnelshift_l(ms0[p], pw[p][j >> 5], 1);
              pw[p][(j + H2) >> 5] = __funnelshift_l(ms1[p], pw[p][(j + H2) >> 5], 1);
            }
            syw[j >> 5] = __funnelshift_l(__float_as_uint(x[j]), syw[j >> 5], 1);
            syw[(j + H2) >> 5] = __funnelshift_l(__float_as_uint(x[j + H2]), syw[(j + H2) >> 5], 1);
          }
#pragma unroll
          for (int w = 0; w < NW; ++w) {
#pragma unroll
            for (int p = 0; p < BV - 1; ++p) pw[p][w] ^= syw[w];
            pw[BV - 1][w] = syw[w];
          }
        }
        const int64_t crow = bh * a.rows_cap + R;
        if (active) a.vnorm[crow] = tq_f32_to_half(nu);
        // column words: lane i gets coordinate 32 w + i of the warp's 32 rows
        const uint32_t act = __ballot_sync(TQ_FULL, active);
        uint32_t *vg = a.vcode + (bh * (a.rows_cap / 32) + (R >> 5)) * (BV * D);
        const WarpTranspose tp(lane);
#pragma unroll
        for (int p = 0; p < BV; ++p) {
#pragma unroll
          for (int w = 0; w < NW; ++w) {
            const uint32_t col = tp(~pw[p][w]);
            uint32_t *dst = vg + p * D + 32 * w + lane;
            if (act == TQ_FULL) {
              *dst = col;
            } else if (act) {
              atomicAnd(dst, ~act);
              atomicOr(dst, col & act);
            }
          }
        }
      }
    }
  }
  if (tid == 0 && abort_s) {
    // this CTA's own copies and MMAs land before its memory is released
    if (issued >= 0) sm100::mbar_wait(&full, issued & 1, 1u << 20);
    if (committed >= 0) sm100::mbar_wait(&z_ready, committed & 1, 1u << 20);
  }
  sm100::fence_before_sync();
  __syncthreads();
  sm100::fence_after_sync();
  if (abort_s && tid == 0 && a.status) atomicOr(a.status, 1u << 31);
  if (QJL && warp == 0) sm100::tmem_dealloc(tm, TALLOC);
}

// ---------------------------------------------------------------- host side

using EncodeFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                              const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                              const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                              CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn encode_fn() {
  static EncodeFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeFn>(p);
  }
  return fn;
}

template <int D, int MBK, int BV, bool QJL>
int run_tile(const TileArgs &a, const CUtensorMap &mk, const CUtensorMap &mv, const CUtensorMap &mc,
             const CUtensorMap &ms, cudaStream_t stream) {
  constexpr int NTL = tiles_per_unit(D);
  // the unit's X tiles, the RoPE table tiles and S
  constexpr size_t shm = 1024 + (NTL + 2) * (D / 64) * BOX + (QJL ? static_cast<size_t>(D) * D * 2 : 0);
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  static bool done[64] = {};
  if (dev < 64 && !done[dev]) {
    if (cudaFuncSetAttribute(qtile_kernel<D, MBK, BV, QJL>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(shm)) != cudaSuccess)
      return tq_check_launch("cudaFuncSetAttribute(qtile)");
    done[dev] = true;
  }
  // one CTA per SM (its tensor memory takes all 512 columns)
  const int grid = static_cast<int>(a.nunits < sms ? a.nunits : sms);
  qtile_kernel<D, MBK, BV, QJL><<<grid, 128 * NTL, shm, stream>>>(mk, mv, mc, ms, a);
  tq_count_launch(1);
  return tq_check_launch("qtile_kernel");
}

bool make_map(CUtensorMap *m, CUtensorMapDataType dt, int rank, void *base, const cuuint64_t *dims,
              const cuuint64_t *strides_bytes, const cuuint32_t *box) {
  EncodeFn fn = encode_fn();
  if (!fn) return false;
  const cuuint32_t es[4] = {1, 1, 1, 1};
  return fn(m, dt, rank, base, dims, strides_bytes, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

// Returns TQ_ERR_UNSUPPORTED (without launching) when the call does not fit
// this kernel's layout rules; the caller then takes another kernel.
int launch_quantize_tile(const tq_codec *c, const void *k, const void *v, int dtype, int B, int H,
                         int T, int64_t sb, int64_t sh, int64_t st, const float *rc,
                         const float *rs, int64_t pos0, const tq_cache *cache, int64_t row0,
                         uint32_t *status, cudaStream_t stream) {
  if (getenv("TQ_QUANT_IMPL")) return TQ_ERR_UNSUPPORTED;   // explicit kernel choice
  if (dtype != TQ_BF16 || (c->d != 64 && c->d != 128) || T <= 0) return TQ_ERR_UNSUPPORTED;
  const int d = c->d;
  const int mbk = c->mse_bits_k, bv = c->bits_v;
  if (mbk < 1 || mbk > 4 || bv < 1 || bv > 4) return TQ_ERR_UNSUPPORTED;
  auto al16 = [](int64_t x) { return (x * 2) % 16 == 0; };
  if (!al16(sb) || !al16(sh) || !al16(st) || (reinterpret_cast<uintptr_t>(k) % 16) ||
      (reinterpret_cast<uintptr_t>(v) % 16))
    return TQ_ERR_UNSUPPORTED;
  if ((rc != nullptr) && ((reinterpret_cast<uintptr_t>(rc) % 16) || (reinterpret_cast<uintptr_t>(rs) % 16)))
    return TQ_ERR_UNSUPPORTED;
  if (pos0 + T > (int64_t(1) << 30) || row0 + T > (int64_t(1) << 30)) return TQ_ERR_UNSUPPORTED;
  TileArgs a;
  a.B = B;
  a.H = H;
  a.T = T;
  a.row0 = row0;
  a.pos0 = pos0;
  a.rows_cap = cache->rows_cap;
  a.R_first = row0 / QR * QR;
  a.nrt = (row0 + T - 1) / QR - row0 / QR + 1;
  const int ntl = tiles_per_unit(d);
  a.groups = (static_cast<int64_t>(B) * H + ntl - 1) / ntl;
  a.nunits = 2 * a.nrt * a.groups;
  a.kcode = cache->kcode;
  a.kscale = cache->kscale;
  a.vcode = cache->vcode;
  a.vnorm = cache->vnorm;
  a.status = status;
  a.S = c->S_dev;
  a.wait_outer = 4096;
  if (const char *e = getenv("TQ_WAIT_LIMIT")) a.wait_outer = static_cast<uint32_t>(strtoul(e, nullptr, 10) >> 14);
  a.rope = rc != nullptr;
  const int hk = 1 << (mbk - 1), hv = 1 << (bv - 1);
  for (int m = 0; m < 8; ++m) {
    a.ck[m] = m < hk ? c->books.ck[hk + m] : 0.f;
    a.tk[m] = m < hk - 1 ? c->books.tk[hk + m] : 0.f;
    a.tv[m] = m < hv - 1 ? c->books.tv[hv + m] : 0.f;
  }
  for (int j = 0; j < 64; ++j) {
    const auto sgn = [&](int i) { return i < d && ((c->books.dneg[i >> 5] >> (i & 31)) & 1u) ? -1.f : 1.f; };
    a.dsg[2 * j] = sgn(j);
    a.dsg[2 * j + 1] = sgn(j + d / 2);
  }
  // tensor maps: K and V [B][H][T][d] bf16 (4-D, innermost d); RoPE tables [pos0 + T][d/2] fp32
  CUtensorMap mk, mv, mc, ms;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(T),
                              static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(B)};
  const cuuint64_t str[3] = {static_cast<cuuint64_t>(st * 2), static_cast<cuuint64_t>(sh * 2),
                             static_cast<cuuint64_t>(sb * 2)};
  const cuuint32_t box[4] = {64, QR, 1, 1};
  if (!make_map(&mk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(k), dims, str, box) ||
      !make_map(&mv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(v), dims, str, box))
    return TQ_ERR_UNSUPPORTED;
  if (a.rope) {
    const cuuint64_t tdims[2] = {static_cast<cuuint64_t>(d / 2), static_cast<cuuint64_t>(pos0 + T)};
    const cuuint64_t tstr[1] = {static_cast<cuuint64_t>(d / 2 * 4)};
    const cuuint32_t tbox[2] = {32, QR};
    if (!make_map(&mc, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float *>(rc), tdims, tstr, tbox) ||
        !make_map(&ms, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float *>(rs), tdims, tstr, tbox))
      return TQ_ERR_UNSUPPORTED;
  } else {
    mc = mk;   // unused
    ms = mk;
  }
  const int key = d * 1000 + mbk * 100 + bv * 10 + c->qjl_k;
  switch (key) {
    case 64231: return run_tile<64, 2, 3, true>(a, mk, mv, mc, ms, stream);
    case 128341: return run_tile<128, 3, 4, true>(a, mk, mv, mc, ms, stream);
    case 128121: return run_tile<128, 1, 2, true>(a, mk, mv, mc, ms, stream);
    case 128231: return run_tile<128, 2, 3, true>(a, mk, mv, mc, ms, stream);
    case 64331: return run_tile<64, 3, 3, true>(a, mk, mv, mc, ms, stream);
    case 128440: return run_tile<128, 4, 4, false>(a, mk, mv, mc, ms, stream);
    case 128330: return run_tile<128, 3, 3, false>(a, mk, mv, mc, ms, stream);
    case 64330: return run_tile<64, 3, 3, false>(a, mk, mv, mc, ms, stream);
    default: return TQ_ERR_UNSUPPORTED;
  }
}
