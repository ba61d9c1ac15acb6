// Prefill quantize for codecs with a dense rotation: the rotation of a tile of
// 128 rows is one tensor-core product.
//
// Sources: "Google presenta TurboQuant ..." ("La mecanica geometrica de
// TurboQuant": one shared random rotation, then per-coordinate Lloyd-Max
// codes; "Eliminacion del sesgo": b-1 MSE bits plus the 1-bit QJL sketch of
// the residual); "FibQuant ..." section 2.1 (Haar rotation) and 2.3 (store nu,
// rotate x / nu, quantize); "TurboESM ..." section 2.A (RoPE first).
//
// One tile = 4 token groups of 32 rows (each of one (batch, head)).  Warps 0-3
// own the key rows of groups 0-3, warps 4-7 the value rows (thread = row, so a
// warp's rows sit in its own quarter of the tensor-memory lanes); thread 0
// issues the MMAs.
//   1. Each thread loads its row (RoPE for keys), takes nu and writes
//      64 x / nu split into fp16 hi + lo into the tile's A operand in shared
//      memory (K-major core matrices).
//   2. U = [x_hi | x_lo] [16 Pi_hi ; 16 Pi_hi]^T + x_hi (16 Pi_lo)^T, fp32 in
//      tensor memory (Pi = 16 Pi_hi + 16 Pi_lo exactly up to 2^-22 relative;
//      the x_lo Pi_lo term is below fp32 rounding), u = U / 1024.
//   3. Each thread reads its row of u back, 32 coordinates at a time: codes by
//      the threshold search, key plane words directly (thread = row), the key
//      residual (bf16 hi + lo) into the A operand of the sketch, value plane
//      words across the 32 tokens of a group by warp ballots.
//   4. The sketch z = S r of the key rows is one more product (S exactly bf16);
//      each key thread reads its row of z and writes the sign plane.
// Every wait is bounded; a give-up is reported in bit 31 of the status word.
#include "tq_device.cuh"
#include "tq_sm100.cuh"

namespace {

constexpr int RT = 256;   // 8 row warps; thread 0 also issues the MMAs

struct RotArgs {
  const void *k, *v;
  int dtype;
  int B, H, T;
  int64_t sb, sh, st;
  const float *rc, *rs;
  int64_t pos0;
  uint8_t *kcode;
  uint16_t *kscale;
  uint32_t *vcode;
  uint16_t *vnorm;
  int64_t rows_cap, row0, g_first, n_groups;
  uint32_t *status;
  const uint16_t *S;
  TqBooks books;
};

template <int D>
constexpr uint32_t rot_smem_bytes(bool qjl) {
  return 2u * 128u * (2 * D) * 2u + 2u * D * D * 2u + (qjl ? D * D * 2u : 0u);
}

// byte offset of element e (16-bit) of row m in a 128-row K-major A operand
__device__ __forceinline__ uint32_t a_off(int m, int e) {
  return static_cast<uint32_t>((e >> 3) * 2048 + (m >> 3) * 128 + (m & 7) * 16 + (e & 7) * 2);
}

// byte offset of element (n, k) (16-bit) in a D x D K-major B operand
template <int D>
__device__ __forceinline__ uint32_t b_off(int n, int k) {
  return static_cast<uint32_t>((k >> 3) * (D * 16) + (n >> 3) * 128 + (n & 7) * 16 + (k & 7) * 2);
}

__device__ __forceinline__ uint32_t pack_h2(float a, float b) {
  const __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<const uint32_t *>(&h);
}

template <int D, bool QJL>
__global__ void __launch_bounds__(RT, D == 64 ? 2 : 1) qrot_kernel(RotArgs a) {
  constexpr int KE = 2 * D;                       // K elements of the rotation product
  constexpr uint32_t A_BYTES = 128u * KE * 2u;
  constexpr uint32_t B_BYTES = static_cast<uint32_t>(D) * D * 2u;
  constexpr uint32_t IDESC_R = sm100::idesc_f16(128, D);
  constexpr uint32_t IDESC_S = sm100::idesc_bf16(128, D);
  constexpr int TCOLS = 3 * D <= 256 ? 256 : 512;   // U_k | U_v | z
  constexpr int NC = D / 32;                         // 32-coordinate chunks of a row
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t *Ak = smem;
  uint8_t *Av = Ak + A_BYTES;
  uint8_t *Bh = Av + A_BYTES;
  uint8_t *Bl = Bh + B_BYTES;
  uint8_t *Bs = Bl + B_BYTES;
  __shared__ float cks[TQ_MAX_LEVELS], tks[TQ_MAX_LEVELS], tvs[TQ_MAX_LEVELS];
  __shared__ __align__(8) uint64_t mb_rot, mb_sk;
  __shared__ uint32_t tmem_s;
  __shared__ int abort_s;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid < TQ_MAX_LEVELS) {
    cks[tid] = a.books.ck[tid];
    tks[tid] = a.books.tk[tid];
    tvs[tid] = a.books.tv[tid];
  }
  // B operands: 16 Pi split into fp16 hi + lo, S (bf16, exact)
  for (int e = tid; e < D * D; e += RT) {
    const int n = e / D, kx = e % D;
    const float p = 16.0f * a.books.pi[e];            // Pi[n][kx], row-major
    const __half hi = __float2half_rn(p);
    const __half lo = __float2half_rn(p - __half2float(hi));
    *reinterpret_cast<__half *>(Bh + b_off<D>(n, kx)) = hi;
    *reinterpret_cast<__half *>(Bl + b_off<D>(n, kx)) = lo;
    if (QJL) *reinterpret_cast<uint16_t *>(Bs + b_off<D>(n, kx)) = a.S[e];
  }
  if (warp == 0) sm100::tmem_alloc(&tmem_s, TCOLS);
  if (tid == 0) {
    sm100::mbar_init(&mb_rot, 1);
    sm100::mbar_init(&mb_sk, 1);
    abort_s = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  sm100::fence_async_smem();
  sm100::fence_before_sync();
  __syncthreads();
  sm100::fence_after_sync();
  const uint32_t tm = tmem_s;
  const uint32_t ak = sm100::smem_addr(Ak), av = sm100::smem_addr(Av);
  const uint32_t bh = sm100::smem_addr(Bh), bl = sm100::smem_addr(Bl), bs = sm100::smem_addr(Bs);
  const int mbk = a.books.mse_bits_k, bv = a.books.bits_v;
  const int planes_k = mbk + (QJL ? 1 : 0);
  const int64_t items = static_cast<int64_t>(a.B) * a.H * a.n_groups;
  const int64_t tiles = (items + 3) / 4;
  uint32_t ph_rot = 0, ph_sk = 0;
  uint32_t n_rot = 0, n_sk = 0;          // commits issued (thread 0)
  const bool is_key = warp < 4, is_row = true;
  const int q = warp & 3;               // group of the tile = tensor-memory lane quarter
  const int m = 32 * q + lane;          // row of the tile

  for (int64_t tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
    // ------------------------------------------------ 1. rows into the A operands
    int64_t g = 0, cbh = 0, r = 0;
    int b = 0, h = 0;
    bool valid = false;
    float nu = 0.f;
    bool bad = false;
    uint32_t gmask = 0u;             // rows of this group the call covers
    if (is_row) {
      const int64_t it = tile * 4 + q;
      if (it < items) {
        g = a.g_first + it % a.n_groups;
        const int64_t bhi = it / a.n_groups;
        b = static_cast<int>(bhi / a.H);
        h = static_cast<int>(bhi % a.H);
        cbh = static_cast<int64_t>(b) * a.H + h;
        const int64_t rb = max(a.row0, g * 32), re = min(a.row0 + a.T, g * 32 + 32);
        r = g * 32 + lane;
        valid = r >= rb && r < re;
        const uint32_t nrows = static_cast<uint32_t>(re - rb);
        gmask = nrows >= 32 ? TQ_FULL : (((1u << nrows) - 1u) << (rb & 31));
      }
      float x[D];
      if (valid) {
        const int64_t t = r - a.row0;
        const int64_t off = b * a.sb + h * a.sh + t * a.st;
        const void *src = is_key ? a.k : a.v;
        const size_t es = a.dtype == TQ_BF16 ? 2 : 4;
        const bool vec = (reinterpret_cast<uintptr_t>(static_cast<const uint8_t *>(src) + off * es) & 15) == 0;
        if (a.dtype == TQ_BF16 && vec) {
          const uint4 *p = reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(src) + off);
#pragma unroll
          for (int c = 0; c < D / 8; ++c) {
            const uint4 w = p[c];
            const uint32_t wd[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              x[8 * c + 2 * e] = __uint_as_float(wd[e] << 16);
              x[8 * c + 2 * e + 1] = __uint_as_float(wd[e] & 0xffff0000u);
            }
          }
        } else if (a.dtype == TQ_F32 && vec) {
          const float4 *p = reinterpret_cast<const float4 *>(static_cast<const float *>(src) + off);
#pragma unroll
          for (int c = 0; c < D / 4; ++c) {
            const float4 w = p[c];
            x[4 * c] = w.x;
            x[4 * c + 1] = w.y;
            x[4 * c + 2] = w.z;
            x[4 * c + 3] = w.w;
          }
        } else {
#pragma unroll
          for (int i = 0; i < D; ++i) x[i] = tq_load_elem(src, off + i, a.dtype);
        }
        if (is_key && a.rc != nullptr) {
          // rotate-half RoPE at position pos0 + t
          const float *pc = a.rc + (a.pos0 + t) * (D / 2), *ps = a.rs + (a.pos0 + t) * (D / 2);
          const bool tv = ((reinterpret_cast<uintptr_t>(pc) | reinterpret_cast<uintptr_t>(ps)) & 15) == 0;
#pragma unroll
          for (int c4 = 0; c4 < D / 8; ++c4) {
            float cc[4], sn[4];
            if (tv) {
              const float4 cv = reinterpret_cast<const float4 *>(pc)[c4];
              const float4 sv = reinterpret_cast<const float4 *>(ps)[c4];
              cc[0] = cv.x, cc[1] = cv.y, cc[2] = cv.z, cc[3] = cv.w;
              sn[0] = sv.x, sn[1] = sv.y, sn[2] = sv.z, sn[3] = sv.w;
            } else {
#pragma unroll
              for (int e = 0; e < 4; ++e) cc[e] = pc[4 * c4 + e], sn[e] = ps[4 * c4 + e];
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int i = 4 * c4 + e;
              const float u = x[i], w = x[i + D / 2];
              x[i] = u * cc[e] - w * sn[e];
              x[i + D / 2] = w * cc[e] + u * sn[e];
            }
          }
        }
        bool finite = true;
        float ss = 0.f;
#pragma unroll
        for (int i = 0; i < D; ++i) {
          finite &= isfinite(x[i]);
          ss += x[i] * x[i];
        }
        nu = sqrtf(ss);
        bad = !finite || isinf(__half2float(__float2half_rn(nu)));
        if (bad) nu = 0.f;
      }
      const float inv = nu > 0.f ? 64.0f / nu : 0.f;
      uint8_t *A = is_key ? Ak : Av;
#pragma unroll
      for (int c = 0; c < D / 8; ++c) {
        uint32_t hw[4], lw[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float v0 = valid && !bad ? x[8 * c + 2 * e] * inv : 0.f;
          const float v1 = valid && !bad ? x[8 * c + 2 * e + 1] * inv : 0.f;
          const __half h0 = __float2half_rn(v0), h1 = __float2half_rn(v1);
          hw[e] = pack_h2(__half2float(h0), __half2float(h1));
          lw[e] = pack_h2(v0 - __half2float(h0), v1 - __half2float(h1));
        }
        *reinterpret_cast<uint4 *>(A + a_off(m, 8 * c)) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
        *reinterpret_cast<uint4 *>(A + a_off(m, D + 8 * c)) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
      }
    }
    sm100::fence_async_smem();
    sm100::fence_before_sync();
    __syncthreads();
    sm100::fence_after_sync();
    // ------------------------------------------------ 2. the rotation products
    if (tid == 0) {
#pragma unroll 1
      for (int part = 0; part < 2; ++part) {
        const uint32_t aa = part == 0 ? ak : av, dcol = tm + part * D;
        for (int s = 0; s < KE / 16; ++s) {
          const int kk = (16 * s) % D;
          sm100::mma_bf16_ss(dcol, sm100::smem_desc(aa + s * 2 * 2048, 2048, 128),
                             sm100::smem_desc(bh + (kk / 8) * (D * 16), D * 16, 128), IDESC_R, s > 0);
        }
        for (int s = 0; s < D / 16; ++s)
          sm100::mma_bf16_ss(dcol, sm100::smem_desc(aa + s * 2 * 2048, 2048, 128),
                             sm100::smem_desc(bl + (16 * s / 8) * (D * 16), D * 16, 128), IDESC_R, 1);
      }
      sm100::mma_commit(&mb_rot);
      ++n_rot;
    }
    // the give-up decision is taken per warp, so the ballots below never diverge
    bool go = false;
    if (is_row) {
      go = __all_sync(TQ_FULL, sm100::mbar_wait(&mb_rot, ph_rot));
      if (!go && lane == 0) abort_s = 1;
    }
    ph_rot ^= 1;
    sm100::fence_after_sync();
    // ------------------------------------------------ 3. codes, planes, residual
    if (go) {
      const uint32_t ucol = tm + (is_key ? 0 : D);
      float r2 = 0.f;
      uint32_t kw[4][NC];
#pragma unroll
      for (int c = 0; c < NC; ++c) {
        uint32_t raw[32];
        sm100::tmem_ld32(sm100::tmem_lane(ucol + 32 * c, q), raw);
        sm100::wait_ld();
        if (is_key) {
#pragma unroll
          for (int p = 0; p < 4; ++p) kw[p][c] = 0u;
#pragma unroll
          for (int c8 = 0; c8 < 4; ++c8) {
            uint32_t hw[4], lw[4];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const int t = 8 * c8 + e;
              const float u = __uint_as_float(raw[t]) * (1.0f / 1024.0f);
              const int code = tq_code<4>(u, tks);
#pragma unroll
              for (int p = 0; p < 4; ++p) kw[p][c] |= static_cast<uint32_t>((code >> p) & 1) << t;
              if (QJL) {
                // residual r = u - c[idx] as bf16 hi + lo into the sketch's A operand
                const float rr = u - cks[code];
                r2 += rr * rr;
                const __nv_bfloat16 hh = __float2bfloat16_rn(rr);
                const __nv_bfloat16 ll = __float2bfloat16_rn(rr - __bfloat162float(hh));
                const uint32_t hb = __bfloat16_as_ushort(hh), lb = __bfloat16_as_ushort(ll);
                if (e & 1) {
                  hw[e >> 1] |= hb << 16;
                  lw[e >> 1] |= lb << 16;
                } else {
                  hw[e >> 1] = hb;
                  lw[e >> 1] = lb;
                }
              }
            }
            if (QJL) {
              const int e0 = 32 * c + 8 * c8;
              *reinterpret_cast<uint4 *>(Ak + a_off(m, e0)) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
              *reinterpret_cast<uint4 *>(Ak + a_off(m, D + e0)) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
            }
          }
        } else {
          // value words across the 32 tokens of the group: lane t keeps
          // coordinate 32 c + t of every plane
          uint32_t vw[4] = {0u, 0u, 0u, 0u};
#pragma unroll
          for (int t = 0; t < 32; ++t) {
            const int code = tq_code<4>(__uint_as_float(raw[t]) * (1.0f / 1024.0f), tvs);
#pragma unroll
            for (int p = 0; p < 4; ++p) {
              const uint32_t w = __ballot_sync(TQ_FULL, valid && ((code >> p) & 1));
              if (lane == t) vw[p] = w;
            }
          }
          if (gmask != 0u) {
            uint32_t *vg = a.vcode + (cbh * (a.rows_cap / 32) + g) * bv * D + 32 * c + lane;
#pragma unroll
            for (int p = 0; p < 4; ++p) {
              if (p >= bv) break;
              if (gmask == TQ_FULL) {
                vg[p * D] = vw[p];
              } else {
                atomicAnd(vg + p * D, ~gmask);
                atomicOr(vg + p * D, vw[p] & gmask);
              }
            }
          }
        }
      }
      if (valid) {
        if (is_key) {
          uint32_t *krow = reinterpret_cast<uint32_t *>(a.kcode + (cbh * a.rows_cap + r) * planes_k * (D / 8));
#pragma unroll
          for (int p = 0; p < 4; ++p) {
            if (p >= mbk) break;
#pragma unroll
            for (int c = 0; c < NC; ++c) krow[p * NC + c] = kw[p][c];
          }
          if (!QJL) a.kscale[2 * (cbh * a.rows_cap + r) + 1] = 0;
          a.kscale[2 * (cbh * a.rows_cap + r)] = tq_f32_to_half(nu);
          if (QJL) a.kscale[2 * (cbh * a.rows_cap + r) + 1] = tq_f32_to_half(sqrtf(r2));
        } else {
          a.vnorm[cbh * a.rows_cap + r] = tq_f32_to_half(nu);
        }
        if (bad && a.status) atomicAdd(a.status, 1u);
      }
    }
    if (QJL) {
      // ---------------------------------------------- 4. the sketch of the key rows
      sm100::fence_async_smem();
      sm100::fence_before_sync();
      __syncthreads();
      sm100::fence_after_sync();
      const bool run = !abort_s;        // uniform: read after the barrier
      if (tid == 0 && run) {
        for (int s = 0; s < KE / 16; ++s) {
          const int kk = (16 * s) % D;
          sm100::mma_bf16_ss(tm + 2 * D, sm100::smem_desc(ak + s * 2 * 2048, 2048, 128),
                             sm100::smem_desc(bs + (kk / 8) * (D * 16), D * 16, 128), IDESC_S, s > 0);
        }
        sm100::mma_commit(&mb_sk);
        ++n_sk;
      }
      bool zok = false;
      if (is_key && run) {
        zok = __all_sync(TQ_FULL, sm100::mbar_wait(&mb_sk, ph_sk));
        if (!zok && lane == 0) abort_s = 1;
      }
      if (run) ph_sk ^= 1;
      sm100::fence_after_sync();
      if (zok) {
        uint32_t sw[NC];
#pragma unroll
        for (int c = 0; c < NC; ++c) {
          uint32_t z[32];
          sm100::tmem_ld32(sm100::tmem_lane(tm + 2 * D + 32 * c, q), z);
          sm100::wait_ld();
          uint32_t w = 0u;
#pragma unroll
          for (int t = 0; t < 32; ++t) w |= (__uint_as_float(z[t]) >= 0.f ? 1u : 0u) << t;
          sw[c] = w;
        }
        if (valid) {
          uint32_t *srow = reinterpret_cast<uint32_t *>(a.kcode + (cbh * a.rows_cap + r) * planes_k * (D / 8) +
                                                        mbk * (D / 8));
#pragma unroll
          for (int c = 0; c < NC; ++c) srow[c] = sw[c];
        }
      }
    }
    sm100::fence_before_sync();
    __syncthreads();
    sm100::fence_after_sync();
    if (abort_s) break;
  }
  if (abort_s) {
    // let this CTA's own MMAs land before its memory is released: wait for
    // the phase of each barrier's last commit
    if (tid == 0) {
      if (n_rot) sm100::mbar_wait(&mb_rot, (n_rot - 1) & 1, 1u << 20);
      if (n_sk) sm100::mbar_wait(&mb_sk, (n_sk - 1) & 1, 1u << 20);
    }
    if (tid == 0 && a.status) atomicOr(a.status, 1u << 31);
  }
  sm100::fence_before_sync();
  __syncthreads();
  sm100::fence_after_sync();
  if (warp == 0) sm100::tmem_dealloc(tm, TCOLS);
}

template <int D, bool QJL>
int run_qrot(const RotArgs &a, cudaStream_t stream) {
  constexpr uint32_t shm = rot_smem_bytes<D>(QJL);
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  static bool done[64] = {};
  if (dev < 64 && !done[dev]) {
    if (cudaFuncSetAttribute(qrot_kernel<D, QJL>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(shm)) != cudaSuccess)
      return tq_check_launch("cudaFuncSetAttribute(qrot)");
    done[dev] = true;
  }
  const int64_t items = static_cast<int64_t>(a.B) * a.H * a.n_groups;
  const int64_t tiles = (items + 3) / 4;
  const int64_t cap = static_cast<int64_t>(sms) * (D == 64 ? 2 : 1);   // resident CTAs
  const int grid = static_cast<int>(tiles < cap ? tiles : cap);
  qrot_kernel<D, QJL><<<grid, RT, shm, stream>>>(a);
  tq_count_launch(1);
  return tq_check_launch("qrot_kernel");
}

}  // namespace

int launch_quantize_rot(const tq_codec *c, const void *k, const void *v, int dtype, int B, int H,
                        int T, int64_t sb, int64_t sh, int64_t st, const float *rc,
                        const float *rs, int64_t pos0, const tq_cache *cache, int64_t row0,
                        uint32_t *status, cudaStream_t stream) {
  if (c->books.pi == nullptr || (c->d != 64 && c->d != 128)) return TQ_ERR_UNSUPPORTED;
  RotArgs a;
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
  a.g_first = row0 / 32;
  a.n_groups = (row0 + T - 1) / 32 - row0 / 32 + 1;
  a.status = status;
  a.S = c->S_dev;
  a.books = c->books;
  if (c->d == 64) return c->qjl_k ? run_qrot<64, true>(a, stream) : run_qrot<64, false>(a, stream);
  return c->qjl_k ? run_qrot<128, true>(a, stream) : run_qrot<128, false>(a, stream);
}
