// append_tc.cu -- the append with a tensor-core prefilter for the centroid
// search (head_dim 128, C a multiple of 16, C <= 512).
//
// The codes written are exactly those of the canonical fp32 definition in
// append.cu (QSAC shortlist by (D_i, i), QSAC score, INT2 groups, PSAC INT8);
// only the search for candidates changes:
//
//   D_i = A_t + d_i,  d_i = B_i - 2 X_ti,  A_t = sum_j s_j k_j^2,
//   B_i = sum_j s_j c_ij^2,  X_ti = sum_j (s_j k_tj) c_ij      (s = 1 for Values)
//
// The tensor cores compute the approximation d~_i for all C centroids at once
// (s*k split into bf16 hi + lo, centroid rows as -2c in bf16, plus one K step
// adding B_i as bf16 hi + lo) into TMEM.  With a bound E >= |d~_i - d_i|
// (representation 2^-17 and fp32-accumulation error, Cauchy-Schwarz:
// sum |s k c| <= sqrt(A_t B_i)) and the canonical fold's relative error
// gamma, every index of the exact top-M must satisfy d~_i <= theta (derived
// below); those survivors, usually about M, are rescored with the canonical fp32
// fold and ranked by (D, i).  A token with more than SURV_MAX survivors is
// rescored over all C centroids.
//
// One CTA per (head, NT tokens), NT threads: thread t owns token t and a TMEM
// lane; the token rows sit in shared memory (16-byte aligned, conflict-free
// rows).  NT = 256 when C <= 256 (two 128-row MMA halves share one centroid
// tile; each half writes its own TMEM column range, token t in lane t % 128),
// else 128.  Thread 0 issues the MMAs.  The
// candidate threshold comes from the M-th smallest minimum over groups of 8
// centroids, and survivors are rescored in pairs.
// After the MMAs the -2c tile stays in shared memory and serves as the
// centroid table for the exact passes (c = -0.5 * (-2c) is exact), so that the
// rescoring, the QSAC score, the INT2 codes and the PSAC coefficients read
// centroid rows from shared memory (from global memory only when C exceeds
// one 256-row tile).  Phases are separated by __syncthreads; the single
// mbarrier wait is bounded.
//
// This file is compiled with --fmad=false; all fused multiply-adds of the
// canonical definition are explicit __fmaf_rn calls.
#include <math.h>

#include "common.cuh"
#include "tc.cuh"

namespace qwm {

__device__ int g_append_timeout;

namespace {
using namespace tc;

constexpr int DH = 128;        // head_dim
constexpr int NCH = 256;       // centroids per MMA chunk (N)
constexpr int SURV_MAX = 16;   // survivors kept per token before falling back
constexpr int KROW = 136;      // bf16 row stride of the token rows (16-byte aligned)

// Shared memory for a CTA of NT threads (NT tokens: 128, or 256 when C <= 256
// and the tokens go through the MMA in two halves of 128 rows).
template <int NT>
struct Lay {
  static constexpr uint32_t TILE_A = 128 * 128 * 2;                // A hi / lo (SW128 K-major)
  static constexpr uint32_t TILE_B = NCH * 128 * 2;                // -2c chunk (SW128 K-major)
  static constexpr uint32_t AHI = 0;
  static constexpr uint32_t ALO = AHI + TILE_A;
  static constexpr uint32_t B = ALO + TILE_A;
  static constexpr uint32_t AEXT = B + TILE_B;                     // [128][16] bf16 no swizzle
  static constexpr uint32_t BEXT = AEXT + 128 * 16 * 2;            // [256][16]
  static constexpr uint32_t SURV = BEXT + NCH * 16 * 2;            // [SURV_MAX][NT] u16
  static constexpr uint32_t S = SURV + NT * SURV_MAX * 2;          // [128] s
  static constexpr uint32_t W = S + 128 * 4;                       // [8] w
  static constexpr uint32_t U = W + 8 * 4;                         // [128][16] U
  static constexpr uint32_t RED = U + 128 * 16 * 4;                // [8]
  static constexpr uint32_t KR = RED + 8 * 4 + 16;                 // [NT][KROW] bf16 token rows
  static constexpr uint32_t BAR = KR + NT * KROW * 2;
  static constexpr uint32_t BYTES = BAR + 16 + 16 + 1024;
};
static_assert(Lay<256>::BYTES <= 227 * 1024, "shared memory of the 256-token CTA");

struct ApArgs {
  const uint16_t* X;      // [n][H][d] bf16
  const uint16_t* cent;   // [H][C][d] bf16
  const float* sens;      // [H][d]
  const float* wgroup;    // [H][ng]
  const float* basis;     // [H][d][r] (slot in force)
  uint8_t* codes;
  uint16_t* params;
  void* idx;
  int8_t* coef;
  uint16_t* cscale;
  uint16_t* tokver;
  uint16_t* centver;
  int64_t n, t0, tcap;
  int H, C, G, M, r, idx_bytes, version, cver;
};

__device__ __forceinline__ bool lex_less(float a, int ia, float b, int ib) {
  return a < b || (a == b && ia < ib);
}

__device__ __forceinline__ uint16_t bf16_rn(float x) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}

__device__ __forceinline__ float lo_f(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float hi_f(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Channels 8q..8q+7 of centroid i as fp32.  With the whole table in the -2c tile
// (C <= NCH) they come from shared memory: -0.5 * (-2c) restores c exactly,
// signed zeros included; otherwise from global memory.
__device__ __forceinline__ void cent_chunk(const uint8_t* bt, const uint16_t* cent, int C, int i,
                                           int q, float (&c)[8]) {
  if (C <= NCH) {
    const uint4 w = *reinterpret_cast<const uint4*>(bt + sw128_off(i, q, NCH));
    const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      c[2 * e] = __fmul_rn(-0.5f, lo_f(wv[e]));
      c[2 * e + 1] = __fmul_rn(-0.5f, hi_f(wv[e]));
    }
  } else {
    const uint4 w = __ldg(reinterpret_cast<const uint4*>(cent + (size_t)i * DH) + q);
    const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      c[2 * e] = lo_f(wv[e]);
      c[2 * e + 1] = hi_f(wv[e]);
    }
  }
}

// Channels 8q..8q+7 of this thread's token row (shared memory) as fp32.
__device__ __forceinline__ void tok_chunk(const uint16_t* krow, int q, float (&k)[8]) {
  const uint4 w = *reinterpret_cast<const uint4*>(krow + q * 8);
  const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    k[2 * e] = lo_f(wv[e]);
    k[2 * e + 1] = hi_f(wv[e]);
  }
}

// Canonical distances of token row r0 to centroid i0 and of row r1 to i1 (two
// independent channel-order folds interleaved for instruction-level
// parallelism).
template <bool KEY>
__device__ __forceinline__ void canon_dist2x(const uint16_t* r0, const uint16_t* r1,
                                             const uint8_t* bt, const uint16_t* cent, int C,
                                             int i0, int i1, const float* s, float& d0,
                                             float& d1) {
  // the two folds as the lanes of f32x2 operations (each lane rounds exactly as
  // the scalar operation would)
  uint64_t acc = 0ull;
#pragma unroll 2
  for (int q = 0; q < DH / 8; ++q) {
    float k0[8], k1[8], c0[8], c1[8];
    tok_chunk(r0, q, k0);
    tok_chunk(r1, q, k1);
    cent_chunk(bt, cent, C, i0, q, c0);
    cent_chunk(bt, cent, C, i1, q, c1);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int j = q * 8 + e;
      const uint64_t l = fsub2(f2pack(k0[e], k1[e]), f2pack(c0[e], c1[e]));
      if (KEY) acc = ffma2(f2pack(s[j], s[j]), fmul2(l, l), acc);
      else acc = ffma2(l, l, acc);
    }
  }
  f2unpack(acc, d0, d1);
}

// The same token row against two centroids.
template <bool KEY>
__device__ __forceinline__ void canon_dist2(const uint16_t* krow, const uint8_t* bt,
                                            const uint16_t* cent, int C, int i0, int i1,
                                            const float* s, float& d0, float& d1) {
  canon_dist2x<KEY>(krow, krow, bt, cent, C, i0, i1, s, d0, d1);
}

template <bool KEY, int G, int NT>
__device__ __forceinline__ void append_tc_body(const ApArgs& A) {
  using L = Lay<NT>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + L::BAR);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::BAR + 8);
  uint16_t* surv = reinterpret_cast<uint16_t*>(smem + L::SURV);
  // the survivors' approximations [SURV_MAX][NT], in the A tiles, which are
  // free once the MMAs have completed
  float* sval = reinterpret_cast<float*>(smem + L::AHI);
  static_assert(SURV_MAX * NT * 4 <= 2 * L::TILE_A, "survivor values fit the A tiles");
  float* s_s = reinterpret_cast<float*>(smem + L::S);
  float* w_s = reinterpret_cast<float*>(smem + L::W);
  float* U_s = reinterpret_cast<float*>(smem + L::U);
  float* red = reinterpret_cast<float*>(smem + L::RED);
  const uint8_t* bt = smem + L::B;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int half = tid >> 7;     // MMA half of the CTA's tokens (TMEM columns half * NCH)
  const int row = tid & 127;     // row of the half = TMEM lane
  const int h = blockIdx.y;
  const int C = A.C, r = A.r, ng = DH / G;
  const int64_t tok = (int64_t)blockIdx.x * NT + tid;
  const bool valid = tok < A.n;
  const uint16_t* cent = A.cent + (size_t)h * C * DH;

  int* qcount = reinterpret_cast<int*>(smem + L::BAR + 16);
  if (tid == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
    *qcount = 0;
  }
  if (warp == 0) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  // the token row, in shared memory for every later pass
  uint16_t* krow = reinterpret_cast<uint16_t*>(smem + L::KR) + tid * KROW;
  {
    const uint4* src = reinterpret_cast<const uint4*>(A.X + ((size_t)tok * A.H + h) * DH);
#pragma unroll 4
    for (int c = 0; c < 16; ++c) {
      uint4 w = make_uint4(0, 0, 0, 0);
      if (valid) w = __ldg(src + c);
      *reinterpret_cast<uint4*>(krow + c * 8) = w;
    }
  }
  // ---- P0: statistics in force; the constant rows of the extra A step
  for (int j = tid; j < DH; j += NT) s_s[j] = KEY ? A.sens[(size_t)h * DH + j] : 1.0f;
  if (KEY) {
    if (tid < ng) w_s[tid] = A.wgroup[(size_t)h * ng + tid];
    for (int e = tid; e < DH * r; e += NT) U_s[e] = A.basis[(size_t)h * DH * r + e];
  }
  if (tid < 128) {
    // extra K step: A row = [1, 1, 0 ...]
    uint8_t* aext = smem + L::AEXT;
    const uint32_t one2 = 0x3F803F80u;  // bf16 1.0, 1.0
    *reinterpret_cast<uint4*>(aext + (tid >> 3) * 256 + (tid & 7) * 16) = make_uint4(one2, 0, 0, 0);
    *reinterpret_cast<uint4*>(aext + (tid >> 3) * 256 + 128 + (tid & 7) * 16) = make_uint4(0, 0, 0, 0);
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  // ---- P1-P3: per chunk of 256 centroids the B operand (-2c and B_i), then per
  // half of the tokens the A operand (s*k as bf16 hi + lo, A_t) and the MMAs into
  // TMEM columns (chunk + half) * NCH
  const int nchunk = (C + NCH - 1) / NCH;  // 1 when NT == 256
  float At = 0.0f;
  float bmax = 0.0f;  // max of B_i over this thread's centroid rows, then over all
  bool ok = true;
  int nmma = 0;
  for (int ch = 0; ch < nchunk; ++ch) {
    const int c0 = ch * NCH, nc = min(NCH, C - c0);
    uint8_t* btw = smem + L::B;
    uint8_t* bext = smem + L::BEXT;
    for (int rr = tid; rr < NCH; rr += NT) {
      const int i = c0 + rr;
      const uint4* c4 = reinterpret_cast<const uint4*>(cent + (size_t)i * DH);
      float bacc = 0.0f;  // B_i = sum_j s_j c_ij^2, channel order
#pragma unroll 4
      for (int c = 0; c < 16; ++c) {
        uint4 w = make_uint4(0, 0, 0, 0);
        if (rr < nc) w = __ldg(c4 + c);
        // -2c is exact in bf16: flip the sign, add one to the exponent (0 stays 0)
        const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
        uint32_t o[4];
#pragma unroll
        for (int e2 = 0; e2 < 4; ++e2) {
          uint32_t x = wv[e2], y = 0;
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const uint32_t hbits = (x >> (16 * u)) & 0xffffu;
            const float f = __uint_as_float(hbits << 16);
            bacc = __fmaf_rn(s_s[c * 8 + e2 * 2 + u], __fmul_rn(f, f), bacc);
            const uint16_t m2 = bf16_rn(-2.0f * f);
            y |= (uint32_t)m2 << (16 * u);
          }
          o[e2] = y;
        }
        *reinterpret_cast<uint4*>(btw + sw128_off(rr, c, NCH)) = make_uint4(o[0], o[1], o[2], o[3]);
      }
      const float b = (rr < nc) ? bacc : 0.0f;
      bmax = fmaxf(bmax, b);
      const uint16_t bh = bf16_rn(b);
      const uint16_t bl = bf16_rn(__fsub_rn(b, bf2f(bh)));
      *reinterpret_cast<uint4*>(bext + (rr >> 3) * 256 + (rr & 7) * 16) =
          make_uint4((uint32_t)bh | ((uint32_t)bl << 16), 0, 0, 0);
      *reinterpret_cast<uint4*>(bext + (rr >> 3) * 256 + 128 + (rr & 7) * 16) = make_uint4(0, 0, 0, 0);
    }
    for (int hp = 0; hp < NT / 128; ++hp) {
      if (ch == 0 && half == hp) {
        uint8_t* ahi = smem + L::AHI;
        uint8_t* alo = smem + L::ALO;
#pragma unroll 1
        for (int c = 0; c < 16; ++c) {
          const uint4 w4 = *reinterpret_cast<const uint4*>(krow + c * 8);
          const uint32_t wk[4] = {w4.x, w4.y, w4.z, w4.w};
          uint32_t hi[4], lo[4];
#pragma unroll
          for (int e2 = 0; e2 < 4; ++e2) {
            const uint32_t wv = wk[e2];
            uint16_t hb[2], lb[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              const int j = c * 8 + e2 * 2 + u;
              const float kj = u ? hi_f(wv) : lo_f(wv);
              At = __fmaf_rn(s_s[j], __fmul_rn(kj, kj), At);
              const float sk = KEY ? __fmul_rn(s_s[j], kj) : kj;
              hb[u] = bf16_rn(sk);
              lb[u] = bf16_rn(__fsub_rn(sk, bf2f(hb[u])));
            }
            hi[e2] = (uint32_t)hb[0] | ((uint32_t)hb[1] << 16);
            lo[e2] = (uint32_t)lb[0] | ((uint32_t)lb[1] << 16);
          }
          *reinterpret_cast<uint4*>(ahi + sw128_off(row, c, 128)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
          if (KEY)
            *reinterpret_cast<uint4*>(alo + sw128_off(row, c, 128)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        }
      }
      fence_proxy_async_smem();
      __syncthreads();
      if (tid == 0) {
        tc_fence_after();
        const uint32_t idesc = idesc_bf16(128, NCH, false, false);
        const uint32_t sa = smem_u32(smem + L::AHI), sl = smem_u32(smem + L::ALO);
        const uint32_t sb = smem_u32(smem + L::B);
        const uint32_t d_t = tmem + (ch + hp) * NCH;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint32_t ko = (k >> 2) * (128 * 128) + (k & 3) * 32;
          const uint32_t kb = (k >> 2) * (NCH * 128) + (k & 3) * 32;
          mma_bf16_ss(d_t, desc_sw128(sa + ko, 16, 1024), desc_sw128(sb + kb, 16, 1024), idesc, k > 0);
        }
        if (KEY) {
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint32_t ko = (k >> 2) * (128 * 128) + (k & 3) * 32;
            const uint32_t kb = (k >> 2) * (NCH * 128) + (k & 3) * 32;
            mma_bf16_ss(d_t, desc_sw128(sl + ko, 16, 1024), desc_sw128(sb + kb, 16, 1024), idesc, 1u);
          }
        }
        mma_bf16_ss(d_t, desc_noswz(smem_u32(smem + L::AEXT), 128, 256),
                    desc_noswz(smem_u32(smem + L::BEXT), 128, 256), idesc, 1u);
        mma_commit(bar);
      }
      ok = ok && mbar_wait(bar, nmma & 1);
      ++nmma;
      tc_fence_after();
      __syncthreads();
    }
  }
  if (!__syncthreads_and(ok)) {
    if (tid == 0) atomicExch(&g_append_timeout, 1);
  }
  for (int o = 16; o >= 1; o >>= 1) bmax = fmaxf(bmax, __shfl_xor_sync(0xffffffffu, bmax, o));
  if (lane == 0) red[warp] = bmax;
  __syncthreads();
  bmax = 0.0f;
  for (int wv = 0; wv < NT / 32; ++wv) bmax = fmaxf(bmax, red[wv]);

  // ---- P4: selection from the approximations (thread t, TMEM lane t)
  const int Mc = KEY ? A.M : 1;
  // |d~ - d| <= (2^-16.9 + 2^-14) sqrt(A_t B_i) + (2^-15 + 2^-17 + 2^-18) B_i: bf16 hi+lo
  // representation of s*k (2^-17.9 per term, Cauchy-Schwarz), fp32 accumulation of
  // 258 terms (<= 258 * 2^-23 of the sum of magnitudes), B_i's fp32 fold and its
  // hi+lo split.  E doubles both coefficients.  The canonical fold of 128
  // positive terms is within (n + 3) 2^-24 < 2^-16.9 relative; gamma = 2^-15.
  const float E = 2.4414062e-4f * sqrtf(At * bmax) + 1.2207031e-4f * bmax;  // 2^-12, 2^-13
  const float gam = 3.0517578e-5f;                                           // 2^-15
  const uint32_t trow = tmem + ((uint32_t)(32 * (warp & 3)) << 16) + half * NCH;
  // dM >= the M-th smallest d~: the M-th smallest of the minima of groups of 8
  // columns (M groups hold an element no larger than it).  Group minima are
  // four independent chains per 32 columns; only they enter the sorted list.
  float topv[8];
#pragma unroll
  for (int m = 0; m < 8; ++m) topv[m] = INFINITY;
  // list length: the shortlist size rounded up to 1, 4 or 8 (shorter lists
  // need fewer compare-exchanges per group)
  const int tl = Mc <= 1 ? 1 : (Mc <= 4 ? 4 : 8);
#pragma unroll 1
  for (int c0 = 0; c0 < nchunk * NCH; c0 += 32) {
    float v[32];
    tmem_ld32(trow + c0, v);
#pragma unroll
    for (int gq = 0; gq < 4; ++gq) {
      float x = INFINITY;
      if (c0 + 8 * gq < C) {  // C is a multiple of 16: groups are all valid or all not
#pragma unroll
        for (int e = 0; e < 8; ++e) x = fminf(x, v[8 * gq + e]);
      }
      // insertion into the sorted list
      if (tl == 1) {
        topv[0] = fminf(topv[0], x);
      } else if (tl == 4) {
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const float lo = fminf(topv[m], x);
          x = fmaxf(topv[m], x);
          topv[m] = lo;
        }
      } else {
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          const float lo = fminf(topv[m], x);
          x = fmaxf(topv[m], x);
          topv[m] = lo;
        }
      }
    }
  }
  float dM = topv[0];
#pragma unroll
  for (int m = 0; m < 8; ++m)
    if (m == Mc - 1) dM = topv[m];
  const float tau = dM + E + gam * (At + fabsf(dM) + E);
  float theta = (tau + E + gam * (At + E)) / (1.0f - gam);
  theta += 1e-6f * (fabsf(theta) + At) + 1e-30f;
  int cnt = 0;
#pragma unroll 1
  for (int c0 = 0; c0 < nchunk * NCH; c0 += 32) {
    float v[32];
    tmem_ld32(trow + c0, v);
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      if (c0 + e < C && v[e] <= theta) {
        if (cnt < SURV_MAX) {
          surv[cnt * NT + tid] = (uint16_t)(c0 + e);
          sval[cnt * NT + tid] = v[e];
        }
        ++cnt;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }

  // ---- P5: exact (canonical) distances of the survivors; top-M by (D, i)
  int cand[8];
  float candD[8];
#pragma unroll
  for (int m = 0; m < 8; ++m) { cand[m] = -1; candD[m] = INFINITY; }
  // With exactly Mc survivors they are the shortlist (every member of the exact
  // top Mc survives); their order by (D, i) is needed only to break a tie of
  // the stage-2 score (or never, for a shortlist of one), so the exact
  // distances are computed later for tied candidates only.
  bool exact_set = (cnt == Mc);
  if (valid && exact_set) {
#pragma unroll
    for (int m = 0; m < 8; ++m)
      if (m < Mc) cand[m] = (int)surv[m * NT + tid];
  } else if (valid && cnt > Mc && cnt <= SURV_MAX) {
    // More survivors: the Mc smallest approximations are still the shortlist
    // when the gap to the next one exceeds what the errors can close.  With
    // S those Mc, any j outside S has d~_j >= d~(Mc+1) (non-survivors lie
    // above theta >= d~(Mc+1)), so for i in S the exact values satisfy
    // D*_j - D*_i >= delta = d~(Mc+1) - d~(Mc) - 2E, and the canonical folds
    // (relative error gamma) keep D_j > D_i when
    // delta (1 - gamma) > 2 gamma D*_i, D*_i <= A_t / (1 - gamma) + d~(Mc) + E.
    float sd[9];
    int si[9];
#pragma unroll
    for (int m = 0; m < 9; ++m) { sd[m] = INFINITY; si[m] = 0x7fffffff; }
#pragma unroll 1
    for (int q = 0; q < cnt; ++q) {
      float xv = sval[q * NT + tid];
      int xi = (int)surv[q * NT + tid];
#pragma unroll
      for (int m = 0; m < 9; ++m) {
        if (m <= Mc && lex_less(xv, xi, sd[m], si[m])) {
          const float tv = sd[m];
          const int ti = si[m];
          sd[m] = xv;
          si[m] = xi;
          xv = tv;
          xi = ti;
        }
      }
    }
    float dm = sd[0], dn = sd[1];
#pragma unroll
    for (int m = 1; m < 9; ++m) {
      if (m == Mc - 1) dm = sd[m];
      if (m == Mc) dn = sd[m];
    }
    // 1 + 2 gamma >= 1 / (1 - gamma); the last term covers this test's own rounding
    const float g2 = 1.0f + 2.0f * gam;
    const float dhi = fmaxf(At * g2 + dm + E, 0.0f);
    const float delta = dn - dm - 2.0f * E;
    const float need = 2.0f * gam * g2 * dhi + 1e-6f * (fabsf(dn) + fabsf(dm) + At + E) + 1e-30f;
    if (delta > need) {
      exact_set = true;
#pragma unroll
      for (int m = 0; m < 8; ++m)
        if (m < Mc) cand[m] = si[m];
    }
  }
  // The remaining tokens' survivors are rescored as one queue of (token,
  // centroid) pairs that every thread of the CTA shares (two pairs per thread
  // at a time), so that a few such tokens do not hold up their whole warps;
  // the owner then ranks its own results.  A token whose survivors overflowed
  // the list, or with fewer than Mc, rescores all C centroids itself.
  const bool all = valid && !exact_set && (cnt > SURV_MAX || cnt < Mc);
  const bool queued = valid && !exact_set && !all;
  int qbase = 0;
  uint32_t* qent = reinterpret_cast<uint32_t*>(smem + L::ALO);     // [NT * SURV_MAX]
  float* qd = reinterpret_cast<float*>(smem + L::ALO) + NT * SURV_MAX;
  static_assert(NT * SURV_MAX * 8 <= L::TILE_A, "the rescoring queue fits one A tile");
  if (queued) {
    qbase = atomicAdd(qcount, cnt);
    for (int q = 0; q < cnt; ++q) qent[qbase + q] = ((uint32_t)tid << 16) | surv[q * NT + tid];
  }
  __syncthreads();
  const int qn = *qcount;
#pragma unroll 1
  for (int e0 = tid; e0 < qn; e0 += 2 * NT) {
    const int e1 = e0 + NT < qn ? e0 + NT : e0;
    const uint32_t x0 = qent[e0], x1 = qent[e1];
    const uint16_t* r0 = reinterpret_cast<const uint16_t*>(smem + L::KR) + (x0 >> 16) * KROW;
    const uint16_t* r1 = reinterpret_cast<const uint16_t*>(smem + L::KR) + (x1 >> 16) * KROW;
    float D0, D1;
    canon_dist2x<KEY>(r0, r1, bt, cent, C, (int)(x0 & 0xffffu), (int)(x1 & 0xffffu), s_s, D0, D1);
    qd[e0] = D0;
    qd[e1] = D1;
  }
  __syncthreads();
  if (queued || all) {
    const int nloop = all ? C : cnt;
#pragma unroll 1
    for (int q = 0; q < nloop; q += 2) {
      const bool two = q + 1 < nloop;
      int i0, i1;
      float D0, D1;
      if (all) {
        i0 = q;
        i1 = two ? q + 1 : q;
        canon_dist2<KEY>(krow, bt, cent, C, i0, i1, s_s, D0, D1);
      } else {
        i0 = (int)surv[q * NT + tid];
        i1 = two ? (int)surv[(q + 1) * NT + tid] : i0;
        D0 = qd[qbase + q];
        D1 = two ? qd[qbase + q + 1] : D0;
      }
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        if (u == 1 && !two) break;
        // insert (D, i) into the sorted candidate list (total order on (D, i))
        float xd = u ? D1 : D0;
        int xi = u ? i1 : i0;
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          if (m < Mc) {
            const bool sw =
                (candD[m] == INFINITY && cand[m] < 0) || lex_less(xd, xi, candD[m], cand[m]);
            if (sw) {
              const float td = candD[m];
              const int ti = cand[m];
              candD[m] = xd;
              cand[m] = xi;
              xd = td;
              xi = ti;
            }
          }
        }
      }
    }
  }
  constexpr int NG = DH / G;     // groups per row
  constexpr int QG = G / 8;      // 8-channel chunks per group
  // Code words, group parameters and INT8 coefficients are staged per token in
  // the A tiles (free again) and written to the cache with coalesced 16-byte
  // stores once the whole CTA has encoded its tokens.
  constexpr uint32_t SO_PAR = NT * (DH / 4), SO_COEF = SO_PAR + NT * NG * 4;
  static_assert(SO_COEF + NT * 16 <= 2 * L::TILE_A, "staged outputs fit the A tiles");
  uint8_t* so = smem + L::AHI;
  if (valid) {

  // ---- P6: QSAC stage 2 (keys): expected squared logit perturbation
  int a = cand[0];
  if (KEY && Mc > 1) {
    float best = 0.0f;
    int bm = -1;
    uint32_t tied = 0;  // candidates whose score equals the lowest so far
    float scores[8];
#pragma unroll 1
    for (int m = 0; m < Mc; ++m) {
      int cm = cand[0];
#pragma unroll
      for (int mm = 0; mm < 8; ++mm)
        if (mm == m) cm = cand[mm];
      float score = 0.0f;
#pragma unroll 1
      for (int g = 0; g < NG; ++g) {
        float lo = 0.0f, hi = 0.0f;
#pragma unroll
        for (int qi = 0; qi < QG; ++qi) {
          const int q = g * QG + qi;
          float k[8], c[8];
          tok_chunk(krow, q, k);
          cent_chunk(bt, cent, C, cm, q, c);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float rho = __fsub_rn(k[e], c[e]);
            lo = (qi == 0 && e == 0) ? rho : fminf(lo, rho);
            hi = (qi == 0 && e == 0) ? rho : fmaxf(hi, rho);
          }
        }
        const float R = __fsub_rn(hi, lo);
        score = __fmaf_rn(w_s[g], __fmul_rn(R, R), score);
      }
#pragma unroll
      for (int mm = 0; mm < 8; ++mm)
        if (mm == m) scores[mm] = score;
      if (bm < 0 || score < best) {
        best = score;
        bm = m;
        a = cm;
        tied = 1u << m;
      } else if (score == best) {
        tied |= 1u << m;
      }
    }
    if (exact_set && __popc(tied) > 1) {
      // a tie among unordered candidates: the earliest in (D, i) order wins
      float bd = INFINITY;
      int bi = -1;
#pragma unroll 1
      for (int m = 0; m < Mc; ++m) {
        if (!((tied >> m) & 1u)) continue;
        int cm = cand[0];
#pragma unroll
        for (int mm = 0; mm < 8; ++mm)
          if (mm == m) cm = cand[mm];
        float D, Dx;
        canon_dist2<KEY>(krow, bt, cent, C, cm, cm, s_s, D, Dx);
        if (bi < 0 || lex_less(D, cm, bd, bi)) {
          bd = D;
          bi = cm;
        }
      }
      a = bi;
    }
    (void)scores;
  }

  // ---- P7: INT2 residual and PSAC coefficients, group by group in channel order
  const size_t slot = (size_t)h * A.tcap + (size_t)(A.t0 + tok);
  uint16_t* codew = reinterpret_cast<uint16_t*>(so + tid * (DH / 4));
  uint32_t* pdst = reinterpret_cast<uint32_t*>(so + SO_PAR) + tid * NG;
  float cq[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) cq[i] = 0.0f;
  uint64_t cq2[4] = {0ull, 0ull, 0ull, 0ull};  // r == 8: coefficient pairs (2i, 2i + 1)
#pragma unroll 1
  for (int g = 0; g < NG; ++g) {
    float lo = 0.0f, hi = 0.0f;
#pragma unroll
    for (int qi = 0; qi < QG; ++qi) {
      const int q = g * QG + qi;
      float k[8], c[8];
      tok_chunk(krow, q, k);
      cent_chunk(bt, cent, C, a, q, c);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float rho = __fsub_rn(k[e], c[e]);
        lo = (qi == 0 && e == 0) ? rho : fminf(lo, rho);
        hi = (qi == 0 && e == 0) ? rho : fmaxf(hi, rho);
      }
    }
    uint16_t mnh, sch;
    float mn, sc;
    int2_params(lo, hi, mnh, sch, mn, sc);
    pdst[g] = (uint32_t)mnh | ((uint32_t)sch << 16);
#pragma unroll 1
    for (int qi = 0; qi < QG; ++qi) {
      const int q = g * QG + qi;
      float k[8], c[8];
      tok_chunk(krow, q, k);
      cent_chunk(bt, cent, C, a, q, c);
      uint32_t bits = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int j = q * 8 + e;
        const float rho = __fsub_rn(k[e], c[e]);
        const int code = int2_code(rho, mn, sc);
        bits |= (uint32_t)code << (2 * e);
        if (KEY) {
          // PSAC: e_j = k_j - (c_j + deq_j); coefficient i accumulates U_ji e_j in channel order
          const float deq = __fmaf_rn((float)code, sc, mn);
          const float ej = __fsub_rn(k[e], __fadd_rn(c[e], deq));
          const float* Uj = U_s + j * r;
          if (r == 8) {
            const float4 u0 = *reinterpret_cast<const float4*>(Uj);
            const float4 u1 = *reinterpret_cast<const float4*>(Uj + 4);
            const uint64_t e2 = f2pack(ej, ej);
            cq2[0] = ffma2(f2pack(u0.x, u0.y), e2, cq2[0]);
            cq2[1] = ffma2(f2pack(u0.z, u0.w), e2, cq2[1]);
            cq2[2] = ffma2(f2pack(u1.x, u1.y), e2, cq2[2]);
            cq2[3] = ffma2(f2pack(u1.z, u1.w), e2, cq2[3]);
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i)
              if (i < r) cq[i] = __fmaf_rn(Uj[i], ej, cq[i]);
          }
        }
      }
      codew[q] = (uint16_t)bits;  // channels 8q..8q+7
    }
  }
  if (A.idx_bytes == 1) ((uint8_t*)A.idx)[slot] = (uint8_t)a;
  else ((uint16_t*)A.idx)[slot] = (uint16_t)a;
  if (KEY) {
    if (h == 0) {
      A.tokver[A.t0 + tok] = (uint16_t)A.version;
      A.centver[A.t0 + tok] = (uint16_t)A.cver;
    }
    if (r == 8) {
#pragma unroll
      for (int q = 0; q < 4; ++q) f2unpack(cq2[q], cq[2 * q], cq[2 * q + 1]);
    }
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i)
      if (i < r) amax = fmaxf(amax, fabsf(cq[i]));
    const uint16_t csh = f2h_ru(__fdiv_rn(amax, 127.0f));
    const float cs = h2f(csh);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      if (i < r) {
        int q8 = 0;
        if (cs != 0.0f) {
          q8 = __float2int_rn(__fdiv_rn(cq[i], cs));
          q8 = max(-127, min(127, q8));
        }
        so[SO_COEF + tid * r + i] = (uint8_t)(int8_t)q8;
      }
    }
    A.cscale[slot] = csh;
  }
  }  // valid
  __syncthreads();
  // the CTA's tokens are contiguous in every field: copy the staged rows out
  const int64_t tok0 = (int64_t)blockIdx.x * NT;
  const int nv = (int)(A.n - tok0 < NT ? A.n - tok0 : NT);
  const size_t slot0 = (size_t)h * A.tcap + (size_t)(A.t0 + tok0);
  {
    const uint4* src = reinterpret_cast<const uint4*>(so);
    uint4* dst = reinterpret_cast<uint4*>(A.codes + slot0 * (DH / 4));
    for (int u = tid; u < nv * (DH / 64); u += NT) dst[u] = src[u];
  }
  {
    const uint4* src = reinterpret_cast<const uint4*>(so + SO_PAR);
    uint4* dst = reinterpret_cast<uint4*>(A.params + slot0 * NG * 2);
    for (int u = tid; u < nv * (NG / 4); u += NT) dst[u] = src[u];
  }
  if (KEY && r > 0) {
    if ((r & 7) == 0) {
      const uint2* src = reinterpret_cast<const uint2*>(so + SO_COEF);
      uint2* dst = reinterpret_cast<uint2*>(A.coef + slot0 * r);
      for (int u = tid; u < nv * (r / 8); u += NT) dst[u] = src[u];
    } else {
      for (int u = tid; u < nv * r; u += NT) A.coef[slot0 * r + u] = (int8_t)so[SO_COEF + u];
    }
  }
}

// Keys (blockIdx.z == 0) and Values (z == 1) in one launch: the Value CTAs,
// which finish sooner, fill the last wave of the Key CTAs.
template <int G, int NT>
__global__ void __launch_bounds__(NT, 1) append_tc_kernel(const ApArgs AK, const ApArgs AV) {
  if (blockIdx.z == 0) append_tc_body<true, G, NT>(AK);
  else append_tc_body<false, G, NT>(AV);
}

template <int G, int NT>
cudaError_t run_tc(const ApArgs& ak, const ApArgs& av, cudaStream_t s) {
  const int smem = (int)Lay<NT>::BYTES;
  cudaError_t e = cudaFuncSetAttribute(append_tc_kernel<G, NT>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)((ak.n + NT - 1) / NT), ak.H, 2);
  append_tc_kernel<G, NT><<<grid, NT, smem, s>>>(ak, av);
  return cudaGetLastError();
}

// 256 tokens per CTA (two MMA halves sharing one B tile) when the centroid
// table fits one 256-row tile, else 128.
cudaError_t run_tc_g(const ApArgs& ak, const ApArgs& av, cudaStream_t s) {
  if (ak.C <= NCH) return ak.G == 32 ? run_tc<32, 256>(ak, av, s) : run_tc<16, 256>(ak, av, s);
  return ak.G == 32 ? run_tc<32, 128>(ak, av, s) : run_tc<16, 128>(ak, av, s);
}

}  // namespace

int read_and_clear_append_timeout() {
  int v = 0, z = 0;
  if (cudaMemcpyFromSymbol(&v, g_append_timeout, sizeof(int)) != cudaSuccess) return -1;
  cudaMemcpyToSymbol(g_append_timeout, &z, sizeof(int));
  return v;
}

bool append_tc_supported(const Dims& D) {
  return D.d == DH && (D.G == 16 || D.G == 32) && D.C % 16 == 0 && D.C <= 512 && D.M <= 8 &&
         D.r <= 16 && !D.qsac_full;
}

cudaError_t launch_append_tc(const Dims& Dm, const CacheView& v, const uint16_t* K,
                             const uint16_t* V, int64_t n, int64_t t0, int version,
                             int cent_version, cudaStream_t s) {
  const size_t coff = (size_t)cent_version * cent_slot_elems(Dm);
  ApArgs a{};
  a.n = n;
  a.t0 = t0;
  a.tcap = Dm.tcap;
  a.H = Dm.H;
  a.C = Dm.C;
  a.G = Dm.G;
  a.M = Dm.M;
  a.r = Dm.r;
  a.idx_bytes = Dm.idx_bytes;
  a.version = version;
  a.cver = cent_version;
  a.X = K;
  a.cent = v.cent_k + coff;
  a.sens = v.sens;
  a.wgroup = v.wgroup;
  a.basis = v.basis + (size_t)version * Dm.H * Dm.d * (Dm.r > 0 ? Dm.r : 1);
  a.codes = v.k_codes;
  a.params = v.k_params;
  a.idx = v.k_idx;
  a.coef = v.k_coef;
  a.cscale = v.k_cscale;
  a.tokver = v.tokver;
  a.centver = v.centver;
  ApArgs b = a;
  b.X = V;
  b.cent = v.cent_v + coff;
  b.codes = v.v_codes;
  b.params = v.v_params;
  b.idx = v.v_idx;
  b.coef = nullptr;
  b.cscale = nullptr;
  return run_tc_g(a, b, s);
}

}  // namespace qwm
