// attention_tc.cu -- attention over the packed QuantWM cache on the sm_100a
// tensor cores (tcgen05.mma; Q, S/P and O live in TMEM).
//
// O = softmax(scale Q K'^T) V' with K' = C_K[a] + deq(R) + U_v (c8 cs) and
// V' = C_V[b] + deq(R_V) reconstructed on the fly (QuantWM, "Flickering after
// quantization?" (SynthePulse), PSAC paragraph: the Key error is compensated
// when the cache is reconstructed; U_v is the basis in force when the key was
// appended).
//
// The compensation term runs on the tensor cores instead of per element:
//   q . (U_v c_t) = (U_v^T q) . c_t,
// so each Q K^T gains one extra K16 step (two for r > 8) whose A operand holds
// AX = [Q U_va | Q U_vb] for the (at most two) basis versions va, vb of the key
// tile and whose B operand holds each key's c8 cs in the slot of its version.
// AX itself is a tensor-core product (Q from TMEM times [U_va | U_vb] in bf16),
// recomputed only when the version pair changes from one key tile to the next;
// a key whose version is neither (a tile spanning three versions) is
// compensated element-wise by its dequant thread instead.
//
// One CTA per (head, 256 query rows = two 128-row Q tiles); 608 threads:
//   warps 0-7   softmax: warp w serves Q tile w/4, TMEM lanes 32(w%4)..+31 =
//               query rows; online softmax in the log2 domain with a lazy
//               rescale of O, P written back into TMEM over S (bf16 pairs).
//   warps 8-15  dequant: four threads per key row of each 64-key tile gather
//               their centroid chunks with 16-byte async copies two tiles
//               ahead, then rewrite them in place as K-hat / V' (bf16, the
//               128B-swizzled layouts the UMMA descriptors read).
//   warps 16-17 MMA: one issuing thread per Q tile, S = Q K^T (+ AX BX^T)
//               then, once the softmax has written P, O += P V'; the two
//               threads interleave on the tensor pipe, which works on one Q
//               tile while the softmax works on the other.
//   warp 18     producer: bulk-copies (TMA engine) the tile's packed codes,
//               group parameters, coefficients, versions and centroid indices
//               into the packed-field ring, and builds [U_va | U_vb] in bf16
//               on changes.
// TMEM (512 columns): per Q tile p, Q at 256p (64 columns of bf16 pairs), S/P
// at 256p+64, O at 256p+128.  Shared memory: a ring of 4 K-hat / V' /
// compensation-slab stages (released by the MMA) and a ring of 5 packed-field
// stages (released by the dequant).
//
// The SEG instance also attends over a bf16 segment after the packed tokens
// (the frame being generated): its tiles follow the packed ones, and the
// dequant warps copy their rows into the same swizzled stages instead of
// decoding; they carry the last packed tile's version pair and zero
// compensation rows.  An optional output receives ln sum exp of the scores.
//
// Every mbarrier wait is bounded (about 1 s); a timeout sets a device flag
// that qwm_device_status() reports, every role then leaves its loop, and
// in-flight copies and MMAs are drained (bounded) before the TMEM is freed.
#include <math.h>

#include "dequant.cuh"
#include "tc.cuh"

namespace qwm {

__device__ int g_tc_timeout;

namespace {
using namespace tc;

constexpr int DH = 128;        // head_dim handled here
constexpr int KT = 64;         // keys per tile
constexpr int QT = 128;        // query rows per Q tile (TMEM lanes)
constexpr int BQ = 2 * QT;     // query rows per CTA
constexpr int NKV = 4;         // K-hat / V' stages (released by the MMA)
constexpr int NPK = 5;         // packed-field stages (released by the dequant)
constexpr int NTHREADS = 608;  // 8 softmax + 8 dequant + 2 MMA + producer warps
constexpr int W_MMA = 16;      // warps 16, 17 issue the MMAs of Q tiles 0, 1
constexpr int W_PROD = 18;
constexpr int NDQW = 8;        // dequant warps

// ---- shared memory (bytes); K-hat and V' tiles 1024-aligned for the swizzle
constexpr uint32_t KV_TILE = KT * DH * 2;  // [2 column halves][64 rows][128 B]
constexpr uint32_t ST_K = 0, ST_V = KV_TILE, ST_BX = 2 * KV_TILE;
constexpr uint32_t BX_BYTES = KT * 32 * 2;  // [64 keys][<= 32] bf16
constexpr uint32_t KVST = ST_BX + BX_BYTES;  // 36 KB
constexpr uint32_t PK_KCODE = 0, PK_VCODE = 2048, PK_KPAR = 4096, PK_VPAR = 6144,
                   PK_KCOEF = 8192, PK_KCS = 9216, PK_TV = 9344, PK_KIDX = 9472,
                   PK_VIDX = 9600, PK_BYTES = 9728;
constexpr uint32_t AX_BYTES = QT * 32 * 2;  // [128 rows][<= 32] bf16 per Q tile
constexpr uint32_t UB_BYTES = 32 * DH * 2;  // [<= 32 rows][128] bf16 per buffer
constexpr uint32_t OFF_KV = 0;
constexpr uint32_t OFF_PK = OFF_KV + NKV * KVST;
constexpr uint32_t OFF_AX = (OFF_PK + NPK * PK_BYTES + 1023) / 1024 * 1024;
constexpr uint32_t OFF_UB = OFF_AX + 2 * AX_BYTES;
constexpr uint32_t OFF_INFO = OFF_UB + 2 * UB_BYTES;  // [NKV] version pair of the tile in stage
constexpr uint32_t OFF_BAR = OFF_INFO + 128;
constexpr int NBAR = 35;
constexpr uint32_t SMEM_BYTES = OFF_BAR + NBAR * 8 + 16 + 1024;

enum {
  B_LOAD_FULL = 0,   // [NPK] producer bulk copies (tx bytes) -> dequant
  B_PK_EMPTY = 5,    // [NPK] dequant (one arrival per warp) -> producer
  B_KV_FULL = 10,    // [NKV] dequant (one arrival per warp) -> MMA
  B_KV_EMPTY = 14,   // [NKV] MMA commit after each Q tile's P V' -> dequant
  B_S_FULL = 18,     // [2] MMA commit after Q K^T, or after AX on a version change
  B_P_FULL = 20,     // [2] softmax (per warp) -> MMA: P of that Q tile is in TMEM
  // 22, 23 unused
  B_AX_FULL = 24,    // [2] softmax (per warp) -> MMA: AX slab in shared memory
  B_UB_FULL = 26,    // [2] producer -> MMA: [U_va | U_vb] in buffer
  B_UB_EMPTY = 28,   // [2] MMA commit after the AX products -> producer
  B_Q_READY = 30,    // softmax (per warp) -> MMA: Q in TMEM
  B_O_LAST = 31,     // [2] MMA commit after the last P V' of that Q tile
  B_DONE = 33        // [2] MMA commit -> MMA (drain before exit)
};

struct TcArgs {
  Dims Dm;
  CacheView v;
  int64_t T;     // packed tokens (key tiles 0 .. ntp - 1)
  const uint16_t* Q;
  int64_t nq;
  float scale_log2;
  uint16_t* O;
  int kx;        // extra K width for the compensation (0, 16 or 32)
  const uint16_t* Ks;  // bf16 segment [nseg][H][d] after the packed tokens (tiles ntp ..)
  const uint16_t* Vs;
  int64_t nseg;
  float* lse;    // [nq][H] natural-log softmax denominators, or null
  int ntp;       // key tiles of the packed part
};

// Valid keys of tile j: packed tiles first, then (SEG) the segment's tiles.
template <bool SEG>
__device__ __forceinline__ int tile_valid(const TcArgs& A, int j) {
  const int64_t rem = (!SEG || j < A.ntp) ? A.T - (int64_t)j * KT
                                          : A.nseg - (int64_t)(j - A.ntp) * KT;
  return (int)(rem < KT ? rem : KT);
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm volatile("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// {a, b} -> bf16x2 with a in the low half (round to nearest even)
__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(b), "f"(a));
  return r;
}

__device__ __forceinline__ void timeout_flag() { atomicExch(&g_tc_timeout, 1); }

// One arrival per warp: every lane has ordered its own writes (proxy fence or
// tcgen05 fence) before calling; __syncwarp orders the lanes, then lane 0
// arrives with release semantics.
__device__ __forceinline__ void warp_arrive(uint64_t* bar) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
}

// Bounded wait taken by a whole warp; false (on every lane) if any lane gave up.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity) {
  const bool w = mbar_wait(bar, parity);
  return __all_sync(0xffffffffu, w);
}

// Versions in force for the first and the last key of tile j, packed as
// first | last << 16 (read from global memory).
__device__ __forceinline__ uint32_t tile_pair_global(const uint16_t* tokver, int64_t T, int j) {
  const int64_t t0 = (int64_t)j * KT;
  const int64_t t1 = ((t0 + KT) < T ? (t0 + KT) : T) - 1;
  return (uint32_t)tokver[t0] | ((uint32_t)tokver[t1] << 16);
}

// Slab layouts (no swizzle, K-major core matrices of 8 rows x 16 B):
//   AX  [128 rows][kx]: core (row group g, K column kc) at kc*2048 + g*128
//   BX  [64 keys][kx] : core (g, kc) at kc*1024 + g*128
//   UB  [kx rows][128]: core (g, kc) at g*2048 + kc*128
__device__ __forceinline__ uint32_t ax_off(int m, int kc) {
  return (uint32_t)(kc * 2048 + (m >> 3) * 128 + (m & 7) * 16);
}
__device__ __forceinline__ uint32_t bx_off(int n, int kc) {
  return (uint32_t)(kc * 1024 + (n >> 3) * 128 + (n & 7) * 16);
}
__device__ __forceinline__ uint32_t ub_off(int n, int kc) {
  return (uint32_t)((n >> 3) * 2048 + kc * 128 + (n & 7) * 16);
}

// ------------------------------------------------------------------ softmax role
// The exponent reference m_used of a row moves only when the row maximum has
// grown by more than TAU (log2 units); P then stays below 2^TAU and O, which
// accumulates in TMEM across tiles, is rescaled in place only on such moves.
constexpr float TAU = 8.0f;

// Row maximum of the first n of 64 scores (n = 64 on all but the last tile).
__device__ __forceinline__ float row_max(const float (&s)[64], int n) {
  float m0 = -INFINITY, m1 = -INFINITY, m2 = -INFINITY, m3 = -INFINITY;
  if (n == KT) {
#pragma unroll
    for (int e = 0; e < 64; e += 8) {
      m0 = fmax3(m0, s[e], s[e + 1]);
      m1 = fmax3(m1, s[e + 2], s[e + 3]);
      m2 = fmax3(m2, s[e + 4], s[e + 5]);
      m3 = fmax3(m3, s[e + 6], s[e + 7]);
    }
  } else {
#pragma unroll
    for (int e = 0; e < 64; ++e)
      if (e < n) m0 = fmaxf(m0, s[e]);
  }
  return fmaxf(fmaxf(m0, m1), fmaxf(m2, m3));
}

template <bool SEG>
__device__ __forceinline__ void softmax_role(const TcArgs& A, uint8_t* smem, uint64_t* bars,
                                             uint32_t tmem, int ntile, int nqt) {
  const int warp = threadIdx.x >> 5;
  const int p = warp >> 2;          // Q tile
  const int m = threadIdx.x & 127;  // row in the Q tile = TMEM lane
  const int h = blockIdx.y;
  const int H = A.Dm.H;
  const int kx = A.kx;
  const int64_t q = (int64_t)blockIdx.x * BQ + p * QT + m;
  const uint32_t trow = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
  const uint32_t tq = trow + 256 * p, ts = tq + 64, to = tq + 128;
  {
    // Q row -> TMEM as bf16 pairs (dims 2i, 2i+1 in column i)
    const uint4* src = reinterpret_cast<const uint4*>(A.Q + ((size_t)q * H + h) * DH);
#pragma unroll
    for (int hlf = 0; hlf < 2; ++hlf) {
      uint32_t w[32];
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        uint4 val = make_uint4(0, 0, 0, 0);
        if (q < A.nq) val = __ldg(src + hlf * 8 + c);
        w[4 * c] = val.x;
        w[4 * c + 1] = val.y;
        w[4 * c + 2] = val.z;
        w[4 * c + 3] = val.w;
      }
      tmem_st32u(tq + 32 * hlf, w);
    }
  }
  tc_fence_before();
  warp_arrive(&bars[B_Q_READY]);
  if (p >= nqt) return;

  uint8_t* ax = smem + OFF_AX + p * AX_BYTES;
  const uint32_t* kvinfo = reinterpret_cast<const uint32_t*>(smem + OFF_INFO);
  uint32_t prev = 0xffffffffu;
  int sph = 0;  // phases of S_FULL seen: one per tile, two when the tile brings AX
  float m_used = -INFINITY;
  uint64_t l2 = 0;  // running row sum, as a pair of partial sums
  const float sl2 = A.scale_log2;
  const uint64_t sc2 = f2pack(sl2, sl2);
  bool ok = true;
  for (int j = 0; j < ntile; ++j) {
    if (!warp_wait(&bars[B_S_FULL + p], sph & 1)) { ok = false; break; }
    ++sph;
    tc_fence_after();
    if (kx) {
      // the version pair of the tile (written by the dequant before the stage
      // was handed to the MMA); on a change the S columns hold AX = Q [U_va | U_vb]
      const uint32_t pr = kvinfo[j % NKV];
      if (pr != prev) {
        prev = pr;
        uint32_t w[16];
        if (kx == 16) {
          float a[16];
          tmem_ld16(ts, a);
#pragma unroll
          for (int e = 0; e < 8; ++e) w[e] = pack_bf16(a[2 * e], a[2 * e + 1]);
#pragma unroll
          for (int e = 8; e < 16; ++e) w[e] = 0u;
        } else {
          float a[32];
          tmem_ld32(ts, a);
#pragma unroll
          for (int e = 0; e < 16; ++e) w[e] = pack_bf16(a[2 * e], a[2 * e + 1]);
        }
#pragma unroll
        for (int kc = 0; kc < 4; ++kc)
          if (kc < kx / 8)
            *reinterpret_cast<uint4*>(ax + ax_off(m, kc)) =
                make_uint4(w[4 * kc], w[4 * kc + 1], w[4 * kc + 2], w[4 * kc + 3]);
        fence_proxy_async_smem();
        tc_fence_before();
        warp_arrive(&bars[B_AX_FULL + p]);
        if (!warp_wait(&bars[B_S_FULL + p], sph & 1)) { ok = false; break; }
        ++sph;
        tc_fence_after();
      }
    }
    const int nvalid = tile_valid<SEG>(A, j);
    float m_row;
    {
      float s[64];
      tmem_ld64(ts, s);
      m_row = row_max(s, nvalid) * sl2;
    }
    if (j == 0) {
      m_used = m_row;
    } else {
      const bool need = m_row > m_used + TAU;
      if (__any_sync(0xffffffffu, need)) {
        // O holds P V' of tiles < j, all complete: the commit behind S_FULL(j)
        // tracks every MMA issued before Q K^T of tile j.
        const float f = need ? ex2(m_used - m_row) : 1.0f;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          float o[32];
          tmem_ld32(to + c * 32, o);
          uint32_t ou[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) ou[e] = __float_as_uint(o[e] * f);
          tmem_st32u(to + c * 32, ou);
        }
        l2 = ffma2(l2, f2pack(f, f), 0ull);
        if (need) m_used = m_row;
      }
    }
    // P (bf16 pairs) over the S columns already read: keys 2i, 2i+1 of the tile
    // in column i (the A-operand layout of the P V' MMA).
    const uint64_t nm2 = f2pack(-m_used, -m_used);
#pragma unroll 1
    for (int c = 0; c < 2; ++c) {
      float s[32];
      tmem_ld32(ts + c * 32, s);
      uint32_t pk[16];
#pragma unroll
      for (int e = 0; e < 32; e += 2) {
        float x0, x1;
        f2unpack(ffma2(f2pack(s[e], s[e + 1]), sc2, nm2), x0, x1);
        float p0 = ex2(x0), p1 = ex2(x1);
        if (nvalid < KT) {
          const int col = c * 32 + e;
          if (col >= nvalid) p0 = 0.0f;
          if (col + 1 >= nvalid) p1 = 0.0f;
        }
        const uint64_t pp = f2pack(p0, p1);
        l2 = fadd2(l2, pp);
        pk[e / 2] = pack_bf16(p0, p1);
      }
      tmem_st16u(ts + c * 16, pk);
    }
    tc_fence_before();
    warp_arrive(&bars[B_P_FULL + p]);
  }
  if (ok) ok = warp_wait(&bars[B_O_LAST + p], 0);
  if (!ok) {
    if ((threadIdx.x & 31) == 0) timeout_flag();
    return;
  }
  tc_fence_after();
  float la, lb;
  f2unpack(l2, la, lb);
  const float inv = 1.0f / (la + lb);
  // sum_t 2^(s_t scale log2 e) = l 2^m_used
  if (A.lse && q < A.nq) A.lse[(size_t)q * H + h] = (m_used + log2f(la + lb)) * 0.6931471805599453f;
  uint4* dst = reinterpret_cast<uint4*>(A.O + ((size_t)q * H + h) * DH);
#pragma unroll 1
  for (int c = 0; c < 4; ++c) {
    float o[32];
    tmem_ld32(to + c * 32, o);
    if (q < A.nq) {
#pragma unroll
      for (int k = 0; k < 4; ++k)
        dst[c * 4 + k] = make_uint4(pack_bf16(o[8 * k] * inv, o[8 * k + 1] * inv),
                                    pack_bf16(o[8 * k + 2] * inv, o[8 * k + 3] * inv),
                                    pack_bf16(o[8 * k + 4] * inv, o[8 * k + 5] * inv),
                                    pack_bf16(o[8 * k + 6] * inv, o[8 * k + 7] * inv));
    }
  }
}

// ------------------------------------------------------------------ dequant role
// Residual decode without an int-to-float conversion: for the code c of
// position i (0..3) of a code byte shifted to bits 15..22, OR-ing the masked
// bits into 1.0f gives exactly 1 + c 2^(2i-8); with S_i = sc 2^(8-2i) and
// M_i = mn - S_i one fma then yields mn + c sc (S_i is exact, and M_i is exact
// whenever mn and S_i lie within 2^13 of each other).  Pairs of positions share
// one f32x2 fma; the centroid is added with one f32x2 add.
struct GroupConst {
  uint64_t s01, s23, m01, m23;  // {S_0, S_1}, {S_2, S_3}, {M_0, M_1}, {M_2, M_3}
};

__device__ __forceinline__ GroupConst group_const(uint32_t par) {
  const float mn = h2f((uint16_t)(par & 0xffff)), sc = h2f((uint16_t)(par >> 16));
  const float s0 = sc * 256.0f, s1 = sc * 64.0f, s2 = sc * 16.0f, s3 = sc * 4.0f;
  GroupConst g;
  g.s01 = f2pack(s0, s1);
  g.s23 = f2pack(s2, s3);
  g.m01 = f2pack(__fsub_rn(mn, s0), __fsub_rn(mn, s1));
  g.m23 = f2pack(__fsub_rn(mn, s2), __fsub_rn(mn, s3));
  return g;
}

__device__ __forceinline__ float magic_code(uint32_t x, int i) {
  return __uint_as_float((x & (3u << (15 + 2 * i))) | 0x3F800000u);
}

// Eight channels: centroid chunk cw (bf16 x 8) plus the residual of the 16-bit
// code word `bits` (channel e at bits 2e), as fp32 pairs.
__device__ __forceinline__ void deq_chunk_f32(uint4 cw, uint32_t bits, const GroupConst& g,
                                              uint64_t (&v)[4]) {
  const uint32_t x0 = bits << 15, x1 = bits << 7;  // channels 0-3, 4-7 at bits 15..22
  const uint32_t w[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
  for (int pi = 0; pi < 4; ++pi) {
    const uint32_t x = pi < 2 ? x0 : x1;
    const int i0 = (2 * pi) & 3;
    const uint64_t mm = f2pack(magic_code(x, i0), magic_code(x, i0 + 1));
    const uint64_t r = ffma2(mm, i0 == 0 ? g.s01 : g.s23, i0 == 0 ? g.m01 : g.m23);
    const uint64_t c = f2pack(__uint_as_float(w[pi] << 16), __uint_as_float(w[pi] & 0xffff0000u));
    v[pi] = fadd2(r, c);
  }
}

__device__ __forceinline__ uint4 pack_chunk(const uint64_t (&v)[4]) {
  uint32_t o[4];
#pragma unroll
  for (int pi = 0; pi < 4; ++pi) {
    float a, b;
    f2unpack(v[pi], a, b);
    o[pi] = pack_bf16(a, b);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

__device__ __forceinline__ int staged_idx(const uint8_t* pk, uint32_t off, int k, int ib) {
  return ib == 1 ? (int)pk[off + k] : (int)reinterpret_cast<const uint16_t*>(pk + off)[k];
}

// Element-wise compensation U (c8 cs) of channels j0..j0+7 (rare path).
__device__ __forceinline__ void compensate_chunk(uint64_t (&v2)[4], const float* U, const uint8_t* pk,
                                              int k, int r, int j0) {
  const float cs = h2f(reinterpret_cast<const uint16_t*>(pk + PK_KCS)[k]);
  const int8_t* cf = reinterpret_cast<const int8_t*>(pk + PK_KCOEF) + k * r;
  for (int pi = 0; pi < 4; ++pi) {
    float a, b, ca = 0.0f, cb = 0.0f;
    f2unpack(v2[pi], a, b);
    for (int i = 0; i < r; ++i) {
      const float ch = (float)cf[i] * cs;
      ca = fmaf(__ldg(U + (size_t)(j0 + 2 * pi) * r + i), ch, ca);
      cb = fmaf(__ldg(U + (size_t)(j0 + 2 * pi + 1) * r + i), ch, cb);
    }
    v2[pi] = f2pack(a + ca, b + cb);
  }
}

// One tensor (K or V) of this thread's quarter row: centroid chunks read from
// the stage, residual added, bf16 written back in place.  U != nullptr adds the
// element-wise compensation U (c8 cs) (a key whose basis version is not one of
// the tile's two slots).
__device__ __forceinline__ void deq_quarter(uint8_t* base, const uint32_t (&offs)[4], uint2 w,
                                            const uint32_t* par, int G, int qq, const float* U,
                                            const uint8_t* pk, int k, int r) {
  uint4 cv[4];
#pragma unroll
  for (int cc = 0; cc < 4; ++cc) cv[cc] = *reinterpret_cast<const uint4*>(base + offs[cc]);
  GroupConst g;
  if (G == 32) g = group_const(par[qq]);
#pragma unroll
  for (int cc = 0; cc < 4; ++cc) {
    const int lc = (cc + qq) & 3;  // chunk within the quarter
    if (G != 32) g = group_const(par[(4 * qq + lc) * 8 / G]);
    const uint32_t bits = (lc < 2 ? w.x : w.y) >> (16 * (lc & 1));
    uint64_t v2[4];
    deq_chunk_f32(cv[cc], bits, g, v2);
    if (U) compensate_chunk(v2, U, pk, k, r, (4 * qq + lc) * 8);
    *reinterpret_cast<uint4*>(base + offs[cc]) = pack_chunk(v2);
  }
}

// Issue this thread's 16-byte centroid-chunk copies for tile jj (key row k,
// channel chunks 4qq..4qq+3 of K and V); one commit group per tile.
__device__ __forceinline__ void issue_gather(const TcArgs& A, uint8_t* smem, const PackedHead& ph,
                                             int jj, int k, int qq) {
  const uint8_t* pk = smem + OFF_PK + (jj % NPK) * PK_BYTES;
  const uint32_t st = smem_u32(smem + OFF_KV + (jj % NKV) * KVST);
  const int64_t t = (int64_t)jj * KT + k;
  if (t < A.T) {
    const int ib = A.Dm.idx_bytes;
    const int a = staged_idx(pk, PK_KIDX, k, ib);
    const int b = staged_idx(pk, PK_VIDX, k, ib);
    const uint16_t* ck = ph.cent_k + (size_t)a * DH;
    const uint16_t* cv = ph.cent_v + (size_t)b * DH;
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
      const int c = 4 * qq + ((cc + qq) & 3);  // same bank-group rotation as the rewrite
      cp_async16(st + ST_K + sw128_off(k, c, KT), ck + c * 8);
      cp_async16(st + ST_V + sw128_off(k, c, KT), cv + c * 8);
    }
  }
  cp_async_commit();
}

// Segment tile jj (jj >= ntp): this thread's 16-byte chunks of the bf16 K and V
// rows copied as they are into the same swizzled stage positions.
__device__ __forceinline__ void issue_seg_gather(const TcArgs& A, uint8_t* smem, int jj, int k,
                                                 int qq) {
  const uint32_t st = smem_u32(smem + OFF_KV + (jj % NKV) * KVST);
  const int64_t t = (int64_t)(jj - A.ntp) * KT + k;
  if (t < A.nseg) {
    const size_t row = ((size_t)t * A.Dm.H + blockIdx.y) * DH;
    const uint16_t* kr = A.Ks + row;
    const uint16_t* vr = A.Vs + row;
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
      const int c = 4 * qq + ((cc + qq) & 3);
      cp_async16(st + ST_K + sw128_off(k, c, KT), kr + c * 8);
      cp_async16(st + ST_V + sw128_off(k, c, KT), vr + c * 8);
    }
  }
  cp_async_commit();
}

template <bool SEG>
__device__ __forceinline__ void dequant_role(const TcArgs& A, uint8_t* smem, uint64_t* bars,
                                             int ntile) {
  const int dq = threadIdx.x - 256;  // 0..255
  const int k = dq >> 2;             // key row in the tile
  const int qq = dq & 3;             // channel quarter [32 qq, 32 qq + 32)
  const Dims& Dm = A.Dm;
  const int h = blockIdx.y;
  const PackedHead ph = packed_head(A.v, Dm, h);
  const int G = Dm.G, ng = Dm.ng, r = Dm.r, kx = A.kx;
  uint32_t* kvinfo = reinterpret_cast<uint32_t*>(smem + OFF_INFO);
  bool ok = true;
  const int ntp = SEG ? A.ntp : ntile;
  // the version pair segment tiles carry: that of the last packed tile, so the
  // compensation slab stays in place (segment keys have zero BX rows)
  const uint32_t seg_pair =
      (SEG && kx && ntp > 0) ? tile_pair_global(A.v.tokver, A.T, ntp - 1) : 0u;
  // prologue: gathers of tiles 0 and 1 (their K-hat / V' stages start free)
  for (int jj = 0; jj < 2 && jj < ntile; ++jj) {
    if (!SEG || jj < ntp) {
      if (!warp_wait(&bars[B_LOAD_FULL + jj], 0)) { ok = false; break; }
      issue_gather(A, smem, ph, jj, k, qq);
    } else {
      issue_seg_gather(A, smem, jj, k, qq);
    }
  }
  for (int j = 0; ok && j < ntile; ++j) {
    if (j + 2 < ntile) {
      const int j2 = j + 2;
      if ((!SEG || j2 < ntp) &&
          !warp_wait(&bars[B_LOAD_FULL + j2 % NPK], (j2 / NPK) & 1)) { ok = false; break; }
      if (j2 >= NKV &&
          !warp_wait(&bars[B_KV_EMPTY + j2 % NKV], ((j2 / NKV) - 1) & 1)) { ok = false; break; }
      if (!SEG || j2 < ntp) issue_gather(A, smem, ph, j2, k, qq);
      else issue_seg_gather(A, smem, j2, k, qq);
      cp_async_wait<2>();
    } else if (j + 1 < ntile) {
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    const int s = j % NKV, sp = j % NPK;
    uint8_t* st = smem + OFF_KV + s * KVST;
    uint8_t* kb = st + ST_K;
    uint8_t* vb = st + ST_V;
    uint8_t* xb = st + ST_BX;
    if (SEG && j >= ntp) {
      // segment tile: rows already in place; zero rows past the segment's end
      // and zero compensation rows
      if ((int64_t)(j - ntp) * KT + k >= A.nseg) {
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          const uint32_t off = sw128_off(k, 4 * qq + cc, KT);
          *reinterpret_cast<uint4*>(kb + off) = make_uint4(0, 0, 0, 0);
          *reinterpret_cast<uint4*>(vb + off) = make_uint4(0, 0, 0, 0);
        }
      }
      if (qq < kx / 8) *reinterpret_cast<uint4*>(xb + bx_off(k, qq)) = make_uint4(0, 0, 0, 0);
      if (dq == 0) kvinfo[s] = seg_pair;
      fence_proxy_async_smem();
      warp_arrive(&bars[B_KV_FULL + s]);
      continue;
    }
    const uint8_t* pk = smem + OFF_PK + sp * PK_BYTES;
    const int64_t t0 = (int64_t)j * KT;
    const int64_t t = t0 + k;
    const int nvalid = (int)((A.T - t0) < KT ? (A.T - t0) : KT);
    const uint16_t* tv = reinterpret_cast<const uint16_t*>(pk + PK_TV);
    const int va = tv[0], vbv = tv[nvalid - 1];
    if (t < A.T) {
      const uint2 kw = *reinterpret_cast<const uint2*>(pk + PK_KCODE + k * 32 + qq * 8);
      const uint2 vw = *reinterpret_cast<const uint2*>(pk + PK_VCODE + k * 32 + qq * 8);
      const uint32_t* kpar = reinterpret_cast<const uint32_t*>(pk + PK_KPAR) + k * ng;
      const uint32_t* vpar = reinterpret_cast<const uint32_t*>(pk + PK_VPAR) + k * ng;
      bool fallback = false;
      int ver = 0;
      if (r > 0) {
        ver = tv[k];
        fallback = (ver != va) && (ver != vbv);
        if (qq < kx / 8) {
          // compensation slab row: c8 cs in the slot of the key's version
          // (slot = K columns [0, kx/2) for va, [kx/2, kx) for vb); thread qq
          // writes core column qq (8 columns)
          const int per = kx / 16;  // core columns per slot: 1 or 2
          const int slot = qq / per, i0 = (qq % per) * 8;
          const int sl = (ver == va) ? 0 : ((ver == vbv) ? 1 : -1);
          uint32_t w[4] = {0u, 0u, 0u, 0u};
          if (slot == sl) {
            const float cs = h2f(reinterpret_cast<const uint16_t*>(pk + PK_KCS)[k]);
            const int8_t* cf = reinterpret_cast<const int8_t*>(pk + PK_KCOEF) + k * r;
#pragma unroll
            for (int e = 0; e < 8; e += 2) {
              const float x0 = (i0 + e < r) ? (float)cf[i0 + e] * cs : 0.0f;
              const float x1 = (i0 + e + 1 < r) ? (float)cf[i0 + e + 1] * cs : 0.0f;
              w[e / 2] = pack_bf16(x0, x1);
            }
          }
          *reinterpret_cast<uint4*>(xb + bx_off(k, qq)) = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      // rotating the chunk order by the quarter keeps the 8 threads of a
      // shared-memory phase on distinct 16-byte bank groups
      uint32_t offs[4];
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) offs[cc] = sw128_off(k, 4 * qq + ((cc + qq) & 3), KT);
      const float* U = fallback ? basis_of(A.v, Dm, ver, h) : nullptr;
      deq_quarter(kb, offs, kw, kpar, G, qq, U, pk, k, r);
      deq_quarter(vb, offs, vw, vpar, G, qq, nullptr, pk, k, r);
    } else {
      // past the end of the cache: zero rows (finite V' under P = 0)
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        const uint32_t off = sw128_off(k, 4 * qq + cc, KT);
        *reinterpret_cast<uint4*>(kb + off) = make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4*>(vb + off) = make_uint4(0, 0, 0, 0);
      }
      if (qq < kx / 8) *reinterpret_cast<uint4*>(xb + bx_off(k, qq)) = make_uint4(0, 0, 0, 0);
    }
    if (dq == 0) kvinfo[s] = (uint32_t)va | ((uint32_t)vbv << 16);
    fence_proxy_async_smem();
    warp_arrive(&bars[B_KV_FULL + s]);
    warp_arrive(&bars[B_PK_EMPTY + sp]);
  }
  cp_async_wait<0>();
  if (!ok && (threadIdx.x & 31) == 0) timeout_flag();
}

// ------------------------------------------------------------------ producer role
__device__ __forceinline__ void producer_role(const TcArgs& A, uint8_t* smem, uint64_t* bars,
                                              int ntile) {
  const int lane = threadIdx.x & 31;
  const Dims& Dm = A.Dm;
  const int h = blockIdx.y;
  const PackedHead ph = packed_head(A.v, Dm, h);
  const int ng = Dm.ng, r = Dm.r, kx = A.kx, ib = Dm.idx_bytes;
  const uint32_t par_bytes = KT * ng * 4, coef_bytes = KT * r, idx_bytes = KT * ib;
  const uint32_t tx = 2 * (KT * DH / 4) + 2 * par_bytes + (r > 0 ? coef_bytes + KT * 2 : 0) +
                      KT * 2 + 2 * idx_bytes;
  const uint16_t* tokver = A.v.tokver;
  uint32_t prev = 0xffffffffu;
  int nchg = 0;
  bool ok = true;
  int issued = 0;
  for (int j = 0; j < ntile; ++j) {
    const int s = j % NPK;
    if (j >= NPK) {
      if (!warp_wait(&bars[B_PK_EMPTY + s], ((j / NPK) - 1) & 1)) { ok = false; break; }
    }
    uint8_t* pk = smem + OFF_PK + s * PK_BYTES;
    const int64_t t0 = (int64_t)j * KT;
    if (lane == 0) {
      uint64_t* bar = &bars[B_LOAD_FULL + s];
      mbar_arrive_expect_tx(bar, tx);
      bulk_g2s(smem_u32(pk + PK_KCODE), ph.k_codes + t0 * (DH / 4), KT * DH / 4, bar);
      bulk_g2s(smem_u32(pk + PK_VCODE), ph.v_codes + t0 * (DH / 4), KT * DH / 4, bar);
      bulk_g2s(smem_u32(pk + PK_KPAR), ph.k_params + t0 * ng * 2, par_bytes, bar);
      bulk_g2s(smem_u32(pk + PK_VPAR), ph.v_params + t0 * ng * 2, par_bytes, bar);
      if (r > 0) {
        bulk_g2s(smem_u32(pk + PK_KCOEF), ph.k_coef + t0 * r, coef_bytes, bar);
        bulk_g2s(smem_u32(pk + PK_KCS), ph.k_cscale + t0, KT * 2, bar);
      }
      bulk_g2s(smem_u32(pk + PK_TV), tokver + t0, KT * 2, bar);
      bulk_g2s(smem_u32(pk + PK_KIDX), (const uint8_t*)ph.k_idx + t0 * ib, idx_bytes, bar);
      bulk_g2s(smem_u32(pk + PK_VIDX), (const uint8_t*)ph.v_idx + t0 * ib, idx_bytes, bar);
    }
    __syncwarp();
    ++issued;
    if (kx) {
      const uint32_t pr = tile_pair_global(tokver, A.T, j);
      if (pr != prev) {
        // two buffers: the wait is for the change before last, whose tile
        // precedes this one by at least two, so the MMA can always reach it
        const int b = nchg & 1;
        if (nchg >= 2) {
          if (!warp_wait(&bars[B_UB_EMPTY + b], ((nchg >> 1) - 1) & 1)) { ok = false; break; }
        }
        // [U_va | U_vb]^T in bf16: row n = slot * sw + i holds column i of the
        // slot's basis (zeros past r, and slot 1 is zero when va == vb)
        const int va = (int)(pr & 0xffff), vbv = (int)(pr >> 16);
        const int sw = kx / 2;
        uint8_t* ub = smem + OFF_UB + b * UB_BYTES;
        const int kc = lane & 15;
        for (int n = lane >> 4; n < kx; n += 2) {
          const int sl = n / sw, i = n % sw;
          const int ver = sl == 0 ? va : (vbv != va ? vbv : -1);
          float x[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) x[e] = 0.0f;
          if (ver >= 0 && i < r) {
            const float* U = basis_of(A.v, Dm, ver, h);
#pragma unroll
            for (int e = 0; e < 8; ++e) x[e] = __ldg(U + (size_t)(kc * 8 + e) * r + i);
          }
          *reinterpret_cast<uint4*>(ub + ub_off(n, kc)) =
              make_uint4(pack_bf16(x[0], x[1]), pack_bf16(x[2], x[3]), pack_bf16(x[4], x[5]),
                         pack_bf16(x[6], x[7]));
        }
        fence_proxy_async_smem();
        warp_arrive(&bars[B_UB_FULL + b]);
        prev = pr;
        ++nchg;
      }
    }
  }
  // drain: every bulk copy issued has landed before the CTA may exit
  for (int jj = (issued > NPK ? issued - NPK : 0); jj < issued; ++jj)
    if (!warp_wait(&bars[B_LOAD_FULL + jj % NPK], (jj / NPK) & 1)) ok = false;
  if (!ok && lane == 0) timeout_flag();
}

// ------------------------------------------------------------------ MMA role
// Descriptors are built once; a stage or K-step offset is added to the start
// address field (bytes / 16; no carry out of the 14-bit field in 227 KB).
struct MmaDesc {
  uint64_t k, v, bx, ax, ub;
};

// S_p = Q_p K-hat^T (8 K16 steps, A from TMEM) + AX_p BX^T for the tile in stage s.
__device__ __forceinline__ void issue_qk(const MmaDesc& D, uint32_t tmem, int p, int s, int kx) {
  constexpr uint32_t IDQ = idesc_bf16(128, KT, false, false);
  const uint32_t tq = tmem + 256 * p, ts = tq + 64;
  const uint64_t kd = D.k + (uint64_t)((s * KVST) >> 4);
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const uint32_t koff = ((k >> 2) * (KT * 128) + (k & 3) * 32) >> 4;
    mma_bf16_ts(ts, tq + 8 * k, kd + koff, IDQ, k > 0);
  }
  if (kx) {
    const uint64_t ad = D.ax + (uint64_t)((p * AX_BYTES) >> 4);
    const uint64_t bd = D.bx + (uint64_t)((s * KVST) >> 4);
    mma_bf16_ss(ts, ad, bd, IDQ, 1u);
    if (kx == 32) mma_bf16_ss(ts, ad + (4096 >> 4), bd + (2048 >> 4), IDQ, 1u);
  }
}

// O_p += P_p V' (stage s) with P read from TMEM (the S columns of Q tile p).
__device__ __forceinline__ void issue_pv(const MmaDesc& D, uint32_t tmem, int p, int s,
                                         bool first) {
  constexpr uint32_t IDP = idesc_bf16(128, DH, false, true);
  const uint32_t ts = tmem + 256 * p + 64, to = tmem + 256 * p + 128;
  const uint64_t vd = D.v + (uint64_t)((s * KVST) >> 4);
#pragma unroll
  for (int k = 0; k < KT / 16; ++k)
    mma_bf16_ts(to, ts + 8 * k, vd + (uint64_t)((k * 2048) >> 4), IDP,
                (!first || k > 0) ? 1u : 0u);
}

// AX_p = Q_p [U_va | U_vb] into the S columns of Q tile p.
__device__ __forceinline__ void issue_ax(const MmaDesc& D, uint32_t tmem, int p, int b, int kx) {
  const uint32_t idx = idesc_bf16(128, kx, false, false);
  const uint32_t tq = tmem + 256 * p, ts = tq + 64;
#pragma unroll
  for (int k = 0; k < 8; ++k)
    mma_bf16_ts(ts, tq + 8 * k, D.ub + (uint64_t)((b * UB_BYTES + 2 * k * 128) >> 4), idx, k > 0);
}

// One issuing thread per Q tile p (warps 16 and 17), each running
//   Q K^T(p, t) [after AX(p) when the version pair changes at t]
//     -> wait for the softmax -> P V'(p, t) -> Q K^T(p, t + 1) -> ...
// with blocking waits; the two threads interleave on the tensor pipe, which
// works on one Q tile while the softmax works on the other.  Q K^T(p, t + 1) and
// AX(p) come after P V'(p, t) in the thread's issue order, so an MMA that
// overwrites the S/P columns never overtakes the P V' that reads them.  A stage
// is released after both threads' P V' (one commit each).
__device__ __forceinline__ void mma_role(const TcArgs& A, uint8_t* smem, uint64_t* bars,
                                         uint32_t tmem, int ntile, int p) {
  const uint32_t sbase = smem_u32(smem);
  const int kx = A.kx;
  MmaDesc D;
  D.k = desc_sw128(sbase + OFF_KV + ST_K, 16, 1024);
  D.v = desc_sw128(sbase + OFF_KV + ST_V, KT * 128, 1024);
  D.bx = desc_noswz(sbase + OFF_KV + ST_BX, 1024, 128);
  D.ax = desc_noswz(sbase + OFF_AX, 2048, 128);
  D.ub = desc_noswz(sbase + OFF_UB, 128, 2048);
  const uint32_t* kvinfo = reinterpret_cast<const uint32_t*>(smem + OFF_INFO);
  bool ok = mbar_wait(&bars[B_Q_READY], 0);
  tc_fence_after();
  uint32_t prev = 0xffffffffu;
  int nchg = 0;
  for (int t = 0; ok && t < ntile; ++t) {
    const int s = t % NKV;
    if (!mbar_wait(&bars[B_KV_FULL + s], (t / NKV) & 1)) { ok = false; break; }
    tc_fence_after();
    if (kx) {
      const uint32_t pr = kvinfo[s];
      if (pr != prev) {
        const int b = nchg & 1;
        if (!mbar_wait(&bars[B_UB_FULL + b], (nchg >> 1) & 1)) { ok = false; break; }
        tc_fence_after();
        issue_ax(D, tmem, p, b, kx);
        mma_commit(&bars[B_S_FULL + p]);
        mma_commit(&bars[B_UB_EMPTY + b]);
        if (!mbar_wait(&bars[B_AX_FULL + p], nchg & 1)) { ok = false; break; }
        tc_fence_after();
        ++nchg;
        prev = pr;
      }
    }
    issue_qk(D, tmem, p, s, kx);
    mma_commit(&bars[B_S_FULL + p]);
    if (!mbar_wait(&bars[B_P_FULL + p], t & 1)) { ok = false; break; }
    tc_fence_after();
    issue_pv(D, tmem, p, s, t == 0);
    mma_commit(&bars[B_KV_EMPTY + s]);
    if (t == ntile - 1) mma_commit(&bars[B_O_LAST + p]);
  }
  mma_commit(&bars[B_DONE + p]);
  if (!mbar_wait(&bars[B_DONE + p], 0)) ok = false;
  if (!ok) timeout_flag();
}

template <bool SEG>
__global__ void __launch_bounds__(NTHREADS, 1) attn_tc_kernel(const TcArgs A) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + OFF_BAR + NBAR * 8);
  const int warp = threadIdx.x / 32;
  const int ntile = SEG ? A.ntp + (int)((A.nseg + KT - 1) / KT) : A.ntp;
  const int nqt = ((int64_t)blockIdx.x * BQ + QT < A.nq) ? 2 : 1;
  if (threadIdx.x == 0) {
    for (int i = 0; i < NPK; ++i) {
      mbar_init(&bars[B_LOAD_FULL + i], 1);
      mbar_init(&bars[B_PK_EMPTY + i], NDQW);
    }
    for (int i = 0; i < NKV; ++i) {
      mbar_init(&bars[B_KV_FULL + i], NDQW);
      mbar_init(&bars[B_KV_EMPTY + i], nqt);  // one commit per Q tile
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars[B_S_FULL + i], 1);
      mbar_init(&bars[B_P_FULL + i], 4);
      mbar_init(&bars[B_AX_FULL + i], 4);
      mbar_init(&bars[B_O_LAST + i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars[B_UB_FULL + i], 1);
      mbar_init(&bars[B_UB_EMPTY + i], nqt);  // one commit per Q tile
    }
    mbar_init(&bars[B_Q_READY], 8);
    mbar_init(&bars[B_DONE], 1);
    mbar_init(&bars[B_DONE + 1], 1);
    fence_mbar_init();
  }
  if (warp == W_MMA) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  if (warp < 8) {
    softmax_role<SEG>(A, smem, bars, tmem, ntile, nqt);
  } else if (warp < 8 + NDQW) {
    dequant_role<SEG>(A, smem, bars, ntile);
  } else if (warp < W_PROD) {
    const int p = warp - W_MMA;
    if ((threadIdx.x & 31) == 0 && p < nqt) mma_role(A, smem, bars, tmem, ntile, p);
    __syncwarp();
  } else {
    producer_role(A, smem, bars, A.ntp);  // packed tiles only
  }
  tc_fence_before();
  __syncthreads();
  if (warp == W_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

bool attention_tc_supported(const Dims& D) { return D.d == DH; }

cudaError_t launch_attention_tc(const Dims& D, const CacheView& v, int64_t T, const uint16_t* Q,
                                int64_t nq, float scale, uint16_t* O, const Segment& sg,
                                cudaStream_t s) {
  TcArgs a;
  a.Dm = D;
  a.v = v;
  a.T = T;
  a.Q = Q;
  a.nq = nq;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.O = O;
  // two slots of 8 or 16 columns; none without packed keys
  a.kx = (D.r == 0 || T == 0) ? 0 : (D.r <= 8 ? 16 : 32);
  a.Ks = sg.K;
  a.Vs = sg.V;
  a.nseg = sg.n;
  a.lse = sg.lse;
  a.ntp = (int)((T + KT - 1) / KT);
  // the segment variant only when there is one (no extra branches otherwise)
  auto kern = sg.n > 0 ? attn_tc_kernel<true> : attn_tc_kernel<false>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)((nq + BQ - 1) / BQ), D.H);
  kern<<<grid, NTHREADS, SMEM_BYTES, s>>>(a);
  return cudaGetLastError();
}

int read_and_clear_tc_timeout() {
  int v = 0, z = 0;
  if (cudaMemcpyFromSymbol(&v, g_tc_timeout, sizeof(int)) != cudaSuccess) return -1;
  cudaMemcpyToSymbol(g_tc_timeout, &z, sizeof(int));
  return v;
}

}  // namespace qwm
