// attention_tc.cu -- attention over the packed QuantWM cache on the sm_100a
// tensor cores (tcgen05.mma; Q, S/P and O live in TMEM).
//
// O = softmax(scale Q K'^T) V' with K' = C_K[a] + deq(R) + U_v (c8 cs) and
// V' = C_V[b] + deq(R_V) reconstructed on the fly (QuantWM, "Flickering after
// quantization?" (SynthePulse), PSAC paragraph: the Key error is compensated
// when the cache is reconstructed; U_v is the basis and C the centroid table in
// force when the key was appended).  Each element of K' and V' is summed in
// fp32 and rounded once to bf16, so the tensor cores read the same bf16 cache
// that the reconstruction returns.
//
// One CTA per (head, 256 query rows = two 128-row Q tiles); 608 threads:
//   warps 0-7   softmax: warp w serves Q tile w/4, TMEM lanes 32(w%4)..+31 =
//               query rows; online softmax in the log2 domain with a lazy
//               rescale of O, P written back into TMEM over S (bf16 pairs).
//   warps 8-15  dequant: warp 8+s owns channels [16s, 16s+16) of every key of
//               a 64-key tile (lane l: keys l and l+32); it gathers those
//               centroid chunks with 16-byte async copies two tiles ahead, then
//               rewrites them in place as K' / V' (bf16, the 128B-swizzled
//               layouts the UMMA descriptors read).  All lanes of a warp read the
//               same basis rows, so the compensation's loads are broadcasts.
//   warps 16-17 MMA: one issuing thread per Q tile, S = Q K'^T then, once the
//               softmax has written P, O += P V'; the two threads interleave on
//               the tensor pipe, which works on one Q tile while the softmax
//               works on the other.
//   warp 18     producer: bulk-copies (TMA engine) the tile's packed codes,
//               group parameters, coefficients, basis and table versions and
//               centroid indices into the packed-field ring.
// TMEM (512 columns): per Q tile p, Q at 256p (64 columns of bf16 pairs), S/P
// at 256p+64, O at 256p+128.  Shared memory: a ring of 5 K' / V' stages
// (released by the MMA) and a ring of 5 packed-field stages (released by the
// dequant).
//
// The SEG instance also attends over a bf16 segment after the packed tokens
// (the frame being generated): its tiles follow the packed ones, and the
// dequant warps copy their rows into the same swizzled stages instead of
// decoding.  An optional output receives ln sum exp of the scores.
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
constexpr int NKV = 5;         // K' / V' stages (released by the MMA)
constexpr int NPK = 5;         // packed-field stages (released by the dequant)
constexpr int NTHREADS = 608;  // 8 softmax + 8 dequant + 2 MMA + producer warps
constexpr int W_MMA = 16;      // warps 16, 17 issue the MMAs of Q tiles 0, 1
constexpr int W_PROD = 18;
constexpr int NDQW = 8;        // dequant warps

// ---- shared memory (bytes); K' and V' tiles 1024-aligned for the swizzle
constexpr uint32_t KV_TILE = KT * DH * 2;  // [2 column halves][64 rows][128 B]
constexpr uint32_t ST_K = 0, ST_V = KV_TILE;
constexpr uint32_t KVST = 2 * KV_TILE;     // 32 KB
constexpr uint32_t PK_KCODE = 0, PK_VCODE = 2048, PK_KPAR = 4096, PK_VPAR = 6144,
                   PK_KCOEF = 8192, PK_KCS = 9216, PK_TV = 9344, PK_KIDX = 9472,
                   PK_VIDX = 9600, PK_CV = 9728, PK_BYTES = 9856;
constexpr uint32_t OFF_KV = 0;
constexpr uint32_t OFF_PK = OFF_KV + NKV * KVST;
constexpr uint32_t OFF_BAR = (OFF_PK + NPK * PK_BYTES + 127) / 128 * 128;
constexpr int NBAR = 32;
constexpr uint32_t SMEM_BYTES = OFF_BAR + NBAR * 8 + 16 + 1024;
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory of the attention CTA");

enum {
  B_LOAD_FULL = 0,   // [NPK] producer bulk copies (tx bytes) -> dequant
  B_PK_EMPTY = 5,    // [NPK] dequant (one arrival per warp) -> producer
  B_KV_FULL = 10,    // [NKV] dequant (one arrival per warp) -> MMA
  B_KV_EMPTY = 15,   // [NKV] MMA commit after each Q tile's P V' -> dequant
  B_S_FULL = 20,     // [2] MMA commit after Q K'^T
  B_P_FULL = 22,     // [2] softmax (per warp) -> MMA: P of that Q tile is in TMEM
  B_Q_READY = 24,    // softmax (per warp) -> MMA: Q in TMEM
  B_O_LAST = 25,     // [2] MMA commit after the last P V' of that Q tile
  B_DONE = 27        // [2] MMA commit -> MMA (drain before exit)
};

struct TcArgs {
  Dims Dm;
  CacheView v;
  int64_t T;     // packed tokens (key tiles 0 .. ntp - 1)
  const uint16_t* Q;
  int64_t nq;
  float scale_log2;
  uint16_t* O;
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
__device__ __forceinline__ void softmax_role(const TcArgs& A, uint64_t* bars, uint32_t tmem,
                                             int ntile, int nqt) {
  const int warp = threadIdx.x >> 5;
  const int p = warp >> 2;          // Q tile
  const int m = threadIdx.x & 127;  // row in the Q tile = TMEM lane
  const int h = blockIdx.y;
  const int H = A.Dm.H;
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

  float m_used = -INFINITY;
  uint64_t l2 = 0;  // running row sum, as a pair of partial sums
  const float sl2 = A.scale_log2;
  const uint64_t sc2 = f2pack(sl2, sl2);
  bool ok = true;
  for (int j = 0; j < ntile; ++j) {
    if (!warp_wait(&bars[B_S_FULL + p], j & 1)) { ok = false; break; }
    tc_fence_after();
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
        // tracks every MMA issued before Q K'^T of tile j.
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

// Rank-8 compensation of one channel for two keys: sum_i U_ji cc_i with the
// coefficients as pairs {cc_2m, cc_2m+1}; row j of each key's basis holds 8
// fp32 values (two 16-byte loads; all lanes of the warp read the same row when
// the keys share a basis version).
__device__ __forceinline__ void corr8_pair(const float* U0, const float* U1, bool same,
                                           const uint64_t (&c0)[4], const uint64_t (&c1)[4],
                                           float& o0, float& o1) {
  const float4 a0 = __ldg(reinterpret_cast<const float4*>(U0));
  const float4 b0 = __ldg(reinterpret_cast<const float4*>(U0) + 1);
  float4 a1 = a0, b1 = b0;
  if (!same) {
    a1 = __ldg(reinterpret_cast<const float4*>(U1));
    b1 = __ldg(reinterpret_cast<const float4*>(U1) + 1);
  }
  uint64_t s0 = ffma2(f2pack(a0.x, a0.y), c0[0], 0ull);
  uint64_t s1 = ffma2(f2pack(a1.x, a1.y), c1[0], 0ull);
  s0 = ffma2(f2pack(a0.z, a0.w), c0[1], s0);
  s1 = ffma2(f2pack(a1.z, a1.w), c1[1], s1);
  s0 = ffma2(f2pack(b0.x, b0.y), c0[2], s0);
  s1 = ffma2(f2pack(b1.x, b1.y), c1[2], s1);
  s0 = ffma2(f2pack(b0.z, b0.w), c0[3], s0);
  s1 = ffma2(f2pack(b1.z, b1.w), c1[3], s1);
  float x, y;
  f2unpack(s0, x, y);
  o0 = x + y;
  f2unpack(s1, x, y);
  o1 = x + y;
}

// Compensation of one channel for any rank: sequential fold of U_ji c8_i cs
// (the coefficients read from the staged packed fields).
__device__ __forceinline__ float corr_any(const float* Uj, const int8_t* cf, float cs, int r) {
  float acc = 0.0f;
  for (int i = 0; i < r; ++i) acc = fmaf(__ldg(Uj + i), (float)cf[i] * cs, acc);
  return acc;
}

// Issue this thread's 16-byte centroid-chunk copies for tile jj: keys l and
// l + 32, channel chunks 2s and 2s + 1 of K and V (s = dequant warp), each from
// the table version the key was encoded with; one commit group per tile.
__device__ __forceinline__ void issue_gather(const TcArgs& A, uint8_t* smem, const PackedHead& ph,
                                             int jj, int lane, int sw) {
  const uint8_t* pk = smem + OFF_PK + (jj % NPK) * PK_BYTES;
  const uint32_t st = smem_u32(smem + OFF_KV + (jj % NKV) * KVST);
  const int ib = A.Dm.idx_bytes;
  const uint16_t* cvs = reinterpret_cast<const uint16_t*>(pk + PK_CV);
#pragma unroll
  for (int kk = 0; kk < 2; ++kk) {
    const int k = lane + 32 * kk;
    const int64_t t = (int64_t)jj * KT + k;
    if (t < A.T) {
      const size_t vo = (size_t)cvs[k] * ph.cstride;
      const uint16_t* ck = ph.cent_k + vo + (size_t)staged_idx(pk, PK_KIDX, k, ib) * DH;
      const uint16_t* cv = ph.cent_v + vo + (size_t)staged_idx(pk, PK_VIDX, k, ib) * DH;
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        const int c = 2 * sw + cc;
        cp_async16(st + ST_K + sw128_off(k, c, KT), ck + c * 8);
        cp_async16(st + ST_V + sw128_off(k, c, KT), cv + c * 8);
      }
    }
  }
  cp_async_commit();
}

// Segment tile jj (jj >= ntp): this thread's 16-byte chunks of the bf16 K and V
// rows copied as they are into the same swizzled stage positions.
__device__ __forceinline__ void issue_seg_gather(const TcArgs& A, uint8_t* smem, int jj, int lane,
                                                 int sw) {
  const uint32_t st = smem_u32(smem + OFF_KV + (jj % NKV) * KVST);
#pragma unroll
  for (int kk = 0; kk < 2; ++kk) {
    const int k = lane + 32 * kk;
    const int64_t t = (int64_t)(jj - A.ntp) * KT + k;
    if (t < A.nseg) {
      const size_t row = ((size_t)t * A.Dm.H + blockIdx.y) * DH;
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        const int c = 2 * sw + cc;
        cp_async16(st + ST_K + sw128_off(k, c, KT), A.Ks + row + c * 8);
        cp_async16(st + ST_V + sw128_off(k, c, KT), A.Vs + row + c * 8);
      }
    }
  }
  cp_async_commit();
}

// Rewrite chunk c (8 channels) of key row k in place: centroid chunk from the
// stage, residual (and compensation) added in fp32, one bf16 rounding.
__device__ __forceinline__ void deq_chunk(uint8_t* base, int k, int c, uint32_t bits16,
                                          uint32_t par, const float* corr) {
  const GroupConst g = group_const(par);
  const uint32_t off = sw128_off(k, c, KT);
  const uint4 cw = *reinterpret_cast<const uint4*>(base + off);
  uint64_t v2[4];
  deq_chunk_f32(cw, bits16, g, v2);
  if (corr) {
#pragma unroll
    for (int pi = 0; pi < 4; ++pi) v2[pi] = fadd2(v2[pi], f2pack(corr[2 * pi], corr[2 * pi + 1]));
  }
  *reinterpret_cast<uint4*>(base + off) = pack_chunk(v2);
}

__device__ __forceinline__ void zero_chunks(uint8_t* kb, uint8_t* vb, int k, int sw) {
#pragma unroll
  for (int cc = 0; cc < 2; ++cc) {
    const uint32_t off = sw128_off(k, 2 * sw + cc, KT);
    *reinterpret_cast<uint4*>(kb + off) = make_uint4(0, 0, 0, 0);
    *reinterpret_cast<uint4*>(vb + off) = make_uint4(0, 0, 0, 0);
  }
}

template <bool SEG>
__device__ __forceinline__ void dequant_role(const TcArgs& A, uint8_t* smem, uint64_t* bars,
                                             int ntile) {
  const int dq = threadIdx.x - 256;  // 0..255
  const int sw = dq >> 5;            // channel slice [16 sw, 16 sw + 16)
  const int lane = dq & 31;          // keys lane, lane + 32
  const Dims& Dm = A.Dm;
  const int h = blockIdx.y;
  const PackedHead ph = packed_head(A.v, Dm, h);
  const int G = Dm.G, ng = Dm.ng, r = Dm.r;
  const int gi = (16 * sw) / G;      // the slice's INT2 group (one group: G = 16 or 32)
  const size_t ustride = (size_t)Dm.H * DH * (r > 0 ? r : 1);  // floats per basis version
  const float* ubase = A.v.basis + (size_t)h * DH * (r > 0 ? r : 1) + (size_t)16 * sw * r;
  bool ok = true;
  const int ntp = SEG ? A.ntp : ntile;
  // prologue: gathers of tiles 0 and 1 (their K' / V' stages start free)
  for (int jj = 0; jj < 2 && jj < ntile; ++jj) {
    if (!SEG || jj < ntp) {
      if (!warp_wait(&bars[B_LOAD_FULL + jj], 0)) { ok = false; break; }
      issue_gather(A, smem, ph, jj, lane, sw);
    } else {
      issue_seg_gather(A, smem, jj, lane, sw);
    }
  }
  for (int j = 0; ok && j < ntile; ++j) {
    if (j + 2 < ntile) {
      const int j2 = j + 2;
      if ((!SEG || j2 < ntp) &&
          !warp_wait(&bars[B_LOAD_FULL + j2 % NPK], (j2 / NPK) & 1)) { ok = false; break; }
      if (j2 >= NKV &&
          !warp_wait(&bars[B_KV_EMPTY + j2 % NKV], ((j2 / NKV) - 1) & 1)) { ok = false; break; }
      if (!SEG || j2 < ntp) issue_gather(A, smem, ph, j2, lane, sw);
      else issue_seg_gather(A, smem, j2, lane, sw);
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
    if (SEG && j >= ntp) {
      // segment tile: rows already in place; zero rows past the segment's end
#pragma unroll
      for (int kk = 0; kk < 2; ++kk) {
        const int k = lane + 32 * kk;
        if ((int64_t)(j - ntp) * KT + k >= A.nseg) {
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            const uint32_t off = sw128_off(k, 2 * sw + cc, KT);
            *reinterpret_cast<uint4*>(kb + off) = make_uint4(0, 0, 0, 0);
            *reinterpret_cast<uint4*>(vb + off) = make_uint4(0, 0, 0, 0);
          }
        }
      }
      fence_proxy_async_smem();
      warp_arrive(&bars[B_KV_FULL + s]);
      continue;
    }
    const uint8_t* pk = smem + OFF_PK + sp * PK_BYTES;
    const int64_t t0 = (int64_t)j * KT;
    const uint16_t* tv = reinterpret_cast<const uint16_t*>(pk + PK_TV);
    const uint16_t* kcs = reinterpret_cast<const uint16_t*>(pk + PK_KCS);
    const int8_t* kcf = reinterpret_cast<const int8_t*>(pk + PK_KCOEF);
    const int k0 = lane, k1 = lane + 32;
    const bool in0 = t0 + k0 < A.T, in1 = t0 + k1 < A.T;
    const uint32_t* kpar = reinterpret_cast<const uint32_t*>(pk + PK_KPAR);
    const uint32_t* vpar = reinterpret_cast<const uint32_t*>(pk + PK_VPAR);
    // ---- K' rows: residual plus the compensation of this slice's channels
    {
      const uint32_t kw0 = *reinterpret_cast<const uint32_t*>(pk + PK_KCODE + k0 * 32 + 4 * sw);
      const uint32_t kw1 = *reinterpret_cast<const uint32_t*>(pk + PK_KCODE + k1 * 32 + 4 * sw);
      const uint32_t p0 = kpar[k0 * ng + gi], p1 = kpar[k1 * ng + gi];
      const int v0 = in0 ? tv[k0] : 0, v1 = in1 ? tv[k1] : v0;
      const float* U0 = ubase + (size_t)v0 * ustride;
      const float* U1 = ubase + (size_t)v1 * ustride;
      const float cs0 = in0 ? h2f(kcs[k0]) : 0.0f, cs1 = in1 ? h2f(kcs[k1]) : 0.0f;
      uint64_t c0[4], c1[4];
      if (r == 8) {
        const int2 w0 = *reinterpret_cast<const int2*>(kcf + 8 * k0);
        const int2 w1 = *reinterpret_cast<const int2*>(kcf + 8 * k1);
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const uint32_t x0 = m < 2 ? (uint32_t)w0.x : (uint32_t)w0.y;
          const uint32_t x1 = m < 2 ? (uint32_t)w1.x : (uint32_t)w1.y;
          const int sh = 16 * (m & 1);
          // c8 * cs is exact in fp32 (8-bit times 11-bit significands)
          c0[m] = f2pack((float)(int8_t)(x0 >> sh) * cs0, (float)(int8_t)(x0 >> (sh + 8)) * cs0);
          c1[m] = f2pack((float)(int8_t)(x1 >> sh) * cs1, (float)(int8_t)(x1 >> (sh + 8)) * cs1);
        }
      }
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        float q0[8], q1[8];
        if (r == 8) {
          const bool same = (v0 == v1);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            corr8_pair(U0 + 8 * (8 * cc + e), U1 + 8 * (8 * cc + e), same, c0, c1, q0[e], q1[e]);
        } else if (r > 0) {
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            q0[e] = corr_any(U0 + (size_t)(8 * cc + e) * r, kcf + k0 * r, cs0, r);
            q1[e] = corr_any(U1 + (size_t)(8 * cc + e) * r, kcf + k1 * r, cs1, r);
          }
        }
        if (in0) deq_chunk(kb, k0, 2 * sw + cc, (kw0 >> (16 * cc)) & 0xffffu, p0, r > 0 ? q0 : nullptr);
        if (in1) deq_chunk(kb, k1, 2 * sw + cc, (kw1 >> (16 * cc)) & 0xffffu, p1, r > 0 ? q1 : nullptr);
      }
    }
    // ---- V' rows
#pragma unroll
    for (int kk = 0; kk < 2; ++kk) {
      const int k = lane + 32 * kk;
      if (kk == 0 ? in0 : in1) {
        const uint32_t vw = *reinterpret_cast<const uint32_t*>(pk + PK_VCODE + k * 32 + 4 * sw);
        const uint32_t vp = vpar[k * ng + gi];
        deq_chunk(vb, k, 2 * sw, vw & 0xffffu, vp, nullptr);
        deq_chunk(vb, k, 2 * sw + 1, vw >> 16, vp, nullptr);
      } else {
        zero_chunks(kb, vb, k, sw);
      }
    }
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
  const int ng = Dm.ng, r = Dm.r, ib = Dm.idx_bytes;
  const uint32_t par_bytes = KT * ng * 4, coef_bytes = KT * r, idx_bytes = KT * ib;
  const uint32_t tx = 2 * (KT * DH / 4) + 2 * par_bytes + (r > 0 ? coef_bytes + KT * 2 : 0) +
                      2 * KT * 2 + 2 * idx_bytes;
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
      bulk_g2s(smem_u32(pk + PK_TV), A.v.tokver + t0, KT * 2, bar);
      bulk_g2s(smem_u32(pk + PK_CV), A.v.centver + t0, KT * 2, bar);
      bulk_g2s(smem_u32(pk + PK_KIDX), (const uint8_t*)ph.k_idx + t0 * ib, idx_bytes, bar);
      bulk_g2s(smem_u32(pk + PK_VIDX), (const uint8_t*)ph.v_idx + t0 * ib, idx_bytes, bar);
    }
    __syncwarp();
    ++issued;
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
  uint64_t k, v;
};

// S_p = Q_p K'^T (8 K16 steps, A from TMEM) for the tile in stage s.
__device__ __forceinline__ void issue_qk(const MmaDesc& D, uint32_t tmem, int p, int s) {
  constexpr uint32_t IDQ = idesc_bf16(128, KT, false, false);
  const uint32_t tq = tmem + 256 * p, ts = tq + 64;
  const uint64_t kd = D.k + (uint64_t)((s * KVST) >> 4);
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const uint32_t koff = ((k >> 2) * (KT * 128) + (k & 3) * 32) >> 4;
    mma_bf16_ts(ts, tq + 8 * k, kd + koff, IDQ, k > 0);
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

// One issuing thread per Q tile p (warps 16 and 17), each running
//   Q K'^T(p, t) -> wait for the softmax -> P V'(p, t) -> Q K'^T(p, t + 1) -> ...
// with blocking waits; the two threads interleave on the tensor pipe, which
// works on one Q tile while the softmax works on the other.  Q K'^T(p, t + 1)
// comes after P V'(p, t) in the thread's issue order, so an MMA that
// overwrites the S/P columns never overtakes the P V' that reads them.  A stage
// is released after both threads' P V' (one commit each).
__device__ __forceinline__ void mma_role(const TcArgs& A, uint8_t* smem, uint64_t* bars,
                                         uint32_t tmem, int ntile, int p) {
  const uint32_t sbase = smem_u32(smem);
  MmaDesc D;
  D.k = desc_sw128(sbase + OFF_KV + ST_K, 16, 1024);
  D.v = desc_sw128(sbase + OFF_KV + ST_V, KT * 128, 1024);
  bool ok = mbar_wait(&bars[B_Q_READY], 0);
  tc_fence_after();
  for (int t = 0; ok && t < ntile; ++t) {
    const int s = t % NKV;
    if (!mbar_wait(&bars[B_KV_FULL + s], (t / NKV) & 1)) { ok = false; break; }
    tc_fence_after();
    issue_qk(D, tmem, p, s);
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
      mbar_init(&bars[B_O_LAST + i], 1);
      mbar_init(&bars[B_DONE + i], 1);
    }
    mbar_init(&bars[B_Q_READY], 8);
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
    softmax_role<SEG>(A, bars, tmem, ntile, nqt);
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
