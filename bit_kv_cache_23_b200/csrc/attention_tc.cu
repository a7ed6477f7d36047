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
// A pair of CTAs on two SMs (a cluster of 2) serves one (head, row block):
// each CTA holds up to 256 query rows (two 128-row Q tiles, one per TMEM lane),
// and the even CTA issues M = 256 tensor-core MMAs (tcgen05 cta_group::2) that
// cover the rows of both.  The B operands of those MMAs are split between the
// two CTAs' shared memory, so each CTA decodes only half of every key tile: K'
// for its 32 of the tile's 64 keys (all 128 channels) and V' for its 64 of the
// 128 channels (all 64 keys).  A pair thus decodes each key once for up to 512
// query rows, and each SM decodes half a tile per tile.
//
// 608 threads per CTA:
//   warps 0-7   softmax of this CTA's rows: warp w serves Q tile w/4, TMEM
//               lanes 32(w%4)..+31; online softmax in the log2 domain with a
//               lazy rescale of O, P written back into TMEM over S (bf16 pairs).
//   warps 8-15  dequant: warp 8+s owns channels [16s, 16s+16) of this CTA's 32
//               keys of K' (lane = key) and channel chunk s of this CTA's half of
//               V' for keys lane and lane+32; it gathers the centroid chunks with
//               16-byte async copies two tiles ahead, then rewrites them in place
//               (bf16, the 128B-swizzled layouts the UMMA descriptors read).  All
//               lanes of a warp read the same basis rows, so the compensation's
//               loads are broadcasts.
//   warps 16-17 MMA (even CTA only): one issuing thread per Q tile, S = Q K'^T
//               then, once the softmax of both CTAs has written P, O += P V';
//               completions are signalled to both CTAs (multicast commits).
//   warp 18     producer: bulk-copies (TMA engine) the tile's packed codes,
//               group parameters, coefficients, basis and table versions and
//               centroid indices into this CTA's packed-field ring.
// TMEM (512 columns, the same in both CTAs): per Q tile p, Q at 256p (64
// columns of bf16 pairs), S/P at 256p+64, O at 256p+128.  Shared memory: a ring
// of K' / V' half-tile stages (released by the MMA commits) and a ring of
// packed-field stages (released by the dequant).
//
// The SEG instance also attends over a bf16 segment after the packed tokens
// (the frame being generated): its tiles follow the packed ones, and the
// dequant warps copy their rows into the same swizzled stages instead of
// decoding.  An optional output receives ln sum exp of the scores.
//
// Every mbarrier wait is bounded (about 1 s); a timeout sets a device flag
// that qwm_device_status() reports, every role then leaves its loop, and
// in-flight copies and MMAs are drained (bounded) before both CTAs meet at the
// final cluster barrier and free the TMEM.
#include <math.h>

#include "dequant.cuh"
#include "tc.cuh"

namespace qwm {

__device__ int g_tc_timeout;

namespace {
using namespace tc;

constexpr int DH = 128;        // head_dim handled here
constexpr int KT = 64;         // keys per tile
constexpr int KH = KT / 2;     // K' rows (keys) per CTA per tile
constexpr int VH = DH / 2;     // V' columns (channels) per CTA
constexpr int QT = 128;        // query rows per Q tile (TMEM lanes)
constexpr int ROWS = 2 * QT;   // query rows per CTA at most
constexpr int NKV = 6;         // K' / V' half-tile stages (released by the MMA)
constexpr int NPK = 6;         // packed-field stages (released by the dequant)
constexpr int NTHREADS = 608;  // 8 softmax + 8 dequant + 2 MMA + producer warps
constexpr int W_MMA = 16;      // warps 16, 17 issue the MMAs of Q tiles 0, 1
constexpr int W_PROD = 18;
constexpr int NDQW = 8;        // dequant warps
constexpr uint16_t BOTH = 3;   // multicast mask: both CTAs of the pair
constexpr uint16_t LEAD = 1;   // the even CTA only

// ---- shared memory (bytes); K' and V' halves 1024-aligned for the swizzle
constexpr uint32_t K_HALF = KH * DH * 2;   // [2 column blocks][32 rows][128 B]
constexpr uint32_t V_HALF = KT * VH * 2;   // [64 rows][128 B]
constexpr uint32_t ST_K = 0, ST_V = K_HALF;
constexpr uint32_t KVST = K_HALF + V_HALF;  // 16 KB
// Packed-field stage: the tile's fields, then the PSAC bases of the versions of
// its first and last key, transposed to [r][d] fp32 (one slot when r > 8).
constexpr uint32_t PK_KCODE = 0, PK_VCODE = 2048, PK_KPAR = 4096, PK_VPAR = 6144,
                   PK_KCOEF = 8192, PK_KCS = 9216, PK_TV = 9344, PK_KIDX = 9472,
                   PK_VIDX = 9600, PK_CV = 9728, PK_U = 9856, PK_U_BYTES = 8192,
                   PK_BYTES = PK_U + PK_U_BYTES;
constexpr uint32_t OFF_KV = 0;
constexpr uint32_t OFF_PK = OFF_KV + NKV * KVST;
constexpr uint32_t OFF_BAR = (OFF_PK + NPK * PK_BYTES + 127) / 128 * 128;
constexpr int NBAR = 40;
constexpr uint32_t SMEM_BYTES = OFF_BAR + NBAR * 8 + 16 + 1024;
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory of the attention CTA");

enum {
  B_LOAD_FULL = 0,         // [NPK] producer bulk copies (tx bytes) -> dequant (local)
  B_PK_EMPTY = NPK,        // [NPK] dequant (one arrival per warp) -> producer (local)
  B_KV_FULL = 2 * NPK,     // [NKV] dequant warps of both CTAs -> MMA (even CTA)
  B_KV_EMPTY = B_KV_FULL + NKV,  // [NKV] MMA commit after each Q tile's P V' -> dequant (both)
  B_S_FULL = B_KV_EMPTY + NKV,   // [2] MMA commit after Q K'^T -> softmax (both)
  B_P_FULL = B_S_FULL + 2,       // [2] softmax warps of both CTAs -> MMA (even CTA)
  B_Q_READY = B_P_FULL + 2,      // softmax warps of both CTAs -> MMA: Q in TMEM
  B_O_LAST = B_Q_READY + 1,      // [2] MMA commit after the last P V' -> softmax (both)
  B_DONE = B_O_LAST + 2          // [2] MMA commit -> MMA (drain before exit)
};
static_assert(B_DONE + 2 <= NBAR, "barrier slots");

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
  int rc;        // query rows per CTA (<= 256); a pair serves 2 rc rows
  int nqt;       // Q tiles per CTA with rows (1 or 2), the same in every pair
  int npairs;    // row blocks (pairs) per key range
  int nsplit;    // key ranges; > 1: fp32 partials to ws_o / ws_l, merged after
  float* ws_o;   // [nsplit][nq][H][d] partial outputs (each over its own keys)
  float* ws_l;   // [nsplit][nq][H] their natural-log softmax denominators
};

// The key tiles [j0, j0 + n) and the row block of this pair.
struct Work {
  int rb, chunk, j0, n;
};

__device__ __forceinline__ Work work_of(const TcArgs& A, int ntile) {
  Work w;
  const int unit = blockIdx.x >> 1;
  w.rb = unit % A.npairs;
  w.chunk = unit / A.npairs;
  w.j0 = (int)((int64_t)w.chunk * ntile / A.nsplit);
  w.n = (int)((int64_t)(w.chunk + 1) * ntile / A.nsplit) - w.j0;
  return w;
}

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

// One arrival per warp on this CTA's barrier: every lane has ordered its own
// writes (proxy fence or tcgen05 fence) before calling; __syncwarp orders the
// lanes, then lane 0 arrives with release semantics.
__device__ __forceinline__ void warp_arrive(uint64_t* bar) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
}

// The same on the even CTA's barrier at `bar`'s offset.
__device__ __forceinline__ void warp_arrive_lead(uint64_t* bar) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive_cta(bar, 0);
}

// Bounded wait taken by a whole warp; false (on every lane) if any lane gave up.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity) {
  const bool w = mbar_wait(bar, parity);
  return __all_sync(0xffffffffu, w);
}

// First query row of this CTA.
__device__ __forceinline__ int64_t cta_row0(const TcArgs& A, const Work& w, uint32_t rank) {
  return (int64_t)w.rb * 2 * A.rc + (int64_t)rank * A.rc;
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
                                             const Work& wk, uint32_t rank) {
  const int warp = threadIdx.x >> 5;
  const int p = warp >> 2;          // Q tile
  const int m = threadIdx.x & 127;  // row in the Q tile = TMEM lane
  const int h = blockIdx.y;
  const int H = A.Dm.H;
  const int64_t r0 = cta_row0(A, wk, rank);
  const int64_t rend = (r0 + A.rc < A.nq) ? r0 + A.rc : A.nq;
  const int64_t q = r0 + p * QT + m;
  const bool valid = (p * QT + m < A.rc) && (q < rend);
  const uint32_t trow = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
  const uint32_t tq = trow + 256 * p, ts = tq + 64, to = tq + 128;
  {
    // Q row -> TMEM as bf16 pairs (dims 2i, 2i+1 in column i); zero rows pad
    const uint4* src = reinterpret_cast<const uint4*>(A.Q + ((size_t)(valid ? q : 0) * H + h) * DH);
#pragma unroll
    for (int hlf = 0; hlf < 2; ++hlf) {
      uint32_t w[32];
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        uint4 val = make_uint4(0, 0, 0, 0);
        if (valid) val = __ldg(src + hlf * 8 + c);
        w[4 * c] = val.x;
        w[4 * c + 1] = val.y;
        w[4 * c + 2] = val.z;
        w[4 * c + 3] = val.w;
      }
      tmem_st32u(tq + 32 * hlf, w);
    }
  }
  tc_fence_before();
  warp_arrive_lead(&bars[B_Q_READY]);
  if (p >= A.nqt) return;

  float m_used = -INFINITY;
  uint64_t l2 = 0;  // running row sum, as a pair of partial sums
  const float sl2 = A.scale_log2;
  const uint64_t sc2 = f2pack(sl2, sl2);
  bool ok = true;
  for (int j = 0; j < wk.n; ++j) {
    if (!warp_wait(&bars[B_S_FULL + p], j & 1)) { ok = false; break; }
    tc_fence_after();
    const int nvalid = tile_valid<SEG>(A, wk.j0 + j);
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
        for (int c = 0; c < 16; ++c) {
          float o[8];
          tmem_ld8(to + c * 8, o);
          uint32_t ou[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) ou[e] = __float_as_uint(o[e] * f);
          tmem_st8u_nw(to + c * 8, ou);
          tmem_wait_st();
        }
        l2 = ffma2(l2, f2pack(f, f), 0ull);
        if (need) m_used = m_row;
      }
    }
    // P (bf16 pairs) over the S columns already read: keys 2i, 2i+1 of the tile
    // in column i (the A-operand layout of the P V' MMA); the scores are read
    // again 32 columns at a time.
    const uint64_t nm2 = f2pack(-m_used, -m_used);
#pragma unroll 1
    for (int h2 = 0; h2 < 2; ++h2) {
      float s[32];
      tmem_ld32(ts + 32 * h2, s);
#pragma unroll
    for (int c = 2 * h2; c < 2 * h2 + 2; ++c) {
      uint32_t pk[8];
#pragma unroll
      for (int e = 0; e < 16; e += 2) {
        float x0, x1;
        f2unpack(ffma2(f2pack(s[16 * (c & 1) + e], s[16 * (c & 1) + e + 1]), sc2, nm2), x0, x1);
        float p0 = ex2(x0), p1 = ex2(x1);
        if (nvalid < KT) {
          const int col = c * 16 + e;
          if (col >= nvalid) p0 = 0.0f;
          if (col + 1 >= nvalid) p1 = 0.0f;
        }
        l2 = fadd2(l2, f2pack(p0, p1));
        pk[e / 2] = pack_bf16(p0, p1);
      }
      tmem_st8u_nw(ts + c * 8, pk);
    }
    }
    tmem_wait_st();
    tc_fence_before();
    warp_arrive_lead(&bars[B_P_FULL + p]);
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
  const float lse = (m_used + log2f(la + lb)) * 0.6931471805599453f;
  if (A.nsplit > 1) {
    // partial over this pair's key range: normalized output and its lse
    const size_t row = ((size_t)wk.chunk * A.nq + (valid ? q : 0)) * H + h;
    if (valid) A.ws_l[row] = lse;
    float4* dstp = reinterpret_cast<float4*>(A.ws_o + row * DH);
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      float o[32];
      tmem_ld32(to + c * 32, o);
      if (valid) {
#pragma unroll
        for (int k = 0; k < 8; ++k)
          dstp[c * 8 + k] = make_float4(o[4 * k] * inv, o[4 * k + 1] * inv, o[4 * k + 2] * inv,
                                        o[4 * k + 3] * inv);
      }
    }
    return;
  }
  if (A.lse && valid) A.lse[(size_t)q * H + h] = lse;
  uint4* dst = reinterpret_cast<uint4*>(A.O + ((size_t)(valid ? q : 0) * H + h) * DH);
#pragma unroll 1
  for (int c = 0; c < 4; ++c) {
    float o[32];
    tmem_ld32(to + c * 32, o);
    if (valid) {
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

// binary16 -> fp32 on the FMA and integer pipes (the conversion unit is left to
// the softmax's exponentials): the 15 magnitude bits moved to the fp32
// exponent/mantissa position give 2^-112 times the value, normals and
// subnormals alike, so one exact multiply by 2^112 restores it.
__device__ __forceinline__ float half_bits_to_f32(uint32_t h) {
  const float m = __uint_as_float((h & 0x7fffu) << 13) * 0x1p112f;
  return __uint_as_float(__float_as_uint(m) | ((h & 0x8000u) << 16));
}

// int8 -> fp32 without a conversion instruction: adding c to the bit pattern of
// 1.5 * 2^23 gives 1.5 * 2^23 + c exactly (|c| < 2^22).
__device__ __forceinline__ float i8_to_f32(int c) {
  return __uint_as_float(0x4B400000u + (uint32_t)c) - 12582912.0f;
}

__device__ __forceinline__ GroupConst group_const(uint32_t par) {
  const float mn = half_bits_to_f32(par & 0xffffu), sc = half_bits_to_f32(par >> 16);
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

// Compensation U (c8 cs) of this thread's 16 channels as 8 channel pairs,
// from the basis staged transposed ([r][d], row i = column i of U): for each
// rank i one broadcast of cc_i and four 16-byte loads that every lane of the
// warp shares when the keys have the same version; 8 independent f32x2 chains.
__device__ __forceinline__ void corr_staged(const float* Ut, const int8_t* cf, float cs, int r,
                                            uint64_t (&acc)[8]) {
#pragma unroll
  for (int q = 0; q < 8; ++q) acc[q] = 0ull;
#pragma unroll 4
  for (int i = 0; i < r; ++i) {
    const float ci = i8_to_f32(cf[i]) * cs;  // exact: 8-bit times 11-bit significands
    const uint64_t cc = f2pack(ci, ci);
    const float4* u = reinterpret_cast<const float4*>(Ut + i * DH);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 x = u[q];
      acc[2 * q] = ffma2(f2pack(x.x, x.y), cc, acc[2 * q]);
      acc[2 * q + 1] = ffma2(f2pack(x.z, x.w), cc, acc[2 * q + 1]);
    }
  }
}

// The same from the basis in global memory ([d][r], channel j at row j) for a
// key whose version is not staged with its tile.
__device__ __forceinline__ void corr_global(const float* Uj0, const int8_t* cf, float cs, int r,
                                            uint64_t (&acc)[8]) {
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    float a = 0.0f, b = 0.0f;
    for (int i = 0; i < r; ++i) {
      const float ci = (float)cf[i] * cs;
      a = fmaf(__ldg(Uj0 + (size_t)(2 * q) * r + i), ci, a);
      b = fmaf(__ldg(Uj0 + (size_t)(2 * q + 1) * r + i), ci, b);
    }
    acc[q] = f2pack(a, b);
  }
}

// Rewrite the 8-channel chunk at byte `off` of a swizzled stage tile in place:
// centroid chunk from the stage, residual (and compensation) added in fp32, one
// bf16 rounding.
__device__ __forceinline__ void deq_chunk(uint8_t* base, uint32_t off, uint32_t bits16,
                                          const GroupConst& g, const uint64_t* corr) {
  const uint4 cw = *reinterpret_cast<const uint4*>(base + off);
  uint64_t v2[4];
  deq_chunk_f32(cw, bits16, g, v2);
  if (corr) {
#pragma unroll
    for (int pi = 0; pi < 4; ++pi) v2[pi] = fadd2(v2[pi], corr[pi]);
  }
  *reinterpret_cast<uint4*>(base + off) = pack_chunk(v2);
}

__device__ __forceinline__ void zero_chunk(uint8_t* base, uint32_t off) {
  *reinterpret_cast<uint4*>(base + off) = make_uint4(0, 0, 0, 0);
}

// This thread's share of a tile (rank = CTA in the pair, sw = dequant warp):
//   K': key kk = 32 rank + lane of the tile, channel chunks 2sw, 2sw+1;
//   V': keys lane and lane + 32, channel chunk cvc = 8 rank + sw (chunk sw of
//       this CTA's 64-channel half).
struct DqShare {
  int kk, sw, lane, cvc;
  uint32_t koff[2];   // stage offsets of the K' chunks (row lane, chunks 2sw, 2sw+1)
  uint32_t voff[2];   // stage offsets of the V' chunk (rows lane, lane+32, chunk sw)
};

// Issue the 16-byte centroid-chunk copies of tile jj, each from the table
// version its key was encoded with; one commit group per tile.
__device__ __forceinline__ void issue_gather(const TcArgs& A, uint8_t* smem, const PackedHead& ph,
                                             int jj, int jl, const DqShare& d) {
  const uint8_t* pk = smem + OFF_PK + (jl % NPK) * PK_BYTES;
  const uint32_t st = smem_u32(smem + OFF_KV + (jl % NKV) * KVST);
  const int ib = A.Dm.idx_bytes;
  const uint16_t* cvs = reinterpret_cast<const uint16_t*>(pk + PK_CV);
  const int64_t t0 = (int64_t)jj * KT;
  if (t0 + d.kk < A.T) {
    const uint16_t* ck = ph.cent_k + (size_t)cvs[d.kk] * ph.cstride +
                         (size_t)staged_idx(pk, PK_KIDX, d.kk, ib) * DH;
    cp_async16_cg(st + d.koff[0], ck + 16 * d.sw);
    cp_async16_cg(st + d.koff[1], ck + 16 * d.sw + 8);
  }
#pragma unroll
  for (int kk = 0; kk < 2; ++kk) {
    const int k = d.lane + 32 * kk;
    if (t0 + k < A.T) {
      const uint16_t* cv = ph.cent_v + (size_t)cvs[k] * ph.cstride +
                           (size_t)staged_idx(pk, PK_VIDX, k, ib) * DH;
      cp_async16_cg(st + d.voff[kk], cv + d.cvc * 8);
    }
  }
  cp_async_commit();
}

// Segment tile jj (jj >= ntp): this thread's 16-byte chunks of the bf16 K and V
// rows copied as they are into the same swizzled stage positions.
__device__ __forceinline__ void issue_seg_gather(const TcArgs& A, uint8_t* smem, int jj, int jl,
                                                 const DqShare& d) {
  const uint32_t st = smem_u32(smem + OFF_KV + (jl % NKV) * KVST);
  const int64_t t0 = (int64_t)(jj - A.ntp) * KT;
  if (t0 + d.kk < A.nseg) {
    const uint16_t* kr = A.Ks + ((size_t)(t0 + d.kk) * A.Dm.H + blockIdx.y) * DH;
    cp_async16_cg(st + d.koff[0], kr + 16 * d.sw);
    cp_async16_cg(st + d.koff[1], kr + 16 * d.sw + 8);
  }
#pragma unroll
  for (int kk = 0; kk < 2; ++kk) {
    const int k = d.lane + 32 * kk;
    if (t0 + k < A.nseg) {
      const uint16_t* vr = A.Vs + ((size_t)(t0 + k) * A.Dm.H + blockIdx.y) * DH;
      cp_async16_cg(st + d.voff[kk], vr + d.cvc * 8);
    }
  }
  cp_async_commit();
}

template <bool SEG>
__device__ __forceinline__ void dequant_role(const TcArgs& A, uint8_t* smem, uint64_t* bars,
                                             const Work& wk, uint32_t rank) {
  const int dq = threadIdx.x - 256;  // 0..255
  DqShare d;
  d.sw = dq >> 5;
  d.lane = dq & 31;
  d.kk = KH * (int)rank + d.lane;
  d.cvc = 8 * (int)rank + d.sw;
  d.koff[0] = ST_K + sw128_off(d.lane, 2 * d.sw, KH);
  d.koff[1] = ST_K + sw128_off(d.lane, 2 * d.sw + 1, KH);
  d.voff[0] = ST_V + sw128_off(d.lane, d.sw, KT);
  d.voff[1] = ST_V + sw128_off(d.lane + 32, d.sw, KT);
  const Dims& Dm = A.Dm;
  const int h = blockIdx.y;
  const PackedHead ph = packed_head(A.v, Dm, h);
  const int G = Dm.G, ng = Dm.ng, r = Dm.r;
  const int gik = (16 * d.sw) / G;   // INT2 group of the K' channels (one group)
  const int giv = (8 * d.cvc) / G;   // INT2 group of the V' chunk
  const size_t ustride = (size_t)Dm.H * DH * (r > 0 ? r : 1);  // floats per basis version
  const float* ubase = A.v.basis + (size_t)h * DH * (r > 0 ? r : 1) + (size_t)16 * d.sw * r;
  bool ok = true;
  const int ntp = A.ntp;  // tiles below ntp are packed, the rest (SEG) the segment's
  const int n = wk.n, j0 = wk.j0;
  // prologue: gathers of the range's first two tiles (their stages start free);
  // ring slots and barrier phases count tiles from the start of the range
  for (int jl = 0; jl < 2 && jl < n; ++jl) {
    if (!SEG || j0 + jl < ntp) {
      if (!warp_wait(&bars[B_LOAD_FULL + jl], 0)) { ok = false; break; }
      issue_gather(A, smem, ph, j0 + jl, jl, d);
    } else {
      issue_seg_gather(A, smem, j0 + jl, jl, d);
    }
  }
  for (int jl = 0; ok && jl < n; ++jl) {
    const int j = j0 + jl;
    if (jl + 2 < n) {
      const int l2 = jl + 2;
      if ((!SEG || j0 + l2 < ntp) &&
          !warp_wait(&bars[B_LOAD_FULL + l2 % NPK], (l2 / NPK) & 1)) { ok = false; break; }
      if (l2 >= NKV &&
          !warp_wait(&bars[B_KV_EMPTY + l2 % NKV], ((l2 / NKV) - 1) & 1)) { ok = false; break; }
      if (!SEG || j0 + l2 < ntp) issue_gather(A, smem, ph, j0 + l2, l2, d);
      else issue_seg_gather(A, smem, j0 + l2, l2, d);
      cp_async_wait<2>();
    } else if (jl + 1 < n) {
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    const int s = jl % NKV, sp = jl % NPK;
    uint8_t* st = smem + OFF_KV + s * KVST;
    if (SEG && j >= ntp) {
      // segment tile: rows already in place; zero rows past the segment's end
      const int64_t t0 = (int64_t)(j - ntp) * KT;
      if (t0 + d.kk >= A.nseg) {
        zero_chunk(st, d.koff[0]);
        zero_chunk(st, d.koff[1]);
      }
#pragma unroll
      for (int kk = 0; kk < 2; ++kk)
        if (t0 + d.lane + 32 * kk >= A.nseg) zero_chunk(st, d.voff[kk]);
      fence_proxy_async_smem();
      warp_arrive_lead(&bars[B_KV_FULL + s]);
      continue;
    }
    const uint8_t* pk = smem + OFF_PK + sp * PK_BYTES;
    const int64_t t0 = (int64_t)j * KT;
    // ---- K': residual plus the compensation of this slice's 16 channels
    if (t0 + d.kk < A.T) {
      const int kk = d.kk;
      const uint32_t kw = *reinterpret_cast<const uint32_t*>(pk + PK_KCODE + kk * 32 + 4 * d.sw);
      const uint32_t kp = reinterpret_cast<const uint32_t*>(pk + PK_KPAR)[kk * ng + gik];
      uint64_t corr[8];
      if (r > 0) {
        // the basis of the key's version: a staged slot (the versions of the
        // tile's first and last key), else global memory
        const uint16_t* tv = reinterpret_cast<const uint16_t*>(pk + PK_TV);
        const int ver = tv[kk];
        const int nval = (int)((A.T - t0) < KT ? (A.T - t0) : KT);
        const float cs = half_bits_to_f32(reinterpret_cast<const uint16_t*>(pk + PK_KCS)[kk]);
        const int8_t* kcf = reinterpret_cast<const int8_t*>(pk + PK_KCOEF) + kk * r;
        const float* us = reinterpret_cast<const float*>(pk + PK_U) + 16 * d.sw;
        if (ver == tv[0]) corr_staged(us, kcf, cs, r, corr);
        else if (r <= 8 && ver == tv[nval - 1]) corr_staged(us + r * DH, kcf, cs, r, corr);
        else corr_global(ubase + (size_t)ver * ustride, kcf, cs, r, corr);
      }
      const GroupConst g = group_const(kp);  // both chunks lie in one INT2 group
      deq_chunk(st, d.koff[0], kw & 0xffffu, g, r > 0 ? corr : nullptr);
      deq_chunk(st, d.koff[1], kw >> 16, g, r > 0 ? corr + 4 : nullptr);
    } else {
      zero_chunk(st, d.koff[0]);
      zero_chunk(st, d.koff[1]);
    }
    // ---- V': this CTA's channel chunk of keys lane and lane + 32
#pragma unroll
    for (int kk = 0; kk < 2; ++kk) {
      const int k = d.lane + 32 * kk;
      if (t0 + k < A.T) {
        const uint32_t vw = *reinterpret_cast<const uint16_t*>(pk + PK_VCODE + k * 32 + 2 * d.cvc);
        const uint32_t vp = reinterpret_cast<const uint32_t*>(pk + PK_VPAR)[k * ng + giv];
        deq_chunk(st, d.voff[kk], vw, group_const(vp), nullptr);
      } else {
        zero_chunk(st, d.voff[kk]);
      }
    }
    fence_proxy_async_smem();
    warp_arrive_lead(&bars[B_KV_FULL + s]);
    warp_arrive(&bars[B_PK_EMPTY + sp]);
  }
  cp_async_wait<0>();
  if (!ok && (threadIdx.x & 31) == 0) timeout_flag();
}

// ------------------------------------------------------------------ producer role
__device__ __forceinline__ void producer_role(const TcArgs& A, uint8_t* smem, uint64_t* bars,
                                              const Work& wk) {
  const int lane = threadIdx.x & 31;
  const Dims& Dm = A.Dm;
  const int h = blockIdx.y;
  const PackedHead ph = packed_head(A.v, Dm, h);
  const int ng = Dm.ng, r = Dm.r, ib = Dm.idx_bytes;
  const uint32_t par_bytes = KT * ng * 4, coef_bytes = KT * r, idx_bytes = KT * ib;
  const uint32_t tx0 = 2 * (KT * DH / 4) + 2 * par_bytes + (r > 0 ? coef_bytes + KT * 2 : 0) +
                       2 * KT * 2 + 2 * idx_bytes;
  const int un = r * DH;  // floats of one basis version of this head
  const float* ub = A.v.basis + (size_t)h * DH * r;
  const size_t vs = (size_t)Dm.H * DH * r;
  int pva = -1, pvb = -1;            // versions staged with the previous tile
  const float* prevU = nullptr;
  bool ok = true;
  int issued = 0;
  // the packed tiles of the range (segment tiles need no fields)
  const int npk = (wk.j0 + wk.n < A.ntp ? wk.j0 + wk.n : A.ntp) - wk.j0;
  for (int jl = 0; jl < npk; ++jl) {
    const int s = jl % NPK;
    if (jl >= NPK) {
      if (!warp_wait(&bars[B_PK_EMPTY + s], ((jl / NPK) - 1) & 1)) { ok = false; break; }
    }
    uint8_t* pk = smem + OFF_PK + s * PK_BYTES;
    const int64_t t0 = (int64_t)(wk.j0 + jl) * KT;
    if (r > 0) {
      // the bases of the versions of the tile's first and last key, transposed
      // to [r][d]: copied from the previous tile's stage when the version was
      // staged there, else gathered from global memory (once per version)
      const int64_t t1 = (t0 + KT < A.T ? t0 + KT : A.T) - 1;
      const int va = A.v.tokver[t0], vb = A.v.tokver[t1];
      const int nsl = (r <= 8 && vb != va) ? 2 : 1;
      float* Ut = reinterpret_cast<float*>(pk + PK_U);
      for (int sl = 0; sl < nsl; ++sl) {
        const int v = sl ? vb : va;
        float* dst = Ut + sl * un;
        const float* src = (v == pva) ? prevU : (v == pvb ? prevU + un : nullptr);
        if (src) {
          for (int e = 4 * lane; e < un; e += 128)
            *reinterpret_cast<float4*>(dst + e) = *reinterpret_cast<const float4*>(src + e);
        } else {
          const float* Ug = ub + (size_t)v * vs;
#pragma unroll 8
          for (int e = lane; e < un; e += 32) dst[e] = __ldg(Ug + (size_t)(e & (DH - 1)) * r + (e >> 7));
        }
      }
      pva = va;
      pvb = nsl == 2 ? vb : -1;
      prevU = Ut;
    }
    __syncwarp();  // the lanes' staged basis is written before lane 0 arrives
    if (lane == 0) {
      uint64_t* bar = &bars[B_LOAD_FULL + s];
      mbar_arrive_expect_tx(bar, tx0);
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
// address field (bytes / 16; no carry out of the 14-bit field in 227 KB).  Both
// CTAs lay out their halves at the same offsets, so one descriptor addresses
// both.
struct MmaDesc {
  uint64_t k, v;
};

// S_p = Q_p K'^T for the tile in stage s: M = 256 rows of the pair, N = 64 keys
// (32 in each CTA's K' half), 8 K16 steps with A = Q from TMEM.
__device__ __forceinline__ void issue_qk(const MmaDesc& D, uint32_t tmem, int p, int s) {
  constexpr uint32_t IDQ = idesc_bf16(256, KT, false, false);
  const uint32_t tq = tmem + 256 * p, ts = tq + 64;
  const uint64_t kd = D.k + (uint64_t)((s * KVST) >> 4);
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const uint32_t koff = ((k >> 2) * (KH * 128) + (k & 3) * 32) >> 4;
    mma2_bf16_ts(ts, tq + 8 * k, kd + koff, IDQ, k > 0);
  }
}

// O_p += P_p V' (stage s): M = 256, N = 128 channels (64 in each CTA's V' half),
// 4 K16 steps over the tile's keys with A = P from TMEM.
__device__ __forceinline__ void issue_pv(const MmaDesc& D, uint32_t tmem, int p, int s,
                                         bool first) {
  constexpr uint32_t IDP = idesc_bf16(256, DH, false, true);
  const uint32_t ts = tmem + 256 * p + 64, to = tmem + 256 * p + 128;
  const uint64_t vd = D.v + (uint64_t)((s * KVST) >> 4);
#pragma unroll
  for (int k = 0; k < KT / 16; ++k)
    mma2_bf16_ts(to, ts + 8 * k, vd + (uint64_t)((k * 16 * 128) >> 4), IDP,
                 (!first || k > 0) ? 1u : 0u);
}

// One issuing thread per Q tile p in the even CTA (warps 16 and 17), each
// running  Q K'^T(p, t) -> wait for P -> P V'(p, t) -> Q K'^T(p, t + 1) -> ...
// with blocking waits; the two threads interleave on the tensor pipes, which
// work on one Q tile while the softmax works on the other.  Q K'^T(p, t + 1)
// comes after P V'(p, t) in the thread's issue order, so an MMA that
// overwrites the S/P columns never overtakes the P V' that reads them.  A stage
// is released in both CTAs after both threads' P V' (one commit each).
__device__ __forceinline__ void mma_role(const TcArgs& A, uint8_t* smem, uint64_t* bars,
                                         uint32_t tmem, int ntile, int p) {
  // ntile: tiles of this pair's key range
  const uint32_t sbase = smem_u32(smem);
  MmaDesc D;
  D.k = desc_sw128(sbase + OFF_KV + ST_K, 16, 1024);
  D.v = desc_sw128(sbase + OFF_KV + ST_V, 16, 1024);
  bool ok = mbar_wait(&bars[B_Q_READY], 0);
  tc_fence_after();
  for (int t = 0; ok && t < ntile; ++t) {
    const int s = t % NKV;
    if (!mbar_wait(&bars[B_KV_FULL + s], (t / NKV) & 1)) { ok = false; break; }
    tc_fence_after();
    issue_qk(D, tmem, p, s);
    mma2_commit_mc(&bars[B_S_FULL + p], BOTH);
    if (!mbar_wait(&bars[B_P_FULL + p], t & 1)) { ok = false; break; }
    tc_fence_after();
    issue_pv(D, tmem, p, s, t == 0);
    mma2_commit_mc(&bars[B_KV_EMPTY + s], BOTH);
    if (t == ntile - 1) mma2_commit_mc(&bars[B_O_LAST + p], BOTH);
  }
  mma2_commit_mc(&bars[B_DONE + p], LEAD);
  if (!mbar_wait(&bars[B_DONE + p], 0)) ok = false;
  if (!ok) timeout_flag();
}

template <bool SEG>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NTHREADS, 1)
    attn_tc_kernel(const TcArgs A) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + OFF_BAR + NBAR * 8);
  const int warp = threadIdx.x / 32;
  const uint32_t rank = cluster_rank();
  const int ntile = SEG ? A.ntp + (int)((A.nseg + KT - 1) / KT) : A.ntp;
  const Work wk = work_of(A, ntile);
  if (threadIdx.x == 0) {
    for (int i = 0; i < NPK; ++i) {
      mbar_init(&bars[B_LOAD_FULL + i], 1);
      mbar_init(&bars[B_PK_EMPTY + i], NDQW);
    }
    for (int i = 0; i < NKV; ++i) {
      mbar_init(&bars[B_KV_FULL + i], 2 * NDQW);  // dequant warps of both CTAs
      mbar_init(&bars[B_KV_EMPTY + i], A.nqt);    // one commit per Q tile
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars[B_S_FULL + i], 1);
      mbar_init(&bars[B_P_FULL + i], 8);           // 4 softmax warps in each CTA
      mbar_init(&bars[B_O_LAST + i], 1);
      mbar_init(&bars[B_DONE + i], 1);
    }
    mbar_init(&bars[B_Q_READY], 16);
    fence_mbar_init();
  }
  if (warp == W_MMA) {
    tmem_alloc2(tmem_holder, 512);
    tmem_relinquish2();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers exist before any arrival crosses the pair
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  if (warp < 8) {
    softmax_role<SEG>(A, bars, tmem, wk, rank);
  } else if (warp < 8 + NDQW) {
    dequant_role<SEG>(A, smem, bars, wk, rank);
  } else if (warp < W_PROD) {
    const int p = warp - W_MMA;
    if (rank == 0 && (threadIdx.x & 31) == 0 && p < A.nqt) mma_role(A, smem, bars, tmem, wk.n, p);
    __syncwarp();
  } else {
    producer_role(A, smem, bars, wk);
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // no MMA of the pair reads this CTA's memory any more
  if (warp == W_MMA) {
    tc_fence_after();
    tmem_dealloc2(tmem, 512);
  }
}

// Merge of the key ranges' partials: for each (query row, head) one warp, lane
// l holding channels 4l .. 4l+3.  With L_c the ranges' log-sum-exps and O_c
// their normalized outputs, O = sum_c e^(L_c - L) O_c / sum_c e^(L_c - L) and
// the row's log-sum-exp is L + ln sum_c e^(L_c - L), L = max_c L_c.
__global__ void __launch_bounds__(256) attn_merge_kernel(const float* __restrict__ ws_o,
                                                         const float* __restrict__ ws_l,
                                                         int nsplit, int64_t rows,
                                                         uint16_t* __restrict__ O,
                                                         float* __restrict__ lse) {
  const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);  // q * H + h
  if (row >= rows) return;
  const int lane = threadIdx.x & 31;
  float L = -INFINITY;
  for (int c = 0; c < nsplit; ++c) L = fmaxf(L, __ldg(ws_l + (size_t)c * rows + row));
  float den = 0.0f;
  float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
  for (int c = 0; c < nsplit; ++c) {
    const float w = expf(__ldg(ws_l + (size_t)c * rows + row) - L);
    const float4 o = __ldg(reinterpret_cast<const float4*>(ws_o + ((size_t)c * rows + row) * DH) + lane);
    den += w;
    acc.x = fmaf(w, o.x, acc.x);
    acc.y = fmaf(w, o.y, acc.y);
    acc.z = fmaf(w, o.z, acc.z);
    acc.w = fmaf(w, o.w, acc.w);
  }
  const float inv = 1.0f / den;
  uint2 out = make_uint2(pack_bf16(acc.x * inv, acc.y * inv), pack_bf16(acc.z * inv, acc.w * inv));
  *reinterpret_cast<uint2*>(O + row * DH + 4 * lane) = out;
  if (lse && lane == 0) lse[row] = L + logf(den);
}

// Number of SMs of the current device (cached per device).
int device_sms() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (!cache[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 2)
      n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

// Key ranges for `units` (row block, head) pairs of CTAs over `ntile` tiles:
// the count that minimizes (rounds of pairs on the GPU) x (tiles per range
// plus a fixed per-range cost of about 4 tiles), within the workspace.
int choose_split(int64_t units, int ntile, int64_t nq, const Dims& D) {
  if (nq > D.max_queries || ntile < 16) return 1;
  const int64_t slots = device_sms() / 2;
  int best = 1;
  double bestc = 1e300;
  for (int s = 1; s <= QWM_ATTN_MAX_SPLIT && s <= ntile / 8; ++s) {
    const double rounds = (double)((units * s + slots - 1) / slots);
    const double c = rounds * ((double)ntile / s + 4.0);
    if (c < bestc * 0.98) {
      bestc = c;
      best = s;
    }
  }
  return best;
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
  // row blocks of at most 2 x 256 rows per pair, spread evenly over the pairs
  const int64_t npairs = (nq + 2 * ROWS - 1) / (2 * ROWS);
  a.rc = (int)((nq + 2 * npairs - 1) / (2 * npairs));
  a.nqt = a.rc > QT ? 2 : 1;
  a.npairs = (int)npairs;
  const int ntile = a.ntp + (int)((sg.n + KT - 1) / KT);
  // key ranges across pairs, so that the last round of pairs on the GPU fills
  a.nsplit = choose_split(npairs * D.H, ntile, nq, D);
  a.ws_o = nullptr;
  a.ws_l = nullptr;
  if (a.nsplit > 1) {
    a.ws_o = reinterpret_cast<float*>(v.workspace);
    a.ws_l = a.ws_o + (size_t)a.nsplit * nq * D.H * DH;
  }
  // the segment variant only when there is one (no extra branches otherwise)
  auto kern = sg.n > 0 ? attn_tc_kernel<true> : attn_tc_kernel<false>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)(2 * npairs * a.nsplit), D.H);
  kern<<<grid, NTHREADS, SMEM_BYTES, s>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess || a.nsplit == 1) return e;
  const int64_t rows = nq * D.H;
  attn_merge_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, s>>>(a.ws_o, a.ws_l, a.nsplit, rows, O,
                                                               sg.lse);
  return cudaGetLastError();
}

int read_and_clear_tc_timeout() {
  int v = 0, z = 0;
  if (cudaMemcpyFromSymbol(&v, g_tc_timeout, sizeof(int)) != cudaSuccess) return -1;
  cudaMemcpyToSymbol(g_tc_timeout, &z, sizeof(int));
  return v;
}

}  // namespace qwm
