// attention_tc.cu -- attention over the packed QuantWM cache on the sm_100a
// tensor cores (tcgen05.mma, accumulators in TMEM).
//
// O = softmax(scale Q K'^T) V' with K' = C_K[a] + deq(R) + U_v (c8 cs) and
// V' = C_V[b] + deq(R_V) reconstructed on the fly (QuantWM, "Flickering after
// quantization?" (SynthePulse), PSAC paragraph: the Key error is compensated
// when the cache is reconstructed; U_v is the basis in force when the key was
// appended).
//
// The compensation term runs on the tensor cores instead of per element:
//   q . (U_v c_t) = (U_v^T q) . c_t,
// so each QK^T gains one extra K16 step (two for r > 8) whose A operand holds
// [Q U_va | Q U_vb] for the (at most two) basis versions va, vb of the tile and
// whose B operand holds each key's c8 cs in the slot of its version.  A key whose
// version is neither (a tile spanning more than two versions) is compensated
// element-wise by the dequant thread instead.
//
// One CTA per (head, 128 query rows); 416 threads in three roles:
//   warps 0-3  softmax: warp w owns TMEM lanes 32w..32w+31 = query rows; loads
//              S from TMEM, online softmax in the log2 domain, writes P (bf16)
//              to shared memory; rescales O in TMEM when a row max moves; builds
//              the [Q U_va | Q U_vb] slab two tiles ahead.
//   warps 4-11 dequant: two threads per key row of each 128-key tile (64
//              channels each) issue all their loads first, then write K-hat and
//              V' (bf16) straight into the 128B-swizzled layout the UMMA
//              descriptors read, plus the key's compensation slab row.
//   warp 12    MMA: one thread issues S = Q K'^T and O += P V' (V' read
//              MN-major) and commits to mbarriers.
// K-hat/V' tiles, the slabs and S are double-buffered, so the QK^T of tile j+1
// runs while the softmax works on tile j.  TMEM: S[2] at columns 0/128, O at
// 256 (512 columns; one CTA per SM by shared memory).  Every mbarrier wait is
// bounded (about 1 s); a timeout sets a device flag that qwm_device_status()
// reports, and every role then leaves its loop.
#include <math.h>

#include "dequant.cuh"
#include "tc.cuh"

namespace qwm {

__device__ int g_tc_timeout;

namespace {
using namespace tc;

constexpr int BQ = 128;        // query rows per CTA
constexpr int KT = 128;        // keys per tile
constexpr int DH = 128;        // head_dim handled here
constexpr int NTHREADS = 416;  // 4 softmax + 8 dequant + 1 MMA warps
constexpr int NDQ = 256;       // dequant threads: two per key row
constexpr uint32_t TILE = 128 * 128 * 2;   // one bf16 128x128 tile
constexpr uint32_t XSLAB = 128 * 32 * 2;   // [128][<=32] bf16 compensation slab
constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_K = OFF_Q + TILE;         // 2 slots
constexpr uint32_t OFF_V = OFF_K + 2 * TILE;     // 2 slots
constexpr uint32_t OFF_AX = OFF_V + 2 * TILE;    // 2 buffers (by tile parity)
constexpr uint32_t OFF_BX = OFF_AX + 2 * XSLAB;  // 2 slots (with K-hat/V')
constexpr uint32_t OFF_BAR = OFF_BX + 2 * XSLAB;
constexpr int NBAR = 16;
constexpr uint32_t SMEM_BYTES = OFF_BAR + NBAR * 8 + 16 + 1024;

enum {
  B_KV_FULL = 0,  // [2] dequant (one arrival per warp) -> MMA
  B_KV_EMPTY = 2, // [2] MMA commit -> dequant
  B_S_FULL = 4,   // [2] MMA commit -> softmax
  B_P_FULL = 6,   // [2] softmax (per warp) -> MMA: P of that parity is in TMEM
  B_AX_FULL = 8,  // [2] softmax (per warp) -> MMA: slab for the tile of that parity
  B_O_FULL = 11,  // MMA commit after each P V'
  B_Q_READY = 12, // softmax (per warp) -> MMA
  B_DONE = 13,    // MMA commit -> MMA (drain before exit)
  B_O_LAST = 14   // MMA commit after the last P V'
};

struct TcArgs {
  Dims Dm;
  CacheView v;
  int64_t T;
  const uint16_t* Q;
  int64_t nq;
  float scale_log2;
  uint16_t* O;
  int kx;  // extra K width for the compensation (0, 16 or 32)
};

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

// byte offset of 16-byte chunk c (8 bf16) of row r in a no-swizzle K-major slab
// with kx columns: core matrices of 8 rows x 16 B, K-adjacent cores 128 B apart,
// 8-row groups kx*16 B apart.
__device__ __forceinline__ uint32_t xslab_off(int r, int c, int kx) {
  return (uint32_t)((r >> 3) * (kx * 16) + c * 128 + (r & 7) * 16);
}

// versions in force for the first and the last key of tile j
__device__ __forceinline__ void tile_versions(const uint16_t* tokver, int64_t T, int j, int& va,
                                              int& vb) {
  const int64_t t0 = (int64_t)j * KT;
  const int64_t t1 = ((t0 + KT) < T ? (t0 + KT) : T) - 1;
  va = tokver[t0];
  vb = tokver[t1];
}

// 32 lanes x 32 fp32 columns to TMEM (the store wait is part of the statement).
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};\n\t"
      "tcgen05.wait::st.sync.aligned;" ::"r"(taddr),
      "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]),
      "f"(v[8]), "f"(v[9]), "f"(v[10]), "f"(v[11]), "f"(v[12]), "f"(v[13]), "f"(v[14]),
      "f"(v[15]), "f"(v[16]), "f"(v[17]), "f"(v[18]), "f"(v[19]), "f"(v[20]), "f"(v[21]),
      "f"(v[22]), "f"(v[23]), "f"(v[24]), "f"(v[25]), "f"(v[26]), "f"(v[27]), "f"(v[28]),
      "f"(v[29]), "f"(v[30]), "f"(v[31])
      : "memory");
}

// ------------------------------------------------------------------ softmax role
// The exponent reference m_used of a row moves only when the row maximum has
// grown by more than TAU (log2 units); P then stays below 2^TAU and O, which
// accumulates in TMEM across tiles, is rescaled in place only on such moves.
constexpr float TAU = 8.0f;

// Slot `sl` (columns [sl*sw, sl*sw + sw), sw = kx/2) of row `row` of the slab
// [Q U_va | Q U_vb] for one tile: (U_v^T q) for version v, zeros when v < 0 or
// past r.
__device__ __forceinline__ void build_ax(const TcArgs& A, uint8_t* slab, int row, int64_t q,
                                         int v, int sl) {
  const Dims& Dm = A.Dm;
  const int r = Dm.r, kx = A.kx, sw = kx / 2, h = blockIdx.y;
  float acc[16];
#pragma unroll
  for (int k = 0; k < 16; ++k) acc[k] = 0.0f;
  if (q < A.nq && v >= 0) {
    const uint4* qrow = reinterpret_cast<const uint4*>(A.Q + ((size_t)q * Dm.H + h) * DH);
    const float* Uv = basis_of(A.v, Dm, v, h);
    for (int c = 0; c < 16; ++c) {
      const uint4 w = __ldg(qrow + c);
      const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float qv = __uint_as_float(e & 1 ? (ww[e / 2] & 0xffff0000u) : (ww[e / 2] << 16));
        const float* Uj = Uv + (c * 8 + e) * r;
#pragma unroll
        for (int k = 0; k < 16; ++k)
          if (k < r) acc[k] = fmaf(qv, __ldg(Uj + k), acc[k]);
      }
    }
  }
#pragma unroll
  for (int c = 0; c < 2; ++c) {
    if (c < sw / 8)
      *reinterpret_cast<uint4*>(slab + xslab_off(row, sl * (sw / 8) + c, kx)) = make_uint4(
          pack_bf16(acc[8 * c], acc[8 * c + 1]), pack_bf16(acc[8 * c + 2], acc[8 * c + 3]),
          pack_bf16(acc[8 * c + 4], acc[8 * c + 5]), pack_bf16(acc[8 * c + 6], acc[8 * c + 7]));
  }
}

__device__ __forceinline__ void build_ax_pair(const TcArgs& A, uint8_t* slab, int row, int64_t q,
                                              int va, int vb) {
  build_ax(A, slab, row, q, va, 0);
  build_ax(A, slab, row, q, vb != va ? vb : -1, 1);
}

__device__ __forceinline__ void softmax_role(const TcArgs& A, uint8_t* smem, uint64_t* bars,
                                             uint32_t tmem, int ntile) {
  const int row = threadIdx.x;  // 0..127
  const int warp = row / 32;
  const int h = blockIdx.y;
  const int H = A.Dm.H;
  const int64_t q = (int64_t)blockIdx.x * BQ + row;
  {
    const uint4* src = reinterpret_cast<const uint4*>(A.Q + ((size_t)q * H + h) * DH);
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      uint4 val = make_uint4(0, 0, 0, 0);
      if (q < A.nq) val = __ldg(src + c);
      *reinterpret_cast<uint4*>(smem + OFF_Q + sw128_off(row, c, BQ)) = val;
    }
  }
  // (va, vb) pair held by slab buffer 0 and 1, packed as va | vb << 16
  uint32_t ax_pair0 = 0xffffffffu, ax_pair1 = 0xffffffffu;
  if (A.kx) {
    for (int j = 0; j < 2 && j < ntile; ++j) {
      int va, vb;
      tile_versions(A.v.tokver, A.T, j, va, vb);
      build_ax_pair(A, smem + OFF_AX + j * XSLAB, row, q, va, vb);
      if (j == 0) ax_pair0 = (uint32_t)va | ((uint32_t)vb << 16);
      else ax_pair1 = (uint32_t)va | ((uint32_t)vb << 16);
    }
  }
  fence_proxy_async_smem();
  warp_arrive(&bars[B_Q_READY]);
  if (A.kx) {
    warp_arrive(&bars[B_AX_FULL + 0]);
    if (ntile > 1) warp_arrive(&bars[B_AX_FULL + 1]);
  }

  float m_used = -INFINITY, l = 0.0f;
  const uint32_t trow = tmem + ((uint32_t)(32 * warp) << 16);
  const uint32_t to = trow + 256;  // O accumulator columns
  const float sl2 = A.scale_log2;
  bool ok = true;
  for (int j = 0; j < ntile; ++j) {
    const int b = j & 1;
    bool w = mbar_wait(&bars[B_S_FULL + b], (j >> 1) & 1);
    if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
    tc_fence_after();
    const int64_t kb = (int64_t)j * KT;
    const int nvalid = (int)((A.T - kb) < KT ? (A.T - kb) : KT);
    float mx = -INFINITY;
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      float s[64];
      tmem_ld64(trow + b * 128 + c * 64, s);
#pragma unroll
      for (int e = 0; e < 64; ++e)
        if (c * 64 + e < nvalid) mx = fmaxf(mx, s[e]);
    }
    const float m_row = mx * sl2;
    if (j == 0) {
      m_used = m_row;
    } else {
      const bool need = m_row > m_used + TAU;
      if (__any_sync(0xffffffffu, need)) {
        // O holds P V' of tiles < j: wait for the last of them, then rescale.
        // S_FULL(j) implies P V' of tile j-2 is done (commits track all earlier
        // MMAs) and P V' of tile j cannot start before P_FULL(j), so O_FULL sits
        // in phase j-1 or j and the parity test is exact.
        bool w2 = mbar_wait(&bars[B_O_FULL], (j - 1) & 1);
        if (!__all_sync(0xffffffffu, w2)) { ok = false; break; }
        tc_fence_after();
        const float f = need ? ex2(m_used - m_row) : 1.0f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float o[32];
          tmem_ld32(to + c * 32, o);
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] *= f;
          tmem_st32(to + c * 32, o);
        }
        l *= f;
        if (need) m_used = m_row;
      }
    }
    // P (bf16 pairs) overwrites the S columns already read: keys 2i, 2i+1 of
    // the tile go to column i of the same TMEM buffer (the A-operand layout of
    // the P V' MMA).
    float lsum = 0.0f;
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      float s[32];
      tmem_ld32(trow + b * 128 + c * 32, s);
      uint32_t pk[16];
#pragma unroll
      for (int e = 0; e < 32; e += 2) {
        const int col = c * 32 + e;
        const float p0 = (col < nvalid) ? ex2(fmaf(s[e], sl2, -m_used)) : 0.0f;
        const float p1 = (col + 1 < nvalid) ? ex2(fmaf(s[e + 1], sl2, -m_used)) : 0.0f;
        lsum += p0 + p1;
        pk[e / 2] = pack_bf16(p0, p1);
      }
      tmem_st16u(trow + b * 128 + c * 16, pk);
    }
    l += lsum;
    tc_fence_before();
    warp_arrive(&bars[B_P_FULL + b]);
    // slab for tile j+2 into buffer b (QK^T of tile j, its last reader, is done)
    if (A.kx && j + 2 < ntile) {
      int va, vb;
      tile_versions(A.v.tokver, A.T, j + 2, va, vb);
      const uint32_t pair = (uint32_t)va | ((uint32_t)vb << 16);
      if (pair != (b ? ax_pair1 : ax_pair0)) {
        build_ax_pair(A, smem + OFF_AX + b * XSLAB, row, q, va, vb);
        if (b) ax_pair1 = pair;
        else ax_pair0 = pair;
        fence_proxy_async_smem();
      }
      warp_arrive(&bars[B_AX_FULL + b]);
    }
  }
  if (ok) {
    bool w = mbar_wait(&bars[B_O_LAST], 0);
    ok = __all_sync(0xffffffffu, w);
  }
  if (!ok) {
    if (row == 0) timeout_flag();
    return;
  }
  tc_fence_after();
  const float inv = 1.0f / l;
  uint4* dst = reinterpret_cast<uint4*>(A.O + ((size_t)q * H + h) * DH);
#pragma unroll
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
// exact float of a 2-bit code: (2^23 + code) - 2^23
__device__ __forceinline__ float code_f(uint32_t bits, int e) {
  return __uint_as_float(0x4B000000u | ((bits >> (2 * e)) & 3u)) - 8388608.0f;
}

__device__ __forceinline__ void dequant_role(const TcArgs& A, uint8_t* smem, uint64_t* bars,
                                             int ntile) {
  const int dq = threadIdx.x - 128;  // 0..255
  const int dt = dq >> 1;            // key row in the tile
  const int hf = dq & 1;             // channel half [64 hf, 64 hf + 64)
  const Dims& Dm = A.Dm;
  const int h = blockIdx.y;
  const PackedHead p = packed_head(A.v, Dm, h);
  const int G = Dm.G, ng = Dm.ng, r = Dm.r, kx = A.kx;
  for (int j = 0; j < ntile; ++j) {
    const int slot = j & 1;
    if (j >= 2) {
      const bool w = mbar_wait(&bars[B_KV_EMPTY + slot], ((j - 2) >> 1) & 1);
      if (!__all_sync(0xffffffffu, w)) {
        timeout_flag();
        return;
      }
    }
    uint8_t* kb = smem + OFF_K + slot * TILE;
    uint8_t* vb = smem + OFF_V + slot * TILE;
    uint8_t* xb = smem + OFF_BX + slot * XSLAB;
    const int64_t t = (int64_t)j * KT + dt;
    if (t < A.T) {
      // ---- all loads of this half-row first (memory-level parallelism)
      const int a = load_idx(p.k_idx, t, Dm.idx_bytes);
      const int bi = load_idx(p.v_idx, t, Dm.idx_bytes);
      const uint4* ck = reinterpret_cast<const uint4*>(p.cent_k + (size_t)a * DH) + hf * 8;
      const uint4* cv = reinterpret_cast<const uint4*>(p.cent_v + (size_t)bi * DH) + hf * 8;
      uint4 kc[8], vc[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        kc[c] = __ldg(ck + c);
        vc[c] = __ldg(cv + c);
      }
      const uint4 kw4 = __ldg(reinterpret_cast<const uint4*>(p.k_codes + t * (DH / 4)) + hf);
      const uint4 vw4 = __ldg(reinterpret_cast<const uint4*>(p.v_codes + t * (DH / 4)) + hf);
      const uint32_t* kpar = reinterpret_cast<const uint32_t*>(p.k_params) + t * ng;
      const uint32_t* vpar = reinterpret_cast<const uint32_t*>(p.v_params) + t * ng;
      const int ver = A.v.tokver[t];
      bool fallback = false;
      float chat[16];
#pragma unroll
      for (int k = 0; k < 16; ++k) chat[k] = 0.0f;
      if (r > 0) {
        int va, vbv;
        tile_versions(A.v.tokver, A.T, j, va, vbv);
        fallback = (ver != va) && (ver != vbv);
        if (hf == 0 || fallback) {
          const float cs = h2f(p.k_cscale[t]);
#pragma unroll
          for (int k = 0; k < 16; ++k)
            if (k < r) chat[k] = (float)p.k_coef[t * r + k] * cs;
        }
        if (hf == 0) {
          // compensation slab row: c8 cs in the slot of the key's version
          const int sw = kx / 2;
          const int sl = (ver == va) ? 0 : ((ver == vbv) ? 1 : -1);
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            if (c < kx / 8) {
              const int cs0 = c - (sl >= 0 ? sl * (sw / 8) : 0);
              const bool mine = sl >= 0 && cs0 >= 0 && cs0 < sw / 8;
              float x[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                float v = 0.0f;
#pragma unroll
                for (int m = 0; m < 16; ++m)
                  if (mine && m == cs0 * 8 + e) v = chat[m];
                x[e] = v;
              }
              *reinterpret_cast<uint4*>(xb + xslab_off(dt, c, kx)) =
                  make_uint4(pack_bf16(x[0], x[1]), pack_bf16(x[2], x[3]), pack_bf16(x[4], x[5]),
                             pack_bf16(x[6], x[7]));
            }
          }
        }
      }
      const float* U = basis_of(A.v, Dm, ver, h);
      const uint32_t kwv[4] = {kw4.x, kw4.y, kw4.z, kw4.w};
      const uint32_t vwv[4] = {vw4.x, vw4.y, vw4.z, vw4.w};
#pragma unroll
      for (int cc = 0; cc < 8; ++cc) {
        const int c = hf * 8 + cc;  // chunk of 8 channels within the row
        const int j0 = c * 8;
        const int g = j0 / G;
        const uint32_t kp = __ldg(kpar + g), vp = __ldg(vpar + g);
        const float kmn = h2f((uint16_t)(kp & 0xffff)), ksc = h2f((uint16_t)(kp >> 16));
        const float vmn = h2f((uint16_t)(vp & 0xffff)), vsc = h2f((uint16_t)(vp >> 16));
        const uint32_t kbits = (kwv[cc / 2] >> (16 * (cc & 1))) & 0xffff;
        const uint32_t vbits = (vwv[cc / 2] >> (16 * (cc & 1))) & 0xffff;
        const uint32_t kw[4] = {kc[cc].x, kc[cc].y, kc[cc].z, kc[cc].w};
        const uint32_t vw[4] = {vc[cc].x, vc[cc].y, vc[cc].z, vc[cc].w};
        float kxv[8], vxv[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float kcf = __uint_as_float(e & 1 ? (kw[e / 2] & 0xffff0000u) : (kw[e / 2] << 16));
          const float vcf = __uint_as_float(e & 1 ? (vw[e / 2] & 0xffff0000u) : (vw[e / 2] << 16));
          kxv[e] = kcf + fmaf(code_f(kbits, e), ksc, kmn);
          vxv[e] = vcf + fmaf(code_f(vbits, e), vsc, vmn);
        }
        if (fallback) {  // a third basis version in this tile: compensate here
          for (int e = 0; e < 8; ++e) {
            float corr = 0.0f;
#pragma unroll
            for (int k = 0; k < 16; ++k)
              if (k < r) corr = fmaf(__ldg(U + (size_t)(j0 + e) * r + k), chat[k], corr);
            kxv[e] += corr;
          }
        }
        *reinterpret_cast<uint4*>(kb + sw128_off(dt, c, KT)) =
            make_uint4(pack_bf16(kxv[0], kxv[1]), pack_bf16(kxv[2], kxv[3]),
                       pack_bf16(kxv[4], kxv[5]), pack_bf16(kxv[6], kxv[7]));
        *reinterpret_cast<uint4*>(vb + sw128_off(dt, c, KT)) =
            make_uint4(pack_bf16(vxv[0], vxv[1]), pack_bf16(vxv[2], vxv[3]),
                       pack_bf16(vxv[4], vxv[5]), pack_bf16(vxv[6], vxv[7]));
      }
    } else {
#pragma unroll
      for (int cc = 0; cc < 8; ++cc) {
        *reinterpret_cast<uint4*>(kb + sw128_off(dt, hf * 8 + cc, KT)) = make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4*>(vb + sw128_off(dt, hf * 8 + cc, KT)) = make_uint4(0, 0, 0, 0);
      }
      if (hf == 0) {
#pragma unroll
        for (int c = 0; c < 4; ++c)
          if (c < kx / 8)
            *reinterpret_cast<uint4*>(xb + xslab_off(dt, c, kx)) = make_uint4(0, 0, 0, 0);
      }
    }
    fence_proxy_async_smem();
    warp_arrive(&bars[B_KV_FULL + slot]);
  }
}

// ------------------------------------------------------------------ MMA role
// S[j&1] = Q K-hat_j^T (8 K16 steps over head_dim, two 64-wide swizzled blocks)
// + the compensation steps [Q U_va | Q U_vb] [c slots]^T.
__device__ __forceinline__ void issue_qk(uint64_t* bars, uint32_t sbase, uint32_t tmem, int j,
                                         int kx) {
  constexpr uint32_t IDQ = idesc_bf16(128, 128, false, false);
  const int slot = j & 1;
  const uint32_t sq = sbase + OFF_Q, sk = sbase + OFF_K + slot * TILE;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const uint32_t koff = (k >> 2) * (128 * 128) + (k & 3) * 32;
    mma_bf16_ss(tmem + slot * 128, desc_sw128(sq + koff, 16, 1024),
                desc_sw128(sk + koff, 16, 1024), IDQ, k > 0);
  }
  const uint32_t sa = sbase + OFF_AX + slot * XSLAB, sb = sbase + OFF_BX + slot * XSLAB;
  for (int k = 0; k < kx / 16; ++k)
    mma_bf16_ss(tmem + slot * 128, desc_noswz(sa + k * 256, 128, kx * 16),
                desc_noswz(sb + k * 256, 128, kx * 16), IDQ, 1u);
  mma_commit(&bars[B_S_FULL + slot]);
}

// O += P_j V'_j with P read from TMEM (the S buffer of tile j).
__device__ __forceinline__ void issue_pv(uint64_t* bars, uint32_t sbase, uint32_t tmem, int j,
                                         int ntile) {
  constexpr uint32_t IDP = idesc_bf16(128, 128, false, true);
  const int b = j & 1;
  const uint32_t sv = sbase + OFF_V + b * TILE;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    // P of keys 16k..16k+15: TMEM columns b*128 + 8k .. +7 (bf16 pairs)
    mma_bf16_ts(tmem + 256, tmem + b * 128 + k * 8, desc_sw128(sv + k * 2048, KT * 128, 1024),
                IDP, (j > 0 || k > 0) ? 1u : 0u);
  }
  mma_commit(&bars[B_O_FULL]);
  mma_commit(&bars[B_KV_EMPTY + b]);
  if (j == ntile - 1) mma_commit(&bars[B_O_LAST]);
}

// ------------------------------------------------------------------ MMA role
// Issues whichever MMA group is ready.  Constraints: QK^T of tile j after P V'
// of tile j-2 has been issued (S/P buffer j&1 is reused; the tensor pipe runs
// in issue order); P V' of tile j after its P is in TMEM.
__device__ __forceinline__ void mma_role(uint8_t* smem, uint64_t* bars, uint32_t tmem, int ntile,
                                         int kx) {
  const uint32_t sbase = smem_u32(smem);
  bool ok = mbar_wait(&bars[B_Q_READY], 0);
  int qn = 0, pn = 0;  // next QK^T tile, next P V' tile
  long long t_idle = 0;
  while (ok && pn < ntile) {
    bool progress = false;
    if (qn < ntile && qn < pn + 2) {
      const int slot = qn & 1;
      if (mbar_test(&bars[B_KV_FULL + slot], (qn >> 1) & 1) &&
          (!kx || mbar_test(&bars[B_AX_FULL + slot], (qn >> 1) & 1))) {
        tc_fence_after();
        issue_qk(bars, sbase, tmem, qn, kx);
        ++qn;
        progress = true;
      }
    }
    if (pn < qn && mbar_test(&bars[B_P_FULL + (pn & 1)], (pn >> 1) & 1)) {
      tc_fence_after();
      issue_pv(bars, sbase, tmem, pn, ntile);
      ++pn;
      progress = true;
    }
    if (progress) {
      t_idle = 0;
    } else if (t_idle == 0) {
      t_idle = clock64();
    } else if (clock64() - t_idle > (1ll << 31)) {
      ok = false;
    }
  }
  mma_commit(&bars[B_DONE]);
  if (!mbar_wait(&bars[B_DONE], 0)) ok = false;
  if (!ok) timeout_flag();
}

__global__ void __launch_bounds__(NTHREADS, 1) attn_tc_kernel(const TcArgs A) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + OFF_BAR + NBAR * 8);
  const int warp = threadIdx.x / 32;
  const int ntile = (int)((A.T + KT - 1) / KT);
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars[B_KV_FULL + i], NDQ / 32);
      mbar_init(&bars[B_KV_EMPTY + i], 1);
      mbar_init(&bars[B_S_FULL + i], 1);
      mbar_init(&bars[B_P_FULL + i], 4);
      mbar_init(&bars[B_AX_FULL + i], 4);
    }
    mbar_init(&bars[B_O_FULL], 1);
    mbar_init(&bars[B_Q_READY], 4);
    mbar_init(&bars[B_DONE], 1);
    mbar_init(&bars[B_O_LAST], 1);
    fence_mbar_init();
  }
  if (warp == 12) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  if (warp < 4) {
    softmax_role(A, smem, bars, tmem, ntile);
  } else if (warp < 12) {
    dequant_role(A, smem, bars, ntile);
  } else if ((threadIdx.x & 31) == 0) {
    mma_role(smem, bars, tmem, ntile, A.kx);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 12) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

bool attention_tc_supported(const Dims& D) { return D.d == DH; }

cudaError_t launch_attention_tc(const Dims& D, const CacheView& v, int64_t T, const uint16_t* Q,
                                int64_t nq, float scale, uint16_t* O, cudaStream_t s) {
  TcArgs a;
  a.Dm = D;
  a.v = v;
  a.T = T;
  a.Q = Q;
  a.nq = nq;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.O = O;
  a.kx = (D.r == 0) ? 0 : (D.r <= 8 ? 16 : 32);  // two slots of 8 or 16 columns
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)SMEM_BYTES);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)((nq + BQ - 1) / BQ), D.H);
  attn_tc_kernel<<<grid, NTHREADS, SMEM_BYTES, s>>>(a);
  return cudaGetLastError();
}

int read_and_clear_tc_timeout() {
  int v = 0, z = 0;
  if (cudaMemcpyFromSymbol(&v, g_tc_timeout, sizeof(int)) != cudaSuccess) return -1;
  cudaMemcpyToSymbol(g_tc_timeout, &z, sizeof(int));
  return v;
}

}  // namespace qwm
