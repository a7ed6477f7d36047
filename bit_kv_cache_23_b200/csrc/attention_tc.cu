// attention_tc.cu -- attention over the packed QuantWM cache on the sm_100a
// tensor cores (tcgen05.mma, accumulators in TMEM).
//
// O = softmax(scale Q K'^T) V' with K' = C_K[a] + deq(R) + U_v (c8 cs) and
// V' = C_V[b] + deq(R_V) reconstructed on the fly (QuantWM, "Flickering after
// quantization?" (SynthePulse), PSAC paragraph: the Key error is compensated
// when the cache is reconstructed; U_v is the basis in force when the key was
// appended).
//
// One CTA per (head, 128 query rows); 288 threads in three roles:
//   warps 0-3  softmax: warp w owns TMEM lanes 32w..32w+31 = query rows; loads
//              S from TMEM, online softmax in the log2 domain, writes P (bf16)
//              to shared memory; rescales O in TMEM when a row max moves.
//   warps 4-7  dequant: thread i reconstructs key row i of each 128-key tile
//              (K' and V', bf16) straight into the 128B-swizzled shared-memory
//              layout the UMMA descriptors read.
//   warp 8     MMA: one thread issues S = Q K'^T (8 x K16 steps, M=128, N=128)
//              and O += P V' (V' read MN-major), commits to mbarriers.
// Buffers: K'/V' tiles, S and P are double-buffered, so the QK^T of tile j+1
// runs while the softmax works on tile j.  O accumulates in TMEM across all
// tiles.  TMEM: S[2] at columns 0/128, O at 256 (512 columns allocated; one
// CTA per SM by shared memory).
// Every mbarrier wait is bounded (about 1 s); a timeout sets a device flag
// that qwm_device_status() reports, and every role then leaves its loop.
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
constexpr int NTHREADS = 288;
constexpr uint32_t TILE = 128 * 128 * 2;  // one bf16 128x128 tile
constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_K = OFF_Q + TILE;          // 2 slots
constexpr uint32_t OFF_V = OFF_K + 2 * TILE;      // 2 slots
constexpr uint32_t OFF_P = OFF_V + 2 * TILE;      // 2 buffers
constexpr uint32_t OFF_BAR = OFF_P + 2 * TILE;
constexpr int NBAR = 16;
constexpr uint32_t SMEM_BYTES = OFF_BAR + NBAR * 8 + 16 + 1024;

enum {
  B_KV_FULL = 0,  // [2] dequant -> MMA (128 arrivals)
  B_KV_EMPTY = 2, // [2] MMA commit -> dequant
  B_S_FULL = 4,   // [2] MMA commit -> softmax
  B_S_FREE = 6,   // [2] softmax (128) -> MMA
  B_P_FULL = 8,   // [2] softmax (128) -> MMA
  B_O_FULL = 10,  // MMA commit after each P V' -> softmax (rescale, epilogue)
  B_Q_READY = 11, // softmax (128) -> MMA
  B_DONE = 12,    // MMA commit -> MMA (drain before exit)
  B_O_LAST = 13   // MMA commit after the last P V' -> softmax epilogue
};

struct TcArgs {
  Dims Dm;
  CacheView v;
  int64_t T;
  const uint16_t* Q;
  int64_t nq;
  float scale_log2;
  uint16_t* O;
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm volatile("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ void timeout_flag() { atomicExch(&g_tc_timeout, 1); }

// ------------------------------------------------------------------ softmax role
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

// The exponent reference m_used of a row moves only when the row maximum has
// grown by more than TAU (log2 units); P then stays below 2^TAU and O, which
// accumulates in TMEM across tiles, is rescaled in place only on such moves.
constexpr float TAU = 8.0f;

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
  fence_proxy_async_smem();
  mbar_arrive(&bars[B_Q_READY]);

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
    for (int c = 0; c < 4; ++c) {
      float s[32];
      tmem_ld32(trow + b * 128 + c * 32, s);
#pragma unroll
      for (int e = 0; e < 32; ++e)
        if (c * 32 + e < nvalid) mx = fmaxf(mx, s[e]);
    }
    const float m_row = mx * sl2;
    if (j == 0) {
      m_used = m_row;
    } else {
      const bool need = m_row > m_used + TAU;
      if (__any_sync(0xffffffffu, need)) {
        // O holds P V' of tiles < j: wait for the last of them, then rescale.
        // S_FULL(j) already implies P V' of tile j-2 is done (commits track all
        // earlier MMAs) and P V' of tile j cannot start before P_FULL(j), so
        // the barrier sits in phase j-1 or j and the parity test is exact.
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
    float lsum = 0.0f;
    uint8_t* pb = smem + OFF_P + b * TILE;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      float s[32];
      tmem_ld32(trow + b * 128 + c * 32, s);
      uint32_t pk[16];
#pragma unroll
      for (int e = 0; e < 32; e += 2) {
        float p0 = (c * 32 + e < nvalid) ? ex2(fmaf(s[e], sl2, -m_used)) : 0.0f;
        float p1 = (c * 32 + e + 1 < nvalid) ? ex2(fmaf(s[e + 1], sl2, -m_used)) : 0.0f;
        lsum += p0 + p1;
        pk[e / 2] = pack_bf16(p0, p1);
      }
#pragma unroll
      for (int k = 0; k < 4; ++k)
        *reinterpret_cast<uint4*>(pb + sw128_off(row, c * 4 + k, BQ)) =
            make_uint4(pk[4 * k], pk[4 * k + 1], pk[4 * k + 2], pk[4 * k + 3]);
    }
    l += lsum;
    tc_fence_before();
    mbar_arrive(&bars[B_S_FREE + b]);
    fence_proxy_async_smem();
    mbar_arrive(&bars[B_P_FULL + b]);
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
__device__ __forceinline__ void dequant_role(const TcArgs& A, uint8_t* smem, uint64_t* bars, int ntile) {
  const int dt = threadIdx.x - 128;  // key row in the tile
  const Dims& Dm = A.Dm;
  const int h = blockIdx.y;
  const PackedHead p = packed_head(A.v, Dm, h);
  const int G = Dm.G, ng = Dm.ng, r = Dm.r;
  for (int j = 0; j < ntile; ++j) {
    const int slot = j & 1;
    if (j >= 2) {
      if (!mbar_wait(&bars[B_KV_EMPTY + slot], ((j - 2) >> 1) & 1)) {
        timeout_flag();
        return;
      }
    }
    uint8_t* kb = smem + OFF_K + slot * TILE;
    uint8_t* vb = smem + OFF_V + slot * TILE;
    const int64_t t = (int64_t)j * KT + dt;
    if (t < A.T) {
      const int a = load_idx(p.k_idx, t, Dm.idx_bytes);
      const int bi = load_idx(p.v_idx, t, Dm.idx_bytes);
      const float* U = basis_of(A.v, Dm, A.v.tokver[t], h);
      float chat[16];
      const float cs = h2f(p.k_cscale[t]);
#pragma unroll
      for (int qq = 0; qq < 16; ++qq) chat[qq] = (qq < r) ? (float)p.k_coef[t * r + qq] * cs : 0.0f;
      const uint4* kc4 = reinterpret_cast<const uint4*>(p.k_codes + t * (DH / 4));
      const uint4* vc4 = reinterpret_cast<const uint4*>(p.v_codes + t * (DH / 4));
      uint32_t kcode[8], vcode[8];
      {
        uint4 x0 = __ldg(kc4), x1 = __ldg(kc4 + 1), y0 = __ldg(vc4), y1 = __ldg(vc4 + 1);
        kcode[0] = x0.x; kcode[1] = x0.y; kcode[2] = x0.z; kcode[3] = x0.w;
        kcode[4] = x1.x; kcode[5] = x1.y; kcode[6] = x1.z; kcode[7] = x1.w;
        vcode[0] = y0.x; vcode[1] = y0.y; vcode[2] = y0.z; vcode[3] = y0.w;
        vcode[4] = y1.x; vcode[5] = y1.y; vcode[6] = y1.z; vcode[7] = y1.w;
      }
      const uint32_t* kpar = reinterpret_cast<const uint32_t*>(p.k_params) + t * ng;
      const uint32_t* vpar = reinterpret_cast<const uint32_t*>(p.v_params) + t * ng;
      const uint4* ck = reinterpret_cast<const uint4*>(p.cent_k + (size_t)a * DH);
      const uint4* cv = reinterpret_cast<const uint4*>(p.cent_v + (size_t)bi * DH);
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const int j0 = c * 8;
        const int g = j0 / G;
        const uint32_t kp = __ldg(kpar + g), vp = __ldg(vpar + g);
        const float kmn = h2f((uint16_t)(kp & 0xffff)), ksc = h2f((uint16_t)(kp >> 16));
        const float vmn = h2f((uint16_t)(vp & 0xffff)), vsc = h2f((uint16_t)(vp >> 16));
        const uint32_t kbits = (kcode[c / 2] >> (16 * (c & 1))) & 0xffff;
        const uint32_t vbits = (vcode[c / 2] >> (16 * (c & 1))) & 0xffff;
        const uint4 kcv = __ldg(ck + c), vcv = __ldg(cv + c);
        const uint32_t kw[4] = {kcv.x, kcv.y, kcv.z, kcv.w};
        const uint32_t vw[4] = {vcv.x, vcv.y, vcv.z, vcv.w};
        float kx[8], vx[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float kc = __uint_as_float(e & 1 ? (kw[e / 2] & 0xffff0000u) : (kw[e / 2] << 16));
          const float vc = __uint_as_float(e & 1 ? (vw[e / 2] & 0xffff0000u) : (vw[e / 2] << 16));
          kx[e] = kc + fmaf((float)((kbits >> (2 * e)) & 3), ksc, kmn);
          vx[e] = vc + fmaf((float)((vbits >> (2 * e)) & 3), vsc, vmn);
        }
        if (r > 0) {
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float* Uj = U + (size_t)(j0 + e) * r;
            float corr = 0.0f;
            if (r == 8) {
              const float4 u0 = __ldg(reinterpret_cast<const float4*>(Uj));
              const float4 u1 = __ldg(reinterpret_cast<const float4*>(Uj) + 1);
              corr = fmaf(u0.x, chat[0], corr);
              corr = fmaf(u0.y, chat[1], corr);
              corr = fmaf(u0.z, chat[2], corr);
              corr = fmaf(u0.w, chat[3], corr);
              corr = fmaf(u1.x, chat[4], corr);
              corr = fmaf(u1.y, chat[5], corr);
              corr = fmaf(u1.z, chat[6], corr);
              corr = fmaf(u1.w, chat[7], corr);
            } else {
#pragma unroll
              for (int qq = 0; qq < 16; ++qq)
                if (qq < r) corr = fmaf(__ldg(Uj + qq), chat[qq], corr);
            }
            kx[e] += corr;
          }
        }
        *reinterpret_cast<uint4*>(kb + sw128_off(dt, c, KT)) =
            make_uint4(pack_bf16(kx[0], kx[1]), pack_bf16(kx[2], kx[3]),
                       pack_bf16(kx[4], kx[5]), pack_bf16(kx[6], kx[7]));
        *reinterpret_cast<uint4*>(vb + sw128_off(dt, c, KT)) =
            make_uint4(pack_bf16(vx[0], vx[1]), pack_bf16(vx[2], vx[3]),
                       pack_bf16(vx[4], vx[5]), pack_bf16(vx[6], vx[7]));
      }
    } else {
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        *reinterpret_cast<uint4*>(kb + sw128_off(dt, c, KT)) = make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4*>(vb + sw128_off(dt, c, KT)) = make_uint4(0, 0, 0, 0);
      }
    }
    fence_proxy_async_smem();
    mbar_arrive(&bars[B_KV_FULL + slot]);
  }
}

// S[j&1] = Q K'_j^T: 8 K-steps of 16 over head_dim (two 64-wide swizzled blocks).
__device__ __forceinline__ bool issue_qk(uint64_t* bars, uint32_t sq, uint32_t sk, uint32_t tmem,
                                         int j) {
  constexpr uint32_t IDQ = idesc_bf16(128, 128, false, false);
  const int slot = j & 1;
  if (!mbar_wait(&bars[B_KV_FULL + slot], (j >> 1) & 1)) return false;
  if (j >= 2 && !mbar_wait(&bars[B_S_FREE + slot], ((j - 2) >> 1) & 1)) return false;
  tc_fence_after();
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const uint32_t koff = (k >> 2) * (128 * 128) + (k & 3) * 32;
    const uint64_t da = desc_sw128(sq + koff, 16, 1024);
    const uint64_t db = desc_sw128(sk + slot * TILE + koff, 16, 1024);
    mma_bf16_ss(tmem + slot * 128, da, db, IDQ, k > 0);
  }
  mma_commit(&bars[B_S_FULL + slot]);
  return true;
}

// ------------------------------------------------------------------ MMA role
__device__ __forceinline__ void mma_role(uint8_t* smem, uint64_t* bars, uint32_t tmem, int ntile) {
  constexpr uint32_t IDP = idesc_bf16(128, 128, false, true);
  const uint32_t sq = smem_u32(smem + OFF_Q);
  const uint32_t sk = smem_u32(smem + OFF_K);
  const uint32_t sv = smem_u32(smem + OFF_V);
  const uint32_t sp = smem_u32(smem + OFF_P);
  bool ok = mbar_wait(&bars[B_Q_READY], 0);
  if (ok) ok = issue_qk(bars, sq, sk, tmem, 0);
  for (int j = 0; ok && j < ntile; ++j) {
    if (j + 1 < ntile && !(ok = issue_qk(bars, sq, sk, tmem, j + 1))) break;
    const int b = j & 1;
    if (!mbar_wait(&bars[B_P_FULL + b], (j >> 1) & 1)) { ok = false; break; }
    tc_fence_after();
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const uint64_t da = desc_sw128(sp + b * TILE + (k >> 2) * (BQ * 128) + (k & 3) * 32, 16, 1024);
      const uint64_t db = desc_sw128(sv + b * TILE + k * 2048, KT * 128, 1024);
      mma_bf16_ss(tmem + 256, da, db, IDP, (j > 0 || k > 0) ? 1u : 0u);
    }
    mma_commit(&bars[B_O_FULL]);
    mma_commit(&bars[B_KV_EMPTY + b]);
    if (j == ntile - 1) mma_commit(&bars[B_O_LAST]);
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
      mbar_init(&bars[B_KV_FULL + i], 128);
      mbar_init(&bars[B_KV_EMPTY + i], 1);
      mbar_init(&bars[B_S_FULL + i], 1);
      mbar_init(&bars[B_S_FREE + i], 128);
      mbar_init(&bars[B_P_FULL + i], 128);
    }
    mbar_init(&bars[B_O_FULL], 1);
    mbar_init(&bars[B_Q_READY], 128);
    mbar_init(&bars[B_DONE], 1);
    mbar_init(&bars[B_O_LAST], 1);
    fence_mbar_init();
  }
  if (warp == 8) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  if (warp < 4) {
    softmax_role(A, smem, bars, tmem, ntile);
  } else if (warp < 8) {
    dequant_role(A, smem, bars, ntile);
  } else if ((threadIdx.x & 31) == 0) {
    mma_role(smem, bars, tmem, ntile);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
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
