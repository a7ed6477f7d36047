// append.cu -- quantize new Keys and Values into the packed cache.
//
// Keys (QuantWM, "Flickering after quantization?" (SynthePulse), QSAC and PSAC
// paragraphs; evolve.pub review, Summary):
//   1. shortlist: the M centroids with the smallest (D_i, i), where
//      D_i = sum_j s_j (k_j - c_ij)^2 is the Query-sensitivity-weighted
//      distance, folded over j in order as acc = fma(s_j, delta*delta, acc);
//   2. choice: the candidate with the smallest expected squared logit
//      perturbation of its INT2 residual, sum_g w_g R_g^2 (R_g the residual's
//      range in group g, w_g = sum of s over the group; the constant 1/108 of
//      step^2/12 with step = R/3 is dropped), folded over groups in order;
//      ties keep the earlier shortlist position.  With the full-quadratic
//      option the score is e^T A e instead (e the Key error the candidate
//      leaves after INT2, A = fp32(M / n) in force; y_i = fold_j fma(A_ij, e_j),
//      then fold_i fma(e_i, y_i));
//   3. INT2 residual: per group mn = fp16 round-down(min), sc = fp16
//      round-up((max - mn)/3), code = #{k : rho >= mn + (k + 0.5) sc};
//   4. PSAC: e = k - (c + mn + code sc); coef_q = fold_j fma(U_jq, e_j, acc);
//      cs = fp16 round-up(max|coef| / 127); c8 = rint(coef / cs) in [-127, 127].
// Values: nearest centroid (fold fma(delta, delta, acc)), same INT2 residual.
//
// Every floating-point decision uses the operations above in that order, so
// the codes, indices and INT8 coefficients are bit-identical to the canonical
// definition.  This file is compiled with --fmad=false; the only fused
// multiply-adds are the explicit __fmaf_rn calls the definition names.
//
// Layout of the work: one CTA per (head, slice of token blocks).  The CTA
// keeps the head's centroid table in shared memory (transposed, bf16), computes
// all C distances of a block of TB tokens with one thread per centroid (so
// each thread's fold runs over the channels in order), then one warp per
// token selects the shortlist, scores it and encodes the winner.
#include "common.cuh"

namespace qwm {
namespace {

constexpr int TB = 16;        // tokens per block iteration
constexpr int NT = 256;       // threads per CTA
constexpr int NW = NT / 32;   // warps per CTA
constexpr int kMaxR = 16;
constexpr int kMaxM = 8;

struct AppendArgs {
  const uint16_t* X;      // [n][H][d] bf16 (K or V)
  const uint16_t* cent;   // [H][C][d] bf16
  const float* sens;      // [H][d]       (keys)
  const float* wgroup;    // [H][ng]      (keys)
  const float* basis;     // [H][d][r]    basis slot in force (keys)
  uint8_t* codes;         // [H][tcap][d/4]
  uint16_t* params;       // [H][tcap][ng][2]
  void* idx;              // [H][tcap]
  int8_t* coef;           // [H][tcap][r]  (keys)
  uint16_t* cscale;       // [H][tcap]     (keys)
  uint16_t* tokver;       // [tcap]        (keys)
  uint16_t* centver;      // [tcap]        (keys)
  double* eigvec;         // refresh state holding A = fp32(M / n) per head (full-quadratic)
  int64_t n, t0, tcap;
  int H, C, G, M, r, idx_bytes, version, cver, qfull;
};

__device__ __forceinline__ bool lex_less(float a, int ia, float b, int ib) {
  return a < b || (a == b && ia < ib);
}

// Full-quadratic QSAC score of one candidate, taken by one warp: lane owns
// channels lane*CPL.. and the group range (lo, hi) of its group.  The Key error
// e of the candidate goes to the warp's row `ew`; y_i = sum_j A_ij e_j is
// folded over j in order by the lane owning row i (A symmetric: row i is read
// as column i, coalesced), then lane 0 folds sum_i e_i y_i over i in order.
template <int D>
__device__ float full_score(const AppendArgs& A, int h, int lane, const float* kv,
                            const uint16_t* crow, float lo, float hi, float* ew) {
  constexpr int CPL = D / 32;
  uint16_t mnh, sch;
  float mn, sc;
  int2_params(lo, hi, mnh, sch, mn, sc);
  __syncwarp();
#pragma unroll
  for (int u = 0; u < CPL; ++u) {
    const float cv = bf2f(crow[u]);
    const float rho = __fsub_rn(kv[u], cv);
    const float deq = __fmaf_rn((float)int2_code(rho, mn, sc), sc, mn);
    ew[lane * CPL + u] = __fsub_rn(kv[u], __fadd_rn(cv, deq));
  }
  __syncwarp();
  const float* Ah = qsnap_of(A.eigvec, D, h);
  float y[CPL];
#pragma unroll
  for (int u = 0; u < CPL; ++u) {
    const int i = u * 32 + lane;
    float acc = 0.0f;
    for (int j = 0; j < D; ++j) acc = __fmaf_rn(Ah[(size_t)j * D + i], ew[j], acc);
    y[u] = acc;
  }
  float score = 0.0f;  // i = 32 u + l in increasing order
#pragma unroll
  for (int u = 0; u < CPL; ++u) {
    for (int l = 0; l < 32; ++l) {
      const float yi = __shfl_sync(0xffffffffu, y[u], l);
      score = __fmaf_rn(ew[32 * u + l], yi, score);
    }
  }
  __syncwarp();  // every lane has read `ew` before the caller reuses it
  return score;  // the same value on every lane
}

template <int D, bool KEY>
__global__ void __launch_bounds__(NT) append_kernel(AppendArgs A) {
  constexpr int CPL = D / 32;  // channels per lane (contiguous: lane*CPL ..)
  extern __shared__ __align__(16) unsigned char smem[];
  const int C = A.C, G = A.G, r = A.r, ng = D / A.G;
  uint16_t* cT = (uint16_t*)smem;                       // [D][C]
  float* ks = (float*)(smem + (size_t)D * C * 2);       // [TB][D]
  float* Ds = ks + TB * D;                              // [TB][C]
  float* s_s = Ds + TB * C;                             // [D]
  float* w_s = s_s + D;                                 // [8]  (ng <= 8)
  float* U_s = w_s + 8;                                 // [D][r]
  float* es = U_s + D * kMaxR;                          // [NW][D]
  int* cand = (int*)(es + NW * D);                      // [TB][kMaxM]

  const int h = blockIdx.y;
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const uint16_t* cent = A.cent + (size_t)h * C * D;

  for (int e = tid; e < C * D; e += NT) {
    int i = e / D, j = e % D;
    cT[j * C + i] = cent[e];
  }
  if (KEY) {
    for (int j = tid; j < D; j += NT) s_s[j] = A.sens[(size_t)h * D + j];
    if (tid < ng) w_s[tid] = A.wgroup[(size_t)h * ng + tid];
    for (int e = tid; e < D * r; e += NT) U_s[e] = A.basis[(size_t)h * D * r + e];
  }

  const int lpg = G / CPL;  // lanes per INT2 group (power of two)
  const int64_t nblk = (A.n + TB - 1) / TB;
  for (int64_t blk = blockIdx.x; blk < nblk; blk += gridDim.x) {
    const int64_t tb0 = blk * TB;
    __syncthreads();
    for (int e = tid; e < TB * D; e += NT) {
      int tt = e / D, j = e % D;
      int64_t t = tb0 + tt;
      ks[e] = (t < A.n) ? bf2f(A.X[((size_t)t * A.H + h) * D + j]) : 0.0f;
    }
    __syncthreads();
    // ---- phase 1: all C distances of the TB tokens, one thread per centroid
    for (int i = tid; i < C; i += NT) {
      float acc[TB];
#pragma unroll
      for (int tt = 0; tt < TB; ++tt) acc[tt] = 0.0f;
      for (int j = 0; j < D; ++j) {
        const float c = bf2f(cT[j * C + i]);
        const float sj = KEY ? s_s[j] : 1.0f;
#pragma unroll
        for (int tt = 0; tt < TB; ++tt) {
          float dl = __fsub_rn(ks[tt * D + j], c);
          if (KEY) acc[tt] = __fmaf_rn(sj, __fmul_rn(dl, dl), acc[tt]);
          else acc[tt] = __fmaf_rn(dl, dl, acc[tt]);
        }
      }
#pragma unroll
      for (int tt = 0; tt < TB; ++tt) Ds[tt * C + i] = acc[tt];
    }
    __syncthreads();
    // ---- phase 2: shortlist, one warp per token
    const int Mc = KEY ? A.M : 1;
    for (int tt = warp; tt < TB; tt += NW) {
      if (tb0 + tt >= A.n) continue;
      float lastD = 0.0f;
      int lastI = -1;
      for (int m = 0; m < Mc; ++m) {
        float bd = 0.0f;
        int bi = -1;
        for (int i = lane; i < C; i += 32) {
          float v = Ds[tt * C + i];
          bool after = (lastI < 0) || lex_less(lastD, lastI, v, i);
          if (after && (bi < 0 || lex_less(v, i, bd, bi))) { bd = v; bi = i; }
        }
        for (int o = 16; o >= 1; o >>= 1) {
          float od = __shfl_xor_sync(0xffffffffu, bd, o);
          int oi = __shfl_xor_sync(0xffffffffu, bi, o);
          if (oi >= 0 && (bi < 0 || lex_less(od, oi, bd, bi))) { bd = od; bi = oi; }
        }
        lastD = bd;
        lastI = bi;
        if (lane == 0) cand[tt * kMaxM + m] = bi;
      }
    }
    __syncwarp();
    // ---- phase 3: QSAC score, INT2 codes, PSAC coefficients
    for (int tt = warp; tt < TB; tt += NW) {
      const int64_t t = tb0 + tt;
      if (t >= A.n) continue;
      float kv[CPL];
#pragma unroll
      for (int u = 0; u < CPL; ++u) kv[u] = ks[tt * D + lane * CPL + u];
      int a = cand[tt * kMaxM + 0];
      if (KEY && Mc > 1) {
        float best = 0.0f;
        int bm = -1;
        for (int m = 0; m < Mc; ++m) {
          const int i = cand[tt * kMaxM + m];
          const uint16_t* crow = cent + (size_t)i * D + lane * CPL;
          float lo, hi;
#pragma unroll
          for (int u = 0; u < CPL; ++u) {
            float rho = __fsub_rn(kv[u], bf2f(crow[u]));
            lo = (u == 0) ? rho : fminf(lo, rho);
            hi = (u == 0) ? rho : fmaxf(hi, rho);
          }
          for (int o = 1; o < lpg; o <<= 1) {
            lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
            hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
          }
          float score = 0.0f;
          if (A.qfull) {
            score = full_score<D>(A, h, lane, kv, crow, lo, hi, es + warp * D);
          } else {
            const float R = __fsub_rn(hi, lo);
            for (int g = 0; g < ng; ++g) {
              float Rg = __shfl_sync(0xffffffffu, R, g * lpg);
              score = __fmaf_rn(w_s[g], __fmul_rn(Rg, Rg), score);
            }
          }
          if (bm < 0 || score < best) { best = score; bm = m; }
        }
        a = cand[tt * kMaxM + bm];
      }
      // encode the winner
      const uint16_t* crow = cent + (size_t)a * D + lane * CPL;
      float cv[CPL], rho[CPL];
      float lo, hi;
#pragma unroll
      for (int u = 0; u < CPL; ++u) {
        cv[u] = bf2f(crow[u]);
        rho[u] = __fsub_rn(kv[u], cv[u]);
        lo = (u == 0) ? rho[u] : fminf(lo, rho[u]);
        hi = (u == 0) ? rho[u] : fmaxf(hi, rho[u]);
      }
      for (int o = 1; o < lpg; o <<= 1) {
        lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
        hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
      }
      uint16_t mnh, sch;
      float mn, sc;
      int2_params(lo, hi, mnh, sch, mn, sc);
      uint32_t bits = 0;
      int code[CPL];
#pragma unroll
      for (int u = 0; u < CPL; ++u) {
        code[u] = int2_code(rho[u], mn, sc);
        bits |= (uint32_t)code[u] << (2 * ((lane * CPL + u) % 4));
      }
      const size_t slot = (size_t)h * A.tcap + (size_t)(A.t0 + t);
      if (CPL == 4) {
        A.codes[slot * (D / 4) + lane] = (uint8_t)bits;
      } else {  // two lanes share a byte
        bits |= __shfl_xor_sync(0xffffffffu, bits, 1);
        if ((lane & 1) == 0) A.codes[slot * (D / 4) + lane / 2] = (uint8_t)bits;
      }
      if ((lane % lpg) == 0) {
        const int g = lane / lpg;
        ((uint32_t*)A.params)[slot * ng + g] = (uint32_t)mnh | ((uint32_t)sch << 16);
      }
      if (lane == 0) {
        if (A.idx_bytes == 1) ((uint8_t*)A.idx)[slot] = (uint8_t)a;
        else ((uint16_t*)A.idx)[slot] = (uint16_t)a;
        if (KEY && h == 0) {
          A.tokver[A.t0 + t] = (uint16_t)A.version;
          A.centver[A.t0 + t] = (uint16_t)A.cver;
        }
      }
      if (KEY) {
        float* ew = es + warp * D;
#pragma unroll
        for (int u = 0; u < CPL; ++u) {
          float deq = __fmaf_rn((float)code[u], sc, mn);
          float khat = __fadd_rn(cv[u], deq);
          ew[lane * CPL + u] = __fsub_rn(kv[u], khat);
        }
        __syncwarp();
        float cq = 0.0f;
        if (lane < r) {
          for (int j = 0; j < D; ++j) cq = __fmaf_rn(U_s[j * r + lane], ew[j], cq);
        }
        float amax = fabsf(cq);
        for (int o = 16; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        const uint16_t csh = f2h_ru(__fdiv_rn(amax, 127.0f));
        const float cs = h2f(csh);
        if (lane < r) {
          int q8 = 0;
          if (cs != 0.0f) {
            q8 = __float2int_rn(__fdiv_rn(cq, cs));
            q8 = max(-127, min(127, q8));
          }
          A.coef[slot * r + lane] = (int8_t)q8;
        }
        if (lane == 0) A.cscale[slot] = csh;
        __syncwarp();
      }
    }
  }
}

template <int D, bool KEY>
cudaError_t run(const AppendArgs& a, cudaStream_t s) {
  size_t smem = (size_t)D * a.C * 2 + (size_t)TB * D * 4 + (size_t)TB * a.C * 4 + D * 4 + 8 * 4 +
                (size_t)D * kMaxR * 4 + (size_t)NW * D * 4 + TB * kMaxM * 4;
  cudaError_t e = cudaFuncSetAttribute(append_kernel<D, KEY>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int64_t nblk = (a.n + TB - 1) / TB;
  int bph = (int)(nblk < 1 ? 1 : nblk);
  int cap = (4 * 148 + a.H - 1) / a.H;
  if (bph > cap) bph = cap;
  append_kernel<D, KEY><<<dim3(bph, a.H), NT, smem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_append_simt(const Dims& Dm, const CacheView& v, const uint16_t* K,
                               const uint16_t* V, int64_t n, int64_t t0, int version,
                               int cent_version, cudaStream_t s);

cudaError_t launch_append(const Dims& Dm, const CacheView& v, const uint16_t* K, const uint16_t* V,
                          int64_t n, int64_t t0, int version, int cent_version, cudaStream_t s) {
  if (append_tc_supported(Dm))
    return launch_append_tc(Dm, v, K, V, n, t0, version, cent_version, s);
  return launch_append_simt(Dm, v, K, V, n, t0, version, cent_version, s);
}

cudaError_t launch_append_simt(const Dims& Dm, const CacheView& v, const uint16_t* K,
                               const uint16_t* V, int64_t n, int64_t t0, int version,
                               int cent_version, cudaStream_t s) {
  const size_t coff = (size_t)cent_version * cent_slot_elems(Dm);
  AppendArgs a{};
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
  // keys
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
  a.eigvec = v.eigvec;
  a.qfull = Dm.qsac_full;
  cudaError_t e = (Dm.d == 128) ? run<128, true>(a, s) : run<64, true>(a, s);
  if (e != cudaSuccess) return e;
  // values
  a.X = V;
  a.cent = v.cent_v + coff;
  a.codes = v.v_codes;
  a.params = v.v_params;
  a.idx = v.v_idx;
  a.coef = nullptr;
  a.cscale = nullptr;
  return (Dm.d == 128) ? run<128, false>(a, s) : run<64, false>(a, s);
}

}  // namespace qwm
