// attention_simt.cu -- CUDA-core kernels over the packed cache: reconstruction
// for inspection, the top-1 key-selection measurement, and a plain attention
// kernel (64 query rows per CTA, 64-key tiles dequantized into shared memory,
// online softmax) that serves configurations the tensor-core kernel does not.
#include <math.h>

#include "dequant.cuh"

namespace qwm {
namespace {

constexpr int QT = 64;   // query rows per CTA
constexpr int KT = 64;   // keys per tile

__device__ __forceinline__ float round_bf16(float x) { return bf2f(f2bf(x)); }

// Keys 0 .. T-1 come from the packed cache, keys T .. T+sg.n-1 from the bf16
// segment.
template <int D>
__global__ void __launch_bounds__(256) attn_simt(const Dims Dm, const CacheView v, int64_t T,
                                                 const uint16_t* __restrict__ Q, int64_t nq,
                                                 float scale_log2, uint16_t* __restrict__ O,
                                                 const Segment sg) {
  extern __shared__ float sm[];
  float* Qs = sm;                   // [QT][D+1]
  float* Ks = Qs + QT * (D + 1);    // [KT][D+1]
  float* Vs = Ks + KT * (D + 1);    // [KT][D]
  float* Ps = Vs + KT * D;          // [QT][KT+1]
  const int h = blockIdx.y;
  const int64_t q0 = (int64_t)blockIdx.x * QT;
  const int tid = threadIdx.x, row = tid / 4, sub = tid % 4;
  const int H = Dm.H;
  for (int e = tid; e < QT * D; e += 256) {
    int rr = e / D, j = e % D;
    int64_t q = q0 + rr;
    Qs[rr * (D + 1) + j] = (q < nq) ? bf2f(Q[((size_t)q * H + h) * D + j]) : 0.0f;
  }
  float m = -INFINITY, l = 0.0f;
  float o[D / 4];
#pragma unroll
  for (int u = 0; u < D / 4; ++u) o[u] = 0.0f;
  const PackedHead p = packed_head(v, Dm, h);
  const int64_t Ttot = T + sg.n;
  for (int64_t k0 = 0; k0 < Ttot; k0 += KT) {
    __syncthreads();
    for (int e = tid; e < KT * D; e += 256) {
      int kk = e / D, j = e % D;
      int64_t t = k0 + kk;
      float kv = 0.0f, vv = 0.0f;
      if (t < T) {
        const float* U_h = basis_of(v, Dm, v.tokver[t], h);
        kv = round_bf16(key_elem(p, Dm, U_h, t, j));
        vv = round_bf16(value_elem(p, Dm, t, j));
      } else if (t < Ttot) {
        const size_t o = ((size_t)(t - T) * H + h) * D + j;
        kv = bf2f(sg.K[o]);
        vv = bf2f(sg.V[o]);
      }
      Ks[kk * (D + 1) + j] = kv;
      Vs[kk * D + j] = vv;
    }
    __syncthreads();
    float s[KT / 4];
#pragma unroll
    for (int u = 0; u < KT / 4; ++u) s[u] = 0.0f;
    for (int j = 0; j < D; ++j) {
      float qv = Qs[row * (D + 1) + j];
#pragma unroll
      for (int u = 0; u < KT / 4; ++u) s[u] = fmaf(qv, Ks[(u * 4 + sub) * (D + 1) + j], s[u]);
    }
    float mx = -INFINITY;
#pragma unroll
    for (int u = 0; u < KT / 4; ++u) {
      int64_t t = k0 + u * 4 + sub;
      s[u] = (t < Ttot) ? s[u] * scale_log2 : -INFINITY;
      mx = fmaxf(mx, s[u]);
    }
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    const float mnew = fmaxf(m, mx);
    const float alpha = exp2f(m - mnew);
    float ls = 0.0f;
#pragma unroll
    for (int u = 0; u < KT / 4; ++u) {
      float pv = exp2f(s[u] - mnew);
      Ps[row * (KT + 1) + u * 4 + sub] = pv;
      ls += pv;
    }
    ls += __shfl_xor_sync(0xffffffffu, ls, 1);
    ls += __shfl_xor_sync(0xffffffffu, ls, 2);
    l = l * alpha + ls;
    m = mnew;
#pragma unroll
    for (int u = 0; u < D / 4; ++u) o[u] *= alpha;
    __syncwarp();
    for (int kk = 0; kk < KT; ++kk) {
      float pv = Ps[row * (KT + 1) + kk];
#pragma unroll
      for (int u = 0; u < D / 4; ++u) o[u] = fmaf(pv, Vs[kk * D + u * 4 + sub], o[u]);
    }
  }
  const int64_t q = q0 + row;
  if (q < nq) {
    const float inv = 1.0f / l;
#pragma unroll
    for (int u = 0; u < D / 4; ++u) O[((size_t)q * H + h) * D + u * 4 + sub] = f2bf(o[u] * inv);
    if (sg.lse && sub == 0) sg.lse[(size_t)q * H + h] = (m + log2f(l)) * 0.6931471805599453f;
  }
}

__global__ void reconstruct_kernel(const Dims Dm, const CacheView v, int64_t t0, int64_t n,
                                   uint16_t* __restrict__ Kp, uint16_t* __restrict__ Vp) {
  const int h = blockIdx.y;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t i = (int64_t)blockIdx.x * (blockDim.x / 32) + warp;
  if (i >= n) return;
  const int64_t t = t0 + i;
  const PackedHead p = packed_head(v, Dm, h);
  const float* U_h = basis_of(v, Dm, v.tokver[t], h);
  for (int j = lane; j < Dm.d; j += 32) {
    Kp[((size_t)h * n + i) * Dm.d + j] = f2bf(key_elem(p, Dm, U_h, t, j));
    Vp[((size_t)h * n + i) * Dm.d + j] = f2bf(value_elem(p, Dm, t, j));
  }
}

template <int D>
__global__ void __launch_bounds__(256) top1_kernel(const Dims Dm, const CacheView v, int64_t T,
                                                   const uint16_t* __restrict__ Q, int64_t nq,
                                                   const uint16_t* __restrict__ Kx,
                                                   int32_t* __restrict__ idx_exact,
                                                   int32_t* __restrict__ idx_quant) {
  extern __shared__ float sm[];
  float* Qs = sm;                   // [QT][D+1]
  float* Ks = Qs + QT * (D + 1);    // [KT][D+1] reconstructed
  float* Xs = Ks + KT * (D + 1);    // [KT][D+1] exact
  const int h = blockIdx.y;
  const int64_t q0 = (int64_t)blockIdx.x * QT;
  const int tid = threadIdx.x, row = tid / 4, sub = tid % 4;
  const int H = Dm.H;
  for (int e = tid; e < QT * D; e += 256) {
    int rr = e / D, j = e % D;
    int64_t q = q0 + rr;
    Qs[rr * (D + 1) + j] = (q < nq) ? bf2f(Q[((size_t)q * H + h) * D + j]) : 0.0f;
  }
  float bx = -INFINITY, bq = -INFINITY;
  int ix = -1, iq = -1;
  const PackedHead p = packed_head(v, Dm, h);
  for (int64_t k0 = 0; k0 < T; k0 += KT) {
    __syncthreads();
    for (int e = tid; e < KT * D; e += 256) {
      int kk = e / D, j = e % D;
      int64_t t = k0 + kk;
      float kv = 0.0f, xv = 0.0f;
      if (t < T) {
        const float* U_h = basis_of(v, Dm, v.tokver[t], h);
        kv = round_bf16(key_elem(p, Dm, U_h, t, j));
        xv = bf2f(Kx[((size_t)t * H + h) * D + j]);
      }
      Ks[kk * (D + 1) + j] = kv;
      Xs[kk * (D + 1) + j] = xv;
    }
    __syncthreads();
    for (int u = 0; u < KT / 4; ++u) {
      int kk = u * 4 + sub;
      int64_t t = k0 + kk;
      if (t >= T) break;
      float a = 0.0f, b = 0.0f;
      for (int j = 0; j < D; ++j) {
        float qv = Qs[row * (D + 1) + j];
        a = fmaf(qv, Xs[kk * (D + 1) + j], a);
        b = fmaf(qv, Ks[kk * (D + 1) + j], b);
      }
      if (a > bx) { bx = a; ix = (int)t; }
      if (b > bq) { bq = b; iq = (int)t; }
    }
  }
  for (int o = 1; o <= 2; o <<= 1) {
    float obx = __shfl_xor_sync(0xffffffffu, bx, o);
    int oix = __shfl_xor_sync(0xffffffffu, ix, o);
    float obq = __shfl_xor_sync(0xffffffffu, bq, o);
    int oiq = __shfl_xor_sync(0xffffffffu, iq, o);
    if (oix >= 0 && (obx > bx || (obx == bx && oix < ix) || ix < 0)) { bx = obx; ix = oix; }
    if (oiq >= 0 && (obq > bq || (obq == bq && oiq < iq) || iq < 0)) { bq = obq; iq = oiq; }
  }
  const int64_t q = q0 + row;
  if (q < nq && sub == 0) {
    idx_exact[(size_t)q * H + h] = ix;
    idx_quant[(size_t)q * H + h] = iq;
  }
}

}  // namespace

cudaError_t launch_attention_simt(const Dims& D, const CacheView& v, int64_t T, const uint16_t* Q,
                                  int64_t nq, float scale, uint16_t* O, const Segment& sg,
                                  cudaStream_t s) {
  const float scale_log2 = scale * 1.4426950408889634f;
  dim3 grid((unsigned)((nq + QT - 1) / QT), D.H);
  if (D.d == 128) {
    size_t smem = (size_t)(QT * 129 + KT * 129 + KT * 128 + QT * (KT + 1)) * 4;
    cudaError_t e = cudaFuncSetAttribute(attn_simt<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    attn_simt<128><<<grid, 256, smem, s>>>(D, v, T, Q, nq, scale_log2, O, sg);
  } else {
    size_t smem = (size_t)(QT * 65 + KT * 65 + KT * 64 + QT * (KT + 1)) * 4;
    cudaError_t e = cudaFuncSetAttribute(attn_simt<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    attn_simt<64><<<grid, 256, smem, s>>>(D, v, T, Q, nq, scale_log2, O, sg);
  }
  return cudaGetLastError();
}

cudaError_t launch_reconstruct(const Dims& D, const CacheView& v, int64_t t0, int64_t n,
                               uint16_t* Kp, uint16_t* Vp, cudaStream_t s) {
  reconstruct_kernel<<<dim3((unsigned)((n + 7) / 8), D.H), 256, 0, s>>>(D, v, t0, n, Kp, Vp);
  return cudaGetLastError();
}

cudaError_t launch_top1(const Dims& D, const CacheView& v, int64_t T, const uint16_t* Q,
                        int64_t nq, const uint16_t* Kexact, int32_t* idx_exact,
                        int32_t* idx_quant, cudaStream_t s) {
  dim3 grid((unsigned)((nq + QT - 1) / QT), D.H);
  if (D.d == 128) {
    size_t smem = (size_t)(QT * 129 + 2 * KT * 129) * 4;
    cudaError_t e = cudaFuncSetAttribute(top1_kernel<128>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    top1_kernel<128><<<grid, 256, smem, s>>>(D, v, T, Q, nq, Kexact, idx_exact, idx_quant);
  } else {
    size_t smem = (size_t)(QT * 65 + 2 * KT * 65) * 4;
    cudaError_t e = cudaFuncSetAttribute(top1_kernel<64>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    top1_kernel<64><<<grid, 256, smem, s>>>(D, v, T, Q, nq, Kexact, idx_exact, idx_quant);
  }
  return cudaGetLastError();
}

// head_dim 128 runs on the tensor cores; other shapes use the CUDA-core kernel.
cudaError_t launch_attention(const Dims& D, const CacheView& v, int64_t T, const uint16_t* Q,
                             int64_t nq, float scale, uint16_t* O, const Segment& sg,
                             cudaStream_t s) {
  if (attention_tc_supported(D)) return launch_attention_tc(D, v, T, Q, nq, scale, O, sg, s);
  return launch_attention_simt(D, v, T, Q, nq, scale, O, sg, s);
}

}  // namespace qwm
