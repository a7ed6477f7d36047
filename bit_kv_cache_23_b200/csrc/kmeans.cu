// kmeans.cu -- centroid tables for the centroid-residual cache (per head,
// Lloyd iterations on the first cached frame).
//
// The QuantWM pages say only that each Key is assigned to a cluster centre
// that keeps higher precision ("Flickering after quantization?", QSAC
// paragraph).  Reading used here: centroid i starts at token floor(i n / C);
// each round assigns every token to the centroid with the smallest fp32
// squared distance (fold acc = fma(delta, delta, acc) over channels in order,
// ties to the lower index), then moves every non-empty centroid to the fp64
// mean of its tokens, summed in token order and rounded to fp32; the final
// table is rounded to bf16.  Every step is deterministic, so the result is
// bit-identical run to run.
//
// Workspace: cent32 [H][C][d] fp32 followed by assign [H][tcap] int32.
#include "common.cuh"

namespace qwm {

size_t kmeans_workspace_bytes(const Dims& D) {
  size_t km = (size_t)D.H * D.C * D.d * 4 + (size_t)D.H * D.tcap * 4;
  size_t eig = (size_t)D.H * D.d * D.d * 8;  // refresh: A V_prev (fp64)
  km = (km + 255) / 256 * 256;
  return km > eig ? km : eig;
}

namespace {

__global__ void km_init(const uint16_t* __restrict__ X, int64_t n, int H, int C, int d,
                        float* __restrict__ cent) {
  int h = blockIdx.y;
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < C * d; e += gridDim.x * blockDim.x) {
    int i = e / d, j = e % d;
    int64_t t = ((int64_t)i * n) / C;
    cent[((size_t)h * C + i) * d + j] = bf2f(X[((size_t)t * H + h) * d + j]);
  }
}

// One thread per token; the token block's rows sit in shared memory as fp32
// [d][TB] (column per thread, conflict-free), centroids stream through shared
// memory in chunks of CH rows (broadcast reads).
template <int TB, int CH>
__global__ void __launch_bounds__(TB) km_assign(const uint16_t* __restrict__ X, int64_t n, int H,
                                                int C, int d, const float* __restrict__ cent,
                                                int32_t* __restrict__ assign, int64_t tcap) {
  extern __shared__ float sm[];
  float* xs = sm;               // [d][TB]
  float* cs = sm + d * TB;      // [CH][d]
  const int h = blockIdx.y;
  const int64_t t0 = (int64_t)blockIdx.x * TB;
  const int tid = threadIdx.x;
  for (int e = tid; e < TB * d; e += TB) {
    int tt = e / d, j = e % d;
    int64_t t = t0 + tt;
    xs[j * TB + tt] = (t < n) ? bf2f(X[((size_t)t * H + h) * d + j]) : 0.0f;
  }
  float best = 0.0f;
  int bi = -1;
  const float* ch = cent + (size_t)h * C * d;
  for (int c0 = 0; c0 < C; c0 += CH) {
    int cn = min(CH, C - c0);
    __syncthreads();
    for (int e = tid; e < cn * d; e += TB) cs[e] = ch[(size_t)c0 * d + e];
    __syncthreads();
    for (int ci = 0; ci < cn; ++ci) {
      float acc = 0.0f;
      for (int j = 0; j < d; ++j) {
        float dl = __fsub_rn(xs[j * TB + tid], cs[ci * d + j]);
        acc = __fmaf_rn(dl, dl, acc);
      }
      if (bi < 0 || acc < best) {
        best = acc;
        bi = c0 + ci;
      }
    }
  }
  int64_t t = t0 + tid;
  if (t < n) assign[(size_t)h * tcap + t] = bi;
}

// One warp per centroid: walk the tokens in order, 32 at a time; the ballot of
// members is consumed lowest token first, so every fp64 sum is taken in token
// order.  Lane l owns channels l, l+32, ...
__global__ void km_update(const uint16_t* __restrict__ X, int64_t n, int H, int C, int d,
                          const int32_t* __restrict__ assign, int64_t tcap,
                          float* __restrict__ cent) {
  const int h = blockIdx.y;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int i = blockIdx.x * (blockDim.x / 32) + warp;
  if (i >= C) return;
  double acc[4] = {0.0, 0.0, 0.0, 0.0};
  int64_t cnt = 0;
  const int32_t* a = assign + (size_t)h * tcap;
  const int per = d / 32;
  for (int64_t b = 0; b < n; b += 32) {
    int64_t t = b + lane;
    bool mine = (t < n) && (a[t] == i);
    unsigned m = __ballot_sync(0xffffffffu, mine);
    while (m) {
      int k = __ffs(m) - 1;
      m &= m - 1;
      const uint16_t* row = X + ((size_t)(b + k) * H + h) * d;
      for (int u = 0; u < per; ++u) acc[u] += (double)bf2f(row[lane + 32 * u]);
      ++cnt;
    }
  }
  if (cnt > 0) {
    float* c = cent + ((size_t)h * C + i) * d;
    for (int u = 0; u < per; ++u) c[lane + 32 * u] = __double2float_rn(acc[u] / (double)cnt);
  }
}

__global__ void km_finalize(const float* __restrict__ cent, size_t count, uint16_t* __restrict__ out) {
  for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < count;
       e += (size_t)gridDim.x * blockDim.x)
    out[e] = f2bf(cent[e]);
}

}  // namespace

cudaError_t launch_kmeans(const Dims& D, const uint16_t* X, int64_t n, int iters, uint16_t* cent_out,
                          void* workspace, cudaStream_t s) {
  float* cent = (float*)workspace;
  size_t cbytes = ((size_t)D.H * D.C * D.d * 4 + 255) / 256 * 256;
  int32_t* assign = (int32_t*)((char*)workspace + cbytes);
  constexpr int TB = 128, CH = 32;
  size_t smem = (size_t)(D.d * TB + CH * D.d) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(km_assign<TB, CH>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  km_init<<<dim3((D.C * D.d + 255) / 256, D.H), 256, 0, s>>>(X, n, D.H, D.C, D.d, cent);
  const int wpb = 8;
  for (int it = 0; it < iters; ++it) {
    km_assign<TB, CH><<<dim3((unsigned)((n + TB - 1) / TB), D.H), TB, smem, s>>>(
        X, n, D.H, D.C, D.d, cent, assign, D.tcap);
    km_update<<<dim3((D.C + wpb - 1) / wpb, D.H), 32 * wpb, 0, s>>>(X, n, D.H, D.C, D.d, assign,
                                                                     D.tcap, cent);
  }
  size_t count = (size_t)D.H * D.C * D.d;
  km_finalize<<<(unsigned)((count + 255) / 256 < 4096 ? (count + 255) / 256 : 4096), 256, 0, s>>>(
      cent, count, cent_out);
  return cudaGetLastError();
}

}  // namespace qwm
