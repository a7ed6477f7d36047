// stats.cu -- historical Query statistics and the PSAC basis.
//
// QuantWM reads two statistics of the queries generated so far (evolve.pub
// review, Summary and Strengths, Eq. 7: the expected squared logit
// perturbation of a Key error e is e^T M e with M = E[q q^T]):
//   - QSAC uses the diagonal s_j = M_jj,
//   - PSAC uses U = the top-r eigenvectors of M (the principal Query
//     directions; the pages use r = 8, Fig. 4 / Table 9).
//
// stats_accumulate: QSTATS[h] += sum_t q_t q_t^T.  Products of bf16 values are
// exact in fp32; each 64-token chunk is summed in fp32 (tokens in order) and
// added to the fp64 running sum, so the result does not depend on scheduling.
//
// refresh: s_j = M_jj / n, w_g = sum_{j in g} s_j (fp32 fold over the group),
// U = top-r eigenvectors of A = M / n by block subspace iteration (see
// refresh_kernel), warm-started from the previous refresh since the statistics
// move little between frames.  Each U column is signed so that its
// largest-magnitude entry (lowest index on ties) is positive.
#include "common.cuh"

namespace qwm {
namespace {

constexpr int kTile = 32;
constexpr int kChunk = 64;

// grid (d/32, d/32, H), block 256: each thread owns a 2x2 block of the 32x32
// output tile.
__global__ void __launch_bounds__(256) stats_acc(const uint16_t* __restrict__ Q, int64_t n, int H,
                                                 int d, double* __restrict__ M) {
  __shared__ float qi[kChunk][kTile + 1];
  __shared__ float qj[kChunk][kTile + 1];
  const int h = blockIdx.z;
  const int i0 = blockIdx.y * kTile, j0 = blockIdx.x * kTile;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  double tot[2][2] = {{0, 0}, {0, 0}};
  for (int64_t b = 0; b < n; b += kChunk) {
    __syncthreads();
    for (int e = threadIdx.x; e < kChunk * kTile; e += 256) {
      int tt = e / kTile, c = e % kTile;
      int64_t t = b + tt;
      bool ok = t < n;
      const uint16_t* row = Q + ((size_t)t * H + h) * d;
      qi[tt][c] = ok ? bf2f(row[i0 + c]) : 0.0f;
      qj[tt][c] = ok ? bf2f(row[j0 + c]) : 0.0f;
    }
    __syncthreads();
    float acc[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
    for (int tt = 0; tt < kChunk; ++tt) {
      float a0 = qi[tt][ty * 2], a1 = qi[tt][ty * 2 + 1];
      float b0 = qj[tt][tx * 2], b1 = qj[tt][tx * 2 + 1];
      acc[0][0] = __fmaf_rn(a0, b0, acc[0][0]);
      acc[0][1] = __fmaf_rn(a0, b1, acc[0][1]);
      acc[1][0] = __fmaf_rn(a1, b0, acc[1][0]);
      acc[1][1] = __fmaf_rn(a1, b1, acc[1][1]);
    }
    for (int u = 0; u < 2; ++u)
      for (int v = 0; v < 2; ++v) tot[u][v] += (double)acc[u][v];
  }
  for (int u = 0; u < 2; ++u)
    for (int v = 0; v < 2; ++v) {
      size_t o = ((size_t)h * d + i0 + ty * 2 + u) * d + j0 + tx * 2 + v;
      M[o] += tot[u][v];
    }
}

// Block subspace ("orthogonal") iteration for the top eigenvectors of the
// symmetric positive semi-definite A = M / n, fp64, one CTA per head.  The
// block X (d x p, p = 16 for r <= 8, else 32) starts from the previous
// refresh's Ritz vectors (warm) or from the columns of A with the largest
// diagonal (cold).  Each step orthonormalizes X by Cholesky-QR (twice) and
// multiplies by A; it stops when the trace of Q^T A Q changes by less than
// 1e-14 relative (or after a cap).  A final Rayleigh-Ritz step diagonalizes
// H = Q^T A Q (p x p) by one-sided Jacobi; the Ritz vectors Q W, sorted by
// descending Ritz value, give U (first r columns) and the next warm start.
struct RefreshSmem {
  double* A;   // [d][d+1] row-major, padded
  double* X;   // [p][d+1] column-major (column k at X + k*(d+1))
  double* Y;   // [p][d+1]
  double* G;   // [p][p]  Gram / projected matrix (column-major for Jacobi)
  double* L;   // [p][p]  Cholesky factor
  double* th;  // [p]     Ritz values
  int* ord;    // [p]
  double* red; // [32]    block reduction scratch
};

// Y = A X  (each warp takes columns, lanes take rows)
__device__ void gemm_AX(const RefreshSmem& S, const double* X, double* Y, int d, int p) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x / 32, nw = blockDim.x / 32;
  for (int k = warp; k < p; k += nw) {
    const double* xk = X + k * (d + 1);
    for (int i = lane; i < d; i += 32) {
      const double* ai = S.A + i * (d + 1);
      double acc = 0.0;
      for (int j = 0; j < d; ++j) acc = fma(ai[j], xk[j], acc);
      Y[k * (d + 1) + i] = acc;
    }
  }
  __syncthreads();
}

// G = X^T Y (p x p); one warp per entry, lanes split the rows.
__device__ void gram(const double* X, const double* Y, double* G, int d, int p) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x / 32, nw = blockDim.x / 32;
  for (int e = warp; e < p * p; e += nw) {
    const int a = e / p, b = e % p;
    const double* xa = X + a * (d + 1);
    const double* yb = Y + b * (d + 1);
    double acc = 0.0;
    for (int i = lane; i < d; i += 32) acc = fma(xa[i], yb[i], acc);
    for (int o = 16; o >= 1; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) G[b * p + a] = acc;  // column-major
  }
  __syncthreads();
}

// One Cholesky-QR pass: X <- X R^-1 with R^T R = X^T X (R = L^T).  One warp
// factors the p x p Gram matrix and inverts L; then every thread applies
// L^-1 to rows of X.  Columns whose pivot vanishes (dependent columns) become
// zero.
__device__ void cholqr(const RefreshSmem& S, double* X, int d, int p) {
  gram(X, X, S.G, d, p);
  if (threadIdx.x < 32) {
    const int i = threadIdx.x;  // row owned by this lane
    double tr = 0.0;
    for (int k = 0; k < p; ++k) tr += S.G[k * p + k];
    for (int k = 0; k < p; ++k) {
      const double piv = S.G[k * p + k];
      const bool ok = piv > 1e-26 * tr && piv > 0.0;
      const double dkk = ok ? sqrt(piv) : 0.0;
      if (i >= k && i < p) S.L[k * p + i] = ok ? (i == k ? dkk : S.G[k * p + i] / dkk) : 0.0;
      __syncwarp();
      if (i > k && i < p) {
        const double lik = S.L[k * p + i];
        for (int j = k + 1; j <= i; ++j) S.G[j * p + i] -= lik * S.L[k * p + j];
      }
      __syncwarp();
    }
    // Linv (lower triangular) into G: lane c computes column c by forward
    // substitution down the column, using only L and its own earlier entries
    __syncwarp();
    if (i < p) {
      const int c = i;
      for (int r2 = 0; r2 < c; ++r2) S.G[c * p + r2] = 0.0;
      for (int r2 = c; r2 < p; ++r2) {
        double v = (r2 == c) ? 1.0 : 0.0;
        for (int m = c; m < r2; ++m) v -= S.L[m * p + r2] * S.G[c * p + m];
        const double l = S.L[r2 * p + r2];
        S.G[c * p + r2] = (l != 0.0) ? v / l : 0.0;
      }
    }
  }
  __syncthreads();
  // Q = X R^-1 = X Linv^T: Q[:, k] = sum_{m <= k} X[:, m] Linv[k][m]
  double* Y = S.Y;
  for (int e = threadIdx.x; e < p * d; e += blockDim.x) {
    const int k = e / d, i = e % d;
    double acc = 0.0;
    for (int m = 0; m <= k; ++m) acc = fma(X[m * (d + 1) + i], S.G[m * p + k], acc);
    Y[k * (d + 1) + i] = acc;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < p * d; e += blockDim.x) {
    const int k = e / d, i = e % d;
    X[k * (d + 1) + i] = Y[k * (d + 1) + i];
  }
  __syncthreads();
}

// One-sided Jacobi on the p x p column-major matrix G (positive semi-definite):
// rotate column pairs until orthogonal; 8 threads per pair.  Also applies the
// rotations to W (p x p, column-major, starts as the identity).
__device__ void small_jacobi(double* G, double* W, int p, double* red) {
  const int tid = threadIdx.x;
  const int grp = tid / 8, sub = tid % 8;
  const int npairs = p / 2;
  for (int e = tid; e < p * p; e += blockDim.x) W[e] = ((e / p) == (e % p)) ? 1.0 : 0.0;
  __syncthreads();
  for (int sweep = 0; sweep < 30; ++sweep) {
    float worst = 0.0f;
    for (int rnd = 0; rnd < p - 1; ++rnd) {
      if (grp < npairs) {
        const int a = (grp == 0) ? 0 : 1 + (grp - 1 + rnd) % (p - 1);
        const int bb = 1 + (p - 1 - grp - 1 + rnd) % (p - 1);
        const int pp = min(a, bb), qq = max(a, bb);
        double* gp = G + pp * p;
        double* gq = G + qq * p;
        double al = 0.0, be = 0.0, ga = 0.0;
        for (int i = sub; i < p; i += 8) {
          al += gp[i] * gp[i];
          be += gq[i] * gq[i];
          ga += gp[i] * gq[i];
        }
        for (int o = 4; o >= 1; o >>= 1) {
          al += __shfl_xor_sync(0xffffffffu, al, o);
          be += __shfl_xor_sync(0xffffffffu, be, o);
          ga += __shfl_xor_sync(0xffffffffu, ga, o);
        }
        const double nrm = sqrt(al * be);
        if (ga != 0.0 && fabs(ga) > 1e-15 * nrm) {
          worst = fmaxf(worst, (float)(fabs(ga) / nrm));
          const double zeta = (be - al) / (2.0 * ga);
          const double t = (zeta >= 0.0 ? 1.0 : -1.0) / (fabs(zeta) + sqrt(1.0 + zeta * zeta));
          const double c = 1.0 / sqrt(1.0 + t * t), s = c * t;
          double* wp = W + pp * p;
          double* wq = W + qq * p;
          for (int i = sub; i < p; i += 8) {
            const double u = gp[i], v = gq[i];
            gp[i] = c * u - s * v;
            gq[i] = s * u + c * v;
            const double wu = wp[i], wv = wq[i];
            wp[i] = c * wu - s * wv;
            wq[i] = s * wu + c * wv;
          }
        }
      }
      __syncthreads();
    }
    for (int o = 16; o >= 1; o >>= 1) worst = fmaxf(worst, __shfl_xor_sync(0xffffffffu, worst, o));
    __syncthreads();
    if ((tid & 31) == 0) red[tid / 32] = worst;
    __syncthreads();
    float m = 0.0f;
    for (int w = 0; w < (int)(blockDim.x / 32); ++w) m = fmaxf(m, (float)red[w]);
    __syncthreads();
    if (m <= 1e-13f) break;
  }
}

// One CTA per head, 512 threads.
__global__ void __launch_bounds__(512) refresh_kernel(const double* __restrict__ Mall, int64_t n,
                                                      int d, int G, int r, int p,
                                                      float* __restrict__ sens,
                                                      float* __restrict__ wgroup,
                                                      float* __restrict__ basis_slot,
                                                      double* __restrict__ eigvec,
                                                      double* __restrict__ flags) {
  extern __shared__ double sm[];
  const int h = blockIdx.x;
  const int tid = threadIdx.x, nt = blockDim.x;
  float* s_out = sens + (size_t)h * d;
  float* w_out = wgroup + (size_t)h * (d / G);
  float* U = basis_slot + (size_t)h * d * (r > 0 ? r : 1);
  if (n <= 0) {
    for (int j = tid; j < d; j += nt) s_out[j] = 1.0f;
    for (int e = tid; e < d * r; e += nt) U[e] = 0.0f;
    __syncthreads();
    if (tid < d / G) {
      float acc = 0.0f;
      for (int j = tid * G; j < (tid + 1) * G; ++j) acc = __fadd_rn(acc, s_out[j]);
      w_out[tid] = acc;
    }
    return;
  }
  RefreshSmem S;
  S.A = sm;
  S.X = S.A + d * (d + 1);
  S.Y = S.X + p * (d + 1);
  S.G = S.Y + p * (d + 1);
  S.L = S.G + p * p;
  S.th = S.L + p * p;
  S.red = S.th + p;
  S.ord = reinterpret_cast<int*>(S.red + 32);
  const double* M = Mall + (size_t)h * d * d;
  const double inv = 1.0 / (double)n;
  for (int e = tid; e < d * d; e += nt) S.A[(e / d) * (d + 1) + (e % d)] = M[e] * inv;
  for (int j = tid; j < d; j += nt) s_out[j] = __double2float_rn(M[(size_t)j * d + j] / (double)n);
  __syncthreads();
  if (tid < d / G) {
    float acc = 0.0f;
    for (int j = tid * G; j < (tid + 1) * G; ++j) acc = __fadd_rn(acc, s_out[j]);
    w_out[tid] = acc;
  }
  // ---- starting block
  const double* Vprev = eigvec + (size_t)h * d * d;
  const bool warm = flags[h] != 0.0;
  if (warm) {
    for (int e = tid; e < p * d; e += nt) S.X[(e / d) * (d + 1) + (e % d)] = Vprev[e];
  } else {
    // columns of A with the p largest diagonal entries (ties: lower index)
    if (tid < d) {
      const double v = S.A[tid * (d + 1) + tid];
      int rank = 0;
      for (int j = 0; j < d; ++j) {
        const double u = S.A[j * (d + 1) + j];
        rank += (u > v) || (u == v && j < tid);
      }
      if (rank < p) S.ord[rank] = tid;
    }
    __syncthreads();
    for (int e = tid; e < p * d; e += nt) {
      const int k = e / d, i = e % d;
      S.X[k * (d + 1) + i] = S.A[i * (d + 1) + S.ord[k]];
    }
  }
  __syncthreads();
  // ---- orthogonal iteration: a fixed number of steps (the top-r subspace
  // converges at rate lambda_{p+1}/lambda_r per step; the trailing part of the
  // block may be nearly degenerate, so the block as a whole is not a stopping
  // test).  Warm starts track a basis that moves little between refreshes.
  const int iters = warm ? 3 : 30;
  for (int it = 0; it < iters; ++it) {
    cholqr(S, S.X, d, p);
    gemm_AX(S, S.X, S.Y, d, p);
    for (int e = tid; e < p * d; e += nt) {
      const int k = e / d, i = e % d;
      S.X[k * (d + 1) + i] = S.Y[k * (d + 1) + i];
    }
    __syncthreads();
  }
  // ---- Rayleigh-Ritz on the final block
  cholqr(S, S.X, d, p);
  cholqr(S, S.X, d, p);
  gemm_AX(S, S.X, S.Y, d, p);
  gram(S.X, S.Y, S.G, d, p);              // H = Q^T A Q (column-major, symmetric)
  double* W = S.Y;                         // Y is free again: W [p][p] in its space
  double* Hc = S.Y + p * p;                // copy of H to rotate
  for (int e = tid; e < p * p; e += nt) Hc[e] = S.G[e];
  __syncthreads();
  small_jacobi(Hc, W, p, S.red);
  __syncthreads();
  if (tid < p) {
    double acc = 0.0;
    for (int i = 0; i < p; ++i) acc += Hc[tid * p + i] * Hc[tid * p + i];
    S.th[tid] = sqrt(acc);
  }
  __syncthreads();
  if (tid < p) {
    const double v = S.th[tid];
    int rank = 0;
    for (int j = 0; j < p; ++j) rank += (S.th[j] > v) || (S.th[j] == v && j < tid);
    S.ord[rank] = tid;
  }
  __syncthreads();
  // Ritz vectors V = Q W (sorted), written to eigvec (column-major) for the
  // next warm start; the first r columns, sign-normalized, are U.
  double* Vout = eigvec + (size_t)h * d * d;
  for (int e = tid; e < p * d; e += nt) {
    const int c = e / d, i = e % d;
    const int k = S.ord[c];
    double acc = 0.0;
    for (int m = 0; m < p; ++m) acc = fma(S.X[m * (d + 1) + i], W[k * p + m], acc);
    Vout[(size_t)c * d + i] = acc;
  }
  __syncthreads();
  const int lane = tid & 31, warp = tid / 32;
  for (int c = warp; c < r; c += nt / 32) {
    const double* v = Vout + (size_t)c * d;
    double big = -1.0;
    int arg = 0;
    for (int i = lane; i < d; i += 32) {
      const double m = fabs(v[i]);
      if (m > big) { big = m; arg = i; }
    }
    for (int o = 16; o >= 1; o >>= 1) {
      const double ob = __shfl_xor_sync(0xffffffffu, big, o);
      const int oa = __shfl_xor_sync(0xffffffffu, arg, o);
      if (ob > big || (ob == big && oa < arg)) { big = ob; arg = oa; }
    }
    const double sg = (v[arg] < 0.0) ? -1.0 : 1.0;
    for (int i = lane; i < d; i += 32) U[(size_t)i * r + c] = __double2float_rn(sg * v[i]);
  }
  if (tid == 0) {
    const double t0 = S.th[S.ord[0]], tl = S.th[S.ord[p - 1]];
    flags[h] = (t0 > 0.0 && tl > 1e-10 * t0) ? 1.0 : 0.0;
  }
}

__global__ void init_state(int H, int d, int G, int r, float* sens, float* wgroup, float* basis0,
                           double* qstats, double* eig_flags) {
  size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x;
  size_t stride = (size_t)gridDim.x * blockDim.x;
  for (size_t e = i; e < (size_t)H * d * d; e += stride) qstats[e] = 0.0;
  for (size_t e = i; e < (size_t)H * d; e += stride) sens[e] = 1.0f;
  for (size_t e = i; e < (size_t)H * (d / G); e += stride) {
    float acc = 0.0f;
    for (int j = 0; j < G; ++j) acc = __fadd_rn(acc, 1.0f);
    wgroup[e] = acc;
  }
  for (size_t e = i; e < (size_t)H * d * (r > 0 ? r : 1); e += stride) basis0[e] = 0.0f;
  for (size_t e = i; e < (size_t)H; e += stride) eig_flags[e] = 0.0;
}

}  // namespace

cudaError_t launch_init_state(const Dims& D, const CacheView& v, cudaStream_t s) {
  double* flags = v.eigvec + (size_t)D.H * D.d * D.d;
  init_state<<<256, 256, 0, s>>>(D.H, D.d, D.G, D.r, v.sens, v.wgroup, v.basis, v.qstats, flags);
  return cudaGetLastError();
}

cudaError_t launch_stats_accumulate(const Dims& D, const uint16_t* Q, int64_t n, double* qstats,
                                    cudaStream_t s) {
  dim3 grid(D.d / kTile, D.d / kTile, D.H);
  stats_acc<<<grid, 256, 0, s>>>(Q, n, D.H, D.d, qstats);
  return cudaGetLastError();
}

int refresh_block(int d, int r) { return (r <= 8 ? 16 : 32) < d ? (r <= 8 ? 16 : 32) : d; }

cudaError_t launch_refresh(const Dims& D, const CacheView& v, int64_t n_total, int version,
                           int /*warm_hint*/, cudaStream_t s) {
  double* flags = v.eigvec + (size_t)D.H * D.d * D.d;
  float* slot = v.basis + (size_t)version * D.H * D.d * (D.r > 0 ? D.r : 1);
  const int p = refresh_block(D.d, D.r);
  size_t smem = ((size_t)D.d * (D.d + 1) + 2 * (size_t)p * (D.d + 1) + 2 * p * p + p + 32) * 8 +
                (size_t)p * 4 + 64;
  cudaError_t e =
      cudaFuncSetAttribute(refresh_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  refresh_kernel<<<D.H, 512, smem, s>>>(v.qstats, n_total, D.d, D.G, D.r, p, v.sens, v.wgroup,
                                        slot, v.eigvec, flags);
  return cudaGetLastError();
}

}  // namespace qwm
