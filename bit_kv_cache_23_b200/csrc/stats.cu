// stats.cu -- historical Query statistics and the PSAC basis.
//
// QuantWM reads two statistics of the queries generated so far (evolve.pub
// review, Summary and Strengths, Eq. 7: the expected squared logit
// perturbation of a Key error e is e^T M e with M = E[q q^T]):
//   - QSAC uses the diagonal s_j = M_jj,
//   - PSAC uses U = the top-r eigenvectors of M (the principal Query
//     directions; the pages use r = 8, Fig. 4 / Table 9).
//
// stats_accumulate: QSTATS[h] += sum_t q_t q_t^T in fp64, each entry summed
// in token order (M_ij <- M_ij + q_ti q_tj, t = 0, 1, ...).  A product of two
// bf16 values has at most 16 significant bits and is exact in fp64, so the
// fused multiply-add rounds exactly as the plain add does: the matrix is the
// sequential fp64 sum, bit for bit, whatever the launch shape.
//
// refresh: s_j = M_jj / n, w_g = sum_{j in g} s_j (fp32 fold over the group),
// U = top-r eigenvectors of A = M / n by block subspace iteration (see
// refresh_kernel), warm-started from the previous refresh since the statistics
// move little between frames.  Each U column is signed so that its
// largest-magnitude entry (lowest index on ties) is positive.
#include "common.cuh"

namespace qwm {
namespace {

constexpr int kTile = 32;   // output tile side
constexpr int kChunk = 32;  // tokens staged per pass

// grid (nt (nt + 1) / 2, H) with nt = d / 32: one CTA per tile (bi <= bj) of
// the upper block triangle, 64 threads, each owning a 4 x 4 block of the
// 32 x 32 tile.  Both tiles' token columns are staged in shared memory as fp64;
// M is symmetric (q_i q_j = q_j q_i exactly), so an off-diagonal tile is
// written to both (bi, bj) and (bj, bi).
__global__ void __launch_bounds__(64) stats_acc(const uint16_t* __restrict__ Q, int64_t n, int H,
                                                int d, double* __restrict__ M) {
  __shared__ __align__(16) double qi[kChunk][kTile];
  __shared__ __align__(16) double qj[kChunk][kTile];
  const int h = blockIdx.y;
  const int nt = d / kTile;
  int bi = 0, rem = blockIdx.x;
  while (rem >= nt - bi) {
    rem -= nt - bi;
    ++bi;
  }
  const int bj = bi + rem;
  const int i0 = bi * kTile, j0 = bj * kTile;
  const int tid = threadIdx.x, ty = tid / 8, tx = tid % 8;
  double* Mh = M + (size_t)h * d * d;
  double acc[4][4];
#pragma unroll
  for (int u = 0; u < 4; ++u)
#pragma unroll
    for (int v = 0; v < 4; ++v) acc[u][v] = Mh[(size_t)(i0 + ty * 4 + u) * d + j0 + tx * 4 + v];

  // staging: 2 sides x 32 tokens x 4 pieces of 8 channels = 256 pieces, 4 per thread
  uint4 pre[4];
  auto fetch = [&](int64_t b) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int e = tid + 64 * k, side = e >> 7, tt = (e & 127) >> 2, part = e & 3;
      const int64_t t = b + tt;
      const int col = (side ? j0 : i0) + part * 8;
      pre[k] = make_uint4(0, 0, 0, 0);
      if (t < n) pre[k] = __ldg(reinterpret_cast<const uint4*>(Q + ((size_t)t * H + h) * d + col));
    }
  };
  auto stage = [&]() {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int e = tid + 64 * k, side = e >> 7, tt = (e & 127) >> 2, part = e & 3;
      double* dst = (side ? &qj[tt][0] : &qi[tt][0]) + part * 8;
      const uint32_t w[4] = {pre[k].x, pre[k].y, pre[k].z, pre[k].w};
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const double lo = (double)__uint_as_float(w[m] << 16);
        const double hi = (double)__uint_as_float(w[m] & 0xffff0000u);
        *reinterpret_cast<double2*>(dst + 2 * m) = make_double2(lo, hi);
      }
    }
  };
  if (n > 0) fetch(0);
  for (int64_t b = 0; b < n; b += kChunk) {
    __syncthreads();
    stage();
    __syncthreads();
    if (b + kChunk < n) fetch(b + kChunk);
    const int cnt = (n - b < kChunk) ? (int)(n - b) : kChunk;
#pragma unroll 4
    for (int tt = 0; tt < cnt; ++tt) {
      const double2 a01 = *reinterpret_cast<const double2*>(&qi[tt][ty * 4]);
      const double2 a23 = *reinterpret_cast<const double2*>(&qi[tt][ty * 4 + 2]);
      const double2 b01 = *reinterpret_cast<const double2*>(&qj[tt][tx * 4]);
      const double2 b23 = *reinterpret_cast<const double2*>(&qj[tt][tx * 4 + 2]);
      const double a[4] = {a01.x, a01.y, a23.x, a23.y};
      const double bb[4] = {b01.x, b01.y, b23.x, b23.y};
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[u][v] = fma(a[u], bb[v], acc[u][v]);
    }
  }
#pragma unroll
  for (int u = 0; u < 4; ++u)
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const int i = i0 + ty * 4 + u, j = j0 + tx * 4 + v;
      Mh[(size_t)i * d + j] = acc[u][v];
      if (bi != bj) Mh[(size_t)j * d + i] = acc[u][v];
    }
}

// Block subspace ("orthogonal") iteration for the top eigenvectors of the
// symmetric positive semi-definite A = M / n, fp64, one CTA per head.  The
// block X (d x p, p = 16 for r <= 8, else 32) starts from the previous
// refresh's Ritz vectors (warm) or from the columns of A with the largest
// diagonal (cold).  Each step orthonormalizes X by Cholesky-QR and multiplies
// by A, a fixed number of steps (3 warm, 30 cold).  A final Rayleigh-Ritz step
// (Cholesky-QR twice, H = Q^T A Q) diagonalizes the p x p matrix H by one-sided
// Jacobi; the Ritz vectors Q W, sorted by descending Ritz value, give U (first
// r columns) and the next warm start.
struct RefreshSmem {
  double* A;   // [d][d+1] row-major, padded
  double* X;   // [p][d+1] column-major (column k at X + k*(d+1))
  double* Y;   // [p][d+1]
  double* G;   // [p][p]  Gram / projected matrix (column-major for Jacobi)
  double* L;   // [p][p]  Cholesky factor (column-major: L[k*p + i] = L_ik)
  double* th;  // [p]     Ritz values
  int* ord;    // [p]
  double* red; // [32]    block reduction scratch
};

// Y = A X.  32 (P / 4) threads: thread (cg, lane) owns rows lane + 32 m and
// columns 4 cg .. 4 cg + 3 (4 D / 32 independent accumulators); rows of A are
// read without bank conflicts (padded stride), entries of X are broadcast.
template <int D, int P>
__device__ void gemm_AX(const double* A, const double* X, double* Y) {
  constexpr int RM = D / 32;
  const int t = threadIdx.x;
  if (t < 32 * (P / 4)) {
    const int lane = t & 31, cg = t >> 5;
    const double* x0 = X + 4 * cg * (D + 1);
    double acc[RM][4];
#pragma unroll
    for (int m = 0; m < RM; ++m)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[m][c] = 0.0;
#pragma unroll 4
    for (int j = 0; j < D; ++j) {
      double a[RM], x[4];
#pragma unroll
      for (int m = 0; m < RM; ++m) a[m] = A[(lane + 32 * m) * (D + 1) + j];
#pragma unroll
      for (int c = 0; c < 4; ++c) x[c] = x0[c * (D + 1) + j];
#pragma unroll
      for (int m = 0; m < RM; ++m)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[m][c] = fma(a[m], x[c], acc[m][c]);
    }
#pragma unroll
    for (int m = 0; m < RM; ++m)
#pragma unroll
      for (int c = 0; c < 4; ++c) Y[(4 * cg + c) * (D + 1) + lane + 32 * m] = acc[m][c];
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

// One Cholesky-QR pass: X <- X R^-1 with R^T R = X^T X (R = L^T).  Warp 0
// factors the Gram matrix with lane i holding row i in registers (right-looking,
// the multipliers passed by shuffles); then each thread takes one row x of X and
// solves L q = x by forward substitution.  A column whose pivot vanishes
// (dependent columns) becomes zero.
template <int D, int P>
__device__ void cholqr(double* X, double* G, double* L) {
  gram(X, X, G, D, P);
  if (threadIdx.x < 32) {
    const int i = threadIdx.x;
    double g[P];
#pragma unroll
    for (int j = 0; j < P; ++j) g[j] = (i < P) ? G[j * P + i] : 0.0;
    double tr = 0.0;
#pragma unroll
    for (int k = 0; k < P; ++k) tr += G[k * P + k];
#pragma unroll
    for (int k = 0; k < P; ++k) {
      const double piv = __shfl_sync(0xffffffffu, g[k], k);
      const bool ok = piv > 1e-26 * tr && piv > 0.0;
      const double dkk = ok ? sqrt(piv) : 0.0;
      double lik = 0.0;
      if (i == k) lik = dkk;
      else if (i > k && i < P && ok) lik = g[k] / dkk;
      if (i < P) L[k * P + i] = lik;
#pragma unroll
      for (int j = k + 1; j < P; ++j) {
        const double ljk = __shfl_sync(0xffffffffu, lik, j);
        g[j] = g[j] - lik * ljk;  // rows below k; the upper triangle is never read
      }
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < D; i += blockDim.x) {
    double q[P];
#pragma unroll
    for (int k = 0; k < P; ++k) {
      double v = X[k * (D + 1) + i];
#pragma unroll
      for (int m = 0; m < k; ++m) v = v - L[m * P + k] * q[m];
      const double lkk = L[k * P + k];
      q[k] = (lkk != 0.0) ? v / lkk : 0.0;
    }
#pragma unroll
    for (int k = 0; k < P; ++k) X[k * (D + 1) + i] = q[k];
  }
  __syncthreads();
}

// One-sided Jacobi on the p x p column-major matrix G (positive semi-definite),
// in warp 0: rotate column pairs until orthogonal, the p / 2 disjoint pairs of
// a round-robin round at once, 64 / p lanes per pair.  Also applies the
// rotations to W (p x p, column-major, starts as the identity).
template <int P>
__device__ void small_jacobi(double* G, double* W) {
  constexpr int LPP = 64 / P;  // lanes per pair
  for (int e = threadIdx.x; e < P * P; e += blockDim.x) W[e] = ((e / P) == (e % P)) ? 1.0 : 0.0;
  __syncthreads();
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x, grp = lane / LPP, sub = lane % LPP;
    for (int sweep = 0; sweep < 30; ++sweep) {
      float worst = 0.0f;
      for (int rnd = 0; rnd < P - 1; ++rnd) {
        const int a = (grp == 0) ? 0 : 1 + (grp - 1 + rnd) % (P - 1);
        const int bb = 1 + (P - 1 - grp - 1 + rnd) % (P - 1);
        const int pp = min(a, bb), qq = max(a, bb);
        double* gp = G + pp * P;
        double* gq = G + qq * P;
        double al = 0.0, be = 0.0, ga = 0.0;
#pragma unroll
        for (int i = sub; i < P; i += LPP) {
          al += gp[i] * gp[i];
          be += gq[i] * gq[i];
          ga += gp[i] * gq[i];
        }
#pragma unroll
        for (int o = LPP / 2; o >= 1; o >>= 1) {
          al += __shfl_xor_sync(0xffffffffu, al, o);
          be += __shfl_xor_sync(0xffffffffu, be, o);
          ga += __shfl_xor_sync(0xffffffffu, ga, o);
        }
        // rotate unless the pair is orthogonal to 1e-15 (compared squared: no root)
        if (ga != 0.0 && ga * ga > 1e-30 * (al * be)) {
          worst = fmaxf(worst, fabsf((float)ga) * rsqrtf((float)al * (float)be));
          const double zeta = (be - al) / (2.0 * ga);
          const double t = (zeta >= 0.0 ? 1.0 : -1.0) / (fabs(zeta) + sqrt(1.0 + zeta * zeta));
          const double c = rsqrt(1.0 + t * t), s = c * t;
          double* wp = W + pp * P;
          double* wq = W + qq * P;
#pragma unroll
          for (int i = sub; i < P; i += LPP) {
            const double u = gp[i], v = gq[i];
            gp[i] = c * u - s * v;
            gq[i] = s * u + c * v;
            const double wu = wp[i], wv = wq[i];
            wp[i] = c * wu - s * wv;
            wq[i] = s * wu + c * wv;
          }
        }
        __syncwarp();
      }
      for (int o = 16; o >= 1; o >>= 1) worst = fmaxf(worst, __shfl_xor_sync(0xffffffffu, worst, o));
      if (worst <= 1e-13f) break;
    }
  }
  __syncthreads();
}

// One CTA per head (512 threads, 256 for P = 32 so that the 32-wide register
// rows fit); head_dim D and block width P fixed at compile time.
template <int D, int P>
__global__ void __launch_bounds__(P == 32 ? 256 : 512) refresh_kernel(const double* __restrict__ Mall, int64_t n,
                                                      int G, int r, int qfull,
                                                      float* __restrict__ sens,
                                                      float* __restrict__ wgroup,
                                                      float* __restrict__ basis_slot,
                                                      double* __restrict__ eigvec,
                                                      double* __restrict__ flags) {
  constexpr int d = D, p = P;
  extern __shared__ double sm[];
  const int h = blockIdx.x;
  const int tid = threadIdx.x, nt = blockDim.x;
  float* s_out = sens + (size_t)h * d;
  float* w_out = wgroup + (size_t)h * (d / G);
  float* U = basis_slot + (size_t)h * d * (r > 0 ? r : 1);
  float* snap = qsnap_of(eigvec, d, h);  // A = fp32(M / n) for the full-quadratic score
  if (n <= 0) {
    for (int j = tid; j < d; j += nt) s_out[j] = 1.0f;
    for (int e = tid; e < d * r; e += nt) U[e] = 0.0f;
    if (qfull)
      for (int e = tid; e < d * d; e += nt) snap[e] = 0.0f;
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
  if (qfull)
    for (int e = tid; e < d * d; e += nt) snap[e] = __double2float_rn(M[e] / (double)n);
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
  // ---- orthogonal iteration (the top-r subspace converges at rate
  // lambda_{p+1}/lambda_r per step), then a Rayleigh-Ritz step whose residuals
  // decide whether to go on: every one of the top r Ritz pairs must satisfy
  // |A v - theta v| <= 1e-7 theta_1, else 8 more steps follow, up to a bound.
  // Warm starts track a basis that moves little between refreshes.
  const int cap = warm ? 64 : 160;
  int target = warm ? 3 : 30;
  int it = 0;
  double* Xc = S.X;  // the current block; the product goes to the other buffer
  double* Yc = S.Y;
  double* Hc = S.G;  // Rayleigh quotient, rotated in place by the Jacobi
  double* W = S.L;   // its eigenvectors
  while (true) {
    for (; it < target; ++it) {
      cholqr<D, P>(Xc, S.G, S.L);
      gemm_AX<D, P>(S.A, Xc, Yc);
      double* t = Xc;
      Xc = Yc;
      Yc = t;
    }
    cholqr<D, P>(Xc, S.G, S.L);
    cholqr<D, P>(Xc, S.G, S.L);
    gemm_AX<D, P>(S.A, Xc, Yc);              // Y = A Q
    gram(Xc, Yc, Hc, d, p);                  // H = Q^T A Q (column-major, symmetric)
    small_jacobi<P>(Hc, W);
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
    if (tid < 32) S.red[tid] = 0.0;
    __syncthreads();
    // squared residuals of the top r Ritz pairs: (Y W_k - theta_k Q W_k)_i
    const int rr = r < p ? r : p;
    for (int e = tid; e < rr * d; e += nt) {
      const int c = e / d, i = e % d;
      const int k = S.ord[c];
      double av = 0.0, v = 0.0;
      for (int m = 0; m < p; ++m) {
        av = fma(Yc[m * (d + 1) + i], W[k * p + m], av);
        v = fma(Xc[m * (d + 1) + i], W[k * p + m], v);
      }
      const double res = av - S.th[k] * v;
      atomicAdd(&S.red[c], res * res);
    }
    __syncthreads();
    bool done = true;
    const double tol = 1e-7 * S.th[S.ord[0]];
    for (int c = 0; c < rr; ++c) done = done && (sqrt(S.red[c]) <= tol);
    if (done || it >= cap) break;
    target = it + 8;
    __syncthreads();
  }
  // Ritz vectors V = Q W (sorted), written to eigvec (column-major) for the
  // next warm start; the first r columns, sign-normalized, are U.
  double* Vout = eigvec + (size_t)h * d * d;
  for (int e = tid; e < p * d; e += nt) {
    const int c = e / d, i = e % d;
    const int k = S.ord[c];
    double acc = 0.0;
    for (int m = 0; m < p; ++m) acc = fma(Xc[m * (d + 1) + i], W[k * p + m], acc);
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
  const int nt = D.d / kTile;
  dim3 grid(nt * (nt + 1) / 2, D.H);
  stats_acc<<<grid, 64, 0, s>>>(Q, n, D.H, D.d, qstats);
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
  auto kern = refresh_kernel<128, 16>;
  if (D.d == 128 && p == 32) kern = refresh_kernel<128, 32>;
  else if (D.d == 64 && p == 16) kern = refresh_kernel<64, 16>;
  else if (D.d == 64 && p == 32) kern = refresh_kernel<64, 32>;
  else if (!(D.d == 128 && p == 16)) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<D.H, p == 32 ? 256 : 512, smem, s>>>(v.qstats, n_total, D.G, D.r, D.qsac_full, v.sens,
                                               v.wgroup, slot, v.eigvec, flags);
  return cudaGetLastError();
}

}  // namespace qwm
