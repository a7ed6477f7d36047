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
// U = top-r eigenvectors of A = M / n.  The eigenvectors come from one-sided
// (Hestenes) Jacobi in fp64 on X = A V0, where V0 is the previous refresh's
// eigenvector matrix (warm start: the statistics move little between frames,
// so one or two sweeps usually suffice) or the identity.  Rotations are
// applied to disjoint column pairs in round-robin order; at convergence the
// columns of X are A v_k = lambda_k v_k (A is positive semi-definite), so
// lambda_k = |x_k| and v_k = x_k / lambda_k.  Columns are ordered by
// descending lambda (ties: lower column) and each U column is signed so that
// its largest-magnitude entry (lowest index on ties) is positive.
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

// X0 (column-major [k][i]) = (M / n) V0 with V0 column-major (warm), or M / n
// (cold; M is symmetric so its rows are its columns).
__global__ void refresh_prep(const double* __restrict__ M, int64_t n, int d,
                             const double* __restrict__ eigvec, const double* __restrict__ flags,
                             double* __restrict__ X0) {
  const int h = blockIdx.y;
  const double* A = M + (size_t)h * d * d;
  const double* V = eigvec + (size_t)h * d * d;
  double* X = X0 + (size_t)h * d * d;
  const bool warm = flags[h] != 0.0;
  const double inv = 1.0 / (double)n;
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < d * d; e += gridDim.x * blockDim.x) {
    int k = e / d, i = e % d;
    double v;
    if (warm) {
      double acc = 0.0;
      for (int j = 0; j < d; ++j) acc += A[(size_t)i * d + j] * V[(size_t)k * d + j];
      v = acc * inv;
    } else {
      v = A[(size_t)k * d + i] * inv;
    }
    X[e] = v;
  }
}

// One CTA per head, 4*d threads (8 per column pair).
__global__ void refresh_jacobi(const double* __restrict__ M, int64_t n, int d, int G, int r,
                               const double* __restrict__ X0, float* __restrict__ sens,
                               float* __restrict__ wgroup, float* __restrict__ basis_slot,
                               double* __restrict__ eigvec, double* __restrict__ flags, int H) {
  extern __shared__ double X[];  // [d][d] column-major
  __shared__ double lam[128];
  __shared__ int order[128];
  __shared__ float sred[32];
  __shared__ int sweeps_done;
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
  const double* A = M + (size_t)h * d * d;
  for (int j = tid; j < d; j += nt) s_out[j] = __double2float_rn(A[(size_t)j * d + j] / (double)n);
  for (int e = tid; e < d * d; e += nt) X[e] = X0[(size_t)h * d * d + e];
  __syncthreads();
  if (tid < d / G) {
    float acc = 0.0f;
    for (int j = tid * G; j < (tid + 1) * G; ++j) acc = __fadd_rn(acc, s_out[j]);
    w_out[tid] = acc;
  }

  const int grp = tid / 8, sub = tid % 8;  // pair slot, lane within the pair group
  const int npairs = d / 2;
  const double tol = 1e-13;
  for (int sweep = 0; sweep < 40; ++sweep) {
    float worst = 0.0f;
    for (int rnd = 0; rnd < d - 1; ++rnd) {
      if (grp < npairs) {
        // circle method: position 0 fixed, the others rotate by `rnd`
        int a = (grp == 0) ? 0 : 1 + (grp - 1 + rnd) % (d - 1);
        int bpos = d - 1 - grp;
        int b = 1 + (bpos - 1 + rnd) % (d - 1);
        int p = min(a, b), q = max(a, b);
        double* xp = X + (size_t)p * d;
        double* xq = X + (size_t)q * d;
        double al = 0.0, be = 0.0, ga = 0.0;
        for (int i = sub; i < d; i += 8) {
          double u = xp[i], v = xq[i];
          al += u * u;
          be += v * v;
          ga += u * v;
        }
        for (int o = 4; o >= 1; o >>= 1) {
          al += __shfl_xor_sync(0xffffffffu, al, o);
          be += __shfl_xor_sync(0xffffffffu, be, o);
          ga += __shfl_xor_sync(0xffffffffu, ga, o);
        }
        double nrm = sqrt(al * be);
        if (ga != 0.0 && fabs(ga) > tol * nrm) {
          worst = fmaxf(worst, (float)(fabs(ga) / nrm));
          double zeta = (be - al) / (2.0 * ga);
          double t = (zeta >= 0.0 ? 1.0 : -1.0) / (fabs(zeta) + sqrt(1.0 + zeta * zeta));
          double c = 1.0 / sqrt(1.0 + t * t), s = c * t;
          for (int i = sub; i < d; i += 8) {
            double u = xp[i], v = xq[i];
            xp[i] = c * u - s * v;
            xq[i] = s * u + c * v;
          }
        }
      }
      __syncthreads();
    }
    // block max of the largest relative off-diagonal seen in this sweep
    for (int o = 16; o >= 1; o >>= 1) worst = fmaxf(worst, __shfl_xor_sync(0xffffffffu, worst, o));
    if (tid % 32 == 0) sred[tid / 32] = worst;
    __syncthreads();
    if (tid == 0) {
      float m = 0.0f;
      for (int w = 0; w < nt / 32; ++w) m = fmaxf(m, sred[w]);
      sweeps_done = (m <= 1e-12f) ? 1 : 0;
    }
    __syncthreads();
    if (sweeps_done) break;
    __syncthreads();
  }
  // eigenvalues as column norms (each 8-lane group handles d/(nt/8) = 2 columns)
  for (int k = grp; k < d; k += nt / 8) {
    double acc = 0.0;
    for (int i = sub; i < d; i += 8) acc += X[(size_t)k * d + i] * X[(size_t)k * d + i];
    for (int o = 4; o >= 1; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (sub == 0) lam[k] = sqrt(acc);
  }
  __syncthreads();
  double lmax = 0.0;
  for (int k = 0; k < d; ++k) lmax = fmax(lmax, lam[k]);
  if (tid < d) {
    double lk = lam[tid];
    int rank = 0;
    for (int j = 0; j < d; ++j) {
      double lj = lam[j];
      rank += (lj > lk) || (lj == lk && j < tid);
    }
    order[rank] = tid;
  }
  __syncthreads();
  const double floor_l = lmax * 1e-12;
  // normalized eigenvectors -> eigvec (column-major, same column order as X)
  for (int e = tid; e < d * d; e += nt) {
    int k = e / d;
    double lk = lam[k];
    eigvec[(size_t)h * d * d + e] = (lk > floor_l) ? X[e] / lk : 0.0;
  }
  // U columns, sign-normalized; every 8-lane group runs the shuffles (r <= nt/8)
  {
    const int c = grp;
    const bool act = c < r;
    const int k = order[act ? c : 0];
    const double lk = lam[k];
    const double* x = X + (size_t)k * d;
    double big = -1.0;
    int arg = 0;
    for (int i = sub; i < d; i += 8) {
      double m = fabs(x[i]);
      if (m > big) { big = m; arg = i; }
    }
    for (int o = 4; o >= 1; o >>= 1) {
      double ob = __shfl_xor_sync(0xffffffffu, big, o);
      int oa = __shfl_xor_sync(0xffffffffu, arg, o);
      if (ob > big || (ob == big && oa < arg)) { big = ob; arg = oa; }
    }
    const double sg = (x[arg] < 0.0) ? -1.0 : 1.0;
    if (act)
      for (int i = sub; i < d; i += 8) {
        double v = (lk > floor_l) ? sg * x[i] / lk : 0.0;
        U[(size_t)i * r + c] = __double2float_rn(v);
      }
  }
  if (tid == 0) {
    bool ok = lmax > 0.0;
    for (int k = 0; k < d; ++k) ok = ok && (lam[k] > lmax * 1e-8);
    flags[h] = ok ? 1.0 : 0.0;
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

cudaError_t launch_refresh(const Dims& D, const CacheView& v, int64_t n_total, int version,
                           int /*warm_hint*/, cudaStream_t s) {
  double* flags = v.eigvec + (size_t)D.H * D.d * D.d;
  double* X0 = (double*)v.workspace;
  float* slot = v.basis + (size_t)version * D.H * D.d * (D.r > 0 ? D.r : 1);
  if (n_total > 0) {
    refresh_prep<<<dim3(16, D.H), 256, 0, s>>>(v.qstats, n_total, D.d, v.eigvec, flags, X0);
  }
  size_t smem = (size_t)D.d * D.d * sizeof(double);
  cudaError_t e =
      cudaFuncSetAttribute(refresh_jacobi, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  refresh_jacobi<<<D.H, 4 * D.d, smem, s>>>(v.qstats, n_total, D.d, D.G, D.r, X0, v.sens,
                                            v.wgroup, slot, v.eigvec, flags, D.H);
  return cudaGetLastError();
}

}  // namespace qwm
