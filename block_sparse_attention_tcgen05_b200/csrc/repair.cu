// SparsePR probe-fitted residual repair.
//
// Sources: "Sparse-block compensation" (mlx-arsenal notes), §SparsePR — probe-fitted
// residual repair (residual R = O_dense - O_sparse on the probe rows; weighted ridge
// fit from the standardised sparse output; projection on the top-16 residual
// directions; applied to every row; per call and per (batch, head)), §Deviations
// (weights normalised to sum 1); "Partition the Support, Reconstruct the Residual"
// (ridge lambda = 0.1, r = 16, affine map, corrections kept inside the output subspace
// seen in the probe residuals).
//
// Per (b, h) with X = out[b,h] (S x D), mu / sigma its column mean and population
// standard deviation (+1e-6 in the variance), Zt = [(X - mu)/sigma, 1], W = diag(w):
//   Bc  = (Zt_pᵀ W Zt_p + lam·diag(1,..,1,0))⁻¹ Zt_pᵀ W R      Cholesky in shared memory
//   V_r = top-r eigenvectors of Rᵀ W R                         Householder tridiagonalisation,
//                                                              bisection, inverse iteration on
//                                                              the smaller of Rᵀ W R and
//                                                              W½ R Rᵀ W½
//   out += Zt Bc V_r V_rᵀ = (X P' + c') V_rᵀ,  P' = diag(1/sigma) Bc[:D] V_r,
//          c' = (Bc[D] - Σ_i mu_i/sigma_i Bc[i]) V_r      (rank-r update, one HBM pass)
#include <cmath>

#include "common.cuh"
#include "ptx.cuh"

namespace bsa {

constexpr int kStatSplit = 32;
constexpr int kFitThreads = 512;

// grid (kStatSplit, B*H), 256 threads: partial column sums of (x - x_0) and its square,
// x_0 = the first row, over a slice of the rows.
__global__ void __launch_bounds__(256) column_stats_kernel(const float* __restrict__ out, int S,
                                                           int D, float* __restrict__ psum,
                                                           float* __restrict__ psq) {
  __shared__ float s1[256], s2[256];
  const int64_t bh = blockIdx.y;
  const float* X = out + bh * S * D;
  const int d = threadIdx.x % D, lane_row = threadIdx.x / D, rows_per = 256 / D;
  const int r0 = static_cast<int>((static_cast<int64_t>(S) * blockIdx.x) / kStatSplit);
  const int r1 = static_cast<int>((static_cast<int64_t>(S) * (blockIdx.x + 1)) / kStatSplit);
  const float x0 = X[d];
  float a = 0.f, b = 0.f;
  for (int r = r0 + lane_row; r < r1; r += rows_per) {
    const float x = X[static_cast<int64_t>(r) * D + d] - x0;
    a += x;
    b = fmaf(x, x, b);
  }
  s1[threadIdx.x] = a;
  s2[threadIdx.x] = b;
  __syncthreads();
  if (threadIdx.x < D) {
    float ta = 0.f, tb = 0.f;
    for (int k = 0; k < rows_per; ++k) {
      ta += s1[k * D + threadIdx.x];
      tb += s2[k * D + threadIdx.x];
    }
    psum[(bh * kStatSplit + blockIdx.x) * D + threadIdx.x] = ta;
    psq[(bh * kStatSplit + blockIdx.x) * D + threadIdx.x] = tb;
  }
}

struct FitArgs {
  const float* out;
  const float* o_probe;
  const int32_t* probe_idx;
  const float* weights;
  int per_head, S, D, M, rank;
  float lam;
  const float* psum;
  const float* psq;
  float* zt;   // [BH][M][D+2]   (used when they do not fit in shared memory)
  float* rr;   // [BH][M][D+1]
  float* rv;   // [BH][M][rank]
  float* vr;   // [BH][D][rank]
  float* pp;   // [BH][D][rank]
  float* cc;   // [BH][rank]
};

__device__ __forceinline__ float block_sum(float v, float* red) {
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  float t = 0.f;
  if (threadIdx.x < 32) {
    t = threadIdx.x < static_cast<int>(blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
    for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
    if (threadIdx.x == 0) red[0] = t;
  }
  __syncthreads();
  return red[0];
}


// Top-k eigenpairs of a symmetric n x n matrix A (n <= 128, row stride ld, in shared
// memory), all threads of the CTA taking part:
//  1. Householder reduction to tridiagonal form T = Hᵀ A H (reflector k in hv row k,
//     A overwritten), diag d, off-diagonal e;
//  2. the k largest eigenvalues of T by multisection on Sturm counts (one warp each:
//     32 points per round split the bracket into 33 parts);
//  3. their eigenvectors by inverse iteration on T (one thread each), then Gram-Schmidt
//     in order of decreasing eigenvalue (classical, applied twice, all warps);
//  4. back-transformation by the reflectors: U = H x.
// Output: U (n x min(k, n), row stride ld >= n) and lam[0..k) in decreasing order
// (zero past n). hv needs n x ld floats, x n x k, work 5n + 2 k n floats.
__device__ void top_eigenpairs(float* A, int ld, int n, int k, float* hv, float* U, float* lam,
                               float* x, float* work, float* red) {
  const int tid = threadIdx.x, nt = blockDim.x;
  const int lane = tid & 31, wid = tid >> 5, nw = nt >> 5;
  float* d = work;
  float* e = work + n;        // e[i] couples i and i+1
  float* pv = work + 2 * n;   // A v
  __shared__ float s_scal[2];
  // 1. Householder: column c below the diagonal is mapped to (alpha, 0, ..., 0). Three
  //    block barriers per step: warp 0 forms the reflector (column norm by shuffles);
  //    the warps form p = A' v; every warp then takes v·p on its own (the same sum in
  //    the same order) and applies the rank-2 update with w = 2 (p - (v·p) v) formed in
  //    place.
  __shared__ int s_skip;
  for (int c = 0; c + 2 < n; ++c) {
    const int m = n - c - 1;  // length of the column below the diagonal
    float* v = hv + c * ld;
    if (wid == 0) {
      float ss = 0.f;
      for (int i = lane; i < m; i += 32) {
        const float xi = A[(c + 1 + i) * ld + c];
        ss = fmaf(xi, xi, ss);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      const float x0 = A[(c + 1) * ld + c];
      const float nrm = sqrtf(ss);
      const float alpha = x0 > 0.f ? -nrm : nrm;
      // v = x - alpha e1, normalised; |v|^2 = ss - 2 alpha x0 + alpha^2 = 2(ss - alpha x0)
      const float vv = 2.f * (ss - alpha * x0);
      const bool skip = !(vv > 1e-30f * (ss + 1e-30f));
      const float inv = skip ? 0.f : rsqrtf(vv);
      for (int i = lane; i < m; i += 32) {
        const float xi = A[(c + 1 + i) * ld + c];
        v[i] = (i == 0 ? xi - alpha : xi) * inv;
      }
      if (lane == 0) {
        d[c] = A[c * ld + c];
        e[c] = skip ? x0 : alpha;
        s_skip = skip ? 1 : 0;
      }
    }
    __syncthreads();
    if (!s_skip) {
      // p = A' v over the trailing block A' = A[c+1.., c+1..]: a warp per row, lanes
      // along it; four rows of a warp at a time, their shuffle sums interleaved
      for (int i0 = wid; i0 < m; i0 += 4 * nw) {
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const int i = i0 + r * nw;
          if (i < m)
            for (int j = lane; j < m; j += 32) acc[r] = fmaf(A[(c + 1 + i) * ld + c + 1 + j], v[j], acc[r]);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
          for (int r = 0; r < 4; ++r) acc[r] += __shfl_xor_sync(0xffffffffu, acc[r], o);
        }
        if (lane == 0) {
#pragma unroll
          for (int r = 0; r < 4; ++r)
            if (i0 + r * nw < m) pv[i0 + r * nw] = acc[r];
        }
      }
      __syncthreads();
      float kk = 0.f;
      for (int i = lane; i < m; i += 32) kk = fmaf(v[i], pv[i], kk);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) kk += __shfl_xor_sync(0xffffffffu, kk, o);
      // A' <- A' - v wᵀ - w vᵀ  (= H A' H with H = I - 2 v vᵀ)
      // a warp per row, lanes along it (no index division)
      for (int i = wid; i < m; i += nw) {
        const float vi = v[i], wi = 2.f * (pv[i] - kk * vi);
        float* row = A + (c + 1 + i) * ld + c + 1;
        for (int j = lane; j < m; j += 32) {
          const float vj = v[j], wj = 2.f * (pv[j] - kk * vj);
          row[j] -= vi * wj + wi * vj;
        }
      }
    }
    __syncthreads();
  }
  if (tid == 0) {
    for (int c = (n >= 2 ? n - 2 : 0); c < n; ++c) d[c] = A[c * ld + c];
    if (n >= 2) e[n - 2] = A[(n - 1) * ld + (n - 2)];
  }
  __syncthreads();
  // 2. multisection: eigenvalue j (ascending) of T is the x where the Sturm count
  //    #{eigenvalues < x} passes j; warp w takes the w-th largest (then w + nw, ...),
  //    j = n - 1 - t
  float* e2 = work + 4 * n;
  for (int i = tid; i < n; i += nt) e2[i] = i + 1 < n ? e[i] * e[i] : 0.f;
  if (tid == 0) {
    float lo = INFINITY, hi = -INFINITY, emax = 0.f;
    for (int i = 0; i < n; ++i) {
      const float r = (i > 0 ? fabsf(e[i - 1]) : 0.f) + (i + 1 < n ? fabsf(e[i]) : 0.f);
      lo = fminf(lo, d[i] - r);
      hi = fmaxf(hi, d[i] + r);
      if (i + 1 < n) emax = fmaxf(emax, e2[i]);
    }
    const float span = fmaxf(hi - lo, 1e-30f);
    s_scal[0] = lo - 1e-6f * span;
    s_scal[1] = hi + 1e-6f * span;
  }
  __syncthreads();
  const int kk = k < n ? k : n;
  const float lo0 = s_scal[0], hi0 = s_scal[1];
  const float pivmin = 1e-30f + 1e-12f * (hi0 - lo0) * (hi0 - lo0);
  for (int t = wid; t < kk; t += nw) {
    const int j = n - 1 - t;
    float a = lo0, b = hi0;
    for (int it = 0; it < 40; ++it) {
      // lane l evaluates the count at the (l+1)-th of 32 interior points of [a, b]
      const float xl = a + (b - a) * (static_cast<float>(lane + 1) * (1.f / 33.f));
      int cnt = 0;
      float q = d[0] - xl;
      for (int i = 0;; ++i) {
        if (fabsf(q) < pivmin) q = -pivmin;
        cnt += q < 0.f;
        if (i + 1 >= n) break;
        q = d[i + 1] - xl - __fdividef(e2[i], q);
      }
      // the first point whose count exceeds j closes the new bracket, the point before
      // it opens it (a and b when there is none)
      const unsigned above = __ballot_sync(0xffffffffu, cnt > j);
      const int p = above ? __ffs(above) - 1 : 32;
      const float xa = __shfl_sync(0xffffffffu, xl, p > 0 ? p - 1 : 0);
      const float xb = __shfl_sync(0xffffffffu, xl, p < 32 ? p : 31);
      const float na = p > 0 ? fmaxf(xa, a) : a;
      const float nb = p < 32 ? fminf(xb, b) : b;
      if (!(nb - na < b - a)) break;  // float resolution reached
      a = na;
      b = nb;
    }
    if (lane == 0) lam[t] = 0.5f * (a + b);
  }
  __syncthreads();
  // 3. inverse iteration: solve (T - lam I) y = x by elimination with guarded pivots
  //    (thread t factors T - lam_t I once, its factors in cs and rmv row t), normalise;
  //    3 rounds. The next step's operands are loaded ahead of the recurrence.
  float* cs = work + 5 * n;   // k x n: f_i = e_i / m_i
  float* rmv = cs + k * n;    // k x n: 1 / m_i
  if (tid < kk) {
    const float lt = lam[tid];
    float* f = cs + tid * n;
    float* rm = rmv + tid * n;
    {
      float fprev = 0.f;
      for (int i = 0; i < n; ++i) {
        float mi = d[i] - lt - (i > 0 ? e[i - 1] * fprev : 0.f);
        if (fabsf(mi) < pivmin) mi = mi < 0.f ? -pivmin : pivmin;
        const float r = 1.f / mi;
        rm[i] = r;
        fprev = i + 1 < n ? e[i] * r : 0.f;
        f[i] = fprev;
      }
    }
    for (int i = 0; i < n; ++i) x[i * k + tid] = 1.f + 0.25f * static_cast<float>((i * 7 + tid * 13) % 11) / 11.f;
    for (int round = 0; round < 3; ++round) {
      // forward: y_i = (x_i - e_{i-1} y_{i-1}) / m_i
      float yprev = 0.f;
      float xn = x[tid], rn_ = rm[0], en = 0.f;
      for (int i = 0; i < n; ++i) {
        const float xi = xn, ri = rn_, ei = en;
        if (i + 1 < n) {
          xn = x[(i + 1) * k + tid];
          rn_ = rm[i + 1];
          en = e[i];
        }
        yprev = (xi - ei * yprev) * ri;
        x[i * k + tid] = yprev;
      }
      // back: y_i -= f_i y_{i+1}
      float nrm = yprev * yprev;
      float ynext = yprev;
      float xp = n >= 2 ? x[(n - 2) * k + tid] : 0.f, fp = n >= 2 ? f[n - 2] : 0.f;
      for (int i = n - 2; i >= 0; --i) {
        const float xi = xp, fi = fp;
        if (i > 0) {
          xp = x[(i - 1) * k + tid];
          fp = f[i - 1];
        }
        const float yi = xi - fi * ynext;
        x[i * k + tid] = yi;
        nrm = fmaf(yi, yi, nrm);
        ynext = yi;
      }
      const float rs = nrm > 0.f ? rsqrtf(nrm) : 0.f;
      for (int i = 0; i < n; ++i) x[i * k + tid] *= rs;
    }
  }
  __syncthreads();
  //    Gram-Schmidt in order of decreasing eigenvalue, classical and applied twice: the
  //    projections of vector t on the vectors before it are taken together (a warp per
  //    projection); repairs the loss of orthogonality of inverse iteration within
  //    clusters of eigenvalues
  for (int t = 0; t < kk; ++t) {
    for (int pass = 0; pass < 2; ++pass) {
      for (int s2 = wid; s2 < t; s2 += nw) {
        float dot = 0.f;
        for (int i = lane; i < n; i += 32) dot = fmaf(x[i * k + s2], x[i * k + t], dot);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
        if (lane == 0) pv[s2] = dot;
      }
      __syncthreads();
      for (int i = tid; i < n; i += nt) {
        float v = x[i * k + t];
        for (int s2 = 0; s2 < t; ++s2) v = fmaf(-pv[s2], x[i * k + s2], v);
        x[i * k + t] = v;
      }
      __syncthreads();
    }
    float nrm = 0.f;
    for (int i = tid; i < n; i += nt) nrm = fmaf(x[i * k + t], x[i * k + t], nrm);
    nrm = block_sum(nrm, red);
    const float rn = nrm > 0.f ? rsqrtf(nrm) : 0.f;
    for (int i = tid; i < n; i += nt) x[i * k + t] *= rn;
    __syncthreads();
  }
  // 4. back-transformation: x <- H_c x for c = n-3 .. 0, H_c = I - 2 v_c v_cᵀ on rows c+1..
  for (int c = n - 3; c >= 0; --c) {
    const int m = n - c - 1;
    if (tid < kk) {
      float s = 0.f;
      for (int i = 0; i < m; ++i) s = fmaf(hv[c * ld + i], x[(c + 1 + i) * k + tid], s);
      pv[tid] = 2.f * s;
    }
    __syncthreads();
    for (int e3 = tid; e3 < m * kk; e3 += nt) {
      const int i = e3 / kk, t = e3 % kk;
      x[(c + 1 + i) * k + t] -= hv[c * ld + i] * pv[t];
    }
    __syncthreads();
  }
  for (int e3 = tid; e3 < n * kk; e3 += nt) {  // only the kk <= n columns that exist
    const int i = e3 / kk, t = e3 % kk;
    U[i * ld + t] = x[i * k + t];
  }
  for (int t = kk + tid; t < k; t += nt) lam[t] = 0.f;
  __syncthreads();
}

// Solves A X = B in place for SPD A (n x n, row stride lda) and B (n x nr): Cholesky
// without the column scaling (after step k the lower triangle holds A[i][k] = L[i][k]·s_k
// with s_k = L[k][k] = sqrt(A[k][k]); one barrier per step), then forward and backward
// substitution by one warp (lanes across 16 right-hand side columns and two row
// parities, no block barrier per step). rpiv (n floats) receives 1 / s_k. All threads of
// the CTA take part.
__device__ void chol_solve(float* A, int n, int lda, float* B, int nr, float* rpiv) {
  const int tid = threadIdx.x, nt = blockDim.x, lane = tid & 31, wid = tid >> 5, nw = nt >> 5;
  for (int k = 0; k < n; ++k) {
    const float rdk = 1.f / fmaxf(A[k * lda + k], 1e-30f);
    for (int i = k + 1 + wid; i < n; i += nw) {  // warps along rows, lanes along columns
      const float aik = A[i * lda + k] * rdk;
      for (int j = k + 1 + lane; j <= i; j += 32) A[i * lda + j] -= aik * A[j * lda + k];
    }
    __syncthreads();
  }
  for (int k = tid; k < n; k += nt) rpiv[k] = 1.f / sqrtf(fmaxf(A[k * lda + k], 1e-30f));
  __syncthreads();
  if (wid == 0) {
    // one warp: lane (c, h) = (l % 16, l / 16) takes right-hand side column c0 + c over
    // the rows of parity h (consecutive lanes on consecutive words of a row of B); eight
    // rows loaded before any is stored
    const int cl = lane & 15, hl = lane >> 4;
    for (int c0 = 0; c0 < nr; c0 += 16) {
      const int c = c0 + cl;
      const bool on = c < nr;
      // forward  b_i -= (A[i][k] / s_k) (b_k / s_k), i > k;  then y_k = b_k / s_k
      for (int k = 0; k < n - 1; ++k) {
        if (on) {
          const float bk = B[k * nr + c] * (rpiv[k] * rpiv[k]);
          for (int i0 = k + 1 + hl; i0 < n; i0 += 16) {
            float bv[8], av[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              const int i = i0 + 2 * u;
              bv[u] = i < n ? B[i * nr + c] : 0.f;
              av[u] = i < n ? A[i * lda + k] : 0.f;
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              const int i = i0 + 2 * u;
              if (i < n) B[i * nr + c] = bv[u] - av[u] * bk;
            }
          }
        }
        __syncwarp();
      }
      if (on)
        for (int i = hl; i < n; i += 2) B[i * nr + c] *= rpiv[i];
      __syncwarp();
      // backward y_i -= (A[k][i] / s_i) (y_k / s_k), i < k;  then x_k = y_k / s_k
      for (int k = n - 1; k > 0; --k) {
        if (on) {
          const float bk = B[k * nr + c] * rpiv[k];
          for (int i0 = hl; i0 < k; i0 += 16) {
            float bv[8], av[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              const int i = i0 + 2 * u;
              bv[u] = i < k ? B[i * nr + c] : 0.f;
              av[u] = i < k ? A[k * lda + i] * rpiv[i] : 0.f;
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              const int i = i0 + 2 * u;
              if (i < k) B[i * nr + c] = bv[u] - av[u] * bk;
            }
          }
        }
        __syncwarp();
      }
      if (on)
        for (int i = hl; i < n; i += 2) B[i * nr + c] *= rpiv[i];
      __syncwarp();
    }
  }
  __syncthreads();
}

// Shared-memory plan of the fit, in floats: the standardised probe rows Zt (M x ldz)
// and residuals R (M x ldr) and R V_r (M x rk) when they fit (else they stay in the
// workspace), a region W used first by the eigen step (the Gram matrix, later its
// eigenvectors, n x ld; the reflectors n x ld; inverse-iteration vectors n x rk and
// scratch) and then by the solve (primal: A n1 x n1 and right-hand sides n1 x rk; dual:
// K M x M, right-hand sides M x rk and the solution n1 x rk), V_r (D x rk) and the
// Cholesky pivots.
struct FitPlan {
  int n1, n, ld, ldz, ldr, rk;
  bool local_zr;                   // Zt, R, R V_r in shared memory
  size_t zt, rr, rv, w, vr, piv;   // offsets (floats) into the dynamic shared memory
  size_t floats;
};
__host__ __device__ inline FitPlan fit_plan(int D, int M, int rk) {
  FitPlan p{};
  p.n1 = D + 1;
  p.n = M < D ? M : D;
  p.ld = (p.n + 1) | 1;  // odd: rows on distinct banks
  p.ldz = D + 3;  // odd: probe rows on distinct banks
  p.ldr = D + 1;
  p.rk = rk;
  const size_t wa = static_cast<size_t>(2) * p.n * p.ld + static_cast<size_t>(3) * p.n * rk +
                    static_cast<size_t>(5) * p.n;
  const size_t wb_primal = static_cast<size_t>(p.n1) * (p.n1 | 1) + static_cast<size_t>(p.n1) * rk;
  const size_t wb_dual = M < p.n1 ? static_cast<size_t>(M) * (M | 1) + static_cast<size_t>(M) * rk +
                                        static_cast<size_t>(p.n1) * rk
                                  : 0;
  const size_t wb = wb_primal > wb_dual ? wb_primal : wb_dual;
  const size_t wsz = wa > wb ? wa : wb;
  const size_t common = wsz + static_cast<size_t>(D) * rk + p.n1;
  const size_t zr = static_cast<size_t>(M) * (p.ldz + p.ldr + rk);
  p.local_zr = (common + zr) * sizeof(float) <= 200 * 1024;
  size_t o = 0;
  if (p.local_zr) {
    p.zt = o; o += static_cast<size_t>(M) * p.ldz;
    p.rr = o; o += static_cast<size_t>(M) * p.ldr;
    p.rv = o; o += static_cast<size_t>(M) * rk;
  }
  p.w = o; o += wsz;
  p.vr = o; o += static_cast<size_t>(D) * rk;
  p.piv = o; o += p.n1;
  p.floats = o;
  return p;
}

// One CTA (512 threads) per (b, h): statistics, the residual subspace V_r, then the
// ridge solve for Bc V_r only (Bc itself is never needed: the apply uses Bc V_r), and
// the folded rank-r factors P', c' for the apply pass.
__global__ void __launch_bounds__(kFitThreads, 1) repair_fit_kernel(const FitArgs a) {
  extern __shared__ float sm_fit[];
  __shared__ float mu[128], isg[128], red[32];
  __shared__ float wv[1024], sqw[1024];  // probe weights and their square roots
  __shared__ int sel[128];
  __shared__ float evl[128];  // eigenvalues of the residual Gram matrix, decreasing
  __shared__ float zbar[128], tbar[128];  // weighted probe means of Z and R V_r (dual solve)
  const int tid = threadIdx.x, nt = blockDim.x;
  const int64_t bh = blockIdx.x;
  const int S = a.S, D = a.D, M = a.M, rk = a.rank;
  const FitPlan pl = fit_plan(D, M, rk);
  const int n1 = pl.n1, n = pl.n, ld = pl.ld, ldz = pl.ldz, ldr = pl.ldr;
  const bool small = M < D;
  const float* X = a.out + bh * S * D;
  const int32_t* idx = a.per_head ? a.probe_idx + bh * M : a.probe_idx;
  const float* w = a.per_head ? a.weights + bh * M : a.weights;
  float* zt = pl.local_zr ? sm_fit + pl.zt : a.zt + bh * M * ldz;
  float* rr = pl.local_zr ? sm_fit + pl.rr : a.rr + bh * M * ldr;
  float* rv = pl.local_zr ? sm_fit + pl.rv : a.rv + bh * M * rk;
  float* W = sm_fit + pl.w;
  float* vrs = sm_fit + pl.vr;
  float* piv = sm_fit + pl.piv;

  // 1. column statistics
  if (tid < D) {
    float s1 = 0.f, s2 = 0.f;
    for (int k = 0; k < kStatSplit; ++k) {
      s1 += a.psum[(bh * kStatSplit + k) * D + tid];
      s2 += a.psq[(bh * kStatSplit + k) * D + tid];
    }
    const float m1 = s1 / static_cast<float>(S);
    const float var = fmaxf(s2 / static_cast<float>(S) - m1 * m1, 0.f);
    mu[tid] = X[tid] + m1;
    isg[tid] = 1.f / sqrtf(var + 1e-6f);
  }
  for (int m = tid; m < M; m += nt) {
    wv[m] = w[m];
    sqw[m] = sqrtf(w[m]);
  }
  for (int k = tid; k < 128; k += nt) sel[k] = -1;
  __syncthreads();
  // 2. standardised probe rows Zt = [(x - mu) / sigma, 1] and residuals R = o_probe - x
  // A probe index outside [0, S) is reported in the device status word (site 70) and
  // clamped, so that the reads stay inside this head's rows.
  for (int m = tid; m < M; m += nt)
    if (idx[m] < 0 || idx[m] >= S) report_device_error(kStatusBadLabel, 70);
  for (int e = tid; e < M * D; e += nt) {
    const int m = e / D, d = e % D;
    int row = idx[m];
    row = row < 0 ? 0 : (row >= S ? S - 1 : row);
    const float x = X[static_cast<int64_t>(row) * D + d];
    zt[m * ldz + d] = (x - mu[d]) * isg[d];
    rr[m * ldr + d] = a.o_probe[(bh * M + m) * D + d] - x;
  }
  for (int m = tid; m < M; m += nt) zt[m * ldz + D] = 1.f;
  __syncthreads();
  // 3. Gram matrix of the weighted residuals, n x n with n = min(M, D):
  //    W½ R Rᵀ W½ (M < D) or Rᵀ W R
  float* G = W;              // n x ld; its eigenvectors later overwrite it (V)
  float* V = W;
  for (int e = tid; e < n * n; e += nt) {
    const int i = e / n, j = e % n;
    float acc = 0.f;
    if (small) {
      for (int d = 0; d < D; ++d) acc = fmaf(rr[i * ldr + d], rr[j * ldr + d], acc);
      acc *= sqrtf(wv[i] * wv[j]);
    } else {
      for (int m = 0; m < M; ++m) acc = fmaf(wv[m] * rr[m * ldr + i], rr[m * ldr + j], acc);
    }
    G[i * ld + j] = acc;
  }
  __syncthreads();
  // 4-5. the rk largest eigenpairs (Householder tridiagonalisation, bisection, inverse
  //      iteration); slots past n stay -1 (those directions are left out)
  {
    float* hvb = W + n * ld;
    float* xb = hvb + n * ld;
    float* wk = xb + n * rk;
    top_eigenpairs(G, ld, n, rk, hvb, V, evl, xb, wk, red);
    for (int t = tid; t < 128; t += nt) sel[t] = t < rk && t < n ? t : -1;
    __syncthreads();
  }
  // 6. V_r (D x rk): eigenvectors of Rᵀ W R, directly (M >= D) or as
  //    (W½ R)ᵀ u / sqrt(l) from those of W½ R Rᵀ W½ (M < D)
  const float lmax = n > 0 && sel[0] >= 0 ? evl[0] : 0.f;
  float* vr = a.vr + bh * D * rk;
  for (int e = tid; e < D * rk; e += nt) {
    const int d = e / rk, k = e % rk;
    const int i = sel[k];
    float val = 0.f;
    if (i >= 0) {
      if (!small) {
        val = V[d * ld + i];
      } else {
        const float lam_i = evl[i];
        if (lam_i > 1e-12f * lmax && lam_i > 0.f) {
          float acc = 0.f;
          for (int m = 0; m < M; ++m) acc = fmaf(sqw[m] * rr[m * ldr + d], V[m * ld + i], acc);
          val = acc / sqrtf(lam_i);
        }
      }
    }
    vrs[e] = val;
    vr[e] = val;
  }
  __syncthreads();
  // 7. R V_r (M x rk)
  for (int e = tid; e < M * rk; e += nt) {
    const int m = e / rk, k = e % rk;
    float acc = 0.f;
    for (int d = 0; d < D; ++d) acc = fmaf(rr[m * ldr + d], vrs[d * rk + k], acc);
    rv[e] = acc;
  }
  __syncthreads();
  // 8-10. X = Bc V_r ((D+1) x rk), the ridge solution for the targets T = R V_r:
  //   primal (M >= D+1): A X = B with A = Ztᵀ W Zt + lam·I' (intercept unpenalised) and
  //     B = Ztᵀ W T, by Cholesky (D+1 steps);
  //   dual (M < D+1, the same solution through M x M): the unpenalised intercept is
  //     taken out by weighted centring (zbar, Tbar: weighted means over the probes), then
  //     beta = Ucᵀ (Uc Ucᵀ + lam I)⁻¹ W½ T_c with Uc = W½ (Z - 1 zbarᵀ) (push-through
  //     identity), and the intercept row Tbar - zbarᵀ beta.
  float* Xs;
  if (M < n1) {
    const int ldk = M | 1;       // odd row stride (distinct banks per row)
    float* Kd = W;               // M x M
    float* Yd = Kd + M * ldk;    // M x rk: W½ T_c, then the dual solution
    Xs = Yd + M * rk;            // (D+1) x rk
    float sw = 0.f;
    for (int m = tid; m < M; m += nt) sw += wv[m];
    sw = block_sum(sw, red);
    const float isw = sw > 0.f ? 1.f / sw : 0.f;
    for (int d = tid; d < D; d += nt) {
      float acc = 0.f;
      for (int m = 0; m < M; ++m) acc = fmaf(wv[m], zt[m * ldz + d], acc);
      zbar[d] = acc * isw;
    }
    for (int k = tid; k < rk; k += nt) {
      float acc = 0.f;
      for (int m = 0; m < M; ++m) acc = fmaf(wv[m], rv[m * rk + k], acc);
      tbar[k] = acc * isw;
    }
    __syncthreads();
    for (int e = tid; e < M * D; e += nt) {  // Uc in place of the probe rows of Z
      const int m = e / D, d = e % D;
      zt[m * ldz + d] = sqw[m] * (zt[m * ldz + d] - zbar[d]);
    }
    for (int e = tid; e < M * rk; e += nt) {
      const int m = e / rk, k = e % rk;
      Yd[e] = sqw[m] * (rv[e] - tbar[k]);
    }
    __syncthreads();
    {
      // K = Uc Ucᵀ + lam I: a warp per row i, lanes along the columns j <= i (M <= 128)
      const int ln = tid & 31, wd = tid >> 5, nwd = nt >> 5;
      for (int i = wd; i < M; i += nwd) {
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        for (int d = 0; d < D; ++d) {
          const float u = zt[i * ldz + d];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const int j = ln + 32 * c;
            if (j <= i) acc[c] = fmaf(u, zt[j * ldz + d], acc[c]);
          }
        }
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int j = ln + 32 * c;
          if (j <= i) {
            const float v = acc[c] + (i == j ? a.lam : 0.f);
            Kd[i * ldk + j] = v;
            Kd[j * ldk + i] = v;
          }
        }
      }
    }
    __syncthreads();
    chol_solve(Kd, M, ldk, Yd, rk, piv);
    for (int e = tid; e < D * rk; e += nt) {  // beta = Ucᵀ Y
      const int d = e / rk, k = e % rk;
      float acc = 0.f;
      for (int m = 0; m < M; ++m) acc = fmaf(zt[m * ldz + d], Yd[m * rk + k], acc);
      Xs[e] = acc;
    }
    __syncthreads();
    for (int k = tid; k < rk; k += nt) {  // intercept row
      float acc = tbar[k];
      for (int d = 0; d < D; ++d) acc = fmaf(-zbar[d], Xs[d * rk + k], acc);
      Xs[D * rk + k] = acc;
    }
    __syncthreads();
  } else {
    const int lda = n1 | 1;    // odd row stride
    float* A = W;              // n1 x n1 (overwrites G, V: no longer needed)
    float* Bm = W + n1 * lda;  // n1 x rk
    Xs = Bm;
    {
      // a warp per row i, lanes along the columns j <= i (at most 5 per lane: n1 <= 129)
      const int lane8 = tid & 31, wid8 = tid >> 5, nw8 = nt >> 5;
      for (int i = wid8; i < n1; i += nw8) {
        float acc[5] = {0.f, 0.f, 0.f, 0.f, 0.f};
        for (int m = 0; m < M; ++m) {
          const float wz = wv[m] * zt[m * ldz + i];
#pragma unroll
          for (int c = 0; c < 5; ++c) {
            const int j = lane8 + 32 * c;
            if (j <= i) acc[c] = fmaf(wz, zt[m * ldz + j], acc[c]);
          }
        }
#pragma unroll
        for (int c = 0; c < 5; ++c) {
          const int j = lane8 + 32 * c;
          if (j <= i) {
            const float v = acc[c] + ((i == j && i < D) ? a.lam : 0.f);
            A[i * lda + j] = v;
            A[j * lda + i] = v;
          }
        }
      }
    }
    for (int e = tid; e < n1 * rk; e += nt) {
      const int i = e / rk, k = e % rk;
      float acc = 0.f;
      for (int m = 0; m < M; ++m) acc = fmaf(wv[m] * zt[m * ldz + i], rv[m * rk + k], acc);
      Bm[e] = acc;
    }
    __syncthreads();
    chol_solve(A, n1, lda, Bm, rk, piv);
  }
  // 11. folded factors from X = Bc V_r: P' = diag(1/sigma) X[:D],
  //     c' = X[D] - Σ_i (mu_i / sigma_i) X[i]
  float* pp = a.pp + bh * D * rk;
  for (int e = tid; e < D * rk; e += nt) pp[e] = Xs[e] * isg[e / rk];
  for (int k = tid; k < rk; k += nt) {
    float acc = Xs[D * rk + k];
    for (int i = 0; i < D; ++i) acc -= mu[i] * isg[i] * Xs[i * rk + k];
    a.cc[bh * rk + k] = acc;
  }
}

// Sum of 16 per-lane values over the warp: a reduce-scatter butterfly (the halves a
// lane gives away shrink 8, 4, 2, 1), then one exchange across lane pairs. Afterwards
// lane l holds the warp total of value slot(l), slot(l) = the bits 4..1 of l
// (i.e. (l >> 1) & 15, read MSB-first: bit 4 -> slot bit 3, ..., bit 1 -> slot bit 0).
__device__ __forceinline__ float warp_sum16_scatter(float (&y)[16], int lane) {
#pragma unroll
  for (int h = 8, o = 16; h >= 1; h >>= 1, o >>= 1) {
    const bool up = (lane & o) != 0;  // this lane keeps the upper half
#pragma unroll
    for (int k = 0; k < h; ++k) {
      const float give = up ? y[k] : y[k + h];
      const float keep = up ? y[k + h] : y[k];
      y[k] = keep + __shfl_xor_sync(0xffffffffu, give, o);
    }
  }
  return y[0] + __shfl_xor_sync(0xffffffffu, y[0], 1);
}

// grid (ceil(S / 64), B*H), 256 threads (8 warps); a warp corrects one row at a time:
// y = x P' + c' (lane l holds columns l, l+32, ...; the factors sit in shared memory
// as [k][d] so the 32 lanes read 32 consecutive words), x += y V_rᵀ. Ranks above 16
// are taken 16 at a time.
template <int D>
__global__ void __launch_bounds__(256) repair_apply_kernel(float* __restrict__ out, int S, int rank,
                                                           const float* __restrict__ pp,
                                                           const float* __restrict__ cc,
                                                           const float* __restrict__ vr) {
  constexpr int EPL = D / 32;
  extern __shared__ float sm_apply[];
  const int64_t bh = blockIdx.y;
  const int nk = (rank + 15) & ~15;    // rank rounded up to 16: zero factors past it
  float* sP = sm_apply;                // [nk][D]
  float* sV = sm_apply + nk * D;       // [nk][D]
  float* sc = sV + nk * D;             // [nk]
  for (int e = threadIdx.x; e < nk * D; e += blockDim.x) {
    const int k = e / D, d = e % D;
    const bool in = k < rank;
    sP[e] = in ? pp[(bh * D + d) * rank + k] : 0.f;
    sV[e] = in ? vr[(bh * D + d) * rank + k] : 0.f;
  }
  for (int e = threadIdx.x; e < nk; e += blockDim.x) sc[e] = e < rank ? cc[bh * rank + e] : 0.f;
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int slot = (lane >> 1) & 15;   // the value this lane holds after warp_sum16_scatter
  const int r0 = blockIdx.x * 64;
  for (int r = r0 + warp; r < min(S, r0 + 64); r += 8) {
    float* row = out + (bh * S + r) * D + lane;
    float x[EPL], acc[EPL];
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      x[e] = row[32 * e];
      acc[e] = x[e];
    }
    for (int k0 = 0; k0 < nk; k0 += 16) {
      float y[16];
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        float t = 0.f;
#pragma unroll
        for (int e = 0; e < EPL; ++e) t = fmaf(x[e], sP[(k0 + k) * D + lane + 32 * e], t);
        y[k] = t;
      }
      const float mine = warp_sum16_scatter(y, lane) + sc[k0 + slot];
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        // the lanes 2k' .. holding slot k: lane l has slot (l >> 1) & 15, so lane 2k has k
        const float yk = __shfl_sync(0xffffffffu, mine, 2 * k);
#pragma unroll
        for (int e = 0; e < EPL; ++e) acc[e] = fmaf(yk, sV[(k0 + k) * D + lane + 32 * e], acc[e]);
      }
    }
#pragma unroll
    for (int e = 0; e < EPL; ++e) row[32 * e] = acc[e];
  }
}

constexpr int kApplyRows = 128;
constexpr int kApplyThreads = 64;  // two rows per thread
constexpr int apply16_smem_bytes(int D) {
  return static_cast<int>(sizeof(float)) * (2 * D * 16 + kApplyRows * (D + 4) + 16);
}

// rank <= 16: tiles of 128 rows staged through shared memory, so that every global
// access is a coalesced 16-byte vector (HBM traffic: one read and one write of out);
// then two rows per thread (rows t and t + 64): y = x P' + c' (each factor row d is a
// broadcast read of 16 floats, all lanes the same address, used for both rows),
// x += y V_rᵀ (V_rᵀ row k broadcast likewise), pairs of outputs per packed f32x2 FMA.
// Rows are padded to D + 4 floats, so the eight rows of a quarter-warp fall on distinct
// 16-byte bank groups. grid (ceil(S / 128), B*H), 64 threads; factors as P'[d][k],
// V_rᵀ[k][d], zero past `rank`.
template <int D>
__global__ void __launch_bounds__(kApplyThreads) repair_apply16_kernel(float* __restrict__ out, int S,
                                                                      int rank,
                                                                      const float* __restrict__ pp,
                                                                      const float* __restrict__ cc,
                                                                      const float* __restrict__ vr) {
  constexpr int TR = kApplyRows, LD = D + 4, V4 = D / 4, NT = kApplyThreads;
  extern __shared__ __align__(16) float apply_smem[];  // apply16_smem_bytes(D)
  float(*sP)[16] = reinterpret_cast<float(*)[16]>(apply_smem);
  float(*sVt)[D] = reinterpret_cast<float(*)[D]>(apply_smem + D * 16);
  float* xs = apply_smem + 2 * D * 16;
  float* sc = xs + TR * LD;
  const int64_t bh = blockIdx.y;
  for (int e = threadIdx.x; e < D * 16; e += NT) {
    const int d = e / 16, k = e % 16;
    const bool in = k < rank;
    sP[d][k] = in ? pp[(bh * D + d) * rank + k] : 0.f;
    sVt[k][d] = in ? vr[(bh * D + d) * rank + k] : 0.f;
  }
  if (threadIdx.x < 16) sc[threadIdx.x] = threadIdx.x < rank ? cc[bh * rank + threadIdx.x] : 0.f;
  const int r0 = blockIdx.x * TR;
  const int nr = min(TR, S - r0);
  const float4* src = reinterpret_cast<const float4*>(out + (bh * S + r0) * D);
  // fixed trip count: each thread's TR * V4 / NT loads are in flight together
#pragma unroll
  for (int i = 0; i < TR * V4 / NT; ++i) {
    const int e = threadIdx.x + NT * i;
    if (e < nr * V4) *reinterpret_cast<float4*>(&xs[(e / V4) * LD + 4 * (e % V4)]) = __ldg(src + e);
  }
  __syncthreads();
  // rows a = t and b = t + 64 (rows past nr hold stale values and are not written back)
  float* xa = &xs[threadIdx.x * LD];
  float* xb = &xs[(threadIdx.x + NT) * LD];
  float ya[16], yb[16];
#pragma unroll
  for (int k = 0; k < 16; ++k) ya[k] = yb[k] = sc[k];
#pragma unroll 2
  for (int d4 = 0; d4 < V4; ++d4) {
    const float4 a4 = *reinterpret_cast<const float4*>(xa + 4 * d4);
    const float4 b4 = *reinterpret_cast<const float4*>(xb + 4 * d4);
    const float av[4] = {a4.x, a4.y, a4.z, a4.w}, bv[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
#pragma unroll
      for (int k4 = 0; k4 < 4; ++k4) {
        const float4 p = *reinterpret_cast<const float4*>(&sP[4 * d4 + j][4 * k4]);
        fma2(ya[4 * k4], ya[4 * k4 + 1], av[j], av[j], p.x, p.y, ya[4 * k4], ya[4 * k4 + 1]);
        fma2(ya[4 * k4 + 2], ya[4 * k4 + 3], av[j], av[j], p.z, p.w, ya[4 * k4 + 2], ya[4 * k4 + 3]);
        fma2(yb[4 * k4], yb[4 * k4 + 1], bv[j], bv[j], p.x, p.y, yb[4 * k4], yb[4 * k4 + 1]);
        fma2(yb[4 * k4 + 2], yb[4 * k4 + 3], bv[j], bv[j], p.z, p.w, yb[4 * k4 + 2], yb[4 * k4 + 3]);
      }
    }
  }
#pragma unroll 2
  for (int c4 = 0; c4 < V4; ++c4) {
    float4 a4 = *reinterpret_cast<const float4*>(xa + 4 * c4);
    float4 b4 = *reinterpret_cast<const float4*>(xb + 4 * c4);
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const float4 v = *reinterpret_cast<const float4*>(&sVt[k][4 * c4]);
      fma2(a4.x, a4.y, ya[k], ya[k], v.x, v.y, a4.x, a4.y);
      fma2(a4.z, a4.w, ya[k], ya[k], v.z, v.w, a4.z, a4.w);
      fma2(b4.x, b4.y, yb[k], yb[k], v.x, v.y, b4.x, b4.y);
      fma2(b4.z, b4.w, yb[k], yb[k], v.z, v.w, b4.z, b4.w);
    }
    *reinterpret_cast<float4*>(xa + 4 * c4) = a4;
    *reinterpret_cast<float4*>(xb + 4 * c4) = b4;
  }
  __syncthreads();
  float4* dst = reinterpret_cast<float4*>(out + (bh * S + r0) * D);
#pragma unroll
  for (int i = 0; i < TR * V4 / NT; ++i) {
    const int e = threadIdx.x + NT * i;
    if (e < nr * V4) dst[e] = *reinterpret_cast<const float4*>(&xs[(e / V4) * LD + 4 * (e % V4)]);
  }
}

namespace {
struct RepairLayout {
  float *psum, *psq, *zt, *rr, *rv, *vr, *pp, *cc;
  size_t bytes;
};
RepairLayout carve_repair(int BH, int D, int M, int rank, void* ws) {
  Carver cv(ws);
  RepairLayout L{};
  L.psum = cv.take<float>(static_cast<size_t>(BH) * kStatSplit * D);
  L.psq = cv.take<float>(static_cast<size_t>(BH) * kStatSplit * D);
  L.zt = cv.take<float>(static_cast<size_t>(BH) * M * (D + 3));  // row stride ldz of the fit plan
  L.rr = cv.take<float>(static_cast<size_t>(BH) * M * (D + 1));
  L.rv = cv.take<float>(static_cast<size_t>(BH) * M * rank);
  L.vr = cv.take<float>(static_cast<size_t>(BH) * D * rank);
  L.pp = cv.take<float>(static_cast<size_t>(BH) * D * rank);
  L.cc = cv.take<float>(static_cast<size_t>(BH) * rank);
  L.bytes = align_up(cv.used, 256);
  return L;
}
}  // namespace

}  // namespace bsa

namespace bsa {
// Argument checks of the repair, shared by the workspace and the allocation-free entry
// points so that both return the same status for the same arguments.
int validate_repair_args(const float* out, const float* o_probe, const int32_t* probe_idx,
                         const float* weights, int B, int H, int S, int D, int M, int rank,
                         float lam) {
  if (!out || !o_probe || !probe_idx || !weights) return fail(BSA_ERR_INVALID_ARG, "null pointer");
  if (B <= 0 || H <= 0 || S <= 0 || M <= 0) return fail(BSA_ERR_INVALID_ARG, "bad sizes");
  if (D != 64 && D != 128) return fail(BSA_ERR_UNSUPPORTED, "head dim %d", D);
  if (M > 1024) return fail(BSA_ERR_UNSUPPORTED, "M %d > 1024", M);
  if (rank < 1 || rank > D) return fail(BSA_ERR_INVALID_ARG, "rank %d outside [1, D]", rank);
  if (!(lam >= 0.f)) return fail(BSA_ERR_INVALID_ARG, "lambda must be >= 0");
  return BSA_OK;
}
}  // namespace bsa

extern "C" size_t bsa_repair_workspace_bytes(int B, int H, int S, int D, int M) {
  if (B <= 0 || H <= 0 || S <= 0 || (D != 64 && D != 128) || M <= 0 || M > 1024) return 0;
  return bsa::carve_repair(B * H, D, M, D, nullptr).bytes;
}

extern "C" int bsa_probe_residual_correction(float* out, const float* o_probe,
                                             const int32_t* probe_idx, const float* weights,
                                             int per_head, int B, int H, int S, int D, int M,
                                             int rank, float lam, void* workspace,
                                             size_t workspace_bytes, void* stream) {
  using namespace bsa;
  cudaStream_t st = as_stream(stream);
  int rc = validate_repair_args(out, o_probe, probe_idx, weights, B, H, S, D, M, rank, lam);
  if (rc) return rc;
  const int BH = B * H;
  RepairLayout L = carve_repair(BH, D, M, rank, workspace);
  if (!workspace || workspace_bytes < L.bytes)
    return fail(BSA_ERR_WORKSPACE, "workspace %zu < %zu bytes", workspace_bytes, L.bytes);
  column_stats_kernel<<<dim3(kStatSplit, BH), 256, 0, st>>>(out, S, D, L.psum, L.psq);
  count_launch();
  if ((rc = check_cuda(cudaGetLastError(), "column_stats_kernel"))) return rc;
  FitArgs fa{out, o_probe, probe_idx, weights, per_head, S, D, M, rank, lam, L.psum, L.psq,
             L.zt,  L.rr,    L.rv,      L.vr,    L.pp,     L.cc};
  const size_t big = fit_plan(D, M, rank).floats * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(repair_fit_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(big));
  if (e != cudaSuccess) return check_cuda(e, "cudaFuncSetAttribute(repair_fit)");
  repair_fit_kernel<<<BH, kFitThreads, big, st>>>(fa);
  count_launch();
  if ((rc = check_cuda(cudaGetLastError(), "repair_fit_kernel"))) return rc;
  if (rank <= 16) {
    auto ap16 = D == 64 ? repair_apply16_kernel<64> : repair_apply16_kernel<128>;
    const int smem16 = apply16_smem_bytes(D);
    e = cudaFuncSetAttribute(ap16, cudaFuncAttributeMaxDynamicSharedMemorySize, smem16);
    if (e != cudaSuccess) return check_cuda(e, "cudaFuncSetAttribute(repair_apply16)");
    ap16<<<dim3((S + kApplyRows - 1) / kApplyRows, BH), kApplyThreads, smem16, st>>>(out, S, rank,
                                                                                    L.pp, L.cc, L.vr);
    count_launch();
    return check_cuda(cudaGetLastError(), "repair_apply16_kernel");
  }
  const int nk = (rank + 15) & ~15;
  const int smem = (2 * D * nk + nk) * static_cast<int>(sizeof(float));
  auto ap = D == 64 ? repair_apply_kernel<64> : repair_apply_kernel<128>;
  if (smem > 48 * 1024) {
    e = cudaFuncSetAttribute(ap, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return check_cuda(e, "cudaFuncSetAttribute(repair_apply)");
  }
  ap<<<dim3((S + 63) / 64, BH), 256, smem, st>>>(out, S, rank, L.pp, L.cc, L.vr);
  count_launch();
  return check_cuda(cudaGetLastError(), "repair_apply_kernel");
}
