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
//   V_r = top-r eigenvectors of Rᵀ W R                         cyclic Jacobi (circle-method
//                                                              pair order) on the smaller
//                                                              of Rᵀ W R and W½ R Rᵀ W½
//   out += Zt Bc V_r V_rᵀ = (X P' + c') V_rᵀ,  P' = diag(1/sigma) Bc[:D] V_r,
//          c' = (Bc[D] - Σ_i mu_i/sigma_i Bc[i]) V_r      (rank-r update, one HBM pass)
#include <cmath>

#include "common.cuh"
#include "ptx.cuh"

namespace bsa {

constexpr int kStatSplit = 32;
constexpr int kFitThreads = 1024;

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
  float* zt;   // [BH][M][D+1]
  float* rr;   // [BH][M][D]
  float* bc;   // [BH][D+1][D]
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

// Circle-method round robin: round r of n (even) players pairs r with n-1 and
// (r+i) with (r-i) (mod n-1) for i = 1 .. n/2-1; every pair meets once per n-1 rounds.
__device__ __forceinline__ void round_pair(int n, int r, int i, int& p, int& q) {
  if (i == 0) {
    p = r;
    q = n - 1;
  } else {
    p = (r + i) % (n - 1);
    q = (r - i + (n - 1)) % (n - 1);
  }
  if (p > q) {
    const int t = p;
    p = q;
    q = t;
  }
}

// One CTA (1024 threads) per (b, h): statistics, normal equations, Cholesky solve,
// residual subspace, and the folded rank-r factors P', c' for the apply pass.
__global__ void __launch_bounds__(kFitThreads, 1) repair_fit_kernel(const FitArgs a) {
  extern __shared__ float big[];
  __shared__ float mu[128], isg[128], red[32];
  __shared__ float wv[1024];
  __shared__ int sel[128];
  __shared__ float csn[64][2];
  __shared__ int cpq[64][2];
  const int tid = threadIdx.x, nt = blockDim.x;
  const int64_t bh = blockIdx.x;
  const int S = a.S, D = a.D, M = a.M, n1 = D + 1;
  const float* X = a.out + bh * S * D;
  const int32_t* idx = a.per_head ? a.probe_idx + bh * M : a.probe_idx;
  const float* w = a.per_head ? a.weights + bh * M : a.weights;
  float* zt = a.zt + bh * M * n1;
  float* rr = a.rr + bh * M * D;

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
  for (int m = tid; m < M; m += nt) wv[m] = w[m];
  __syncthreads();
  // 2. standardised probe rows and residuals
  for (int e = tid; e < M * D; e += nt) {
    const int m = e / D, d = e % D;
    int row = idx[m];
    row = row < 0 ? 0 : (row >= S ? S - 1 : row);
    const float x = X[static_cast<int64_t>(row) * D + d];
    zt[m * n1 + d] = (x - mu[d]) * isg[d];
    rr[m * D + d] = a.o_probe[(bh * M + m) * D + d] - x;
  }
  for (int m = tid; m < M; m += nt) zt[m * n1 + D] = 1.f;
  __syncthreads();
  // 3. normal equations: A = Ztᵀ W Zt + lam·I' (intercept unpenalised), Y = Ztᵀ W R
  float* A = big;            // n1 x n1
  float* Y = big + n1 * n1;  // n1 x D
  for (int e = tid; e < n1 * n1; e += nt) {
    const int i = e / n1, j = e % n1;
    if (j > i) continue;
    float acc = 0.f;
    for (int m = 0; m < M; ++m) acc = fmaf(wv[m] * zt[m * n1 + i], zt[m * n1 + j], acc);
    if (i == j && i < D) acc += a.lam;
    A[i * n1 + j] = acc;
    A[j * n1 + i] = acc;
  }
  for (int e = tid; e < n1 * D; e += nt) {
    const int i = e / D, c = e % D;
    float acc = 0.f;
    for (int m = 0; m < M; ++m) acc = fmaf(wv[m] * zt[m * n1 + i], rr[m * D + c], acc);
    Y[i * D + c] = acc;
  }
  __syncthreads();
  // 4. Cholesky A = L Lᵀ (lower triangle, in place)
  for (int k = 0; k < n1; ++k) {
    if (tid == 0) A[k * n1 + k] = sqrtf(fmaxf(A[k * n1 + k], 1e-30f));
    __syncthreads();
    const float piv = A[k * n1 + k];
    for (int i = k + 1 + tid; i < n1; i += nt) A[i * n1 + k] /= piv;
    __syncthreads();
    const int rem = n1 - k - 1;
    for (int e = tid; e < rem * rem; e += nt) {
      const int i = k + 1 + e / rem, j = k + 1 + e % rem;
      if (j <= i) A[i * n1 + j] -= A[i * n1 + k] * A[j * n1 + k];
    }
    __syncthreads();
  }
  // 5. solve L Lᵀ Bc = Y, one right-hand side column per thread
  if (tid < D) {
    const int c = tid;
    for (int i = 0; i < n1; ++i) {
      float acc = Y[i * D + c];
      for (int j = 0; j < i; ++j) acc -= A[i * n1 + j] * Y[j * D + c];
      Y[i * D + c] = acc / A[i * n1 + i];
    }
    for (int i = n1 - 1; i >= 0; --i) {
      float acc = Y[i * D + c];
      for (int j = i + 1; j < n1; ++j) acc -= A[j * n1 + i] * Y[j * D + c];
      Y[i * D + c] = acc / A[i * n1 + i];
    }
  }
  __syncthreads();
  float* bc = a.bc + bh * n1 * D;
  for (int e = tid; e < n1 * D; e += nt) bc[e] = Y[e];
  __syncthreads();

  // 6. Gram matrix of the weighted residuals: n x n with n = min(M, D)
  const bool small = M < D;
  const int n = small ? M : D;
  const int ne = n + (n & 1);
  const int ld = ne + 1;      // padded row stride: column sweeps hit distinct banks
  float* G = big;             // ne x ne in ld-strided rows (padding row/col zero)
  float* V = big + ne * ld;   // ne x ne in ld-strided rows
  for (int e = tid; e < ne * ne; e += nt) {
    const int i = e / ne, j = e % ne;
    float acc = 0.f;
    if (i < n && j < n) {
      if (small) {
        const float s = sqrtf(wv[i] * wv[j]);
        for (int d = 0; d < D; ++d) acc = fmaf(rr[i * D + d], rr[j * D + d], acc);
        acc *= s;
      } else {
        for (int m = 0; m < M; ++m) acc = fmaf(wv[m] * rr[m * D + i], rr[m * D + j], acc);
      }
    }
    G[i * ld + j] = acc;
    V[i * ld + j] = (i == j) ? 1.f : 0.f;
  }
  __syncthreads();
  // 7. cyclic Jacobi sweeps, until the off-diagonal mass is below 1e-12 of the total
  //    (about the float32 resolution of the squared entries)
  for (int sweep = 0; sweep < 20; ++sweep) {
    float off = 0.f, tot = 0.f;
    for (int e = tid; e < ne * ne; e += nt) {
      const float g = G[(e / ne) * ld + e % ne];
      tot += g * g;
      if (e / ne != e % ne) off += g * g;
    }
    off = block_sum(off, red);
    tot = block_sum(tot, red);
    if (off <= 1e-12f * tot || tot == 0.f) break;
    for (int r = 0; r < ne - 1; ++r) {
      if (tid < ne / 2) {
        int p, q;
        round_pair(ne, r, tid, p, q);
        float c = 1.f, s = 0.f;
        if (q < n) {
          const float apq = G[p * ld + q];
          if (apq != 0.f) {
            const float tau = (G[q * ld + q] - G[p * ld + p]) / (2.f * apq);
            const float t = (tau >= 0.f ? 1.f : -1.f) / (fabsf(tau) + sqrtf(1.f + tau * tau));
            c = 1.f / sqrtf(1.f + t * t);
            s = t * c;
          }
        }
        csn[tid][0] = c;
        csn[tid][1] = s;
        cpq[tid][0] = p;
        cpq[tid][1] = q;
      }
      __syncthreads();
      for (int e = tid; e < (ne / 2) * ne; e += nt) {  // rows p, q  <- Jᵀ G
        const int i = e / ne, j = e % ne;
        const int p = cpq[i][0], q = cpq[i][1];
        const float c = csn[i][0], s = csn[i][1];
        const float gp = G[p * ld + j], gq = G[q * ld + j];
        G[p * ld + j] = c * gp - s * gq;
        G[q * ld + j] = s * gp + c * gq;
      }
      __syncthreads();
      for (int e = tid; e < (ne / 2) * ne; e += nt) {  // columns p, q  <- G J, V J
        const int i = e / ne, j = e % ne;
        const int p = cpq[i][0], q = cpq[i][1];
        const float c = csn[i][0], s = csn[i][1];
        const float gp = G[j * ld + p], gq = G[j * ld + q];
        G[j * ld + p] = c * gp - s * gq;
        G[j * ld + q] = s * gp + c * gq;
        const float vp = V[j * ld + p], vq = V[j * ld + q];
        V[j * ld + p] = c * vp - s * vq;
        V[j * ld + q] = s * vp + c * vq;
      }
      __syncthreads();
    }
  }
  // 8. the `rank` largest eigenvalues
  const int rk = a.rank;
  if (tid == 0) {
    for (int k = 0; k < rk; ++k) {
      int best = -1;
      float bv = -INFINITY;
      for (int i = 0; i < n; ++i) {
        bool used = false;
        for (int j = 0; j < k; ++j) used |= sel[j] == i;
        if (!used && G[i * ld + i] > bv) {
          bv = G[i * ld + i];
          best = i;
        }
      }
      sel[k] = best;  // -1 when rank exceeds n: that direction is left out
    }
  }
  __syncthreads();
  float* vr = a.vr + bh * D * rk;
  const float lmax = n > 0 && sel[0] >= 0 ? G[sel[0] * ld + sel[0]] : 0.f;
  for (int e = tid; e < D * rk; e += nt) {
    const int d = e / rk, k = e % rk;
    const int i = sel[k];
    float val = 0.f;
    if (i >= 0) {
      if (!small) {
        val = V[d * ld + i];
      } else {
        const float lam_i = G[i * ld + i];
        if (lam_i > 1e-12f * lmax && lam_i > 0.f) {
          float acc = 0.f;
          for (int m = 0; m < M; ++m) acc = fmaf(sqrtf(wv[m]) * rr[m * D + d], V[m * ld + i], acc);
          val = acc / sqrtf(lam_i);
        }
      }
    }
    vr[d * rk + k] = val;
  }
  __syncthreads();
  // 9. folded factors: P' = diag(1/sigma) Bc[:D] V_r, c' = (Bc[D] - Σ mu/sigma Bc) V_r
  float* c0 = big;  // D (reuses the Gram region, no longer needed)
  __syncthreads();
  if (tid < D) {
    float acc = bc[D * D + tid];
    for (int i = 0; i < D; ++i) acc -= mu[i] * isg[i] * bc[i * D + tid];
    c0[tid] = acc;
  }
  __syncthreads();
  float* pp = a.pp + bh * D * rk;
  for (int e = tid; e < D * rk; e += nt) {
    const int d = e / rk, k = e % rk;
    float acc = 0.f;
    for (int c = 0; c < D; ++c) acc = fmaf(bc[d * D + c], vr[c * rk + k], acc);
    pp[d * rk + k] = acc * isg[d];
  }
  if (tid < rk) {
    float acc = 0.f;
    for (int c = 0; c < D; ++c) acc = fmaf(c0[c], vr[c * rk + tid], acc);
    a.cc[bh * rk + tid] = acc;
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

namespace {
struct RepairLayout {
  float *psum, *psq, *zt, *rr, *bc, *vr, *pp, *cc;
  size_t bytes;
};
RepairLayout carve_repair(int BH, int D, int M, int rank, void* ws) {
  Carver cv(ws);
  RepairLayout L{};
  L.psum = cv.take<float>(static_cast<size_t>(BH) * kStatSplit * D);
  L.psq = cv.take<float>(static_cast<size_t>(BH) * kStatSplit * D);
  L.zt = cv.take<float>(static_cast<size_t>(BH) * M * (D + 1));
  L.rr = cv.take<float>(static_cast<size_t>(BH) * M * D);
  L.bc = cv.take<float>(static_cast<size_t>(BH) * (D + 1) * D);
  L.vr = cv.take<float>(static_cast<size_t>(BH) * D * rank);
  L.pp = cv.take<float>(static_cast<size_t>(BH) * D * rank);
  L.cc = cv.take<float>(static_cast<size_t>(BH) * rank);
  L.bytes = align_up(cv.used, 256);
  return L;
}
}  // namespace

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
  if (!out || !o_probe || !probe_idx || !weights) return fail(BSA_ERR_INVALID_ARG, "null pointer");
  if (B <= 0 || H <= 0 || S <= 0 || M <= 0) return fail(BSA_ERR_INVALID_ARG, "bad sizes");
  if (D != 64 && D != 128) return fail(BSA_ERR_UNSUPPORTED, "head dim %d", D);
  if (M > 1024) return fail(BSA_ERR_UNSUPPORTED, "M %d > 1024", M);
  if (rank < 1 || rank > D) return fail(BSA_ERR_INVALID_ARG, "rank %d outside [1, D]", rank);
  if (!(lam >= 0.f)) return fail(BSA_ERR_INVALID_ARG, "lambda must be >= 0");
  const int BH = B * H;
  RepairLayout L = carve_repair(BH, D, M, rank, workspace);
  if (!workspace || workspace_bytes < L.bytes)
    return fail(BSA_ERR_WORKSPACE, "workspace %zu < %zu bytes", workspace_bytes, L.bytes);
  int rc;
  column_stats_kernel<<<dim3(kStatSplit, BH), 256, 0, st>>>(out, S, D, L.psum, L.psq);
  count_launch();
  if ((rc = check_cuda(cudaGetLastError(), "column_stats_kernel"))) return rc;
  FitArgs fa{out, o_probe, probe_idx, weights, per_head, S, D, M, rank, lam, L.psum, L.psq,
             L.zt,  L.rr,    L.bc,      L.vr,    L.pp,     L.cc};
  const int n = M < D ? M : D;
  const int ne = n + (n & 1);
  const size_t big = std::max(static_cast<size_t>(D + 1) * (D + 1) + static_cast<size_t>(D + 1) * D,
                              2 * static_cast<size_t>(ne) * (ne + 1)) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(repair_fit_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(big));
  if (e != cudaSuccess) return check_cuda(e, "cudaFuncSetAttribute(repair_fit)");
  repair_fit_kernel<<<BH, kFitThreads, big, st>>>(fa);
  count_launch();
  if ((rc = check_cuda(cudaGetLastError(), "repair_fit_kernel"))) return rc;
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
