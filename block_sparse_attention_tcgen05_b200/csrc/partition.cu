// SparsePR Response-Coupled Partitioning: query and key clusters from the current
// call's responses.
//
// Source: "Partition the Support, Reconstruct the Residual" (paper summary): queries
// are sampled from the call and keys grouped by their pre-softmax response; key-group
// centroids define query coordinates, so queries with a similar response direction
// share a route; one asymmetric pass; feature ranks rK = 48 and rQ = 64; K/V partitions
// and routes shared by a KV head's query heads; an online k-means.
//
// Per (batch, KV head g) with G = Hq / Hkv query heads:
//   samples         rK query rows: sample s = token floor((s + 1/2) Sq / rK) of query
//                   head g G + (s mod G)
//   key features    f_j = scale * Q_s k_j                                 (Sk x rK)
//   key groups      k-means of the key features into Ck clusters
//   query coords    x_i = (scale * q_{h,i} . kbar_{c_t}) over the rQ' = min(rQ, Ck)
//                   groups c_t = floor((t + 1/2) Ck / rQ') and the G heads, divided by
//                   its norm                                              (Sq x rQ' G)
//   query groups    k-means of the query coordinates into Cq clusters
// k-means (Lloyd): centroids start at rows floor((c + 1/2) N / C); each round assigns
// rows to the nearest centroid (squared distance, ties to the lower index) and moves
// each centroid to its rows' mean (an empty cluster keeps its centroid); after `iters`
// rounds a last assignment gives the labels. Every sum runs in a fixed order, so a
// call is deterministic.
#include <cuda_bf16.h>

#include <cmath>

#include "common.cuh"
#include "ptx.cuh"

namespace bsa {

constexpr int kRcpMaxF = 256;       // feature dimension limit (rK, rQ' G)
constexpr int kRcpRows = 128;       // rows per assignment CTA
constexpr int kRcpCentChunk = 32;   // centroids per shared-memory chunk

__device__ __forceinline__ float rcp_f(float x) { return x; }
__device__ __forceinline__ float rcp_f(__nv_bfloat16 x) { return __bfloat162float(x); }

// grid (ceil(Sk / 64), Hkv, B), 256 threads: feat[b,g,j,s] = scale * q[b, h_s, t_s] . k[b,g,j].
template <typename T, int D>
__global__ void __launch_bounds__(256) rcp_key_features_kernel(const T* __restrict__ q,
                                                               const T* __restrict__ k, int Hq,
                                                               int Hkv, int Sq, int Sk, int rk,
                                                               float scale,
                                                               float* __restrict__ feat) {
  extern __shared__ float sm_rcp[];
  float* qs = sm_rcp;              // rk x (D + 1): odd row stride, the lanes' samples on distinct banks
  float* ks = qs + rk * (D + 1);   // 64 x (D + 1)
  const int g = blockIdx.y, b = blockIdx.z, G = Hq / Hkv;
  const int j0 = blockIdx.x * 64;
  for (int e = threadIdx.x; e < rk * D; e += 256) {
    const int s = e / D, d = e % D;
    const int tok = static_cast<int>((static_cast<int64_t>(2 * s + 1) * Sq) / (2 * rk));
    const int h = g * G + s % G;
    qs[s * (D + 1) + d] = rcp_f(q[((static_cast<int64_t>(b) * Hq + h) * Sq + tok) * D + d]);
  }
  const int64_t kb = (static_cast<int64_t>(b) * Hkv + g) * Sk;
  for (int e = threadIdx.x; e < 64 * D; e += 256) {
    const int j = e / D, d = e % D;
    ks[j * (D + 1) + d] = j0 + j < Sk ? rcp_f(k[(kb + j0 + j) * D + d]) : 0.f;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < 64 * rk; e += 256) {
    const int j = e / rk, s = e % rk;
    if (j0 + j >= Sk) continue;
    float acc = 0.f;
#pragma unroll 8
    for (int d = 0; d < D; ++d) acc = fmaf(qs[s * (D + 1) + d], ks[j * (D + 1) + d], acc);
    feat[(kb + j0 + j) * rk + s] = scale * acc;
  }
}

// grid (C, n_problems): cent[p, c, :] = x[p, floor((2c + 1) N / (2C)), :].
__global__ void kmeans_init_kernel(const float* __restrict__ x, int N, int F, int C,
                                   float* __restrict__ cent) {
  const int c = blockIdx.x;
  const int64_t p = blockIdx.y;
  const int row = static_cast<int>((static_cast<int64_t>(2 * c + 1) * N) / (2 * C));
  for (int f = threadIdx.x; f < F; f += blockDim.x)
    cent[(p * C + c) * F + f] = x[(p * N + row) * F + f];
}

// grid (ceil(N / 128), n_problems), 256 threads: the nearest of the C centroids for 128
// rows (squared distance summed in feature order, ties to the lower index). Rows are
// staged feature-major in shared memory, centroids 32 at a time as rows of F4 =
// ceil(F / 4) * 4 floats (zero padded, which adds exact zeros), read four features per
// broadcast load. Thread t takes row t % 128 against centroid quarter t / 128 of every
// chunk (warp-uniform, so every centroid read is a broadcast); the four quarters' bests
// are merged at the end.
constexpr int kRcpGroups = 4;
constexpr int kRcpThreads = kRcpGroups * kRcpRows;
__global__ void __launch_bounds__(kRcpThreads) kmeans_assign_kernel(const float* __restrict__ x,
                                                                    int N, int F, int C,
                                                                    const float* __restrict__ cent,
                                                                    int32_t* __restrict__ label) {
  extern __shared__ __align__(16) float sm_km[];
  constexpr int HC = kRcpCentChunk / kRcpGroups;   // centroids per group
  __shared__ float s_best[kRcpGroups][kRcpRows];
  __shared__ int s_bc[kRcpGroups][kRcpRows];
  const int F4 = (F + 3) / 4 * 4;
  float* xs = sm_km;                       // F4 x 128
  float* cs = xs + F4 * kRcpRows;          // 32 x F4
  const int64_t p = blockIdx.y;
  const int i0 = blockIdx.x * kRcpRows, tid = threadIdx.x;
  const int r = tid % kRcpRows, grp = tid / kRcpRows;
  for (int e = tid; e < kRcpRows * F4; e += kRcpThreads) {
    const int rr = e / F4, f = e % F4;
    xs[f * kRcpRows + rr] = (i0 + rr < N && f < F) ? x[(p * N + i0 + rr) * F + f] : 0.f;
  }
  float best = INFINITY;
  int bc = 0x7fffffff;
  for (int c0 = 0; c0 < C; c0 += kRcpCentChunk) {
    const int nc = min(kRcpCentChunk, C - c0);
    __syncthreads();
    for (int e = tid; e < kRcpCentChunk * F4; e += kRcpThreads) {
      const int c = e / F4, f = e % F4;
      cs[e] = (c < nc && f < F) ? cent[(p * C + c0 + c) * F + f] : 0.f;
    }
    __syncthreads();
    const float* ch = cs + grp * HC * F4;
    float d[HC];
#pragma unroll
    for (int c = 0; c < HC; ++c) d[c] = 0.f;
    for (int f = 0; f < F4; f += 4) {
      const float x0 = xs[f * kRcpRows + r], x1 = xs[(f + 1) * kRcpRows + r];
      const float x2 = xs[(f + 2) * kRcpRows + r], x3 = xs[(f + 3) * kRcpRows + r];
#pragma unroll
      for (int c = 0; c < HC; ++c) {
        const float4 cv = *reinterpret_cast<const float4*>(ch + c * F4 + f);
        float t = x0 - cv.x;
        d[c] = fmaf(t, t, d[c]);
        t = x1 - cv.y;
        d[c] = fmaf(t, t, d[c]);
        t = x2 - cv.z;
        d[c] = fmaf(t, t, d[c]);
        t = x3 - cv.w;
        d[c] = fmaf(t, t, d[c]);
      }
    }
#pragma unroll
    for (int c = 0; c < HC; ++c) {
      const int ci = grp * HC + c;
      if (ci < nc && d[c] < best) {
        best = d[c];
        bc = c0 + ci;
      }
    }
  }
  s_best[grp][r] = best;
  s_bc[grp][r] = bc;
  __syncthreads();
  if (grp == 0 && i0 + r < N) {
#pragma unroll
    for (int g = 1; g < kRcpGroups; ++g) {
      const float b1 = s_best[g][r];
      const int c1 = s_bc[g][r];
      if (b1 < best || (b1 == best && c1 < bc)) {
        best = b1;
        bc = c1;
      }
    }
    label[p * N + i0 + r] = bc == 0x7fffffff ? 0 : bc;  // no finite distance: cluster 0
  }
}

// grid (n_problems), 1024 threads: stable sort of each problem's labels into member
// lists (cluster c's rows, in index order, at slot[p][off[p][c] ..]).
__global__ void __launch_bounds__(1024) kmeans_members_kernel(const int32_t* __restrict__ label, int N,
                                                              int C, int32_t* slot, int32_t* count,
                                                              int32_t* off) {
  extern __shared__ int32_t sm_mem[];
  const int64_t p = blockIdx.x;
  LabelSortJob j{};
  j.labels = label + p * N;
  j.S = N;
  j.C = C;
  j.cluster_pad = 1;
  j.n_slots = N;
  j.slot_token = slot + p * N;
  j.count = count + p * C;
  j.off = off + p * (C + 1);
  label_sort_cta(j, sm_mem);
}

// grid (C, n_problems), 256 threads (thread f holds feature f): the mean of the rows of
// cluster c, summed in index order from its member list (eight rows in flight); an
// empty cluster keeps its centroid. With T != float the rows come from a (n_problems,
// N, F) source of that type (the key-space centroids).
template <typename T>
__global__ void __launch_bounds__(256) kmeans_update_kernel(const T* __restrict__ x, int N, int F,
                                                            int C, const int32_t* __restrict__ slot,
                                                            const int32_t* __restrict__ count,
                                                            const int32_t* __restrict__ off,
                                                            float* __restrict__ cent) {
  const int c = blockIdx.x, tid = threadIdx.x;
  const int64_t p = blockIdx.y;
  const int n = count[p * C + c];
  if (tid >= F || n == 0) return;
  const int32_t* mem = slot + p * N + off[p * (C + 1) + c];
  const T* xp = x + p * N * F + tid;
  float acc = 0.f;
  int m = 0;
  for (; m + 8 <= n; m += 8) {
    float v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) v[u] = rcp_f(xp[static_cast<int64_t>(mem[m + u]) * F]);
#pragma unroll
    for (int u = 0; u < 8; ++u) acc += v[u];
  }
  for (; m < n; ++m) acc += rcp_f(xp[static_cast<int64_t>(mem[m]) * F]);
  cent[(p * C + c) * F + tid] = acc / static_cast<float>(n);
}

// grid (ceil(Sq / 64), Hkv, B), 256 threads: x[b,g,i,:] = (scale q_{h,i} . kbar_{c_t})
// over t < rq and the G heads h of KV head g, divided by its norm. The group vectors sit
// transposed in shared memory (d-major, rq padded to rq4 = ceil(rq / 4) * 4 with zeros),
// so a thread takes four groups of one (row, head) per query element: one load of q and
// one broadcast-free float4 of the four groups' components per d.
template <typename T, int D>
__global__ void __launch_bounds__(256) rcp_query_coords_kernel(const T* __restrict__ q,
                                                               const float* __restrict__ kbar,
                                                               int Hq, int Hkv, int Sq, int Ck,
                                                               int rq, float scale,
                                                               float* __restrict__ xq) {
  extern __shared__ __align__(16) float sm_rq[];
  const int rq4 = (rq + 3) / 4 * 4, n4 = rq4 / 4;
  float* kcT = sm_rq;                // D x rq4
  float* out = kcT + D * rq4;        // 64 x F
  const int g = blockIdx.y, b = blockIdx.z, G = Hq / Hkv, F = rq * G;
  const int i0 = blockIdx.x * 64;
  const int64_t pg = static_cast<int64_t>(b) * Hkv + g;
  for (int e = threadIdx.x; e < D * rq4; e += 256) {
    const int d = e / rq4, t = e % rq4;
    const int c = static_cast<int>((static_cast<int64_t>(2 * t + 1) * Ck) / (2 * rq));
    kcT[e] = t < rq ? kbar[(pg * Ck + c) * D + d] : 0.f;
  }
  __syncthreads();
  for (int item = threadIdx.x; item < 64 * G * n4; item += 256) {
    const int g4 = item % n4, rest = item / n4;
    const int hh = rest % G, i = rest / G;
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
    if (i0 + i < Sq) {
      const T* qrow = q + ((static_cast<int64_t>(b) * Hq + g * G + hh) * Sq + i0 + i) * D;
#pragma unroll 8
      for (int d = 0; d < D; ++d) {
        const float qv = rcp_f(qrow[d]);
        const float4 k4 = *reinterpret_cast<const float4*>(kcT + d * rq4 + 4 * g4);
        a0 = fmaf(qv, k4.x, a0);
        a1 = fmaf(qv, k4.y, a1);
        a2 = fmaf(qv, k4.z, a2);
        a3 = fmaf(qv, k4.w, a3);
      }
    }
    const float av[4] = {a0, a1, a2, a3};
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int t = 4 * g4 + u;
      if (t < rq) out[i * F + hh * rq + t] = scale * av[u];
    }
  }
  __syncthreads();
  // one warp per row: norm, then the normalised row
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = warp; i < 64; i += 8) {
    if (i0 + i >= Sq) continue;
    float ss = 0.f;
    for (int f = lane; f < F; f += 32) ss = fmaf(out[i * F + f], out[i * F + f], ss);
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float inv = ss > 0.f ? 1.f / sqrtf(ss) : 0.f;
    for (int f = lane; f < F; f += 32) xq[(pg * Sq + i0 + i) * F + f] = out[i * F + f] * inv;
  }
}

namespace {
struct RcpLayout {
  float *fk, *xq, *kcent, *qcent, *kbar;
  int32_t *mslot, *mcount, *moff;  // k-means member lists: rows of each cluster, per problem
  size_t bytes;
};
RcpLayout carve_rcp(const bsa_shape& s, int Cq, int Ck, int rk, int rq, void* ws) {
  Carver cv(ws);
  RcpLayout L{};
  const size_t P = static_cast<size_t>(s.B) * s.Hkv;
  const int G = s.Hq / s.Hkv;
  const int rqe = rq < Ck ? rq : Ck;
  L.fk = cv.take<float>(P * s.Sk * rk);
  L.xq = cv.take<float>(P * s.Sq * rqe * G);
  L.kcent = cv.take<float>(P * Ck * rk);
  L.qcent = cv.take<float>(P * Cq * rqe * G);
  L.kbar = cv.take<float>(P * Ck * s.D);
  const size_t Nmax = s.Sq > s.Sk ? s.Sq : s.Sk;
  const size_t Cmax = Cq > Ck ? Cq : Ck;
  L.mslot = cv.take<int32_t>(P * Nmax);
  L.mcount = cv.take<int32_t>(P * Cmax);
  L.moff = cv.take<int32_t>(P * (Cmax + 1));
  L.bytes = align_up(cv.used, 256);
  return L;
}

int validate_rcp(const bsa_shape& s, int Cq, int Ck, int rk, int rq, int iters) {
  if (s.B <= 0 || s.Hq <= 0 || s.Hkv <= 0 || s.Sq <= 0 || s.Sk <= 0)
    return fail(BSA_ERR_INVALID_ARG, "non-positive shape");
  if (s.Hq % s.Hkv) return fail(BSA_ERR_INVALID_ARG, "Hq (%d) not a multiple of Hkv (%d)", s.Hq, s.Hkv);
  if (s.D != 64 && s.D != 128) return fail(BSA_ERR_UNSUPPORTED, "head dim %d not in {64,128}", s.D);
  if (s.dtype != BSA_BF16 && s.dtype != BSA_F32) return fail(BSA_ERR_UNSUPPORTED, "dtype %d", s.dtype);
  if (Cq < 1 || Ck < 1 || Cq > s.Sq || Ck > s.Sk)
    return fail(BSA_ERR_INVALID_ARG, "cluster counts Cq=%d Ck=%d outside [1, S]", Cq, Ck);
  if (Cq > 4096 || Ck > 4096) return fail(BSA_ERR_UNSUPPORTED, "cluster counts above 4096");
  if (rk < 1 || rq < 1 || iters < 0) return fail(BSA_ERR_INVALID_ARG, "rK, rQ >= 1, iters >= 0");
  const int G = s.Hq / s.Hkv;
  const int rqe = rq < Ck ? rq : Ck;
  if (rk > kRcpMaxF || rqe * G > kRcpMaxF)
    return fail(BSA_ERR_UNSUPPORTED, "feature dims rK=%d, rQ'*G=%d above %d", rk, rqe * G, kRcpMaxF);
  return BSA_OK;
}

// Lloyd iterations on (P, N, F) features: init, `iters` rounds, last assignment.
// Member lists of every cluster (stable sort of each problem's labels).
int run_members(const int32_t* label, int P, int N, int C, const RcpLayout& L, cudaStream_t st) {
  const int smem = label_sort_smem(C);
  cudaError_t e = cudaFuncSetAttribute(kmeans_members_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       smem > 48 * 1024 ? smem : 48 * 1024);
  if (e != cudaSuccess) return check_cuda(e, "cudaFuncSetAttribute(kmeans_members)");
  kmeans_members_kernel<<<P, 1024, smem, st>>>(label, N, C, L.mslot, L.mcount, L.moff);
  count_launch();
  return check_cuda(cudaGetLastError(), "kmeans_members_kernel");
}

int run_kmeans(const float* x, int P, int N, int F, int C, int iters, float* cent,
               int32_t* label, const RcpLayout& L, cudaStream_t st) {
  kmeans_init_kernel<<<dim3(C, P), 128, 0, st>>>(x, N, F, C, cent);
  count_launch();
  const int F4 = (F + 3) / 4 * 4;
  const int smem = (F4 * kRcpRows + kRcpCentChunk * F4) * 4;
  cudaError_t e = cudaFuncSetAttribute(kmeans_assign_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       smem > 48 * 1024 ? smem : 48 * 1024);
  if (e != cudaSuccess) return check_cuda(e, "cudaFuncSetAttribute(kmeans_assign)");
  for (int it = 0; it <= iters; ++it) {
    kmeans_assign_kernel<<<dim3((N + kRcpRows - 1) / kRcpRows, P), kRcpThreads, smem, st>>>(x, N, F, C,
                                                                                           cent, label);
    count_launch();
    if (it == iters) break;
    int rc = run_members(label, P, N, C, L, st);
    if (rc) return rc;
    kmeans_update_kernel<float><<<dim3(C, P), 256, 0, st>>>(x, N, F, C, L.mslot, L.mcount, L.moff, cent);
    count_launch();
  }
  return check_cuda(cudaGetLastError(), "k-means kernels");
}

template <typename T, int D>
int run_rcp(const void* qv, const void* kv, const bsa_shape& s, int Cq, int Ck, int rk, int rq,
            int iters, float scale, int32_t* q_labels, int32_t* k_labels, const RcpLayout& L,
            cudaStream_t st) {
  const T* q = static_cast<const T*>(qv);
  const T* k = static_cast<const T*>(kv);
  const int P = s.B * s.Hkv, G = s.Hq / s.Hkv;
  const int rqe = rq < Ck ? rq : Ck;
  int rc;
  {
    const int smem = (rk * (D + 1) + 64 * (D + 1)) * 4;
    cudaError_t e = cudaFuncSetAttribute(rcp_key_features_kernel<T, D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         smem > 48 * 1024 ? smem : 48 * 1024);
    if (e != cudaSuccess) return check_cuda(e, "cudaFuncSetAttribute(rcp_key_features)");
    rcp_key_features_kernel<T, D><<<dim3((s.Sk + 63) / 64, s.Hkv, s.B), 256, smem, st>>>(
        q, k, s.Hq, s.Hkv, s.Sq, s.Sk, rk, scale, L.fk);
    count_launch();
  }
  if ((rc = run_kmeans(L.fk, P, s.Sk, rk, Ck, iters, L.kcent, k_labels, L, st))) return rc;
  // key-group centroids in key space
  if ((rc = run_members(k_labels, P, s.Sk, Ck, L, st))) return rc;
  kmeans_update_kernel<T><<<dim3(Ck, P), 256, 0, st>>>(k, s.Sk, D, Ck, L.mslot, L.mcount, L.moff, L.kbar);
  count_launch();
  {
    const int smem = (D * ((rqe + 3) / 4 * 4) + 64 * rqe * G) * 4;
    cudaError_t e = cudaFuncSetAttribute(rcp_query_coords_kernel<T, D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         smem > 48 * 1024 ? smem : 48 * 1024);
    if (e != cudaSuccess) return check_cuda(e, "cudaFuncSetAttribute(rcp_query_coords)");
    rcp_query_coords_kernel<T, D><<<dim3((s.Sq + 63) / 64, s.Hkv, s.B), 256, smem, st>>>(
        q, L.kbar, s.Hq, s.Hkv, s.Sq, Ck, rqe, scale, L.xq);
    count_launch();
  }
  return run_kmeans(L.xq, P, s.Sq, rqe * G, Cq, iters, L.qcent, q_labels, L, st);
}
}  // namespace

}  // namespace bsa

extern "C" size_t bsa_partition_workspace_bytes(bsa_shape shape, int Cq, int Ck, int r_k, int r_q) {
  if (bsa::validate_rcp(shape, Cq, Ck, r_k, r_q, 0)) return 0;
  return bsa::carve_rcp(shape, Cq, Ck, r_k, r_q, nullptr).bytes;
}

extern "C" int bsa_response_coupled_partition(const void* q, const void* k, bsa_shape shape, int Cq,
                                              int Ck, int r_k, int r_q, int iters, float scale,
                                              int32_t* q_labels, int32_t* k_labels, void* workspace,
                                              size_t workspace_bytes, void* stream) {
  using namespace bsa;
  int rc = validate_rcp(shape, Cq, Ck, r_k, r_q, iters);
  if (rc) return rc;
  if (!q || !k || !q_labels || !k_labels) return fail(BSA_ERR_INVALID_ARG, "null pointer argument");
  RcpLayout L = carve_rcp(shape, Cq, Ck, r_k, r_q, workspace);
  if (!workspace || workspace_bytes < L.bytes)
    return fail(BSA_ERR_WORKSPACE, "workspace %zu bytes < required %zu", workspace_bytes, L.bytes);
  if (reinterpret_cast<uintptr_t>(workspace) % 256)
    return fail(BSA_ERR_INVALID_ARG, "workspace not 256-byte aligned");
  const float sc = scale > 0.f ? scale : 1.f / std::sqrt(static_cast<float>(shape.D));
  cudaStream_t st = as_stream(stream);
  if (shape.dtype == BSA_F32)
    return shape.D == 64 ? run_rcp<float, 64>(q, k, shape, Cq, Ck, r_k, r_q, iters, sc, q_labels,
                                              k_labels, L, st)
                         : run_rcp<float, 128>(q, k, shape, Cq, Ck, r_k, r_q, iters, sc, q_labels,
                                               k_labels, L, st);
  return shape.D == 64 ? run_rcp<__nv_bfloat16, 64>(q, k, shape, Cq, Ck, r_k, r_q, iters, sc,
                                                    q_labels, k_labels, L, st)
                       : run_rcp<__nv_bfloat16, 128>(q, k, shape, Cq, Ck, r_k, r_q, iters, sc,
                                                     q_labels, k_labels, L, st);
}
