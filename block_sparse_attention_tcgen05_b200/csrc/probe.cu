// SparsePR probe rows: selection and their exact dense attention.
//
// Sources: "Sparse-block compensation" (mlx-arsenal notes), §What mlx-arsenal ships
// (select_probe_rows: round-robin over query clusters, |G_a| / m_a weights), §Recipe
// (dense attention of q[:, :, probe_idx] over every key), §Deviations (middle-out
// member; weights normalised to sum 1); "Partition the Support, Reconstruct the
// Residual" (probes stratified across query groups, ordered by distance to the group
// centroid; M query rows evaluated exactly against all keys).
#include <cuda_bf16.h>

#include "common.cuh"
#include "ptx.cuh"

namespace bsa {

int run_label_sort(const int32_t* labels, int S, int C, int cluster_pad, int n_slots,
                   int32_t* slot_token, int32_t* slot_label, int32_t* count, int32_t* off,
                   int32_t* group_cluster, int32_t* group_valid, int n_groups, float* bias2,
                   int C_pad, uint32_t* nonempty, cudaStream_t st);
int centroid_compensated_attention(const void* q, const void* k, const void* v,
                                   const bsa_shape& s, const int32_t* q_labels, int Cq,
                                   const int32_t* k_labels, int Ck, const uint8_t* mask,
                                   int64_t mbs, int64_t mhs, float scale, int compensate,
                                   float* out, void* ws, size_t ws_bytes, cudaStream_t st,
                                   int prof_id, bool dense, bool reuse_plan);
size_t attention_workspace_bytes(const bsa_shape& s, int Cq, int Ck);

constexpr int kMaxCentroidCluster = 4096;
constexpr int kMaxProbes = 1024;

// k-th member (0-based) of a cluster of n rows in middle-out order: rank by distance
// of the member's position r to the centre (n-1)/2, the lower position first on ties.
__device__ __forceinline__ int middle_out(int n, int k) {
  if (n & 1) {
    const int c = (n - 1) / 2;
    return (k == 0) ? c : ((k & 1) ? c - (k + 1) / 2 : c + k / 2);
  }
  const int lo = n / 2 - 1, hi = n / 2;
  return (k & 1) ? hi + (k - 1) / 2 : lo - k / 2;
}

template <typename T>
__device__ __forceinline__ float to_f(T x);
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }
template <>
__device__ __forceinline__ float to_f<float>(float x) { return x; }

// epl consecutive elements of a row as fp32, read as one vector per lane (epl * sizeof(T)
// bytes: 4, 8 or 16; rows start on D * sizeof(T) and lanes on epl * sizeof(T) boundaries).
template <typename T>
__device__ __forceinline__ void load_lane(const T* p, int epl, float (&x)[4]);
template <>
__device__ __forceinline__ void load_lane<__nv_bfloat16>(const __nv_bfloat16* p, int epl, float (&x)[4]) {
  if (epl == 4) {
    const uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
    x[0] = a.x; x[1] = a.y; x[2] = b.x; x[3] = b.y;
  } else {
    const uint32_t u = __ldg(reinterpret_cast<const unsigned int*>(p));
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u));
    x[0] = a.x; x[1] = a.y; x[2] = x[3] = 0.f;
  }
}
template <>
__device__ __forceinline__ void load_lane<float>(const float* p, int epl, float (&x)[4]) {
  if (epl == 4) {
    const float4 u = __ldg(reinterpret_cast<const float4*>(p));
    x[0] = u.x; x[1] = u.y; x[2] = u.z; x[3] = u.w;
  } else {
    const float2 u = __ldg(reinterpret_cast<const float2*>(p));
    x[0] = u.x; x[1] = u.y; x[2] = x[3] = 0.f;
  }
}

// (distance, token) order: the smaller distance first, ties to the lower token index.
__device__ __forceinline__ bool dist_before(float da, int ta, float db, int tb) {
  return da < db || (da == db && ta < tb);
}

// grid (C, Hq, B), 256 threads: members of cluster a ordered by the Euclidean distance
// of q_i to the cluster's mean query (fp32), ties to the lower token index. When fewer
// probes than non-empty clusters are drawn (M < C'), the selection reads only each
// cluster's first member, so only that one (the arg-min) is written; otherwise the
// whole cluster is sorted.
template <typename T>
__global__ void __launch_bounds__(256) centroid_order_kernel(
    const T* __restrict__ q, int S, int D, int H, int C, int M, const int32_t* __restrict__ slot_token,
    const int32_t* __restrict__ count, const int32_t* __restrict__ off, int32_t* __restrict__ order) {
  __shared__ float mean[128];
  __shared__ float dist[kMaxCentroidCluster];
  __shared__ int tokn[kMaxCentroidCluster];
  __shared__ float part[8][128];
  __shared__ int red_n[8];
  __shared__ float red_d[8];
  __shared__ int red_t[8];
  const int a = blockIdx.x;
  const int64_t bh = static_cast<int64_t>(blockIdx.z) * H + blockIdx.y;
  const int n = count[a], start = off[a];
  if (n == 0) return;
  if (n > kMaxCentroidCluster) {
    // too large to order on chip: keep index order and report it
    for (int i = threadIdx.x; i < n; i += blockDim.x) order[bh * S + start + i] = slot_token[start + i];
    if (threadIdx.x == 0) report_device_error(kStatusUnsupported, 50);
    return;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  // non-empty clusters C' (the same count the selection makes)
  int ne = 0;
  for (int c = threadIdx.x; c < C; c += blockDim.x) ne += count[c] > 0;
  ne = __reduce_add_sync(0xffffffffu, ne);
  if (lane == 0) red_n[warp] = ne;
  // Rows are read warp by warp (lane l holds elements [l·D/32, (l+1)·D/32) of a row,
  // so a warp reads whole rows coalesced); warps stride over the members.
  const T* qb = q + bh * S * D;
  const int epl = D / 32;  // 2 or 4
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
  for (int i = warp; i < n; i += nw) {
    float x[4];
    load_lane<T>(qb + static_cast<int64_t>(slot_token[start + i]) * D + lane * epl, epl, x);
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[e] += x[e];
  }
#pragma unroll
  for (int e = 0; e < 4; ++e)
    if (e < epl) part[warp][lane * epl + e] = acc[e];
  __syncthreads();
  int cp = 0;
  for (int w = 0; w < nw; ++w) cp += red_n[w];
  const bool argmin_only = M < cp;
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    float t = 0.f;
    for (int w = 0; w < nw; ++w) t += part[w][d];
    mean[d] = t / static_cast<float>(n);
  }
  __syncthreads();
  int np = 1;
  while (np < n) np <<= 1;
  float best_d = INFINITY;
  int best_t = 0x7fffffff;
#pragma unroll 4
  for (int i = warp; i < np; i += nw) {
    if (i < n) {
      const int tok = slot_token[start + i];
      float x[4];
      load_lane<T>(qb + static_cast<int64_t>(tok) * D + lane * epl, epl, x);
      float sq = 0.f;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if (e < epl) {
          const float y = x[e] - mean[lane * epl + e];
          sq = fmaf(y, y, sq);
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
      const float dd = sqrtf(sq);
      if (argmin_only) {
        if (dist_before(dd, tok, best_d, best_t)) {
          best_d = dd;
          best_t = tok;
        }
      } else if (lane == 0) {
        dist[i] = dd;
        tokn[i] = tok;
      }
    } else if (!argmin_only && lane == 0) {
      dist[i] = INFINITY;
      tokn[i] = 0x7fffffff;
    }
  }
  if (argmin_only) {
    // every lane of a warp holds the warp's best; then the best of the warps
    if (lane == 0) {
      red_d[warp] = best_d;
      red_t[warp] = best_t;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      for (int w = 1; w < nw; ++w)
        if (dist_before(red_d[w], red_t[w], best_d, best_t)) {
          best_d = red_d[w];
          best_t = red_t[w];
        }
      order[bh * S + start] = best_t;
    }
    return;
  }
  __syncthreads();
  for (int k = 2; k <= np; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = threadIdx.x; i < np; i += blockDim.x) {
        const int p = i ^ j;
        if (p > i) {
          const bool up = (i & k) == 0;
          const float da = dist[i], db = dist[p];
          const int ta = tokn[i], tb = tokn[p];
          const bool a_first = dist_before(da, ta, db, tb);
          if (up ? !a_first : a_first) {
            dist[i] = db;
            dist[p] = da;
            tokn[i] = tb;
            tokn[p] = ta;
          }
        }
      }
      __syncthreads();
    }
  }
  for (int i = threadIdx.x; i < n; i += blockDim.x) order[bh * S + start + i] = tokn[i];
}

// Cluster sizes staged in shared memory for the selecting thread (C above this reads
// them from global memory).
constexpr int kRoundRobinStage = 4096;

// One CTA per head (or one in total for the shared variant): round-robin stratified
// selection across non-empty clusters, then w = |G_a| / m_a normalised to sum 1.
__global__ void __launch_bounds__(256) round_robin_kernel(
    const int32_t* __restrict__ slot_token, const int32_t* __restrict__ order, int S, int C, int M,
    const int32_t* __restrict__ count, const int32_t* __restrict__ off, int32_t* __restrict__ idx,
    float* __restrict__ weights) {
  __shared__ int owner[kMaxProbes];
  __shared__ int chosen[kMaxProbes];
  __shared__ float wsum[256];
  __shared__ int n_taken;
  __shared__ int cnt_s[kRoundRobinStage];  // cluster sizes, read by the selecting thread
  const int bh = blockIdx.x;
  const int32_t* ord = order ? order + static_cast<int64_t>(bh) * S : nullptr;
  const bool staged = C <= kRoundRobinStage;
  for (int a = threadIdx.x; a < C && staged; a += blockDim.x) cnt_s[a] = count[a];
  __syncthreads();
  auto cnt = [&](int a) -> int { return staged ? cnt_s[a] : count[a]; };
  auto member = [&](int a, int k) -> int {
    const int n = cnt(a);
    return ord ? ord[off[a] + k] : slot_token[off[a] + middle_out(n, k)];
  };
  if (threadIdx.x == 0) {
    int cp = 0;
    for (int a = 0; a < C; ++a) cp += cnt(a) > 0;
    int taken = 0;
    if (M < cp) {
      int a = -1, seen = -1;
      for (int i = 0; i < M; ++i) {
        const int target = static_cast<int>((static_cast<int64_t>(i) * cp) / M);
        while (seen < target) {
          ++a;
          if (cnt(a) > 0) ++seen;
        }
        owner[taken] = a;
        chosen[taken++] = member(a, 0);
      }
    } else {
      for (int p = 0; taken < M; ++p) {
        bool any = false;
        for (int a = 0; a < C && taken < M; ++a) {
          if (cnt(a) > p) {
            owner[taken] = a;
            chosen[taken++] = member(a, p);
            any = true;
          }
        }
        if (!any) break;
      }
    }
    n_taken = taken;
  }
  __syncthreads();
  const int taken = n_taken;
  float local = 0.f;
  for (int i = threadIdx.x; i < M; i += blockDim.x) {
    if (i < taken) {
      int m = 0;
      for (int j = 0; j < taken; ++j) m += owner[j] == owner[i];
      const float w = static_cast<float>(cnt(owner[i])) / static_cast<float>(m);
      weights[static_cast<int64_t>(bh) * M + i] = w;
      local += w;
    }
  }
  wsum[threadIdx.x] = local;
  __syncthreads();
  for (int o = 128; o > 0; o >>= 1) {
    if (threadIdx.x < o) wsum[threadIdx.x] += wsum[threadIdx.x + o];
    __syncthreads();
  }
  const float inv = 1.f / wsum[0];
  for (int i = threadIdx.x; i < M; i += blockDim.x) {
    float* w = weights + static_cast<int64_t>(bh) * M + i;
    if (i < taken) {
      idx[static_cast<int64_t>(bh) * M + i] = chosen[i];
      *w = *w * inv;
    } else {
      idx[static_cast<int64_t>(bh) * M + i] = chosen[0];  // fewer rows than M exist
      *w = 0.f;
    }
  }
}

// qp[b,h,m] = q[b,h,idx[m]] (shared) or q[b,h,idx[b,h,m]] (per head); 16-byte vectors.
__global__ void gather_probe_rows_kernel(const uint4* __restrict__ q, uint4* __restrict__ qp,
                                         const int32_t* __restrict__ idx, int per_head, int S,
                                         int M, int vpr, int H) {
  const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t bh = static_cast<int64_t>(blockIdx.z) * H + blockIdx.y;
  const int m = static_cast<int>(t / vpr), v = static_cast<int>(t % vpr);
  if (m >= M) return;
  const int row = per_head ? idx[bh * M + m] : idx[m];
  uint4 val = make_uint4(0, 0, 0, 0);
  if (row >= 0 && row < S) val = q[(bh * S + row) * vpr + v];
  else if (v == 0) report_device_error(kStatusBadLabel, 51);
  qp[(bh * M + m) * vpr + v] = val;
}

namespace {
struct ProbeSelLayout {
  int32_t *slot_token, *count, *off, *order;
  size_t bytes;
};
ProbeSelLayout carve_sel(int S, int C, int BH, void* ws) {
  Carver cv(ws);
  ProbeSelLayout L{};
  L.slot_token = cv.take<int32_t>(S);
  L.count = cv.take<int32_t>(C);
  L.off = cv.take<int32_t>(C + 1);
  L.order = cv.take<int32_t>(static_cast<size_t>(BH) * S);
  L.bytes = align_up(cv.used, 256);
  return L;
}
}  // namespace

}  // namespace bsa

extern "C" size_t bsa_probe_select_workspace_bytes(int S, int C, int n_heads) {
  if (S <= 0 || C <= 0 || n_heads <= 0) return 0;
  return bsa::carve_sel(S, C, n_heads, nullptr).bytes;
}

extern "C" int bsa_select_probe_rows(const int32_t* labels, int S, int C, int M, const void* q,
                                     bsa_shape shape, int32_t* probe_idx, float* weights,
                                     void* workspace, size_t workspace_bytes, void* stream) {
  using namespace bsa;
  cudaStream_t st = as_stream(stream);
  if (!labels || !probe_idx || !weights) return fail(BSA_ERR_INVALID_ARG, "null pointer argument");
  if (S <= 0 || C <= 0 || M <= 0) return fail(BSA_ERR_INVALID_ARG, "bad sizes");
  if (S > 65536 || C > 16384 || M > kMaxProbes)
    return fail(BSA_ERR_UNSUPPORTED, "S<=65536, C<=16384, M<=%d required", kMaxProbes);
  const int BH = q ? shape.B * shape.Hq : 1;
  if (q) {
    if (shape.Sq != S || (shape.D != 64 && shape.D != 128) || shape.D > 128)
      return fail(BSA_ERR_INVALID_ARG, "q shape does not match labels");
    if (shape.dtype != BSA_BF16 && shape.dtype != BSA_F32) return fail(BSA_ERR_UNSUPPORTED, "dtype");
  }
  ProbeSelLayout L = carve_sel(S, C, BH, workspace);
  if (!workspace || workspace_bytes < L.bytes)
    return fail(BSA_ERR_WORKSPACE, "workspace %zu < %zu bytes", workspace_bytes, L.bytes);
  int rc = run_label_sort(labels, S, C, 1, S, L.slot_token, nullptr, L.count, L.off, nullptr,
                          nullptr, 0, nullptr, 0, nullptr, st);
  if (rc) return rc;
  if (q) {
    const dim3 grid(C, shape.Hq, shape.B);
    if (shape.dtype == BSA_BF16)
      centroid_order_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(
          static_cast<const __nv_bfloat16*>(q), S, shape.D, shape.Hq, C, M, L.slot_token, L.count,
          L.off, L.order);
    else
      centroid_order_kernel<float><<<grid, 256, 0, st>>>(static_cast<const float*>(q), S,
                                                          shape.D, shape.Hq, C, M, L.slot_token,
                                                          L.count, L.off, L.order);
    count_launch();
    if ((rc = check_cuda(cudaGetLastError(), "centroid_order_kernel"))) return rc;
  }
  round_robin_kernel<<<BH, 256, 0, st>>>(L.slot_token, q ? L.order : nullptr, S, C, M, L.count,
                                         L.off, probe_idx, weights);
  count_launch();
  return check_cuda(cudaGetLastError(), "round_robin_kernel");
}

namespace bsa {
// The gathered probe rows, (B, Hq, M, D), are the same memory as (B, Hkv, G M, D) with
// G = Hq / Hkv: the probe rows of the G query heads that share a KV head run as one
// attention problem of G M rows per KV head (fewer, fuller 128-row tiles than one
// problem of M rows per query head), and o_probe comes out in the same layout.
inline bsa_shape probe_attention_shape(const bsa_shape& shape, int M) {
  bsa_shape ps = shape;
  const int G = shape.Hkv > 0 ? shape.Hq / shape.Hkv : 1;
  ps.Hq = shape.Hkv;
  ps.Sq = G * M;
  return ps;
}
}  // namespace bsa

extern "C" size_t bsa_probe_attention_workspace_bytes(bsa_shape shape, int M) {
  using namespace bsa;
  if (M <= 0 || M > kMaxProbes) return 0;
  if (shape.Hkv <= 0 || shape.Hq <= 0 || shape.Hq % shape.Hkv) return 0;
  const int es = shape.dtype == BSA_F32 ? 4 : 2;
  const bsa_shape ps = probe_attention_shape(shape, M);
  Carver cv(nullptr);
  cv.take<uint8_t>(static_cast<size_t>(shape.B) * shape.Hq * M * shape.D * es);
  cv.take<int32_t>(static_cast<size_t>(ps.Sq > shape.Sk ? ps.Sq : shape.Sk));
  cv.take<uint8_t>(16);
  const size_t att = attention_workspace_bytes(ps, 1, 1);
  return align_up(cv.used, 256) + att;
}

extern "C" int bsa_probe_dense_attention(const void* q, const void* k, const void* v,
                                         bsa_shape shape, const int32_t* probe_idx, int M,
                                         int per_head, float scale, float* o_probe,
                                         void* workspace, size_t workspace_bytes, void* stream) {
  using namespace bsa;
  cudaStream_t st = as_stream(stream);
  if (!q || !k || !v || !probe_idx || !o_probe) return fail(BSA_ERR_INVALID_ARG, "null pointer");
  if (M <= 0 || M > kMaxProbes) return fail(BSA_ERR_UNSUPPORTED, "M must be in [1, %d]", kMaxProbes);
  if (shape.Hkv <= 0 || shape.Hq <= 0 || shape.Hq % shape.Hkv)
    return fail(BSA_ERR_INVALID_ARG, "Hq (%d) not a positive multiple of Hkv (%d)", shape.Hq, shape.Hkv);
  const size_t need = bsa_probe_attention_workspace_bytes(shape, M);
  if (!need) return fail(BSA_ERR_INVALID_ARG, "bad shape");
  if (!workspace || workspace_bytes < need)
    return fail(BSA_ERR_WORKSPACE, "workspace %zu < %zu bytes", workspace_bytes, need);
  const int es = shape.dtype == BSA_F32 ? 4 : 2;
  Carver cv(workspace);
  void* qp = cv.take<uint8_t>(static_cast<size_t>(shape.B) * shape.Hq * M * shape.D * es);
  const bsa_shape ps = probe_attention_shape(shape, M);
  const int nz = ps.Sq > shape.Sk ? ps.Sq : shape.Sk;
  int32_t* zeros = cv.take<int32_t>(nz);
  uint8_t* one = cv.take<uint8_t>(16);
  const size_t used = align_up(cv.used, 256);
  int rc;
  const int vpr = shape.D * es / 16;
  const int64_t n = static_cast<int64_t>(M) * vpr;
  gather_probe_rows_kernel<<<dim3(static_cast<unsigned>((n + 255) / 256), shape.Hq, shape.B), 256, 0,
                             st>>>(static_cast<const uint4*>(q), static_cast<uint4*>(qp), probe_idx,
                                   per_head, shape.Sq, M, vpr, shape.Hq);
  count_launch();
  if ((rc = check_cuda(cudaGetLastError(), "gather_probe_rows_kernel"))) return rc;
  // Every probe row keeps every key: one query cluster, one key cluster, one kept block
  // (the sorts and the tile plan are identities, filled directly; the label and mask
  // buffers passed along are never read on that path).
  return centroid_compensated_attention(qp, k, v, ps, zeros, 1, zeros, 1, one, 0, 0, scale, 0,
                                        o_probe, static_cast<char*>(workspace) + used,
                                        workspace_bytes - used, st, kProfProbe, true, false);
}
