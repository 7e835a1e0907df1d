// SVG-EAR error-aware routing: which (query cluster, key cluster) blocks to compute
// exactly.
//
// Sources: "Sparse-block compensation" (mlx-arsenal notes), §SVG-EAR — centroid
// compensation (the paper adds an error-aware router choosing which blocks to compute
// exactly); the SVG-EAR abstract (a lightweight probe estimates each block's
// compensation error; the blocks with the highest error-to-cost ratio are computed
// exactly, the others compensated).
//
// Per (batch, query head):
//   probe of query cluster a   q̄_a, the mean query of the cluster
//   block error                err_ac = || E_ac - A_ac ||_2 with, for dense logits
//                              l_j = scale q̄_a . k_j, m their max, Z = sum_j exp(l_j - m):
//                              E_ac = sum_{j in c} exp(l_j - m) v_j / Z (exact) and
//                              A_ac = n_c exp(scale q̄_a . k̄_c - m) v̄_c / Z (centroid term)
//   cost, ratio                n_a n_c token pairs; ratio = err_ac / n_c
//   selection                  blocks of non-empty clusters by descending ratio (equal
//                              ratios: lower a*Ck + c), the longest prefix whose pairs
//                              sum to at most floor(density * Sq * Sk)
//
// Kernels (caller's stream): label sorts of both label arrays (the attention's sort),
// per-cluster means of Q, K and V (fp32), the probe kernel (one CTA per 16 probes of a
// head, streaming the head's keys cluster by cluster through shared memory), and one
// CTA per head that selects the prefix exactly by a radix descent over the ratios'
// bits with 64-bit pair counts.
#include <cuda_bf16.h>

#include <cmath>

#include "common.cuh"
#include "ptx.cuh"

namespace bsa {

// ---------------------------------------------------------------- cluster means
// grid (C, H, B), 128 threads: dst[b,h,c,:] = mean of src[b,h,tok,:] over the tokens of
// cluster c (slots off[c] .. off[c] + count[c] of the sorted order); 0 if empty.
template <typename T>
__global__ void __launch_bounds__(128) cluster_mean_kernel(const T* __restrict__ src,
                                                           const int32_t* __restrict__ sort_token,
                                                           const int32_t* __restrict__ count,
                                                           const int32_t* __restrict__ off, int C,
                                                           int S, int D, int H,
                                                           float* __restrict__ dst) {
  const int c = blockIdx.x;
  const int64_t bh = static_cast<int64_t>(blockIdx.z) * H + blockIdx.y;
  const int n = count[c], o = off[c];
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    float acc = 0.f;
    for (int i = 0; i < n; ++i) {
      const int tok = sort_token[o + i];
      acc += static_cast<float>(src[(bh * S + tok) * D + d]);
    }
    dst[(bh * C + c) * D + d] = n > 0 ? acc / static_cast<float>(n) : 0.f;
  }
}

// ---------------------------------------------------------------- probe errors
constexpr int kRouteProbes = 16;   // probes per CTA
constexpr int kRouteKeys = 32;     // keys per shared-memory chunk
constexpr int kRouteThreads = 256; // 16 threads per probe

__device__ __forceinline__ float route_f(float x) { return x; }
__device__ __forceinline__ float route_f(__nv_bfloat16 x) { return __bfloat162float(x); }

struct RouteArgs {
  int B, Hq, Hkv, S, D, Cq, Ck;
  float scale;
  const float* qbar;   // (B, Hq, Cq, D)
  const float* kbar;   // (B, Hkv, Ck, D)
  const float* vbar;   // (B, Hkv, Ck, D)
  const int32_t* q_count;
  const int32_t* k_sort_token;
  const int32_t* k_count;
  const int32_t* k_off;
  float* err;   // (B, Hq, Cq, Ck): written
  float* mref;  // (B, Hq, Cq, Ck): per-block reference of the unscaled error (scratch)
};

// grid (ceil(Cq / 16), Hq, B), 256 threads: the 16 probes (query clusters a0 .. a0+15)
// of one head against every key of its KV head. kp / vp hold the keys and values of each
// (batch, KV head) in cluster-major order (cluster c at rows off[c] .. off[c] + n_c).
// Warp w takes the key clusters w, w + 8, ...; inside a cluster lane j holds key j of
// each 32-key chunk and computes its 16 probe logits (probe rows stored transposed, so
// one broadcast float4 feeds four probes through packed f32x2 FMAs); each lane also
// owns dims [DL lane, DL lane + DL) of the 16 running difference vectors
// sum_j exp(l_j - m) v_j, fed by shuffles of the keys' weights. Every warp keeps its
// own running reference m (the largest logit it has seen, centroid logits included)
// and sum z per probe; at the end of a cluster the norm of (difference - n_c exp(lc - m)
// vbar_c) is stored with the reference it was taken with, and once all warps are done
// every error is brought to the common reference and divided by the total Z.
template <typename T, int D>
__global__ void __launch_bounds__(kRouteThreads) route_probe_kernel(const T* __restrict__ kp,
                                                                     const T* __restrict__ vp,
                                                                     const RouteArgs a) {
  constexpr int NP = kRouteProbes;        // 16
  constexpr int NW = kRouteThreads / 32;  // 8 warps
  constexpr int DL = D / 32;              // dims per lane
  constexpr int EPV = 16 / sizeof(T);     // elements per 16-byte vector
  __shared__ __align__(16) float sqt[D][NP];   // probe rows, transposed
  __shared__ __align__(16) float s_w[NW][32][NP];  // per warp: the 16 weights of each key of a chunk
  __shared__ float s_m[NW][NP], s_z[NW][NP];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int h = blockIdx.y, b = blockIdx.z;
  const int hkv = h / (a.Hq / a.Hkv);
  const int a0 = blockIdx.x * NP;
  const int64_t bq = static_cast<int64_t>(b) * a.Hq + h;
  const int64_t bk = static_cast<int64_t>(b) * a.Hkv + hkv;
  for (int e = tid; e < NP * D; e += kRouteThreads) {
    const int pp = e / D, d = e % D;
    sqt[d][pp] = (a0 + pp < a.Cq) ? a.qbar[(bq * a.Cq + a0 + pp) * D + d] : 0.f;
  }
  __syncthreads();
  const float* kb = a.kbar + bk * a.Ck * D;
  const float* vb = a.vbar + bk * a.Ck * D;
  const T* kbase = kp + bk * a.S * D;
  const T* vbase = vp + bk * a.S * D;
  float m[NP], z[NP], diff[NP][DL];
#pragma unroll
  for (int p = 0; p < NP; ++p) {
    m[p] = -INFINITY;
    z[p] = 0.f;
  }
  for (int c = warp; c < a.Ck; c += NW) {
    const int n = a.k_count[c], o = a.k_off[c];
    // the (probe, cluster) slots of this cluster: lane p < 16 writes probe p's
    float* err_p = a.err + (bq * a.Cq + a0 + (lane & (NP - 1))) * a.Ck;
    float* mref_p = a.mref + (bq * a.Cq + a0 + (lane & (NP - 1))) * a.Ck;
    const bool writer = lane < NP && a0 + lane < a.Cq;
    if (n == 0) {
      if (writer) {
        err_p[c] = 0.f;
        mref_p[c] = 0.f;
      }
      continue;
    }
    // centroid logits: lane p (< 16) computes probe p's, then every lane gets all 16
    float lcl = 0.f;
    if (lane < NP)
#pragma unroll 8
      for (int d = 0; d < D; ++d) lcl = fmaf(sqt[d][lane], kb[c * D + d], lcl);
    float lc[NP];
#pragma unroll
    for (int p = 0; p < NP; ++p) {
      lc[p] = __shfl_sync(0xffffffffu, lcl, p) * a.scale;
      if (lc[p] > m[p]) {
        z[p] *= __expf(m[p] - lc[p]);
        m[p] = lc[p];
      }
#pragma unroll
      for (int i = 0; i < DL; ++i) diff[p][i] = 0.f;
    }
    // one 32-key group: chunk maxima, new references, weights and their sums, then the
    // difference vectors (the lane's dims of each key's value row; a key's 16 weights
    // come as four broadcast loads)
    auto group = [&](const float (&l)[NP], int jb, int nk) {
      const bool mine = lane < nk;
      float w[NP];
#pragma unroll
      for (int p = 0; p < NP; ++p) {
        const float lp = mine ? l[p] * a.scale : -INFINITY;
        float mx = lp;
#pragma unroll
        for (int o2 = 16; o2 > 0; o2 >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o2));
        if (mx > m[p]) {
          const float f = __expf(m[p] - mx);
          z[p] *= f;
#pragma unroll
          for (int i = 0; i < DL; ++i) diff[p][i] *= f;
          m[p] = mx;
        }
        w[p] = mine ? __expf(lp - m[p]) : 0.f;
        s_w[warp][lane][p] = w[p];
        float ws = w[p];
#pragma unroll
        for (int o2 = 16; o2 > 0; o2 >>= 1) ws += __shfl_xor_sync(0xffffffffu, ws, o2);
        z[p] += ws;
      }
      __syncwarp();
      for (int jj = 0; jj < nk; ++jj) {
        const T* vrow = vbase + static_cast<int64_t>(o + jb + jj) * D + DL * lane;
        float vx[DL];
        if constexpr (DL == 4) {
          const uint2 u = *reinterpret_cast<const uint2*>(vrow);
          if constexpr (sizeof(T) == 2) {
            const float2 lo = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
            const float2 hi = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
            vx[0] = lo.x; vx[1] = lo.y; vx[2] = hi.x; vx[3] = hi.y;
          }
        }
        if constexpr (sizeof(T) == 4 || DL != 4) {
#pragma unroll
          for (int i = 0; i < DL; ++i) vx[i] = route_f(vrow[i]);
        }
#pragma unroll
        for (int p4 = 0; p4 < NP; p4 += 4) {
          const float4 w4 = *reinterpret_cast<const float4*>(&s_w[warp][jj][p4]);
#pragma unroll
          for (int i = 0; i < DL; ++i) {
            fma2(diff[p4][i], diff[p4 + 1][i], w4.x, w4.y, vx[i], vx[i], diff[p4][i], diff[p4 + 1][i]);
            fma2(diff[p4 + 2][i], diff[p4 + 3][i], w4.z, w4.w, vx[i], vx[i], diff[p4 + 2][i],
                 diff[p4 + 3][i]);
          }
        }
      }
      __syncwarp();
    };
    // 64 keys at a time: the 16 logits of the lane's two keys (j0 + lane, j0 + 32 + lane),
    // one broadcast float4 of probe rows feeding both
    for (int j0 = 0; j0 < n; j0 += 64) {
      const int nk0 = min(32, n - j0), nk1 = max(0, min(32, n - j0 - 32));
      float l0[NP], l1[NP];
#pragma unroll
      for (int p = 0; p < NP; ++p) l0[p] = l1[p] = 0.f;
      const T* krow0 = kbase + static_cast<int64_t>(o + j0 + (lane < nk0 ? lane : 0)) * D;
      const T* krow1 = kbase + static_cast<int64_t>(o + j0 + 32 + (lane < nk1 ? lane : 0) - (nk1 ? 0 : 32)) * D;
#pragma unroll 4
      for (int v0 = 0; v0 < D; v0 += EPV) {
        float k0[EPV], k1[EPV];
        unpack16<T>(__ldg(reinterpret_cast<const uint4*>(krow0 + v0)), k0);
        unpack16<T>(__ldg(reinterpret_cast<const uint4*>(krow1 + v0)), k1);
#pragma unroll
        for (int t = 0; t < EPV; ++t) {
#pragma unroll
          for (int p4 = 0; p4 < NP; p4 += 4) {
            const float4 qv = *reinterpret_cast<const float4*>(&sqt[v0 + t][p4]);
            fma2(l0[p4], l0[p4 + 1], k0[t], k0[t], qv.x, qv.y, l0[p4], l0[p4 + 1]);
            fma2(l0[p4 + 2], l0[p4 + 3], k0[t], k0[t], qv.z, qv.w, l0[p4 + 2], l0[p4 + 3]);
            fma2(l1[p4], l1[p4 + 1], k1[t], k1[t], qv.x, qv.y, l1[p4], l1[p4 + 1]);
            fma2(l1[p4 + 2], l1[p4 + 3], k1[t], k1[t], qv.z, qv.w, l1[p4 + 2], l1[p4 + 3]);
          }
        }
      }
      group(l0, j0, nk0);
      if (nk1 > 0) group(l1, j0 + 32, nk1);
    }
    // cluster c done: the norm of (difference - centroid term), taken with reference m
    float vbl[DL];
#pragma unroll
    for (int i = 0; i < DL; ++i) vbl[i] = vb[c * D + DL * lane + i];
    float e2w = 0.f;  // lane p (< 16) ends with probe p's squared norm
#pragma unroll
    for (int p = 0; p < NP; ++p) {
      const float wc = static_cast<float>(n) * __expf(lc[p] - m[p]);
      float e2 = 0.f;
#pragma unroll
      for (int i = 0; i < DL; ++i) {
        const float dd = diff[p][i] - wc * vbl[i];
        e2 = fmaf(dd, dd, e2);
      }
#pragma unroll
      for (int o2 = 16; o2 > 0; o2 >>= 1) e2 += __shfl_xor_sync(0xffffffffu, e2, o2);
      if (lane == p) e2w = e2;
    }
    float mw = m[0];
#pragma unroll
    for (int p = 1; p < NP; ++p) mw = lane == p ? m[p] : mw;
    if (writer) {
      err_p[c] = sqrtf(e2w);
      mref_p[c] = mw;
    }
  }
  // every warp's references and sums, combined per probe
  if (lane == 0) {
#pragma unroll
    for (int p = 0; p < NP; ++p) {
      s_m[warp][p] = m[p];
      s_z[warp][p] = z[p];
    }
  }
  __syncthreads();
  for (int e = tid; e < NP * a.Ck; e += kRouteThreads) {
    const int pp = e / a.Ck, c = e % a.Ck;
    if (a0 + pp >= a.Cq) continue;
    float M = -INFINITY;
    for (int ww = 0; ww < NW; ++ww) M = fmaxf(M, s_m[ww][pp]);
    float Z = 0.f;
    for (int ww = 0; ww < NW; ++ww)
      if (s_z[ww][pp] > 0.f) Z += s_z[ww][pp] * __expf(s_m[ww][pp] - M);
    float* err = a.err + (bq * a.Cq + a0 + pp) * a.Ck;
    const float* mref = a.mref + (bq * a.Cq + a0 + pp) * a.Ck;
    const bool ok = a.q_count[a0 + pp] > 0 && a.k_count[c] > 0 && Z > 0.f;
    err[c] = ok ? err[c] * __expf(mref[c] - M) / Z : 0.f;
  }
}

// ---------------------------------------------------------------- budgeted selection
// One CTA (1024 threads) per (batch, head). Keys are the bit patterns of the
// non-negative float ratios err / n_c (monotone in the value); invalid blocks (an
// empty cluster) take no part. A radix descent, 8 bits per pass from the top, finds
// the key k* at which the pair count of the blocks above it, plus those at k*, first
// exceeds the budget; blocks above k* are kept, and those equal to k* in index order
// while the running count stays within the budget.
__global__ void __launch_bounds__(1024) route_select_kernel(const float* __restrict__ err,
                                                            const int32_t* __restrict__ q_count,
                                                            const int32_t* __restrict__ k_count,
                                                            int Cq, int Ck, double density,
                                                            uint8_t* __restrict__ mask) {
  // per-warp histograms (most ratios share their top bits: one histogram for the whole
  // CTA would serialise its atomics), summed into hist after each pass
  extern __shared__ unsigned long long whist[];  // 32 x 256
  __shared__ unsigned long long hist[256];
  __shared__ unsigned long long s_part[32];
  __shared__ unsigned long long s_sq, s_sk;
  __shared__ uint32_t s_prefix;
  __shared__ long long s_rem;
  __shared__ int s_all;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t bh = blockIdx.x;
  const int64_t E = static_cast<int64_t>(Cq) * Ck;
  const float* e_bh = err + bh * E;
  uint8_t* m_bh = mask + bh * E;
  // totals of valid query and key rows
  unsigned long long sq = 0, sk = 0;
  for (int a = tid; a < Cq; a += 1024) sq += static_cast<unsigned long long>(max(q_count[a], 0));
  for (int c = tid; c < Ck; c += 1024) sk += static_cast<unsigned long long>(max(k_count[c], 0));
  if (tid == 0) { s_sq = 0; s_sk = 0; }
  __syncthreads();
  sq = __reduce_add_sync(0xffffffffu, static_cast<unsigned>(sq));
  sk = __reduce_add_sync(0xffffffffu, static_cast<unsigned>(sk));
  if (lane == 0) { atomicAdd(&s_sq, sq); atomicAdd(&s_sk, sk); }
  __syncthreads();
  const long long budget = static_cast<long long>(
      floor(density * static_cast<double>(s_sq) * static_cast<double>(s_sk)));
  auto key_of = [&](int64_t e, uint32_t& key, long long& cost) -> bool {
    const int a_ = static_cast<int>(e / Ck), c_ = static_cast<int>(e % Ck);
    const int na = q_count[a_], nc = k_count[c_];
    if (na <= 0 || nc <= 0) return false;
    const float r = __fdiv_rn(e_bh[e], static_cast<float>(nc));
    key = __float_as_uint(fmaxf(r, 0.f));
    cost = static_cast<long long>(na) * nc;
    return true;
  };
  if (tid == 0) { s_prefix = 0; s_rem = budget; s_all = 0; }
  __syncthreads();
  // radix descent: after pass p the top 8(p+1) bits of k* are known
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int i = tid; i < 32 * 256; i += 1024) whist[i] = 0;
    __syncthreads();
    const uint32_t pre = s_prefix;
    const uint32_t hi_mask = pass == 0 ? 0u : (0xffffffffu << (shift + 8));
    for (int64_t e = tid; e < E; e += 1024) {
      uint32_t key;
      long long cost;
      if (!key_of(e, key, cost)) continue;
      if ((key & hi_mask) != (pre & hi_mask)) continue;
      atomicAdd(&whist[warp * 256 + ((key >> shift) & 255u)], static_cast<unsigned long long>(cost));
    }
    __syncthreads();
    for (int i = tid; i < 256; i += 1024) {
      unsigned long long t = 0;
      for (int w = 0; w < 32; ++w) t += whist[w * 256 + i];
      hist[i] = t;
    }
    __syncthreads();
    if (tid == 0) {
      long long rem = s_rem;
      int digit = -1;
      for (int d = 255; d >= 0; --d) {
        const long long hcost = static_cast<long long>(hist[d]);
        if (hcost > rem) { digit = d; break; }
        rem -= hcost;
      }
      if (digit < 0) {
        s_all = 1;  // every block under this prefix fits
      } else {
        s_prefix = pre | (static_cast<uint32_t>(digit) << shift);
        s_rem = rem;
      }
    }
    __syncthreads();
    if (s_all) break;
  }
  const bool all = s_all != 0;
  const uint32_t kstar = s_prefix;
  const long long rem_at_k = s_rem;  // budget left for the blocks equal to k*
  // blocks above k* (or every block when all fit); blocks at k* in index order
  unsigned long long carry = 0;
  for (int64_t t0 = 0; t0 < E; t0 += 1024) {
    const int64_t e = t0 + tid;
    uint32_t key = 0;
    long long cost = 0;
    const bool valid = e < E && key_of(e, key, cost);
    uint8_t keep = 0;
    unsigned long long tie_cost = 0;
    if (valid) {
      if (all || key > kstar) keep = 1;
      else if (key == kstar) tie_cost = static_cast<unsigned long long>(cost);
    }
    // inclusive block scan of tie_cost
    unsigned long long x = tie_cost;
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned long long y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) s_part[warp] = x;
    __syncthreads();
    if (warp == 0) {
      unsigned long long w = s_part[lane];
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned long long y = __shfl_up_sync(0xffffffffu, w, o);
        if (lane >= o) w += y;
      }
      s_part[lane] = w;  // inclusive over warps
    }
    __syncthreads();
    const unsigned long long before = warp > 0 ? s_part[warp - 1] : 0ull;
    const unsigned long long incl = carry + before + x;
    if (tie_cost > 0 && static_cast<long long>(incl) <= rem_at_k) keep = 1;
    carry += s_part[31];
    __syncthreads();
    if (e < E) m_bh[e] = keep;
  }
}

// ---------------------------------------------------------------- centroid mass
// grid (Cq, Hq, B), 128 threads: mass[b,h,a,c] = softmax over the key clusters of
// scale * qbar_a . kbar_c + ln n_c (empty key clusters 0; an empty query cluster's row
// is 0): the share of the mean query's attention that falls on each key cluster when
// every key is replaced by its cluster centroid.
template <int D>
__global__ void __launch_bounds__(128) centroid_mass_kernel(const RouteArgs a,
                                                            float* __restrict__ mass) {
  __shared__ float qa[D];
  __shared__ float red[4];
  const int c0 = blockIdx.x, h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const int hkv = h / (a.Hq / a.Hkv);
  const int64_t bq = static_cast<int64_t>(b) * a.Hq + h;
  const int64_t bk = static_cast<int64_t>(b) * a.Hkv + hkv;
  float* row = mass + (bq * a.Cq + c0) * a.Ck;
  if (a.q_count[c0] <= 0) {
    for (int c = tid; c < a.Ck; c += 128) row[c] = 0.f;
    return;
  }
  for (int d = tid; d < D; d += 128) qa[d] = a.qbar[(bq * a.Cq + c0) * D + d];
  __syncthreads();
  float mx = -INFINITY;
  for (int c = tid; c < a.Ck; c += 128) {
    const int n = a.k_count[c];
    float l = -INFINITY;
    if (n > 0) {
      float acc = 0.f;
      const float* kc = a.kbar + (bk * a.Ck + c) * D;
#pragma unroll 8
      for (int d = 0; d < D; ++d) acc = fmaf(qa[d], kc[d], acc);
      l = a.scale * acc + logf(static_cast<float>(n));
    }
    row[c] = l;
    mx = fmaxf(mx, l);
  }
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if ((tid & 31) == 0) red[tid >> 5] = mx;
  __syncthreads();
  mx = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
  __syncthreads();
  float sum = 0.f;
  for (int c = tid; c < a.Ck; c += 128) {
    const float e = row[c] == -INFINITY ? 0.f : __expf(row[c] - mx);
    row[c] = e;
    sum += e;
  }
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if ((tid & 31) == 0) red[tid >> 5] = sum;
  __syncthreads();
  const float inv = 1.f / ((red[0] + red[1]) + (red[2] + red[3]));
  for (int c = tid; c < a.Ck; c += 128) row[c] *= inv;
}

namespace {
struct RouteLayout {
  int32_t *q_tok, *q_count, *q_off, *k_tok, *k_count, *k_off;
  float *qbar, *kbar, *vbar, *err, *mref;
  void *kp, *vp;  // keys and values in cluster-major order
  size_t bytes;
};
RouteLayout carve_route(const bsa_shape& s, int Cq, int Ck, void* ws) {
  Carver cv(ws);
  RouteLayout L{};
  L.q_tok = cv.take<int32_t>(s.Sq);
  L.q_count = cv.take<int32_t>(Cq);
  L.q_off = cv.take<int32_t>(Cq + 1);
  L.k_tok = cv.take<int32_t>(s.Sk);
  L.k_count = cv.take<int32_t>(Ck);
  L.k_off = cv.take<int32_t>(Ck + 1);
  L.qbar = cv.take<float>(static_cast<size_t>(s.B) * s.Hq * Cq * s.D);
  L.kbar = cv.take<float>(static_cast<size_t>(s.B) * s.Hkv * Ck * s.D);
  L.vbar = cv.take<float>(static_cast<size_t>(s.B) * s.Hkv * Ck * s.D);
  L.err = cv.take<float>(static_cast<size_t>(s.B) * s.Hq * Cq * Ck);
  L.mref = cv.take<float>(static_cast<size_t>(s.B) * s.Hq * Cq * Ck);
  const int es = s.dtype == BSA_F32 ? 4 : 2;
  L.kp = cv.take<uint8_t>(static_cast<size_t>(s.B) * s.Hkv * s.Sk * s.D * es);
  L.vp = cv.take<uint8_t>(static_cast<size_t>(s.B) * s.Hkv * s.Sk * s.D * es);
  L.bytes = align_up(cv.used, 256);
  return L;
}

int validate_route(const bsa_shape& s, int Cq, int Ck) {
  if (s.B <= 0 || s.Hq <= 0 || s.Hkv <= 0 || s.Sq <= 0 || s.Sk <= 0)
    return fail(BSA_ERR_INVALID_ARG, "non-positive shape");
  if (s.Hq % s.Hkv) return fail(BSA_ERR_INVALID_ARG, "Hq (%d) not a multiple of Hkv (%d)", s.Hq, s.Hkv);
  if (s.D != 64 && s.D != 128) return fail(BSA_ERR_UNSUPPORTED, "head dim %d not in {64,128}", s.D);
  if (s.dtype != BSA_BF16 && s.dtype != BSA_F32) return fail(BSA_ERR_UNSUPPORTED, "dtype %d", s.dtype);
  if (Cq <= 0 || Ck <= 0 || Cq > 16384 || Ck > 16384)
    return fail(BSA_ERR_UNSUPPORTED, "cluster counts Cq=%d Ck=%d outside [1,16384]", Cq, Ck);
  if (static_cast<int64_t>(Cq) * Ck > (int64_t(1) << 24))
    return fail(BSA_ERR_UNSUPPORTED, "Cq * Ck = %lld blocks per head exceeds 2^24",
                static_cast<long long>(Cq) * Ck);
  return BSA_OK;
}

template <typename T, int D>
void launch_route_probe(const void* k, const void* v, const RouteArgs& ra, cudaStream_t st) {
  route_probe_kernel<T, D><<<dim3((ra.Cq + kRouteProbes - 1) / kRouteProbes, ra.Hq, ra.B),
                             kRouteThreads, 0, st>>>(static_cast<const T*>(k),
                                                     static_cast<const T*>(v), ra);
}
}  // namespace

int route_prologue(const void* q, const void* k, const void* v, const bsa_shape& shape,
                   const int32_t* q_labels, int Cq, const int32_t* k_labels, int Ck, float scale,
                   uint8_t* mask, float* err, const RouteLayout& L, cudaStream_t st, float density,
                   int M);

}  // namespace bsa

extern "C" size_t bsa_routing_workspace_bytes(bsa_shape shape, int Cq, int Ck) {
  if (bsa::validate_route(shape, Cq, Ck)) return 0;
  return bsa::carve_route(shape, Cq, Ck, nullptr).bytes;
}

extern "C" int bsa_error_aware_block_mask(const void* q, const void* k, const void* v,
                                          bsa_shape shape, const int32_t* q_labels, int Cq,
                                          const int32_t* k_labels, int Ck, float density,
                                          float scale, uint8_t* mask, float* err,
                                          void* workspace, size_t workspace_bytes,
                                          void* stream) {
  using namespace bsa;
  int rc = validate_route(shape, Cq, Ck);
  if (rc) return rc;
  if (!q || !k || !v || !q_labels || !k_labels || !mask)
    return fail(BSA_ERR_INVALID_ARG, "null pointer argument");
  if (!(density >= 0.f && density <= 1.f))
    return fail(BSA_ERR_INVALID_ARG, "density %g outside [0, 1]", static_cast<double>(density));
  RouteLayout L = carve_route(shape, Cq, Ck, workspace);
  if (!workspace || workspace_bytes < L.bytes)
    return fail(BSA_ERR_WORKSPACE, "workspace %zu bytes < required %zu", workspace_bytes, L.bytes);
  if (reinterpret_cast<uintptr_t>(workspace) % 256)
    return fail(BSA_ERR_INVALID_ARG, "workspace not 256-byte aligned");
  return route_prologue(q, k, v, shape, q_labels, Cq, k_labels, Ck, scale, mask, err, L,
                        as_stream(stream), density, -1);
}

namespace bsa {
// Shared steps of both routers: label sorts, cluster means, then either the probe
// errors (M < 0: SVG-EAR) or the centroid masses (M >= 0: probe budget), and the exact
// budgeted selection at `density` (less M / Sq for the probe budget).
int route_prologue(const void* q, const void* k, const void* v, const bsa_shape& shape,
                   const int32_t* q_labels, int Cq, const int32_t* k_labels, int Ck, float scale,
                   uint8_t* mask, float* err, const RouteLayout& L, cudaStream_t st, float density,
                   int M) {
  int rc;
  const bsa_shape& s = shape;
  // 1. stable label sorts (cluster-major token order, counts, offsets)
  {
    const LabelSortJob jk{k_labels, s.Sk, Ck, 1, s.Sk, L.k_tok, nullptr, L.k_count, L.k_off,
                          nullptr, nullptr, 0, nullptr, 0, nullptr};
    const LabelSortJob jq{q_labels, s.Sq, Cq, 1, s.Sq, L.q_tok, nullptr, L.q_count, L.q_off,
                          nullptr, nullptr, 0, nullptr, 0, nullptr};
    if ((rc = launch_label_sorts(jk, &jq, st))) return rc;
  }
  // 2. cluster means of Q (probes), K and V (centroids), fp32
  const bool with_v = M < 0;
  if (s.dtype == BSA_F32) {
    cluster_mean_kernel<float><<<dim3(Cq, s.Hq, s.B), 128, 0, st>>>(
        static_cast<const float*>(q), L.q_tok, L.q_count, L.q_off, Cq, s.Sq, s.D, s.Hq, L.qbar);
    cluster_mean_kernel<float><<<dim3(Ck, s.Hkv, s.B), 128, 0, st>>>(
        static_cast<const float*>(k), L.k_tok, L.k_count, L.k_off, Ck, s.Sk, s.D, s.Hkv, L.kbar);
    if (with_v)
      cluster_mean_kernel<float><<<dim3(Ck, s.Hkv, s.B), 128, 0, st>>>(
          static_cast<const float*>(v), L.k_tok, L.k_count, L.k_off, Ck, s.Sk, s.D, s.Hkv, L.vbar);
  } else {
    using bf = __nv_bfloat16;
    cluster_mean_kernel<bf><<<dim3(Cq, s.Hq, s.B), 128, 0, st>>>(
        static_cast<const bf*>(q), L.q_tok, L.q_count, L.q_off, Cq, s.Sq, s.D, s.Hq, L.qbar);
    cluster_mean_kernel<bf><<<dim3(Ck, s.Hkv, s.B), 128, 0, st>>>(
        static_cast<const bf*>(k), L.k_tok, L.k_count, L.k_off, Ck, s.Sk, s.D, s.Hkv, L.kbar);
    if (with_v)
      cluster_mean_kernel<bf><<<dim3(Ck, s.Hkv, s.B), 128, 0, st>>>(
          static_cast<const bf*>(v), L.k_tok, L.k_count, L.k_off, Ck, s.Sk, s.D, s.Hkv, L.vbar);
  }
  for (int i = 0; i < (with_v ? 3 : 2); ++i) count_launch();
  if ((rc = check_cuda(cudaGetLastError(), "cluster_mean_kernel"))) return rc;
  // 3. probe errors
  RouteArgs ra{};
  ra.B = s.B;
  ra.Hq = s.Hq;
  ra.Hkv = s.Hkv;
  ra.S = s.Sk;
  ra.D = s.D;
  ra.Cq = Cq;
  ra.Ck = Ck;
  ra.scale = scale > 0.f ? scale : 1.f / std::sqrt(static_cast<float>(s.D));
  ra.qbar = L.qbar;
  ra.kbar = L.kbar;
  ra.vbar = L.vbar;
  ra.q_count = L.q_count;
  ra.k_sort_token = L.k_tok;
  ra.k_count = L.k_count;
  ra.k_off = L.k_off;
  ra.err = err ? err : L.err;
  ra.mref = L.mref;
  double route_density = static_cast<double>(density);
  if (with_v) {
    // keys and values in cluster-major order (rows off[c] .. off[c] + n_c per head)
    const int es = s.dtype == BSA_F32 ? 4 : 2;
    const int vpr = s.D * es / 16;
    const int64_t nvec = static_cast<int64_t>(s.Sk) * vpr;
    const dim3 gg(static_cast<unsigned>((nvec + 255) / 256), s.Hkv, s.B);
    gather_rows_kernel<<<gg, 256, 0, st>>>(static_cast<const uint4*>(k), static_cast<uint4*>(L.kp),
                                           L.k_tok, s.Sk, s.Sk, vpr, s.Hkv);
    gather_rows_kernel<<<gg, 256, 0, st>>>(static_cast<const uint4*>(v), static_cast<uint4*>(L.vp),
                                           L.k_tok, s.Sk, s.Sk, vpr, s.Hkv);
    count_launch();
    count_launch();
    if (s.dtype == BSA_F32) {
      if (s.D == 64) launch_route_probe<float, 64>(L.kp, L.vp, ra, st);
      else launch_route_probe<float, 128>(L.kp, L.vp, ra, st);
    } else {
      if (s.D == 64) launch_route_probe<__nv_bfloat16, 64>(L.kp, L.vp, ra, st);
      else launch_route_probe<__nv_bfloat16, 128>(L.kp, L.vp, ra, st);
    }
  } else {
    if (s.D == 64)
      centroid_mass_kernel<64><<<dim3(Cq, s.Hq, s.B), 128, 0, st>>>(ra, ra.err);
    else
      centroid_mass_kernel<128><<<dim3(Cq, s.Hq, s.B), 128, 0, st>>>(ra, ra.err);
    // the probe rows' M x Sk pairs come out of the budget first
    route_density = route_density - static_cast<double>(M) / static_cast<double>(s.Sq);
    if (route_density < 0.0) route_density = 0.0;
  }
  count_launch();
  if ((rc = check_cuda(cudaGetLastError(), "route score kernel"))) return rc;
  // 4. budgeted prefix per (batch, head)
  {
    const int smem = 32 * 256 * 8;
    cudaError_t e = cudaFuncSetAttribute(route_select_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return check_cuda(e, "cudaFuncSetAttribute(route_select)");
    route_select_kernel<<<s.B * s.Hq, 1024, smem, st>>>(ra.err, L.q_count, L.k_count, Cq, Ck,
                                                         route_density, mask);
  }
  count_launch();
  return check_cuda(cudaGetLastError(), "route_select_kernel");
}
}  // namespace bsa

extern "C" int bsa_probe_budget_block_mask(const void* q, const void* k, bsa_shape shape,
                                           const int32_t* q_labels, int Cq,
                                           const int32_t* k_labels, int Ck, float density, int M,
                                           float scale, uint8_t* mask, float* mass,
                                           void* workspace, size_t workspace_bytes,
                                           void* stream) {
  using namespace bsa;
  int rc = validate_route(shape, Cq, Ck);
  if (rc) return rc;
  if (!q || !k || !q_labels || !k_labels || !mask)
    return fail(BSA_ERR_INVALID_ARG, "null pointer argument");
  if (!(density >= 0.f && density <= 1.f))
    return fail(BSA_ERR_INVALID_ARG, "density %g outside [0, 1]", static_cast<double>(density));
  if (M < 0) return fail(BSA_ERR_INVALID_ARG, "M %d < 0", M);
  RouteLayout L = carve_route(shape, Cq, Ck, workspace);
  if (!workspace || workspace_bytes < L.bytes)
    return fail(BSA_ERR_WORKSPACE, "workspace %zu bytes < required %zu", workspace_bytes, L.bytes);
  if (reinterpret_cast<uintptr_t>(workspace) % 256)
    return fail(BSA_ERR_INVALID_ARG, "workspace not 256-byte aligned");
  return route_prologue(q, k, nullptr, shape, q_labels, Cq, k_labels, Ck, scale, mask, mass, L,
                        as_stream(stream), density, M);
}
