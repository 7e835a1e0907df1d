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
// one gather-and-mean pass per operand (fp32 means of Q, K and V; K and V also copied
// into cluster-major order), then the probe errors: for bf16 inputs the centroid
// logits and a tensor-core kernel (tcgen05 MMAs for q̄ . k_j and the weighted value
// sums, per 128 probes and a key-balanced range of clusters) followed by a
// normalisation to one reference per probe; for fp32 inputs an FMA-pipe kernel (one CTA
// per 16 probes of a head, streaming the head's keys cluster by cluster through shared
// memory). Last, one CTA per head selects the prefix exactly by a radix descent over
// the ratios' bits with 64-bit pair counts.
#include <cuda_bf16.h>

#include <algorithm>
#include <cmath>

#include "common.cuh"
#include "ptx.cuh"

namespace bsa {

// ---------------------------------------------------------------- cluster means
// grid (C, H, B), 256 threads: mean[b,h,c,:] = mean of src[b,h,tok,:] over the tokens of
// cluster c (slots off[c] .. off[c] + count[c] of the sorted order; 0 if empty), fp32.
// With dst, the rows are also copied to dst in cluster-major order (row off[c] + i of
// the (b, h) slab), so one pass gathers and averages. Each warp takes 32 / VPR rows per
// pass (VPR 16-byte vectors per row, one per lane) and each thread keeps four rows in
// flight; the row slots' partial sums meet in shared memory.
template <typename T, int VPR>
__global__ void __launch_bounds__(256) gather_mean_kernel(const uint4* __restrict__ src,
                                                          uint4* __restrict__ dst,
                                                          const int32_t* __restrict__ sort_token,
                                                          const int32_t* __restrict__ count,
                                                          const int32_t* __restrict__ off, int C,
                                                          int S, int H, float* __restrict__ mean) {
  constexpr int EPV = 16 / sizeof(T);   // elements per vector
  constexpr int RPW = 32 / VPR;         // rows per warp pass
  constexpr int SLOTS = 8 * RPW;        // row slots of the CTA
  constexpr int D = VPR * EPV;
  __shared__ float part[SLOTS][D];
  const int c = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t bh = static_cast<int64_t>(blockIdx.z) * H + blockIdx.y;
  const int n = count[c], o = off[c];
  const int slot = warp * RPW + lane / VPR, vi = lane % VPR;
  float acc[EPV];
#pragma unroll
  for (int e = 0; e < EPV; ++e) acc[e] = 0.f;
  for (int r0 = slot; r0 < n; r0 += 4 * SLOTS) {
    int tok[4];
    uint4 u[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int rr = r0 + j * SLOTS;
      tok[j] = rr < n ? __ldg(sort_token + o + rr) : -1;
    }
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (tok[j] >= 0) u[j] = __ldg(src + (bh * S + tok[j]) * VPR + vi);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (tok[j] < 0) continue;
      float f[EPV];
      unpack16<T>(u[j], f);
#pragma unroll
      for (int e = 0; e < EPV; ++e) acc[e] += f[e];
      if (dst) dst[(bh * S + o + r0 + j * SLOTS) * VPR + vi] = u[j];
    }
  }
#pragma unroll
  for (int e = 0; e < EPV; ++e) part[slot][vi * EPV + e] = acc[e];
  __syncthreads();
  const float inv = n > 0 ? 1.f / static_cast<float>(n) : 0.f;
  for (int d = tid; d < D; d += 256) {
    float t = 0.f;
#pragma unroll
    for (int k = 0; k < SLOTS; ++k) t += part[k][d];
    mean[(bh * C + c) * D + d] = t * inv;
  }
}

template <typename T>
void launch_gather_mean(const void* src, void* dst, const int32_t* tok, const int32_t* cnt,
                        const int32_t* off, int C, int S, int H, int B, int D, float* mean,
                        cudaStream_t st) {
  const dim3 g(C, H, B);
  const uint4* s4 = static_cast<const uint4*>(src);
  uint4* d4 = static_cast<uint4*>(dst);
  const int vpr = D * static_cast<int>(sizeof(T)) / 16;
  if (vpr == 8) gather_mean_kernel<T, 8><<<g, 256, 0, st>>>(s4, d4, tok, cnt, off, C, S, H, mean);
  else if (vpr == 16) gather_mean_kernel<T, 16><<<g, 256, 0, st>>>(s4, d4, tok, cnt, off, C, S, H, mean);
  else gather_mean_kernel<T, 32><<<g, 256, 0, st>>>(s4, d4, tok, cnt, off, C, S, H, mean);
  count_launch();
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

// ---------------------------------------------------------------- probe errors, tensor cores
// bf16 keys and values. The two sums per (probe, key) of the error above, the logit
// q̄_a . k_j and the weighted value sum over a cluster's keys, are dense contractions:
// S = Q̄ Kᵀ over a piece of up to 128 keys of one cluster, then E += P V over the same
// keys, on tcgen05 with fp32 accumulators in TMEM. Both bf16 operands that are not
// exact in bf16 are carried as a high and a low bf16 part (x = hi + lo to about 16
// mantissa bits; keys and values are bf16 already): Q̄ = q̄ scale log2(e) is split once
// per CTA, the weights w = 2^(s - m) once per piece, and each K-step issues one MMA per
// part, so logits and sums keep close to fp32 precision.
//
// One CTA (one per SM: 512 TMEM columns, ~205 KB of shared memory) takes 128 probes of
// one head and a range of key clusters (balanced by keys); clusters are cut into pieces
// of at most 128 keys. 288 threads: warp 0 issues the TMA copies (double-buffered K and
// V stages) and the MMAs; warps 1..8 hold each probe as a pair of threads (one per half
// of a piece's key columns and of E's dims). TMEM columns: S/P of pieces i even / odd
// at 0 / 128 (P's high part over S columns 0..63, low part over 64..127), E of
// clusters k even / odd at 256 / 384. The MMA order is QK(i+1), PV(i),
// QK(i+2), ..., so the next piece's logits are computed while the softmax threads take
// the weights of this one. Per cluster the running reference m starts at the centroid
// logit and follows the largest logit seen (E rescaled in TMEM when a later piece
// raises it); after the cluster's last piece the softmax threads read E and store
// || E - n_c 2^(lc - m) v̄_c ||, m and the weight sum z of the cluster (all in log2
// units), one piece later so that its PV runs meanwhile. route_finish_kernel brings the
// clusters of a probe to one reference and divides by the dense sum.
struct RouteTcArgs {
  int B, Hq, Hkv, S, Cq, Ck, nsplit;
  float scale_log2;       // scale * log2(e)
  const float* qbar;      // (B, Hq, Cq, D)
  const float* lc;        // (B, Hq, Cq, Ck): scale_log2 * q̄_a . k̄_c
  const float* vbar;      // (B, Hkv, Ck, D)
  const int32_t* q_count;
  const int32_t* k_count;
  const int32_t* k_off;   // Ck + 1 offsets into the cluster-major key rows
  float* err;             // (B, Hq, Cq, Ck): || E - A || against reference mref
  float* mref;            // (B, Hq, Cq, Ck)
  float* zc;              // (B, Hq, Cq, Ck): sum of the cluster's weights against mref
};

// Tile (x, y) of a 2-D tensor map into L2 only (no shared memory, no barrier).
__device__ __forceinline__ void tma_prefetch_l2_2d(const void* tmap, int x, int y) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(tmap), "r"(x),
               "r"(y)
               : "memory");
}

// Pieces of the non-empty clusters in [c, c_hi), in order; k counts the clusters. Run by
// a whole warp on warp-uniform values: the lanes hold the counts and offsets of a window
// of 32 consecutive clusters (one coalesced load each), so finding the next non-empty
// cluster is a ballot rather than a chain of dependent loads.
struct RtIter {
  int c, c_hi, p, nc, off, k;
  int wbase, wcnt, woff;  // window [wbase, wbase + 32): this lane's cluster wbase + lane
  __device__ __forceinline__ void seek(const int32_t* cnt, const int32_t* offs) {
    const int lane = threadIdx.x & 31;
    while (c < c_hi) {
      if (c < wbase || c >= wbase + 32) {
        wbase = c;
        const int cc = c + lane;
        wcnt = cc < c_hi ? __ldg(cnt + cc) : 0;
        woff = cc < c_hi ? __ldg(offs + cc) : 0;
      }
      const uint32_t nz = __ballot_sync(0xffffffffu, wcnt > 0) & (0xffffffffu << (c - wbase));
      if (nz) {
        const int j = __ffs(nz) - 1;
        c = wbase + j;
        nc = __shfl_sync(0xffffffffu, wcnt, j);
        off = __shfl_sync(0xffffffffu, woff, j);
        return;
      }
      c = wbase + 32;
    }
  }
  __device__ __forceinline__ void init(int lo, int hi, const int32_t* cnt, const int32_t* offs) {
    c = lo;
    c_hi = hi;
    p = 0;
    k = 0;
    nc = 0;
    off = 0;
    wbase = -64;
    wcnt = woff = 0;
    seek(cnt, offs);
  }
  __device__ __forceinline__ void advance(const int32_t* cnt, const int32_t* offs) {
    if (++p * 128 >= nc) {
      p = 0;
      ++c;
      ++k;
      seek(cnt, offs);
    }
  }
  __device__ __forceinline__ bool valid() const { return c < c_hi; }
  __device__ __forceinline__ int n() const { return min(128, nc - 128 * p); }
  __device__ __forceinline__ int row() const { return off + 128 * p; }
  __device__ __forceinline__ bool first() const { return p == 0; }
  __device__ __forceinline__ bool last() const { return (p + 1) * 128 >= nc; }
};

enum {
  RT_QR = 0, RT_KF0, RT_KF1, RT_KE0, RT_KE1, RT_VF0, RT_VF1, RT_VE0, RT_VE1, RT_SF0, RT_SF1,
  RT_PF0, RT_PF1, RT_OF0, RT_OF1, RT_OE0, RT_OE1, RT_XB0, RT_XB1, RT_XE, RT_DRAIN, RT_NBAR
};

template <int D>
struct RouteTcCfg {
  static constexpr int NATOM = D / 64;        // 128-byte column chunks of a bf16 row
  static constexpr int TILE = 128 * D * 2;    // one 128-row bf16 operand tile
  static constexpr int SMEM = 6 * TILE + 1024 + 8192;  // tiles, alignment, barriers + exchange
};

// First cluster of key-balanced range `split` of nsplit (offsets are non-decreasing).
__device__ __forceinline__ int route_range_start(const int32_t* off, int Ck, int S, int split,
                                                 int nsplit) {
  if (split <= 0) return 0;
  if (split >= nsplit) return Ck;
  const int target = static_cast<int>((static_cast<int64_t>(S) * split) / nsplit);
  int lo = 0, hi = Ck;  // first c with off[c] >= target
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(off + mid) < target) lo = mid + 1;
    else hi = mid;
  }
  return lo;
}

template <int D>
__global__ void __launch_bounds__(288, 1)
    route_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                    const RouteTcArgs a) {
  using Cfg = RouteTcCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sQh = smem_u32(smem), sQl = sQh + Cfg::TILE;
  const uint32_t sK = sQh + 2 * Cfg::TILE, sV = sQh + 4 * Cfg::TILE;  // two stages each
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + 6 * Cfg::TILE);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + RT_NBAR);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* never = reinterpret_cast<int*>(tmem_slot + 2);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // the probe tiles of one key range are neighbours in the grid, so they run together
  // and share the range's K and V through L2
  const int tiles = (a.Cq + 127) / 128;
  const int tile = blockIdx.x % tiles, split = blockIdx.x / tiles;
  const int h = blockIdx.y, b = blockIdx.z;
  const int hkv = h / (a.Hq / a.Hkv);
  const int64_t bq = static_cast<int64_t>(b) * a.Hq + h;
  const int64_t bk = static_cast<int64_t>(b) * a.Hkv + hkv;
  const int a0 = tile * 128;
  const int c_lo = route_range_start(a.k_off, a.Ck, a.S, split, a.nsplit);
  const int c_hi = route_range_start(a.k_off, a.Ck, a.S, split + 1, a.nsplit);
  const uint32_t bar0 = smem_u32(bars);
#define RBAR(i) (bar0 + 8u * static_cast<uint32_t>(i))
  if (tid == 0) {
    for (int i = 0; i < RT_NBAR; ++i)
      mbar_init(RBAR(i), (i == RT_QR || i == RT_PF0 || i == RT_PF1 || i == RT_OE0 || i == RT_OE1 ||
                          i == RT_XB0 || i == RT_XB1 || i == RT_XE)
                             ? 8u   // one arrival per softmax warp
                             : 1u);
    *abort_flag = 0;
    *never = 0;
    fence_mbarrier_init();
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------ control warp: TMA + tcgen05.mma
    const bool leader = lane == 0;
    auto wait_all = [&](uint32_t bar, uint32_t parity, int where) -> bool {
      const bool r = mbar_wait(bar, parity, abort_flag, where);
      return __all_sync(0xffffffffu, r);
    };
    auto commit = [&](uint32_t bar) {
      if (elect_one()) tc_commit(bar);
      __syncwarp();
    };
    constexpr uint32_t kIdescQK = make_idesc(false, 128, 0, false, false);
    constexpr uint32_t kIdescPV = make_idesc(false, 128, D, false, true);
    const uint64_t dQh = smem_desc(sQh, 16, 1024), dQl = smem_desc(sQl, 16, 1024);
    const int grow0 = static_cast<int>(bk * a.S);
    int lk0 = 0, lk1 = 0, lv0 = 0, lv1 = 0;  // copies issued into each K / V stage
    auto load = [&](bool is_v, int stage, int row) {
      if (leader) {
        const uint32_t bar = RBAR((is_v ? RT_VF0 : RT_KF0) + stage);
        const uint32_t dst = (is_v ? sV : sK) + stage * Cfg::TILE;
        mbar_arrive_expect_tx(bar, Cfg::TILE);
#pragma unroll
        for (int cc = 0; cc < Cfg::NATOM; ++cc)
          tma_load_2d(dst + cc * 16384, is_v ? &tmV : &tmK, bar, cc * 64, grow0 + row);
      }
      __syncwarp();
      if (is_v) (stage ? lv1 : lv0) += 1;
      else (stage ? lk1 : lk0) += 1;
    };
    // S[stage] = Q̄_hi Kᵀ + Q̄_lo Kᵀ over the piece's n16 key columns
    auto issue_qk = [&](int stage, int n) {
      const uint32_t n16 = static_cast<uint32_t>((n + 15) & ~15);
      const uint32_t idesc = kIdescQK | ((n16 >> 3) << 17);
      const uint64_t dK = smem_desc(sK + stage * Cfg::TILE, 16, 1024);
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t off = static_cast<uint64_t>(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4);
          mma_ss<false>(tmem + 128 * stage, dQh + off, dK + off, idesc, kk > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t off = static_cast<uint64_t>(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4);
          mma_ss<false>(tmem + 128 * stage, dQl + off, dK + off, idesc, 1u);
        }
      }
      __syncwarp();
    };
    // E[o] (+)= P_hi V + P_lo V over the piece's keys, 16 per K-step
    auto issue_pv = [&](int stage, int o, int n, bool first) {
      const int nst = (n + 15) >> 4;
      const uint64_t dV = smem_desc(sV + stage * Cfg::TILE, 16384, 1024, kLayoutSW128);
      const uint32_t tE = tmem + 256 + 128 * o, tP = tmem + 128 * stage;
      if (elect_one()) {
        for (int t = 0; t < nst; ++t) {
          const uint64_t bv = dV + static_cast<uint64_t>((t * 16 * 128) >> 4);
          mma_ts<false>(tE, tP + 8 * t, bv, kIdescPV, (first && t == 0) ? 0u : 1u);
          mma_ts<false>(tE, tP + 64 + 8 * t, bv, kIdescPV, 1u);
        }
      }
      __syncwarp();
    };
    RtIter it;
    it.init(c_lo, c_hi, a.k_count, a.k_off);
    bool ok = true;
    if (it.valid()) {
      load(false, 0, it.row());
      load(true, 0, it.row());
      RtIter n1 = it;
      n1.advance(a.k_count, a.k_off);
      if (n1.valid()) load(false, 1, n1.row());
      ok = wait_all(RBAR(RT_QR), 0, 40) && wait_all(RBAR(RT_KF0), 0, 41);
      if (ok) {
        tc_fence_after();
        issue_qk(0, it.n());
        commit(RBAR(RT_SF0));
        commit(RBAR(RT_KE0));
      }
    }
    int i = 0;
    while (ok && it.valid()) {
      const int s = i & 1, s1 = s ^ 1;
      RtIter nx = it;
      nx.advance(a.k_count, a.k_off);
      if (nx.valid()) {
        // the next piece's logits go first, so they are ready when this softmax ends
        if (!(ok = wait_all(RBAR(RT_KF0 + s1), ((i + 1) >> 1) & 1, 42))) break;
        tc_fence_after();
        issue_qk(s1, nx.n());
        commit(RBAR(RT_SF0 + s1));
        commit(RBAR(RT_KE0 + s1));
        // K of piece i + 2 as soon as QK(i) has read its stage (it has, or nearly: the
        // softmax of piece i started from it), a whole softmax ahead of its QK
        RtIter nn = nx;
        nn.advance(a.k_count, a.k_off);
        if (nn.valid()) {
          if (!(ok = wait_all(RBAR(RT_KE0 + s), (i >> 1) & 1, 47))) break;
          load(false, s, nn.row());
          // K and V of piece i + 4 into L2, two pieces ahead of their copies
          RtIter n4 = nn;
          n4.advance(a.k_count, a.k_off);
          if (n4.valid()) n4.advance(a.k_count, a.k_off);
          if (n4.valid() && leader) {
#pragma unroll
            for (int cc = 0; cc < Cfg::NATOM; ++cc) {
              tma_prefetch_l2_2d(&tmK, cc * 64, grow0 + n4.row());
              tma_prefetch_l2_2d(&tmV, cc * 64, grow0 + n4.row());
            }
          }
          __syncwarp();
        }
        // V of piece i + 1: its stage was last read by PV(i - 1)
        if (i >= 1 && !(ok = wait_all(RBAR(RT_VE0 + s1), ((i - 1) >> 1) & 1, 43))) break;
        load(true, s1, nx.row());
      }
      if (!(ok = wait_all(RBAR(RT_PF0 + s), (i >> 1) & 1, 44))) break;
      // a cluster's first PV overwrites its E buffer: the epilogue of cluster k - 2 is done
      if (it.first() && it.k >= 2 &&
          !(ok = wait_all(RBAR(RT_OE0 + (it.k & 1)), ((it.k - 2) >> 1) & 1, 45)))
        break;
      if (!(ok = wait_all(RBAR(RT_VF0 + s), (i >> 1) & 1, 46))) break;
      tc_fence_after();
      issue_pv(s, it.k & 1, it.n(), it.first());
      commit(RBAR(RT_VE0 + s));
      if (it.last()) commit(RBAR(RT_OF0 + (it.k & 1)));
      it = nx;
      ++i;
    }
    // Before the CTA may exit: every MMA has completed and every issued copy has landed.
    commit(RBAR(RT_DRAIN));
    mbar_wait(RBAR(RT_DRAIN), 0, never, 48);
    if (lk0) mbar_wait(RBAR(RT_KF0), (lk0 - 1) & 1, never, 49);
    if (lk1) mbar_wait(RBAR(RT_KF1), (lk1 - 1) & 1, never, 49);
    if (lv0) mbar_wait(RBAR(RT_VF0), (lv0 - 1) & 1, never, 49);
    if (lv1) mbar_wait(RBAR(RT_VF1), (lv1 - 1) & 1, never, 49);
  } else {
    // ------------------------------------------------ softmax / epilogue (256 threads)
    // Two threads per probe: warps 1..4 take key columns 0..63 of each piece and E's
    // first half of dims, warps 5..8 columns 64..127 and the second half (warp w reads
    // TMEM lanes 32*(w%4)..+31). The pair exchanges its piece maxima, and at a cluster's
    // end its halves of the error and of the weight sum, through shared memory, each
    // exchange closed by an mbarrier (bounded waits). Every hand-off is one arrival per
    // warp: the lanes fence their own stores, meet at __syncwarp, and lane 0 arrives.
    constexpr int DH = D / 2;  // E columns per thread
    const int quarter = warp & 3, hh = (warp - 1) >> 2;
    const int r = quarter * 32 + lane;
    const int pa = a0 + r;  // this thread's probe (query cluster)
    const bool live = pa < a.Cq;
    const uint32_t lanes = static_cast<uint32_t>(quarter * 32) << 16;
    float* xmax = reinterpret_cast<float*>(tmem_slot + 4);   // [2 parity][2 halves][128]
    float* xe2 = xmax + 2 * 2 * 128;                         // [2 halves][128]
    float* xz = xe2 + 2 * 128;                               // [2 halves][128]
    // Q̄ rows, high and low bf16 parts, into the K-major 128-byte-swizzled tiles (each
    // thread of the pair writes half of the row's 16-byte chunks)
    {
      const float* qrow = a.qbar + (bq * a.Cq + (live ? pa : 0)) * D;
#pragma unroll
      for (int j = 0; j < Cfg::NATOM * 4; ++j) {
        const int g = hh * Cfg::NATOM * 4 + j;  // 16-byte chunk of the row (8 elements)
        const int cc = g >> 3, ch = g & 7;
        float x[8];
        if (live) {
          const float4 u0 = __ldg(reinterpret_cast<const float4*>(qrow + g * 8));
          const float4 u1 = __ldg(reinterpret_cast<const float4*>(qrow + g * 8 + 4));
          x[0] = u0.x; x[1] = u0.y; x[2] = u0.z; x[3] = u0.w;
          x[4] = u1.x; x[5] = u1.y; x[6] = u1.z; x[7] = u1.w;
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) x[e] = 0.f;
        }
        uint32_t hw[4], lw[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float x0 = x[2 * e] * a.scale_log2, x1 = x[2 * e + 1] * a.scale_log2;
          const __nv_bfloat162 hb = __floats2bfloat162_rn(x0, x1);
          const float2 hf = __bfloat1622float2(hb);
          hw[e] = *reinterpret_cast<const uint32_t*>(&hb);
          lw[e] = pack_bf16x2(x0 - hf.x, x1 - hf.y);
        }
        const uint32_t off = cc * 16384 + r * 128 + ((ch ^ (r & 7)) << 4);
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(sQh + off), "r"(hw[0]),
                     "r"(hw[1]), "r"(hw[2]), "r"(hw[3]) : "memory");
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(sQl + off), "r"(lw[0]),
                     "r"(lw[1]), "r"(lw[2]), "r"(lw[3]) : "memory");
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(RBAR(RT_QR));
    }
    auto warp_arrive = [&](uint32_t bar) {
      __syncwarp();
      if (lane == 0) mbar_arrive(bar);
    };
    // waits are warp-uniform: the iterator's ballots need every lane of the warp
    auto wait_w = [&](uint32_t bar, uint32_t parity, int where) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, where));
    };
    const float* lc_row = a.lc + (bq * a.Cq + (live ? pa : 0)) * a.Ck;
    const int64_t out_row = (bq * a.Cq + (live ? pa : 0)) * a.Ck;
    bool ok = true;
    // the cluster whose E is still to be read: ordinal, index, count, m, z, lc
    bool pend = false;
    int pk = 0, pc = 0, pn = 0, ne = 0;  // ne: epilogues done
    float pm = 0.f, pz = 0.f, plc = 0.f;
    auto epilogue = [&]() -> bool {
      // v̄_c (this thread's half; prefetched into L1 when the cluster started)
      const float4* vb = reinterpret_cast<const float4*>(a.vbar + (bk * a.Ck + pc) * D + hh * DH);
      if (!wait_w(RBAR(RT_OF0 + (pk & 1)), (pk >> 1) & 1, 50)) return false;
      tc_fence_after();
      const float wc = static_cast<float>(pn) * ex2(plc - pm);
      const uint32_t tE = tmem + lanes + 256 + 128 * (pk & 1) + hh * DH;
      float e2a = 0.f, e2b = 0.f;
#pragma unroll
      for (int q = 0; q < DH / 32; ++q) {
        float o[32];
        tmem_ld32(tE + 32 * q, o);
        tmem_wait_ld();
#pragma unroll
        for (int c4 = 0; c4 < 8; ++c4) {
          const float4 v4 = __ldg(vb + 8 * q + c4);
          const float d0 = fmaf(-wc, v4.x, o[4 * c4]), d1 = fmaf(-wc, v4.y, o[4 * c4 + 1]);
          const float d2 = fmaf(-wc, v4.z, o[4 * c4 + 2]), d3 = fmaf(-wc, v4.w, o[4 * c4 + 3]);
          e2a = fmaf(d0, d0, fmaf(d1, d1, e2a));
          e2b = fmaf(d2, d2, fmaf(d3, d3, e2b));
        }
      }
      tc_fence_before();
      xe2[hh * 128 + r] = e2a + e2b;
      xz[hh * 128 + r] = pz;
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(RBAR(RT_OE0 + (pk & 1)));
        mbar_arrive(RBAR(RT_XE));
      }
      if (!wait_w(RBAR(RT_XE), ne & 1, 53)) return false;
      ++ne;
      if (live && hh == 0) {
        a.err[out_row + pc] = sqrtf(xe2[r] + xe2[128 + r]);
        a.mref[out_row + pc] = pm;
        a.zc[out_row + pc] = xz[r] + xz[128 + r];
      }
      pend = false;
      return true;
    };
    RtIter it;
    it.init(c_lo, c_hi, a.k_count, a.k_off);
    float m = 0.f, z = 0.f, lc2 = 0.f;
    int i = 0;
#pragma unroll 1
    while (it.valid()) {
      const int s = i & 1;
      const int nh = min(64, it.n() - 64 * hh);  // this thread's key columns (may be <= 0)
      if (it.first()) {
        lc2 = live ? __ldg(lc_row + it.c) : 0.f;
        m = lc2;
        z = 0.f;
        const float* vh = a.vbar + (bk * a.Ck + it.c) * D + hh * DH;
#pragma unroll
        for (int j = 0; j < DH; j += 32)
          asm volatile("prefetch.global.L1 [%0];" ::"l"(vh + j));
      }
      if (!(ok = wait_w(RBAR(RT_SF0 + s), (i >> 1) & 1, 51))) break;
      tc_fence_after();
      const uint32_t tS = tmem + lanes + 128 * s;
      float v[2][32];
#pragma unroll
      for (int q = 0; q < 2; ++q)
        if (32 * q < nh) tmem_ld32(tS + 64 * hh + 32 * q, v[q]);
      tmem_wait_ld();
      float mx = -INFINITY;
#pragma unroll
      for (int q = 0; q < 2; ++q)
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          v[q][c] = 32 * q + c < nh ? v[q][c] : -INFINITY;
          mx = fmaxf(mx, v[q][c]);
        }
      // (the exchange also orders both threads' S loads before either's P stores, which
      // overlap the partner's S columns)
      xmax[(s * 2 + hh) * 128 + r] = mx;
      tc_fence_before();
      warp_arrive(RBAR(RT_XB0 + s));
      if (!(ok = wait_w(RBAR(RT_XB0 + s), (i >> 1) & 1, 54))) break;
      tc_fence_after();
      mx = fmaxf(mx, xmax[(s * 2 + (hh ^ 1)) * 128 + r]);
      const bool need = mx > m;
      float alpha = 1.f;
      if (need) {
        alpha = ex2(m - mx);
        z *= alpha;
        m = mx;
      }
      if (!it.first() && __any_sync(0xffffffffu, need)) {
        // E holds this cluster's earlier pieces against the old reference: wait for
        // PV(i - 1), then scale this thread's half of it
        if (!(ok = wait_w(RBAR(RT_VE0 + (s ^ 1)), ((i - 1) >> 1) & 1, 52))) break;
        tc_fence_after();
        const uint32_t tE = tmem + lanes + 256 + 128 * (it.k & 1) + hh * DH;
#pragma unroll 1
        for (int q = 0; q < DH / 32; ++q) {
          float o[32];
          tmem_ld32(tE + 32 * q, o);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] *= alpha;
          tmem_st32(tE + 32 * q, *reinterpret_cast<uint32_t(*)[32]>(o));
        }
      }
      // weights, their sum, and the high / low bf16 parts over S
      float za = 0.f, zb = 0.f;
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        if (32 * q < nh) {
          uint32_t hw[16], lw[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float w0 = ex2(v[q][2 * e] - m), w1 = ex2(v[q][2 * e + 1] - m);
            za += w0;
            zb += w1;
            const __nv_bfloat162 hb = __floats2bfloat162_rn(w0, w1);
            const float2 hf = __bfloat1622float2(hb);
            hw[e] = *reinterpret_cast<const uint32_t*>(&hb);
            lw[e] = pack_bf16x2(w0 - hf.x, w1 - hf.y);
          }
          tmem_st16(tS + 32 * hh + 16 * q, hw);
          tmem_st16(tS + 64 + 32 * hh + 16 * q, lw);
        }
      }
      z += za + zb;
      tmem_wait_st();
      tc_fence_before();
      warp_arrive(RBAR(RT_PF0 + s));
      // the previous cluster's E: its last PV was issued before this piece's
      if (pend && !(ok = epilogue())) break;
      if (it.last()) {
        pend = true;
        pk = it.k;
        pc = it.c;
        pn = it.nc;
        pm = m;
        pz = z;
        plc = lc2;
      }
      it.advance(a.k_count, a.k_off);
      ++i;
    }
    if (ok && pend) epilogue();
  }
#undef RBAR
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// grid (ceil(Cq / 32), Hq, B), 256 threads: lc[b,h,a,c] = scale_log2 * q̄_a . k̄_c (fp32)
// for 32 probes a per CTA; thread c streams k̄_c once (float4) against the 32 probe rows
// held in shared memory (broadcast reads).
constexpr int kLcProbes = 32;
template <int D>
__global__ void __launch_bounds__(256) centroid_logit_kernel(const float* __restrict__ qbar,
                                                             const float* __restrict__ kbar,
                                                             int Hq, int Hkv, int Cq, int Ck,
                                                             float scale_log2,
                                                             float* __restrict__ lc) {
  __shared__ __align__(16) float qa[kLcProbes][D];
  const int a0 = blockIdx.x * kLcProbes, h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const int hkv = h / (Hq / Hkv);
  const int64_t bq = static_cast<int64_t>(b) * Hq + h;
  const int64_t bk = static_cast<int64_t>(b) * Hkv + hkv;
  const int np = min(kLcProbes, Cq - a0);
  for (int e = tid; e < kLcProbes * D; e += 256) {
    const int p = e / D, d = e % D;
    qa[p][d] = p < np ? qbar[(bq * Cq + a0 + p) * D + d] : 0.f;
  }
  __syncthreads();
  for (int c = tid; c < Ck; c += 256) {
    const float4* kc = reinterpret_cast<const float4*>(kbar + (bk * Ck + c) * D);
    float acc[kLcProbes];
#pragma unroll
    for (int p = 0; p < kLcProbes; ++p) acc[p] = 0.f;
#pragma unroll 2
    for (int d4 = 0; d4 < D / 4; ++d4) {
      const float4 k4 = __ldg(kc + d4);
#pragma unroll
      for (int p = 0; p < kLcProbes; ++p) {
        const float4 q4 = *reinterpret_cast<const float4*>(&qa[p][4 * d4]);
        acc[p] = fmaf(q4.x, k4.x, fmaf(q4.y, k4.y, fmaf(q4.z, k4.z, fmaf(q4.w, k4.w, acc[p]))));
      }
    }
#pragma unroll
    for (int p = 0; p < kLcProbes; ++p)
      if (p < np) lc[(bq * Cq + a0 + p) * Ck + c] = scale_log2 * acc[p];
  }
}

// One warp per (batch, head, probe) row: M = max_c mref, Z = sum_c zc 2^(mref - M) over
// the non-empty key clusters; err <- err 2^(mref - M) / Z (0 for an empty probe or key
// cluster, or Z = 0).
__global__ void __launch_bounds__(256) route_finish_kernel(const int32_t* __restrict__ q_count,
                                                           const int32_t* __restrict__ k_count,
                                                           int Cq, int Ck, int64_t rows,
                                                           const float* __restrict__ mref,
                                                           const float* __restrict__ zc,
                                                           float* __restrict__ err) {
  const int lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int pa = static_cast<int>(row % Cq);
  const float* mr = mref + row * Ck;
  const float* zr = zc + row * Ck;
  float* er = err + row * Ck;
  float M = -INFINITY;
  for (int c = lane; c < Ck; c += 32)
    if (__ldg(k_count + c) > 0) M = fmaxf(M, mr[c]);
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  float Z = 0.f;
  if (M > -INFINITY)
    for (int c = lane; c < Ck; c += 32)
      if (__ldg(k_count + c) > 0) Z += zr[c] * ex2(mr[c] - M);
  for (int o = 16; o > 0; o >>= 1) Z += __shfl_xor_sync(0xffffffffu, Z, o);
  const bool qok = __ldg(q_count + pa) > 0 && Z > 0.f;
  const float invZ = qok ? 1.f / Z : 0.f;
  for (int c = lane; c < Ck; c += 32) {
    const bool ok = qok && __ldg(k_count + c) > 0;
    er[c] = ok ? er[c] * ex2(mr[c] - M) * invZ : 0.f;
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
  float *qbar, *kbar, *vbar, *err, *mref, *lc, *zc;
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
  L.lc = cv.take<float>(static_cast<size_t>(s.B) * s.Hq * Cq * Ck);
  L.zc = cv.take<float>(static_cast<size_t>(s.B) * s.Hq * Cq * Ck);
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
  if (static_cast<int64_t>(s.B) * s.Hkv * s.Sk >= (int64_t(1) << 31))
    return fail(BSA_ERR_UNSUPPORTED, "B * Hkv * Sk = %lld key rows exceeds 2^31 - 1",
                static_cast<long long>(s.B) * s.Hkv * s.Sk);
  return BSA_OK;
}

// Probe errors of bf16 keys and values on the tensor cores: centroid logits, the probe
// kernel over key-balanced cluster ranges, and the common-reference normalisation.
template <int D>
int launch_route_tc(const RouteLayout& L, const bsa_shape& s, int Cq, int Ck, float scale,
                    float* err, cudaStream_t st) {
  int rc;
  const float scale_log2 = scale * 1.4426950408889634f;
  centroid_logit_kernel<D><<<dim3((Cq + kLcProbes - 1) / kLcProbes, s.Hq, s.B), 256, 0, st>>>(
      L.qbar, L.kbar, s.Hq, s.Hkv, Cq, Ck, scale_log2, L.lc);
  count_launch();
  if ((rc = check_cuda(cudaGetLastError(), "centroid_logit_kernel"))) return rc;
  CUtensorMap mk, mv;
  const uint64_t rows = static_cast<uint64_t>(s.B) * s.Hkv * s.Sk;
  if ((rc = make_tmap_2d(&mk, L.kp, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, rows, s.D, 128, 64)) ||
      (rc = make_tmap_2d(&mv, L.vp, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, rows, s.D, 128, 64)))
    return rc;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // one CTA per SM: split the key clusters so that the grid fills whole waves best
  const int tiles = (Cq + 127) / 128;
  const int64_t units = static_cast<int64_t>(tiles) * s.Hq * s.B;
  int nsplit = 1;
  double best = -1.0;
  const int lo = static_cast<int>(std::max<int64_t>(1, (2 * sms + units - 1) / units));
  for (int n = lo; n <= 2 * lo && n <= Ck; ++n) {
    const int64_t ctas = units * n;
    const double fill = static_cast<double>(ctas) / (static_cast<double>((ctas + sms - 1) / sms) * sms);
    if (fill > best + 1e-9) {
      best = fill;
      nsplit = n;
    }
  }
  if (nsplit > Ck) nsplit = Ck;
  if (units * nsplit > 0x7fffffffLL || static_cast<int64_t>(tiles) * nsplit > 0x7fffffffLL)
    return fail(BSA_ERR_UNSUPPORTED, "routing grid too large");
  RouteTcArgs ta{};
  ta.B = s.B;
  ta.Hq = s.Hq;
  ta.Hkv = s.Hkv;
  ta.S = s.Sk;
  ta.Cq = Cq;
  ta.Ck = Ck;
  ta.nsplit = nsplit;
  ta.scale_log2 = scale_log2;
  ta.qbar = L.qbar;
  ta.lc = L.lc;
  ta.vbar = L.vbar;
  ta.q_count = L.q_count;
  ta.k_count = L.k_count;
  ta.k_off = L.k_off;
  ta.err = err;
  ta.mref = L.mref;
  ta.zc = L.zc;
  auto kern = route_tc_kernel<D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       RouteTcCfg<D>::SMEM);
  if (e != cudaSuccess) return check_cuda(e, "cudaFuncSetAttribute(route_tc_kernel)");
  kern<<<dim3(tiles * nsplit, s.Hq, s.B), 288, RouteTcCfg<D>::SMEM, st>>>(mk, mv, ta);
  count_launch();
  if ((rc = check_cuda(cudaGetLastError(), "route_tc_kernel"))) return rc;
  const int64_t nrows = static_cast<int64_t>(s.B) * s.Hq * Cq;
  route_finish_kernel<<<static_cast<unsigned>((nrows + 7) / 8), 256, 0, st>>>(
      L.q_count, L.k_count, Cq, Ck, nrows, L.mref, L.zc, err);
  count_launch();
  return check_cuda(cudaGetLastError(), "route_finish_kernel");
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
  // 2. cluster means of Q (probes), K and V (centroids), fp32; for the probe errors K and
  // V are gathered into cluster-major order in the same pass
  const bool with_v = M < 0;
  if (s.dtype == BSA_F32) {
    launch_gather_mean<float>(q, nullptr, L.q_tok, L.q_count, L.q_off, Cq, s.Sq, s.Hq, s.B, s.D,
                              L.qbar, st);
    launch_gather_mean<float>(k, with_v ? L.kp : nullptr, L.k_tok, L.k_count, L.k_off, Ck, s.Sk,
                              s.Hkv, s.B, s.D, L.kbar, st);
    if (with_v)
      launch_gather_mean<float>(v, L.vp, L.k_tok, L.k_count, L.k_off, Ck, s.Sk, s.Hkv, s.B, s.D,
                                L.vbar, st);
  } else {
    using bf = __nv_bfloat16;
    launch_gather_mean<bf>(q, nullptr, L.q_tok, L.q_count, L.q_off, Cq, s.Sq, s.Hq, s.B, s.D,
                           L.qbar, st);
    launch_gather_mean<bf>(k, with_v ? L.kp : nullptr, L.k_tok, L.k_count, L.k_off, Ck, s.Sk,
                           s.Hkv, s.B, s.D, L.kbar, st);
    if (with_v)
      launch_gather_mean<bf>(v, L.vp, L.k_tok, L.k_count, L.k_off, Ck, s.Sk, s.Hkv, s.B, s.D,
                             L.vbar, st);
  }
  if ((rc = check_cuda(cudaGetLastError(), "gather_mean_kernel"))) return rc;
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
    // keys and values are in cluster-major order (rows off[c] .. off[c] + n_c per head)
    if (s.dtype == BSA_F32) {
      if (s.D == 64) launch_route_probe<float, 64>(L.kp, L.vp, ra, st);
      else launch_route_probe<float, 128>(L.kp, L.vp, ra, st);
    } else {
      rc = s.D == 64 ? launch_route_tc<64>(L, s, Cq, Ck, ra.scale, ra.err, st)
                     : launch_route_tc<128>(L, s, Cq, Ck, ra.scale, ra.err, st);
      if (rc) return rc;
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
  if (!(with_v && s.dtype != BSA_F32)) {  // the tensor-core path counts and checks its own
    count_launch();
    if ((rc = check_cuda(cudaGetLastError(), "route score kernel"))) return rc;
  }
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
