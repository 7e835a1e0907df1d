// HEART temporal mask reuse: per-head drift/anchor mask cache.
//
// Source: "Dynamic block masks and head-wise mask reuse" (mlx-arsenal notes), §HEART —
// head-wise temporal mask reuse (per head an anchor: the token means q̄, k̄ at the step
// its mask was last built, and that mask; drift ‖q̄_anchor − q̄_t‖₁ + ‖k̄_anchor − k̄_t‖₁;
// rebuild above a global delta, else reuse; a layer-level override refreshes nothing
// under 40 % of the heads and everything above 80 %), §What mlx-arsenal ships
// (pooled_qk, qk_drift, HeadMaskCache), §Recipe (all heads refresh on the first
// call), §Deviations (relative drift divides by the anchor's L1 norm), "Reuse needs a
// fixed token grid" (reset on a grid change).
//
// The whole state is one caller-owned device buffer (header, anchors, pending pooled
// means, cached mask, pooling partials), so it can be saved and restored as bytes.
#include <cuda_bf16.h>

#include "common.cuh"
#include "ptx.cuh"

namespace bsa {

constexpr int kPoolSplit = 32;

struct CacheHeader {
  int B, H, Cq, Ck, D;
  int has_anchor;
  float delta;
  int relative;
  float gate_lo, gate_hi;
  int n_refresh;
  int magic;
  int pad[4];
};
static_assert(sizeof(CacheHeader) == 64, "cache header is 64 bytes");
constexpr int kCacheMagic = 0x48454152;  // "HEAR"

struct CacheLayout {
  CacheHeader* hdr;
  float *aq, *ak, *pq, *pk, *part;
  uint8_t* mask;
  size_t bytes;
};

__host__ __device__ inline CacheLayout cache_layout(void* base, int B, int H, int Cq, int Ck, int D) {
  CacheLayout L{};
  char* p = static_cast<char*>(base);
  size_t off = 0;
  auto take = [&](size_t n) {
    off = (off + 255) / 256 * 256;
    char* r = p ? p + off : nullptr;
    off += n;
    return r;
  };
  const size_t bhd = static_cast<size_t>(B) * H * D * sizeof(float);
  L.hdr = reinterpret_cast<CacheHeader*>(take(sizeof(CacheHeader)));
  L.aq = reinterpret_cast<float*>(take(bhd));
  L.ak = reinterpret_cast<float*>(take(bhd));
  L.pq = reinterpret_cast<float*>(take(bhd));
  L.pk = reinterpret_cast<float*>(take(bhd));
  L.part = reinterpret_cast<float*>(take(static_cast<size_t>(B) * H * kPoolSplit * 2 * D * sizeof(float)));
  L.mask = reinterpret_cast<uint8_t*>(take(static_cast<size_t>(B) * H * Cq * Ck));
  L.bytes = (off + 255) / 256 * 256;
  return L;
}

__global__ void cache_init_kernel(CacheHeader* h, int B, int H, int Cq, int Ck, int D, float delta,
                                  int relative, float gate_lo, float gate_hi) {
  h->B = B;
  h->H = H;
  h->Cq = Cq;
  h->Ck = Ck;
  h->D = D;
  h->has_anchor = 0;
  h->delta = delta;
  h->relative = relative;
  h->gate_lo = gate_lo;
  h->gate_hi = gate_hi;
  h->n_refresh = 0;
  h->magic = kCacheMagic;
}

__global__ void cache_reset_kernel(CacheHeader* h) { h->has_anchor = 0; }

__device__ __forceinline__ CacheLayout device_layout(void* state) {
  const CacheHeader* h = static_cast<const CacheHeader*>(state);
  return cache_layout(state, h->B, h->H, h->Cq, h->Ck, h->D);
}

__device__ __forceinline__ bool header_matches(const void* state, int B, int H, int D) {
  const CacheHeader* h = static_cast<const CacheHeader*>(state);
  return h->magic == kCacheMagic && h->B == B && h->H == H && h->D == D;
}

// grid (kPoolSplit, B*H): partial column sums of q and k over a slice of the tokens.
// Rows are read as 16-byte vectors (thread = one vector column of a row; the CTA walks
// 256 / (vectors per row) rows at a time), partial sums combined in shared memory.
template <typename T>
__global__ void __launch_bounds__(256) pool_kernel(void* state, const T* __restrict__ q,
                                                   const T* __restrict__ k, int B, int H, int S,
                                                   int D) {
  constexpr int EPV = 16 / sizeof(T);
  __shared__ float red[2][256 * EPV];
  if (!header_matches(state, B, H, D)) {
    if (threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.y == 0) report_device_error(kStatusBadLabel, 60);
    return;
  }
  float* part = device_layout(state).part;
  const int64_t bh = blockIdx.y;
  const int vpr = D / EPV, rpi = 256 / vpr;
  const int rin = threadIdx.x / vpr, v = threadIdx.x % vpr;
  const int r0 = static_cast<int>((static_cast<int64_t>(S) * blockIdx.x) / kPoolSplit);
  const int r1 = static_cast<int>((static_cast<int64_t>(S) * (blockIdx.x + 1)) / kPoolSplit);
  const uint4* q4 = reinterpret_cast<const uint4*>(q) + bh * S * vpr;
  const uint4* k4 = reinterpret_cast<const uint4*>(k) + bh * S * vpr;
  float a[EPV], c[EPV];
#pragma unroll
  for (int e = 0; e < EPV; ++e) a[e] = c[e] = 0.f;
  // four rows per thread in flight: enough outstanding bytes per SM to cover HBM latency
#pragma unroll 4
  for (int r = r0 + rin; r < r1; r += rpi) {
    const uint4 xq = __ldg(q4 + static_cast<int64_t>(r) * vpr + v);
    const uint4 xk = __ldg(k4 + static_cast<int64_t>(r) * vpr + v);
    float fq[EPV], fk[EPV];
    unpack16<T>(xq, fq);
    unpack16<T>(xk, fk);
#pragma unroll
    for (int e = 0; e < EPV; ++e) {
      a[e] += fq[e];
      c[e] += fk[e];
    }
  }
  if (rin < rpi) {
#pragma unroll
    for (int e = 0; e < EPV; ++e) {
      red[0][rin * D + v * EPV + e] = a[e];
      red[1][rin * D + v * EPV + e] = c[e];
    }
  }
  __syncthreads();
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    float ta = 0.f, tb = 0.f;
    for (int i = 0; i < rpi; ++i) {
      ta += red[0][i * D + d];
      tb += red[1][i * D + d];
    }
    float* o = part + (bh * kPoolSplit + blockIdx.x) * 2 * D;
    o[d] = ta;
    o[D + d] = tb;
  }
}

// One CTA: pooled means, per-head drift, delta test, layer gate, refresh flags.
__global__ void __launch_bounds__(1024) decide_kernel(void* state, int B, int H, int D, int S,
                                                      uint8_t* __restrict__ refresh,
                                                      float* __restrict__ drift_out) {
  __shared__ int cnt;
  if (!header_matches(state, B, H, D)) return;  // reported by pool_kernel
  const CacheLayout L = device_layout(state);
  CacheHeader* hdr = L.hdr;
  if (threadIdx.x == 0) cnt = 0;
  const int BH = B * H;
  const float invS = 1.f / static_cast<float>(S);
  for (int e = threadIdx.x; e < BH * D; e += blockDim.x) {
    const int bh = e / D, d = e % D;
    float a = 0.f, b = 0.f;
    for (int i = 0; i < kPoolSplit; ++i) {
      a += L.part[(static_cast<int64_t>(bh) * kPoolSplit + i) * 2 * D + d];
      b += L.part[(static_cast<int64_t>(bh) * kPoolSplit + i) * 2 * D + D + d];
    }
    L.pq[e] = a * invS;
    L.pk[e] = b * invS;
  }
  __syncthreads();
  const int has = hdr->has_anchor;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int bh = warp; bh < BH; bh += blockDim.x >> 5) {
    float dist = 0.f, nrm = 0.f;
    if (has) {
      for (int d = lane; d < D; d += 32) {
        const int64_t e = static_cast<int64_t>(bh) * D + d;
        dist += fabsf(L.aq[e] - L.pq[e]) + fabsf(L.ak[e] - L.pk[e]);
        nrm += fabsf(L.aq[e]) + fabsf(L.ak[e]);
      }
    }
    for (int o = 16; o > 0; o >>= 1) {
      dist += __shfl_xor_sync(0xffffffffu, dist, o);
      nrm += __shfl_xor_sync(0xffffffffu, nrm, o);
    }
    if (lane == 0) {
      const float dd = has ? (hdr->relative ? dist / nrm : dist) : INFINITY;
      const int r = has ? (dd > hdr->delta ? 1 : 0) : 1;
      refresh[bh] = static_cast<uint8_t>(r);
      if (drift_out) drift_out[bh] = dd;
      if (r) atomicAdd(&cnt, 1);
    }
  }
  __syncthreads();
  int n = cnt;
  if (has && hdr->gate_lo >= 0.f) {
    const float frac = static_cast<float>(n) / static_cast<float>(BH);
    const int force = frac < hdr->gate_lo ? 0 : (frac > hdr->gate_hi ? 1 : -1);
    if (force >= 0) {
      for (int bh = threadIdx.x; bh < BH; bh += blockDim.x) refresh[bh] = static_cast<uint8_t>(force);
      n = force ? BH : 0;
    }
  }
  if (threadIdx.x == 0) hdr->n_refresh = n;
}

// Layer gate over heads held by several caches (a layer's heads split across GPUs):
// with the layer-wide refresh count n_layer of n_heads heads, fewer than gate_lo of them
// -> no local head refreshes, more than gate_hi -> every local head does; otherwise the
// per-head decisions stand. Not applied on a cache's first call (no anchors: every head
// refreshes). One CTA; the header's n_refresh becomes the local count after the gate.
__global__ void __launch_bounds__(256) layer_gate_kernel(void* state, uint8_t* __restrict__ refresh,
                                                         int n_layer, int n_heads, float gate_lo,
                                                         float gate_hi) {
  const CacheLayout L = device_layout(state);
  CacheHeader* hdr = L.hdr;
  if (hdr->magic != kCacheMagic) return;
  const int BH = hdr->B * hdr->H;
  if (!hdr->has_anchor || gate_lo < 0.f) return;
  const float frac = static_cast<float>(n_layer) / static_cast<float>(n_heads);
  const int force = frac < gate_lo ? 0 : (frac > gate_hi ? 1 : -1);
  if (force < 0) return;
  for (int bh = threadIdx.x; bh < BH; bh += blockDim.x) refresh[bh] = static_cast<uint8_t>(force);
  if (threadIdx.x == 0) hdr->n_refresh = force ? BH : 0;
}

// Grid-stride over the cached mask: refreshed heads (every head on the first update)
// take new_mask; the result is copied to out.
__global__ void update_mask_kernel(void* state, const uint8_t* __restrict__ new_mask,
                                   const uint8_t* __restrict__ refresh, uint8_t* __restrict__ out) {
  const CacheLayout L = device_layout(state);
  const CacheHeader* hdr = L.hdr;
  if (hdr->magic != kCacheMagic) return;
  const int64_t per = static_cast<int64_t>(hdr->Cq) * hdr->Ck;
  const int64_t n = static_cast<int64_t>(hdr->B) * hdr->H * per;
  const int has = hdr->has_anchor;
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < n;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t bh = e / per;
    uint8_t m = L.mask[e];
    if (new_mask && (!has || refresh[bh])) m = new_mask[e] ? 1 : 0;
    L.mask[e] = m;
    out[e] = m;
  }
}

// Anchors of refreshed heads move to the pooled means of the last should_refresh.
__global__ void update_anchor_kernel(void* state, const uint8_t* __restrict__ refresh,
                                     int have_new_mask) {
  const CacheLayout L = device_layout(state);
  CacheHeader* hdr = L.hdr;
  if (hdr->magic != kCacheMagic) return;
  const int has = hdr->has_anchor;
  const int BH = hdr->B * hdr->H, D = hdr->D;
  for (int e = threadIdx.x; e < BH * D; e += blockDim.x) {
    const int bh = e / D;
    if (have_new_mask && (!has || refresh[bh])) {
      L.aq[e] = L.pq[e];
      L.ak[e] = L.pk[e];
    }
  }
  __syncthreads();
  if (threadIdx.x == 0 && have_new_mask) hdr->has_anchor = 1;
}

}  // namespace bsa

extern "C" size_t bsa_mask_cache_state_bytes(int B, int H, int Cq, int Ck, int D) {
  if (B <= 0 || H <= 0 || Cq <= 0 || Ck <= 0 || D <= 0) return 0;
  return bsa::cache_layout(nullptr, B, H, Cq, Ck, D).bytes;
}

extern "C" int bsa_mask_cache_init(void* state, int B, int H, int Cq, int Ck, int D, float delta,
                                   int relative, float gate_lo, float gate_hi, void* stream) {
  using namespace bsa;
  if (!state) return fail(BSA_ERR_INVALID_ARG, "state is null");
  if (B <= 0 || H <= 0 || Cq <= 0 || Ck <= 0 || D <= 0 || D > 256 || 256 % D)
    return fail(BSA_ERR_INVALID_ARG, "bad sizes (D must divide 256)");
  if (reinterpret_cast<uintptr_t>(state) % 256) return fail(BSA_ERR_INVALID_ARG, "state not 256-byte aligned");
  CacheLayout L = cache_layout(state, B, H, Cq, Ck, D);
  cudaStream_t st = as_stream(stream);
  int rc;
  if ((rc = check_cuda(cudaMemsetAsync(state, 0, L.bytes, st), "memset state"))) return rc;
  cache_init_kernel<<<1, 1, 0, st>>>(L.hdr, B, H, Cq, Ck, D, delta, relative ? 1 : 0, gate_lo, gate_hi);
  count_launch();
  return check_cuda(cudaGetLastError(), "cache_init_kernel");
}

extern "C" int bsa_mask_cache_should_refresh(void* state, const void* q, const void* k,
                                             bsa_shape shape, uint8_t* refresh, float* drift_out,
                                             int* n_refresh_host, void* stream) {
  using namespace bsa;
  if (!state || !q || !k || !refresh) return fail(BSA_ERR_INVALID_ARG, "null pointer");
  if (shape.Hq != shape.Hkv) return fail(BSA_ERR_INVALID_ARG, "the cache needs Hkv == Hq");
  const int es = shape.dtype == BSA_F32 ? 4 : 2;
  if (shape.B <= 0 || shape.Hq <= 0 || shape.Sq <= 0 || shape.D <= 0 || shape.D > 256 ||
      256 % shape.D || (shape.D * es) % 16)
    return fail(BSA_ERR_UNSUPPORTED, "head dim %d must divide 256 and rows be 16-byte multiples",
                shape.D);
  if ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k)) % 16)
    return fail(BSA_ERR_INVALID_ARG, "q and k must be 16-byte aligned");
  cudaStream_t st = as_stream(stream);
  const int BH = shape.B * shape.Hq;
  int rc;
  if (shape.dtype == BSA_BF16)
    pool_kernel<__nv_bfloat16><<<dim3(kPoolSplit, BH), 256, 0, st>>>(
        state, static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
        shape.B, shape.Hq, shape.Sq, shape.D);
  else if (shape.dtype == BSA_F32)
    pool_kernel<float><<<dim3(kPoolSplit, BH), 256, 0, st>>>(
        state, static_cast<const float*>(q), static_cast<const float*>(k), shape.B, shape.Hq,
        shape.Sq, shape.D);
  else
    return fail(BSA_ERR_UNSUPPORTED, "dtype");
  count_launch();
  if ((rc = check_cuda(cudaGetLastError(), "pool_kernel"))) return rc;
  decide_kernel<<<1, 1024, 0, st>>>(state, shape.B, shape.Hq, shape.D, shape.Sq, refresh, drift_out);
  count_launch();
  if ((rc = check_cuda(cudaGetLastError(), "decide_kernel"))) return rc;
  if (n_refresh_host) {
    const CacheLayout L = cache_layout(state, 1, 1, 1, 1, 1);  // header offset only
    if ((rc = check_cuda(cudaMemcpyAsync(n_refresh_host, &L.hdr->n_refresh, sizeof(int),
                                         cudaMemcpyDeviceToHost, st), "copy n_refresh")))
      return rc;
    if ((rc = check_cuda(cudaStreamSynchronize(st), "cudaStreamSynchronize"))) return rc;
  }
  return BSA_OK;
}

extern "C" int bsa_mask_cache_layer_gate(void* state, uint8_t* refresh, int n_refresh_layer,
                                         int n_heads_layer, float gate_lo, float gate_hi,
                                         void* stream) {
  using namespace bsa;
  if (!state || !refresh) return fail(BSA_ERR_INVALID_ARG, "null pointer");
  if (n_heads_layer <= 0 || n_refresh_layer < 0 || n_refresh_layer > n_heads_layer)
    return fail(BSA_ERR_INVALID_ARG, "refresh count %d of %d heads", n_refresh_layer, n_heads_layer);
  layer_gate_kernel<<<1, 256, 0, as_stream(stream)>>>(state, refresh, n_refresh_layer, n_heads_layer,
                                                      gate_lo, gate_hi);
  count_launch();
  return check_cuda(cudaGetLastError(), "layer_gate_kernel");
}

extern "C" int bsa_mask_cache_update(void* state, const uint8_t* new_mask, const uint8_t* refresh,
                                     uint8_t* block_mask_out, void* stream) {
  using namespace bsa;
  if (!state || !refresh || !block_mask_out) return fail(BSA_ERR_INVALID_ARG, "null pointer");
  cudaStream_t st = as_stream(stream);
  int rc;
  update_mask_kernel<<<148 * 4, 256, 0, st>>>(state, new_mask, refresh, block_mask_out);
  count_launch();
  if ((rc = check_cuda(cudaGetLastError(), "update_mask_kernel"))) return rc;
  update_anchor_kernel<<<1, 1024, 0, st>>>(state, refresh, new_mask ? 1 : 0);
  count_launch();
  return check_cuda(cudaGetLastError(), "update_anchor_kernel");
}

extern "C" int bsa_mask_cache_reset(void* state, void* stream) {
  using namespace bsa;
  if (!state) return fail(BSA_ERR_INVALID_ARG, "state is null");
  const CacheLayout L = cache_layout(state, 1, 1, 1, 1, 1);
  cache_reset_kernel<<<1, 1, 0, as_stream(stream)>>>(L.hdr);
  count_launch();
  return check_cuda(cudaGetLastError(), "cache_reset_kernel");
}
