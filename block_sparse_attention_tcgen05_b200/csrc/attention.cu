// Block-sparse attention with SVG-EAR centroid compensation on sm_100a.
//
// Sources: "Sparse-block compensation" (mlx-arsenal notes) §The problem, §SVG-EAR —
// centroid compensation, §No LSE needed; "Partition the Support, Reconstruct the
// Residual" (Q, K, V permuted into group-major order; renormalised hard drop).
//
// Pipeline of one call (all on the caller's stream):
//   1. mask_cbits_kernel        the uint8 cluster mask -> per query cluster bitsets over
//                               key clusters (centroid columns).
//   2. prep_kernel (2 CTAs)     CTA 0: slot-layout order of the key clusters (a nearest-
//                               neighbour chain over the mask columns, so clusters kept
//                               by the same query clusters sit side by side), then the
//                               stable counting sort of the key labels into cluster-
//                               major slots in that order, each key cluster padded to a
//                               multiple of 16 slots (every 16-key group belongs to one
//                               cluster). CTA 1: the query label sort, then the row
//                               order of the 128-row query tiles (whole tiles of one
//                               cluster, then the leftover rows packed by a nearest-
//                               neighbour chain over the clusters' mask rows).
//   3. mask_gbits_kernel        per query cluster bitsets over the 16-key groups.
//   4. gather_rows_kernel       Q rows into tile order, only when the attention kernel
//                               cannot gather them itself by TMA.
//   5. gather_kv_centroids      K, V rows into cluster-major padded order, fused with
//                               the per-cluster mean k̄_c, v̄_c (fp32 sums).
//   6. attn_kernel              one CTA per 128-row query tile: kept key groups are
//                               walked as chunks of up to 128 keys (runs of kept
//                               groups); skipped clusters follow as 128-wide centroid
//                               chunks with column bias log2(n_c); both go through
//                               the same online softmax, so no log-sum-exp leaves
//                               the chip. S = QKᵀ and O += PV run on tcgen05 with
//                               TMEM accumulators; P overwrites S in TMEM.
#include <cuda_bf16.h>

#include <cmath>
#include <cstdio>

#include "common.cuh"
#include "ptx.cuh"

namespace bsa {

// ============================================================== label sort
// One CTA of 1024 threads. Cluster c gets slots [off[c], off[c] + roundup(n_c,
// cluster_pad)), filled with its tokens in increasing token order (a stable sort);
// remaining slots hold token -1 / label -1. With group arrays given, 16-slot group g
// is described by the cluster owning it and its number of real tokens.
struct LabelSortJob {
  const int32_t* labels;
  int S, C, cluster_pad, n_slots;
  int32_t *slot_token, *slot_label, *count, *off, *group_cluster, *group_valid;
  int n_groups;
  float* bias2;
  int C_pad;
  uint32_t* nonempty_bits;
  const int32_t* order;  // nullable: position p of the slot layout holds cluster order[p]
};

// Label sorts with at most kSortFastC clusters take a stable path without CTA-wide
// barriers inside the token loops: warp w owns the contiguous tokens
// [w ceil(S/32), (w+1) ceil(S/32)), counts them per label in its own histogram row,
// and after one scan over (label, warp) scatters them again in token order.
constexpr int kSortFastC = 512;

// Dynamic shared memory (bytes) a label sort of C clusters needs.
__host__ __device__ constexpr int label_sort_smem(int C) {
  return (C <= kSortFastC ? 34 * C + 1 : 2 * C + 1) * 4;
}

// One CTA of 1024 threads sorts one job; `sm` is label_sort_smem(C) bytes of shared memory.
__device__ void label_sort_cta(const LabelSortJob& jb, int32_t* sm) {
  const int32_t* __restrict__ labels = jb.labels;
  const int S = jb.S, C = jb.C, cluster_pad = jb.cluster_pad, n_slots = jb.n_slots;
  int32_t* __restrict__ slot_token = jb.slot_token;
  int32_t* __restrict__ slot_label = jb.slot_label;
  int32_t* __restrict__ count = jb.count;
  int32_t* __restrict__ off = jb.off;
  int32_t* __restrict__ group_cluster = jb.group_cluster;
  int32_t* __restrict__ group_valid = jb.group_valid;
  const int n_groups = jb.n_groups;
  float* __restrict__ bias2 = jb.bias2;
  const int C_pad = jb.C_pad;
  uint32_t* __restrict__ nonempty_bits = jb.nonempty_bits;
  const int32_t* __restrict__ order = jb.order;
  int32_t* cnt = sm;           // C
  int32_t* run = cnt + C;      // C + 1
  int32_t* hist = run + C + 1;  // 32 x C (fast path): warp-major counts, then slot cursors
  __shared__ int32_t warp_tot[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  // One cluster whose labels are all valid (the probe attention's keys): the stable
  // order is the identity, filled directly; anything else takes the general path.
  __shared__ int n_bad;
  if (tid == 0) n_bad = 0;
  __syncthreads();
  if (C == 1) {
    int bad = 0;
    for (int i = tid; i < S; i += 1024) bad += labels[i] != 0;
    bad = __reduce_add_sync(0xffffffffu, bad);
    if (lane == 0 && bad) atomicAdd(&n_bad, bad);
    __syncthreads();
    if (n_bad == 0) {
      const int padded = (S + cluster_pad - 1) / cluster_pad * cluster_pad;
      for (int i = tid; i < n_slots; i += 1024) {
        slot_token[i] = i < S ? i : -1;
        if (slot_label) slot_label[i] = i < S ? 0 : -1;
      }
      if (tid == 0) {
        count[0] = S;
        off[0] = 0;
        off[1] = padded;
      }
      if (group_cluster) {
        for (int g = tid; g < n_groups; g += 1024) {
          const int slot = g * 16;
          group_cluster[g] = slot < padded ? 0 : -1;
          group_valid[g] = slot < padded ? min(16, S - slot) : 0;
        }
      }
      if (bias2) {
        for (int c = tid; c < C_pad; c += 1024)
          bias2[c] = (c == 0 && S > 0) ? log2f(static_cast<float>(S)) : -INFINITY;
        if (tid == 0) nonempty_bits[0] = S > 0 ? 1u : 0u;
      }
      return;
    }
  }
  const bool fast = C <= kSortFastC;
  const int per_w = (S + 31) / 32;
  const int t_lo = min(S, warp * per_w), t_hi = min(S, t_lo + per_w);
  for (int c = tid; c < C; c += 1024) cnt[c] = 0;
  if (fast)
    for (int e = tid; e < 32 * C; e += 1024) hist[e] = 0;
  for (int i = tid; i < n_slots; i += 1024) {
    slot_token[i] = -1;
    if (slot_label) slot_label[i] = -1;
  }
  __syncthreads();
  if (fast) {
    // eight loads of 32 labels in flight per warp, then their counts
    for (int b8 = t_lo; b8 < t_hi; b8 += 256) {
      int lb[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = b8 + 32 * u + lane;
        lb[u] = i < t_hi ? labels[i] : -1;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const bool in = b8 + 32 * u + lane < t_hi;
        int l = lb[u];
        if (in && (l < 0 || l >= C)) report_device_error(kStatusBadLabel, 30);
        if (!in || l < 0 || l >= C) l = -1;
        const unsigned peers = __match_any_sync(0xffffffffu, l);
        if (l >= 0 && lane == __ffs(peers) - 1) hist[warp * C + l] += __popc(peers);
        __syncwarp();
      }
    }
    __syncthreads();
    for (int c = tid; c < C; c += 1024) {
      int t = 0;
#pragma unroll 8
      for (int w = 0; w < 32; ++w) t += hist[w * C + c];
      cnt[c] = t;
    }
  } else {
    for (int i = tid; i < S; i += 1024) {
      const int l = labels[i];
      if (l >= 0 && l < C) atomicAdd(&cnt[l], 1);
      else report_device_error(kStatusBadLabel, 30);
    }
  }
  __syncthreads();

  // Exclusive scan of the padded cluster sizes in slot-layout order (label order, or
  // `order`); thread t owns a contiguous range of positions.
  const int per = (C + 1023) / 1024;
  const int c0 = min(C, tid * per), c1 = min(C, c0 + per);
  int local = 0;
  for (int q = c0; q < c1; ++q) {
    const int c = order ? order[q] : q;
    local += (cnt[c] + cluster_pad - 1) / cluster_pad * cluster_pad;
  }
  int incl = local;
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int t = warp_tot[lane];
    int ti = t;
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, ti, o);
      if (lane >= o) ti += y;
    }
    warp_tot[lane] = ti - t;
  }
  __syncthreads();
  int base = warp_tot[warp] + incl - local;
  for (int q = c0; q < c1; ++q) {
    const int c = order ? order[q] : q;
    run[c] = base;
    off[c] = base;
    count[c] = cnt[c];
    base += (cnt[c] + cluster_pad - 1) / cluster_pad * cluster_pad;
  }
  if (tid == 1023) {
    run[C] = base;
    off[C] = base;  // total slots in use
  }
  __syncthreads();

  if (fast) {
    // slot cursor of (warp, label): the label's first slot plus the tokens of the
    // warps before it
    for (int c = tid; c < C; c += 1024) {
      int r = run[c];
      for (int w = 0; w < 32; ++w) {
        const int t = hist[w * C + c];
        hist[w * C + c] = r;
        r += t;
      }
    }
    __syncthreads();
    for (int b8 = t_lo; b8 < t_hi; b8 += 256) {
      int lb[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = b8 + 32 * u + lane;
        lb[u] = i < t_hi ? labels[i] : -1;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = b8 + 32 * u + lane;
        int l = lb[u];
        if (l >= C) l = -1;  // out-of-range labels were reported above; the token is dropped
        const unsigned peers = __match_any_sync(0xffffffffu, l);
        const int rank = __popc(peers & ((1u << lane) - 1u));
        const int sb = l >= 0 ? hist[warp * C + l] : 0;
        __syncwarp();
        if (l >= 0 && lane == __ffs(peers) - 1) hist[warp * C + l] = sb + __popc(peers);
        __syncwarp();
        if (l >= 0) {
          slot_token[sb + rank] = i;
          if (slot_label) slot_label[sb + rank] = l;
        }
      }
    }
  } else {
    // Stable scatter, 1024 tokens at a time: ranks inside a warp from match_any, warps
    // take their slots one after another so earlier tokens get earlier slots.
    for (int t0 = 0; t0 < S; t0 += 1024) {
      const int i = t0 + tid;
      int l = (i < S) ? labels[i] : -1;
      if (l >= C) l = -1;  // out-of-range labels were reported above; the token is dropped
      const unsigned peers = __match_any_sync(0xffffffffu, l);
      const int rank = __popc(peers & ((1u << lane) - 1u));
      const int leader = __ffs(peers) - 1;
      int slot_base = 0;
      for (int w = 0; w < 32; ++w) {
        if (warp == w && l >= 0 && lane == leader) {
          slot_base = run[l];
          run[l] += __popc(peers);
        }
        __syncthreads();
      }
      slot_base = __shfl_sync(0xffffffffu, slot_base, leader);
      if (l >= 0) {
        const int s = slot_base + rank;
        slot_token[s] = i;
        if (slot_label) slot_label[s] = l;
      }
    }
  }
  __syncthreads();

  if (group_cluster) {
    // groups of every cluster, written by the thread owning it; groups past the last
    // cluster's slots belong to none
    const int total = off[C];
    for (int g = total / 16 + tid; g < n_groups; g += 1024) {
      group_cluster[g] = -1;
      group_valid[g] = 0;
    }
    for (int c = tid; c < C; c += 1024) {
      const int n = cnt[c], g0 = off[c] / 16, ng = (n + 15) / 16;  // cluster_pad is 16 here
      for (int i = 0; i < ng; ++i) {
        group_cluster[g0 + i] = c;
        group_valid[g0 + i] = min(16, n - 16 * i);
      }
    }
  }
  if (bias2) {
    for (int c = tid; c < C_pad; c += 1024)
      bias2[c] = (c < C && cnt[c] > 0) ? log2f(static_cast<float>(cnt[c])) : -INFINITY;
    for (int w = tid; w < (C + 31) / 32; w += 1024) {
      uint32_t bits = 0;
      for (int j = 0; j < 32; ++j) {
        const int c = w * 32 + j;
        if (c < C && cnt[c] > 0) bits |= 1u << j;
      }
      nonempty_bits[w] = bits;
    }
  }
}

// CTA b sorts job b (two sorts of one call side by side).
__global__ void __launch_bounds__(1024) label_sort_kernel(const LabelSortJob j0,
                                                          const LabelSortJob j1) {
  extern __shared__ int32_t sm_i32[];
  label_sort_cta(blockIdx.x == 0 ? j0 : j1, sm_i32);
}

// ============================================================== mask bitsets
// grid (Cq, n_h_slices, n_b_slices). cbits[slice][a][w]: bit c of word w = mask[a][32w+c].
__global__ void __launch_bounds__(256) mask_cbits_kernel(const uint8_t* __restrict__ mask,
                                                         int64_t bstride, int64_t hstride, int nh,
                                                         int Cq, int Ck, int Wc,
                                                         uint32_t* __restrict__ cbits) {
  const int a = blockIdx.x, hs = blockIdx.y, bs = blockIdx.z;
  const uint8_t* row = mask + bs * bstride + hs * hstride + static_cast<int64_t>(a) * Ck;
  const size_t slice = static_cast<size_t>(bs) * nh + hs;
  uint32_t* crow = cbits + (slice * Cq + a) * Wc;
  for (int w = threadIdx.x; w < Wc; w += blockDim.x) {
    uint32_t bits = 0;
    for (int j = 0; j < 32; ++j) {
      const int c = w * 32 + j;
      if (c < Ck && row[c]) bits |= 1u << j;
    }
    crow[w] = bits;
  }
}

// grid (Cq, n_slices). gbits[slice][a][w]: bit j = kept(a, cluster of 16-key group 32w+j),
// from the cluster bitsets; gfull: bit j = group 32w+j holds 16 real keys.
__global__ void __launch_bounds__(256) mask_gbits_kernel(const uint32_t* __restrict__ cbits,
                                                         int Cq, int Wc,
                                                         const int32_t* __restrict__ group_cluster,
                                                         const int32_t* __restrict__ group_valid,
                                                         int n_groups, int Wg,
                                                         uint32_t* __restrict__ gbits,
                                                         uint32_t* __restrict__ gfull) {
  const int a = blockIdx.x;
  const size_t slice = blockIdx.y;
  const uint32_t* crow = cbits + (slice * Cq + a) * Wc;
  uint32_t* grow = gbits + (slice * Cq + a) * Wg;
  for (int w = threadIdx.x; w < Wg; w += blockDim.x) {
    uint32_t bits = 0;
    for (int j = 0; j < 32; ++j) {
      const int g = w * 32 + j;
      if (g < n_groups) {
        const int c = group_cluster[g];
        if (c >= 0 && ((crow[c >> 5] >> (c & 31)) & 1u)) bits |= 1u << j;
      }
    }
    grow[w] = bits;
  }
  if (a == 0 && slice == 0) {
    for (int w = threadIdx.x; w < Wg; w += blockDim.x) {
      uint32_t bits = 0;
      for (int j = 0; j < 32; ++j) {
        const int g = w * 32 + j;
        if (g < n_groups && group_valid[g] == 16) bits |= 1u << j;
      }
      gfull[w] = bits;
    }
  }
}

// ============================================================== nearest-neighbour chain
// Order of n items (n <= kChainMax) given as bitsets of W words, stored transposed in
// shared memory (bitsT[w * n + i] = word w of item i): start at item 0, then move, step
// by step, to the unvisited item whose bitset differs from the current one in the
// fewest bits (Hamming distance; ties: lower index). `dist` is shared scratch of
// n x chain_stride(n) uint16. All threads of the CTA call it; warp 0 walks the chain and
// writes ord[0..n).
constexpr int kChainMax = 288;

// Row stride of the distance matrix: even (two entries per 32-bit load) with an odd
// number of words, so that the mirrored column writes hit distinct banks.
__host__ __device__ constexpr int chain_stride(int n) {
  return ((n + 1) / 2 % 2 == 0) ? (n + 1) / 2 * 2 + 2 : (n + 1) / 2 * 2;
}

__device__ void nn_chain(const uint32_t* bitsT, int n, int W, uint16_t* dist, int32_t* ord) {
  if (n <= 0) return;
  constexpr int kK = (kChainMax + 31) / 32;   // items per lane in the distance rows
  constexpr int kK2 = (kChainMax + 63) / 64;  // item pairs per lane in the chain
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = blockDim.x >> 5;
  const int np = chain_stride(n);
  // distances: warp per item i, lane per item j > i (mirrored into column i); 8 words
  // of item i at a time in registers
  for (int i = warp; i < n; i += nwarps) {
    int d[kK];
#pragma unroll
    for (int k = 0; k < kK; ++k) d[k] = 0;
    for (int w0 = 0; w0 < W; w0 += 8) {
      uint32_t ri[8];
#pragma unroll
      for (int t = 0; t < 8; ++t) ri[t] = w0 + t < W ? bitsT[(w0 + t) * n + i] : 0u;
#pragma unroll
      for (int k = 0; k < kK; ++k) {
        const int j = lane + 32 * k;
        if (j > i && j < n) {
#pragma unroll
          for (int t = 0; t < 8; ++t)
            if (w0 + t < W) d[k] += __popc(ri[t] ^ bitsT[(w0 + t) * n + j]);
        }
      }
    }
#pragma unroll
    for (int k = 0; k < kK; ++k) {
      const int j = lane + 32 * k;
      if (j > i && j < n) {
        const uint16_t v = static_cast<uint16_t>(min(d[k], 65534));
        dist[i * np + j] = v;
        dist[j * np + i] = v;
      } else if (j == i) {
        dist[i * np + i] = 0;
      } else if (j >= n && j < np) {
        dist[i * np + j] = 0xffffu;
      }
    }
  }
  __syncthreads();
  if (warp == 0) {
    // lane owns items 2 lane + 64 k and 2 lane + 64 k + 1; bit 2k (+1) of `vis` marks
    // them visited
    uint32_t vis = lane == 0 ? 1u : 0u;
    int cur = 0;
    if (lane == 0) ord[0] = 0;
    for (int step = 1; step < n; ++step) {
      const uint32_t* row = reinterpret_cast<const uint32_t*>(dist + cur * np);
      uint32_t best = 0xffffffffu;
#pragma unroll
      for (int k = 0; k < kK2; ++k) {
        const int j = 2 * lane + 64 * k;
        if (j < n) {
          const uint32_t wd = row[j >> 1];
          const uint32_t k0 = ((vis >> (2 * k)) & 1u) ? 0xffffffffu : ((wd & 0xffffu) << 16) | j;
          const uint32_t k1 = (j + 1 >= n || ((vis >> (2 * k + 1)) & 1u))
                                  ? 0xffffffffu
                                  : ((wd >> 16) << 16) | (j + 1);
          best = min(best, min(k0, k1));
        }
      }
      best = __reduce_min_sync(0xffffffffu, best);
      cur = static_cast<int>(best & 0xffffu);
      if (lane == ((cur & 63) >> 1)) vis |= 1u << (2 * (cur >> 6) + (cur & 1));
      if (lane == 0) ord[step] = cur;
    }
  }
}

// OR of the mask bitsets over every (batch, head) slice: any[a][w] (Cq x Wc words).
__device__ void or_slices(const uint32_t* __restrict__ cbits, int n_slices, int Cq, int Wc,
                          uint32_t* any) {
  for (int e = threadIdx.x; e < Cq * Wc; e += blockDim.x) {
    uint32_t x = 0;
    for (int sl = 0; sl < n_slices; ++sl) x |= cbits[static_cast<size_t>(sl) * Cq * Wc + e];
    any[e] = x;
  }
}

// ============================================================== key cluster order
// The slot layout of the key clusters decides how a query tile's kept key groups fall
// into runs, and so how many chunks (of at most 128 keys) the attention kernel walks.
// Clusters whose columns of the mask (the query clusters keeping them, OR-ed over every
// (batch, head) slice) are alike are laid out next to each other: the nearest-neighbour
// chain above over the key clusters' columns. Without room for it (more than kChainMax
// key clusters, or too many query clusters) the label order is kept.
struct KeyOrderArgs {
  const uint32_t* cbits;
  int n_slices, Cq, Ck, Wc;
  int chain;
  int32_t* order;  // out: Ck
};

// Shared memory of the chain over the key clusters.
__host__ __device__ constexpr size_t key_order_smem(int Cq, int Ck) {
  return (static_cast<size_t>(Cq) * ((Ck + 31) / 32) + static_cast<size_t>((Cq + 31) / 32) * Ck) * 4 +
         static_cast<size_t>(Ck) * chain_stride(Ck) * 2;
}

__device__ void key_order_cta(const KeyOrderArgs& ka, uint8_t* sm) {
  const int Cq = ka.Cq, Ck = ka.Ck, Wc = ka.Wc, Wq = (Cq + 31) / 32;
  if (!ka.chain) {
    for (int c = threadIdx.x; c < Ck; c += blockDim.x) ka.order[c] = c;
    return;
  }
  uint32_t* any = reinterpret_cast<uint32_t*>(sm);  // Cq x Wc
  uint32_t* colT = any + Cq * Wc;                    // Wq x Ck: word w of column c at w*Ck + c
  uint16_t* dist = reinterpret_cast<uint16_t*>(colT + Wq * Ck);
  or_slices(ka.cbits, ka.n_slices, Cq, Wc, any);
  __syncthreads();
  for (int e = threadIdx.x; e < Wq * Ck; e += blockDim.x) {
    const int w = e / Ck, c = e % Ck;
    uint32_t bits = 0;
    for (int j = 0; j < 32 && 32 * w + j < Cq; ++j)
      bits |= ((any[(32 * w + j) * Wc + (c >> 5)] >> (c & 31)) & 1u) << j;
    colT[e] = bits;
  }
  __syncthreads();
  nn_chain(colT, Ck, Wq, dist, ka.order);
}

// ============================================================== query tile plan
// The attention kernel computes every key group that any row of a 128-row query tile
// keeps, for all 128 rows. With query rows in plain cluster order a tile straddles two
// clusters whenever cluster sizes are not multiples of 128 (3x6x8 video tiles hold 144
// tokens), and the rows of one cluster then also compute the other cluster's kept keys.
// The plan lays the rows out so that tiles mix as few kept sets as possible:
//   1. every query cluster fills floor(n_a / 128) whole tiles with its own rows (no mix);
//   2. the remaining n_a mod 128 rows of each cluster (its leftover) are laid out in the
//      order of a nearest-neighbour chain over the clusters' kept sets: the chain starts
//      at the lowest label with a leftover and moves, step by step, to the unvisited
//      cluster whose mask row differs from the current one in the fewest key clusters
//      (Hamming distance; ties: lower label); consecutive leftovers then share tiles.
// Kept sets are the OR of the mask over every (batch, head) slice. The leftover tiles
// come first (padded to a tile boundary: they are the costliest and start earliest), the
// whole tiles follow; the tile count stays ceil(Sq / 128). When the chain does not fit
// in shared memory (more than kChainMax clusters with a leftover, or mask rows too long)
// the leftovers follow in label order. Any layout gives the same result; only the work
// differs. One CTA of 1024 threads.

struct PlanArgs {
  const int32_t* sort_token;  // stable label sort of the query rows (cluster-major)
  const int32_t* sort_label;  // label of each sorted slot (-1 past the valid rows)
  const int32_t* count;       // rows per query cluster
  const int32_t* off;         // first sorted slot of each cluster
  const uint32_t* cbits;      // mask bitsets (slice, Cq, Wc) over key clusters
  int n_slices, Cq, Wc, Sqpad;
  int chain;                  // 1: nearest-neighbour chain over the leftovers, 0: label order
  int32_t* row_token;         // out: token of each planned row (-1 = pad)
  int32_t* row_label;         // out: its label (-1 = pad)
  int32_t* scratch;           // 5 * Cq ints of workspace
};

// Shared memory of the chain over the leftover clusters.
__host__ __device__ constexpr size_t plan_smem(int Cq, int Wc) {
  return (static_cast<size_t>(Cq) * Wc + static_cast<size_t>(Wc) * kChainMax) * 4 +
         static_cast<size_t>(kChainMax) * chain_stride(kChainMax) * 2;
}

__device__ void plan_cta(const PlanArgs& pa, uint8_t* sm) {
  const int Cq = pa.Cq, Wc = pa.Wc;
  int32_t* rem = pa.scratch;                                          // Cq
  int32_t* poff = rem + Cq;                                           // Cq
  int32_t* lcl = poff + Cq;                                           // Cq: clusters with a leftover
  int32_t* ord = lcl + Cq;                                            // Cq: chain order (indices into lcl)
  int32_t* dstp = ord + Cq;                                           // Cq: first row of each leftover
  uint32_t* any = reinterpret_cast<uint32_t*>(sm);   // Cq x Wc (chain only)
  uint32_t* anyT = any + Cq * Wc;                     // Wc x L: the leftovers' rows, transposed
  uint16_t* dist = reinterpret_cast<uint16_t*>(anyT + Wc * kChainMax);  // L x chain_stride(L)
  __shared__ int warp_tot[32];
  __shared__ int s_total, s_full, s_L;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  if (pa.chain) or_slices(pa.cbits, pa.n_slices, Cq, Wc, any);
  // exclusive scan of 128 * floor(n_a / 128): first row of cluster a's whole tiles
  const int per = (Cq + 1023) / 1024;
  const int c0 = min(Cq, tid * per), c1 = min(Cq, c0 + per);
  int local = 0, valid = 0;
  for (int c = c0; c < c1; ++c) {
    local += pa.count[c] / 128 * 128;
    valid += pa.count[c];
  }
  int incl = local;
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  valid = __reduce_add_sync(0xffffffffu, valid);
  const int fsum = __reduce_add_sync(0xffffffffu, local);
  if (lane == 31) warp_tot[warp] = incl;
  if (tid == 0) {
    s_total = 0;
    s_full = 0;
  }
  __syncthreads();
  if (lane == 0) {
    atomicAdd(&s_total, valid);
    atomicAdd(&s_full, fsum);
  }
  if (warp == 0) {
    const int t = warp_tot[lane];
    int ti = t;
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, ti, o);
      if (lane >= o) ti += y;
    }
    warp_tot[lane] = ti - t;
  }
  __syncthreads();
  const int total = s_total;  // rows with a valid label
  // The leftover tiles come first, padded to a tile boundary; the whole tiles follow.
  const int full_rows = s_full, left_rows = total - full_rows;
  const int pure0 = (left_rows + 127) / 128 * 128;
  int base = pure0 + warp_tot[warp] + incl - local;
  for (int c = c0; c < c1; ++c) {
    const int n = pa.count[c], full = n / 128 * 128;
    rem[c] = n - full;
    poff[c] = base;
    base += full;
  }
  __syncthreads();
  // whole tiles: rows [0, 128 k_a) of each cluster, in cluster order (warp per cluster)
  {
    const int32_t* __restrict__ st = pa.sort_token;
    int32_t* __restrict__ rt = pa.row_token;
    int32_t* __restrict__ rl = pa.row_label;
    for (int c = warp; c < Cq; c += 32) {
      const int full = pa.count[c] / 128 * 128, src = pa.off[c], dst = poff[c];
      for (int i0 = 0; i0 < full; i0 += 128) {
        int tk[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) tk[u] = st[src + i0 + 32 * u + lane];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          rt[dst + i0 + 32 * u + lane] = tk[u];
          rl[dst + i0 + 32 * u + lane] = c;
        }
      }
    }
  }
  for (int r = left_rows + tid; r < pure0; r += 1024) {  // pad of the last leftover tile
    pa.row_token[r] = -1;
    pa.row_label[r] = -1;
  }
  for (int r = pure0 + full_rows + tid; r < pa.Sqpad; r += 1024) {
    pa.row_token[r] = -1;
    pa.row_label[r] = -1;
  }
  // ------------------------------------------------ leftovers: the clusters that have
  // one, in label order (warp 0 compacts them)
  if (warp == 0) {
    int L = 0;
    for (int c0w = 0; c0w < Cq; c0w += 32) {
      const int c = c0w + lane;
      const bool has = c < Cq && rem[c] > 0;
      const unsigned bal = __ballot_sync(0xffffffffu, has);
      if (has) lcl[L + __popc(bal & ((1u << lane) - 1u))] = c;
      L += __popc(bal);
    }
    if (lane == 0) s_L = L;
  }
  __syncthreads();
  const int L = s_L;
  const bool chain = pa.chain && L <= kChainMax;
  if (chain) {
    for (int e = tid; e < Wc * L; e += 1024) anyT[e] = any[lcl[e % L] * Wc + e / L];
    __syncthreads();
    nn_chain(anyT, L, Wc, dist, ord);
  } else {
    for (int t = tid; t < L; t += 1024) ord[t] = t;  // label order
  }
  __syncthreads();
  // first row of each leftover in chain order (warp 0 scans)
  if (warp == 0) {
    int run = 0;
    for (int t0 = 0; t0 < L; t0 += 32) {
      const int t = t0 + lane;
      const int r = t < L ? rem[lcl[ord[t]]] : 0;
      int x = r;
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      if (t < L) dstp[t] = run + x - r;
      run += __shfl_sync(0xffffffffu, x, 31);
    }
  }
  __syncthreads();
  // copy the leftover rows, one warp per cluster
  for (int t = warp; t < L; t += 32) {
    const int c = lcl[ord[t]];
    const int r = rem[c];
    const int src = pa.off[c] + pa.count[c] - r;
    const int dst = dstp[t];
    for (int i = lane; i < r; i += 32) {
      pa.row_token[dst + i] = pa.sort_token[src + i];
      pa.row_label[dst + i] = c;
    }
  }
}

// ============================================================== call preparation
// CTA 0: key cluster order, then the key label sort in that order. CTA 1: query label
// sort, then the query tile plan. The two chains are independent and run side by side.
__global__ void __launch_bounds__(1024) prep_kernel(const KeyOrderArgs ka, const LabelSortJob jk,
                                                    const LabelSortJob jq, const PlanArgs pa) {
  extern __shared__ __align__(16) uint8_t sm_prep[];
  if (blockIdx.x == 0) {
    key_order_cta(ka, sm_prep);
    __syncthreads();
    label_sort_cta(jk, reinterpret_cast<int32_t*>(sm_prep));
  } else {
    label_sort_cta(jq, reinterpret_cast<int32_t*>(sm_prep));
    __syncthreads();
    plan_cta(pa, sm_prep);
  }
}

// ============================================================== dense call preparation
// One query cluster, one key cluster, the block kept, no compensation (the probe rows'
// dense attention): the sorts and the plan are identities, so their outputs are filled
// directly (grid-stride, 256 threads per CTA) instead of by the sparse call's chain.
__global__ void __launch_bounds__(256) dense_prep_kernel(int Sq, int Sqpad, int Sk, int Skpad, int G,
                                                         int Wg, int Ckpad, int32_t* qrow_token,
                                                         int32_t* qrow_label, int32_t* kslot_token,
                                                         int32_t* group_cluster, int32_t* group_valid,
                                                         int32_t* k_count, int32_t* k_off,
                                                         uint32_t* cbits, uint32_t* gbits,
                                                         uint32_t* gfull, uint32_t* cnonempty,
                                                         float* bias2) {
  const int stride = gridDim.x * blockDim.x;
  const int t0 = blockIdx.x * blockDim.x + threadIdx.x;
  for (int i = t0; i < Sqpad; i += stride) {
    qrow_token[i] = i < Sq ? i : -1;
    qrow_label[i] = i < Sq ? 0 : -1;
  }
  for (int i = t0; i < Skpad; i += stride) kslot_token[i] = i < Sk ? i : -1;
  for (int g = t0; g < G; g += stride) {
    const int nv = min(16, max(0, Sk - 16 * g));
    group_cluster[g] = nv > 0 ? 0 : -1;
    group_valid[g] = nv;
  }
  for (int w = t0; w < Wg; w += stride) {
    uint32_t kept = 0, full = 0;
    for (int j = 0; j < 32; ++j) {
      const int g = 32 * w + j;
      if (g < G && 16 * g < Sk) kept |= 1u << j;
      if (g < G && 16 * g + 16 <= Sk) full |= 1u << j;
    }
    gbits[w] = kept;
    gfull[w] = full;
  }
  for (int c = t0; c < Ckpad; c += stride) bias2[c] = c == 0 && Sk > 0 ? log2f(static_cast<float>(Sk)) : -INFINITY;
  if (t0 == 0) {
    cbits[0] = 1u;
    cnonempty[0] = Sk > 0 ? 1u : 0u;
    k_count[0] = Sk;
    k_off[0] = 0;
    k_off[1] = (Sk + 15) / 16 * 16;
  }
}

// ============================================================== gathers
// dst[bh][r] = src[bh][row_token[r]] (zero row when the token is -1); 16-byte vectors.
__global__ void __launch_bounds__(256) gather_rows_kernel(const uint4* __restrict__ src,
                                                          uint4* __restrict__ dst,
                                                          const int32_t* __restrict__ row_token,
                                                          int S, int Spad, int vpr, int H) {
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int r = static_cast<int>(idx / vpr), v = static_cast<int>(idx % vpr);
  if (r >= Spad) return;
  const int64_t bh = static_cast<int64_t>(blockIdx.z) * H + blockIdx.y;
  const int tok = row_token[r];
  uint4 val = make_uint4(0, 0, 0, 0);
  if (tok >= 0) val = __ldg(src + (bh * S + tok) * vpr + v);
  dst[(bh * Spad + r) * vpr + v] = val;
}

template <typename T>
__device__ __forceinline__ void unpack16(const uint4& u, float* f);
template <>
__device__ __forceinline__ void unpack16<__nv_bfloat16>(const uint4& u, float* f) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 x = __bfloat1622float2(h[i]);
    f[2 * i] = x.x;
    f[2 * i + 1] = x.y;
  }
}
template <>
__device__ __forceinline__ void unpack16<float>(const uint4& u, float* f) {
  f[0] = __uint_as_float(u.x);
  f[1] = __uint_as_float(u.y);
  f[2] = __uint_as_float(u.z);
  f[3] = __uint_as_float(u.w);
}
__device__ __forceinline__ void store_elt(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }
__device__ __forceinline__ void store_elt(float* p, float x) { *p = x; }

// grid (C_pad, Hkv, B), 256 threads. Copies the rows of cluster c into their padded
// cluster-major slots of kp / vp and writes the cluster means k̄_c, v̄_c (fp32 sums,
// rounded once to T). Clusters that are empty or beyond C get zero centroids.
template <typename T>
__global__ void __launch_bounds__(256) gather_kv_centroids_kernel(
    const T* __restrict__ k, const T* __restrict__ v, T* __restrict__ kp, T* __restrict__ vp,
    T* __restrict__ kc, T* __restrict__ vc, const int32_t* __restrict__ slot_token,
    const int32_t* __restrict__ count, const int32_t* __restrict__ off, int S, int Skpad, int C,
    int Cpad, int D, int Hkv) {
  constexpr int EPV = 16 / sizeof(T);
  __shared__ float red[2][2048];
  const int c = blockIdx.x;
  const int64_t bh = static_cast<int64_t>(blockIdx.z) * Hkv + blockIdx.y;
  const int vpr = D / EPV, rpi = 256 / vpr;
  const int rin = threadIdx.x / vpr, part = threadIdx.x % vpr;
  const int n = c < C ? count[c] : 0;
  const int start = c < C ? off[c] : 0;
  const int padded = (n + 15) / 16 * 16;
  float ak[EPV], av[EPV];
#pragma unroll
  for (int e = 0; e < EPV; ++e) ak[e] = av[e] = 0.f;
  const uint4* k4 = reinterpret_cast<const uint4*>(k);
  const uint4* v4 = reinterpret_cast<const uint4*>(v);
  uint4* kp4 = reinterpret_cast<uint4*>(kp);
  uint4* vp4 = reinterpret_cast<uint4*>(vp);
  for (int s = rin; s < padded; s += rpi) {
    const int slot = start + s;
    const int tok = slot_token[slot];
    uint4 xk = make_uint4(0, 0, 0, 0), xv = make_uint4(0, 0, 0, 0);
    if (tok >= 0) {
      xk = __ldg(k4 + (bh * S + tok) * vpr + part);
      xv = __ldg(v4 + (bh * S + tok) * vpr + part);
    }
    kp4[(bh * Skpad + slot) * vpr + part] = xk;
    vp4[(bh * Skpad + slot) * vpr + part] = xv;
    float fk[EPV], fv[EPV];
    unpack16<T>(xk, fk);
    unpack16<T>(xv, fv);
#pragma unroll
    for (int e = 0; e < EPV; ++e) {
      ak[e] += fk[e];
      av[e] += fv[e];
    }
  }
#pragma unroll
  for (int e = 0; e < EPV; ++e) {
    red[0][rin * D + part * EPV + e] = ak[e];
    red[1][rin * D + part * EPV + e] = av[e];
  }
  __syncthreads();
  const float inv = n > 0 ? 1.f / static_cast<float>(n) : 0.f;
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    float sk = 0.f, sv = 0.f;
    for (int r = 0; r < rpi; ++r) {
      sk += red[0][r * D + d];
      sv += red[1][r * D + d];
    }
    store_elt(kc + (bh * Cpad + c) * D + d, sk * inv);
    store_elt(vc + (bh * Cpad + c) * D + d, sv * inv);
  }
}

// ============================================================== attention kernel
struct AttnArgs {
  int B, Hq, Hkv, Sq, Sqpad, Skpad, Ck, Ckpad, Cq, G, Wg, Wc;
  int kstride;  // rows per (batch, KV head) in the tensors the K/V maps address
  int q_gather;   // 1: the Q map addresses the caller's q (B*Hq*Sq rows, one-row boxes) and
                  // the tile's rows are gathered through qrow_token; 0: a permuted copy
  int ksplit;   // CTAs per query tile, each over a contiguous range of key groups
  float* part;  // ksplit > 1: per split, unnormalised O, running max and sum per row
  int nh_slices, b_sliced, h_sliced;
  int compensate;
  float scale_log2;
  const int32_t* qrow_token;
  const int32_t* qrow_label;
  const int32_t* group_valid;
  const uint32_t* cbits;
  const uint32_t* gbits;
  const uint32_t* gfull;
  const uint32_t* cnonempty;
  const float* bias2;
  float* out;
};

// Chunk records per CTA: at most 2048 token chunks (G <= 4096) plus 128 centroid chunks.
constexpr int kChunkListCap = 2176;

template <int D, bool TF32>
struct AttnCfg {
  static constexpr int ESIZE = TF32 ? 4 : 2;
  static constexpr int ATOM = 128 / ESIZE;          // elements per 128-byte swizzled row
  static constexpr int NATOM = D / ATOM;            // 128-byte column chunks per row
  static constexpr int TILE = 128 * D * ESIZE;      // one 128-row operand tile
  static constexpr int KSTEP = 32 / ESIZE;          // K of one MMA instruction
  static constexpr int MISC = 2048 + kChunkListCap * 4 + 512;  // barriers, bitsets, chunk list
  static constexpr int SMEM = 3 * TILE + MISC + 1024;
  // At least ~100 KB so that at most two CTAs share an SM (two 256-column TMEM
  // allocations fill the 512 columns).
  static constexpr int SMEM_LAUNCH = SMEM > 100 * 1024 ? SMEM : 100 * 1024;
};

// Q/K/V full (TMA), K/V empty (MMA done reading), S-low / S-high full (QK of key
// columns 0..63 / 64..127 done), P-low / P-high ready (softmax of those columns
// written), PV-low done, O final, drain.
enum { BAR_Q = 0, BAR_KF, BAR_KE, BAR_VF, BAR_VE, BAR_SFLO, BAR_SFHI, BAR_PLO, BAR_PHI, BAR_OLO,
       BAR_OF, BAR_DRAIN, NBAR };

struct Chunk {
  int start;   // first key slot (token chunk) or first centroid (centroid chunk)
  int n;       // number of columns, multiple of 16, <= 128
  int g0, ng;  // token chunk: first group and number of groups
  bool uniform, centroid;
};

__device__ __forceinline__ bool bit_at(const uint32_t* bits, int i) {
  return (bits[i >> 5] >> (i & 31)) & 1u;
}

// A CTA's chunk list, built once by one warp so that no role walks the bitsets per
// chunk. The chunks, in order: every run of consecutive kept 16-key groups inside the
// CTA's key range [g_lo, g_hi) (groups outside it count as dropped), cut into chunks of
// at most 8 groups from the run's start; then one 128-wide chunk per needed centroid
// chunk. A token chunk is uniform when every row of the tile keeps all of its groups
// and none of them holds pad slots. Records are 32-bit (bit 31 centroid, bit 30
// uniform, bits 16..19 groups - 1, bits 0..15 first group or centroid chunk index).
// Lane L scans groups [128 L, 128 L + 128); the position inside a run at its first
// group comes from the trailing kept groups of the lanes before it (whole kept segments
// add 128 = 0 mod 8). At most 2048 token chunks (runs are separated by a dropped group
// and G <= 4096) plus 128 centroid chunks.
__device__ __forceinline__ uint32_t kept_word(const uint32_t* any, int w, int Wg, int g_lo, int g_hi) {
  if (w < 0 || w >= Wg) return 0u;
  uint32_t x = any[w];
  const int lo = g_lo - 32 * w, hi = g_hi - 32 * w;  // keep bits [lo, hi)
  if (hi <= 0 || lo >= 32) return 0u;
  if (hi < 32) x &= (1u << hi) - 1u;
  if (lo > 0) x &= ~((1u << lo) - 1u);
  return x;
}

__device__ int build_chunk_list(const uint32_t* any, const uint32_t* uni, int g_lo, int g_hi,
                                int Wg, const uint32_t* cneed, int ncc, uint32_t* list, int lane,
                                int gbase) {
  const int seg0 = 128 * lane;
  int tail = 0;  // trailing kept groups of this lane's segment
  for (int w = 4 * lane + 3; w >= 4 * lane; --w) {
    const uint32_t x = kept_word(any, w, Wg, g_lo, g_hi);
    if (x == 0xffffffffu) {
      tail += 32;
      continue;
    }
    tail += __clz(~x);
    break;
  }
  const unsigned nonfull = __ballot_sync(0xffffffffu, tail < 128);
  const int tail_prev = __shfl_up_sync(0xffffffffu, tail, 1);
  const unsigned before = nonfull & ((1u << lane) - 1u);
  const int src = before ? 31 - __clz(before) : 0;
  const int tail_src = __shfl_sync(0xffffffffu, tail, src);
  // groups of the run before this segment's first group, mod 8
  const int r0 = (lane > 0 && tail_prev > 0) ? ((before ? tail_src : 0) & 7) : 0;
  const int seg_end = min(seg0 + 128, g_hi);
  auto run_from = [&](int g) -> int {  // consecutive kept groups from g, at most 8
    const int w = g >> 5, sh = g & 31;
    const uint64_t win = ((static_cast<uint64_t>(kept_word(any, w + 1, Wg, g_lo, g_hi)) << 32) |
                          kept_word(any, w, Wg, g_lo, g_hi)) >> sh;
    const int run = __ffsll(static_cast<long long>(~win)) - 1;
    return (run < 0 || run > 8) ? 8 : run;
  };
  int total = 0, base = 0;
#pragma unroll 1
  for (int pass = 0; pass < 2; ++pass) {
    int g = seg0, r = r0, k = 0;
    while (g < seg_end) {
      const int w = g >> 5;
      uint32_t x = kept_word(any, w, Wg, g_lo, g_hi) & (0xffffffffu << (g & 31));
      if (!(x & (1u << (g & 31)))) {
        int ww = w;  // next kept group inside the segment
        while (x == 0u && ++ww < 4 * lane + 4) x = kept_word(any, ww, Wg, g_lo, g_hi);
        if (x == 0u) break;
        g = 32 * ww + __ffs(x) - 1;
        r = 0;
        if (g >= seg_end) break;
      }
      const int run = run_from(g);
      if (r == 0) {
        if (pass == 1) {
          const int wu = g >> 5, su = g & 31;
          const uint64_t uw = ((static_cast<uint64_t>(wu + 1 < Wg ? uni[wu + 1] : 0u) << 32) |
                               (wu < Wg ? uni[wu] : 0u)) >> su;
          const uint64_t m = (1ull << run) - 1ull;
          const uint32_t uniform = (uw & m) == m ? (1u << 30) : 0u;
          list[base + k] = uniform | (static_cast<uint32_t>(run - 1) << 16) | static_cast<uint32_t>(g + gbase);
        }
        ++k;
        g += run;
      } else {
        g += min(8 - r, run);
      }
      r = 0;
    }
    if (pass == 0) {  // exclusive prefix sum of the lanes' counts
      int incl = k;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      base = incl - k;
      total = __shfl_sync(0xffffffffu, incl, 31);
    }
  }
  int nc = total;  // centroid chunks after the token chunks, in index order
  for (int w = 0; w < 4 && 32 * w < ncc; ++w) {
    uint32_t bits = cneed[w];
    if (32 * w + 32 > ncc) bits &= (1u << (ncc - 32 * w)) - 1u;
    if ((bits >> lane) & 1u) list[nc + __popc(bits & ((1u << lane) - 1u))] = 0x80000000u | (32 * w + lane);
    nc += __popc(bits);
  }
  __syncwarp();
  return nc;
}

__device__ __forceinline__ Chunk decode_chunk(uint32_t rec) {
  Chunk c;
  c.centroid = rec >> 31;
  if (c.centroid) {
    c.start = static_cast<int>(rec & 0xffffu) * 128;
    c.n = 128;
    c.g0 = c.ng = 0;
    c.uniform = false;
  } else {
    c.g0 = static_cast<int>(rec & 0xffffu);
    c.ng = static_cast<int>((rec >> 16) & 0xfu) + 1;
    c.start = c.g0 * 16;
    c.n = c.ng * 16;
    c.uniform = (rec >> 30) & 1u;
  }
  return c;
}

// Pairs of every 8 whose exponentials use the FMA-pipe polynomial instead of MUFU ex2
// (the two CTAs' softmax warps share each sub-partition's MUFU). Measured at the video
// workload: 0 -> 8.15 ms, 1 -> 7.99 ms, 2 -> 8.21 ms per kernel.
constexpr int kPolyPairsOf8 = 1;

// Max of 16 / 64 register values as shallow trees of 3-input maxes.
__device__ __forceinline__ float max16(const float* v) {
  return fmaxf(max3(max3(v[0], v[1], v[2]), max3(v[3], v[4], v[5]), fmaxf(v[6], v[7])),
               max3(max3(v[8], v[9], v[10]), max3(v[11], v[12], v[13]), fmaxf(v[14], v[15])));
}
__device__ __forceinline__ float max64(const float (&a)[32], const float (&b)[32]) {
  return fmaxf(max3(max16(a), max16(a + 16), max16(b)), max16(b + 16));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

template <int D, bool TF32>
// 160 threads (control warp + 4 softmax warps); two CTAs share an SM.
__global__ void __launch_bounds__(160, 2)
    attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmKc,
                const __grid_constant__ CUtensorMap tmVc, const AttnArgs a) {
  using Cfg = AttnCfg<D, TF32>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sQ = smem_u32(smem), sK = sQ + Cfg::TILE, sV = sK + Cfg::TILE;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + 3 * Cfg::TILE);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + NBAR);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* n_distinct = reinterpret_cast<int*>(tmem_slot + 2);
  int* never = reinterpret_cast<int*>(tmem_slot + 3);
  int* distinct = reinterpret_cast<int*>(tmem_slot + 4);     // 128
  uint32_t* any_bits = reinterpret_cast<uint32_t*>(distinct + 128);  // 128 words
  uint32_t* uni_bits = any_bits + 128;                                // 128 words
  uint32_t* cneed = uni_bits + 128;                                   // 4 words
  int* nchunks = reinterpret_cast<int*>(cneed + 4);
  uint32_t* clist = reinterpret_cast<uint32_t*>(smem + 3 * Cfg::TILE + 2048);  // kChunkListCap

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tile = blockIdx.x / a.ksplit, split = blockIdx.x % a.ksplit;
  const int h = blockIdx.y, b = blockIdx.z;
  // this CTA's key groups [g_lo, g_hi); the centroid chunks belong to the last split
  // (ranges start on 32-group words; one range spans at most 4096 groups, the window of
  // the CTA's bitsets, which start at word wbase)
  const int g_lo = static_cast<int>((static_cast<int64_t>(a.G) * split) / a.ksplit) & ~31;
  const int g_hi = split + 1 == a.ksplit ? a.G
                                         : static_cast<int>((static_cast<int64_t>(a.G) * (split + 1)) / a.ksplit) & ~31;
  const int wbase = g_lo >> 5;
  const int hkv = h / (a.Hq / a.Hkv);
  const int slice = (a.b_sliced ? b : 0) * a.nh_slices + (a.h_sliced ? h : 0);
  const uint32_t bar0 = smem_u32(bars);
#define BAR(i) (bar0 + 8u * static_cast<uint32_t>(i))

  if (tid == 0) {
    for (int i = 0; i < NBAR; ++i) mbar_init(BAR(i), (i == BAR_PLO || i == BAR_PHI) ? 128u : 1u);
    *abort_flag = 0;
    *n_distinct = 0;
    *never = 0;
    fence_mbarrier_init();
  }
  if (tid == 0) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), 256);
    tmem_relinquish();
  }
  if (tid < 4) cneed[tid] = 0;
  __syncthreads();

  // Query clusters present in this tile (rows are sorted by label, pads last).
  if (tid < 128) {
    const int r = tile * 128 + tid;
    const int lab = a.qrow_label[r];
    const int prev = tid > 0 ? a.qrow_label[r - 1] : -2;
    if (lab >= 0 && lab != prev) distinct[atomicAdd(n_distinct, 1)] = lab;
  }
  __syncthreads();
  const int nd = *n_distinct;
  const uint32_t* gb = a.gbits + static_cast<size_t>(slice) * a.Cq * a.Wg;
  const uint32_t* cb = a.cbits + static_cast<size_t>(slice) * a.Cq * a.Wc;
  for (int w = tid; w < 128; w += blockDim.x) {
    uint32_t any = 0, all = 0;
    const int wa = wbase + w;  // absolute word
    if (wa < a.Wg && nd > 0) {
      all = 0xffffffffu;
      for (int i = 0; i < nd; ++i) {
        const uint32_t x = gb[static_cast<size_t>(distinct[i]) * a.Wg + wa];
        any |= x;
        all &= x;
      }
      all &= a.gfull[wa];
    }
    any_bits[w] = any;
    uni_bits[w] = all & any;
  }
  if (a.compensate) {
    for (int w = tid; w < a.Wc; w += blockDim.x) {
      uint32_t need = 0;
      for (int i = 0; i < nd; ++i) need |= ~cb[static_cast<size_t>(distinct[i]) * a.Wc + w];
      need &= a.cnonempty[w];
      if (need) atomicOr(&cneed[(w >> 2) >> 5], 1u << ((w >> 2) & 31));
    }
  }
  __syncthreads();
  const int ncc = (a.compensate && split == a.ksplit - 1) ? a.Ckpad / 128 : 0;
  if (warp == 1) {
    const int n = build_chunk_list(any_bits, uni_bits, g_lo - 32 * wbase, g_hi - 32 * wbase,
                                   min(128, a.Wg - wbase), cneed, ncc, clist, lane, 32 * wbase);
    if (lane == 0) *nchunks = n;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int nch = *nchunks;

  if (warp == 0) {
    // ------------------------------------------------ control warp: TMA + tcgen05.mma
    // The whole warp runs this loop on warp-uniform values, so MMA descriptors live in
    // uniform registers and each tcgen05.mma issues without per-lane conversion; lane
    // 0 alone issues the per-thread operations (TMA copies, expect_tx, commits). The
    // single K and V stages are refilled as soon as the MMA that read them completes,
    // while the softmax warps work on the current chunk.
    const bool leader = lane == 0;
    auto wait_all = [&](uint32_t bar, uint32_t parity, int where) -> bool {
      const bool r = mbar_wait(bar, parity, abort_flag, where);
      return __all_sync(0xffffffffu, r);
    };
    auto commit = [&](uint32_t bar) {
      if (elect_one()) tc_commit(bar);
      __syncwarp();
    };
    constexpr uint32_t kIdescQK = make_idesc(TF32, 128, 0, false, false);
    constexpr uint32_t kIdescPV = make_idesc(TF32, 128, D, false, true);
    // Base descriptors; a K-step only moves the start address (bits 0..13, in 16-byte
    // units), so each MMA adds a constant instead of rebuilding them.
    const uint64_t dQ = smem_desc(sQ, 16, 1024);
    const uint64_t dK = smem_desc(sK, 16, 1024);
    const uint64_t dV = TF32 ? smem_desc(sV, 16384, 512, kLayoutSW128Atom32B)
                             : smem_desc(sV, 16384, 1024, kLayoutSW128);
    const int qrow0 = (b * a.Hq + h) * a.Sqpad + tile * 128;
    const int krow0 = (b * a.Hkv + hkv) * a.kstride;
    const int crow0 = (b * a.Hkv + hkv) * a.Ckpad;
    auto load_kv = [&](const Chunk& c, bool is_v) {
      if (leader) {
        const CUtensorMap* m = c.centroid ? (is_v ? &tmVc : &tmKc) : (is_v ? &tmV : &tmK);
        const int row = (c.centroid ? crow0 : krow0) + c.start;
        const uint32_t dst = is_v ? sV : sK;
        const uint32_t bar = BAR(is_v ? BAR_VF : BAR_KF);
        mbar_arrive_expect_tx(bar, Cfg::TILE);
#pragma unroll
        for (int cc = 0; cc < Cfg::NATOM; ++cc) tma_load_2d(dst + cc * 16384, m, bar, cc * Cfg::ATOM, row);
      }
      __syncwarp();
    };
    int ci = 0, j = 0, nk = 0, nv = 0;
    auto next = [&](Chunk& c) -> bool {
      if (ci >= nch) return false;
      c = decode_chunk(clist[ci++]);
      return true;
    };
    Chunk cur, nxt, nn;
    bool have = next(cur);
    if (have) {
      load_kv(cur, false);
      ++nk;
      load_kv(cur, true);
      ++nv;
    }
    if (a.q_gather) {
      // the tile's 128 rows straight from the caller's q: lane L gathers rows 4L..4L+3
      // (their tokens through the row map; pad rows point past the last row and read
      // zeros), one tile::gather4 per 128-byte column chunk
      if (leader) mbar_arrive_expect_tx(BAR(BAR_Q), Cfg::TILE);
      __syncwarp();
      const int64_t qbase = (static_cast<int64_t>(b) * a.Hq + h) * a.Sq;
      const int oob = a.B * a.Hq * a.Sq;
      int rr[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int t = a.qrow_token[tile * 128 + 4 * lane + i];
        rr[i] = t >= 0 ? static_cast<int>(qbase + t) : oob;
      }
#pragma unroll
      for (int cc = 0; cc < Cfg::NATOM; ++cc)
        tma_gather4_2d(sQ + cc * 16384 + lane * 512, &tmQ, BAR(BAR_Q), cc * Cfg::ATOM, rr[0], rr[1],
                       rr[2], rr[3]);
      __syncwarp();
    } else {
      if (leader) {
        mbar_arrive_expect_tx(BAR(BAR_Q), Cfg::TILE);
#pragma unroll
        for (int cc = 0; cc < Cfg::NATOM; ++cc)
          tma_load_2d(sQ + cc * 16384, &tmQ, BAR(BAR_Q), cc * Cfg::ATOM, qrow0);
      }
      __syncwarp();
    }
    // S = Q Kᵀ for key columns [64h, 64h + n_h) of chunk c into TMEM columns 64h.. (N = n_h).
    auto issue_qk_half = [&](const Chunk& c, int hlf) {
      const int nh = min(64, c.n - 64 * hlf);
      if (nh > 0) {
        const uint32_t idesc = kIdescQK | (static_cast<uint32_t>(nh >> 3) << 17);
        const uint64_t krow = static_cast<uint64_t>((hlf * 64 * 128) >> 4);  // 64 rows of 128 B
        // one elected lane issues the half's K-steps back to back
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < D / Cfg::KSTEP; ++kk) {
            const uint64_t off = static_cast<uint64_t>(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4);
            mma_ss<TF32>(tmem + 64 * hlf, dQ + off, dK + off + krow, idesc, kk > 0 ? 1u : 0u);
          }
        }
        __syncwarp();
      }
    };
    // O += P V for key rows [64h, 64h + n_h); P of step h sits at TMEM columns 64h..
    // (bf16 pairs: 32 columns, fp32: 64). V is MN-major (d contiguous): 128-byte rows,
    // d chunks 16 KB apart; bf16 uses 8-row swizzle groups (1 KB), tf32 the
    // 32-byte-unit swizzle with 4-row groups; a K-step of KSTEP rows moves KSTEP*128 B.
    auto issue_pv_half = [&](const Chunk& c, int hlf, bool first_chunk) {
      constexpr int kHalfSteps = 64 / Cfg::KSTEP;
      const int nsteps = c.n / Cfg::KSTEP;
      if (elect_one()) {
#pragma unroll
        for (int t = 0; t < kHalfSteps; ++t) {
          const int kk = hlf * kHalfSteps + t;
          if (kk < nsteps)
            mma_ts<TF32>(tmem + 128, tmem + 64 * hlf + t * 8,
                         dV + static_cast<uint64_t>((kk * Cfg::KSTEP * 128) >> 4), kIdescPV,
                         (!first_chunk || kk > 0) ? 1u : 0u);
        }
      }
      __syncwarp();
    };
    bool ok = wait_all(BAR(BAR_Q), 0, 3);
    bool have_next = false, have_nn = false;
    int hi_c = 0;  // chunks with a high step whose P-high the control has waited for
    if (ok && have) {
      ok = wait_all(BAR(BAR_KF), 0, 5);
      if (ok) {
        tc_fence_after();
        issue_qk_half(cur, 0);
        commit(BAR(BAR_SFLO));
        if (cur.n > 64) {
          issue_qk_half(cur, 1);
          commit(BAR(BAR_SFHI));
        }
        commit(BAR(BAR_KE));
        have_next = next(nxt);
        if (have_next && (ok = wait_all(BAR(BAR_KE), 0, 1))) {
          load_kv(nxt, false);
          ++nk;
        }
      }
    }
    // Steady state for chunk j: PV-low(j) | QK-low(j+1) | PV-high(j) | QK-high(j+1), so
    // the tensor core works on the next chunk's low keys while the softmax warps are on
    // chunk j's high keys, and on the next chunk's high keys while they start chunk j+1.
    while (ok && have) {
      if (!(ok = wait_all(BAR(BAR_PLO), j & 1, 6))) break;
      if (!(ok = wait_all(BAR(BAR_VF), j & 1, 7))) break;
      tc_fence_after();
      issue_pv_half(cur, 0, j == 0);
      commit(BAR(BAR_OLO));
      if (have_next) {
        // MMAs of one thread run in issue order: QK-low(j+1) overwrites P-low(j) only
        // after PV-low(j) has read it.
        if (!(ok = wait_all(BAR(BAR_KF), (j + 1) & 1, 5))) break;
        tc_fence_after();
        issue_qk_half(nxt, 0);
        commit(BAR(BAR_SFLO));
      }
      // The high step exists only for chunks of more than 64 keys; its barriers count
      // those chunks alone (hi_c / hi_n), on both sides.
      if (cur.n > 64) {
        if (!(ok = wait_all(BAR(BAR_PHI), hi_c & 1, 8))) break;
        ++hi_c;
        tc_fence_after();
        issue_pv_half(cur, 1, j == 0);
      }
      commit(BAR(BAR_VE));
      have_nn = false;
      if (have_next) {
        if (nxt.n > 64) {
          issue_qk_half(nxt, 1);
          commit(BAR(BAR_SFHI));
        }
        commit(BAR(BAR_KE));
        // V stage: refill with the next chunk once PV(j) has read it
        if (!(ok = wait_all(BAR(BAR_VE), j & 1, 4))) break;
        load_kv(nxt, true);
        ++nv;
        // K stage: refill with the chunk after once QK(j+1) has read it
        have_nn = next(nn);
        if (have_nn) {
          if (!(ok = wait_all(BAR(BAR_KE), (j + 1) & 1, 1))) break;
          load_kv(nn, false);
          ++nk;
        }
      }
      cur = nxt;
      nxt = nn;
      have = have_next;
      have_next = have_nn;
      ++j;
    }
    commit(BAR(BAR_OF));
    // Before the CTA may exit: every issued copy has landed, every MMA has completed.
    commit(BAR(BAR_DRAIN));
    mbar_wait(BAR(BAR_DRAIN), 0, never, 23);
    mbar_wait(BAR(BAR_Q), 0, never, 20);
    if (nk) mbar_wait(BAR(BAR_KF), (nk - 1) & 1, never, 21);
    if (nv) mbar_wait(BAR(BAR_VF), (nv - 1) & 1, never, 22);
  } else {
    // ------------------------------------------------ softmax / epilogue (128 threads)
    // One thread per query row (warps 1..4; warp w reads TMEM lanes 32*(w%4)..+31).
    // Each chunk is taken as two online-softmax steps over key columns 0..63 and
    // 64..127; after the first the PV of those keys starts while the second runs.
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const int qrow = tile * 128 + r;
    const int lab = a.qrow_label[qrow];
    const int tok = a.qrow_token[qrow];
    const uint32_t* grow = gb + static_cast<size_t>(lab < 0 ? 0 : lab) * a.Wg;
    const uint32_t* crow = cb + static_cast<size_t>(lab < 0 ? 0 : lab) * a.Wc;
    const uint32_t tS = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const uint32_t tO = tS + 128;
    const float scl = a.scale_log2;
    float m_run = -INFINITY, l_run = 0.f;
    int j = 0, hi_n = 0;  // hi_n: high steps taken so far
    bool ok = true;
#pragma unroll 1
    for (int ci = 0; ci < nch; ++ci) {
      const Chunk ch = decode_chunk(clist[ci]);
      const int nsteps = ch.n > 64 ? 2 : 1;
      // Token chunks are masked per 16-key group (a key cluster is kept or dropped
      // whole): this row's keep bits for the chunk's groups, the groups holding pad
      // slots, and the warp's votes (whether no row, every row or some rows keep each
      // group). None of it depends on S, so it is read before S is ready.
      uint32_t kb8 = 0u, part8 = 0u, any8 = 0xffu, mixed8 = 0u;
      if (!ch.centroid) {
        const uint32_t present = (1u << ch.ng) - 1u;
        kb8 = present;
        if (!ch.uniform) {
          const int w = ch.g0 >> 5, sh = ch.g0 & 31;
          const bool two = w + 1 < a.Wg;
          const uint64_t kw = static_cast<uint64_t>(__ldg(grow + w)) |
                              (two ? static_cast<uint64_t>(__ldg(grow + w + 1)) << 32 : 0ull);
          const uint64_t fw = static_cast<uint64_t>(__ldg(a.gfull + w)) |
                              (two ? static_cast<uint64_t>(__ldg(a.gfull + w + 1)) << 32 : 0ull);
          kb8 = static_cast<uint32_t>(kw >> sh) & present;
          part8 = ~static_cast<uint32_t>(fw >> sh) & present;
        }
        if (lab < 0) kb8 = 0u;
        any8 = __reduce_or_sync(0xffffffffu, kb8);
        mixed8 = any8 & ~__reduce_and_sync(0xffffffffu, kb8);
      }
#pragma unroll 1
      for (int half = 0; half < nsteps; ++half) {
        const int c0 = half * 64;         // first key column of this step
        {
          if (!(ok = mbar_wait(BAR(half == 0 ? BAR_SFLO : BAR_SFHI), half == 0 ? (j & 1) : (hi_n & 1),
                               abort_flag, 9)))
            break;
          tc_fence_after();
          // Groups no row of the warp keeps get P = 0 without exponentials, groups every
          // row keeps need no select. Columns past a cluster's last token (pad slots of
          // its last group) and pad query rows are set to -inf. Centroid chunks are
          // masked per column and carry the log2 n_c bias.
          float v0[32], v1[32];
          tmem_ld32(tS + c0, v0);
          tmem_ld32(tS + c0 + 32, v1);
          uint32_t any4 = 0xfu;  // groups of this step whose exponentials the warp computes
          float mx;
          float sx = scl;        // exponent argument x = v * sx - m
          if (!ch.centroid) {
            const int gh0 = ch.g0 + half * 4;  // this step covers groups gh0 .. gh0+3
            const uint32_t kb = (kb8 >> (4 * half)) & 0xfu;
            const uint32_t partial = (part8 >> (4 * half)) & 0xfu;
            const uint32_t mixed = (mixed8 >> (4 * half)) & 0xfu;
            any4 = (any8 >> (4 * half)) & 0xfu;
            tmem_wait_ld();
            if (partial | mixed) {
              // -inf for the pad slots of a cluster's last group, and for rows that drop
              // a group another row of the warp keeps
#pragma unroll
              for (int jj = 0; jj < 4; ++jj) {
                float* v = jj < 2 ? v0 : v1;
                const int o = (jj & 1) * 16;
                if ((partial >> jj) & 1u) {
                  const int nv = __ldg(a.group_valid + gh0 + jj);
#pragma unroll
                  for (int c = 1; c < 16; ++c) v[o + c] = c < nv ? v[o + c] : -INFINITY;
                }
                if ((mixed >> jj) & 1u) {
                  const bool keep = (kb >> jj) & 1u;
#pragma unroll
                  for (int c = 0; c < 16; ++c) v[o + c] = keep ? v[o + c] : -INFINITY;
                }
              }
            }
            // raw logits; scale > 0, so the max of scale*s is scale*max(s)
            if (any4 == 0xfu) {
              mx = max64(v0, v1) * scl;
            } else {
              mx = -INFINITY;
#pragma unroll
              for (int jj = 0; jj < 4; ++jj)
                if ((any4 >> jj) & 1u) mx = fmaxf(mx, max16((jj < 2 ? v0 : v1) + (jj & 1) * 16));
              mx *= scl;
            }
          } else {
            uint32_t mk0 = 0u, mk1 = 0u;  // bit c: column c0 + c (+ 32) kept
            if (lab >= 0) {
              const int ww = (ch.start + c0) >> 5;
              mk0 = ww < a.Wc ? (~__ldg(crow + ww) & __ldg(a.cnonempty + ww)) : 0u;
              mk1 = ww + 1 < a.Wc ? (~__ldg(crow + ww + 1) & __ldg(a.cnonempty + ww + 1)) : 0u;
            }
            const float* bias = a.bias2 + ch.start + c0;
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c) {
              v0[c] = ((mk0 >> c) & 1u) ? fmaf(v0[c], scl, __ldg(bias + c)) : -INFINITY;
              v1[c] = ((mk1 >> c) & 1u) ? fmaf(v1[c], scl, __ldg(bias + 32 + c)) : -INFINITY;
            }
            mx = max64(v0, v1);
            sx = 1.f;  // log2-unit logits or -inf
          }
          // Lazy rescaling: the running max only moves when the step max exceeds it by
          // more than 8 (log2 units), so P stays below 256 and O is rarely touched.
          const bool need = mx > m_run + 8.f;
          const bool any_need = __any_sync(0xffffffffu, need);
          float alpha = 1.f;
          if (need) {
            alpha = ex2(m_run - mx);
            l_run *= alpha;
            m_run = mx;
          }
          const float neg_mu = (m_run == -INFINITY) ? 0.f : -m_run;
          // Two independent pair sums keep the add chain short. Groups no row of the
          // warp keeps are zero; the common all-groups case runs as straight-line code.
          float sa0 = 0.f, sa1 = 0.f, sb0 = 0.f, sb1 = 0.f;
          if (any4 == 0xfu) {
#pragma unroll
            for (int q = 0; q < 32; ++q) {
              float* v = q < 16 ? v0 : v1;
              const int c = (q & 15) * 2;
              float x0, x1;
              fma2(x0, x1, v[c], v[c + 1], sx, sx, neg_mu, neg_mu);
              if ((q & 7) < kPolyPairsOf8) {
                exp2_poly2<true>(v[c], v[c + 1], x0, x1);
              } else {
                v[c] = ex2(x0);
                v[c + 1] = ex2(x1);
              }
              if (q & 1) add2(sb0, sb1, sb0, sb1, v[c], v[c + 1]);
              else add2(sa0, sa1, sa0, sa1, v[c], v[c + 1]);
            }
          } else {
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
              float* v = jj < 2 ? v0 : v1;
              const int o = (jj & 1) * 16;
              if ((any4 >> jj) & 1u) {
#pragma unroll
                for (int p = 0; p < 8; ++p) {
                  const int c = o + 2 * p;
                  float x0, x1;
                  fma2(x0, x1, v[c], v[c + 1], sx, sx, neg_mu, neg_mu);
                  v[c] = ex2(x0);
                  v[c + 1] = ex2(x1);
                  if (p & 1) add2(sb0, sb1, sb0, sb1, v[c], v[c + 1]);
                  else add2(sa0, sa1, sa0, sa1, v[c], v[c + 1]);
                }
              } else {
#pragma unroll
                for (int c = 0; c < 16; ++c) v[o + c] = 0.f;
              }
            }
          }
          l_run += (sa0 + sa1) + (sb0 + sb1);
          // P over S in place: bf16 pairs of step h in columns [64h, 64h+32) (step 0's
          // S columns were read above; step 1 lands on its own S columns), fp32 in the
          // step's own 64 columns.
          if constexpr (TF32) {
            tmem_st32(tS + c0, *reinterpret_cast<uint32_t(*)[32]>(v0));
            tmem_st32(tS + c0 + 32, *reinterpret_cast<uint32_t(*)[32]>(v1));
          } else {
            uint32_t* w0 = reinterpret_cast<uint32_t*>(v0);
            uint32_t* w1 = reinterpret_cast<uint32_t*>(v1);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              w0[i] = pack_bf16x2(v0[2 * i], v0[2 * i + 1]);
              w1[i] = pack_bf16x2(v1[2 * i], v1[2 * i + 1]);
            }
            tmem_st16(tS + c0, w0);
            tmem_st16(tS + c0 + 16, w1);
          }
          // O follows the running max before this step's PV adds to it. Step 0: wait
          // for the last PV of the previous chunk; step 1: for the PV of step 0.
          if (any_need && j > 0) {
            if (!(ok = mbar_wait(BAR(half == 0 ? BAR_VE : BAR_OLO), half == 0 ? ((j - 1) & 1) : (j & 1),
                                 abort_flag, 12)))
              break;
            tc_fence_after();
#pragma unroll 1
            for (int p = 0; p < D / 32; ++p) {
              float o[32];
              tmem_ld32(tO + p * 32, o);
              tmem_wait_ld();
#pragma unroll
              for (int c = 0; c < 32; ++c) o[c] *= alpha;
              tmem_st32(tO + p * 32, *reinterpret_cast<uint32_t(*)[32]>(o));
            }
          } else if (any_need && half == 1 && j == 0) {
            // first chunk: the PV of step 0 wrote O without accumulation; rescale it too
            if (!(ok = mbar_wait(BAR(BAR_OLO), 0, abort_flag, 12))) break;
            tc_fence_after();
#pragma unroll 1
            for (int p = 0; p < D / 32; ++p) {
              float o[32];
              tmem_ld32(tO + p * 32, o);
              tmem_wait_ld();
#pragma unroll
              for (int c = 0; c < 32; ++c) o[c] *= alpha;
              tmem_st32(tO + p * 32, *reinterpret_cast<uint32_t(*)[32]>(o));
            }
          }
          tmem_wait_st();
        }
        tc_fence_before();
        mbar_arrive(BAR(half == 0 ? BAR_PLO : BAR_PHI));
        hi_n += half;
      }
      if (!ok) break;
      ++j;
    }
    const bool o_final = ok && mbar_wait(BAR(BAR_OF), 0, abort_flag, 10);
    if (o_final && a.ksplit > 1) {
      // one key range of several: unnormalised O plus running max and sum, merged later
      tc_fence_after();
      const size_t prow = (((static_cast<size_t>(b) * a.Hq + h) * a.ksplit + split) * a.Sqpad) + qrow;
      float* po = a.part + prow * D;
      float* pml = a.part + static_cast<size_t>(a.B) * a.Hq * a.ksplit * a.Sqpad * D + prow * 2;
#pragma unroll 1
      for (int p = 0; p < D / 32; ++p) {
        float o[32];
        tmem_ld32(tO + p * 32, o);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 8; ++i)
          *reinterpret_cast<float4*>(po + p * 32 + 4 * i) =
              make_float4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
      }
      pml[0] = m_run;
      pml[1] = l_run;
    } else if (o_final) {
      tc_fence_after();
      const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
      float* orow = a.out + ((static_cast<size_t>(b) * a.Hq + h) * a.Sq + (tok >= 0 ? tok : 0)) * D;
#pragma unroll 1
      for (int p = 0; p < D / 32; ++p) {
        float o[32];
        tmem_ld32(tO + p * 32, o);
        tmem_wait_ld();
        if (tok >= 0) {
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            float4 v4 = l_run > 0.f ? make_float4(o[4 * i] * inv, o[4 * i + 1] * inv,
                                                  o[4 * i + 2] * inv, o[4 * i + 3] * inv)
                                    : make_float4(0.f, 0.f, 0.f, 0.f);
            *reinterpret_cast<float4*>(orow + p * 32 + 4 * i) = v4;
          }
        }
      }
    }
  }
#undef BAR
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}


// Merge of the key-range splits of one query row (one warp per row, grid (ceil(Sqpad / 8),
// Hq, B), 256 threads): m = max_s m_s, l = sum_s l_s 2^(m_s - m),
// O = sum_s O_s 2^(m_s - m) / l, written to the row's token position (log2 units, as
// the kernel keeps them). A row no split saw (l = 0) is written as zeros.
template <int D>
__global__ void __launch_bounds__(256) combine_splits_kernel(const float* __restrict__ part,
                                                             const int32_t* __restrict__ qrow_token,
                                                             int B, int Hq, int ksplit, int Sqpad,
                                                             int Sq, float* __restrict__ out) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qrow = blockIdx.x * 8 + warp;
  const int h = blockIdx.y, b = blockIdx.z;
  if (qrow >= Sqpad) return;
  const int tok = qrow_token[qrow];
  if (tok < 0) return;
  const size_t bhs = (static_cast<size_t>(b) * Hq + h) * ksplit;
  const float* ml = part + static_cast<size_t>(B) * Hq * ksplit * Sqpad * D;
  // the splits' maxima and sums read by the lanes side by side (lane s, s + 32, ...)
  float m = -INFINITY;
  for (int s = lane; s < ksplit; s += 32) m = fmaxf(m, ml[((bhs + s) * Sqpad + qrow) * 2]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  float l = 0.f, acc[D / 32];
#pragma unroll
  for (int e = 0; e < D / 32; ++e) acc[e] = 0.f;
  for (int s0 = 0; s0 < ksplit; s0 += 32) {
    // weight of split s0 + lane (0 for a split that saw no key of this row)
    float f = 0.f;
    if (s0 + lane < ksplit) {
      const size_t prow = (bhs + s0 + lane) * Sqpad + qrow;
      const float ls = ml[prow * 2 + 1];
      if (ls > 0.f) {
        f = exp2f(ml[prow * 2] - m);
        l = fmaf(ls, f, l);
      }
    }
    const int ns = min(32, ksplit - s0);
#pragma unroll 4
    for (int t = 0; t < ns; ++t) {
      const float ft = __shfl_sync(0xffffffffu, f, t);
      if (ft > 0.f) {  // a split that saw no key of this row left its partial row unset
        const size_t prow = (bhs + s0 + t) * Sqpad + qrow;
#pragma unroll
        for (int e = 0; e < D / 32; ++e) acc[e] = fmaf(part[prow * D + e * 32 + lane], ft, acc[e]);
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
  const float inv = l > 0.f ? 1.f / l : 0.f;
  float* orow = out + ((static_cast<size_t>(b) * Hq + h) * Sq + tok) * D;
#pragma unroll
  for (int e = 0; e < D / 32; ++e) orow[e * 32 + lane] = acc[e] * inv;
}

// ============================================================== host side
namespace {

struct AttnLayout {
  int Sqpad, Skpad, G, Wg, Ckpad, Wc, Cqpad;
  int ksplit;   // CTAs per query tile over disjoint key ranges (1 = no split)
  float* part;  // ksplit > 1: partial O (B,Hq,ksplit,Sqpad,D), then max and sum (...,2)
  int32_t *qrow_token, *qrow_label, *qsort_token, *qsort_label, *q_count, *q_off;
  int32_t* plan_scratch;  // query tile plan: 5 * Cq ints
  int q_gather;     // the kernel gathers Q rows itself (no permuted copy)
  int32_t *kslot_token, *group_cluster, *group_valid, *k_count, *k_off;
  int32_t* korder;  // slot-layout order of the key clusters
  float* bias2;
  uint32_t *cnonempty, *cbits, *gbits, *gfull;
  void *qp, *kp, *vp, *kc, *vc;
  size_t bytes;
};

AttnLayout carve(const bsa_shape& s, int Cq, int Ck, void* ws) {
  AttnLayout L{};
  const int es = s.dtype == BSA_F32 ? 4 : 2;
  L.Sqpad = ceil_div(s.Sq, 128) * 128;
  L.Skpad = ceil_div(s.Sk + 15 * Ck, 128) * 128;
  L.G = L.Skpad / 16;
  L.Wg = ceil_div(L.G, 32);
  L.Ckpad = ceil_div(Ck, 128) * 128;
  L.Wc = ceil_div(Ck, 32);
  Carver cv(ws);
  L.qrow_token = cv.take<int32_t>(L.Sqpad);
  L.qrow_label = cv.take<int32_t>(L.Sqpad);
  L.qsort_token = cv.take<int32_t>(L.Sqpad);
  L.qsort_label = cv.take<int32_t>(L.Sqpad);
  L.plan_scratch = cv.take<int32_t>(static_cast<size_t>(5) * Cq);
  L.q_count = cv.take<int32_t>(Cq);
  L.q_off = cv.take<int32_t>(Cq + 1);
  L.kslot_token = cv.take<int32_t>(L.Skpad);
  L.group_cluster = cv.take<int32_t>(L.G);
  L.group_valid = cv.take<int32_t>(L.G);
  L.k_count = cv.take<int32_t>(Ck);
  L.k_off = cv.take<int32_t>(Ck + 1);
  L.korder = cv.take<int32_t>(Ck);
  L.bias2 = cv.take<float>(L.Ckpad);
  L.cnonempty = cv.take<uint32_t>(L.Wc);
  const size_t slices = static_cast<size_t>(s.B) * s.Hq;
  L.cbits = cv.take<uint32_t>(slices * Cq * L.Wc);
  L.gbits = cv.take<uint32_t>(slices * Cq * L.Wg);
  L.gfull = cv.take<uint32_t>(L.Wg);
  // Q rows are gathered straight from the caller's q by the attention kernel whenever
  // every row index fits a TMA coordinate; otherwise a cluster-major copy is made.
  L.q_gather = static_cast<int64_t>(s.B) * s.Hq * s.Sq < (int64_t(1) << 31) - 1;
  L.qp = L.q_gather ? nullptr
                    : cv.take<uint8_t>(static_cast<size_t>(s.B) * s.Hq * L.Sqpad * s.D * es);
  L.kp = cv.take<uint8_t>(static_cast<size_t>(s.B) * s.Hkv * L.Skpad * s.D * es);
  L.vp = cv.take<uint8_t>(static_cast<size_t>(s.B) * s.Hkv * L.Skpad * s.D * es);
  L.kc = cv.take<uint8_t>(static_cast<size_t>(s.B) * s.Hkv * L.Ckpad * s.D * es);
  L.vc = cv.take<uint8_t>(static_cast<size_t>(s.B) * s.Hkv * L.Ckpad * s.D * es);
  // Key-range split when the query tiles alone leave most of the GPU idle (e.g. the
  // 64 probe rows per head): about 2 CTAs per SM of a 148-SM part, each split at least
  // 8 key groups (128 keys), at most 16 splits.
  const int64_t ctas = static_cast<int64_t>(L.Sqpad / 128) * s.Hq * s.B;
  int ks = ctas >= 148 ? 1 : static_cast<int>(296 / ctas);
  ks = std::min(ks, std::min(16, L.G / 8));
  // one CTA's key range spans at most 4096 groups (its bitset window); longer key
  // sequences are always split (ranges start on 32-group words)
  ks = std::max(ks, ceil_div(L.G, 4064));
  L.ksplit = std::max(ks, 1);
  L.part = L.ksplit > 1 ? cv.take<float>(static_cast<size_t>(s.B) * s.Hq * L.ksplit * L.Sqpad * (s.D + 2))
                        : nullptr;
  L.bytes = align_up(cv.used, 256);
  return L;
}

template <int D, bool TF32>
int launch_attn(const CUtensorMap* maps, const AttnArgs& args, dim3 grid, int prof_id,
                cudaStream_t st) {
  using Cfg = AttnCfg<D, TF32>;
  auto kern = attn_kernel<D, TF32>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       Cfg::SMEM_LAUNCH);
  if (e != cudaSuccess) return check_cuda(e, "cudaFuncSetAttribute(attn_kernel)");
  prof_begin(prof_id, st);
  kern<<<grid, 160, Cfg::SMEM_LAUNCH, st>>>(maps[0], maps[1], maps[2], maps[3], maps[4], args);
  count_launch();
  if (args.ksplit > 1) {
    combine_splits_kernel<D><<<dim3((args.Sqpad + 7) / 8, args.Hq, args.B), 256, 0, st>>>(
        args.part, args.qrow_token, args.B, args.Hq, args.ksplit, args.Sqpad, args.Sq, args.out);
    count_launch();
  }
  prof_end(prof_id, st);
  return check_cuda(cudaGetLastError(), "attn_kernel launch");
}

}  // namespace

int validate_attention_shape(const bsa_shape& s, int Cq, int Ck) {
  if (s.B <= 0 || s.Hq <= 0 || s.Hkv <= 0 || s.Sq <= 0 || s.Sk <= 0)
    return fail(BSA_ERR_INVALID_ARG, "non-positive shape");
  if (s.Hq % s.Hkv) return fail(BSA_ERR_INVALID_ARG, "Hq (%d) not a multiple of Hkv (%d)", s.Hq, s.Hkv);
  if (s.D != 64 && s.D != 128) return fail(BSA_ERR_UNSUPPORTED, "head dim %d not in {64,128}", s.D);
  if (s.dtype != BSA_BF16 && s.dtype != BSA_F32) return fail(BSA_ERR_UNSUPPORTED, "dtype %d", s.dtype);
  if (Cq <= 0 || Ck <= 0 || Cq > 16384 || Ck > 16384)
    return fail(BSA_ERR_UNSUPPORTED, "cluster counts Cq=%d Ck=%d outside [1,16384]", Cq, Ck);
  // chunk records hold a 16-bit first key group: at most 65536 groups of 16 slots
  if (static_cast<int64_t>(s.Sk) + 15LL * Ck > (int64_t(1) << 20) - 128)
    return fail(BSA_ERR_UNSUPPORTED, "Sk + 15*Ck = %lld exceeds %lld",
                static_cast<long long>(s.Sk) + 15LL * Ck, static_cast<long long>((1 << 20) - 128));
  // row indices of the query maps, the key maps and the split partials fit 32 bits
  const int64_t sqpad = (static_cast<int64_t>(s.Sq) + 127) / 128 * 128;
  const int64_t skpad = (static_cast<int64_t>(s.Sk) + 15LL * Ck + 127) / 128 * 128;
  if (static_cast<int64_t>(s.B) * s.Hq * sqpad * 16 >= (int64_t(1) << 31) ||
      static_cast<int64_t>(s.B) * s.Hkv * skpad >= (int64_t(1) << 31))
    return fail(BSA_ERR_UNSUPPORTED, "B*Hq*Sq or B*Hkv*Sk too large for 32-bit row indices");
  return BSA_OK;
}

size_t attention_workspace_bytes(const bsa_shape& s, int Cq, int Ck) {
  return carve(s, Cq, Ck, nullptr).bytes;
}

// One or two label sorts in one launch (one CTA each).
static int launch_label_sorts(const LabelSortJob& j0, const LabelSortJob* j1, cudaStream_t st) {
  const int smem = j1 && label_sort_smem(j1->C) > label_sort_smem(j0.C) ? label_sort_smem(j1->C)
                                                                        : label_sort_smem(j0.C);
  cudaError_t e = cudaFuncSetAttribute(label_sort_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       smem > 48 * 1024 ? smem : 48 * 1024);
  if (e != cudaSuccess) return check_cuda(e, "cudaFuncSetAttribute(label_sort)");
  label_sort_kernel<<<j1 ? 2 : 1, 1024, smem, st>>>(j0, j1 ? *j1 : j0);
  count_launch();
  return check_cuda(cudaGetLastError(), "label_sort_kernel launch");
}

int run_label_sort(const int32_t* labels, int S, int C, int cluster_pad, int n_slots,
                   int32_t* slot_token, int32_t* slot_label, int32_t* count, int32_t* off,
                   int32_t* group_cluster, int32_t* group_valid, int n_groups, float* bias2,
                   int C_pad, uint32_t* nonempty, cudaStream_t st) {
  const LabelSortJob j{labels,        S,           C,     cluster_pad,   n_slots, slot_token,
                       slot_label,    count,       off,   group_cluster, group_valid,
                       n_groups,      bias2,       C_pad, nonempty};
  return launch_label_sorts(j, nullptr, st);
}

int centroid_compensated_attention(const void* q, const void* k, const void* v,
                                   const bsa_shape& s, const int32_t* q_labels, int Cq,
                                   const int32_t* k_labels, int Ck, const uint8_t* mask,
                                   int64_t mbs, int64_t mhs, float scale, int compensate,
                                   float* out, void* ws, size_t ws_bytes, cudaStream_t st,
                                   int prof_id, bool dense, bool reuse_plan) {
  int rc = validate_attention_shape(s, Cq, Ck);
  if (rc) return rc;
  if (!q || !k || !v || !q_labels || !k_labels || !mask || !out)
    return fail(BSA_ERR_INVALID_ARG, "null pointer argument");
  if (mbs < 0 || mhs < 0) return fail(BSA_ERR_INVALID_ARG, "negative mask stride");
  AttnLayout L = carve(s, Cq, Ck, ws);
  if (!ws || ws_bytes < L.bytes)
    return fail(BSA_ERR_WORKSPACE, "workspace %zu bytes < required %zu", ws_bytes, L.bytes);
  if (reinterpret_cast<uintptr_t>(ws) % 256)
    return fail(BSA_ERR_INVALID_ARG, "workspace not 256-byte aligned");
  const int es = s.dtype == BSA_F32 ? 4 : 2;
  if ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) |
       reinterpret_cast<uintptr_t>(v)) % 16)
    return fail(BSA_ERR_INVALID_ARG, "q/k/v must be 16-byte aligned");

  const int nb = mbs ? s.B : 1, nh = mhs ? s.Hq : 1;
  if (dense) {
    // every query row keeps every key: identities instead of steps 1-3
    if (Cq != 1 || Ck != 1 || compensate || mbs || mhs)
      return fail(BSA_ERR_INVALID_ARG, "dense preparation needs one cluster each, no compensation");
    const int n = std::max(L.Sqpad, L.Skpad);
    dense_prep_kernel<<<(n + 255) / 256, 256, 0, st>>>(
        s.Sq, L.Sqpad, s.Sk, L.Skpad, L.G, L.Wg, L.Ckpad, L.qrow_token, L.qrow_label, L.kslot_token,
        L.group_cluster, L.group_valid, L.k_count, L.k_off, L.cbits, L.gbits, L.gfull, L.cnonempty,
        L.bias2);
    count_launch();
    if ((rc = check_cuda(cudaGetLastError(), "dense_prep_kernel"))) return rc;
  } else if (!reuse_plan) {
  // Steps 1-3 depend only on the labels and the mask: a call that reuses the plan of an
  // earlier call on this workspace (same shape, labels, mask) skips them.
  // 1. cluster bitsets of the mask (label order)
  mask_cbits_kernel<<<dim3(Cq, nh, nb), 256, 0, st>>>(mask, mbs, mhs, nh, Cq, Ck, L.Wc, L.cbits);
  count_launch();
  if ((rc = check_cuda(cudaGetLastError(), "mask_cbits_kernel"))) return rc;
  // 2. key cluster order + key label sort (CTA 0) beside query label sort + query tile
  //    plan (CTA 1)
  {
    KeyOrderArgs ka{L.cbits, nb * nh, Cq, Ck, L.Wc, 0, L.korder};
    const size_t ko_bytes = key_order_smem(Cq, Ck);
    ka.chain = Ck <= kChainMax && ko_bytes <= 200 * 1024 ? 1 : 0;
    LabelSortJob jk{k_labels,       s.Sk,           Ck,      16,         L.Skpad,
                    L.kslot_token,  nullptr,        L.k_count, L.k_off,  L.group_cluster,
                    L.group_valid,  L.G,            L.bias2, L.Ckpad,    L.cnonempty};
    jk.order = L.korder;
    const LabelSortJob jq{q_labels, s.Sq,    Cq,      1,       L.Sqpad, L.qsort_token, L.qsort_label,
                          L.q_count, L.q_off, nullptr, nullptr, 0,       nullptr,      0,
                          nullptr};
    PlanArgs pa{};
    pa.sort_token = L.qsort_token;
    pa.sort_label = L.qsort_label;
    pa.count = L.q_count;
    pa.off = L.q_off;
    pa.cbits = L.cbits;
    pa.n_slices = nb * nh;
    pa.Cq = Cq;
    pa.Wc = L.Wc;
    pa.Sqpad = L.Sqpad;
    const size_t plan_bytes = plan_smem(Cq, L.Wc);
    pa.chain = plan_bytes <= 200 * 1024 ? 1 : 0;
    pa.row_token = L.qrow_token;
    pa.row_label = L.qrow_label;
    pa.scratch = L.plan_scratch;
    size_t smem = std::max(label_sort_smem(Ck), label_sort_smem(Cq));
    if (ka.chain) smem = std::max(smem, ko_bytes);
    if (pa.chain) smem = std::max(smem, plan_bytes);
    cudaError_t e = cudaFuncSetAttribute(prep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         smem > 48 * 1024 ? static_cast<int>(smem) : 48 * 1024);
    if (e != cudaSuccess) return check_cuda(e, "cudaFuncSetAttribute(prep_kernel)");
    prep_kernel<<<2, 1024, smem, st>>>(ka, jk, jq, pa);
    count_launch();
    if ((rc = check_cuda(cudaGetLastError(), "prep_kernel"))) return rc;
  }
  // 3. key-group bitsets (slot layout)
  mask_gbits_kernel<<<dim3(Cq, nb * nh), 256, 0, st>>>(L.cbits, Cq, L.Wc, L.group_cluster,
                                                       L.group_valid, L.G, L.Wg, L.gbits, L.gfull);
  count_launch();
  if ((rc = check_cuda(cudaGetLastError(), "mask_gbits_kernel"))) return rc;
  }
  // 4. Q gather (only when the kernel cannot gather the rows itself)
  const int vpr = s.D * es / 16;
  if (!L.q_gather) {
    const int64_t n = static_cast<int64_t>(L.Sqpad) * vpr;
    gather_rows_kernel<<<dim3(static_cast<unsigned>((n + 255) / 256), s.Hq, s.B), 256, 0, st>>>(
        static_cast<const uint4*>(q), static_cast<uint4*>(L.qp), L.qrow_token, s.Sq, L.Sqpad, vpr,
        s.Hq);
    count_launch();
    if ((rc = check_cuda(cudaGetLastError(), "gather_rows_kernel"))) return rc;
  }
  // 5. K/V gather + centroids. One key cluster without compensation (the probe path)
  //    permutes nothing and needs no centroid: the K/V maps then read the caller's
  //    tensors directly (key slot = token, rows per head = Sk).
  const bool kv_identity = Ck == 1 && !compensate && s.Sk % 16 == 0;
  if (!kv_identity) {
    if (s.dtype == BSA_F32) {
      gather_kv_centroids_kernel<float><<<dim3(L.Ckpad, s.Hkv, s.B), 256, 0, st>>>(
          static_cast<const float*>(k), static_cast<const float*>(v), static_cast<float*>(L.kp),
          static_cast<float*>(L.vp), static_cast<float*>(L.kc), static_cast<float*>(L.vc),
          L.kslot_token, L.k_count, L.k_off, s.Sk, L.Skpad, Ck, L.Ckpad, s.D, s.Hkv);
      count_launch();
    } else {
      gather_kv_centroids_kernel<__nv_bfloat16><<<dim3(L.Ckpad, s.Hkv, s.B), 256, 0, st>>>(
          static_cast<const __nv_bfloat16*>(k), static_cast<const __nv_bfloat16*>(v),
          static_cast<__nv_bfloat16*>(L.kp), static_cast<__nv_bfloat16*>(L.vp),
          static_cast<__nv_bfloat16*>(L.kc), static_cast<__nv_bfloat16*>(L.vc), L.kslot_token,
          L.k_count, L.k_off, s.Sk, L.Skpad, Ck, L.Ckpad, s.D, s.Hkv);
      count_launch();
    }
    if ((rc = check_cuda(cudaGetLastError(), "gather_kv_centroids_kernel"))) return rc;
  }

  // 6. tensor maps + attention
  const CUtensorMapDataType tdt =
      s.dtype == BSA_F32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const uint32_t atom = 128 / es;
  // V tiles feed the MMA as MN-major operands; for tf32 those must use the 32-byte-unit
  // 128-byte swizzle, the other tiles use the 16-byte-unit one.
  const CUtensorMapSwizzle vsw =
      s.dtype == BSA_F32 ? CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B : CU_TENSOR_MAP_SWIZZLE_128B;
  CUtensorMap maps[5];
  if ((rc = L.q_gather
                ? make_tmap_2d(&maps[0], q, tdt, es, static_cast<uint64_t>(s.B) * s.Hq * s.Sq, s.D, 1, atom)
                : make_tmap_2d(&maps[0], L.qp, tdt, es, static_cast<uint64_t>(s.B) * s.Hq * L.Sqpad, s.D, 128,
                               atom)) ||
      (rc = make_tmap_2d(&maps[1], kv_identity ? k : L.kp, tdt, es,
                         static_cast<uint64_t>(s.B) * s.Hkv * (kv_identity ? s.Sk : L.Skpad), s.D, 128, atom)) ||
      (rc = make_tmap_2d(&maps[2], kv_identity ? v : L.vp, tdt, es,
                         static_cast<uint64_t>(s.B) * s.Hkv * (kv_identity ? s.Sk : L.Skpad), s.D, 128, atom, vsw)) ||
      (rc = make_tmap_2d(&maps[3], L.kc, tdt, es, static_cast<uint64_t>(s.B) * s.Hkv * L.Ckpad, s.D, 128, atom)) ||
      (rc = make_tmap_2d(&maps[4], L.vc, tdt, es, static_cast<uint64_t>(s.B) * s.Hkv * L.Ckpad, s.D, 128, atom, vsw)))
    return rc;
  AttnArgs args{};
  args.B = s.B;
  args.Hq = s.Hq;
  args.Hkv = s.Hkv;
  args.Sq = s.Sq;
  args.Sqpad = L.Sqpad;
  args.Skpad = L.Skpad;
  args.kstride = kv_identity ? s.Sk : L.Skpad;
  args.q_gather = L.q_gather;
  args.Ck = Ck;
  args.Ckpad = L.Ckpad;
  args.Cq = Cq;
  args.G = L.G;
  args.Wg = L.Wg;
  args.Wc = L.Wc;
  args.nh_slices = nh;
  args.b_sliced = mbs ? 1 : 0;
  args.h_sliced = mhs ? 1 : 0;
  args.compensate = compensate ? 1 : 0;
  const float sc = scale > 0.f ? scale : 1.f / std::sqrt(static_cast<float>(s.D));
  args.scale_log2 = sc * 1.4426950408889634f;
  args.qrow_token = L.qrow_token;
  args.qrow_label = L.qrow_label;
  args.group_valid = L.group_valid;
  args.cbits = L.cbits;
  args.gbits = L.gbits;
  args.gfull = L.gfull;
  args.cnonempty = L.cnonempty;
  args.bias2 = L.bias2;
  args.out = out;
  args.ksplit = L.ksplit;
  args.part = L.part;
  const dim3 grid((L.Sqpad / 128) * L.ksplit, s.Hq, s.B);
  if (s.dtype == BSA_F32) {
    return s.D == 64 ? launch_attn<64, true>(maps, args, grid, prof_id, st)
                     : launch_attn<128, true>(maps, args, grid, prof_id, st);
  }
  return s.D == 64 ? launch_attn<64, false>(maps, args, grid, prof_id, st)
                   : launch_attn<128, false>(maps, args, grid, prof_id, st);
}

}  // namespace bsa

extern "C" size_t bsa_attention_workspace_bytes(bsa_shape shape, int Cq, int Ck) {
  if (bsa::validate_attention_shape(shape, Cq, Ck)) return 0;
  return bsa::attention_workspace_bytes(shape, Cq, Ck);
}

extern "C" int bsa_centroid_compensated_attention(const void* q, const void* k, const void* v,
                                                  bsa_shape shape, const int32_t* q_labels, int Cq,
                                                  const int32_t* k_labels, int Ck,
                                                  const uint8_t* block_mask, int64_t mask_b_stride,
                                                  int64_t mask_h_stride, float scale, int compensate,
                                                  float* out, void* workspace,
                                                  size_t workspace_bytes, void* stream) {
  return bsa::centroid_compensated_attention(q, k, v, shape, q_labels, Cq, k_labels, Ck, block_mask,
                                             mask_b_stride, mask_h_stride, scale, compensate, out,
                                             workspace, workspace_bytes, bsa::as_stream(stream),
                                             bsa::kProfAttention, false, false);
}

extern "C" int bsa_centroid_compensated_attention_ex(
    const void* q, const void* k, const void* v, bsa_shape shape, const int32_t* q_labels, int Cq,
    const int32_t* k_labels, int Ck, const uint8_t* block_mask, int64_t mask_b_stride,
    int64_t mask_h_stride, float scale, int compensate, float* out, void* workspace,
    size_t workspace_bytes, int flags, void* stream) {
  if (flags & ~BSA_REUSE_PLAN) return bsa::fail(BSA_ERR_INVALID_ARG, "unknown flags 0x%x", flags);
  return bsa::centroid_compensated_attention(q, k, v, shape, q_labels, Cq, k_labels, Ck, block_mask,
                                             mask_b_stride, mask_h_stride, scale, compensate, out,
                                             workspace, workspace_bytes, bsa::as_stream(stream),
                                             bsa::kProfAttention, false,
                                             (flags & BSA_REUSE_PLAN) != 0);
}

namespace bsa {
namespace {
// One (batch, KV head) problem of the per-KV-head call: its G query heads and one KV head.
bsa_shape kv_head_problem(const bsa_shape& s) {
  bsa_shape p = s;
  p.B = 1;
  p.Hkv = 1;
  p.Hq = s.Hkv > 0 ? s.Hq / s.Hkv : s.Hq;
  return p;
}
}  // namespace
}  // namespace bsa

extern "C" size_t bsa_per_kv_head_attention_workspace_bytes(bsa_shape shape, int Cq, int Ck) {
  if (shape.B <= 0 || shape.Hkv <= 0 || shape.Hq <= 0 || shape.Hq % shape.Hkv) return 0;
  return bsa_attention_workspace_bytes(bsa::kv_head_problem(shape), Cq, Ck);
}

extern "C" int bsa_per_kv_head_attention(const void* q, const void* k, const void* v, bsa_shape shape,
                                         const int32_t* q_labels, int Cq, const int32_t* k_labels,
                                         int Ck, const uint8_t* block_mask, int64_t mask_b_stride,
                                         int64_t mask_g_stride, float scale, int compensate, float* out,
                                         void* workspace, size_t workspace_bytes, void* stream) {
  using namespace bsa;
  if (shape.B <= 0 || shape.Hkv <= 0 || shape.Hq <= 0 || shape.Sq <= 0 || shape.Sk <= 0)
    return fail(BSA_ERR_INVALID_ARG, "non-positive shape");
  if (shape.Hq % shape.Hkv)
    return fail(BSA_ERR_INVALID_ARG, "Hq (%d) not a multiple of Hkv (%d)", shape.Hq, shape.Hkv);
  if (!q || !k || !v || !q_labels || !k_labels || !block_mask || !out)
    return fail(BSA_ERR_INVALID_ARG, "null pointer argument");
  if (mask_b_stride < 0 || mask_g_stride < 0) return fail(BSA_ERR_INVALID_ARG, "negative mask stride");
  const bsa_shape p = kv_head_problem(shape);
  const int es = shape.dtype == BSA_F32 ? 4 : 2;
  const int G = p.Hq;
  for (int b = 0; b < shape.B; ++b) {
    for (int g = 0; g < shape.Hkv; ++g) {
      const int64_t qh = static_cast<int64_t>(b) * shape.Hq + static_cast<int64_t>(g) * G;
      const int64_t kh = static_cast<int64_t>(b) * shape.Hkv + g;
      const char* qs = static_cast<const char*>(q) + qh * shape.Sq * shape.D * es;
      const char* ks = static_cast<const char*>(k) + kh * shape.Sk * shape.D * es;
      const char* vs = static_cast<const char*>(v) + kh * shape.Sk * shape.D * es;
      const int rc = centroid_compensated_attention(
          qs, ks, vs, p, q_labels + kh * shape.Sq, Cq, k_labels + kh * shape.Sk, Ck,
          block_mask + b * mask_b_stride + g * mask_g_stride, 0, 0, scale, compensate,
          out + qh * shape.Sq * shape.D, workspace, workspace_bytes, as_stream(stream),
          kProfAttention, false, false);
      if (rc) return rc;
    }
  }
  return BSA_OK;
}
