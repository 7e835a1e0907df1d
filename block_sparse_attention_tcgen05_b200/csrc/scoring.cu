// XAttention anti-diagonal block scoring on sm_100a.
//
// Source: "Dynamic block masks and head-wise mask reuse" (mlx-arsenal notes),
// §XAttention — anti-diagonal block scoring (every stride x stride sub-block of QKᵀ
// summarised by its anti-diagonal sum, strided logits softmaxed per row, summed per
// block x block tile), §Deviations (rows normalised to 1), §Out of scope (transient
// memory of the strided matrix; padded keys take softmax mass).
//
// The anti-diagonal sums form a dense GEMM: with Q'[I] = (q_{Is}, ..., q_{Is+s-1}) and
// K'[J] = (k_{Js+s-1}, ..., k_{Js}), A = Q' K'ᵀ with inner dimension s·D. Both operands
// are strided row selections of Q and K, so 3-D TMA boxes over (D, s, rows/s) fetch
// them directly: slot t of Q' is rows I·s + t, slot t of K' is rows J·s + s-1-t.
//
// One CTA owns 128 strided query rows. For each 256-column tile of A (tcgen05, fp32
// accumulator in TMEM) four epilogue warps take the tile row max and, per key block
// (r = block/stride consecutive columns), the sum of 2^((a - m_tile)·scale·log2 e);
// those per-tile partial sums stay in TMEM next to the accumulator. After the last
// tile each row rescales its partials to the global row max and total, and groups of
// r consecutive rows (r lanes of a warp) add their rows up with shuffles. The strided
// logit matrix never reaches device memory.
//
// Long sequences (more than 2048 strided rows or 256 key blocks, where the per-tile
// partials no longer fit next to the accumulator) take two passes of the same GEMM: the
// first keeps each row's running max and sum (online over the tiles) and parks them in
// the row's own query block of the output (2 r floats of its nb), the second reads them
// back and writes every tile's normalised block sums directly.
#include <cuda_bf16.h>

#include <cmath>

#include "common.cuh"
#include "ptx.cuh"

namespace bsa {

struct ScoreArgs {
  int Hq, Hkv, ns, s, r, n_tiles;  // ns = N/s strided rows; n_tiles = ceil(ns/256)
  int nb;                          // N / block
  float scale_log2;
  float* scores;                   // (B, Hq, nb, nb)
};

constexpr int kScoreStages = 3;
constexpr int kScoreStageBytes = 16384 + 32768;  // Q box (128 x 128 B) + K box (256 x 128 B)

// MODE 0: one pass (partials in TMEM); 1: row max and sum only; 2: normalised block sums
// from the first pass's row statistics.
template <int D, int R, int MODE>
__global__ void __launch_bounds__(192, 1)
    score_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                 const ScoreArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kScoreStages * kScoreStageBytes);
  // bars: [0,S) full, [S,2S) empty, 2S = acc full, 2S+1 = acc free, 2S+2 = drain
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * kScoreStages + 3);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* never = reinterpret_cast<int*>(tmem_slot + 2);
  float* mtile = reinterpret_cast<float*>(tmem_slot + 4);  // [8][128]
  float* ltile = mtile + 8 * 128;                           // [8][128]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int itile = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int hk = h / (a.Hq / a.Hkv);
  const uint32_t bar0 = smem_u32(bars);
  auto FULL = [&](int i) { return bar0 + 8u * i; };
  auto EMPTY = [&](int i) { return bar0 + 8u * (kScoreStages + i); };
  const uint32_t ACC_FULL = bar0 + 8u * (2 * kScoreStages);
  const uint32_t ACC_FREE = ACC_FULL + 8u;
  const uint32_t DRAIN = ACC_FULL + 16u;
  constexpr int KCH = D / 64;                // 128-byte column chunks per row of Q/K
  const int steps = a.s * KCH;               // K-loop steps per tile (64 elements each)

  if (tid == 0) {
    for (int i = 0; i < kScoreStages; ++i) {
      mbar_init(FULL(i), 1);
      mbar_init(EMPTY(i), 1);
    }
    mbar_init(ACC_FULL, 1);
    mbar_init(ACC_FREE, 128);
    mbar_init(DRAIN, 1);
    *abort_flag = 0;
    *never = 0;
    fence_mbarrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      const int qrow = (b * a.Hq + h) * a.ns + itile * 128;
      int it = 0, issued = 0;
      for (int jt = 0; jt < a.n_tiles && !*abort_flag; ++jt) {
        const int krow = (b * a.Hkv + hk) * a.ns + jt * 256;
        for (int st = 0; st < steps; ++st, ++it) {
          const int slot = it % kScoreStages;
          if (it >= kScoreStages &&
              !mbar_wait(EMPTY(slot), ((it / kScoreStages) - 1) & 1, abort_flag, 40))
            break;
          const int t = st / KCH, c = st % KCH;
          const uint32_t dst = sbase + slot * kScoreStageBytes;
          mbar_arrive_expect_tx(FULL(slot), kScoreStageBytes);
          tma_load_3d(dst, &tmQ, FULL(slot), c * 64, t, qrow);
          tma_load_3d(dst + 16384, &tmK, FULL(slot), c * 64, a.s - 1 - t, krow);
          issued = it + 1;
        }
      }
      // every issued copy must land before the CTA exits
      for (int i = issued - kScoreStages; i < issued; ++i)
        if (i >= 0) mbar_wait(FULL(i % kScoreStages), (i / kScoreStages) & 1, never, 41);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int jt = 0; jt < a.n_tiles && ok; ++jt) {
        const int ncols = min(256, a.ns - jt * 256);
        const uint32_t idesc = make_idesc(false, 128, ncols, false, false);
        // the epilogue must have read the previous tile before it is overwritten
        if (jt > 0 && !(ok = mbar_wait(ACC_FREE, (jt - 1) & 1, abort_flag, 42))) break;
        for (int st = 0; st < steps; ++st, ++it) {
          const int slot = it % kScoreStages;
          if (!(ok = mbar_wait(FULL(slot), (it / kScoreStages) & 1, abort_flag, 43))) break;
          tc_fence_after();
          const uint32_t sa = sbase + slot * kScoreStageBytes;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ss<false>(tmem, smem_desc(sa + kk * 32, 16, 1024),
                          smem_desc(sa + 16384 + kk * 32, 16, 1024), idesc,
                          (st > 0 || kk > 0) ? 1u : 0u);
          tc_commit(EMPTY(slot));
        }
        if (ok) tc_commit(ACC_FULL);
      }
      tc_commit(DRAIN);
      mbar_wait(DRAIN, 0, never, 44);
    }
  } else {
    // epilogue: thread = strided row (TMEM lane), warps 2..5 cover lane quarters 2,3,0,1
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t tl = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const float scl = a.scale_log2;
    if constexpr (MODE == 0) {
      constexpr int per_tile = 256 / R;  // key blocks per full tile
      bool ok = true;
      for (int jt = 0; jt < a.n_tiles; ++jt) {
        if (!(ok = mbar_wait(ACC_FULL, jt & 1, abort_flag, 45))) break;
        tc_fence_after();
        const int ncols = min(256, a.ns - jt * 256);
        const int npc = ncols / 32;
        float mx = -INFINITY;  // raw logits; scale > 0 so the max commutes with it
        for (int p = 0; p < npc; ++p) {
          float t[32];
          tmem_ld32(tl + p * 32, t);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) mx = fmaxf(mx, t[c]);
        }
        float lsum = 0.f;
        // partial block sums of this tile, written to TMEM columns 256 + jt*per_tile + ...
        for (int p = 0; p < npc; ++p) {
          float t[32];
          tmem_ld32(tl + p * 32, t);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            t[c] = ex2((t[c] - mx) * scl);
            lsum += t[c];
          }
          // sums over groups of R consecutive columns = one key block each
          constexpr int G = 32 / R;
          uint32_t gs[G];
#pragma unroll
          for (int g = 0; g < G; ++g) {
            float acc = 0.f;
#pragma unroll
            for (int c = 0; c < R; ++c) acc += t[g * R + c];
            gs[g] = __float_as_uint(acc);
          }
          tmem_st_n<G>(tl + 256 + jt * per_tile + p * G, gs);
          tmem_wait_st();
        }
        mtile[jt * 128 + row] = mx;
        ltile[jt * 128 + row] = lsum;
        tc_fence_before();
        mbar_arrive(ACC_FREE);
      }
      if (ok && !*abort_flag) {
        float M = -INFINITY;
        for (int jt = 0; jt < a.n_tiles; ++jt) M = fmaxf(M, mtile[jt * 128 + row]);
        float L = 0.f;
        for (int jt = 0; jt < a.n_tiles; ++jt)
          L += ltile[jt * 128 + row] * ex2((mtile[jt * 128 + row] - M) * scl);
        const float inv_rl = 1.f / (L * static_cast<float>(R));
        // query block of this row and the lane leading its group of r rows
        const int qrow_global = itile * 128 + row;
        const int iblk = qrow_global / R;
        const bool leader = (qrow_global % R) == 0;
        float* out = a.scores + ((static_cast<size_t>(b) * a.Hq + h) * a.nb + iblk) * a.nb;
        for (int jt = 0; jt < a.n_tiles; ++jt) {
          const float f = ex2((mtile[jt * 128 + row] - M) * scl) * inv_rl;
          const int ncols = min(256, a.ns - jt * 256);
          const int nblk = ncols / R;
          for (int c0 = 0; c0 < nblk; c0 += 32) {
            float t[32];
            tmem_ld32(tl + 256 + jt * per_tile + c0, t);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c) {
              float v = t[c] * f;
              // sum over the r rows of the query block (r consecutive lanes, r <= 32)
#pragma unroll
              for (int o = 1; o < R; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
              t[c] = v;
            }
            if (leader) {
              for (int c = 0; c < 32 && c0 + c < nblk; ++c) out[jt * per_tile + c0 + c] = t[c];
            }
          }
        }
      }
    } else {
      // the row's query block and the lane leading its group of r rows; the block row of
      // the output first holds the r rows' (max, sum) pairs from the first pass
      const int qrow_global = itile * 128 + row;
      const int iblk = qrow_global / R;
      const bool leader = (qrow_global % R) == 0;
      float* out = a.scores + ((static_cast<size_t>(b) * a.Hq + h) * a.nb + iblk) * a.nb;
      float M = -INFINITY, L = 0.f;
      if constexpr (MODE == 2) {
        M = out[2 * (qrow_global % R)];
        L = out[2 * (qrow_global % R) + 1];
      }
      __syncwarp();  // every row of the block has its statistics before the leader writes
      const float inv_rl = 1.f / (L * static_cast<float>(R));
      bool ok = true;
      for (int jt = 0; jt < a.n_tiles; ++jt) {
        if (!(ok = mbar_wait(ACC_FULL, jt & 1, abort_flag, 45))) break;
        tc_fence_after();
        const int ncols = min(256, a.ns - jt * 256);
        const int npc = ncols / 32;
        if constexpr (MODE == 1) {
          float mx = -INFINITY;  // raw logits; scale > 0 so the max commutes with it
          for (int p = 0; p < npc; ++p) {
            float t[32];
            tmem_ld32(tl + p * 32, t);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c) mx = fmaxf(mx, t[c]);
          }
          if (mx > M) {
            L *= ex2((M - mx) * scl);
            M = mx;
          }
          for (int p = 0; p < npc; ++p) {
            float t[32];
            tmem_ld32(tl + p * 32, t);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c) L += ex2((t[c] - M) * scl);
          }
        } else {
          constexpr int G = 32 / R;
          constexpr int per_tile = 256 / R;
          for (int p = 0; p < npc; ++p) {
            float t[32];
            tmem_ld32(tl + p * 32, t);
            tmem_wait_ld();
            float gs[G];
#pragma unroll
            for (int g = 0; g < G; ++g) {
              float acc = 0.f;
#pragma unroll
              for (int c = 0; c < R; ++c) acc += ex2((t[g * R + c] - M) * scl);
              // sum over the r rows of the query block (r consecutive lanes, r <= 32)
              float v = acc * inv_rl;
#pragma unroll
              for (int o = 1; o < R; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
              gs[g] = v;
            }
            if (leader) {
#pragma unroll
              for (int g = 0; g < G; ++g) out[jt * per_tile + p * G + g] = gs[g];
            }
          }
        }
        tc_fence_before();
        mbar_arrive(ACC_FREE);
      }
      if constexpr (MODE == 1) {
        if (ok && !*abort_flag) {
          out[2 * (qrow_global % R)] = M;
          out[2 * (qrow_global % R) + 1] = L;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

int antidiagonal_block_scores(const void* q, const void* k, const bsa_shape& s, int block,
                              int stride, float logit_scale, float* scores, cudaStream_t st) {
  if (!q || !k || !scores) return fail(BSA_ERR_INVALID_ARG, "null pointer argument");
  if (s.B <= 0 || s.Hq <= 0 || s.Hkv <= 0 || s.Sq <= 0 || s.Hq % s.Hkv)
    return fail(BSA_ERR_INVALID_ARG, "bad shape");
  if (s.Sq != s.Sk) return fail(BSA_ERR_INVALID_ARG, "scoring needs Sq == Sk");
  if (s.dtype != BSA_BF16) return fail(BSA_ERR_UNSUPPORTED, "scoring supports bf16 inputs only");
  if (s.D != 64 && s.D != 128) return fail(BSA_ERR_UNSUPPORTED, "head dim %d", s.D);
  if (stride <= 0 || block <= 0 || block % stride)
    return fail(BSA_ERR_INVALID_ARG, "block (%d) must be a positive multiple of stride (%d)",
                block, stride);
  const int N = s.Sq, r = block / stride;
  if (N % block) return fail(BSA_ERR_INVALID_ARG, "S (%d) not a multiple of block (%d)", N, block);
  if (r > 32 || (r & (r - 1)))
    return fail(BSA_ERR_UNSUPPORTED, "block/stride = %d must be a power of two <= 32", r);
  const int ns = N / stride;
  if (ns % 128) return fail(BSA_ERR_UNSUPPORTED, "S/stride (%d) must be a multiple of 128", ns);
  const int nb = N / block;
  // one pass while the per-tile partials fit beside the accumulator in TMEM (at most 8
  // tiles of 256 strided columns, 256 key blocks); two passes beyond, which park each
  // row's statistics in its query block of the output (2 r floats of nb)
  const bool one_pass = ns <= 2048 && nb <= 256;
  if (!one_pass && nb < 2 * r)
    return fail(BSA_ERR_UNSUPPORTED, "two-pass scoring needs S/block (%d) >= 2 block/stride (%d)", nb,
                2 * r);
  if (static_cast<int64_t>(s.B) * s.Hq * ns >= (int64_t(1) << 31))
    return fail(BSA_ERR_UNSUPPORTED, "B * Hq * S/stride exceeds the TMA row range");
  if ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k)) % 16)
    return fail(BSA_ERR_INVALID_ARG, "q/k must be 16-byte aligned");

  CUtensorMap mq, mk;
  int rc;
  const uint64_t rowb = static_cast<uint64_t>(s.D) * 2;
  if ((rc = make_tmap_3d(&mq, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, s.D, stride,
                         static_cast<uint64_t>(s.B) * s.Hq * ns, rowb, rowb * stride, 64, 1, 128)))
    return rc;
  if ((rc = make_tmap_3d(&mk, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, s.D, stride,
                         static_cast<uint64_t>(s.B) * s.Hkv * ns, rowb, rowb * stride, 64, 1, 256)))
    return rc;
  ScoreArgs a{};
  a.Hq = s.Hq;
  a.Hkv = s.Hkv;
  a.ns = ns;
  a.s = stride;
  a.r = r;
  a.n_tiles = (ns + 255) / 256;
  a.nb = nb;
  const float sc = logit_scale > 0.f ? logit_scale : 1.f / std::sqrt(static_cast<float>(s.D));
  a.scale_log2 = sc * 1.4426950408889634f;
  a.scores = scores;
  const int smem = kScoreStages * kScoreStageBytes + 1024 + 2 * 8 * 128 * 4 + 1024;
  using Kern = void (*)(CUtensorMap, CUtensorMap, ScoreArgs);
  Kern k0 = nullptr, k1 = nullptr, k2 = nullptr;
#define BSA_SCORE_CASE(RR)                                                        \
  case RR:                                                                        \
    k0 = s.D == 64 ? score_kernel<64, RR, 0> : score_kernel<128, RR, 0>;           \
    k1 = s.D == 64 ? score_kernel<64, RR, 1> : score_kernel<128, RR, 1>;           \
    k2 = s.D == 64 ? score_kernel<64, RR, 2> : score_kernel<128, RR, 2>;           \
    break;
  switch (r) {
    BSA_SCORE_CASE(1)
    BSA_SCORE_CASE(2)
    BSA_SCORE_CASE(4)
    BSA_SCORE_CASE(8)
    BSA_SCORE_CASE(16)
    BSA_SCORE_CASE(32)
    default: return fail(BSA_ERR_UNSUPPORTED, "block/stride = %d", r);
  }
#undef BSA_SCORE_CASE
  const dim3 grid(ns / 128, s.Hq, s.B);
  prof_begin(kProfScoring, st);
  for (Kern kern : {one_pass ? k0 : k1, one_pass ? nullptr : k2}) {
    if (!kern) continue;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return check_cuda(e, "cudaFuncSetAttribute(score_kernel)");
    kern<<<grid, 192, smem, st>>>(mq, mk, a);
    count_launch();
    if ((rc = check_cuda(cudaGetLastError(), "score_kernel launch"))) return rc;
  }
  prof_end(kProfScoring, st);
  return BSA_OK;
}

}  // namespace bsa

extern "C" int bsa_antidiagonal_block_scores(const void* q, const void* k, bsa_shape shape,
                                             int block, int stride, float logit_scale,
                                             float* scores, void* stream) {
  return bsa::antidiagonal_block_scores(q, k, shape, block, stride, logit_scale, scores,
                                        bsa::as_stream(stream));
}
