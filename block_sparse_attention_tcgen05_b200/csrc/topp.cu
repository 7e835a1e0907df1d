// Per-row top-p block selection.
//
// Source: "Dynamic block masks and head-wise mask reuse" (mlx-arsenal notes),
// §XAttention (each query block keeps the smallest set of key blocks whose mass
// reaches a fraction tau of its total), §Deviations (at least one block per row; key
// block 0 is not forced), §What mlx-arsenal ships (scalar or per-head tau).
//
// One warp per row: a bitonic sort in shared memory orders the row by (score
// descending, key index ascending); the running float32 sum is then taken in that
// order by one lane, sequentially, so the decision is reproducible bit for bit.
#include "common.cuh"
#include "ptx.cuh"

namespace bsa {

constexpr int kTopPWarps = 4;
constexpr int kTopPMaxN = 1024;

__device__ __forceinline__ bool comes_before(float sa, int ia, float sb, int ib) {
  return sa > sb || (sa == sb && ia < ib);
}

__global__ void __launch_bounds__(kTopPWarps * 32) top_p_kernel(
    const float* __restrict__ scores, int H, int Nq, int Nk, int rows, const float* __restrict__ tau,
    int n_tau, uint8_t* __restrict__ mask, uint8_t* __restrict__ tie_rows) {
  extern __shared__ uint8_t sm_topp[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int n = 1;
  while (n < Nk) n <<= 1;
  float* sv = reinterpret_cast<float*>(sm_topp) + warp * 2 * n;
  int* si = reinterpret_cast<int*>(sv + n);
  const int row = blockIdx.x * kTopPWarps + warp;
  if (row >= rows) return;
  const int h = (row / Nq) % H;
  const float t = tau[n_tau == 1 ? 0 : h];
  const float* in = scores + static_cast<size_t>(row) * Nk;
  for (int i = lane; i < n; i += 32) {
    sv[i] = i < Nk ? in[i] : -INFINITY;
    si[i] = i;
  }
  __syncwarp();
  // bitonic sort; the sorted order is "comes_before" ascending
  for (int k = 2; k <= n; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = lane; i < n; i += 32) {
        const int p = i ^ j;
        if (p > i) {
          const bool up = (i & k) == 0;
          const float a = sv[i], b = sv[p];
          const int ia = si[i], ib = si[p];
          const bool swap = up ? comes_before(b, ib, a, ia) : comes_before(a, ia, b, ib);
          if (swap) {
            sv[i] = b;
            sv[p] = a;
            si[i] = ib;
            si[p] = ia;
          }
        }
      }
      __syncwarp();
    }
  }
  int m = Nk - 1;
  int tie = 0;
  if (lane == 0) {
    float acc = 0.f;
    bool found = false;
    // Scores are non-negative, so the running sum never decreases: once it is past
    // tau by more than the tie tolerance, no later prefix decides or flags anything.
#pragma unroll 4
    for (int i = 0; i < Nk; ++i) {
      acc = __fadd_rn(acc, sv[i]);
      if (fabsf(acc - t) <= 1e-5f) tie = 1;
      if (!found && acc >= t) {
        m = i;
        found = true;
      }
      if (found && acc - t > 1e-5f) break;
    }
    if (m + 1 < Nk && sv[m] - sv[m + 1] <= 1e-5f) tie = 1;
  }
  m = __shfl_sync(0xffffffffu, m, 0);
  tie = __shfl_sync(0xffffffffu, tie, 0);
  uint8_t* out = mask + static_cast<size_t>(row) * Nk;
  for (int i = lane; i < Nk; i += 32) out[si[i]] = i <= m ? 1 : 0;
  if (tie_rows && lane == 0) tie_rows[row] = static_cast<uint8_t>(tie);
}

}  // namespace bsa

extern "C" int bsa_top_p_block_mask(const float* scores, int B, int H, int Nq, int Nk,
                                    const float* tau, int n_tau, uint8_t* mask, uint8_t* tie_rows,
                                    void* stream) {
  using namespace bsa;
  if (!scores || !tau || !mask) return fail(BSA_ERR_INVALID_ARG, "null pointer argument");
  if (B <= 0 || H <= 0 || Nq <= 0 || Nk <= 0) return fail(BSA_ERR_INVALID_ARG, "bad shape");
  if (Nk > kTopPMaxN) return fail(BSA_ERR_UNSUPPORTED, "Nk %d > %d", Nk, kTopPMaxN);
  if (n_tau != 1 && n_tau != H) return fail(BSA_ERR_INVALID_ARG, "n_tau must be 1 or H");
  int n = 1;
  while (n < Nk) n <<= 1;
  const int smem = kTopPWarps * 2 * n * 4;
  const int rows = B * H * Nq;
  cudaError_t e = cudaFuncSetAttribute(top_p_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       smem > 48 * 1024 ? smem : 48 * 1024);
  if (e != cudaSuccess) return check_cuda(e, "cudaFuncSetAttribute(top_p)");
  top_p_kernel<<<(rows + kTopPWarps - 1) / kTopPWarps, kTopPWarps * 32, smem, as_stream(stream)>>>(
      scores, H, Nq, Nk, rows, tau, n_tau, mask, tie_rows);
  count_launch();
  return check_cuda(cudaGetLastError(), "top_p_kernel launch");
}
