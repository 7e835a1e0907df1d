// Status codes, error details, tensor-map encoding and the small label kernel.
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "ptx.cuh"

namespace bsa {

namespace {
thread_local char g_detail[512] = "";

std::atomic<long long> g_launches{0};

struct ProfState {
  std::mutex mu;
  int enabled = 0;
  int capacity = 0;
  std::vector<cudaEvent_t> ev[kProfCount][2];
  int used[kProfCount] = {0, 0, 0};
};
ProfState& prof() {
  static ProfState p;
  return p;
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}
}  // namespace

int fail(int status, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_detail, sizeof(g_detail), fmt, ap);
  va_end(ap);
  return status;
}

void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

void prof_begin(int kernel, cudaStream_t st) {
  ProfState& p = prof();
  std::lock_guard<std::mutex> lk(p.mu);
  if (!p.enabled || p.used[kernel] >= p.capacity) return;
  cudaEventRecord(p.ev[kernel][0][p.used[kernel]], st);
}

void prof_end(int kernel, cudaStream_t st) {
  ProfState& p = prof();
  std::lock_guard<std::mutex> lk(p.mu);
  if (!p.enabled || p.used[kernel] >= p.capacity) return;
  cudaEventRecord(p.ev[kernel][1][p.used[kernel]], st);
  ++p.used[kernel];
}

int check_cuda(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return BSA_OK;
  return fail(BSA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

int make_tmap_3d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype, int elem_bytes,
                 uint64_t d0, uint64_t d1, uint64_t d2, uint64_t stride1_bytes,
                 uint64_t stride2_bytes, uint32_t box0, uint32_t box1, uint32_t box2) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(BSA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  if (reinterpret_cast<uintptr_t>(base) % 16 || stride1_bytes % 16 || stride2_bytes % 16 ||
      (box0 * elem_bytes) % 16)
    return fail(BSA_ERR_INVALID_ARG, "tensor map operands not 16-byte aligned");
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {stride1_bytes, stride2_bytes};
  cuuint32_t box[3] = {box0, box1, box2};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, dtype, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(BSA_ERR_CUDA, "cuTensorMapEncodeTiled (3d) failed: %d", int(r));
  return BSA_OK;
}

int make_tmap_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype, int elem_bytes,
                 uint64_t rows, uint64_t cols, uint32_t box_rows, uint32_t box_cols,
                 CUtensorMapSwizzle swizzle) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(BSA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const uint64_t row_bytes = cols * elem_bytes;
  if (reinterpret_cast<uintptr_t>(base) % 16 || row_bytes % 16 || (box_cols * elem_bytes) % 16)
    return fail(BSA_ERR_INVALID_ARG, "tensor map operands not 16-byte aligned");
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(BSA_ERR_CUDA, "cuTensorMapEncodeTiled (2d) failed: %d", int(r));
  return BSA_OK;
}

// Label of every token of a T x H x W grid for tiles (tt, th, tw), edge tiles partial.
__global__ void tile_labels_kernel(int T, int H, int W, int tt, int th, int tw, int nH, int nW,
                                   int32_t* __restrict__ labels) {
  const int64_t s = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t S = static_cast<int64_t>(T) * H * W;
  if (s >= S) return;
  const int w = static_cast<int>(s % W);
  const int h = static_cast<int>((s / W) % H);
  const int t = static_cast<int>(s / (static_cast<int64_t>(W) * H));
  labels[s] = ((t / tt) * nH + h / th) * nW + w / tw;
}

// Sliding Tile Attention window along one axis of n tiles, w tiles wide: key tile c is
// inside query tile a's window when |c - centre| <= w / 2, the centre being a moved
// inward at the borders (clamped to [w / 2, n - 1 - w / 2]); a window at least as wide
// as the axis holds every tile.
__device__ __forceinline__ bool sta_axis_keep(int a, int c, int n, int w) {
  const int r = w / 2;
  if (2 * r + 1 >= n) return true;
  const int centre = min(max(a, r), n - 1 - r);
  return abs(c - centre) <= r;
}

// Tile-resolution STA mask: one thread per (query tile, key tile) byte, tiles in the
// raster order of tile_labels.
__global__ void sliding_tile_mask_kernel(int nT, int nH, int nW, int wt, int wh, int ww,
                                         uint8_t* __restrict__ mask) {
  const int64_t C = static_cast<int64_t>(nT) * nH * nW;
  const int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (e >= C * C) return;
  const int a = static_cast<int>(e / C), c = static_cast<int>(e % C);
  const int at = a / (nH * nW), ah = (a / nW) % nH, aw = a % nW;
  const int ct = c / (nH * nW), ch = (c / nW) % nH, cw = c % nW;
  mask[e] = (sta_axis_keep(at, ct, nT, wt) && sta_axis_keep(ah, ch, nH, wh) &&
             sta_axis_keep(aw, cw, nW, ww))
                ? 1
                : 0;
}

// One warp waits on an mbarrier that nothing arrives on (expected count 1, no arrival),
// through the bounded wait every kernel uses; the wait gives up after limit_ns, which
// records BSA_ERR_TIMEOUT (site 90) in the status word. The barrier then still has its
// arrival pending; it lives in this CTA's shared memory and ends with it.
__global__ void __launch_bounds__(32) wait_timeout_selftest_kernel(uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1u);
    abort_flag = 0;
    fence_mbarrier_init();
  }
  __syncwarp();
  if (threadIdx.x == 0) mbar_wait(smem_u32(&bar), 0, &abort_flag, 90, limit_ns);
  __syncwarp();
}

}  // namespace bsa

extern "C" {

const char* bsa_status_string(int status) {
  switch (status) {
    case BSA_OK: return "BSA_OK";
    case BSA_ERR_INVALID_ARG: return "BSA_ERR_INVALID_ARG";
    case BSA_ERR_UNSUPPORTED: return "BSA_ERR_UNSUPPORTED";
    case BSA_ERR_CUDA: return "BSA_ERR_CUDA";
    case BSA_ERR_TIMEOUT: return "BSA_ERR_TIMEOUT";
    case BSA_ERR_WORKSPACE: return "BSA_ERR_WORKSPACE";
    default: return "BSA_UNKNOWN_STATUS";
  }
}

void bsa_last_error_detail(char* buf, size_t len) {
  if (!buf || !len) return;
  std::strncpy(buf, bsa::g_detail, len - 1);
  buf[len - 1] = '\0';
}

int bsa_version(void) { return 100; }

long long bsa_launch_count(void) { return bsa::g_launches.load(); }

int bsa_profile_enable(int max_launches) {
  bsa::ProfState& p = bsa::prof();
  std::lock_guard<std::mutex> lk(p.mu);
  if (max_launches < 0) return bsa::fail(BSA_ERR_INVALID_ARG, "max_launches < 0");
  for (int k = 0; k < bsa::kProfCount; ++k) {
    for (int j = 0; j < 2; ++j) {
      while (static_cast<int>(p.ev[k][j].size()) < max_launches) {
        cudaEvent_t e;
        cudaError_t r = cudaEventCreate(&e);
        if (r != cudaSuccess) return bsa::check_cuda(r, "cudaEventCreate");
        p.ev[k][j].push_back(e);
      }
    }
    p.used[k] = 0;
  }
  p.capacity = max_launches;
  p.enabled = max_launches > 0;
  return BSA_OK;
}

int bsa_profile_read(int kernel, float* total_ms, int* launches) {
  bsa::ProfState& p = bsa::prof();
  std::lock_guard<std::mutex> lk(p.mu);
  if (kernel < 0 || kernel >= bsa::kProfCount) return bsa::fail(BSA_ERR_INVALID_ARG, "kernel id");
  float sum = 0.f;
  for (int i = 0; i < p.used[kernel]; ++i) {
    cudaError_t r = cudaEventSynchronize(p.ev[kernel][1][i]);
    if (r != cudaSuccess) return bsa::check_cuda(r, "cudaEventSynchronize");
    float ms = 0.f;
    r = cudaEventElapsedTime(&ms, p.ev[kernel][0][i], p.ev[kernel][1][i]);
    if (r != cudaSuccess) return bsa::check_cuda(r, "cudaEventElapsedTime");
    sum += ms;
  }
  if (total_ms) *total_ms = sum;
  if (launches) *launches = p.used[kernel];
  return BSA_OK;
}

int bsa_wait_timeout_selftest(long long limit_ns, void* stream) {
  const long long lim = limit_ns < 1000 ? 1000 : (limit_ns > 2000000000LL ? 2000000000LL : limit_ns);
  bsa::wait_timeout_selftest_kernel<<<1, 32, 0, bsa::as_stream(stream)>>>(static_cast<uint64_t>(lim));
  bsa::count_launch();
  return bsa::check_cuda(cudaGetLastError(), "wait_timeout_selftest_kernel");
}

int bsa_get_device_status(void* stream, int* where) {
  cudaError_t e = cudaStreamSynchronize(bsa::as_stream(stream));
  if (e != cudaSuccess) return bsa::check_cuda(e, "cudaStreamSynchronize");
  int st = 0, wh = 0, zero = 0;
  if ((e = cudaMemcpyFromSymbol(&st, bsa::g_device_status, sizeof(int))) != cudaSuccess)
    return bsa::check_cuda(e, "read device status");
  if ((e = cudaMemcpyFromSymbol(&wh, bsa::g_device_status_where, sizeof(int))) != cudaSuccess)
    return bsa::check_cuda(e, "read device status site");
  if (st != 0) {
    cudaMemcpyToSymbol(bsa::g_device_status, &zero, sizeof(int));
    cudaMemcpyToSymbol(bsa::g_device_status_where, &zero, sizeof(int));
  }
  if (where) *where = wh;
  return st == 0 ? BSA_OK : st;
}

int bsa_tile_labels(int T, int H, int W, int tt, int th, int tw, int32_t* labels, int* n_clusters,
                    void* stream) {
  if (T <= 0 || H <= 0 || W <= 0 || tt <= 0 || th <= 0 || tw <= 0)
    return bsa::fail(BSA_ERR_INVALID_ARG, "non-positive grid or tile size");
  if (!labels) return bsa::fail(BSA_ERR_INVALID_ARG, "labels is null");
  const int64_t S = static_cast<int64_t>(T) * H * W;
  const int nT = bsa::ceil_div(T, tt), nH = bsa::ceil_div(H, th), nW = bsa::ceil_div(W, tw);
  if (static_cast<int64_t>(nT) * nH * nW > INT32_MAX || S > INT32_MAX)
    return bsa::fail(BSA_ERR_UNSUPPORTED, "grid too large");
  if (n_clusters) *n_clusters = nT * nH * nW;
  bsa::tile_labels_kernel<<<static_cast<unsigned>((S + 255) / 256), 256, 0,
                            bsa::as_stream(stream)>>>(T, H, W, tt, th, tw, nH, nW, labels);
  bsa::count_launch();
  return bsa::check_cuda(cudaGetLastError(), "tile_labels_kernel");
}

int bsa_sliding_tile_block_mask(int nT, int nH, int nW, int wt, int wh, int ww, uint8_t* mask,
                                void* stream) {
  if (nT <= 0 || nH <= 0 || nW <= 0 || wt <= 0 || wh <= 0 || ww <= 0)
    return bsa::fail(BSA_ERR_INVALID_ARG, "non-positive tile grid or window");
  if (!mask) return bsa::fail(BSA_ERR_INVALID_ARG, "mask is null");
  const int64_t C = static_cast<int64_t>(nT) * nH * nW;
  if (C > 16384) return bsa::fail(BSA_ERR_UNSUPPORTED, "%lld tiles > 16384", static_cast<long long>(C));
  bsa::sliding_tile_mask_kernel<<<static_cast<unsigned>((C * C + 255) / 256), 256, 0,
                                  bsa::as_stream(stream)>>>(nT, nH, nW, wt, wh, ww, mask);
  bsa::count_launch();
  return bsa::check_cuda(cudaGetLastError(), "sliding_tile_mask_kernel");
}

}  // extern "C"
