// Allocation-free variant of the SparsePR residual repair.
//
// bsa_probe_residual_correction needs a few megabytes of scratch that the caller
// normally passes in. Some callers cannot obtain that memory at the moment they call:
// runtimes without a device allocator of their own, code on a path that must not call
// the allocator, and serving loops whose device memory is fixed before the first
// request and may not grow afterwards. For
// them this file keeps a fixed scratch buffer inside the library itself and runs the
// same repair with it; nothing is allocated per call.
//
// The buffer below is a file-scope device array: every GPU that loads libbsa.so holds
// its 16 MiB until the process exits. In host code its name is only a host-side
// stand-in, so its device address is looked up with cudaGetSymbolAddress, once per
// device, with that device current, the first time the entry point runs there.
#include <mutex>

#include "common.cuh"

namespace bsa {

constexpr size_t kNoAllocRepairScratchBytes = size_t(16) << 20;  // 16 MiB

static __device__ __align__(256) unsigned char g_repair_scratch[kNoAllocRepairScratchBytes];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of g_repair_scratch on the current device (looked up on first use).
int noalloc_scratch(void** ptr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return check_cuda(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(BSA_ERR_UNSUPPORTED, "device ordinal %d", dev);
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_repair_scratch);
    if (e != cudaSuccess) return check_cuda(e, "cudaGetSymbolAddress(repair scratch)");
    g_noalloc_ptr[dev] = p;
  }
  *ptr = g_noalloc_ptr[dev];
  return BSA_OK;
}
}  // namespace

}  // namespace bsa

extern "C" int bsa_probe_residual_correction_noalloc(float* out, const float* o_probe,
                                                     const int32_t* probe_idx,
                                                     const float* weights, int per_head, int B,
                                                     int H, int S, int D, int M, int rank,
                                                     float lam, void* stream) {
  using namespace bsa;
  int rc = validate_repair_args(out, o_probe, probe_idx, weights, B, H, S, D, M, rank, lam);
  if (rc) return rc;
  const size_t need = bsa_repair_workspace_bytes(B, H, S, D, M);
  if (need > kNoAllocRepairScratchBytes)
    return fail(BSA_ERR_UNSUPPORTED,
                "this repair needs %zu bytes of scratch; the built-in buffer holds %zu bytes "
                "(16 MiB): use bsa_probe_residual_correction with a workspace",
                need, kNoAllocRepairScratchBytes);
  void* scratch = nullptr;
  rc = noalloc_scratch(&scratch);
  if (rc) return rc;
  // Every scratch word the repair reads is written earlier in the same call, so the
  // buffer needs no clearing between calls.
  return bsa_probe_residual_correction(out, o_probe, probe_idx, weights, per_head, B, H, S, D,
                                       M, rank, lam, scratch, kNoAllocRepairScratchBytes, stream);
}
