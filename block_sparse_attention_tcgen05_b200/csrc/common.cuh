// Host-side helpers shared by the library's translation units.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>
#include <string>

#include "../../include/bsa.h"

namespace bsa {

// Records a formatted error detail for bsa_last_error_detail() and returns `status`.
int fail(int status, const char* fmt, ...);

// Returns BSA_ERR_CUDA (with detail) if `e` is an error.
int check_cuda(cudaError_t e, const char* what);

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
inline int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Bump allocator over a caller-provided workspace (never allocates).
struct Carver {
  char* base;
  size_t used = 0;
  explicit Carver(void* p) : base(static_cast<char*>(p)) {}
  template <class T>
  T* take(size_t count) {
    used = align_up(used, 256);
    T* p = reinterpret_cast<T*>(base ? base + used : nullptr);
    used += count * sizeof(T);
    return p;
  }
};

// Encodes a 2-D tiled TMA descriptor over a row-major (rows x cols) matrix with a
// 128-byte swizzle; box = (box_cols x box_rows). Returns 0 on success.
int make_tmap_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype, int elem_bytes,
                 uint64_t rows, uint64_t cols, uint32_t box_rows, uint32_t box_cols,
                 CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B);

// Same, 3-D: dims (inner, mid, outer) with byte strides for mid and outer.
int make_tmap_3d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype, int elem_bytes,
                 uint64_t d0, uint64_t d1, uint64_t d2, uint64_t stride1_bytes,
                 uint64_t stride2_bytes, uint32_t box0, uint32_t box1, uint32_t box2);

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

// Kernel timing hooks (bsa_profile_*): when enabled, the launch sites of the main
// kernels record a CUDA event pair around the launch on the launch stream.
enum ProfKernel { kProfAttention = 0, kProfScoring = 1, kProfProbe = 2, kProfCount = 3 };
void prof_begin(int kernel, cudaStream_t st);
void prof_end(int kernel, cudaStream_t st);
// Counts kernel launches made by the library (bsa_launch_count).
void count_launch();

}  // namespace bsa
