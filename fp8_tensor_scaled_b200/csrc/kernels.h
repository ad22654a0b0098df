// kernels.h — internal launchers behind the C ABI (not part of the public API).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace fp8amax {

cudaError_t launch_amax(const void* x, int dt, size_t n, float* amax, cudaStream_t s);
cudaError_t launch_compute_bias(const float* amax, int fmt, int32_t margin, int32_t* bias,
                                cudaStream_t s);
cudaError_t launch_cast(const void* x, int dt, size_t n, const int32_t* bias, int fmt,
                        uint8_t* out, cudaStream_t s);
cudaError_t launch_quantize(const void* x, int dt, size_t n, int fmt, int32_t margin,
                            float* amax, int32_t* bias, uint8_t* out, cudaStream_t s);

// One FP8 GEMM D[M,N] = (A . B^T) * 2^-(bias_a + bias_b), D row-major with
// leading dimension N.  A is [M,K] K-major (a_mn_major = false: A[m*K + k])
// or MN-major (true: A[k*M + m]); B likewise with N.  D is bf16 or fp32.
struct GemmArgs {
  const uint8_t* a;
  const uint8_t* b;
  int a_fmt, b_fmt;
  bool a_mn_major, b_mn_major;
  const int32_t* bias_a;
  const int32_t* bias_b;
  void* d;
  bool d_fp32;
  float* d_amax;   // optional: receives max |D| (must be zeroed before the launch)
  int64_t M, N, K;
  // optional split-K workspace (problems with few tiles); nullptr = never split
  void* workspace = nullptr;
  size_t workspace_bytes = 0;
};

// Returns 0 on success, an fp8_status_t code otherwise.
int launch_gemm(const GemmArgs& g, cudaStream_t s);

// Bytes of split-K workspace launch_gemm would use for this problem when given
// one (0: the problem is never split).  a/b/d pointers are not read.
size_t gemm_workspace_bytes(const GemmArgs& g);

// The launch launch_gemm makes for this problem: tile shape, CTAs per tile
// and K splits.  `g.workspace` non-null means the caller supplies
// gemm_workspace_bytes(g) bytes.  a/b/d pointers are not read.
struct GemmPlan {
  int tile_m, tile_n, ctas_per_tile, k_splits;
};
void gemm_plan(const GemmArgs& g, GemmPlan* plan);

// launch_gemm with the split-K scratch taken from a static device array
// instead of a caller workspace (FP8_ERR_UNSUPPORTED beyond its 16 MiB).
int launch_gemm_noalloc(GemmArgs g, cudaStream_t s);

cudaError_t launch_selftest_wait(uint64_t timeout_ns);
int device_error_site(bool clear);

}  // namespace fp8amax
