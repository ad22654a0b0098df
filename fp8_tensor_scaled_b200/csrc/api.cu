// api.cu — the extern "C" entry points declared in include/fp8amax.h.
//
// Each call validates its arguments on the host (returning a status, never
// aborting), then enqueues the kernels of its step on the caller's stream.
// The passes of the linear layer are mapped onto the one GEMM kernel:
//   fwd    Y [T,out]  = X  [T,in]  . W [out,in]^T      (A K-major,  B K-major)
//   dgrad  dX [T,in]  = dY [T,out] . W [out,in]        (A K-major,  B MN-major)
//   wgrad  dW [out,in]= dY [T,out]^T . X [T,in]        (A MN-major, B MN-major)
#include <cstdint>
#include <cuda_runtime.h>

#include "fp8amax.h"
#include "kernels.h"

using namespace fp8amax;

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool valid_fmt(int f) { return f == FP8_E4M3 || f == FP8_E5M2; }
bool valid_dtype(int d) { return d == FP8_DTYPE_BF16 || d == FP8_DTYPE_FP32; }
cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

fp8_status_t from_cuda(cudaError_t e) { return e == cudaSuccess ? FP8_OK : FP8_ERR_CUDA; }

// The current device must be an sm_100 part (B200 class).
fp8_status_t check_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return FP8_ERR_NO_DEVICE;
  }
  int major = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) {
    cudaGetLastError();
    return FP8_ERR_NO_DEVICE;
  }
  return major == 10 ? FP8_OK : FP8_ERR_NO_DEVICE;
}

// Largest element count accepted by the elementwise kernels (their index math
// and their 4-byte-per-element inputs stay well inside 64 bits; 2^40 elements
// is far beyond any device's memory).
constexpr size_t kMaxElements = size_t(1) << 40;

// `*_tok` marks the tensors whose size is proportional to T: with T == 0
// they are empty and may be null.
fp8_status_t check_linear(const uint8_t* a, bool a_tok, int fa, const int32_t* ba,
                          const uint8_t* b, bool b_tok, int fb, const int32_t* bb, int64_t T,
                          int64_t in, int64_t out, const void* d, bool d_tok, int ddt) {
  const bool empty = T == 0;
  if (!ba || !bb) return FP8_ERR_INVALID_ARGUMENT;
  if ((!a && !(a_tok && empty)) || (!b && !(b_tok && empty)) || (!d && !(d_tok && empty)))
    return FP8_ERR_INVALID_ARGUMENT;
  if (!valid_fmt(fa) || !valid_fmt(fb) || !valid_dtype(ddt)) return FP8_ERR_INVALID_ARGUMENT;
  if (T < 0 || in <= 0 || out <= 0) return FP8_ERR_INVALID_ARGUMENT;
  if (in % 16 != 0 || out % 16 != 0) return FP8_ERR_UNSUPPORTED;
  if (T > (int64_t(1) << 31) - 1024 || in > (int64_t(1) << 31) - 1024 ||
      out > (int64_t(1) << 31) - 1024)
    return FP8_ERR_UNSUPPORTED;
  if ((a && !aligned16(a)) || (b && !aligned16(b)) || (d && !aligned16(d)))
    return FP8_ERR_MISALIGNED;
  if ((reinterpret_cast<uintptr_t>(ba) & 3u) || (reinterpret_cast<uintptr_t>(bb) & 3u))
    return FP8_ERR_MISALIGNED;
  return FP8_OK;
}

fp8_status_t run_gemm(const uint8_t* a, int fa, bool a_mn, const int32_t* ba, const uint8_t* b,
                      int fb, bool b_mn, const int32_t* bb, int64_t M, int64_t N, int64_t K,
                      void* d, int ddt, cudaStream_t s, float* d_amax = nullptr) {
  GemmArgs g;
  g.a = a;
  g.b = b;
  g.a_fmt = fa;
  g.b_fmt = fb;
  g.a_mn_major = a_mn;
  g.b_mn_major = b_mn;
  g.bias_a = ba;
  g.bias_b = bb;
  g.d = d;
  g.d_fp32 = ddt == FP8_DTYPE_FP32;
  g.d_amax = d_amax;
  g.M = M;
  g.N = N;
  g.K = K;
  return static_cast<fp8_status_t>(launch_gemm(g, s));
}

}  // namespace

extern "C" {

int fp8_abi_version(void) { return 1; }

const char* fp8_status_string(fp8_status_t st) {
  switch (st) {
    case FP8_OK: return "FP8_OK";
    case FP8_ERR_INVALID_ARGUMENT: return "FP8_ERR_INVALID_ARGUMENT";
    case FP8_ERR_UNSUPPORTED: return "FP8_ERR_UNSUPPORTED";
    case FP8_ERR_MISALIGNED: return "FP8_ERR_MISALIGNED";
    case FP8_ERR_CUDA: return "FP8_ERR_CUDA";
    case FP8_ERR_TIMEOUT: return "FP8_ERR_TIMEOUT";
    case FP8_ERR_NO_DEVICE: return "FP8_ERR_NO_DEVICE";
  }
  return "FP8_ERR_UNKNOWN";
}

fp8_status_t fp8_amax(const void* x, fp8_dtype_t dt, size_t n, float* amax, void* stream) {
  if (!amax || (n > 0 && !x) || !valid_dtype(dt)) return FP8_ERR_INVALID_ARGUMENT;
  if (n > kMaxElements) return FP8_ERR_UNSUPPORTED;
  if ((n > 0 && !aligned16(x)) || (reinterpret_cast<uintptr_t>(amax) & 3u))
    return FP8_ERR_MISALIGNED;
  if (fp8_status_t st = check_device()) return st;
  return from_cuda(launch_amax(x, dt, n, amax, as_stream(stream)));
}

fp8_status_t fp8_compute_bias(const float* amax, fp8_format_t fmt, int32_t margin, int32_t* bias,
                              void* stream) {
  if (!amax || !bias || !valid_fmt(fmt)) return FP8_ERR_INVALID_ARGUMENT;
  if ((reinterpret_cast<uintptr_t>(amax) & 3u) || (reinterpret_cast<uintptr_t>(bias) & 3u))
    return FP8_ERR_MISALIGNED;
  if (fp8_status_t st = check_device()) return st;
  return from_cuda(launch_compute_bias(amax, fmt, margin, bias, as_stream(stream)));
}

fp8_status_t fp8_cast_scaled(const void* x, fp8_dtype_t dt, size_t n, const int32_t* bias,
                             fp8_format_t fmt, uint8_t* out, void* stream) {
  if (!bias || !valid_dtype(dt) || !valid_fmt(fmt) || (n > 0 && (!x || !out)))
    return FP8_ERR_INVALID_ARGUMENT;
  if (n > kMaxElements) return FP8_ERR_UNSUPPORTED;
  if ((n > 0 && (!aligned16(x) || !aligned16(out))) || (reinterpret_cast<uintptr_t>(bias) & 3u))
    return FP8_ERR_MISALIGNED;
  if (fp8_status_t st = check_device()) return st;
  return from_cuda(launch_cast(x, dt, n, bias, fmt, out, as_stream(stream)));
}

fp8_status_t fp8_quantize(const void* x, fp8_dtype_t dt, size_t n, fp8_format_t fmt,
                          int32_t margin, float* amax, int32_t* bias, uint8_t* out,
                          void* stream) {
  if (!amax || !bias || !valid_dtype(dt) || !valid_fmt(fmt) || (n > 0 && (!x || !out)))
    return FP8_ERR_INVALID_ARGUMENT;
  if (n > kMaxElements) return FP8_ERR_UNSUPPORTED;
  if ((n > 0 && (!aligned16(x) || !aligned16(out))) ||
      (reinterpret_cast<uintptr_t>(amax) & 3u) || (reinterpret_cast<uintptr_t>(bias) & 3u))
    return FP8_ERR_MISALIGNED;
  if (fp8_status_t st = check_device()) return st;
  return from_cuda(launch_quantize(x, dt, n, fmt, margin, amax, bias, out, as_stream(stream)));
}

fp8_status_t fp8_linear_fwd(const uint8_t* x8, fp8_format_t fx, const int32_t* bias_x,
                            const uint8_t* w8, fp8_format_t fw, const int32_t* bias_w, int64_t T,
                            int64_t in, int64_t out, void* y, fp8_dtype_t y_dtype, void* stream) {
  if (fp8_status_t st = check_linear(x8, true, fx, bias_x, w8, false, fw, bias_w, T, in, out, y, true, y_dtype))
    return st;
  if (fp8_status_t st = check_device()) return st;
  if (T == 0) return FP8_OK;
  return run_gemm(x8, fx, false, bias_x, w8, fw, false, bias_w, T, out, in, y, y_dtype,
                  as_stream(stream));
}

fp8_status_t fp8_linear_bwd_dgrad(const uint8_t* dy8, fp8_format_t fdy, const int32_t* bias_dy,
                                  const uint8_t* w8, fp8_format_t fw, const int32_t* bias_w,
                                  int64_t T, int64_t in, int64_t out, void* dx,
                                  fp8_dtype_t dx_dtype, void* stream) {
  if (fp8_status_t st = check_linear(dy8, true, fdy, bias_dy, w8, false, fw, bias_w, T, in, out, dx, true,
                                             dx_dtype))
    return st;
  if (fp8_status_t st = check_device()) return st;
  if (T == 0) return FP8_OK;
  return run_gemm(dy8, fdy, false, bias_dy, w8, fw, true, bias_w, T, in, out, dx, dx_dtype,
                  as_stream(stream));
}

fp8_status_t fp8_linear_bwd_wgrad(const uint8_t* dy8, fp8_format_t fdy, const int32_t* bias_dy,
                                  const uint8_t* x8, fp8_format_t fx, const int32_t* bias_x,
                                  int64_t T, int64_t in, int64_t out, void* dw,
                                  fp8_dtype_t dw_dtype, void* stream) {
  if (fp8_status_t st = check_linear(dy8, true, fdy, bias_dy, x8, true, fx, bias_x, T, in, out, dw, false,
                                             dw_dtype))
    return st;
  if (fp8_status_t st = check_device()) return st;
  if (T == 0) {
    const size_t bytes = static_cast<size_t>(out) * static_cast<size_t>(in) *
                         (dw_dtype == FP8_DTYPE_FP32 ? 4 : 2);
    return from_cuda(cudaMemsetAsync(dw, 0, bytes, as_stream(stream)));
  }
  return run_gemm(dy8, fdy, true, bias_dy, x8, fx, true, bias_x, out, in, T, dw, dw_dtype,
                  as_stream(stream));
}

fp8_status_t fp8_linear_fwd_amax(const uint8_t* x8, fp8_format_t fx, const int32_t* bias_x,
                                 const uint8_t* w8, fp8_format_t fw, const int32_t* bias_w,
                                 int64_t T, int64_t in, int64_t out, void* y, fp8_dtype_t y_dtype,
                                 float* y_amax, void* stream) {
  if (!y_amax) return FP8_ERR_INVALID_ARGUMENT;
  if (reinterpret_cast<uintptr_t>(y_amax) & 3u) return FP8_ERR_MISALIGNED;
  if (fp8_status_t st = check_linear(x8, true, fx, bias_x, w8, false, fw, bias_w, T, in, out, y,
                                     true, y_dtype))
    return st;
  if (fp8_status_t st = check_device()) return st;
  if (cudaMemsetAsync(y_amax, 0, sizeof(float), as_stream(stream)) != cudaSuccess)
    return FP8_ERR_CUDA;
  if (T == 0) return FP8_OK;
  return run_gemm(x8, fx, false, bias_x, w8, fw, false, bias_w, T, out, in, y, y_dtype,
                  as_stream(stream), y_amax);
}

fp8_status_t fp8_linear_bwd_dgrad_amax(const uint8_t* dy8, fp8_format_t fdy,
                                       const int32_t* bias_dy, const uint8_t* w8, fp8_format_t fw,
                                       const int32_t* bias_w, int64_t T, int64_t in, int64_t out,
                                       void* dx, fp8_dtype_t dx_dtype, float* dx_amax,
                                       void* stream) {
  if (!dx_amax) return FP8_ERR_INVALID_ARGUMENT;
  if (reinterpret_cast<uintptr_t>(dx_amax) & 3u) return FP8_ERR_MISALIGNED;
  if (fp8_status_t st = check_linear(dy8, true, fdy, bias_dy, w8, false, fw, bias_w, T, in, out,
                                     dx, true, dx_dtype))
    return st;
  if (fp8_status_t st = check_device()) return st;
  if (cudaMemsetAsync(dx_amax, 0, sizeof(float), as_stream(stream)) != cudaSuccess)
    return FP8_ERR_CUDA;
  if (T == 0) return FP8_OK;
  return run_gemm(dy8, fdy, false, bias_dy, w8, fw, true, bias_w, T, in, out, dx, dx_dtype,
                  as_stream(stream), dx_amax);
}

size_t fp8_linear_fwd_workspace_size(int64_t T, int64_t in, int64_t out) {
  if (T <= 0 || in <= 0 || out <= 0 || check_device() != FP8_OK) return 0;
  GemmArgs g = {};
  g.M = T;
  g.N = out;
  g.K = in;
  return gemm_workspace_bytes(g);
}

fp8_status_t fp8_linear_fwd_ws(const uint8_t* x8, fp8_format_t fx, const int32_t* bias_x,
                               const uint8_t* w8, fp8_format_t fw, const int32_t* bias_w,
                               int64_t T, int64_t in, int64_t out, void* y, fp8_dtype_t y_dtype,
                               void* workspace, size_t workspace_bytes, void* stream) {
  if (fp8_status_t st = check_linear(x8, true, fx, bias_x, w8, false, fw, bias_w, T, in, out, y,
                                     true, y_dtype))
    return st;
  if (workspace_bytes > 0 && !workspace) return FP8_ERR_INVALID_ARGUMENT;
  if (reinterpret_cast<uintptr_t>(workspace) & 255u) return FP8_ERR_MISALIGNED;
  if (fp8_status_t st = check_device()) return st;
  if (T == 0) return FP8_OK;
  GemmArgs g = {};
  g.a = x8;
  g.b = w8;
  g.a_fmt = fx;
  g.b_fmt = fw;
  g.bias_a = bias_x;
  g.bias_b = bias_w;
  g.d = y;
  g.d_fp32 = y_dtype == FP8_DTYPE_FP32;
  g.M = T;
  g.N = out;
  g.K = in;
  const size_t need = gemm_workspace_bytes(g);
  if (need > 0) {
    if (workspace_bytes < need) return FP8_ERR_INVALID_ARGUMENT;
    g.workspace = workspace;
    g.workspace_bytes = workspace_bytes;
  }
  return static_cast<fp8_status_t>(launch_gemm(g, as_stream(stream)));
}

fp8_status_t fp8_linear_fwd_noalloc(const uint8_t* x8, fp8_format_t fx, const int32_t* bias_x,
                                    const uint8_t* w8, fp8_format_t fw, const int32_t* bias_w,
                                    int64_t T, int64_t in, int64_t out, void* y,
                                    fp8_dtype_t y_dtype, void* stream) {
  if (fp8_status_t st = check_linear(x8, true, fx, bias_x, w8, false, fw, bias_w, T, in, out, y,
                                     true, y_dtype))
    return st;
  if (fp8_status_t st = check_device()) return st;
  if (T == 0) return FP8_OK;
  GemmArgs g = {};
  g.a = x8;
  g.b = w8;
  g.a_fmt = fx;
  g.b_fmt = fw;
  g.bias_a = bias_x;
  g.bias_b = bias_w;
  g.d = y;
  g.d_fp32 = y_dtype == FP8_DTYPE_FP32;
  g.M = T;
  g.N = out;
  g.K = in;
  return static_cast<fp8_status_t>(launch_gemm_noalloc(g, as_stream(stream)));
}

size_t fp8_linear_bwd_wgrad_workspace_size(int64_t T, int64_t in, int64_t out) {
  if (T <= 0 || in <= 0 || out <= 0 || check_device() != FP8_OK) return 0;
  GemmArgs g = {};
  g.M = out;
  g.N = in;
  g.K = T;
  return gemm_workspace_bytes(g);
}

fp8_status_t fp8_linear_bwd_wgrad_ws(const uint8_t* dy8, fp8_format_t fdy, const int32_t* bias_dy,
                                     const uint8_t* x8, fp8_format_t fx, const int32_t* bias_x,
                                     int64_t T, int64_t in, int64_t out, void* dw,
                                     fp8_dtype_t dw_dtype, void* workspace,
                                     size_t workspace_bytes, void* stream) {
  if (fp8_status_t st = check_linear(dy8, true, fdy, bias_dy, x8, true, fx, bias_x, T, in, out, dw,
                                     false, dw_dtype))
    return st;
  if (workspace_bytes > 0 && !workspace) return FP8_ERR_INVALID_ARGUMENT;
  if (reinterpret_cast<uintptr_t>(workspace) & 255u) return FP8_ERR_MISALIGNED;
  if (fp8_status_t st = check_device()) return st;
  if (T == 0) {
    const size_t bytes = static_cast<size_t>(out) * static_cast<size_t>(in) *
                         (dw_dtype == FP8_DTYPE_FP32 ? 4 : 2);
    return from_cuda(cudaMemsetAsync(dw, 0, bytes, as_stream(stream)));
  }
  GemmArgs g = {};
  g.a = dy8;
  g.b = x8;
  g.a_fmt = fdy;
  g.b_fmt = fx;
  g.a_mn_major = true;
  g.b_mn_major = true;
  g.bias_a = bias_dy;
  g.bias_b = bias_x;
  g.d = dw;
  g.d_fp32 = dw_dtype == FP8_DTYPE_FP32;
  g.M = out;
  g.N = in;
  g.K = T;
  const size_t need = gemm_workspace_bytes(g);
  if (need > 0) {
    if (workspace_bytes < need) return FP8_ERR_INVALID_ARGUMENT;
    g.workspace = workspace;
    g.workspace_bytes = workspace_bytes;
  }
  return static_cast<fp8_status_t>(launch_gemm(g, as_stream(stream)));
}

fp8_status_t fp8_linear_plan(fp8_pass_t pass, int64_t T, int64_t in, int64_t out,
                             int with_workspace, fp8_gemm_plan_t* plan) {
  if (!plan || T < 0 || in < 0 || out < 0) return FP8_ERR_INVALID_ARGUMENT;
  if (pass != FP8_PASS_FWD && pass != FP8_PASS_DGRAD && pass != FP8_PASS_WGRAD)
    return FP8_ERR_INVALID_ARGUMENT;
  if (fp8_status_t st = check_device()) return st;
  GemmArgs g = {};
  g.M = pass == FP8_PASS_WGRAD ? out : T;
  g.N = pass == FP8_PASS_FWD ? out : in;
  g.K = pass == FP8_PASS_FWD ? in : (pass == FP8_PASS_DGRAD ? out : T);
  g.a_mn_major = pass == FP8_PASS_WGRAD;
  g.b_mn_major = pass != FP8_PASS_FWD;
  // the passes with a workspace entry point: fwd and wgrad
  static unsigned char marker;
  if (with_workspace && pass != FP8_PASS_DGRAD) g.workspace = &marker;
  GemmPlan p = {};
  gemm_plan(g, &p);
  plan->tile_m = p.tile_m;
  plan->tile_n = p.tile_n;
  plan->ctas_per_tile = p.ctas_per_tile;
  plan->k_splits = p.k_splits;
  return FP8_OK;
}

fp8_status_t fp8_device_error(int clear, int32_t* where) {
  if (fp8_status_t st = check_device()) return st;
  const int site = device_error_site(clear != 0);
  if (where) *where = site;
  if (site < 0) return FP8_ERR_CUDA;
  return site == 0 ? FP8_OK : FP8_ERR_TIMEOUT;
}

fp8_status_t fp8_selftest_bounded_wait(uint64_t timeout_ns) {
  if (timeout_ns < 1000000ull || timeout_ns > 5000000000ull) return FP8_ERR_INVALID_ARGUMENT;
  if (fp8_status_t st = check_device()) return st;
  if (device_error_site(true) < 0) return FP8_ERR_CUDA;
  if (launch_selftest_wait(timeout_ns) != cudaSuccess) return FP8_ERR_CUDA;
  int32_t where = 0;
  const fp8_status_t st = fp8_device_error(1, &where);
  if (st == FP8_ERR_TIMEOUT && where != 6) return FP8_ERR_CUDA;   // wrong site recorded
  return st;
}

}  // extern "C"
