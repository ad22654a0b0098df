/*
 * A plain C caller of the FP8-AMAX library: no Python, no torch.  It owns its
 * device memory (cudaMalloc), runs the whole per-tensor step and a forward
 * GEMM through include/fp8amax.h, and checks the results against the CPU
 * oracle's C functions (linked from oracle/liboracle.so, test use only).
 *
 *   T x in = 200 x 272 activations, out = 400: ragged against every tile edge.
 *
 * Exit status 0 on success; prints the first mismatch otherwise.
 */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cuda_runtime.h>

#include "fp8amax.h"

/* oracle (test infrastructure) */
float oracle_amax_f32(const float *x, size_t n);
int32_t oracle_compute_bias(float amax, int fmt, int margin);
void oracle_cast_scaled_f32(const float *x, size_t n, int32_t bias, int fmt, uint8_t *out);
void oracle_linear_full(int pass, const uint8_t *A, int fa, int32_t bias_a, const uint8_t *B,
                        int fb, int32_t bias_b, int64_t T, int64_t in, int64_t out, double *val,
                        double *absval);

#define CK(call)                                                                  \
  do {                                                                            \
    cudaError_t e_ = (call);                                                      \
    if (e_ != cudaSuccess) {                                                      \
      fprintf(stderr, "%s failed: %s\n", #call, cudaGetErrorString(e_));           \
      return 2;                                                                   \
    }                                                                             \
  } while (0)
#define FP(call)                                                                  \
  do {                                                                            \
    fp8_status_t s_ = (call);                                                     \
    if (s_ != FP8_OK) {                                                           \
      fprintf(stderr, "%s failed: %s\n", #call, fp8_status_string(s_));            \
      return 3;                                                                   \
    }                                                                             \
  } while (0)

static float frand(uint64_t *s) { /* xorshift, then a sum of uniforms (about N(0,1)) */
  float acc = 0.0f;
  for (int i = 0; i < 4; ++i) {
    *s ^= *s << 13; *s ^= *s >> 7; *s ^= *s << 17;
    acc += (float)((*s >> 11) * (1.0 / 9007199254740992.0)) - 0.5f;
  }
  return acc * 1.7320508f;
}

int main(void) {
  const int64_t T = 200, IN = 272, OUT = 400;
  const size_t nx = (size_t)(T * IN), nw = (size_t)(OUT * IN), ny = (size_t)(T * OUT);
  uint64_t seed = 0x9E3779B97F4A7C15ull;
  float *hx = malloc(nx * 4), *hw = malloc(nw * 4), *hy = malloc(ny * 4);
  uint8_t *hx8 = malloc(nx), *hw8 = malloc(nw), *rx8 = malloc(nx), *rw8 = malloc(nw);
  double *ref = malloc(ny * 8), *absref = malloc(ny * 8);
  for (size_t i = 0; i < nx; ++i) hx[i] = frand(&seed);
  for (size_t i = 0; i < nw; ++i) hw[i] = 0.02f * frand(&seed);

  float *dx, *dw, *dy, *damax;
  uint8_t *dx8, *dw8;
  int32_t *dbias;
  CK(cudaMalloc((void **)&dx, nx * 4));
  CK(cudaMalloc((void **)&dw, nw * 4));
  CK(cudaMalloc((void **)&dy, ny * 4));
  CK(cudaMalloc((void **)&dx8, nx));
  CK(cudaMalloc((void **)&dw8, nw));
  CK(cudaMalloc((void **)&damax, 2 * sizeof(float)));
  CK(cudaMalloc((void **)&dbias, 2 * sizeof(int32_t)));
  CK(cudaMemcpy(dx, hx, nx * 4, cudaMemcpyHostToDevice));
  CK(cudaMemcpy(dw, hw, nw * 4, cudaMemcpyHostToDevice));

  cudaStream_t st;
  CK(cudaStreamCreate(&st));
  FP(fp8_quantize(dx, FP8_DTYPE_FP32, nx, FP8_E4M3, 0, damax, dbias, dx8, st));
  FP(fp8_quantize(dw, FP8_DTYPE_FP32, nw, FP8_E4M3, 0, damax + 1, dbias + 1, dw8, st));
  FP(fp8_linear_fwd(dx8, FP8_E4M3, dbias, dw8, FP8_E4M3, dbias + 1, T, IN, OUT, dy,
                    FP8_DTYPE_FP32, st));
  CK(cudaStreamSynchronize(st));

  float amax[2];
  int32_t bias[2];
  CK(cudaMemcpy(amax, damax, sizeof amax, cudaMemcpyDeviceToHost));
  CK(cudaMemcpy(bias, dbias, sizeof bias, cudaMemcpyDeviceToHost));
  CK(cudaMemcpy(hx8, dx8, nx, cudaMemcpyDeviceToHost));
  CK(cudaMemcpy(hw8, dw8, nw, cudaMemcpyDeviceToHost));
  CK(cudaMemcpy(hy, dy, ny * 4, cudaMemcpyDeviceToHost));

  /* oracle: the same steps on the CPU */
  const float ra[2] = {oracle_amax_f32(hx, nx), oracle_amax_f32(hw, nw)};
  const int32_t rb[2] = {oracle_compute_bias(ra[0], 0, 0), oracle_compute_bias(ra[1], 0, 0)};
  oracle_cast_scaled_f32(hx, nx, rb[0], 0, rx8);
  oracle_cast_scaled_f32(hw, nw, rb[1], 0, rw8);
  for (int i = 0; i < 2; ++i)
    if (memcmp(&amax[i], &ra[i], 4) != 0 || bias[i] != rb[i]) {
      fprintf(stderr, "tensor %d: amax %g vs %g, bias %d vs %d\n", i, amax[i], ra[i], bias[i],
              rb[i]);
      return 1;
    }
  if (memcmp(hx8, rx8, nx) != 0 || memcmp(hw8, rw8, nw) != 0) {
    fprintf(stderr, "FP8 codes differ\n");
    return 1;
  }
  oracle_linear_full(0, rx8, 0, rb[0], rw8, 0, rb[1], T, IN, OUT, ref, absref);
  for (size_t i = 0; i < ny; ++i) {
    const double a = fabs(ref[i]);
    double ulp = a > 0 ? ldexp(1.0, (int)floor(log2(a)) - 7) : 0.0;
    if (ulp < ldexp(1.0, -133)) ulp = ldexp(1.0, -133);
    if (fabs((double)hy[i] - ref[i]) > 1e-3 * absref[i] + ulp) {
      fprintf(stderr, "Y[%zu] = %.9g, oracle %.9g\n", i, hy[i], ref[i]);
      return 1;
    }
  }
  printf("C ABI example ok: amax %g/%g bias %d/%d, %lld x %lld Y within tolerance\n", amax[0],
         amax[1], bias[0], bias[1], (long long)T, (long long)OUT);
  return 0;
}
