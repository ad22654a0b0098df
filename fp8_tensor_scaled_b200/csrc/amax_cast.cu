// amax_cast.cu — the memory-bound steps of FP8-AMAX on sm_100a.
//
//   K1  amax          max |x| over a whole tensor: 128-bit loads (8 in flight
//                     per thread), integer max on the |x| bit patterns (packed
//                     2 x bf16 per 32-bit word with __vmaxu2), warp redux.sync
//                     max, block max in shared memory, one atomicMax per block
//                     into the caller's amax.
//   K1b compute_bias  floor(log2(fmt_max / amax)) - margin from the bits of
//                     amax, exact integer arithmetic (one thread).
//   K2  cast_scaled   q = cvt.rn.satfinite.{e4m3x2,e5m2x2}(x * 2^bias): one
//                     128-bit load and one coalesced 8-byte (bf16) or 4-byte
//                     (fp32) store per thread per item, 8 items in flight,
//                     walking the tensor from its end (see cast_kernel).
//
// Method: review page "Training and inference of large language models using
// 8-bit floating point", section "Proposed method" (per-tensor amax ->
// compute_bias with a margin -> scale before the FP8 cast; FP8_E4 for weights
// and activations, FP8_E5 for gradients).
//
// Non-negative IEEE floats order like their bit patterns read as unsigned
// integers, and every NaN pattern with the sign cleared is larger than the
// +inf pattern: an unsigned max over |x| bits is the float max that lets a NaN
// win over everything and an inf over every finite value.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <atomic>

#include "common.cuh"
#include "kernels.h"

namespace fp8amax {

namespace {

constexpr int kThreads = 256;
// Launch shapes, measured on 2^26-2^30-element BF16/FP32 tensors with L2
// flushed (unroll 4 / 8 x 4 / 8 / 16 blocks of 256 threads per SM): 8 loads in
// flight per thread and 8 blocks per SM for both kernels gave the fastest
// amax -> cast sequence (2^30 BF16: 0.840 ms = 6.39 TB/s of algorithmic bytes,
// against 0.858 ms for 4 loads per thread); the cast alone ran best at 4 blocks
// per SM, but not when it follows the amax pass.
constexpr int kAmaxUnroll = 8;
constexpr int kAmaxBlocksPerSm = 8;
constexpr int kCastUnroll = 8;
constexpr int kCastBlocksPerSm = 8;

// Bits of the largest finite value of each format: 448 = 1.75 * 2^8 and
// 57344 = 1.75 * 2^15, i.e. exponent 8 / 15 with mantissa 1.11b.
__device__ __forceinline__ int fmt_max_exponent(int fmt) { return fmt == FP8_E4M3 ? 8 : 15; }

// floor(log2(fmt_max / amax)) - margin, computed exactly from the fp32 bits.
// amax = (1 + m / 2^23) * 2^E (normalising subnormals).  fmt_max = 1.75 * 2^Ef.
// log2(fmt_max / amax) = Ef - E + log2(1.75 / (1 + m/2^23)); the last term is
// in [0, 0.81) when 1 + m/2^23 <= 1.75 (m <= 0x600000) and in (-0.2, 0)
// otherwise, so the floor is Ef - E - (m > 0x600000).
__device__ __forceinline__ int32_t bias_from_amax_bits(uint32_t u, int fmt, int32_t margin) {
  u &= 0x7FFFFFFFu;
  if (u == 0u || u >= 0x7F800000u) return 0;  // zero, inf, NaN
  int E;
  uint32_t m;
  if (u >= 0x00800000u) {
    E = static_cast<int>(u >> 23) - 127;
    m = u & 0x007FFFFFu;
  } else {
    const int p = 31 - __clz(u);  // subnormal: u * 2^-149, MSB at bit p < 23
    E = p - 149;
    m = (u << (23 - p)) & 0x007FFFFFu;
  }
  return fmt_max_exponent(fmt) - E - (m > 0x600000u ? 1 : 0) - margin;
}

// --------------------------------------------------------------------------
// K1: amax
// --------------------------------------------------------------------------
template <bool kBF16>
__global__ void __launch_bounds__(kThreads)
amax_kernel(const uint4* __restrict__ xv, size_t n_vec, const void* __restrict__ tail,
            uint32_t n_tail, uint32_t* __restrict__ amax_bits) {
  uint32_t m = 0;  // for bf16: two packed 16-bit |x| maxima
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const uint32_t mask = kBF16 ? 0x7FFF7FFFu : 0x7FFFFFFFu;

  for (; i + (kAmaxUnroll - 1) * stride < n_vec; i += kAmaxUnroll * stride) {
    uint4 v[kAmaxUnroll];
#pragma unroll
    for (int u = 0; u < kAmaxUnroll; ++u) v[u] = __ldg(xv + i + u * stride);
#pragma unroll
    for (int u = 0; u < kAmaxUnroll; ++u) {
      if (kBF16) {
        m = __vmaxu2(m, v[u].x & mask);
        m = __vmaxu2(m, v[u].y & mask);
        m = __vmaxu2(m, v[u].z & mask);
        m = __vmaxu2(m, v[u].w & mask);
      } else {
        m = max(m, max(max(v[u].x & mask, v[u].y & mask), max(v[u].z & mask, v[u].w & mask)));
      }
    }
  }
  for (; i < n_vec; i += stride) {
    const uint4 v = __ldg(xv + i);
    if (kBF16) {
      m = __vmaxu2(m, v.x & mask);
      m = __vmaxu2(m, v.y & mask);
      m = __vmaxu2(m, v.z & mask);
      m = __vmaxu2(m, v.w & mask);
    } else {
      m = max(m, max(max(v.x & mask, v.y & mask), max(v.z & mask, v.w & mask)));
    }
  }
  // ragged tail (< one 16-byte vector), handled by the first threads of block 0
  if (blockIdx.x == 0 && threadIdx.x < n_tail) {
    if (kBF16) {
      const uint32_t b = static_cast<const uint16_t*>(tail)[threadIdx.x] & 0x7FFFu;
      m = __vmaxu2(m, b);
    } else {
      m = max(m, static_cast<const uint32_t*>(tail)[threadIdx.x] & 0x7FFFFFFFu);
    }
  }
  // widen to fp32 bit patterns: a bf16 is the top half of an fp32
  uint32_t bits = kBF16 ? (max(m & 0xFFFFu, m >> 16) << 16) : m;
  bits = __reduce_max_sync(0xFFFFFFFFu, bits);

  __shared__ uint32_t warp_max[kThreads / 32];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (lane == 0) warp_max[warp] = bits;
  __syncthreads();
  if (warp == 0) {
    bits = lane < kThreads / 32 ? warp_max[lane] : 0u;
    bits = __reduce_max_sync(0xFFFFFFFFu, bits);
    if (lane == 0 && bits != 0u) atomicMax(amax_bits, bits);
  }
}

// --------------------------------------------------------------------------
// K1b: compute_bias
// --------------------------------------------------------------------------
__global__ void compute_bias_kernel(const uint32_t* __restrict__ amax_bits, int fmt,
                                    int32_t margin, int32_t* __restrict__ bias) {
  *bias = bias_from_amax_bits(*amax_bits, fmt, margin);
}

// --------------------------------------------------------------------------
// K2: scale + cast
// --------------------------------------------------------------------------
// Two fp32 values -> two FP8 codes, element `lo` in the low byte (memory
// order).  cvt's first source goes to the upper byte of the result.
template <int kFmt>
__device__ __forceinline__ uint32_t cvt_pair(float lo, float hi) {
  uint16_t r;
  if (kFmt == FP8_E4M3)
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  else
    asm("cvt.rn.satfinite.e5m2x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// 8 bf16 (one uint4) -> 8 codes (one uint2)
template <int kFmt>
__device__ __forceinline__ uint2 cast8_bf16(const uint4 v, const Pow2Scale& s) {
  uint2 o;
  o.x = cvt_pair<kFmt>(apply_pow2(bf16_lo(v.x), s), apply_pow2(bf16_hi(v.x), s)) |
        (cvt_pair<kFmt>(apply_pow2(bf16_lo(v.y), s), apply_pow2(bf16_hi(v.y), s)) << 16);
  o.y = cvt_pair<kFmt>(apply_pow2(bf16_lo(v.z), s), apply_pow2(bf16_hi(v.z), s)) |
        (cvt_pair<kFmt>(apply_pow2(bf16_lo(v.w), s), apply_pow2(bf16_hi(v.w), s)) << 16);
  return o;
}

// 4 fp32 (one uint4) -> 4 codes (one uint32)
template <int kFmt>
__device__ __forceinline__ uint32_t cast4_f32(const uint4 v, const Pow2Scale& s) {
  return cvt_pair<kFmt>(apply_pow2(__uint_as_float(v.x), s), apply_pow2(__uint_as_float(v.y), s)) |
         (cvt_pair<kFmt>(apply_pow2(__uint_as_float(v.z), s), apply_pow2(__uint_as_float(v.w), s))
          << 16);
}

// kFromAmax: the bias is derived here from *amax_bits (fused compute_bias);
// block 0 also writes it to bias_out.  Otherwise *bias_in is used as given.
template <bool kBF16, int kFmt, bool kFromAmax>
__global__ void __launch_bounds__(kThreads)
cast_kernel(const uint4* __restrict__ xv, size_t n_items, const void* __restrict__ tail,
            uint32_t n_tail, const int32_t* __restrict__ bias_in,
            const uint32_t* __restrict__ amax_bits, int32_t margin, int32_t* __restrict__ bias_out,
            uint8_t* __restrict__ out) {
  int32_t bias;
  if (kFromAmax) {
    bias = bias_from_amax_bits(*amax_bits, kFmt, margin);
    if (blockIdx.x == 0 && threadIdx.x == 0) *bias_out = bias;
  } else {
    bias = *bias_in;
  }
  const Pow2Scale s = make_pow2_scale(bias);
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;

  // Items are visited from the end of the tensor towards its start, so that
  // right after an amax pass over the same tensor the first reads here hit the
  // part of it that is still resident in L2.
  const size_t last = n_items - 1;
  if (kBF16) {
    uint2* o = reinterpret_cast<uint2*>(out);
    for (; i + (kCastUnroll - 1) * stride < n_items; i += kCastUnroll * stride) {
      uint4 v[kCastUnroll];
#pragma unroll
      for (int u = 0; u < kCastUnroll; ++u) v[u] = __ldcs(xv + (last - i - u * stride));
#pragma unroll
      for (int u = 0; u < kCastUnroll; ++u) o[last - i - u * stride] = cast8_bf16<kFmt>(v[u], s);
    }
    for (; i < n_items; i += stride) o[last - i] = cast8_bf16<kFmt>(__ldcs(xv + (last - i)), s);
  } else {
    uint32_t* o = reinterpret_cast<uint32_t*>(out);
    for (; i + (kCastUnroll - 1) * stride < n_items; i += kCastUnroll * stride) {
      uint4 v[kCastUnroll];
#pragma unroll
      for (int u = 0; u < kCastUnroll; ++u) v[u] = __ldcs(xv + (last - i - u * stride));
#pragma unroll
      for (int u = 0; u < kCastUnroll; ++u) o[last - i - u * stride] = cast4_f32<kFmt>(v[u], s);
    }
    for (; i < n_items; i += stride) o[last - i] = cast4_f32<kFmt>(__ldcs(xv + (last - i)), s);
  }
  // ragged tail (< one item): one element per thread of block 0
  if (blockIdx.x == 0 && threadIdx.x < n_tail) {
    const float x = kBF16 ? bf16_lo(static_cast<const uint16_t*>(tail)[threadIdx.x])
                          : static_cast<const float*>(tail)[threadIdx.x];
    const size_t base = n_items * (kBF16 ? 8 : 4);
    out[base + threadIdx.x] = static_cast<uint8_t>(cvt_pair<kFmt>(apply_pow2(x, s), 0.0f) & 0xFFu);
  }
}

// SM count per device, filled on first use (possibly by several host threads
// at once, all storing the same value).
std::atomic<int> g_num_sms[64];

int num_sms() {
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  int n = g_num_sms[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    n = n > 0 ? n : 148;
    g_num_sms[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

// Blocks for a streaming kernel over `items` 16-byte vectors: `blocks_per_sm`
// blocks on every SM, but no more than one item per thread per unrolled
// iteration needs.
unsigned grid_for(size_t items, int unroll, int blocks_per_sm) {
  const size_t per_block = static_cast<size_t>(kThreads) * unroll;
  size_t want = (items + per_block - 1) / per_block;
  const size_t cap = static_cast<size_t>(num_sms()) * blocks_per_sm;
  if (want > cap) want = cap;
  if (want < 1) want = 1;
  return static_cast<unsigned>(want);
}

}  // namespace

cudaError_t launch_amax(const void* x, int dt, size_t n, float* amax, cudaStream_t s) {
  cudaError_t e = cudaMemsetAsync(amax, 0, sizeof(float), s);
  if (e != cudaSuccess || n == 0) return e;
  const size_t per_vec = dt == FP8_DTYPE_BF16 ? 8 : 4;
  const size_t n_vec = n / per_vec;
  const uint32_t n_tail = static_cast<uint32_t>(n % per_vec);
  const size_t esz = dt == FP8_DTYPE_BF16 ? 2 : 4;
  const void* tail = static_cast<const uint8_t*>(x) + n_vec * per_vec * esz;
  const unsigned grid = grid_for(n_vec, kAmaxUnroll, kAmaxBlocksPerSm);
  if (dt == FP8_DTYPE_BF16)
    amax_kernel<true><<<grid, kThreads, 0, s>>>(static_cast<const uint4*>(x), n_vec, tail, n_tail,
                                                reinterpret_cast<uint32_t*>(amax));
  else
    amax_kernel<false><<<grid, kThreads, 0, s>>>(static_cast<const uint4*>(x), n_vec, tail, n_tail,
                                                 reinterpret_cast<uint32_t*>(amax));
  return cudaGetLastError();
}

cudaError_t launch_compute_bias(const float* amax, int fmt, int32_t margin, int32_t* bias,
                                cudaStream_t s) {
  compute_bias_kernel<<<1, 1, 0, s>>>(reinterpret_cast<const uint32_t*>(amax), fmt, margin, bias);
  return cudaGetLastError();
}

namespace {
template <bool kBF16, bool kFromAmax>
cudaError_t launch_cast_t(const void* x, size_t n, int fmt, const int32_t* bias_in,
                          const float* amax, int32_t margin, int32_t* bias_out, uint8_t* out,
                          cudaStream_t s) {
  const size_t per_item = kBF16 ? 8 : 4;
  const size_t n_items = n / per_item;
  const uint32_t n_tail = static_cast<uint32_t>(n % per_item);
  const void* tail = static_cast<const uint8_t*>(x) + n_items * per_item * (kBF16 ? 2 : 4);
  const unsigned grid = grid_for(n_items, kCastUnroll, kCastBlocksPerSm);
  const uint4* xv = static_cast<const uint4*>(x);
  const uint32_t* ab = reinterpret_cast<const uint32_t*>(amax);
  if (fmt == FP8_E4M3)
    cast_kernel<kBF16, FP8_E4M3, kFromAmax><<<grid, kThreads, 0, s>>>(
        xv, n_items, tail, n_tail, bias_in, ab, margin, bias_out, out);
  else
    cast_kernel<kBF16, FP8_E5M2, kFromAmax><<<grid, kThreads, 0, s>>>(
        xv, n_items, tail, n_tail, bias_in, ab, margin, bias_out, out);
  return cudaGetLastError();
}
}  // namespace

cudaError_t launch_cast(const void* x, int dt, size_t n, const int32_t* bias, int fmt,
                        uint8_t* out, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  if (dt == FP8_DTYPE_BF16)
    return launch_cast_t<true, false>(x, n, fmt, bias, nullptr, 0, nullptr, out, s);
  return launch_cast_t<false, false>(x, n, fmt, bias, nullptr, 0, nullptr, out, s);
}

cudaError_t launch_quantize(const void* x, int dt, size_t n, int fmt, int32_t margin,
                            float* amax, int32_t* bias, uint8_t* out, cudaStream_t s) {
  cudaError_t e = launch_amax(x, dt, n, amax, s);
  if (e != cudaSuccess) return e;
  if (n == 0) return launch_compute_bias(amax, fmt, margin, bias, s);
  if (dt == FP8_DTYPE_BF16)
    return launch_cast_t<true, true>(x, n, fmt, nullptr, amax, margin, bias, out, s);
  return launch_cast_t<false, true>(x, n, fmt, nullptr, amax, margin, bias, out, s);
}

}  // namespace fp8amax
