// gemm_sm100.cu — the FP8 matmuls of the FP8-AMAX linear layer on sm_100a.
//
// D[M,N] = (A[M,K] . B[N,K]^T) * 2^-(bias_a + bias_b), FP8 operands (E4M3 or
// E5M2, any mix), fp32 accumulation in tensor memory, one RNE conversion to
// BF16 or FP32 in the epilogue.  The three passes of a linear layer map to it
// without any transpose copy (review page "Training and inference of large
// language models using 8-bit floating point", "Proposed method": the matmul
// runs on the scaled FP8 operands and its output is unscaled afterwards):
//   fwd    Y  = X . W^T      A = X  [T,in]  K-major,  B = W [out,in] K-major
//   dgrad  dX = dY . W       A = dY [T,out] K-major,  B = W [out,in] MN-major
//   wgrad  dW = dY^T . X     A = dY [T,out] MN-major, B = X [T,in]   MN-major
//
// Design (one CTA per SM, persistent, warp-specialised, 192 threads):
//   Tiles of 256 x 256 are computed by a CTA pair (a cluster of two) with
//   tcgen05.mma.cta_group::2 (M=256, N=256, K=32): CTA r holds rows
//   [128r, 128r+128) of the A tile, rows [128r, 128r+128) of the B tile and of
//   the accumulator.  Problems with M <= 128 use one CTA per 128 x 256 tile;
//   problems of many tiles use 256 x 512 tiles (two such MMAs per K step that
//   share the A stage: a quarter less L2 traffic per FLOP).
//   warp 0      TMA producer: 128 x 128-byte FP8 boxes with 128-byte swizzle
//               (no multicast: each CTA loads its own halves) into a ring of
//               192 KB per CTA (6 x 32 KB for 256 x 256 tiles, 4 x 48 KB for
//               256 x 512 and 128 x 256 tiles); the pair's copies complete on
//               the leader's mbarrier, armed with the bytes of both CTAs.
//   warp 1      TMEM allocator (512 columns = two 128 x 256 fp32 accumulators
//               per CTA, or one 128 x 512 for 256 x 512 tiles); in the
//               leader, one thread issues the MMAs and tcgen05.commit,
//               multicast to both CTAs' barriers, which frees each stage and
//               publishes each finished accumulator.
//   warps 2-5   epilogue: tcgen05.ld 32x32b of the CTA's accumulator rows,
//               multiply by the power of two 2^-(bias_a+bias_b), one rounding
//               to BF16/FP32 into a swizzled shared-memory box, one TMA store
//               per box.  Two accumulators (or two halves of one) let it
//               overlap the next tile's mainloop.
// Tiles are visited in groups of 16 N-blocks, N fastest inside a group, so
// that the clusters running at one time share A and B panels in L2.
//
// Every mbarrier wait is bounded in time.  A wait that runs out records its
// site in a device error word, raises a block-wide abort flag, and every role
// leaves its loop; the MMA thread and the producer then drain their own
// in-flight tensor-core work and copies (again with bounded waits) before the
// tensor memory is released and the block exits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <atomic>

#include "common.cuh"
#include "kernels.h"

namespace fp8amax {

// Device error word: 0 or the site of the first bounded wait that ran out.
static __device__ int g_device_error = 0;

namespace {

enum WaitSite : int {
  kSiteProducerEmpty = 1,
  kSiteMmaFull = 2,
  kSiteMmaTmemEmpty = 3,
  kSiteEpilogueTmemFull = 4,
  kSiteDrain = 5,
  kSiteSelfTest = 6,
};

constexpr uint64_t kWaitLimitNs = 2000000000ull;   // 2 s; a correct kernel waits microseconds
constexpr uint64_t kDrainLimitNs = 100000000ull;   // 100 ms for draining after an abort

__device__ __forceinline__ void record_device_error(int site) {
  atomicCAS(&g_device_error, 0, site);
}

// Wait until the phase with the given parity has completed, for at most
// `limit_ns`.  Returns false when the wait gave up: either the limit ran out
// (the site is recorded and *abort raised) or another role raised *abort.
// Called by ONE thread.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity,
                                                  volatile int* abort_flag, int site,
                                                  uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > limit_ns) {
      *abort_flag = 1;
      record_device_error(site);
      return false;
    }
  }
}

// Tile shapes (kTile):
//   kTileSingle  one CTA computes a 128 x 256 tile with tcgen05.mma.cta_group::1
//                (M=128, N=256); B may be K- or MN-major.
//   kTilePair    a pair of CTAs (a cluster of 2) computes a 256 x 256 tile with
//                cta_group::2 (M=256, N=256): CTA r loads rows [128r, 128r+128)
//                of the A tile and of the B tile into its own shared memory and
//                holds rows [128r, 128r+128) of the accumulator in its own tensor
//                memory; the leader (r = 0) issues the MMAs for both.
//   kTileNarrow  one CTA computes a 128 x 64 tile (M=128, N=64), K-major B only:
//                for few rows (decode-sized T) the GEMM streams the weights, and
//                narrow tiles give every SM a share of them.
//   kTileDouble  a CTA pair computes a 256 x 512 tile as two cta_group::2 MMAs
//                (M=256, N=256) per K step that share the A stage: CTA r loads
//                A rows [128r, +128) and B rows [128r, +128) and [256+128r, +128)
//                of the tile.  A CTA moves 48 KB from L2 per 128 x 512 x 128
//                block instead of 64 KB for two 128 x 256 blocks (a quarter
//                less L2 -> shared memory traffic per FLOP), at the price of a
//                single 512-column accumulator: the epilogue drains it in two
//                256-column halves, and the next tile's MMAs into a half wait
//                only for that half.
constexpr int BK = 128;                 // K per stage: one 128-byte swizzle row of FP8
constexpr int UK = 32;                  // K per tcgen05.mma of kind::f8f6f4
constexpr uint32_t A_BYTES = 128 * BK;  // 16 KB: 128 rows of A per CTA
constexpr int kThreads = 192;           // 6 warps

enum TileKind : int { kTileSingle = 0, kTilePair = 1, kTileNarrow = 2, kTileDouble = 3 };

// BN: tile columns; MMA_N: N of one tcgen05.mma; B_ROWS: B rows per CTA and stage.
template <int kTile> struct Cfg;
template <> struct Cfg<kTileSingle> {
  static constexpr int CTAS = 1, BM = 128, BN = 256, MMA_N = 256, B_ROWS = 256, STAGES = 4;
};
template <> struct Cfg<kTilePair> {
  static constexpr int CTAS = 2, BM = 256, BN = 256, MMA_N = 256, B_ROWS = 128, STAGES = 6;
};
template <> struct Cfg<kTileNarrow> {
  static constexpr int CTAS = 1, BM = 128, BN = 64, MMA_N = 64, B_ROWS = 64, STAGES = 8;
};
template <> struct Cfg<kTileDouble> {
  static constexpr int CTAS = 2, BM = 256, BN = 512, MMA_N = 256, B_ROWS = 256, STAGES = 4;
};
constexpr uint32_t B_HALF_BYTES = 128 * BK;   // 16 KB: one 128-row B box
// Double-width tile: stages of a new tile multiplied into the first half of
// the accumulator only, while the epilogue still drains the second half
// (1 <= kDeferStages <= the ring depth).
constexpr int kDeferStages = 4;
template <int kTile> constexpr uint32_t b_bytes() { return Cfg<kTile>::B_ROWS * BK; }
template <int kTile> constexpr uint32_t stage_bytes() { return A_BYTES + b_bytes<kTile>(); }
// two fp32 accumulators of BN columns each; the wide tile has one of 512
template <int kTile> constexpr uint32_t tmem_cols() {
  return kTile == kTileDouble ? 512u : 2u * Cfg<kTile>::BN;
}
template <int kTile> constexpr int num_bars() { return 2 * Cfg<kTile>::STAGES + 2 + 2 + 1; }
// Epilogue staging for the TMA store of D: per epilogue warp, 32 rows x 128
// bytes, twice (two 32-column fp32 boxes or one 64-column BF16 box).
constexpr uint32_t kStageOutBytesPerWarp = 2 * 32 * 128;
constexpr uint32_t kStageOutBytes = 4 * kStageOutBytesPerWarp;   // 32 KB
template <int kTile> constexpr size_t smem_bytes() {
  return 1024 + Cfg<kTile>::STAGES * stage_bytes<kTile>() + kStageOutBytes +
         num_bars<kTile>() * 8 + 16;
}
static_assert(smem_bytes<kTileSingle>() <= 232448 && smem_bytes<kTilePair>() <= 232448 &&
                  smem_bytes<kTileNarrow>() <= 232448 && smem_bytes<kTileDouble>() <= 232448,
              "227 KB of shared memory per block");

struct Params {
  int M, N, K;
  int num_m_blocks, num_n_blocks, num_k_blocks, num_tiles;
  int group_n;
  // Split K: each tile's K range is cut into `splits` ranges of kb_per_split
  // k-blocks; work unit u is (tile u / splits, range u % splits).  With
  // splits > 1 every unit writes its raw fp32 partial to ws[range][M][N] and
  // splitk_reduce_kernel, launched next on the same stream, adds the partials
  // in range order and runs the epilogue.
  int splits, kb_per_split, num_work;
  float* ws;
  uint32_t idesc;
  const int32_t* bias_a;
  const int32_t* bias_b;
  void* d;
  uint32_t* amax_out;        // fp32 bits of max |D|; used when the kernel has kAmax
  uint64_t wait_limit_ns;
};

// Shared-memory matrix descriptor (tcgen05 format): start address, leading
// and stride byte offsets (all >> 4), descriptor version 1 at bit 46,
// 128-byte swizzle (layout type 2) in bits 61-63.
__device__ __forceinline__ uint64_t make_sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= 1ull << 46;
  d |= 2ull << 61;
  return d;
}

// K-major operand (rows of 128 K-bytes, 8-row swizzle atoms of 1 KB):
// SBO = 1024 between 8-row groups, LBO unused (16); sub-step k advances the
// start address by 32 bytes inside the swizzle row.
// MN-major operand (rows of 128 MN-bytes, one per K index): SBO = 1024 between
// groups of 8 K rows, LBO = 16 KB between 128-wide MN chunks; sub-step k
// advances by 32 K rows = 4 KB.
template <bool kMN>
__device__ __forceinline__ uint64_t operand_desc(uint32_t stage_base, int k) {
  if (kMN) return make_sdesc(stage_base + k * (UK * 128), BK * 128, 1024);
  return make_sdesc(stage_base + k * UK, 16, 1024);
}

__device__ __forceinline__ void tile_coords(int t, const Params& p, int& mb, int& nb) {
  const int group_size = p.group_n * p.num_m_blocks;
  const int g = t / group_size;
  const int first_n = g * p.group_n;
  const int gn = min(p.group_n, p.num_n_blocks - first_n);
  const int r = t - g * group_size;
  mb = r / gn;
  nb = first_n + r % gn;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

template <int kCta>
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                         int site, uint64_t limit_ns) {
  if (kCta == 1) return mbar_wait_bounded(bar, parity, abort_flag, site, limit_ns);
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait_cluster(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > limit_ns) {
      *abort_flag = 1;
      record_device_error(site);
      return false;
    }
  }
}

// 2^e applied as one multiply when e is a normal exponent (the usual case:
// the whole tile is checked once), else as the split multiplies.
template <bool kSplit>
__device__ __forceinline__ float scale_pow2(float x, const Pow2Scale& s) {
  if (!kSplit) return x * s.f0;
  return (x * s.f0 * s.f1) * s.f2;
}

template <bool kOutF32, bool kAmax, bool kSplit>
__device__ __forceinline__ void stage_out_chunks_t(uint32_t stage, int lane,
                                                   const uint32_t (&r0)[32],
                                                   const uint32_t (&r1)[32], const Pow2Scale& sc,
                                                   uint32_t& dmax) {
  const uint32_t row_base = stage + static_cast<uint32_t>(lane) * 128u;
  const uint32_t sw = static_cast<uint32_t>(lane & 7);
  if (kOutF32) {
#pragma unroll
    for (int b = 0; b < 2; ++b) {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint32_t bits = b == 0 ? r0[4 * j + e] : r1[4 * j + e];
          w[e] = __float_as_uint(scale_pow2<kSplit>(__uint_as_float(bits), sc));
          if (kAmax) dmax = max(dmax, w[e] & 0x7FFFFFFFu);
        }
        const uint32_t addr = row_base + static_cast<uint32_t>(b) * 4096u +
                              ((static_cast<uint32_t>(j) ^ sw) << 4);
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};"
                     ::"r"(addr), "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]) : "memory");
      }
    }
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      uint32_t w[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int col = 8 * j + 2 * e;          // 0..63
        const uint32_t lo = col < 32 ? r0[col] : r1[col - 32];
        const uint32_t hi = col < 32 ? r0[col + 1] : r1[col - 31];
        w[e] = pack_bf16x2(scale_pow2<kSplit>(__uint_as_float(lo), sc),
                           scale_pow2<kSplit>(__uint_as_float(hi), sc));
        if (kAmax) dmax = __vmaxu2(dmax, w[e] & 0x7FFF7FFFu);
      }
      const uint32_t addr = row_base + ((static_cast<uint32_t>(j) ^ sw) << 4);
      asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};"
                   ::"r"(addr), "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]) : "memory");
    }
  }
}

// Scale and round one row's 64 accumulator columns (fp32 bits: r0 = columns
// 0..31, r1 = 32..63) and write them to the warp's staging buffer at `stage`
// (row `lane`, 128-byte rows, 128-byte swizzle: 16-byte piece j of a row
// goes to piece j ^ (lane % 8)).  BF16: one 64-column box of 128-byte rows.
// FP32: two 32-column boxes, the second 4 KB after the first.  With kAmax
// also fold max |stored| into dmax.
template <bool kOutF32, bool kAmax>
__device__ __forceinline__ void stage_out_chunks(uint32_t stage, int lane, const uint32_t (&r0)[32],
                                                 const uint32_t (&r1)[32], const Pow2Scale& sc,
                                                 uint32_t& dmax) {
  if (sc.split) stage_out_chunks_t<kOutF32, kAmax, true>(stage, lane, r0, r1, sc, dmax);
  else          stage_out_chunks_t<kOutF32, kAmax, false>(stage, lane, r0, r1, sc, dmax);
}

// kAmax: the epilogue also takes the max of |D| over the values it stores
// (after the rounding to the output type), reduces it per warp and combines
// it into *p.amax_out with one atomicMax per warp (NaN > inf > finite, as in
// the amax kernel), so the next layer's quantization needs no read of D.
template <int kTile, bool kAMN, bool kBMN, bool kOutF32, bool kAmax>
__global__ void __launch_bounds__(kThreads, 1)
fp8_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a,
                const __grid_constant__ CUtensorMap tmap_b,
                const __grid_constant__ CUtensorMap tmap_d, const Params p) {
  using C = Cfg<kTile>;
  constexpr int kCta = C::CTAS;
  constexpr int BN = C::BN;
  constexpr int STAGES = C::STAGES;
  constexpr uint32_t B_BYTES = b_bytes<kTile>();
  constexpr uint32_t STAGE_BYTES = stage_bytes<kTile>();
  constexpr uint32_t TMEM_COLS = tmem_cols<kTile>();
  constexpr int kNumBars = num_bars<kTile>();
  // wide tile: one accumulator in two halves; tempty_bar(h) frees half h
  constexpr bool kDbl = kTile == kTileDouble;
  constexpr int kHalves = kDbl ? 2 : 1;
  static_assert(kTile != kTileNarrow || !kBMN, "narrow tiles take a K-major B only");
  static_assert(TMEM_COLS <= 512, "tensor memory holds 512 columns");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * A_BYTES;
  uint8_t* sOut = smem + STAGES * STAGE_BYTES;                 // 1024-byte aligned
  uint64_t* bars = reinterpret_cast<uint64_t*>(sOut + kStageOutBytes);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + a); };
  auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + 2 + a); };
  const uint32_t drain_bar = bar0 + 8u * (2 * STAGES + 4);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const uint32_t rank = kCta == 2 ? cluster_ctarank() : 0u;     // 0 = leader
  const bool leader = rank == 0;
  const int unit = kCta == 2 ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int num_units = kCta == 2 ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);            // the leader's producer arrives (with expect_tx)
      mbar_init(empty_bar(s), 1);           // one tcgen05.commit per stage use
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), 4 * kCta);   // one arrival per epilogue warp of the pair
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
    tma_prefetch_desc(&tmap_a);
    tma_prefetch_desc(&tmap_b);
    tma_prefetch_desc(&tmap_d);
  }
  if (warp == 1) {
    if (kCta == 2) {
      tmem_alloc_pair(smem_u32(tmem_slot), TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  if (kCta == 2) cluster_sync();            // both CTAs' barriers and TMEM ready
  else __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ----------------------------- TMA producer -----------------------------
    // Both CTAs load their own halves; the copies complete on the leader's
    // full barrier, which the leader arms with the bytes of both CTAs.
    int stage = 0;
    uint32_t phase = 0;
    uint32_t armed_mask = 0, armed_parity = 0;   // leader: last armed phase per stage
    for (int u = unit; u < p.num_work && !*abort_flag; u += num_units) {
      const int t = u / p.splits;
      const int kb0 = (u - t * p.splits) * p.kb_per_split;
      const int kb1 = min(kb0 + p.kb_per_split, p.num_k_blocks);
      int mb, nb;
      tile_coords(t, p, mb, nb);
      const int a_row = mb * C::BM + static_cast<int>(rank) * 128;
      const int b_row = nb * BN + (kCta == 2 ? static_cast<int>(rank) * 128 : 0);
      // double-width tile: whether its second 256 columns hold any of D (else
      // that half is neither loaded nor multiplied)
      const bool half1 = kDbl && nb * BN + 256 < p.N;
      const uint32_t tx_bytes = kDbl ? (half1 ? STAGE_BYTES : A_BYTES + B_HALF_BYTES) : STAGE_BYTES;
      bool ok = true;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!wait_bar<kCta>(empty_bar(stage), phase ^ 1u, abort_flag, kSiteProducerEmpty,
                            p.wait_limit_ns)) {
          ok = false;
          break;
        }
        const uint32_t fb = full_bar(stage);
        if (leader) {
          mbar_arrive_expect_tx(fb, kCta * tx_bytes);
          armed_mask |= 1u << stage;
          armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
        }
        const uint32_t a_dst = smem_u32(sA + stage * A_BYTES);
        const uint32_t b_dst = smem_u32(sB + stage * B_BYTES);
        const int k0 = kb * BK;
        if (kCta == 2) {
          const uint32_t fb_leader = mapa_shared(fb, 0);
          if (kAMN) tma_load_2d_pair(a_dst, &tmap_a, fb_leader, a_row, k0);
          else      tma_load_2d_pair(a_dst, &tmap_a, fb_leader, k0, a_row);
          if (kBMN) tma_load_2d_pair(b_dst, &tmap_b, fb_leader, b_row, k0);
          else      tma_load_2d_pair(b_dst, &tmap_b, fb_leader, k0, b_row);
          if (half1) {
            if (kBMN) tma_load_2d_pair(b_dst + B_HALF_BYTES, &tmap_b, fb_leader, b_row + 256, k0);
            else      tma_load_2d_pair(b_dst + B_HALF_BYTES, &tmap_b, fb_leader, k0, b_row + 256);
          }
        } else {
          if (kAMN) tma_load_2d(a_dst, &tmap_a, fb, a_row, k0);
          else      tma_load_2d(a_dst, &tmap_a, fb, k0, a_row);
          if (kBMN) {
            tma_load_2d(b_dst, &tmap_b, fb, b_row, k0);
            tma_load_2d(b_dst + BK * 128, &tmap_b, fb, b_row + 128, k0);
          } else {
            tma_load_2d(b_dst, &tmap_b, fb, k0, b_row);
          }
        }
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
      if (!ok) break;
    }
    // Every copy the leader armed completes its stage's full barrier; wait for
    // the last one of each stage so that no copy is still landing when the
    // block exits (immediate in the normal case; the pair's final cluster
    // barrier covers the peer's copies, which count on the same barriers).
    int never = 0;
    if (leader)
      for (int s = 0; s < STAGES; ++s)
        if (armed_mask & (1u << s))
          wait_bar<kCta>(full_bar(s), (armed_parity >> s) & 1u, &never, kSiteDrain, kDrainLimitNs);
  } else if (warp == 1 && lane == 0 && leader) {
    // ------------------------------ MMA issuer ------------------------------
    int stage = 0;
    uint32_t phase = 0;
    int local = 0;
    for (int u = unit; u < p.num_work; u += num_units, ++local) {
      const int t = u / p.splits;
      const int kb0 = (u - t * p.splits) * p.kb_per_split;
      const int kb1 = min(kb0 + p.kb_per_split, p.num_k_blocks);
      const int acc = kDbl ? 0 : (local & 1);
      const uint32_t use = static_cast<uint32_t>(kDbl ? local : (local >> 1));
      int mb_, nb_;
      tile_coords(t, p, mb_, nb_);
      const bool half1 = kDbl && nb_ * BN + 256 < p.N;
      if (!wait_bar<kCta>(tempty_bar(acc), (use & 1u) ^ 1u, abort_flag, kSiteMmaTmemEmpty,
                          p.wait_limit_ns))
        break;
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
      bool ok = true;
      // Double-width tile: the epilogue frees columns 0..255 of the single
      // accumulator before 256..511.  The first `defer` stages of a tile are
      // multiplied into the first half only, while the second half drains;
      // their second-half MMAs follow once it is free, and only then are
      // those stages released (at most STAGES are held, all of which the
      // producer can fill).  The rest run both halves stage by stage.
      int defer = 0;
      if (kDbl) {
        defer = min(kDeferStages, kb1 - kb0);
        int st = stage;
        uint32_t ph = phase;
        for (int i = 0; i < defer; ++i) {
          if (!wait_bar<kCta>(full_bar(st), ph, abort_flag, kSiteMmaFull, p.wait_limit_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = smem_u32(sA + st * A_BYTES);
          const uint32_t b_base = smem_u32(sB + st * B_BYTES);
#pragma unroll
          for (int k = 0; k < BK / UK; ++k)
            mma_f8f6f4_pair(d_tmem, operand_desc<kAMN>(a_base, k), operand_desc<kBMN>(b_base, k),
                            p.idesc, (i != 0 || k != 0) ? 1u : 0u);
          if (++st == STAGES) { st = 0; ph ^= 1u; }
        }
        if (ok && !wait_bar<kCta>(tempty_bar(1), (use & 1u) ^ 1u, abort_flag, kSiteMmaTmemEmpty,
                                  p.wait_limit_ns))
          ok = false;
        if (!ok) break;
        tc_fence_after();
        for (int i = 0; i < defer; ++i) {
          if (half1) {
            const uint32_t a_base = smem_u32(sA + stage * A_BYTES);
            const uint32_t b_base = smem_u32(sB + stage * B_BYTES) + B_HALF_BYTES;
#pragma unroll
            for (int k = 0; k < BK / UK; ++k)
              mma_f8f6f4_pair(d_tmem + 256u, operand_desc<kAMN>(a_base, k),
                              operand_desc<kBMN>(b_base, k), p.idesc, (i != 0 || k != 0) ? 1u : 0u);
          }
          mma_commit_pair_mc(empty_bar(stage), 0x3);   // both halves have read the stage
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      for (int kb = kb0 + defer; kb < kb1; ++kb) {
        if (!wait_bar<kCta>(full_bar(stage), phase, abort_flag, kSiteMmaFull, p.wait_limit_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a_base = smem_u32(sA + stage * A_BYTES);
        const uint32_t b_base = smem_u32(sB + stage * B_BYTES);
#pragma unroll
        for (int k = 0; k < BK / UK; ++k) {
          const uint64_t ad = operand_desc<kAMN>(a_base, k);
          const uint64_t bd = operand_desc<kBMN>(b_base, k);
          const uint32_t accum = (kb != kb0 || k != 0) ? 1u : 0u;
          if (kCta == 2) mma_f8f6f4_pair(d_tmem, ad, bd, p.idesc, accum);
          else           mma_f8f6f4(d_tmem, ad, bd, p.idesc, accum);
        }
        if (kDbl && half1) {
#pragma unroll
          for (int k = 0; k < BK / UK; ++k)
            mma_f8f6f4_pair(d_tmem + 256u, operand_desc<kAMN>(a_base, k),
                            operand_desc<kBMN>(b_base + B_HALF_BYTES, k), p.idesc, 1u);
        }
        // frees the stage (in both CTAs) once these MMAs have read it
        if (kCta == 2) mma_commit_pair_mc(empty_bar(stage), 0x3);
        else           mma_commit(empty_bar(stage));
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
      if (!ok) break;
      // accumulator complete (in both CTAs)
      if (kCta == 2) mma_commit_pair_mc(tfull_bar(acc), 0x3);
      else           mma_commit(tfull_bar(acc));
    }
    // Drain: the commit arrives only after every MMA this thread issued is done.
    if (kCta == 2) mma_commit_pair_mc(drain_bar, 0x1);
    else           mma_commit(drain_bar);
    int never = 0;
    wait_bar<kCta>(drain_bar, 0, &never, kSiteDrain, kDrainLimitNs);
  } else if (warp >= 2) {
    // ------------------------------- epilogue -------------------------------
    const int quarter = warp & 3;                 // TMEM lanes 32*quarter .. +31
    const int row_in_tile = static_cast<int>(rank) * 128 + quarter * 32 + lane;
    const uint32_t out_stage = smem_u32(sOut) + static_cast<uint32_t>(warp - 2) * kStageOutBytesPerWarp;
    const Pow2Scale sc = make_pow2_scale(-(*p.bias_a + *p.bias_b));
    uint32_t dmax = 0;   // kAmax: this thread's max |D| bits (packed bf16 pair or fp32)
    int local = 0;
    for (int u = unit; u < p.num_work; u += num_units, ++local) {
      const int t = u / p.splits;
      const int split = u - t * p.splits;
      const int acc = kDbl ? 0 : (local & 1);
      const uint32_t use = static_cast<uint32_t>(kDbl ? local : (local >> 1));
      int ok = 1;
      if (lane == 0)
        ok = wait_bar<kCta>(tfull_bar(acc), use & 1u, abort_flag, kSiteEpilogueTmemFull,
                            p.wait_limit_ns) ? 1 : 0;
      ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      int mb, nb;
      tile_coords(t, p, mb, nb);
      const int64_t row = static_cast<int64_t>(mb) * C::BM + row_in_tile;
      const bool row_ok = row < p.M;
      // first row of this warp's 32-row box of D
      const int row_box = mb * C::BM + static_cast<int>(rank) * 128 + quarter * 32;
      if (!kDbl && p.splits > 1) {
        // ---- split K: store this range's raw fp32 partial and free the
        // accumulator; splitk_reduce_kernel sums the ranges afterwards
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          const int col0 = nb * BN + c * 32;
          if (col0 >= p.N) break;
          uint32_t r[32];
          tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                                 static_cast<uint32_t>(acc * BN + c * 32), r);
          tmem_ld_wait();
          if (row_ok) {
            float4* dst = reinterpret_cast<float4*>(
                p.ws + (static_cast<int64_t>(split) * p.M + row) * p.N + col0);
#pragma unroll
            for (int j = 0; j < 8; ++j)
              if (col0 + 4 * j < p.N)
                __stcg(dst + j, make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
                                            __uint_as_float(r[4 * j + 2]),
                                            __uint_as_float(r[4 * j + 3])));
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (kCta == 2) mbar_arrive_cluster(mapa_shared(tempty_bar(acc), 0));
          else           mbar_arrive(tempty_bar(acc));
        }
        continue;
      }
      constexpr int kChunks = BN / 32 / kHalves;  // 32-column chunks per half
      static_assert(kChunks % 2 == 0, "chunks are drained in pairs");
#pragma unroll 1
      for (int h = 0; h < kHalves; ++h) {
        // Two 32-column TMEM loads in flight per wait (kChunks is even).
        // The 64 columns are scaled, rounded and written to this warp's
        // staging buffer in the 128-byte-swizzled layout of the D tensor
        // map's box (row = lane; 16-byte piece j of a 128-byte row at
        // j ^ (row % 8)), then stored by one TMA store (BF16: one 64-column
        // box; FP32: two 32-column boxes).  Rows and columns outside D are
        // clipped by the TMA unit.
#pragma unroll 1
        for (int c = h * kChunks; c < (h + 1) * kChunks; c += 2) {
          const int col0 = nb * BN + c * 32;
          if (col0 >= p.N) break;                 // warp-uniform
          const bool two = col0 + 32 < p.N;       // warp-uniform
          const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                                 static_cast<uint32_t>(acc * BN + c * 32);
          uint32_t r0[32], r1[32];
          tmem_ld_32x32b_x32(taddr, r0);
          if (two) tmem_ld_32x32b_x32(taddr + 32u, r1);
          else {
#pragma unroll
            for (int j = 0; j < 32; ++j) r1[j] = 0u;
          }
          // the staging buffer is free once the previous stores have read it
          if (lane == 0) bulk_wait_group_read0();
          __syncwarp();
          tmem_ld_wait();
          stage_out_chunks<kOutF32, kAmax>(out_stage, lane, r0, r1, sc, dmax);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0 && row_box < p.M) {
            tma_store_2d(&tmap_d, out_stage, col0, row_box);
            if (kOutF32 && two) tma_store_2d(&tmap_d, out_stage + 4096u, col0 + 32, row_box);
            bulk_commit_group();
          }
        }
        // these columns are free for the next tile's MMAs
        tc_fence_before();
        __syncwarp();
        const uint32_t tb = tempty_bar(kDbl ? h : acc);
        if (lane == 0) {
          if (kCta == 2) mbar_arrive_cluster(mapa_shared(tb, 0));  // leader's barrier
          else           mbar_arrive(tb);
        }
      }
    }
    // every TMA store of this warp has completed before the block can exit
    if (lane == 0) bulk_wait_group0();
    __syncwarp();
    if (kAmax) {
      // a bf16 is the top half of an fp32: widen the packed pair's max
      uint32_t bits = kOutF32 ? dmax : (max(dmax & 0xFFFFu, dmax >> 16) << 16);
      bits = __reduce_max_sync(0xFFFFFFFFu, bits);
      if (lane == 0 && bits != 0u) atomicMax(p.amax_out, bits);
    }
  }

  // Teardown: every role has left its loop (all waits are bounded).  The pair
  // meets once more so that no CTA exits or frees its tensor memory while the
  // other can still reach its shared memory or tensor memory.
  __syncthreads();
  __syncwarp();
  tc_fence_before();
  if (kCta == 2) cluster_sync();
  tc_fence_after();
  if (warp == 1) {
    if (kCta == 2) tmem_dealloc_pair(tmem_base, TMEM_COLS);
    else           tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// One thread waits on a barrier nothing completes; the bounded wait must give
// up after `limit_ns`, record the self-test site and return.
__global__ void selftest_wait_kernel(uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(smem_u32(&bar), 1);
    fence_mbarrier_init();
    mbar_wait_bounded(smem_u32(&bar), 0, &abort_flag, kSiteSelfTest, limit_ns);
  }
}

// Split-K epilogue: D = (sum over ranges of ws[range]) * 2^-(bias_a+bias_b),
// one rounding to the output type (fp32 sums in range order: the result does
// not depend on which unit finished first).  A separate launch rather than
// "the last unit of a tile adds the partials": that left one CTA per tile
// reading all of the tile's partials with a few loads in flight per thread,
// while here every SM streams them, all ranges' loads of a 4-column group in
// flight together.  N % 4 == 0, so a 4-column group never crosses a row.
constexpr int kReduceThreads = 256;
constexpr int kReduceUnroll = 8;     // ranges whose loads are issued together

template <bool kOutF32, bool kAmax>
__global__ void __launch_bounds__(kReduceThreads)
splitk_reduce_kernel(const float4* __restrict__ ws, int splits, int64_t n4,
                     const int32_t* bias_a, const int32_t* bias_b, void* d, uint32_t* amax_out) {
  const Pow2Scale sc = make_pow2_scale(-(*bias_a + *bias_b));
  uint32_t dmax = 0;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
       i += stride) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s0 = 0; s0 < splits; s0 += kReduceUnroll) {
      float4 v[kReduceUnroll];
#pragma unroll
      for (int u = 0; u < kReduceUnroll; ++u)
        if (s0 + u < splits) v[u] = __ldcs(ws + static_cast<int64_t>(s0 + u) * n4 + i);
#pragma unroll
      for (int u = 0; u < kReduceUnroll; ++u) {
        if (s0 + u < splits) {
          acc.x += v[u].x; acc.y += v[u].y; acc.z += v[u].z; acc.w += v[u].w;
        }
      }
    }
    const float x = apply_pow2(acc.x, sc), y = apply_pow2(acc.y, sc);
    const float z = apply_pow2(acc.z, sc), w = apply_pow2(acc.w, sc);
    if (kOutF32) {
      reinterpret_cast<float4*>(d)[i] = make_float4(x, y, z, w);
      if (kAmax)
        dmax = max(dmax, max(max(__float_as_uint(x) & 0x7FFFFFFFu, __float_as_uint(y) & 0x7FFFFFFFu),
                             max(__float_as_uint(z) & 0x7FFFFFFFu, __float_as_uint(w) & 0x7FFFFFFFu)));
    } else {
      uint2 o;
      o.x = pack_bf16x2(x, y);
      o.y = pack_bf16x2(z, w);
      reinterpret_cast<uint2*>(d)[i] = o;
      if (kAmax) {
        dmax = __vmaxu2(dmax, o.x & 0x7FFF7FFFu);
        dmax = __vmaxu2(dmax, o.y & 0x7FFF7FFFu);
      }
    }
  }
  if (kAmax) {
    uint32_t bits = kOutF32 ? dmax : (max(dmax & 0xFFFFu, dmax >> 16) << 16);
    bits = __reduce_max_sync(0xFFFFFFFFu, bits);
    if ((threadIdx.x & 31) == 0 && bits != 0u) atomicMax(amax_out, bits);
  }
}

// ----------------------------------------------------------------------------
// Host side
// ----------------------------------------------------------------------------
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// Host-side caches below (entry point, SM count, co-resident units, scratch
// address) are filled on first use and may be filled by several host threads
// at once: they are atomics, and every writer stores the same value (or, for
// the pair count, the minimum).
EncodeTiledFn encode_fn() {
  static std::atomic<EncodeTiledFn> fn{nullptr};
  EncodeTiledFn f = fn.load(std::memory_order_acquire);
  if (!f) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess && q == cudaDriverEntryPointSuccess) {
      f = reinterpret_cast<EncodeTiledFn>(p);
      fn.store(f, std::memory_order_release);
    }
  }
  return f;
}

// 2-D row-major uint8 tensor [outer, inner], box [box_outer, box_inner],
// 128-byte swizzle, zero fill out of bounds.
bool encode_2d(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer,
               uint32_t box_inner, uint32_t box_outer) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D row-major D [rows, cols] (BF16 or FP32) for the epilogue's TMA stores:
// box of 128 bytes (64 BF16 / 32 FP32 columns) x 32 rows, 128-byte swizzle.
bool encode_out_2d(CUtensorMap* m, const void* ptr, bool fp32, uint64_t cols, uint64_t rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const uint64_t esz = fp32 ? 4 : 2;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * esz};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(128 / esz), 32};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, fp32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
            const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

std::atomic<int> g_sm_count[64];

int sm_count() {
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  int n = g_sm_count[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    n = n > 0 ? n : 148;
    g_sm_count[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

// Tile order.  Tiles are walked in groups of `group_n` N-blocks, N fastest
// inside a group; the clusters running at one time cover a window of about
// 74 consecutive tiles, i.e. group_n N-blocks x 74/group_n M-blocks, whose
// panels they share in L2.  Measured on the Llama-2-70B projections (each of
// the 12 GEMMs of a step, same clocks): group_n = 16 beat 8, 4 and the orders
// that sweep one whole operand (M fastest or N fastest) by 1-5 %, except
// where both operands are large (K = 28672: both > 128 MB), where 8 won by
// 1-2 %; an evict-last hint on either operand only slowed it down.
// Split-K workspace: fp32 partials [splits][M][N] (256-byte aligned).
size_t splitk_partials_bytes(int splits, int64_t M, int64_t N) {
  return ((static_cast<size_t>(splits) * M * N * sizeof(float)) + 255) & ~size_t(255);
}
size_t splitk_workspace_bytes(int splits, int64_t M, int64_t N) {
  return splitk_partials_bytes(splits, M, N);
}

int pick_group_n(uint64_t a_bytes, uint64_t b_bytes) {
  return (a_bytes > (128ull << 20) && b_bytes > (128ull << 20)) ? 8 : 16;
}

// Split K for problems whose tiles cannot fill the GPU (few rows: the
// weight-streaming GEMMs of decode).  Cut K into ranges so that tiles x splits
// work units still fit in one wave, each range at least 16 k-blocks.
// Measured on the Llama-2-70B projections (T = 1 .. 128, weights streamed,
// splitk_reduce_kernel summing the partials): QKV (K = 8192) 3.1-3.4 ->
// 3.7-3.9 TB/s of weights at T <= 64, down (K = 28672) 2.3-3.3 -> 4.1-5.0 TB/s
// up to T = 128; ranges of >= 24 or >= 48 k-blocks split less and gained less.
// Returns 1 for no split.
int plan_splits(int64_t M, int num_tiles, int num_k_blocks, int* kb_per_split) {
  const int sms = sm_count();
  int splits = 1;
  if (M <= 128 && 2 * num_tiles <= sms) {
    splits = sms / num_tiles;
    splits = splits < num_k_blocks / 16 ? splits : num_k_blocks / 16;
    splits = splits < 16 ? splits : 16;
    if (splits < 1) splits = 1;
  }
  int per = (num_k_blocks + splits - 1) / splits;
  *kb_per_split = per;
  return (num_k_blocks + per - 1) / per;     // no empty range
}

// Split K for CTA-pair tiles (M > 128) when the 256 x 256 tiles cannot fill
// half of the pairs: small outputs with a long K, e.g. the weight gradients
// of small layers (GPT-111M: a 768 x 768 dW over 8192 tokens is 9 tiles for 74
// pairs).  At least 8 k-blocks per range.
int plan_pair_splits(int num_tiles, int num_k_blocks, int num_pairs, int* kb_per_split) {
  int splits = 1;
  if (2 * num_tiles <= num_pairs) {
    splits = num_pairs / num_tiles;
    splits = splits < num_k_blocks / 8 ? splits : num_k_blocks / 8;
    splits = splits < 16 ? splits : 16;
    if (splits < 1) splits = 1;
  }
  int per = (num_k_blocks + splits - 1) / splits;
  *kb_per_split = per;
  return (num_k_blocks + per - 1) / per;
}

// Pairs the pair kernels may run at once on this device: the occupancy query
// made at their first launch, or one pair per two SMs before that.
std::atomic<int> g_pair_units[64];
int pair_units() {
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  const int n = g_pair_units[dev].load(std::memory_order_relaxed);
  return n > 0 ? n : sm_count() / 2;
}
void record_pair_units(int dev, int clusters) {
  int cur = g_pair_units[dev].load(std::memory_order_relaxed);
  while ((cur == 0 || clusters < cur) &&
         !g_pair_units[dev].compare_exchange_weak(cur, clusters, std::memory_order_relaxed)) {
  }
}

template <int kTile, bool kAMN, bool kBMN, bool kOutF32, bool kAmax>
int launch_t(const GemmArgs& g, cudaStream_t s) {
  constexpr int kCta = Cfg<kTile>::CTAS;
  constexpr int BM = Cfg<kTile>::BM;
  constexpr int BN = Cfg<kTile>::BN;
  constexpr size_t kSmem = smem_bytes<kTile>();
  // TMA boxes: 128 x 128 bytes for A (this CTA's rows); for a K-major B, the
  // CTA's B rows (256, 128 or 64) x 128 bytes; for an MN-major B, 128 MN
  // columns x 128 K rows (the single-CTA tile loads two of them).
  const uint32_t b_box_rows = (kBMN || kTile == kTileDouble) ? 128 : Cfg<kTile>::B_ROWS;
  CUtensorMap ta, tb;
  const uint64_t M = g.M, N = g.N, K = g.K;
  const bool ok_a = kAMN ? encode_2d(&ta, g.a, M, K, 128, BK) : encode_2d(&ta, g.a, K, M, BK, 128);
  const bool ok_b = kBMN ? encode_2d(&tb, g.b, N, K, 128, BK)
                         : encode_2d(&tb, g.b, K, N, BK, b_box_rows);
  CUtensorMap td;
  const bool ok_d = encode_out_2d(&td, g.d, g.d_fp32, N, M);
  if (!ok_a || !ok_b || !ok_d) return FP8_ERR_CUDA;

  Params p;
  p.M = static_cast<int>(g.M);
  p.N = static_cast<int>(g.N);
  p.K = static_cast<int>(g.K);
  p.num_m_blocks = (p.M + BM - 1) / BM;
  p.num_n_blocks = (p.N + BN - 1) / BN;
  p.num_k_blocks = (p.K + BK - 1) / BK;
  p.num_tiles = p.num_m_blocks * p.num_n_blocks;
  p.group_n = pick_group_n(M * K, N * K);
  if (kTile == kTileDouble) p.group_n /= 2;   // the same columns in half as many tiles
  p.splits = 1;
  p.kb_per_split = p.num_k_blocks;
  p.ws = nullptr;
  if (g.workspace != nullptr && kTile != kTileDouble) {
    int per = 0;
    const int sp = kCta == 1 ? plan_splits(g.M, p.num_tiles, p.num_k_blocks, &per)
                             : plan_pair_splits(p.num_tiles, p.num_k_blocks, pair_units(), &per);
    if (sp > 1) {
      const size_t need = splitk_workspace_bytes(sp, g.M, g.N);
      if (need > g.workspace_bytes) return FP8_ERR_INVALID_ARGUMENT;
      p.splits = sp;
      p.kb_per_split = per;
      p.ws = static_cast<float*>(g.workspace);
    }
  }
  p.num_work = p.num_tiles * p.splits;
  p.idesc = (1u << 4)                                      // D = fp32
            | (static_cast<uint32_t>(g.a_fmt) << 7)       // A: 0 E4M3, 1 E5M2
            | (static_cast<uint32_t>(g.b_fmt) << 10)      // B: 0 E4M3, 1 E5M2
            | (static_cast<uint32_t>(kAMN) << 15)         // A major: 0 K, 1 MN
            | (static_cast<uint32_t>(kBMN) << 16)         // B major
            | (static_cast<uint32_t>(Cfg<kTile>::MMA_N >> 3) << 17)   // N / 8 of one MMA
            | (static_cast<uint32_t>(BM >> 4) << 24);     // M / 16 (256 for a pair)
  p.bias_a = g.bias_a;
  p.bias_b = g.bias_b;
  p.d = g.d;
  p.amax_out = reinterpret_cast<uint32_t*>(g.d_amax);
  p.wait_limit_ns = kWaitLimitNs;

  static std::atomic<int> max_units[64];   // co-resident CTAs (1-CTA) or clusters (pair), per device
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  auto kern = fp8_gemm_kernel<kTile, kAMN, kBMN, kOutF32, kAmax>;

  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmem;
  cfg.stream = s;
  if (kCta == 2) {
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
  int units_max = max_units[dev].load(std::memory_order_relaxed);
  if (units_max == 0) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kSmem)) != cudaSuccess)
      return FP8_ERR_CUDA;
    int units = sm_count();
    if (kCta == 2) {
      int clusters = 0;
      cfg.gridDim = dim3(2 * (sm_count() / 2), 1, 1);
      if (cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg) != cudaSuccess || clusters < 1) {
        cudaGetLastError();
        clusters = sm_count() / 2;
      }
      units = clusters;
      record_pair_units(dev, clusters);
    }
    units_max = units;
    max_units[dev].store(units, std::memory_order_relaxed);
  }
  const int units = p.num_work < units_max ? p.num_work : units_max;
  cfg.gridDim = dim3(static_cast<unsigned>(units * kCta), 1, 1);
  if (cudaLaunchKernelEx(&cfg, kern, ta, tb, td, p) != cudaSuccess) return FP8_ERR_CUDA;
  if (p.splits > 1) {
    const int64_t n4 = static_cast<int64_t>(g.M) * g.N / 4;
    int64_t blocks = (n4 + kReduceThreads - 1) / kReduceThreads;
    const int64_t cap = static_cast<int64_t>(sm_count()) * 8;
    if (blocks > cap) blocks = cap;
    splitk_reduce_kernel<kOutF32, kAmax><<<static_cast<unsigned>(blocks), kReduceThreads, 0, s>>>(
        reinterpret_cast<const float4*>(p.ws), p.splits, n4, g.bias_a, g.bias_b, g.d,
        p.amax_out);
  }
  return cudaGetLastError() == cudaSuccess ? FP8_OK : FP8_ERR_CUDA;
}

// Few rows (M <= 128): the GEMM streams B and its 128 x 256 tiles may not
// fill the GPU.  With a workspace, such problems split K (plan_splits);
// without one, narrow 128 x 64 tiles are used when 128 x 256 tiles would
// leave more than half of the SMs idle and the narrow ones still fit in one
// wave (measured on the Llama-2-70B projections at T <= 128: a second, mostly
// empty wave of narrow tiles costs more than the idle SMs of the wide ones).
constexpr double kDoubleGain = 1.05;

bool few_wide_tiles(int64_t M, int64_t N) {
  const int64_t wide = ((M + 127) / 128) * ((N + 255) / 256);
  return M <= 128 && 2 * wide <= sm_count();
}

// 256 x 512 pair tiles where they fill the GPU about as evenly as 256 x 256
// ones: the fraction of pair-slots busy over the waves of each tile shape,
// the wide one credited with its lower L2 traffic per FLOP.
bool use_double(const GemmArgs& g) {
  if (g.M <= 128 || g.N <= 256) return false;
  const int64_t pairs = pair_units();
  const int64_t mb = (g.M + 255) / 256;
  const int64_t t256 = mb * ((g.N + 255) / 256);
  const int64_t t512 = mb * ((g.N + 511) / 512);
  const double e256 = static_cast<double>(t256) / (((t256 + pairs - 1) / pairs) * pairs);
  const double e512 = static_cast<double>(t512) / (((t512 + pairs - 1) / pairs) * pairs);
  return e512 * kDoubleGain >= e256;
}

int choose_tile(const GemmArgs& g) {
  if (g.workspace == nullptr && use_double(g)) return kTileDouble;
  if (g.M <= 128) {
    const int64_t narrow = (g.N + 63) / 64;
    if (!g.b_mn_major && g.workspace == nullptr && few_wide_tiles(g.M, g.N) &&
        narrow <= sm_count())
      return kTileNarrow;
    return kTileSingle;
  }
  return kTilePair;
}

template <bool kAMN, bool kBMN, bool kOutF32, bool kAmax = false>
int launch_pick(const GemmArgs& g, cudaStream_t s) {
  switch (choose_tile(g)) {
    case kTileDouble: return launch_t<kTileDouble, kAMN, kBMN, kOutF32, kAmax>(g, s);
    case kTileNarrow: return launch_t<kTileNarrow, kAMN, false, kOutF32, kAmax>(g, s);
    case kTileSingle: return launch_t<kTileSingle, kAMN, kBMN, kOutF32, kAmax>(g, s);
    default:          return launch_t<kTilePair, kAMN, kBMN, kOutF32, kAmax>(g, s);
  }
}

}  // namespace

int launch_gemm(const GemmArgs& g, cudaStream_t s) {
  // limits of the 32-bit tile arithmetic and of the TMA tensor map
  if (g.M > (1LL << 31) - 1 - 256 || g.N > (1LL << 31) - 1 - 256 || g.K > (1LL << 31) - 1 - BK)
    return FP8_ERR_UNSUPPORTED;
  const int key = (g.a_mn_major ? 4 : 0) | (g.b_mn_major ? 2 : 0) | (g.d_fp32 ? 1 : 0);
  if (g.d_amax) {
    // output amax: the passes whose output feeds another quantization (fwd, dgrad)
    switch (key) {
      case 0: return launch_pick<false, false, false, true>(g, s);
      case 1: return launch_pick<false, false, true, true>(g, s);
      case 2: return launch_pick<false, true, false, true>(g, s);
      case 3: return launch_pick<false, true, true, true>(g, s);
      default: return FP8_ERR_UNSUPPORTED;
    }
  }
  switch (key) {
    case 0: return launch_pick<false, false, false>(g, s);
    case 1: return launch_pick<false, false, true>(g, s);
    case 2: return launch_pick<false, true, false>(g, s);
    case 3: return launch_pick<false, true, true>(g, s);
    case 6: return launch_pick<true, true, false>(g, s);
    case 7: return launch_pick<true, true, true>(g, s);
    default: return FP8_ERR_UNSUPPORTED;   // MN-major A with K-major B: no pass uses it
  }
}

void gemm_plan(const GemmArgs& g, GemmPlan* plan) {
  GemmArgs h = g;
  const size_t need = gemm_workspace_bytes(g);
  if (g.workspace == nullptr || need == 0) h.workspace = nullptr;
  const int kind = choose_tile(h);
  int bm = 256, bn = 256, ctas = 2;
  if (kind == kTileDouble) bn = 512;
  if (kind == kTileSingle || kind == kTileNarrow) { bm = 128; ctas = 1; }
  if (kind == kTileNarrow) bn = 64;
  const int nkb = static_cast<int>((g.K + BK - 1) / BK);
  const int tiles = static_cast<int>(((g.M + bm - 1) / bm) * ((g.N + bn - 1) / bn));
  int splits = 1, per = 0;
  if (h.workspace != nullptr)
    splits = ctas == 1 ? plan_splits(g.M, tiles, nkb, &per)
                       : plan_pair_splits(tiles, nkb, pair_units(), &per);
  plan->tile_m = bm;
  plan->tile_n = bn;
  plan->ctas_per_tile = ctas;
  plan->k_splits = splits;
}

size_t gemm_workspace_bytes(const GemmArgs& g) {
  const int nkb = static_cast<int>((g.K + BK - 1) / BK);
  int per = 0;
  if (g.M > 128) {
    const int tiles = static_cast<int>(((g.M + 255) / 256) * ((g.N + 255) / 256));
    const int sp = plan_pair_splits(tiles, nkb, pair_units(), &per);
    return sp > 1 ? splitk_workspace_bytes(sp, g.M, g.N) : 0;
  }
  if (!few_wide_tiles(g.M, g.N)) return 0;
  const int tiles = static_cast<int>(((g.M + 127) / 128) * ((g.N + 255) / 256));
  const int sp = plan_splits(g.M, tiles, nkb, &per);
  return sp > 1 ? splitk_workspace_bytes(sp, g.M, g.N) : 0;
}

// ----------------------------------------------------------------------------
// Forward GEMM that allocates nothing (fp8_linear_fwd_noalloc).
//
// Some callers cannot allocate device memory at the point where they run a
// forward: code inside a region that must not call cudaMalloc (an allocator
// that is locked, a pre-sized memory pool that may not grow, a serving loop
// that forbids allocation on its hot path), or plain C callers with no device
// allocator of their own.  For them the split-K scratch lives in the array
// below, which every GPU that loads this library holds until the process
// exits.  Host code may not use the array's name as a device address: it is
// looked up once per device with cudaGetSymbolAddress, with that device
// current, on the first call made there.
// ----------------------------------------------------------------------------
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;     // 16 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

int launch_gemm_noalloc(GemmArgs g, cudaStream_t s) {
  static std::atomic<void*> scratch_addr[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return FP8_ERR_CUDA;
  void* scratch = scratch_addr[dev].load(std::memory_order_relaxed);
  if (scratch == nullptr) {
    if (cudaGetSymbolAddress(&scratch, g_noalloc_scratch) != cudaSuccess || scratch == nullptr)
      return FP8_ERR_CUDA;
    scratch_addr[dev].store(scratch, std::memory_order_relaxed);
  }
  size_t need = gemm_workspace_bytes(g);
  if (need > kNoAllocScratchBytes) {
    if (g.M <= 64) return FP8_ERR_UNSUPPORTED;
    need = 0;     // more rows: split only when the partials fit, else run unsplit
  }
  if (need > 0) {
    // every fp32 partial is written by the GEMM before the reduction reads it
    g.workspace = scratch;
    g.workspace_bytes = kNoAllocScratchBytes;
  }
  return launch_gemm(g, s);
}

cudaError_t launch_selftest_wait(uint64_t timeout_ns) {
  selftest_wait_kernel<<<1, 32>>>(timeout_ns);
  return cudaGetLastError();
}

int device_error_site(bool clear) {
  int v = 0;
  if (cudaDeviceSynchronize() != cudaSuccess) return -1;
  if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof(int)) != cudaSuccess) return -1;
  if (clear && v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int)) != cudaSuccess) return -1;
  }
  return v;
}

}  // namespace fp8amax
