// Persistent ternary x int8 GEMM on the 5th-generation tensor cores
// (tcgen05, kind::i8), for the prefill regime, with the dequant epilogue
// fused and overlapped with the next tile's MMAs.
//
// BitNet v2 architecture walkthrough, section 3.4 "H-BitLinear: The Composite
// Layer", Eq. 9: acc[m, n] = sum_k c[m, k] * t[n, k]; Y = acc * s[m] * alpha.
//
// One CTA per SM walks a static list of 128 (output rows) x 128 (tokens)
// tiles. Warp roles:
//   warp 0     TMA producer: per 256-k stage, the codes tile (128 tokens x
//              256 k as two 128-byte-wide 128B-swizzled boxes) and the packed
//              weight tile (128 rows x 64 bytes), into a 4-stage ring.
//   warps 2-5  converters: one weight row per thread (one TMEM lane); unpack
//              64 packed bytes to 256 unsigned bytes (u = t + 1) in registers
//              and tcgen05.st them into the stage's 64 TMEM columns, which are
//              the MMA's A operand.
//   warp 1     MMA issuer: 8 x tcgen05.mma.kind::i8 (M=128, N=128, K=32) per
//              stage into one of two TMEM accumulators (columns [0,128) and
//              [128,256)), tcgen05.commit to free the stage / hand over the
//              finished accumulator.
//   warps 6-9  epilogue: tcgen05.ld the finished accumulator, release it at
//              once (the MMA warp starts the next tile into it two tiles on),
//              then subtract the code sums, scale by s[m] * alpha and store.
// TMEM: 512 columns = 2 accumulators x 128 + 4 A stages x 64.
// Every mbarrier wait is bounded; on timeout the CTA sets the device error
// word, every role stops, the CTA waits (bounded) for its own outstanding copies
// and MMAs, frees its tensor memory and exits.
#pragma once
#include <cuda.h>
#include "hbl_common.cuh"
#include "gemm_tc.cuh"

namespace hbl {
namespace tc2 {

using tc::mbar_init;
using tc::mbar_expect_tx;
using tc::mbar_arrive;
using tc::mbar_try_wait;
using tc::mbar_wait;
using tc::tma_load_2d;
using tc::tmem_alloc;
using tc::tmem_relinquish;
using tc::tmem_dealloc;
using tc::tc_fence_before;
using tc::tc_fence_after;
using tc::tc_commit;
using tc::tc_wait_st;
using tc::tc_wait_ld;
using tc::mma_i8_ts;
using tc::smem_desc_sw128;
using tc::su32;

constexpr int kRows = 128;                       // weight rows per tile (MMA M)
constexpr int kToks = 128;                       // tokens per tile (MMA N)
constexpr int kStages = 4;
constexpr int kBBytes = kToks * kKBlock;         // 32 KB of codes per stage
constexpr int kABytes = kRows * (kKBlock / 4);   // 8 KB of packed weights per stage
constexpr int kStageTx = kBBytes + kABytes;
constexpr int kACol0 = 2 * kToks;                // A stages start after the two accumulators
constexpr int kACols = kKBlock / 4;              // 64 columns per A stage
constexpr int kTmemCols = 512;
constexpr int kThreads = 320;
constexpr long long kSpinLimit = tc::kSpinLimit;

struct __align__(8) Smem {
  uint8_t b[kStages][kBBytes];     // 1024-byte aligned
  uint8_t a[kStages][kABytes];
  uint64_t full[kStages];
  uint64_t aready[kStages];
  uint64_t empty[kStages];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t done;
  uint32_t tmem_base;
  int abort;
};
constexpr size_t kSmemBytes = sizeof(Smem) + 1024;

constexpr uint32_t kIdesc = (2u << 4) | (0u << 7) | (1u << 10) | ((uint32_t)(kToks >> 3) << 17) |
                            ((uint32_t)(kRows >> 4) << 24);

HBL_DEVINL void tile_coords(int t, int n_tiles, int* n0, int* m0) {
  *n0 = (t % n_tiles) * kRows;
  *m0 = (t / n_tiles) * kToks;
}

template <bool OUT_BF16>
__global__ void __launch_bounds__(kThreads, 1)
gemm_tc2_kernel(const __grid_constant__ CUtensorMap map_codes, const __grid_constant__ CUtensorMap map_w, int M,
                int K, int N, const int32_t* __restrict__ csum, const float* __restrict__ scales,
                const float* __restrict__ alpha, uint16_t* __restrict__ Y, int32_t* __restrict__ acc_out) {
  extern __shared__ uint8_t smem_raw[];
  Smem& S = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tiles = (N + kRows - 1) / kRows;
  const int m_tiles = (M + kToks - 1) / kToks;
  const int tiles = n_tiles * m_tiles;
  const int nblk = K / kKBlock;
  volatile int* abort = &S.abort;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&S.full[s], 1);
      mbar_init(&S.aready[s], 128);
      mbar_init(&S.empty[s], 1);
    }
    for (int d = 0; d < 2; ++d) {
      mbar_init(&S.acc_full[d], 1);
      mbar_init(&S.acc_empty[d], 128);
    }
    mbar_init(&S.done, 1);
    S.abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    asm volatile("prefetch.tensormap [%0];\n" ::"l"(reinterpret_cast<uint64_t>(&map_codes)) : "memory");
    asm volatile("prefetch.tensormap [%0];\n" ::"l"(reinterpret_cast<uint64_t>(&map_w)) : "memory");
  }
  if (warp == 1) {
    tmem_alloc(&S.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S.tmem_base;
  int issued_stages = 0;   // producer: stages issued (for the bounded drain)

  if (warp == 0) {
    if (lane == 0) {
      int g = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
        int n0, m0;
        tile_coords(t, n_tiles, &n0, &m0);
        for (int kb = 0; kb < nblk; ++kb, ++g) {
          const int s = g % kStages;
          const uint32_t ph = (uint32_t)(g / kStages) & 1u;
          if (g >= kStages && !mbar_wait(&S.empty[s], ph ^ 1u, abort)) { ok = false; break; }
          mbar_expect_tx(&S.full[s], kStageTx);
          tma_load_2d(&S.b[s][0], &map_codes, &S.full[s], kb * kKBlock, m0);
          tma_load_2d(&S.b[s][kBBytes / 2], &map_codes, &S.full[s], kb * kKBlock + 128, m0);
          tma_load_2d(&S.a[s][0], &map_w, &S.full[s], kb * (kKBlock / 4), n0);
          issued_stages = g + 1;
        }
      }
      // bounded drain: the last loads issued must land before the CTA may exit
      for (int q = (issued_stages > kStages ? issued_stages - kStages : 0); q < issued_stages; ++q) {
        const long long t0 = clock64();
        while (!mbar_try_wait(&S.full[q % kStages], (uint32_t)(q / kStages) & 1u) && clock64() - t0 < kSpinLimit) {
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int g = 0, i = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x, ++i) {
        const int d = i & 1, u = i >> 1;
        if (u >= 1 && !mbar_wait(&S.acc_empty[d], (uint32_t)(u - 1) & 1u, abort)) break;
        tc_fence_after();
        const uint32_t dcol = tmem + (uint32_t)(d * kToks);
        for (int kb = 0; kb < nblk; ++kb, ++g) {
          const int s = g % kStages;
          const uint32_t ph = (uint32_t)(g / kStages) & 1u;
          ok = mbar_wait(&S.full[s], ph, abort) && mbar_wait(&S.aready[s], ph, abort);
          if (!ok) break;
          tc_fence_after();
          const uint32_t bbase = su32(&S.b[s][0]);
#pragma unroll
          for (int j = 0; j < kKBlock / 32; ++j) {
            const uint32_t a_addr = tmem + (uint32_t)(kACol0 + s * kACols + 8 * j);
            const uint64_t bdesc = smem_desc_sw128(bbase + (uint32_t)((j >> 2) * (kBBytes / 2) + (j & 3) * 32));
            mma_i8_ts(dcol, a_addr, bdesc, kIdesc, (kb > 0 || j > 0) ? 1u : 0u);
          }
          tc_commit(&S.empty[s]);
        }
        if (!ok) break;
        tc_commit(&S.acc_full[d]);
      }
      tc_commit(&S.done);   // arrives once every MMA issued above has completed
    }
  } else if (warp <= 5) {
    // converters: TMEM lane quadrant warp % 4
    const int quad = warp & 3;
    const int row = 32 * quad + lane;
    const uint32_t lane_addr = (uint32_t)(32 * quad) << 16;
    int g = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
      for (int kb = 0; kb < nblk; ++kb, ++g) {
        const int s = g % kStages;
        const uint32_t ph = (uint32_t)(g / kStages) & 1u;
        if (!__all_sync(0xffffffffu, mbar_wait(&S.full[s], ph, abort))) { ok = false; break; }
        // 64B-swizzled tile: chunk q of the row sits at q ^ ((row >> 1) & 3)
        const uint4* src = reinterpret_cast<const uint4*>(&S.a[s][row * (kKBlock / 4)]);
        uint32_t wv[16];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint4 v = src[q ^ ((row >> 1) & 3)];
          wv[4 * q] = v.x; wv[4 * q + 1] = v.y; wv[4 * q + 2] = v.z; wv[4 * q + 3] = v.w;
        }
        uint32_t c0[32], c1[32];
#pragma unroll
        for (int tig = 0; tig < 4; ++tig)
#pragma unroll
          for (int w = 0; w < 4; ++w)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int col = 16 * w + 8 * (j >> 1) + 2 * tig + (j & 1);
              const uint32_t v = unpack_u8x4(wv[4 * tig + w], j);
              if (col < 32) c0[col] = v; else c1[col - 32] = v;
            }
        const uint32_t abase = tmem + lane_addr + (uint32_t)(kACol0 + s * kACols);
        HBL_TMEM_ST32(abase, c0);
        HBL_TMEM_ST32(abase + 32, c1);
        tc_wait_st();
        tc_fence_before();
        mbar_arrive(&S.aready[s]);
      }
    }
  } else {
    // epilogue warps 6..9: TMEM lane quadrant warp % 4
    const int quad = warp & 3;
    const uint32_t lane_addr = (uint32_t)(32 * quad) << 16;
    const float a = OUT_BF16 ? __ldg(alpha) : 0.f;
    int i = 0;
    for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++i) {
      const int d = i & 1, u = i >> 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&S.acc_full[d], (uint32_t)u & 1u, abort))) break;
      tc_fence_after();
      int n0, m0;
      tile_coords(t, n_tiles, &n0, &m0);
      const int n = n0 + 32 * quad + lane;
#pragma unroll 1
      for (int c = 0; c < kToks / 32; ++c) {
        uint32_t acc[32];
        HBL_TMEM_LD32(tmem + lane_addr + (uint32_t)(d * kToks + 32 * c), acc);
        tc_wait_ld();
        if (c == kToks / 32 - 1) {
          tc_fence_before();
          mbar_arrive(&S.acc_empty[d]);   // the accumulator may be reused now
        }
        if (n < N) {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int m = m0 + 32 * c + j;
            if (m < M) {
              const int v = (int)acc[j] - __ldg(csum + m);
              if constexpr (OUT_BF16) {
                const float y = __fmul_rn(__fmul_rn((float)v, __ldg(scales + m)), a);
                Y[(size_t)m * N + n] = float_to_bf16_bits(y);
              } else {
                acc_out[(size_t)m * N + n] = v;
              }
            }
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    // every MMA this CTA issued has completed once `done` flips (bounded wait)
    if (lane == 0) {
      const long long t0 = clock64();
      while (!mbar_try_wait(&S.done, 0) && clock64() - t0 < kSpinLimit) {
      }
    }
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace tc2
}  // namespace hbl
