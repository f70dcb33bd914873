// Persistent ternary x int8 GEMM on the 5th-generation tensor cores
// (tcgen05, kind::i8) with a wide weight tile, for the prefill regime.
//
// BitNet v2 architecture walkthrough, section 3.4 "H-BitLinear: The Composite
// Layer", Eq. 9: acc[m, n] = sum_k c[m, k] * t[n, k]; Y = acc * s[m] * alpha.
//
// Why this tile: with 128 weight rows per tile every code byte is fetched from
// L2 once per 128 rows, and the code feed (about 72 bytes per SM clock at the
// int8 MMA rate) exceeds what L2 delivers to an SM. Here one CTA owns 256
// weight rows x 128 tokens: each 128-token code tile in shared memory feeds
// two M=128 MMAs (rows 0-127 and 128-255), which halves the code bytes per
// multiply-add; the weights, 2 bits each, stay cheap to fetch twice as often.
//
// One CTA per SM walks a static list of tiles (row tile fastest). Warp roles:
//   warp 0     TMA producer: per 256-k stage, the codes tile (128 tokens x
//              256 k as two 128-byte-wide 128B-swizzled boxes, 32 KB) and the
//              packed weight tile (256 rows x 64 bytes, 64B-swizzled, 16 KB)
//              into a 4-stage ring.
//   warp 1     MMA issuer: per stage and 32-k step, two tcgen05.mma.kind::i8
//              (M=128, N=128, K=32), A (unpacked weights) from TMEM, B (codes)
//              from shared memory, int32 accumulators in TMEM columns
//              [0,128) and [128,256); tcgen05.commit frees the shared-memory
//              stage and the TMEM A slot.
//   warps 2-9  converters: warp w owns weight-row half (w-2)/4 and TMEM lane
//              quadrant w%4; each thread unpacks its row's 64 packed bytes
//              into 256 unsigned bytes (u = t + 1) and writes them with
//              tcgen05.st into the stage's A slot (two slots of 128 columns,
//              columns [256,512)). The same warps run the epilogue of the
//              previous tile once the first two stages of the next tile are
//              converted: tcgen05.ld of their 128 accumulator columns, release
//              of the accumulator, then D - sum(c), times s[m] * alpha, bf16.
// Every mbarrier wait is bounded; on timeout the CTA sets the device error
// word, every role stops, the CTA waits (bounded) for its own copies and MMAs,
// frees its tensor memory and exits.
#pragma once
#include <cuda.h>
#include "hbl_common.cuh"
#include "gemm_tc.cuh"

namespace hbl {
namespace tcw {

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

constexpr int kHalf = 128;                       // weight rows per MMA (M)
constexpr int kRows = 2 * kHalf;                 // weight rows per tile
constexpr int kToks = 128;                       // tokens per tile (MMA N)
constexpr int kStages = 4;                       // shared-memory ring
constexpr int kASlots = 2;                       // TMEM A ring
constexpr int kBBytes = kToks * kKBlock;         // 32 KB of codes per stage
constexpr int kABytes = kRows * (kKBlock / 4);   // 16 KB of packed weights per stage
constexpr int kStageTx = kBBytes + kABytes;
constexpr int kAColsHalf = kKBlock / 4;          // 64 TMEM columns per half-tile and stage
constexpr int kAColsSlot = 2 * kAColsHalf;       // 128 per slot
constexpr int kACol0 = 2 * kToks;                // A slots after the two accumulators
constexpr int kTmemCols = 512;
constexpr int kConvWarps = 8;
constexpr int kThreads = 32 * (2 + kConvWarps);
constexpr long long kSpinLimit = tc::kSpinLimit;
static_assert(kACol0 + kASlots * kAColsSlot <= kTmemCols, "TMEM columns");

struct __align__(8) Smem {
  uint8_t b[kStages][kBBytes];     // 1024-byte aligned (swizzle atoms)
  uint8_t a[kStages][kABytes];
  uint64_t full[kStages];          // TMA bytes landed
  uint64_t s_empty[kStages];       // MMAs of the stage done (shared memory reusable)
  uint64_t aready[kASlots];        // converters wrote the A slot
  uint64_t a_empty[kASlots];       // MMAs reading the A slot done
  uint64_t acc_full;               // tile's MMAs done
  uint64_t acc_empty;              // epilogue has read the accumulators
  uint64_t done;                   // every MMA of the CTA done
  uint32_t tmem_base;
  int abort;
};
constexpr size_t kSmemBytes = sizeof(Smem) + 1024;

// Instruction descriptor: D s32, A u8, B s8, both K-major, M = 128, N = 128.
constexpr uint32_t kIdesc = (2u << 4) | (0u << 7) | (1u << 10) | ((uint32_t)(kToks >> 3) << 17) |
                            ((uint32_t)(kHalf >> 4) << 24);

HBL_DEVINL void tile_coords(int t, int n_tiles, int* n0, int* m0) {
  *n0 = (t % n_tiles) * kRows;
  *m0 = (t / n_tiles) * kToks;
}

// Unpack one weight row's 64 packed bytes (one 256-k block, 64B-swizzled in
// shared memory) and write them into 64 TMEM columns of this thread's lane.
HBL_DEVINL void convert_row(const uint8_t* tile, int row, uint32_t taddr) {
  const uint4* src = reinterpret_cast<const uint4*>(tile + row * (kKBlock / 4));
  uint32_t wv[16];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint4 v = src[q ^ ((row >> 1) & 3)];
    wv[4 * q] = v.x; wv[4 * q + 1] = v.y; wv[4 * q + 2] = v.z; wv[4 * q + 3] = v.w;
  }
  // word (tig, w) register j holds k = 64w + 32(j>>1) + 8tig + 4(j&1) + i, i.e.
  // TMEM column 16w + 8(j>>1) + 2tig + (j&1) of the slot
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
  HBL_TMEM_ST32(taddr, c0);
  HBL_TMEM_ST32(taddr + 32, c1);
}

template <bool OUT_BF16>
__global__ void __launch_bounds__(kThreads, 1)
gemm_tcw_kernel(const __grid_constant__ CUtensorMap map_codes, const __grid_constant__ CUtensorMap map_w, int M,
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
      mbar_init(&S.s_empty[s], 1);
    }
    for (int s = 0; s < kASlots; ++s) {
      mbar_init(&S.aready[s], kConvWarps);
      mbar_init(&S.a_empty[s], 1);
    }
    mbar_init(&S.acc_full, 1);
    mbar_init(&S.acc_empty, kConvWarps);
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
  // Programmatic dependent launch: everything above overlapped the previous
  // kernel's tail; the codes, code sums and scales it writes are read below.
  asm volatile("griddepcontrol.wait;\n" ::: "memory");

  if (warp == 0) {
    if (lane == 0) {
      int g = 0, issued = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
        int n0, m0;
        tile_coords(t, n_tiles, &n0, &m0);
        for (int kb = 0; kb < nblk; ++kb, ++g) {
          const int s = g % kStages;
          if (g >= kStages && !mbar_wait(&S.s_empty[s], ((uint32_t)(g / kStages) & 1u) ^ 1u, abort)) {
            ok = false;
            break;
          }
          mbar_expect_tx(&S.full[s], kStageTx);
          tma_load_2d(&S.b[s][0], &map_codes, &S.full[s], kb * kKBlock, m0);
          tma_load_2d(&S.b[s][kBBytes / 2], &map_codes, &S.full[s], kb * kKBlock + 128, m0);
          tma_load_2d(&S.a[s][0], &map_w, &S.full[s], kb * (kKBlock / 4), n0);
          issued = g + 1;
        }
      }
      // bounded drain: the last loads issued must land before the CTA may exit
      for (int q = (issued > kStages ? issued - kStages : 0); q < issued; ++q) {
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
        if (i >= 1 && !mbar_wait(&S.acc_empty, (uint32_t)(i - 1) & 1u, abort)) break;
        tc_fence_after();
        for (int kb = 0; kb < nblk; ++kb, ++g) {
          const int s = g % kStages, as = g % kASlots;
          ok = mbar_wait(&S.full[s], (uint32_t)(g / kStages) & 1u, abort) &&
               mbar_wait(&S.aready[as], (uint32_t)(g / kASlots) & 1u, abort);
          if (!ok) break;
          tc_fence_after();
          const uint32_t bbase = su32(&S.b[s][0]);
          const uint32_t abase = tmem + (uint32_t)(kACol0 + as * kAColsSlot);
#pragma unroll
          for (int j = 0; j < kKBlock / 32; ++j) {
            const uint64_t bdesc = smem_desc_sw128(bbase + (uint32_t)((j >> 2) * (kBBytes / 2) + (j & 3) * 32));
            const uint32_t acc = (kb > 0 || j > 0) ? 1u : 0u;
            mma_i8_ts(tmem, abase + (uint32_t)(8 * j), bdesc, kIdesc, acc);
            mma_i8_ts(tmem + (uint32_t)kToks, abase + (uint32_t)(kAColsHalf + 8 * j), bdesc, kIdesc, acc);
          }
          tc_commit(&S.s_empty[s]);
          tc_commit(&S.a_empty[as]);
        }
        if (!ok) break;
        tc_commit(&S.acc_full);
      }
      tc_commit(&S.done);   // arrives once every MMA issued above has completed
    }
  } else {
    // converters + epilogue: half h of the tile's weight rows, TMEM lane quadrant warp % 4
    const int quad = warp & 3;
    const int h = (warp - 2) >> 2;
    const int row = kHalf * h + 32 * quad + lane;      // row within the tile
    const uint32_t lane_addr = (uint32_t)(32 * quad) << 16;
    const float a = OUT_BF16 ? __ldg(alpha) : 0.f;
    const int conv_before_epi = nblk < 2 ? nblk : 2;   // next-tile stages converted before the epilogue
    int g = 0, i = 0, prev_t = -1;
    bool ok = true;

    // Epilogue of tile pt (ordinal pi): read the accumulator columns of this
    // warp's half, release them, then dequantise and store.
    auto epilogue = [&](int pt, int pi) -> bool {
      if (!__all_sync(0xffffffffu, mbar_wait(&S.acc_full, (uint32_t)pi & 1u, abort))) return false;
      tc_fence_after();
      uint32_t acc[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) HBL_TMEM_LD32(tmem + lane_addr + (uint32_t)(kToks * h + 32 * c), acc[c]);
      tc_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.acc_empty);
      int n0, m0;
      tile_coords(pt, n_tiles, &n0, &m0);
      const int n = n0 + row;
      if (n < N) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int m = m0 + 32 * c + j;
            if (m < M) {
              const int v = (int)acc[c][j] - __ldg(csum + m);
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
      return true;
    };

    for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x, ++i) {
      for (int kb = 0; kb < nblk; ++kb, ++g) {
        const int s = g % kStages, as = g % kASlots;
        bool w = mbar_wait(&S.full[s], (uint32_t)(g / kStages) & 1u, abort);
        if (w && g >= kASlots) w = mbar_wait(&S.a_empty[as], ((uint32_t)(g / kASlots) & 1u) ^ 1u, abort);
        if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
        tc_fence_after();
        convert_row(&S.a[s][0], row, tmem + lane_addr + (uint32_t)(kACol0 + as * kAColsSlot + kAColsHalf * h));
        tc_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.aready[as]);
        if (kb == conv_before_epi - 1 && prev_t >= 0) {
          if (!epilogue(prev_t, i - 1)) { ok = false; break; }
        }
      }
      prev_t = t;
    }
    if (ok && prev_t >= 0) epilogue(prev_t, i - 1);
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

}  // namespace tcw
}  // namespace hbl
