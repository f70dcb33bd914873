// Ternary x int8 GEMM on the 5th-generation tensor cores with the MMA spread
// over a pair of SMs (tcgen05.mma.cta_group::2, kind::i8), for the prefill
// regime.
//
// BitNet v2 architecture walkthrough, section 3.4 "H-BitLinear: The Composite
// Layer", Eq. 9: acc[m, n] = sum_k c[m, k] * t[n, k], then the dequant
// acc * s[m] * alpha (Eq. 1, Eq. 7 / Eq. 8).
//
// Why a pair: one SM computing a 128 x 256 tile must pull 64 KB of codes and
// 8 KB of packed weights into shared memory per 1024 tensor-pipe cycles, more
// than it is fed at. A cluster of two CTAs on two SMs computes one 256 (output
// rows) x 256 (tokens) tile with M=256 MMAs: CTA r holds weight rows
// [128r, 128r+128) of the tile (unpacked into its own tensor memory) and the
// codes of tokens [128r, 128r+128) (in its own shared memory); each SM's
// tensor core reads the other half of the codes from the peer. Each SM thus
// loads 32 KB of codes and 8 KB of weights per 1024 cycles.
//
// Roles in each CTA of the pair (rank 0 is the leader, which issues the MMAs):
//   warp 0 (one lane): TMA producer. Per 256-k stage: its token half of the
//     codes (two 128-byte-wide 128B-swizzled boxes, 32 KB), completing on the
//     LEADER's code barrier, and its 128 weight rows (64B-swizzled, 8 KB),
//     completing on its own weight barrier.
//   warps 2..5: converters. Each thread owns one weight row (one TMEM lane),
//     unpacks its 64 packed bytes into 256 unsigned bytes (u = t + 1) and
//     writes them into the stage's 64 TMEM columns; one arrive per warp on the
//     leader's A-ready barrier (remote for the second CTA).
//   warp 1 of the leader (one lane): per stage, eight
//     tcgen05.mma.cta_group::2.kind::i8 (M=256, N=256, K=32), A from both
//     tensor memories, B from both shared memories, int32 accumulators in
//     TMEM columns [0, 256) of both SMs; commits free the stage in both CTAs.
//   warps 2..5 again: epilogue on each SM's own 128 rows.
// Every mbarrier wait is bounded; on timeout the CTA sets the device error
// word and stops issuing. Both CTAs always reach the final cluster barrier,
// so neither frees its shared or tensor memory while the pair's MMAs can
// still read it.
#pragma once
#include <cuda.h>
#include "hbl_common.cuh"
#include "gemm_tc.cuh"

namespace hbl {
namespace tcp {

using tc::mbar_init;
using tc::mbar_expect_tx;
using tc::mbar_arrive;
using tc::mbar_try_wait;
using tc::mbar_wait;
using tc::tma_load_2d;
using tc::tc_fence_before;
using tc::tc_fence_after;
using tc::tc_wait_st;
using tc::tc_wait_ld;
using tc::smem_desc_sw128;
using tc::su32;

constexpr int kRows = 128;                       // weight rows per CTA (the pair: MMA M = 256)
constexpr int kToks = 256;                       // tokens per tile (MMA N); 128 per CTA
constexpr int kStages = 4;
constexpr int kCBytes = (kToks / 2) * kKBlock;   // 32 KB: this CTA's token half, 256 k
constexpr int kABytes = kRows * (kKBlock / 4);   // 8 KB packed weights per stage
constexpr int kACols = kKBlock / 4;              // 64 TMEM columns of A per stage
constexpr int kDCols = kToks;                    // accumulator columns
constexpr int kTmemCols = 512;
constexpr int kThreads = 192;
constexpr long long kSpinLimit = tc::kSpinLimit;
static_assert(kDCols + kStages * kACols <= kTmemCols, "TMEM columns");

struct __align__(8) Smem {
  uint8_t b[kStages][kCBytes];     // 1024-byte aligned (swizzle atoms); same offset in both CTAs
  uint8_t a[kStages][kABytes];
  uint64_t c_full[kStages];        // leader: both token halves of the codes landed
  uint64_t w_full[kStages];        // own packed weights landed
  uint64_t aready[kStages];        // leader: both CTAs' converters wrote the A stage
  uint64_t empty[kStages];         // the pair's MMAs on the stage are done
  uint64_t done;                   // every MMA of the pair is done
  uint32_t tmem_base;
  int abort;
};
constexpr size_t kSmemBytes = sizeof(Smem) + 1024;

// Instruction descriptor: D s32, A u8, B s8, both K-major, M = 256, N = 256.
constexpr uint32_t kIdesc = (2u << 4) | (0u << 7) | (1u << 10) | ((uint32_t)(kToks >> 3) << 17) |
                            ((uint32_t)((2 * kRows) >> 4) << 24);

HBL_DEVINL uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;\n" : "=r"(r));
  return r;
}
// Shared::cluster address of the same shared variable in CTA `rank` of the cluster.
HBL_DEVINL uint32_t map_to(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;\n" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
HBL_DEVINL void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;\n" ::: "memory");
}
HBL_DEVINL void arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];\n" ::"r"(cluster_addr) : "memory");
}
// TMA tile load into this CTA's shared memory whose completion is counted on
// a barrier of either CTA of the pair (cluster address).
HBL_DEVINL void tma_load_2d_pair(void* dst, const CUtensorMap* map, uint32_t bar_cluster, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];\n" ::"r"(
          su32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(x), "r"(y)
      : "memory");
}
HBL_DEVINL void tmem_alloc2(uint32_t* slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(su32(slot)), "r"(ncols)
               : "memory");
}
HBL_DEVINL void tmem_relinquish2() { asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;\n" ::); }
HBL_DEVINL void tmem_dealloc2(uint32_t addr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;\n" ::"r"(addr), "r"(ncols) : "memory");
}
// D[tmem, both SMs] (+)= A[tmem, both SMs] * B[smem desc, both SMs], kind::i8, M = 256.
HBL_DEVINL void mma2_i8(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc, uint32_t accum) {
  asm volatile(
      "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
      "tcgen05.mma.cta_group::2.kind::i8 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accum)
      : "memory");
}
// Arrive on a barrier (of either CTA of the pair) once every MMA this thread issued has completed.
HBL_DEVINL void commit2(uint32_t bar_cluster) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(bar_cluster)
               : "memory");
}

// Tile of a pair: CTAs 2p and 2p+1 form pair p; row tiles of 256 are fastest.
HBL_DEVINL void pair_tile(int p, int n_tiles, int* n0, int* m0) {
  *n0 = (p % n_tiles) * (2 * kRows);
  *m0 = (p / n_tiles) * kToks;
}

// OUT_BF16: Y = bf16((D - csum) * s * alpha); else acc (int32) = D - csum.
// map_codes loads [128 tokens][128 B] boxes, map_w [128 rows][64 B] boxes.
template <bool OUT_BF16>
__global__ void __launch_bounds__(kThreads, 1)
gemm_tc2sm_kernel(const __grid_constant__ CUtensorMap map_codes, const __grid_constant__ CUtensorMap map_w, int M,
                  int K, int N, const int32_t* __restrict__ csum, const float* __restrict__ scales,
                  const float* __restrict__ alpha, uint16_t* __restrict__ Y, int32_t* __restrict__ acc_out) {
  extern __shared__ uint8_t smem_raw[];
  Smem& S = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  int n0, m0;
  pair_tile((int)(blockIdx.x >> 1), (N + 2 * kRows - 1) / (2 * kRows), &n0, &m0);
  n0 += (int)rank * kRows;                 // this CTA's weight rows
  const int mt0 = m0 + (int)rank * (kToks / 2);   // this CTA's token half of the codes
  const int nblk = K / kKBlock;
  volatile int* abort = &S.abort;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&S.c_full[s], 1);
      mbar_init(&S.w_full[s], 1);
      mbar_init(&S.aready[s], 8);      // 4 converter warps in each CTA
      mbar_init(&S.empty[s], 1);
    }
    mbar_init(&S.done, 1);
    S.abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    asm volatile("prefetch.tensormap [%0];\n" ::"l"(reinterpret_cast<uint64_t>(&map_codes)) : "memory");
    asm volatile("prefetch.tensormap [%0];\n" ::"l"(reinterpret_cast<uint64_t>(&map_w)) : "memory");
  }
  if (warp == 1) {
    tmem_alloc2(&S.tmem_base, kTmemCols);
    tmem_relinquish2();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();            // both CTAs' barriers are initialised before any remote use
  tc_fence_after();
  const uint32_t tmem = S.tmem_base;
  // the leader's barriers, as addresses the peer can reach
  const uint32_t lead_cfull0 = map_to(su32(&S.c_full[0]), 0);
  const uint32_t lead_aready0 = map_to(su32(&S.aready[0]), 0);
  const uint32_t peer_empty0 = map_to(su32(&S.empty[0]), 1);
  const uint32_t peer_done = map_to(su32(&S.done), 1);

  if (warp == 0) {
    if (lane == 0) {
      int issued = 0;
      for (int kb = 0; kb < nblk; ++kb) {
        const int s = kb % kStages;
        const uint32_t ph = (uint32_t)(kb / kStages) & 1u;
        if (kb >= kStages && !mbar_wait(&S.empty[s], ph ^ 1u, abort)) break;
        if (leader) mbar_expect_tx(&S.c_full[s], 2u * kCBytes);   // both token halves
        const uint32_t cfull = lead_cfull0 + 8u * (uint32_t)s;
        tma_load_2d_pair(&S.b[s][0], &map_codes, cfull, kb * kKBlock, mt0);
        tma_load_2d_pair(&S.b[s][kCBytes / 2], &map_codes, cfull, kb * kKBlock + 128, mt0);
        mbar_expect_tx(&S.w_full[s], (uint32_t)kABytes);
        tma_load_2d(&S.a[s][0], &map_w, &S.w_full[s], kb * (kKBlock / 4), n0);
        issued = kb + 1;
      }
      // bounded drain of this CTA's own weight loads (the code loads complete
      // on the leader's barrier; the pair's MMAs, which consume them, are
      // waited for through `done` before anything is freed)
      for (int q = (issued > kStages ? issued - kStages : 0); q < issued; ++q) {
        const long long t0 = clock64();
        while (!mbar_try_wait(&S.w_full[q % kStages], (uint32_t)(q / kStages) & 1u) && clock64() - t0 < kSpinLimit) {
        }
      }
    }
  } else if (warp == 1) {
    if (leader && lane == 0) {
      bool ok = true;
      for (int kb = 0; kb < nblk && ok; ++kb) {
        const int s = kb % kStages;
        const uint32_t ph = (uint32_t)(kb / kStages) & 1u;
        ok = mbar_wait(&S.c_full[s], ph, abort) && mbar_wait(&S.aready[s], ph, abort);
        if (!ok) break;
        tc_fence_after();
        const uint32_t bbase = su32(&S.b[s][0]);
#pragma unroll
        for (int j = 0; j < kKBlock / 32; ++j) {
          const uint32_t a_addr = tmem + (uint32_t)(kDCols + s * kACols + 8 * j);
          const uint64_t bdesc = smem_desc_sw128(bbase + (uint32_t)((j >> 2) * (kCBytes / 2) + (j & 3) * 32));
          mma2_i8(tmem, a_addr, bdesc, kIdesc, (kb > 0 || j > 0) ? 1u : 0u);
        }
        commit2(su32(&S.empty[s]));
        commit2(peer_empty0 + 8u * (uint32_t)s);
      }
      commit2(su32(&S.done));   // arrive once every MMA issued above has completed
      commit2(peer_done);
    }
  } else {
    // converter warps 2..5: TMEM lane quadrant (warp % 4), row = 32 * quadrant + lane
    const int quad = warp & 3;
    const int row = 32 * quad + lane;
    const uint32_t lane_addr = (uint32_t)(32 * quad) << 16;
    for (int kb = 0; kb < nblk; ++kb) {
      const int s = kb % kStages;
      const uint32_t ph = (uint32_t)(kb / kStages) & 1u;
      // the weights landed; the producer reloads a stage only once the pair's
      // MMAs on its previous use are done, so its TMEM A stage is free
      if (!__all_sync(0xffffffffu, mbar_wait(&S.w_full[s], ph, abort))) break;
      tc_fence_after();
      const uint4* src = reinterpret_cast<const uint4*>(&S.a[s][row * (kKBlock / 4)]);
      uint32_t wv[16];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const uint4 q = src[t ^ ((row >> 1) & 3)];
        wv[4 * t] = q.x; wv[4 * t + 1] = q.y; wv[4 * t + 2] = q.z; wv[4 * t + 3] = q.w;
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
      const uint32_t abase = tmem + lane_addr + (uint32_t)(kDCols + s * kACols);
      HBL_TMEM_ST32(abase, c0);
      HBL_TMEM_ST32(abase + 32, c1);
      tc_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) arrive_remote(lead_aready0 + 8u * (uint32_t)s);
    }
    // epilogue: this SM's 128 rows x 256 tokens
    const bool ok = __all_sync(0xffffffffu, mbar_wait(&S.done, 0, abort));
    if (ok && !*abort) {
      tc_fence_after();
      const int n = n0 + row;
      const float a = OUT_BF16 ? __ldg(alpha) : 0.f;
#pragma unroll 1
      for (int c = 0; c < kToks / 32; ++c) {
        uint32_t d[32];
        HBL_TMEM_LD32(tmem + lane_addr + (uint32_t)(32 * c), d);
        tc_wait_ld();
        if (n < N) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int m = m0 + 32 * c + i;
            if (m < M) {
              const int v = (int)d[i] - __ldg(csum + m);
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
  if (warp == 1 && lane == 0 && *abort) {
    // on abort, give the pair's outstanding MMAs a bounded chance to finish
    const long long t0 = clock64();
    while (!mbar_try_wait(&S.done, 0) && clock64() - t0 < kSpinLimit) {
    }
  }
  __syncwarp();
  cluster_sync();            // neither CTA frees memory the pair's MMAs may still read
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc2(tmem, kTmemCols);
  }
}

}  // namespace tcp
}  // namespace hbl
