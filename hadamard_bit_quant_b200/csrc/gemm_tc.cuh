// Ternary x int8 GEMM on the 5th-generation tensor cores (tcgen05, kind::i8),
// for the prefill regime (many tokens per weight row).
//
// BitNet v2 architecture walkthrough, section 3.4 "H-BitLinear: The Composite
// Layer", Eq. 9: acc[m, n] = sum_k c[m, k] * t[n, k], then the dequant
// acc * s[m] * alpha (Eq. 1, Eq. 7 / Eq. 8).
//
// One CTA computes a 128 (output features) x 256 (tokens) tile of D = sum c*u
// (u = t + 1 in {0,1,2}; the exact product is D - sum_k c). When the tiles do
// not fill the last wave of CTAs (one CTA per SM), the tiles of that wave are
// split into two 128-token halves run by two CTAs, so the wave takes about half
// as long (the tail CTAs carry the highest indices and start last):
//   * warp 0 (one lane): TMA producer. Per 256-k stage it loads the codes
//     tile (256 or 128 tokens x 256 k, two 128-byte-wide boxes, 128B swizzle)
//     and the packed weight tile (128 rows x 64 bytes, 64B swizzle).
//   * warps 2..5: converters. Each thread owns one weight row (one TMEM lane),
//     unpacks its 64 packed bytes into 256 unsigned bytes in registers and
//     writes them into the stage's 64 TMEM columns with tcgen05.st. The
//     weights thus become the MMA's A operand straight from tensor memory and
//     never pass through shared memory unpacked.
//   * warp 1 (one lane): MMA issuer. Eight tcgen05.mma.kind::i8 (M=128,
//     N=256 or 128, K=32) per stage, A from TMEM, B (codes) from shared memory,
//     int32 accumulator in TMEM columns [0, N); tcgen05.commit frees the stage.
//   * warps 2..5 again: epilogue. tcgen05.ld of the accumulator, subtract the
//     code sum, scale by s[m] * alpha, store bf16 (or the int32 result).
// Every mbarrier wait is bounded (about a second of clock cycles); on timeout
// the CTA sets the device error word, stops issuing, waits (bounded) for the
// copies and MMAs it already issued, frees its tensor memory and exits.
#pragma once
#include <cuda.h>
#include "hbl_common.cuh"

namespace hbl {
namespace tc {

constexpr int kRows = 128;         // weight rows per tile (MMA M)
constexpr int kStages = 3;
constexpr int kABytes = kRows * (kKBlock / 4);    // 8 KB packed weights per stage
constexpr int kACols = kKBlock / 4;               // 64 TMEM columns of A per stage
constexpr int kTmemCols = 512;
constexpr int kThreads = 192;
constexpr long long kSpinLimit = 4000000000ll;    // ~2 s of SM clock

constexpr int kToks = 256;                        // tokens of a full tile (MMA N)
constexpr int kBBytes = kToks * kKBlock;          // codes per stage (two [256][128 B] boxes)
constexpr int kDCols = kToks;                     // accumulator columns (A stages follow)
static_assert(kDCols + kStages * kACols <= kTmemCols, "TMEM columns");

struct __align__(8) Smem {
  uint8_t b[kStages][kBBytes];      // 1024-byte aligned (swizzle atoms)
  uint8_t a[kStages][kABytes];
  uint64_t full[kStages];           // the stage's codes landed
  uint64_t w_full[kStages];         // the stage's packed weights landed
  uint64_t aready[kStages];
  uint64_t empty[kStages];
  uint64_t done;
  uint32_t tmem_base;
  int abort;
};
constexpr size_t kSmemBytes = sizeof(Smem) + 1024;  // + alignment slack

// Instruction descriptor: D s32, A u8, B s8, both K-major, M = 128, N = toks.
HBL_DEVINL uint32_t idesc_for(int toks) {
  return (2u << 4) | (0u << 7) | (1u << 10) | ((uint32_t)(toks >> 3) << 17) | ((uint32_t)(kRows >> 4) << 24);
}

// Tile of CTA b: CTAs [0, full) own 128 x 256 tiles (output rows fastest);
// each later pair of CTAs splits one of the remaining tiles into two
// 128-token halves.
HBL_DEVINL void cta_tile(int b, int full, int n_tiles, int* n0, int* m0, int* toks) {
  if (b < full) {
    *n0 = (b % n_tiles) * kRows;
    *m0 = (b / n_tiles) * kToks;
    *toks = kToks;
  } else {
    const int h = b - full, t = full + h / 2;
    *n0 = (t % n_tiles) * kRows;
    *m0 = (t / n_tiles) * kToks + (h & 1) * (kToks / 2);
    *toks = kToks / 2;
  }
}

HBL_DEVINL uint32_t su32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

HBL_DEVINL void mbar_init(uint64_t* b, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(su32(b)), "r"(count) : "memory");
}
HBL_DEVINL void mbar_expect_tx(uint64_t* b, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(su32(b)), "r"(bytes) : "memory");
}
HBL_DEVINL void mbar_arrive(uint64_t* b) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(su32(b)) : "memory");
}
HBL_DEVINL bool mbar_try_wait(uint64_t* b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n.reg .pred p;\nmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\nselp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(su32(b)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait. Returns false (and raises the CTA abort flag and the device
// error word) when the phase did not complete within kSpinLimit cycles, or
// when another warp of the CTA already aborted.
HBL_DEVINL bool mbar_wait(uint64_t* b, uint32_t parity, volatile int* abort) {
  const long long t0 = clock64();
  while (!mbar_try_wait(b, parity)) {
    if (*abort) return false;
    if (clock64() - t0 > kSpinLimit) {
      *abort = 1;
      set_device_error(HBL_ERR_TIMEOUT);
      return false;
    }
  }
  return true;
}

HBL_DEVINL void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];\n" ::"r"(
          su32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(su32(bar)), "r"(x), "r"(y)
      : "memory");
}

HBL_DEVINL void tmem_alloc(uint32_t* slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(su32(slot)), "r"(ncols)
               : "memory");
}
HBL_DEVINL void tmem_relinquish() { asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::); }
HBL_DEVINL void tmem_dealloc(uint32_t addr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(addr), "r"(ncols) : "memory");
}
HBL_DEVINL void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory"); }
HBL_DEVINL void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory"); }
HBL_DEVINL void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(su32(bar))
               : "memory");
}
HBL_DEVINL void tc_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory"); }
HBL_DEVINL void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory"); }

// D[tmem] (+)= A[tmem] * B[smem desc], kind::i8, cta_group::1.
HBL_DEVINL void mma_i8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc, uint32_t accum) {
  asm volatile(
      "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accum)
      : "memory");
}


// Shared-memory descriptor of a K-major, 128B-swizzled tile whose rows are
// 128 bytes and whose 8-row groups are 1024 bytes apart.
HBL_DEVINL uint64_t smem_desc_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3fffu);           // start address
  d |= (uint64_t)1u << 16;                            // leading byte offset (unused for swizzled K-major)
  d |= (uint64_t)(1024u >> 4) << 32;                  // stride byte offset: 8 rows x 128 B
  d |= (uint64_t)1u << 46;                            // descriptor version (sm_100)
  d |= (uint64_t)2u << 61;                            // layout: 128B swizzle
  return d;
}

#define HBL_TMEM_ST32(addr, r)                                                                                   \
  asm volatile(                                                                                                  \
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"    \
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n" ::"r"(addr),                         \
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),         \
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), \
      "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), \
      "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])                                                 \
      : "memory")

#define HBL_TMEM_LD32(addr, r)                                                                                   \
  asm volatile(                                                                                                  \
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,"   \
      "%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"                                       \
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),          \
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),    \
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),  \
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])   \
      : "r"(addr)                                                                                                \
      : "memory")

// OUT_BF16: Y = bf16((D - csum) * s * alpha); else acc (int32) = D - csum.
// map_codes loads 256-token boxes, map_codes_half 128-token boxes (split tiles).
template <bool OUT_BF16>
__global__ void __launch_bounds__(kThreads, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap map_codes, const __grid_constant__ CUtensorMap map_codes_half,
               const __grid_constant__ CUtensorMap map_w, int M, int K, int N, int full,
               const int32_t* __restrict__ csum, const float* __restrict__ scales,
               const float* __restrict__ alpha, uint16_t* __restrict__ Y, int32_t* __restrict__ acc_out) {
  extern __shared__ uint8_t smem_raw[];
  Smem& S = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int n0, m0, toks;
  cta_tile(blockIdx.x, full, (N + kRows - 1) / kRows, &n0, &m0, &toks);
  const int bbytes = toks * kKBlock;                 // codes bytes per stage
  const uint32_t idesc = idesc_for(toks);
  const int nblk = K / kKBlock;
  volatile int* abort = &S.abort;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&S.full[s], 1);
      mbar_init(&S.w_full[s], 1);
      mbar_init(&S.aready[s], 128);
      mbar_init(&S.empty[s], 1);
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
  // number of stages the producer issued / MMAs committed (for the bounded drain on abort)
  int issued = 0;

  if (warp == 0) {
    if (lane == 0) {
      for (int kb = 0; kb < nblk; ++kb) {
        const int s = kb % kStages;
        const uint32_t ph = (uint32_t)(kb / kStages) & 1u;
        if (kb >= kStages && !mbar_wait(&S.empty[s], ph ^ 1u, abort)) break;
        const CUtensorMap* mc = toks == kToks ? &map_codes : &map_codes_half;
        // the weights first, on their own barrier: the converters unpack them
        // while the codes are still arriving
        mbar_expect_tx(&S.w_full[s], (uint32_t)kABytes);
        tma_load_2d(&S.a[s][0], &map_w, &S.w_full[s], kb * (kKBlock / 4), n0);
        mbar_expect_tx(&S.full[s], (uint32_t)bbytes);
        tma_load_2d(&S.b[s][0], mc, &S.full[s], kb * kKBlock, m0);
        tma_load_2d(&S.b[s][bbytes / 2], mc, &S.full[s], kb * kKBlock + 128, m0);
        ++issued;
      }
      // drain: wait (bounded) for the last loads issued to land before anyone may exit
      for (int kb = (issued > kStages ? issued - kStages : 0); kb < issued; ++kb) {
        const int s = kb % kStages;
        const long long t0 = clock64();
        while (!mbar_try_wait(&S.full[s], (uint32_t)(kb / kStages) & 1u) && clock64() - t0 < kSpinLimit) {
        }
        while (!mbar_try_wait(&S.w_full[s], (uint32_t)(kb / kStages) & 1u) && clock64() - t0 < kSpinLimit) {
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      bool ok = true;
      for (int kb = 0; kb < nblk && ok; ++kb) {
        const int s = kb % kStages;
        const uint32_t ph = (uint32_t)(kb / kStages) & 1u;
        ok = mbar_wait(&S.full[s], ph, abort) && mbar_wait(&S.aready[s], ph, abort);
        if (!ok) break;
        tc_fence_after();
        const uint32_t bbase = su32(&S.b[s][0]);
#pragma unroll
        for (int j = 0; j < kKBlock / 32; ++j) {
          const uint32_t a_addr = tmem + (uint32_t)(kDCols + s * kACols + 8 * j);
          const uint64_t bdesc = smem_desc_sw128(bbase + (uint32_t)((j >> 2) * (bbytes / 2) + (j & 3) * 32));
          mma_i8_ts(tmem, a_addr, bdesc, idesc, (kb > 0 || j > 0) ? 1u : 0u);
        }
        tc_commit(&S.empty[s]);
        ++issued;
      }
      tc_commit(&S.done);   // arrives once every MMA issued above has completed
    }
  } else {
    // converter warps 2..5: TMEM lane quadrant (warp % 4), row = 32 * quadrant + lane
    const int quad = warp & 3;
    const int row = 32 * quad + lane;
    const uint32_t lane_addr = (uint32_t)(32 * quad) << 16;
    for (int kb = 0; kb < nblk; ++kb) {
      const int s = kb % kStages;
      const uint32_t ph = (uint32_t)(kb / kStages) & 1u;
      // the weights landed; the producer reloads a stage only once its
      // previous MMAs are done, so its TMEM A stage is free
      if (!__all_sync(0xffffffffu, mbar_wait(&S.w_full[s], ph, abort))) break;
      tc_fence_after();
      // the tile arrives 64B-swizzled: 16-byte chunk t of row `row` sits at
      // chunk t ^ ((row >> 1) & 3), which spreads a quarter-warp's 8 rows over
      // all 32 banks
      const uint4* src = reinterpret_cast<const uint4*>(&S.a[s][row * (kKBlock / 4)]);
      uint32_t wv[16];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const uint4 q = src[t ^ ((row >> 1) & 3)];
        wv[4 * t] = q.x; wv[4 * t + 1] = q.y; wv[4 * t + 2] = q.z; wv[4 * t + 3] = q.w;
      }
      // word (tig, w) register j holds k = 64w + 32(j>>1) + 8tig + 4(j&1) + i, i.e.
      // TMEM column 16w + 8(j>>1) + 2tig + (j&1) of this stage.
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
      mbar_arrive(&S.aready[s]);
    }
    // epilogue
    const bool ok = __all_sync(0xffffffffu, mbar_wait(&S.done, 0, abort));
    if (ok && !*abort) {
      tc_fence_after();
      const int n = n0 + row;
      const float a = OUT_BF16 ? __ldg(alpha) : 0.f;
#pragma unroll 1
      for (int c = 0; c < toks / 32; ++c) {
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
  if (warp == 1) {
    // on abort, give outstanding MMAs a bounded chance to finish before freeing TMEM
    if (*abort) {
      const long long t0 = clock64();
      while (!mbar_try_wait(&S.done, 0) && clock64() - t0 < kSpinLimit) {
      }
    }
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace tc
}  // namespace hbl
