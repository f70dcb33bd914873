// Weight-streaming ternary x int8 GEMM for the decode regime (1..16 tokens),
// with the dequant epilogue fused.
//
// BitNet v2 architecture walkthrough, section 3.4 "H-BitLinear: The Composite
// Layer", Eq. 9: acc[m, n] = sum_k c[m, k] * t[n, k]; Y = acc * s[m] * alpha.
//
// With few tokens the forward moves N*K/4 bytes of packed weights and little
// else, so the kernel is built to keep HBM busy:
//   * one CTA per SM (persistent); each CTA owns a contiguous run of 16-row
//     groups (the runs differ by at most one group) over the whole of K, so no
//     partial sums ever leave the CTA;
//   * K is walked in chunks of 2048; a chunk's codes (M x 2048 int8) sit in
//     one of two shared-memory buffers, brought by ONE 3-D TMA copy (sixteen
//     128B-swizzled [token][128 B] tiles; token rows past M read as zeros):
//     a copy costs the TMA unit a few hundred cycles whatever its size, and
//     one copy per token row left the unit, not HBM, setting the pace;
//   * the weights stream in units of two neighbouring groups and one chunk --
//     32 rows x 512 bytes, one 16 KB 3-D TMA copy laid out as eight
//     [32 rows][64 B] tiles (an odd last group: one 8 KB copy of [16][64 B]
//     tiles) -- through a ring of 10 (two token tiles) or 12 (one) slots,
//     160 or 192 KB, as much as shared memory holds beside the codes. Copies of
//     8 KB left the copy unit's fixed cost per copy setting the pace. The ring
//     is filled before the kernel waits for the quantiser grid (programmatic
//     dependent launch), so a layer's weights arrive while the previous
//     kernel still runs;
//   * 8 consumer warps take one 256-k block of each unit each: weights as the
//     m16n8k32 A operand (u = t + 1 unpacked in registers, read free of bank
//     conflicts), codes as B (read step by step, at most a 2-way conflict),
//     accumulating in registers across chunks; a dedicated producer warp
//     issues the copies, weights two chunks ahead of the consumers;
//   * at the end the 8 warps' partial sums are added in shared memory, the
//     code sums subtracted, scaled and stored as bf16 (or int32).
// Every mbarrier wait is bounded; a CTA that gives up sets the device error
// word, lets its outstanding copies land (bounded) and exits.
#pragma once
#include <cuda.h>
#include "hbl_common.cuh"
#include "gemm_mma.cuh"

namespace hbl {
namespace strm {

constexpr int kGroupRows = 16;
constexpr int kChunk = 2048;                       // k per chunk
constexpr int kBlocksPerChunk = kChunk / kKBlock;  // 8 = one per consumer warp
constexpr int kConsumers = 8;
constexpr int kThreads = 32 * (kConsumers + 1);
constexpr int kGroupBytes = kGroupRows * (kChunk / 4);  // 8 KB: one group's chunk of weights
constexpr int kUnitBytes = 2 * kGroupBytes;             // ring slot: two groups
constexpr int kMaxGroups = 8;                      // per CTA
constexpr long long kSpinLimit = 4000000000ll;

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
// Non-blocking probe (test_wait never suspends the thread).
HBL_DEVINL bool mbar_test(uint64_t* b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n.reg .pred p;\nmbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\nselp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(su32(b)), "r"(parity)
      : "memory");
  return ok != 0;
}
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
HBL_DEVINL void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];\n" ::"r"(
          su32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(su32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// One chunk of codes: kChunk / 128 column tiles of [MT tokens][128 B], each
// 128B-swizzled (16-byte unit u of token row m at u ^ (m & 7)). A fragment
// read (half-warp: 4 tokens x 32 bytes) meets at most a 2-way bank conflict;
// it happens once per chunk and serves every unit of the chunk.
template <int MT>
struct Layout {
  static constexpr int kStages = MT == 8 ? 12 : 10;       // weight ring slots
  static constexpr int kCodeTile = MT * 128;
  static constexpr int kCodeBuf = (kChunk / 128) * kCodeTile;
  static constexpr size_t kRing = (size_t)kStages * kUnitBytes;
  // wfull, wempty [kStages]; cfull, cempty [2]; abort flag
  static constexpr size_t kBarBytes = (size_t)(2 * kStages + 4) * 8 + 16;
  static constexpr size_t kBytes = 1024 + kRing + 2 * (size_t)kCodeBuf + kBarBytes;
  static_assert(kBytes <= 227 * 1024, "shared memory per block");
};

// Consumer side for a CTA that owns exactly NG groups (NU = ceil(NG / 2)
// units per chunk; group b sits in unit b / 2, rows 16 * (b % 2) on): per
// chunk, wait for the chunk's codes and all NU weight units, load every
// fragment, release the slots, then issue the chunk's MMAs q by q over all
// groups (2*NG independent accumulator chains; with one token tile, even and
// odd q accumulate separately). The unit barriers are probed back to back with
// test_wait (non-blocking), so their round trips (on the order of a hundred
// cycles each) overlap; only a unit still in flight is waited for. Ends by writing this warp's partial sums into shared memory
// (aliasing the ring) once every consumer warp is past its last unit.
template <int NG, int TN, int MT>
HBL_DEVINL bool consume(int nchunks, uint8_t* ring, const uint8_t* cbuf, uint64_t* wfull, uint64_t* wempty,
                        uint64_t* cfull, uint64_t* cempty, volatile int* abort, int warp, int lane) {
  using Lay = Layout<MT>;
  constexpr int kStages = Lay::kStages;
  constexpr int SPLIT = TN == 1 ? 2 : 1;
  const int g = lane >> 2, tig = lane & 3;
  int acc[NG][TN * SPLIT][4];
#pragma unroll
  for (int a = 0; a < NG; ++a)
#pragma unroll
    for (int i = 0; i < TN * SPLIT; ++i)
#pragma unroll
      for (int r = 0; r < 4; ++r) acc[a][i][r] = 0;
  bool ok = true;
  for (int c = 0; c < nchunks && ok; ++c) {
    if (!__all_sync(0xffffffffu, mbar_wait(&cfull[c & 1], (uint32_t)(c >> 1) & 1u, abort))) { ok = false; break; }
    const uint8_t* cb = cbuf + (size_t)(c & 1) * Lay::kCodeBuf;
    constexpr int NU = (NG + 1) / 2;
    uint32_t A4[NG][4], B4[NG][4];
    bool landed[NU];
#pragma unroll
    for (int v = 0; v < NU; ++v) {
      const int u = c * NU + v;
      landed[v] = mbar_test(&wfull[u % kStages], (uint32_t)(u / kStages) & 1u);
    }
#pragma unroll
    for (int v = 0; v < NU; ++v) {
      const int u = c * NU + v;
      if (!__all_sync(0xffffffffu, landed[v] || mbar_wait(&wfull[u % kStages], (uint32_t)(u / kStages) & 1u, abort)))
        ok = false;
    }
#pragma unroll
    for (int b = 0; b < NG; ++b) {
      const int v = b >> 1;
      const int s = (c * NU + v) % kStages;
      constexpr int kLastRows = (NG & 1) ? kGroupRows : 2 * kGroupRows;
      const int rows = (v == NU - 1) ? kLastRows : 2 * kGroupRows;   // rows of the unit's tiles
      // block `warp` of the unit: tile `warp`, [rows][64 B]; rows 64 B apart,
      // so the two rows a quarter-warp reads fall in different bank halves
      const uint8_t* wb = ring + (size_t)s * kUnitBytes + warp * (rows * 64) + (b & 1) * (kGroupRows * 64);
      const uint4 pa = *reinterpret_cast<const uint4*>(wb + g * 64 + (tig << 4));
      const uint4 pb = *reinterpret_cast<const uint4*>(wb + (g + 8) * 64 + (tig << 4));
      A4[b][0] = pa.x; A4[b][1] = pa.y; A4[b][2] = pa.z; A4[b][3] = pa.w;
      B4[b][0] = pb.x; B4[b][1] = pb.y; B4[b][2] = pb.z; B4[b][3] = pb.w;
    }
    __syncwarp();
    if (lane == 0) {
#pragma unroll
      for (int v = 0; v < NU; ++v) mbar_arrive(&wempty[(c * NU + v) % kStages]);
    }
    if (!ok) break;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int w = q >> 1, jj = 2 * (q & 1);
      // codes as the B operand, read per step (they serve every group; held
      // for the whole chunk they pushed the warp's registers into spilling):
      // k = 256 * warp + 32 * q + 8 * tig .. + 7 of the chunk -> column tile
      // 2 * warp + q / 4, 16-byte unit 2 * (q % 4) + tig / 2, half tig % 2
      uint2 bf[TN];
#pragma unroll
      for (int i = 0; i < TN; ++i) {
        const int m = 8 * i + g;
        const int unit = (2 * (q & 3) + (tig >> 1)) ^ (m & 7);
        bf[i] = *reinterpret_cast<const uint2*>(cb + (2 * warp + (q >> 2)) * Lay::kCodeTile + m * 128 + (unit << 4) +
                                                ((tig & 1) << 3));
      }
#pragma unroll
      for (int b = 0; b < NG; ++b) {
        const uint32_t a[4] = {unpack_u8x4(A4[b][w], jj), unpack_u8x4(B4[b][w], jj), unpack_u8x4(A4[b][w], jj + 1),
                               unpack_u8x4(B4[b][w], jj + 1)};
#pragma unroll
        for (int i = 0; i < TN; ++i) mma_u8s8_16832(acc[b][SPLIT == 2 ? (q & 1) : i], a, bf[i].x, bf[i].y);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&cempty[c & 1]);   // this warp no longer reads the chunk's codes
  }
  if constexpr (SPLIT == 2) {
#pragma unroll
    for (int a = 0; a < NG; ++a)
#pragma unroll
      for (int r = 0; r < 4; ++r) acc[a][0][r] += acc[a][1][r];
  }
  // partial sums of the 8 warps -> shared memory (aliases the ring, so only
  // after every warp is done with it): red[warp][group][token][row], so the
  // epilogue's threads (consecutive rows of one token) read without bank
  // conflicts
  asm volatile("bar.sync 1, %0;\n" ::"n"(kConsumers * 32) : "memory");
  if (ok && *abort == 0) {
    int* red = reinterpret_cast<int*>(ring);
#pragma unroll
    for (int gl = 0; gl < NG; ++gl)
#pragma unroll
      for (int i = 0; i < TN; ++i)
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const int row = g + ((r >> 1) << 3);
          const int tok = 8 * i + 2 * tig + (r & 1);
          red[((warp * kMaxGroups + gl) * MT + tok) * kGroupRows + row] = acc[gl][i][r];
        }
  }
  return ok;
}

template <int TN, bool OUT_BF16>
__global__ void __launch_bounds__(kThreads, 1)
gemm_stream_kernel(const __grid_constant__ CUtensorMap map_w2, const __grid_constant__ CUtensorMap map_w1,
                   const __grid_constant__ CUtensorMap map_codes,
                   const int32_t* __restrict__ csum, const float* __restrict__ scales,
                   const float* __restrict__ alpha, int M, int K, int N, uint16_t* __restrict__ Y,
                   int32_t* __restrict__ acc_out) {
  constexpr int MT = 8 * TN;
  using Lay = Layout<MT>;
  constexpr int kStages = Lay::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* ring = base;
  uint8_t* cbuf = ring + Lay::kRing;
  uint64_t* bars = reinterpret_cast<uint64_t*>(cbuf + 2 * Lay::kCodeBuf);
  uint64_t* wfull = bars;                 // [kStages]
  uint64_t* wempty = bars + kStages;      // [kStages]
  uint64_t* cfull = bars + 2 * kStages;   // [2]
  uint64_t* cempty = cfull + 2;           // [2]
  volatile int* abort = reinterpret_cast<volatile int*>(cempty + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int groups = N / kGroupRows;
  const int G = gridDim.x;
  const int gbeg = (int)((long long)groups * blockIdx.x / G);          // this CTA's groups: [gbeg, gend)
  const int ng = (int)((long long)groups * (blockIdx.x + 1) / G) - gbeg;
  const int nu = (ng + 1) / 2;                                         // weight units per chunk
  const int nchunks = K / kChunk;
  const int units = nchunks * nu;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&wfull[s], 1);
      mbar_init(&wempty[s], kConsumers);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&cfull[b], 1);
      mbar_init(&cempty[b], kConsumers);
    }
    *abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  __syncthreads();

  if (warp == kConsumers) {
    // ----- producer -----
    if (lane == 0) {
      auto issue_w = [&](int u) {
        const int s = u % kStages;
        const int c = u / nu, v = u % nu;
        const int row0 = (gbeg + 2 * v) * kGroupRows;
        // 8 blocks x 32 (or 16) rows x 64 B: eight [rows][64 B] tiles in one copy
        const bool pair = 2 * v + 1 < ng;
        mbar_expect_tx(&wfull[s], pair ? kUnitBytes : kGroupBytes);
        tma_load_3d(ring + (size_t)s * kUnitBytes, pair ? &map_w2 : &map_w1, &wfull[s], 0, row0,
                    c * (kChunk / kKBlock));
      };
      auto issue_c = [&](int c) {
        // the whole box counts, zero-filled token rows included
        mbar_expect_tx(&cfull[c & 1], (uint32_t)Lay::kCodeBuf);
        tma_load_3d(cbuf + (size_t)(c & 1) * Lay::kCodeBuf, &map_codes, &cfull[c & 1], 0, 0, c * (kChunk / 128));
      };
      int u = 0;
      for (; u < units && u < kStages; ++u) issue_w(u);             // weights do not depend on the previous grid
      asm volatile("griddepcontrol.wait;\n" ::: "memory");          // codes do
      int issued_c = 0;
      if (nchunks > 0) { issue_c(0); issued_c = 1; }
      bool ok = true;
      // The consumers free chunk c-1's weight slots when they start it (the
      // fragments are then in registers) and its code buffer when they finish
      // it. Iteration c therefore first refills weight slots up to chunk c+1
      // (free since the start of chunk c-1), then chunk c+1's codes (free at
      // the end of chunk c-1): neither waits behind the other. Blocking waits
      // (try_wait suspends the thread), so the producer takes no issue slots
      // from the consumer warps beside it.
      for (int c = 0; c < nchunks && ok; ++c) {
        for (; u < units && u < (c + 2) * nu; ++u) {
          const int s = u % kStages;
          if (!mbar_wait(&wempty[s], (uint32_t)((u / kStages) - 1) & 1u, abort)) { ok = false; break; }
          issue_w(u);
        }
        if (ok && c + 1 < nchunks) {
          if (c + 1 >= 2 && !mbar_wait(&cempty[(c + 1) & 1], (uint32_t)(((c + 1) >> 1) - 1) & 1u, abort)) {
            ok = false;
            break;
          }
          issue_c(c + 1);
          issued_c = c + 2;
        }
      }
      // bounded drain of the copies issued last
      const int last = u;
      for (int q = (last > kStages ? last - kStages : 0); q < last; ++q) {
        const long long t0 = clock64();
        while (!mbar_try_wait(&wfull[q % kStages], (uint32_t)(q / kStages) & 1u) && clock64() - t0 < kSpinLimit) {
        }
      }
      for (int c = (issued_c > 2 ? issued_c - 2 : 0); c < issued_c; ++c) {
        const long long t0 = clock64();
        while (!mbar_try_wait(&cfull[c & 1], (uint32_t)(c >> 1) & 1u) && clock64() - t0 < kSpinLimit) {
        }
      }
    }
    asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
  } else {
    // ----- consumers: warp w takes 256-k block w of every unit -----
    asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
    bool ok = true;
    switch (ng) {
      case 1: ok = consume<1, TN, MT>(nchunks, ring, cbuf, wfull, wempty, cfull, cempty, abort, warp, lane); break;
      case 2: ok = consume<2, TN, MT>(nchunks, ring, cbuf, wfull, wempty, cfull, cempty, abort, warp, lane); break;
      case 3: ok = consume<3, TN, MT>(nchunks, ring, cbuf, wfull, wempty, cfull, cempty, abort, warp, lane); break;
      case 4: ok = consume<4, TN, MT>(nchunks, ring, cbuf, wfull, wempty, cfull, cempty, abort, warp, lane); break;
      case 5: ok = consume<5, TN, MT>(nchunks, ring, cbuf, wfull, wempty, cfull, cempty, abort, warp, lane); break;
      case 6: ok = consume<6, TN, MT>(nchunks, ring, cbuf, wfull, wempty, cfull, cempty, abort, warp, lane); break;
      case 7: ok = consume<7, TN, MT>(nchunks, ring, cbuf, wfull, wempty, cfull, cempty, abort, warp, lane); break;
      default: ok = consume<8, TN, MT>(nchunks, ring, cbuf, wfull, wempty, cfull, cempty, abort, warp, lane); break;
    }
    (void)ok;
  }
  // every copy was consumed (or the CTA gave up); the ring may be reused
  const bool all_ok = __syncthreads_and(*abort == 0) != 0;
  if (all_ok && warp < kConsumers) {
    const int* red = reinterpret_cast<const int*>(ring);
    const float a = OUT_BF16 ? __ldg(alpha) : 0.f;
    const int per_group = kGroupRows * MT;
    for (int e = threadIdx.x; e < ng * per_group; e += kConsumers * 32) {
      const int gl = e / per_group, rem = e % per_group;
      const int tok = rem / kGroupRows, row = rem % kGroupRows;
      const int n = (gbeg + gl) * kGroupRows + row;
      if (tok < M) {
        int s = 0;
#pragma unroll
        for (int w = 0; w < kConsumers; ++w) s += red[((w * kMaxGroups + gl) * MT + tok) * kGroupRows + row];
        s -= __ldg(csum + tok);
        if constexpr (OUT_BF16) {
          const float y = __fmul_rn(__fmul_rn((float)s, __ldg(scales + tok)), a);
          Y[(size_t)tok * N + n] = float_to_bf16_bits(y);
        } else {
          acc_out[(size_t)tok * N + n] = s;
        }
      }
    }
  }
}

}  // namespace strm
}  // namespace hbl
