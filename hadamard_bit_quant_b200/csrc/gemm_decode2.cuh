// Decode-regime ternary x int8 GEMM with a K-split across a thread-block
// cluster and the dequant epilogue fused.
//
// BitNet v2 architecture walkthrough, section 3.4 "H-BitLinear: The Composite
// Layer", Eq. 9: acc[m, n] = sum_k c[m, k] * t[n, k]; Y = acc * s[m] * alpha.
//
// A cluster of C CTAs owns 64 output rows; CTA r of the cluster owns the K
// slice [r*KC, (r+1)*KC), KC = K / C. Each CTA
//   1. TMA-loads its 64 x KC/4 bytes of packed weights into 128B-swizzled
//      shared memory as its first action, before waiting for the quantiser
//      grid (programmatic dependent launch), so the weight stream overlaps
//      the Hadamard/quantise kernel;
//   2. after the wait, TMA-loads only its M x KC slice of the int8 codes;
//   3. runs m16n8k32 MMAs in 8 warps (4 row groups x 2 halves of the slice),
//      weights as the A operand unpacked in registers (u = t + 1), codes as B;
//   4. adds the two halves in shared memory, then the cluster reduces over its
//      C slices through distributed shared memory: CTA r sums rows
//      [r*64/C, (r+1)*64/C) across the cluster, subtracts the code sums and
//      stores bf16 (or the int32 result).
// Every wait is bounded. A CTA that gives up still takes part in both cluster
// barriers (so no CTA waits on an exited peer) and writes nothing.
#pragma once
#include <cuda.h>
#include "hbl_common.cuh"
#include "gemm_mma.cuh"

namespace hbl {
namespace dec2 {

constexpr int kRows = 64;
constexpr int kWarps = 8;
constexpr int kThreads = 32 * kWarps;
constexpr long long kSpinLimit = 4000000000ll;

HBL_DEVINL uint32_t su32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

HBL_DEVINL uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;\n" : "=r"(r));
  return r;
}
HBL_DEVINL uint32_t cluster_size() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;\n" : "=r"(r));
  return r;
}
HBL_DEVINL void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;\n" ::: "memory");
}
HBL_DEVINL int ld_dsmem_i32(const void* local, uint32_t rank) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;\n" : "=r"(remote) : "r"(su32(local)), "r"(rank));
  int v;
  asm volatile("ld.shared::cluster.s32 %0, [%1];\n" : "=r"(v) : "r"(remote) : "memory");
  return v;
}

HBL_DEVINL void mbar_init(uint64_t* b, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(su32(b)), "r"(count) : "memory");
}
HBL_DEVINL void mbar_expect_tx(uint64_t* b, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(su32(b)), "r"(bytes) : "memory");
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
HBL_DEVINL bool mbar_wait_bounded(uint64_t* b) {
  const long long t0 = clock64();
  while (!mbar_try_wait(b, 0)) {
    if (clock64() - t0 > kSpinLimit) return false;
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

// Shared memory for a K slice of KC: weights KC/512 boxes of [64][128 B],
// codes KC/128 boxes of [MT][128 B] (both 128B-swizzled, 1024-aligned),
// partial sums [2][64][MT] int32, two mbarriers.
inline size_t smem_bytes(int KC, int MT) {
  const size_t w = (size_t)(KC / 512) * kRows * 128;
  const size_t c = (size_t)(KC / 128) * (size_t)((MT * 128 + 1023) / 1024 * 1024);
  return 1024 + w + c + (size_t)2 * kRows * MT * 4 + 64;
}

template <int TN, bool OUT_BF16>
__global__ void __launch_bounds__(kThreads)
gemm_decode_cluster_kernel(const __grid_constant__ CUtensorMap map_w, const __grid_constant__ CUtensorMap map_c,
                           const int32_t* __restrict__ csum, const float* __restrict__ scales,
                           const float* __restrict__ alpha, int M, int K, int N, int KC, uint16_t* __restrict__ Y,
                           int32_t* __restrict__ acc_out) {
  constexpr int MT = 8 * TN;
  constexpr int CBOX = (MT * 128 + 1023) / 1024 * 1024;   // bytes per codes box, 1024-aligned
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const int nwbox = KC / 512, ncbox = KC / 128;
  uint8_t* wsm = base;
  uint8_t* csm = wsm + (size_t)nwbox * kRows * 128;
  int* part = reinterpret_cast<int*>(csm + (size_t)ncbox * CBOX);
  uint64_t* bars = reinterpret_cast<uint64_t*>(part + 2 * kRows * MT);

  const uint32_t crank = cluster_rank();
  const uint32_t csize = cluster_size();
  const int n0 = blockIdx.y * kRows;
  const int k0 = (int)crank * KC;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, tig = lane & 3;

  if (threadIdx.x == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    mbar_expect_tx(&bars[0], (uint32_t)(nwbox * kRows * 128));
    for (int b = 0; b < nwbox; ++b) tma_load_2d(wsm + (size_t)b * kRows * 128, &map_w, &bars[0], k0 / 4 + b * 128, n0);
  }
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
  __syncthreads();
  asm volatile("griddepcontrol.wait;\n" ::: "memory");   // codes, code sums, scales are ready past this point
  if (threadIdx.x == 0) {
    mbar_expect_tx(&bars[1], (uint32_t)(ncbox * MT * 128));
    for (int b = 0; b < ncbox; ++b) tma_load_2d(csm + (size_t)b * CBOX, &map_c, &bars[1], k0 + b * 128, 0);
  }
  const bool ok = __syncthreads_and(mbar_wait_bounded(&bars[0]) && mbar_wait_bounded(&bars[1])) != 0;
  if (!ok && threadIdx.x == 0) set_device_error(HBL_ERR_TIMEOUT);

  if (ok) {
    int acc[TN][4];
#pragma unroll
    for (int i = 0; i < TN; ++i)
#pragma unroll
      for (int r = 0; r < 4; ++r) acc[i][r] = 0;
    const int rg = warp & 3, kh = warp >> 2;
    const int nb = KC / kKBlock;
    const int b0 = kh * (nb / 2 + (nb & 1)), b1 = min(nb, b0 + nb / 2 + (nb & 1));
    const int ra = 16 * rg + g, rb = ra + 8;
    for (int blk = b0; blk < b1; ++blk) {
      // weights: row r, 16-byte chunk (blk % 2) * 4 + tig of box blk / 2, XOR-swizzled by row % 8
      const int wb = blk >> 1, ch = ((blk & 1) << 2) + tig;
      const uint4 pa = *reinterpret_cast<const uint4*>(wsm + (size_t)wb * kRows * 128 + ra * 128 + ((ch ^ (ra & 7)) << 4));
      const uint4 pb = *reinterpret_cast<const uint4*>(wsm + (size_t)wb * kRows * 128 + rb * 128 + ((ch ^ (rb & 7)) << 4));
      const uint32_t A4[4] = {pa.x, pa.y, pa.z, pa.w};
      const uint32_t B4[4] = {pb.x, pb.y, pb.z, pb.w};
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int w = q >> 1, jj = 2 * (q & 1);
        const uint32_t a[4] = {unpack_u8x4(A4[w], jj), unpack_u8x4(B4[w], jj), unpack_u8x4(A4[w], jj + 1),
                               unpack_u8x4(B4[w], jj + 1)};
        // codes: k = blk*256 + 32q + 8tig -> box 2*blk + q/4, chunk 2*(q%4) + tig/2, 8-byte half tig%2
        const int cb = 2 * blk + (q >> 2), cch = 2 * (q & 3) + (tig >> 1);
#pragma unroll
        for (int i = 0; i < TN; ++i) {
          const int m = 8 * i + g;
          const uint2 bv = *reinterpret_cast<const uint2*>(csm + (size_t)cb * CBOX + m * 128 +
                                                           ((cch ^ (m & 7)) << 4) + ((tig & 1) << 3));
          mma_u8s8_16832(acc[i], a, bv.x, bv.y);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < TN; ++i)
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int row = 16 * rg + g + ((r >> 1) << 3);
        const int tok = 8 * i + 2 * tig + (r & 1);
        part[(kh * kRows + row) * MT + tok] = acc[i][r];
      }
    __syncthreads();
    for (int e = threadIdx.x; e < kRows * MT; e += kThreads) part[e] += part[kRows * MT + e];
  }
  cluster_sync();   // every CTA's partial tile is complete and visible to the cluster
  if (__syncthreads_and(ok) != 0) {
    const int rows_per = kRows / (int)csize;
    const float a = OUT_BF16 ? __ldg(alpha) : 0.f;
    for (int e = threadIdx.x; e < rows_per * MT; e += kThreads) {
      const int tok = e / rows_per, row = (int)crank * rows_per + e % rows_per;
      const int n = n0 + row;
      if (tok < M && n < N) {
        int s = 0;
        for (uint32_t q = 0; q < csize; ++q) s += ld_dsmem_i32(&part[row * MT + tok], q);
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
  cluster_sync();   // keep this CTA's shared memory alive until the peers have read it
}

}  // namespace dec2
}  // namespace hbl
