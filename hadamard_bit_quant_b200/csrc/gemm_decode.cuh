// Ternary x int8 GEMM for the decode regime (few tokens per forward), with the
// dequant epilogue fused.
//
// BitNet v2 architecture walkthrough, section 3.4 "H-BitLinear: The Composite
// Layer", Eq. 9: acc[m, n] = sum_k c[m, k] * t[n, k]; Y = acc * s[m] * alpha.
//
// With few tokens the forward is bound by streaming the packed weights from
// HBM. One CTA owns 16 output rows over the whole of K. Their packed bytes are
// contiguous in the weight layout (16 * K/4 bytes), so the CTA fetches them
// with a single bulk copy into shared memory as its first action -- before it
// waits for the quantiser that produces the codes (programmatic dependent
// launch: the weight stream overlaps the Hadamard/quantise kernel). After the
// wait, the 8 warps split K, run m16n8k32 MMAs (weights as the A operand,
// unpacked in registers; codes as the B operand, read from L2), reduce their
// partial sums through shared memory, subtract the code sums and store bf16.
#pragma once
#include "hbl_common.cuh"
#include "gemm_mma.cuh"

namespace hbl {
namespace dec {

constexpr int kRows = 16;
constexpr int kWarps = 8;
constexpr int kThreads = 32 * kWarps;
constexpr long long kSpinLimit = 4000000000ll;

HBL_DEVINL uint32_t su32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

HBL_DEVINL void pdl_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
HBL_DEVINL void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }

HBL_DEVINL uint2 ldg_nc_u2(const void* p) {
  uint2 r;
  asm volatile("ld.global.nc.v2.u32 {%0, %1}, [%2];\n" : "=r"(r.x), "=r"(r.y) : "l"(p));
  return r;
}

inline size_t smem_bytes(int K, int TN) {
  return (size_t)kRows * (K / 4) + (size_t)kWarps * kRows * (8 * TN) * 4 + 64;
}

// OUT_BF16: Y = bf16((acc - csum) * s * alpha); else acc_out = acc - csum (int32).
template <int TN, bool OUT_BF16>
__global__ void __launch_bounds__(kThreads)
gemm_decode_kernel(const int8_t* __restrict__ codes, const int32_t* __restrict__ csum,
                   const float* __restrict__ scales, const float* __restrict__ alpha, int M, int K, int N,
                   const uint8_t* __restrict__ Wpk, uint16_t* __restrict__ Y, int32_t* __restrict__ acc_out) {
  constexpr int MT = 8 * TN;
  extern __shared__ __align__(128) uint8_t sm[];
  const int wbytes = kRows * (K / 4);
  uint8_t* wsm = sm;
  int* red = reinterpret_cast<int*>(sm + wbytes);
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + wbytes + kWarps * kRows * MT * 4);
  const int n0 = blockIdx.x * kRows;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, tig = lane & 3;

  if (threadIdx.x == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;\n" ::"r"(su32(bar)) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(su32(bar)), "r"(wbytes)
                 : "memory");
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(su32(wsm)),
        "l"(Wpk + (size_t)n0 * (K / 4)), "r"(wbytes), "r"(su32(bar))
        : "memory");
  }
  pdl_launch_dependents();
  __syncthreads();
  pdl_wait();   // codes, code sums and scales come from the previous kernel

  {  // bounded wait for the weights
    uint32_t ok = 0;
    const long long t0 = clock64();
    while (true) {
      asm volatile(
          "{\n.reg .pred p;\nmbarrier.try_wait.parity.shared::cta.b64 p, [%1], 0;\nselp.u32 %0, 1, 0, p;\n}\n"
          : "=r"(ok)
          : "r"(su32(bar))
          : "memory");
      if (ok) break;
      if (clock64() - t0 > kSpinLimit) {
        set_device_error(HBL_ERR_TIMEOUT);
        break;
      }
    }
    if (!__all_sync(0xffffffffu, ok != 0)) {
      // the copy may still be in flight: give it a bounded chance to land before exiting
      const long long t1 = clock64();
      while (clock64() - t1 < kSpinLimit) {
        asm volatile(
            "{\n.reg .pred p;\nmbarrier.try_wait.parity.shared::cta.b64 p, [%1], 0;\nselp.u32 %0, 1, 0, p;\n}\n"
            : "=r"(ok)
            : "r"(su32(bar))
            : "memory");
        if (ok) break;
      }
      return;
    }
  }

  int acc[TN][4];
#pragma unroll
  for (int i = 0; i < TN; ++i)
#pragma unroll
    for (int r = 0; r < 4; ++r) acc[i][r] = 0;

  const int nblk = K / kKBlock;
  const int per = (nblk + kWarps - 1) / kWarps;
  const int b0 = warp * per, b1 = min(b0 + per, nblk);
  const uint8_t* rowa = wsm + (size_t)g * (K / 4) + tig * 16;
  const uint8_t* rowb = wsm + (size_t)(g + 8) * (K / 4) + tig * 16;
  for (int blk = b0; blk < b1; ++blk) {
    const uint4 pa = *reinterpret_cast<const uint4*>(rowa + blk * 64);
    const uint4 pb = *reinterpret_cast<const uint4*>(rowb + blk * 64);
    const uint32_t A4[4] = {pa.x, pa.y, pa.z, pa.w};
    const uint32_t B4[4] = {pb.x, pb.y, pb.z, pb.w};
    uint2 bf[TN][8];
#pragma unroll
    for (int i = 0; i < TN; ++i) {
      const int m = 8 * i + g;
#pragma unroll
      for (int q = 0; q < 8; ++q)
        bf[i][q] = (m < M) ? ldg_nc_u2(codes + (size_t)m * K + (size_t)blk * kKBlock + 32 * q + 8 * tig)
                           : make_uint2(0u, 0u);
    }
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int w = q >> 1, jj = 2 * (q & 1);
      const uint32_t a[4] = {unpack_u8x4(A4[w], jj), unpack_u8x4(B4[w], jj), unpack_u8x4(A4[w], jj + 1),
                             unpack_u8x4(B4[w], jj + 1)};
#pragma unroll
      for (int i = 0; i < TN; ++i) mma_u8s8_16832(acc[i], a, bf[i][q].x, bf[i][q].y);
    }
  }
  // partial sums of the 8 warps -> shared memory: red[warp][row][token]
#pragma unroll
  for (int i = 0; i < TN; ++i)
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int row = g + ((r >> 1) << 3);
      const int tok = 8 * i + 2 * tig + (r & 1);
      red[(warp * kRows + row) * MT + tok] = acc[i][r];
    }
  __syncthreads();
  const float a = OUT_BF16 ? __ldg(alpha) : 0.f;
  for (int t = threadIdx.x; t < kRows * MT; t += kThreads) {
    const int tok = t / kRows, row = t % kRows;
    const int n = n0 + row;
    if (tok < M && n < N) {
      int s = 0;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) s += red[(w * kRows + row) * MT + tok];
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

}  // namespace dec
}  // namespace hbl
