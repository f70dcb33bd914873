// Ternary x int8 GEMM on the warp-level tensor-core path (mma.sync m16n8k32),
// plus the dequant epilogue.
//
// BitNet v2 architecture walkthrough, section 3.4 "H-BitLinear: The Composite
// Layer", Eq. 9: Y = Q_w(W) . Q_INT8/4(X_r). The integer part is
// acc[m, n] = sum_k c[m, k] * t[n, k]; the dequant is acc * s[m] * alpha
// (Eq. 1 for alpha, Eq. 7 / Eq. 8 for s).
//
// Weights enter the MMA as the A operand (swap-AB: output features in the MMA
// M slot, tokens in the N slot), unpacked in registers straight from the
// packed stream: each lane loads one 16-byte segment per row and 256-k block
// and shifts/masks it into four m16n8k32 A fragments of u = t + 1. The codes
// are the B operand, staged in shared memory by cp.async. D holds
// sum c*u; the exact product is D - sum_k c[m, k].
#pragma once
#include "hbl_common.cuh"

namespace hbl {

HBL_DEVINL void mma_u8s8_16832(int (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

HBL_DEVINL uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

HBL_DEVINL void cp_async16(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(src_bytes));
}
HBL_DEVINL void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N_>
HBL_DEVINL void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N_)); }

constexpr int kMmaRowsPerCta = 64;     // 4 warps x 16 output features
constexpr int kCodesRowBytes = 256 + 32;  // padded: conflict-free 8-byte fragment reads

// D (M x N int32) = sum over this CTA's k-slice of c * u; atomicAdd when split.
template <int TN>
__global__ void __launch_bounds__(128) gemm_mma_kernel(const int8_t* __restrict__ codes, int M, int K,
                                                       int N, const uint4* __restrict__ Wpk,
                                                       int kblocks_per_split, int32_t* __restrict__ D,
                                                       int atomic) {
  constexpr int MT = 8 * TN;
  __shared__ __align__(16) int8_t cs[2][MT * kCodesRowBytes];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, tig = lane & 3;
  const int n0 = blockIdx.x * kMmaRowsPerCta + warp * 16;
  const int m0 = blockIdx.y * MT;
  const int nblk = K / kKBlock;
  const int kb0 = blockIdx.z * kblocks_per_split;
  const int kb1 = min(kb0 + kblocks_per_split, nblk);
  const int ra = min(n0 + g, N - 1), rb = min(n0 + g + 8, N - 1);
  const uint4* wa = Wpk + (size_t)ra * (K / 64) + tig;
  const uint4* wb = Wpk + (size_t)rb * (K / 64) + tig;

  int acc[TN][4];
#pragma unroll
  for (int i = 0; i < TN; ++i)
#pragma unroll
    for (int r = 0; r < 4; ++r) acc[i][r] = 0;

  auto load_codes = [&](int stage, int kb) {
    for (int c = threadIdx.x; c < MT * 16; c += 128) {
      const int row = c >> 4, ch = c & 15;
      const int m = m0 + row;
      const int8_t* src = codes + (size_t)min(m, M - 1) * K + (size_t)kb * kKBlock + ch * 16;
      cp_async16(smem_u32(&cs[stage][row * kCodesRowBytes + ch * 16]), src, m < M ? 16 : 0);
    }
    cp_async_commit();
  };

  if (kb0 < kb1) load_codes(0, kb0);
  uint4 pa = make_uint4(0, 0, 0, 0), pb = pa;
  if (kb0 < kb1) { pa = __ldg(wa + (size_t)kb0 * 4); pb = __ldg(wb + (size_t)kb0 * 4); }
  for (int kb = kb0; kb < kb1; ++kb) {
    const int st = (kb - kb0) & 1;
    const bool more = kb + 1 < kb1;
    if (more) load_codes(st ^ 1, kb + 1);
    uint4 na = pa, nb = pb;
    if (more) { na = __ldg(wa + (size_t)(kb + 1) * 4); nb = __ldg(wb + (size_t)(kb + 1) * 4); }
    if (more) cp_async_wait<1>(); else cp_async_wait<0>();
    __syncthreads();
    const uint32_t A4[4] = {pa.x, pa.y, pa.z, pa.w};
    const uint32_t B4[4] = {pb.x, pb.y, pb.z, pb.w};
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int w = q >> 1, jj = 2 * (q & 1);
      const uint32_t a[4] = {unpack_u8x4(A4[w], jj), unpack_u8x4(B4[w], jj), unpack_u8x4(A4[w], jj + 1),
                             unpack_u8x4(B4[w], jj + 1)};
#pragma unroll
      for (int i = 0; i < TN; ++i) {
        const uint2 b = *reinterpret_cast<const uint2*>(&cs[st][(8 * i + g) * kCodesRowBytes + 32 * q + 8 * tig]);
        mma_u8s8_16832(acc[i], a, b.x, b.y);
      }
    }
    __syncthreads();
    pa = na; pb = nb;
  }
#pragma unroll
  for (int i = 0; i < TN; ++i)
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int n = n0 + g + ((r >> 1) << 3);
      const int m = m0 + 8 * i + 2 * tig + (r & 1);
      if (n < N && m < M) {
        int32_t* p = D + (size_t)m * N + n;
        if (atomic) atomicAdd(p, acc[i][r]); else *p = acc[i][r];
      }
    }
}

// Y[m, n] = bf16( (D[m, n] - csum[m]) * s[m] * alpha ); 8 outputs per thread.
__global__ void __launch_bounds__(256) dequant_store_kernel(const int32_t* __restrict__ D,
                                                            const int32_t* __restrict__ csum,
                                                            const float* __restrict__ scales,
                                                            const float* __restrict__ alpha, int M, int N,
                                                            uint16_t* __restrict__ Y) {
  const long long i8 = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long total8 = (long long)M * N / 8;
  if (i8 >= total8) return;
  const long long e0 = i8 * 8;
  const int m = (int)(e0 / N);
  const float s = __ldg(scales + m), a = __ldg(alpha);
  const int cs = __ldg(csum + m);
  const int4* src = reinterpret_cast<const int4*>(D + e0);
  const int4 d0 = src[0], d1 = src[1];
  const int dv[8] = {d0.x, d0.y, d0.z, d0.w, d1.x, d1.y, d1.z, d1.w};
  uint32_t out[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float y0 = __fmul_rn(__fmul_rn((float)(dv[2 * q] - cs), s), a);
    const float y1 = __fmul_rn(__fmul_rn((float)(dv[2 * q + 1] - cs), s), a);
    out[q] = (uint32_t)float_to_bf16_bits(y0) | ((uint32_t)float_to_bf16_bits(y1) << 16);
  }
  *reinterpret_cast<uint4*>(Y + e0) = make_uint4(out[0], out[1], out[2], out[3]);
}

// acc[m, n] = D[m, n] - csum[m] (integer result of hbl_gemm_codes).
__global__ void __launch_bounds__(256) sub_rowsum_kernel(int32_t* __restrict__ D,
                                                         const int32_t* __restrict__ csum, int M, int N) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (long long)M * N) return;
  D[i] -= __ldg(csum + i / N);
}

}  // namespace hbl
