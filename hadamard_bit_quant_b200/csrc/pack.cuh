// Ternary weight quantiser and 2-bit packer.
//
// BitNet v2 architecture walkthrough, section 3.4 "Weight Quantization",
// Eq. 1-2: alpha = mean|W| per tensor, codes RoundClip(W / (alpha + eps), -1, 1),
// two bits per weight plus one fp32 scalar.
//
// alpha is made independent of summation order: every |w| (an fp32) is an
// integer significand m < 2^24 times 2^(E-150), E = max(biased exponent, 1).
// With E = 32*b + r, m << r is added into one of eight 128-bit integer
// accumulators (b = 0..7). Integer addition is exact and commutative, so the
// 8 accumulators hold the exact sum whatever the thread order. A single
// thread then rounds the exact sum once to fp64, divides by N*K in fp64 and
// rounds to fp32.
#pragma once
#include "hbl_common.cuh"

namespace hbl {

struct AbsSumAcc {             // global accumulator, 8 x (lo, hi)
  unsigned long long w[16];
};

HBL_DEVINL void add128(unsigned long long& lo, unsigned long long& hi, unsigned long long v) {
  unsigned long long n = lo + v;
  hi += (n < v) ? 1ull : 0ull;
  lo = n;
}

// Adds |w| (an fp32 bit pattern) to the thread's exact accumulators: most
// weights of a tensor share one exponent bucket, so a thread first tries the
// bucket of its previous value (one compare, one 128-bit add) and only else
// walks the eight buckets.
HBL_DEVINL void abs_acc_add(uint32_t bits, unsigned long long (&lo)[8], unsigned long long (&hi)[8], int& hot,
                            unsigned long long& hlo, unsigned long long& hhi, bool& bad) {
  bits &= 0x7fffffffu;
  uint32_t e = bits >> 23;
  uint32_t m = bits & 0x7fffffu;
  if (e == 255u) { bad = true; return; }
  if (e) m |= 0x800000u; else e = 1u;
  const int bkt = (int)(e >> 5);
  const unsigned long long v = ((unsigned long long)m) << (e & 31u);
  if (bkt == hot) {
    add128(hlo, hhi, v);
    return;
  }
  // flush the hot bucket into its slot and make this one hot
#pragma unroll
  for (int b = 0; b < 8; ++b)
    if (hot == b) { add128(lo[b], hi[b], hlo); hi[b] += hhi; }
  hot = bkt;
  hlo = v;
  hhi = 0ull;
}

__global__ void __launch_bounds__(256) abs_sum_kernel(const float* __restrict__ W, long long n,
                                                      AbsSumAcc* __restrict__ acc) {
  unsigned long long lo[8], hi[8];
#pragma unroll
  for (int b = 0; b < 8; ++b) { lo[b] = 0ull; hi[b] = 0ull; }
  int hot = -1;
  unsigned long long hlo = 0ull, hhi = 0ull;
  bool bad = false;
  const long long stride = (long long)gridDim.x * blockDim.x;
  const long long tid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if ((reinterpret_cast<uintptr_t>(W) & 15u) == 0 && (n & 3) == 0) {
    const uint4* W4 = reinterpret_cast<const uint4*>(W);
    for (long long i = tid; i < n / 4; i += stride) {
      const uint4 q = __ldg(W4 + i);
      abs_acc_add(q.x, lo, hi, hot, hlo, hhi, bad);
      abs_acc_add(q.y, lo, hi, hot, hlo, hhi, bad);
      abs_acc_add(q.z, lo, hi, hot, hlo, hhi, bad);
      abs_acc_add(q.w, lo, hi, hot, hlo, hhi, bad);
    }
  } else {
    for (long long i = tid; i < n; i += stride) abs_acc_add(__float_as_uint(__ldg(W + i)), lo, hi, hot, hlo, hhi, bad);
  }
#pragma unroll
  for (int b = 0; b < 8; ++b)
    if (hot == b) { add128(lo[b], hi[b], hlo); hi[b] += hhi; }
  if (bad) set_device_error(HBL_ERR_INVALID_ARG);
  // warp reduction of each 128-bit bucket
#pragma unroll
  for (int b = 0; b < 8; ++b) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      unsigned long long olo = __shfl_xor_sync(0xffffffffu, lo[b], off);
      unsigned long long ohi = __shfl_xor_sync(0xffffffffu, hi[b], off);
      hi[b] += ohi;
      add128(lo[b], hi[b], olo);
    }
  }
  if ((threadIdx.x & 31) == 0) {
#pragma unroll
    for (int b = 0; b < 8; ++b) {
      if ((lo[b] | hi[b]) == 0ull) continue;
      unsigned long long old = atomicAdd(&acc->w[2 * b], lo[b]);
      unsigned long long carry = (old + lo[b] < lo[b]) ? 1ull : 0ull;
      atomicAdd(&acc->w[2 * b + 1], hi[b] + carry);
    }
  }
}

// Exact sum (8 buckets, value = B_b * 2^(32b - 150)) -> fp64 round-to-nearest-even
// -> / count in fp64 -> fp32. One thread.
__global__ void alpha_finalize_kernel(const AbsSumAcc* __restrict__ acc, long long count,
                                      float* __restrict__ alpha) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  // 14 limbs of 32 bits: bucket b (128 bits) starts at limb b.
  uint32_t L[14];
  for (int i = 0; i < 14; ++i) L[i] = 0u;
  for (int b = 0; b < 8; ++b) {
    const unsigned long long lo = acc->w[2 * b], hi = acc->w[2 * b + 1];
    uint32_t part[4] = {(uint32_t)lo, (uint32_t)(lo >> 32), (uint32_t)hi, (uint32_t)(hi >> 32)};
    unsigned long long carry = 0ull;
    for (int i = 0; i < 4 || carry; ++i) {
      const int li = b + i;
      if (li >= 14) break;
      unsigned long long s = (unsigned long long)L[li] + (i < 4 ? part[i] : 0u) + carry;
      L[li] = (uint32_t)s;
      carry = s >> 32;
    }
  }
  int top = -1;  // index of the highest set bit
  for (int i = 13; i >= 0 && top < 0; --i)
    if (L[i]) top = 32 * i + 31 - __clz(L[i]);
  double sum = 0.0;
  if (top >= 0) {
    auto bit = [&](int p) -> uint32_t { return (p < 0) ? 0u : ((L[p >> 5] >> (p & 31)) & 1u); };
    int shift = top - 52;  // keep 53 bits
    unsigned long long mant = 0ull;
    if (shift <= 0) {
      for (int p = top; p >= 0; --p) mant = (mant << 1) | bit(p);
      shift = 0;
    } else {
      for (int p = top; p >= shift; --p) mant = (mant << 1) | bit(p);
      const uint32_t rb = bit(shift - 1);
      bool sticky = false;
      for (int p = shift - 2; p >= 0 && !sticky; --p) sticky = bit(p) != 0u;
      if (rb && (sticky || (mant & 1ull))) {
        ++mant;
        if (mant == (1ull << 53)) { mant >>= 1; ++shift; }
      }
    }
    sum = ldexp((double)mant, shift - 150);
  }
  const double mean = sum / (double)count;
  *alpha = __double2float_rn(mean);
}

// One thread per packed 32-bit word (16 weights). Word index within a row:
// 16*block + 4*tig + w.
__global__ void __launch_bounds__(256) ternary_pack_kernel(const float* __restrict__ W, int N, int K,
                                                           const float* __restrict__ alpha,
                                                           uint32_t* __restrict__ Wpk) {
  const long long words_per_row = K / 16;
  const long long total = (long long)N * words_per_row;
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= total) return;
  const int n = (int)(idx / words_per_row);
  const int wr = (int)(idx % words_per_row);
  const int blk = wr >> 4, tig = (wr >> 2) & 3, w = wr & 3;
  const float den = __fadd_rn(__ldg(alpha), kEps);
  const float* row = W + (size_t)n * K + (size_t)blk * kKBlock;
  uint32_t out = 0u;
#pragma unroll
  for (int j = 0; j < 4; ++j)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float q = __fdiv_rn(__ldg(row + packed_k_of(tig, w, j, i)), den);
      const int t = clampi((int)rintf(q), -1, 1);
      out |= (uint32_t)(t + 1) << (8 * i + 2 * j);
    }
  Wpk[idx] = out;
}

__global__ void __launch_bounds__(256) ternary_unpack_kernel(const uint32_t* __restrict__ Wpk, int N,
                                                             int K, int8_t* __restrict__ T) {
  const long long words_per_row = K / 16;
  const long long total = (long long)N * words_per_row;
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= total) return;
  const int n = (int)(idx / words_per_row);
  const int wr = (int)(idx % words_per_row);
  const int blk = wr >> 4, tig = (wr >> 2) & 3, w = wr & 3;
  const uint32_t word = __ldg(Wpk + idx);
  int8_t* row = T + (size_t)n * K + (size_t)blk * kKBlock;
#pragma unroll
  for (int j = 0; j < 4; ++j)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int u = (int)((word >> (8 * i + 2 * j)) & 3u);
      row[packed_k_of(tig, w, j, i)] = (int8_t)(u - 1);
    }
}

}  // namespace hbl
