// Post-RoPE QKV quantiser: unsigned integers from the absmax of each head.
//
// BitNet v2 architecture walkthrough, section 3.4 "QKV Attention
// Quantization": the query, key and value heads are quantised after RoPE,
// directly, to unsigned b-bit integers (range [0, 2^b - 1]) using the absmax
// of each head; the BOS token's heads keep 8 bits.
//
// Reading of "unsigned absmax": gamma = max|x| over one head vector of one
// token, and [-gamma, gamma] maps affinely onto [0, 2^b - 1]:
//   u = RoundClip((2^b - 1)/2 * (x / (gamma + eps) + 1), 0, 2^b - 1),
// dequantised as (2u / (2^b - 1) - 1) * gamma.
//
// One warp per head vector; each lane holds d/32 consecutive values (one
// 4-, 8- or 16-byte load), so a warp reads the head in one coalesced sweep.
// The kernel is bound by HBM: it reads 2d bytes and writes d + 4 per head.
#pragma once
#include "hbl_common.cuh"

namespace hbl {

template <int VPL>   // values per lane: d = 32 * VPL
__global__ void __launch_bounds__(256) qkv_quant_kernel(const uint16_t* __restrict__ X, int rows, int heads,
                                                        int bits, int bos_token, uint8_t* __restrict__ codes,
                                                        float* __restrict__ gamma_out) {
  constexpr int D = 32 * VPL;
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (row >= rows) return;
  const uint16_t* src = X + (size_t)row * D + VPL * lane;
  float v[VPL];
  if constexpr (VPL == 2) {
    const uint32_t w = __ldg(reinterpret_cast<const uint32_t*>(src));
    v[0] = __uint_as_float(w << 16); v[1] = __uint_as_float(w & 0xffff0000u);
  } else if constexpr (VPL == 4) {
    const uint2 w = __ldg(reinterpret_cast<const uint2*>(src));
    v[0] = __uint_as_float(w.x << 16); v[1] = __uint_as_float(w.x & 0xffff0000u);
    v[2] = __uint_as_float(w.y << 16); v[3] = __uint_as_float(w.y & 0xffff0000u);
  } else {
    const uint4 w = __ldg(reinterpret_cast<const uint4*>(src));
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = __uint_as_float(ws[i] << 16);
      v[2 * i + 1] = __uint_as_float(ws[i] & 0xffff0000u);
    }
  }
  float g = 0.f;
#pragma unroll
  for (int i = 0; i < VPL; ++i) g = fmaxf(g, fabsf(v[i]));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) g = fmaxf(g, __shfl_xor_sync(0xffffffffu, g, off));
  const int b = (bos_token >= 0 && row / heads == bos_token) ? 8 : bits;
  const int top = (1 << b) - 1;
  const float half_top = 0.5f * (float)top;
  const float den = __fadd_rn(g, kEps);
  uint8_t u[VPL];
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const float q = __fdiv_rn(v[i], den);
    const float x = __fmul_rn(half_top, __fadd_rn(q, 1.f));
    u[i] = (uint8_t)clampi(__float2int_rn(x), 0, top);
  }
  uint8_t* dst = codes + (size_t)row * D + VPL * lane;
  if constexpr (VPL == 2) {
    *reinterpret_cast<uint16_t*>(dst) = (uint16_t)(u[0] | (u[1] << 8));
  } else if constexpr (VPL == 4) {
    *reinterpret_cast<uint32_t*>(dst) = (uint32_t)u[0] | ((uint32_t)u[1] << 8) | ((uint32_t)u[2] << 16) |
                                        ((uint32_t)u[3] << 24);
  } else {
    uint2 w;
    w.x = (uint32_t)u[0] | ((uint32_t)u[1] << 8) | ((uint32_t)u[2] << 16) | ((uint32_t)u[3] << 24);
    w.y = (uint32_t)u[4] | ((uint32_t)u[5] << 8) | ((uint32_t)u[6] << 16) | ((uint32_t)u[7] << 24);
    *reinterpret_cast<uint2*>(dst) = w;
  }
  if (lane == 0) gamma_out[row] = g;
}

}  // namespace hbl
