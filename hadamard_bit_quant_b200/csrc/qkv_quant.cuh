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
// Each lane holds d/32 consecutive values of a head (one 4-, 8- or 16-byte
// load), so a warp reads a head in one coalesced sweep; a warp takes four
// heads. The kernel is bound by HBM: it reads 2d bytes and writes d + 4 per head.
#pragma once
#include "hbl_common.cuh"

namespace hbl {

constexpr int kQkvRowsPerWarp = 4;   // head vectors per warp, all loaded before any is reduced

template <int VPL>   // values per lane: d = 32 * VPL
HBL_DEVINL void qkv_load(const uint16_t* src, float (&v)[VPL]) {
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
}

// Each warp quantises kQkvRowsPerWarp head vectors: their loads are all in
// flight before the first reduction (the kernel is bound by HBM latency x
// bytes in flight). x / (gamma + eps) is computed as x * (1 / (gamma + eps)),
// one reciprocal per head; that moves q by at most an ulp, so a code can
// differ from the exact division only at a rounding tie.
template <int VPL>
__global__ void __launch_bounds__(256) qkv_quant_kernel(const uint16_t* __restrict__ X, int rows, int heads,
                                                        int bits, int bos_token, uint8_t* __restrict__ codes,
                                                        float* __restrict__ gamma_out) {
  constexpr int D = 32 * VPL;
  constexpr int R = kQkvRowsPerWarp;
  const int lane = threadIdx.x & 31;
  const int row0 = (blockIdx.x * 8 + (threadIdx.x >> 5)) * R;
  float v[R][VPL];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    if (row0 + r < rows) qkv_load<VPL>(X + (size_t)(row0 + r) * D + VPL * lane, v[r]);
    else {
#pragma unroll
      for (int i = 0; i < VPL; ++i) v[r][i] = 0.f;
    }
  }
  float g[R];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    g[r] = 0.f;
#pragma unroll
    for (int i = 0; i < VPL; ++i) g[r] = fmaxf(g[r], fabsf(v[r][i]));
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1)
#pragma unroll
    for (int r = 0; r < R; ++r) g[r] = fmaxf(g[r], __shfl_xor_sync(0xffffffffu, g[r], off));
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int row = row0 + r;
    if (row >= rows) break;
    const int b = (bos_token >= 0 && row / heads == bos_token) ? 8 : bits;
    const int top = (1 << b) - 1;
    const float half_top = 0.5f * (float)top;
    const float rden = __fdiv_rn(1.f, __fadd_rn(g[r], kEps));
    uint32_t packed[(VPL + 3) / 4] = {};
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const float x = __fmul_rn(half_top, __fadd_rn(__fmul_rn(v[r][i], rden), 1.f));
      packed[i / 4] |= (uint32_t)clampi(__float2int_rn(x), 0, top) << (8 * (i % 4));
    }
    uint8_t* dst = codes + (size_t)row * D + VPL * lane;
    if constexpr (VPL == 2) *reinterpret_cast<uint16_t*>(dst) = (uint16_t)packed[0];
    else if constexpr (VPL == 4) *reinterpret_cast<uint32_t*>(dst) = packed[0];
    else *reinterpret_cast<uint2*>(dst) = make_uint2(packed[0], packed[1]);
    if (lane == 0) gamma_out[row] = g[r];
  }
}

}  // namespace hbl
