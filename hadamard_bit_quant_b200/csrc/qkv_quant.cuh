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
// flight before the first reduction. Per head: gamma by one warp max
// reduction over the bit patterns of |x| (for non-negative floats the bit
// pattern orders like the value); r = 1 / (gamma + eps) correctly rounded
// (the same value as the division); then per value
//   q = x * (half_top * r) + half_top      (one fused multiply-add),
// rounded to the nearest integer, ties to even, by adding 1.5 * 2^23 (the
// integer then sits in the low bits), and packed four to a word. In exact
// arithmetic q lies in [0, 2^b - 1] (|x| <= gamma < gamma + eps), and the
// fp32 rounding moves it by far less than a half, so no clamp is needed; the
// result can differ from the exact map only at a rounding tie.
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
  uint32_t gbits[R];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    float m = 0.f;
#pragma unroll
    for (int i = 0; i < VPL; ++i) m = fmaxf(m, fabsf(v[r][i]));
    gbits[r] = __reduce_max_sync(0xffffffffu, __float_as_uint(m));
  }
  // rows [bos_lo, bos_hi) are the BOS token's heads
  const long long bos_lo = bos_token >= 0 ? (long long)bos_token * heads : -1;
  const long long bos_hi = bos_token >= 0 ? bos_lo + heads : -1;
  const float2 magic = make_float2(12582912.0f, 12582912.0f);   // 1.5 * 2^23
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int row = row0 + r;
    if (row >= rows) break;
    const float g = __uint_as_float(gbits[r]);
    const int b = (row >= bos_lo && row < bos_hi) ? 8 : bits;
    const float half_top = 0.5f * (float)((1 << b) - 1);
    const float a = __fmul_rn(half_top, __frcp_rn(__fadd_rn(g, kEps)));
    const float2 a2 = make_float2(a, a), h2 = make_float2(half_top, half_top);
    uint32_t q[VPL];
#pragma unroll
    for (int i = 0; i < VPL; i += 2) {
      const float2 t = __fadd2_rn(__ffma2_rn(make_float2(v[r][i], v[r][i + 1]), a2, h2), magic);
      q[i] = __float_as_uint(t.x);
      q[i + 1] = __float_as_uint(t.y);
    }
    // the low byte of each q is its code: bytes 0 of q0, q1 (, q2, q3) side by side
    uint32_t packed[(VPL + 3) / 4];
    if constexpr (VPL >= 4) {
#pragma unroll
      for (int w = 0; w < VPL / 4; ++w)
        packed[w] = __byte_perm(__byte_perm(q[4 * w], q[4 * w + 1], 0x0040),
                                __byte_perm(q[4 * w + 2], q[4 * w + 3], 0x0040), 0x5410);
    } else {
      packed[0] = __byte_perm(q[0], q[1], 0x0040) & 0xffffu;
    }
    uint8_t* dst = codes + (size_t)row * D + VPL * lane;
    if constexpr (VPL == 2) *reinterpret_cast<uint16_t*>(dst) = (uint16_t)packed[0];
    else if constexpr (VPL == 4) *reinterpret_cast<uint32_t*>(dst) = packed[0];
    else *reinterpret_cast<uint2*>(dst) = make_uint2(packed[0], packed[1]);
    if (lane == 0) gamma_out[row] = g;
  }
}

}  // namespace hbl
