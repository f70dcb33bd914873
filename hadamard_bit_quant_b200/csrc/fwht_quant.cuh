// Online Hadamard transform + per-token activation quantiser.
//
// BitNet v2 architecture walkthrough, section 3.4:
//   * "The Hadamard Transformation", Eq. 3-6: X_r = H_m x, Sylvester H_m with
//     2^(-m/2) scaling, computed by the fast Walsh-Hadamard transform
//     (log2 K butterfly stages).
//   * "Activation Quantization", Eq. 7 (INT8, absmax/127) and Eq. 8 (INT4,
//     absmean/sqrt7), per token, RoundClip with round-half-to-even.
//
// Kernel structure (one token per T = K/E threads, E = 2^G values per thread):
// the log2 K butterfly stages commute, so they are grouped into passes of G
// index bits, processed top-down. In a pass that owns bits [lo, lo+G), thread
// t holds the E values whose indices differ only in those bits, and the
// butterflies run in registers. Between passes the values are exchanged
// through shared memory (one pad word per 2^G values keeps every access
// pattern free of bank conflicts). The first pass owns the top bits, so its loads are
// coalesced across threads; the last pass owns bits [0, G), so each thread
// ends with E consecutive values and stores E consecutive codes.
#pragma once
#include "hbl_common.cuh"

namespace hbl {

enum QuantMode { kModeInt4 = 0, kModeInt8 = 1, kModeF32 = 2 };


template <int LOG_K, int G>
struct FwhtCfg {
  static constexpr int K = 1 << LOG_K;
  static constexpr int E = 1 << G;
  static constexpr int T = K / E;                       // threads per token
  static constexpr int TPC = T >= 128 ? 1 : 128 / T;    // tokens per CTA
  static constexpr int THREADS = T * TPC;
  static constexpr int P = (LOG_K + G - 1) / G;         // passes
  static constexpr int WARPS_PER_TOKEN = T >= 32 ? T / 32 : 1;
  // Two-pass configurations whose token fills whole warps pad 4 words per E
  // values (instead of 1), so the last pass reads its E consecutive values
  // with 16-byte shared-memory loads, still free of bank conflicts.
  static constexpr int PADW = (P == 2 && T >= 32) ? 4 : 1;
  static constexpr int KPAD = K + PADW * (K / E);
  static constexpr size_t SMEM = (size_t)TPC * KPAD * sizeof(float);
};

template <int G>
HBL_DEVINL int pass_index(int t, int j, int lo) {
  const int low = t & ((1 << lo) - 1);
  const int high = t >> lo;
  return low | (j << lo) | (high << (lo + G));
}

// Shared-memory position of index idx: one pad word after every 2^G values.
// For every exchange pattern used here (32 consecutive threads, one register
// index) the padded positions fall in 32 distinct banks, and because the
// thread part and the register part of idx occupy disjoint bits, the
// position splits into (thread part) + (compile-time offset per register).
template <int G, int PADW = 1>
HBL_DEVINL int pad(int idx) { return idx + PADW * (idx >> G); }

// Packed two-lane fp32 arithmetic of sm_100 (each lane an IEEE operation with
// round-to-nearest-even, the same result as the scalar instruction).
HBL_DEVINL float2 f2_add(float2 a, float2 b) {
  unsigned long long r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(*reinterpret_cast<unsigned long long*>(&a)),
      "l"(*reinterpret_cast<unsigned long long*>(&b)));
  return *reinterpret_cast<float2*>(&r);
}
HBL_DEVINL float2 f2_sub(float2 a, float2 b) {
  unsigned long long r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(*reinterpret_cast<unsigned long long*>(&a)),
      "l"(*reinterpret_cast<unsigned long long*>(&b)));
  return *reinterpret_cast<float2*>(&r);
}
HBL_DEVINL float2 f2_fma(float2 a, float2 b, float2 c) {
  unsigned long long r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(*reinterpret_cast<unsigned long long*>(&a)),
      "l"(*reinterpret_cast<unsigned long long*>(&b)), "l"(*reinterpret_cast<unsigned long long*>(&c)));
  return *reinterpret_cast<float2*>(&r);
}

// Codes of four values, RoundClip(mult * v, lo, hi) with round half to even,
// packed little-endian into one word. One fused multiply-add per value forms
// mult * v + 1.5 * 2^23 with a single rounding: for |mult * v| < 2^22 the sum
// lies in [2^23, 2^24), where the float spacing is 1, so the rounding is the
// round-half-to-even of the exact product mult * v to an integer n, and the
// low mantissa byte of the sum is n's two's-complement low byte. With CLAMP
// the sum is then clamped to [1.5 * 2^23 + lo, 1.5 * 2^23 + hi] (exact; a
// product beyond +-2^22 lands outside that range and is clamped the same
// way). Without CLAMP the caller guarantees |mult * v| < 127.5 (the absmax
// quantiser: |v| <= gamma < gamma + eps).
template <bool CLAMP>
HBL_DEVINL uint32_t quant4(float v0, float v1, float v2, float v3, float mult, float lo, float hi) {
  constexpr float kMagic = 12582912.0f;   // 1.5 * 2^23
  const float2 m2 = make_float2(mult, mult);
  const float2 magic = make_float2(kMagic, kMagic);
  float2 a = f2_fma(make_float2(v0, v1), m2, magic);
  float2 b = f2_fma(make_float2(v2, v3), m2, magic);
  if constexpr (CLAMP) {
    const float l = kMagic + lo, h = kMagic + hi;
    a.x = fminf(fmaxf(a.x, l), h);
    a.y = fminf(fmaxf(a.y, l), h);
    b.x = fminf(fmaxf(b.x, l), h);
    b.y = fminf(fmaxf(b.y, l), h);
  }
  const uint32_t lo2 = __byte_perm(__float_as_uint(a.x), __float_as_uint(a.y), 0x0040);
  const uint32_t hi2 = __byte_perm(__float_as_uint(b.x), __float_as_uint(b.y), 0x0040);
  return __byte_perm(lo2, hi2, 0x5410);
}

// Sum of the four signed bytes of a packed code word, added to acc.
HBL_DEVINL int code_sum4(uint32_t w, int acc) { return __dp4a((int)w, 0x01010101, acc); }

// Sum / max over the T threads of one token. Threads of a token are T
// consecutive lanes (T < 32) or T/32 whole warps (T >= 32). `red` holds one
// slot per warp. Deterministic (fixed reduction order).
template <int T, int WPT, bool IS_MAX>
HBL_DEVINL float token_reduce_f(float x, float* red, int token_sub) {
  constexpr int W = T < 32 ? T : 32;
#pragma unroll
  for (int off = W / 2; off > 0; off >>= 1) {
    float o = __shfl_xor_sync(0xffffffffu, x, off);
    x = IS_MAX ? fmaxf(x, o) : x + o;
  }
  if constexpr (T > 32) {
    const int lane = threadIdx.x & 31;
    const int wt = (threadIdx.x % T) >> 5;
    __syncthreads();
    if (lane == 0) red[token_sub * WPT + wt] = x;
    __syncthreads();
    float r = red[token_sub * WPT];
#pragma unroll
    for (int i = 1; i < WPT; ++i) r = IS_MAX ? fmaxf(r, red[token_sub * WPT + i]) : r + red[token_sub * WPT + i];
    x = r;
  }
  return x;
}

template <int T, int WPT>
HBL_DEVINL int token_reduce_i(int x, int* red, int token_sub) {
  constexpr int W = T < 32 ? T : 32;
#pragma unroll
  for (int off = W / 2; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
  if constexpr (T > 32) {
    const int lane = threadIdx.x & 31;
    const int wt = (threadIdx.x % T) >> 5;
    __syncthreads();
    if (lane == 0) red[token_sub * WPT + wt] = x;
    __syncthreads();
    int r = 0;
#pragma unroll
    for (int i = 0; i < WPT; ++i) r += red[token_sub * WPT + i];
    x = r;
  }
  return x;
}

// Quantise E consecutive values v[] of a token whose T threads hold the whole
// row (K values), write codes / scale / code sum, or the fp32 values (kModeF32).
// v holds the values before the scale `nrm` (> 0) of the transform is applied:
// X_r = nrm * v. The scale is applied to the statistic and folded into the
// quantiser's multiplier, so each value is multiplied once.
template <int E, int T, int WPT, int MODE>
HBL_DEVINL void quant_tail(float (&v)[E], int K, int t, int token_sub, bool active, size_t m,
                           float* red_f, int* red_i, int8_t* __restrict__ codes,
                           float* __restrict__ scales, int32_t* __restrict__ csum,
                           float* __restrict__ Xr, float nrm = 1.f) {
  if constexpr (MODE == kModeF32) {
    const float2 n2 = make_float2(nrm, nrm);
#pragma unroll
    for (int j = 0; j < E; j += 2) {
      const float2 r = __fmul2_rn(make_float2(v[j], v[j + 1]), n2);
      v[j] = r.x;
      v[j + 1] = r.y;
    }
    if (active) {
      float4* dst = reinterpret_cast<float4*>(Xr + m * (size_t)K + (size_t)E * t);
#pragma unroll
      for (int q = 0; q < E / 4; ++q) dst[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
    }
    return;
  } else {
    float part = 0.f;
    if constexpr (MODE == kModeInt4 && E >= 64) {
      // many values per thread (configurations with no fused counterpart):
      // eight interleaved partial sums, added in a fixed tree, instead of one
      // chain of E dependent additions
      float p8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int j = 0; j < E; ++j) p8[j & 7] += fabsf(v[j]);
      part = ((p8[0] + p8[1]) + (p8[2] + p8[3])) + ((p8[4] + p8[5]) + (p8[6] + p8[7]));
    } else if constexpr (MODE == kModeInt4) {
#pragma unroll
      for (int j = 0; j < E; ++j) part += fabsf(v[j]);
    } else {
      // the maximum does not depend on the order: eight interleaved chains
      float p8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int j = 0; j < E; ++j) p8[j & 7] = fmaxf(p8[j & 7], fabsf(v[j]));
      part = fmaxf(fmaxf(fmaxf(p8[0], p8[1]), fmaxf(p8[2], p8[3])), fmaxf(fmaxf(p8[4], p8[5]), fmaxf(p8[6], p8[7])));
    }
    const float r = __fmul_rn(token_reduce_f<T, WPT, MODE == kModeInt8>(part, red_f, token_sub), nrm);
    float mult, scale;
    int lo, hi;
    if constexpr (MODE == kModeInt4) {
      const float beta = __fdiv_rn(r, (float)K);               // mean |x|
      mult = __fdiv_rn(kSqrt7, __fadd_rn(beta, kEps));
      scale = __fdiv_rn(beta, kSqrt7);
      lo = -8; hi = 7;
    } else {
      mult = __fdiv_rn(127.f, __fadd_rn(r, kEps));              // gamma = max |x|
      scale = __fdiv_rn(r, 127.f);
      lo = -128; hi = 127;
    }
    mult = __fmul_rn(mult, nrm);
    int cs = 0;
    uint32_t packed[E / 4];
#pragma unroll
    for (int q = 0; q < E / 4; ++q) {
      packed[q] = MODE == kModeInt4
                      ? quant4<true>(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3], mult, (float)lo, (float)hi)
                      : quant4<false>(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3], mult, 0.f, 0.f);
      cs = code_sum4(packed[q], cs);
    }
    if (csum != nullptr) cs = token_reduce_i<T, WPT>(cs, red_i, token_sub);   // uniform branch
    if (active) {
      if constexpr (E >= 16) {
        uint4* dst = reinterpret_cast<uint4*>(codes + m * (size_t)K + (size_t)E * t);
#pragma unroll
        for (int q = 0; q < E / 16; ++q)
          dst[q] = make_uint4(packed[4 * q], packed[4 * q + 1], packed[4 * q + 2], packed[4 * q + 3]);
      } else {
        *reinterpret_cast<uint2*>(codes + m * (size_t)K + (size_t)E * t) = make_uint2(packed[0], packed[1]);
      }
      if (t == 0) {
        scales[m] = scale;
        if (csum) csum[m] = cs;
      }
    }
  }
}

// Butterflies over register-index bits 0..nb-1 of v[0..E). Bit 0 pairs the two
// halves of a register pair (scalar adds); every higher bit pairs whole
// register pairs, done with the packed two-lane fp32 add of sm_100 -- the
// same IEEE additions, half the instructions.
template <int E>
HBL_DEVINL void butterflies(float (&v)[E], int nb) {
  if (nb > 0) {
#pragma unroll
    for (int j = 0; j < E; j += 2) {
      const float a = v[j], b = v[j + 1];
      v[j] = a + b;
      v[j + 1] = a - b;
    }
  }
#pragma unroll
  for (int r = 1; r < 8; ++r) {
    if (r < nb && (1 << r) < E) {
#pragma unroll
      for (int j = 0; j < E; j += 2) {
        if ((j >> r) & 1) continue;
        const int k = j | (1 << r);
        const float2 a = make_float2(v[j], v[j + 1]);
        const float2 b = make_float2(v[k], v[k + 1]);
        const float2 s = f2_add(a, b);
        const float2 d = f2_sub(a, b);
        v[j] = s.x; v[j + 1] = s.y;
        v[k] = d.x; v[k + 1] = d.y;
      }
    }
  }
}

// RMSNorm epsilon of the LN prologue (a reading: the pages give none; the
// quantisers' 1e-5 is reused).
constexpr float kRmsEps = 1e-5f;

// IN_F32: X is fp32 (gradients, latent weights) instead of bf16.
// LN: apply the RMSNorm of Eq. 9 first: x * gain / sqrt(mean(x^2) + eps). The
// per-channel gain is applied on load; the per-token factor commutes with the
// transform and is folded into the final normalisation.
template <int LOG_K, int G, int MODE, bool IN_F32 = false, bool LN = false>
__global__ void __launch_bounds__(FwhtCfg<LOG_K, G>::THREADS)
fwht_quant_kernel(const void* __restrict__ Xv, int M, const float* __restrict__ gain, int8_t* __restrict__ codes,
                  float* __restrict__ scales, int32_t* __restrict__ csum, float* __restrict__ Xr) {
  using C = FwhtCfg<LOG_K, G>;
  constexpr int K = C::K, E = C::E, T = C::T, P = C::P;
  extern __shared__ __align__(16) float smem[];
  __shared__ float red_f[C::TPC * C::WARPS_PER_TOKEN];
  __shared__ int red_i[C::TPC * C::WARPS_PER_TOKEN];
  __shared__ __align__(8) uint64_t stage_bar;

  const int token_sub = threadIdx.x / T;
  const int t = threadIdx.x % T;
  const size_t m = (size_t)blockIdx.x * C::TPC + token_sub;
  const bool active = m < (size_t)M;
  float* sm = smem + (size_t)token_sub * C::KPAD;
  constexpr uint32_t kRowBytes = (uint32_t)K * (IN_F32 ? 4u : 2u);
  const uint32_t bar = (uint32_t)__cvta_generic_to_shared(&stage_bar);

  if (threadIdx.x == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;\n" ::"r"(bar) : "memory");
    // make the initialised barrier visible to the bulk-copy (async) proxy before
    // a copy completes on it: without this, the copy may act on whatever barrier
    // state an earlier CTA left at the same shared-memory address
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  __syncthreads();
  // Programmatic dependent launch: let the consumer grid launch now (it only
  // prefetches weights until this grid completes), and wait for the producer
  // of X before reading it. Both are no-ops without the launch attribute.
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
  // Each token's row arrives by one bulk copy into its exchange buffer; the
  // first pass then reads its strided values (idx = t + j*T) from shared memory.
  if (threadIdx.x == 0) {
    const size_t m0 = (size_t)blockIdx.x * C::TPC;
    const int n = (int)((size_t)M - m0 < (size_t)C::TPC ? (size_t)M - m0 : (size_t)C::TPC);
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(bar), "r"((uint32_t)n * kRowBytes)
                 : "memory");
    for (int i = 0; i < n; ++i) {
      const char* src = reinterpret_cast<const char*>(Xv) + (m0 + i) * (size_t)kRowBytes;
      const uint32_t dst = (uint32_t)__cvta_generic_to_shared(smem + (size_t)i * C::KPAD);
      asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(dst),
                   "l"(src), "r"(kRowBytes), "r"(bar)
                   : "memory");
    }
  }
  {
    uint32_t done = 0;
    const long long t0 = clock64();
    while (true) {
      asm volatile("{\n.reg .pred p;\nmbarrier.try_wait.parity.shared::cta.b64 p, [%1], 0;\nselp.u32 %0, 1, 0, p;\n}\n"
                   : "=r"(done)
                   : "r"(bar)
                   : "memory");
      if (done || clock64() - t0 > 4000000000ll) break;
    }
    if (!done && threadIdx.x == 0) set_device_error(HBL_ERR_TIMEOUT);
  }
  float v[E];
  float ssq = 0.f;
  // Pass 0 owns the top G bits: idx = t + j*T.
  if (active) {
    if constexpr (IN_F32) {
#pragma unroll
      for (int j = 0; j < E; ++j) v[j] = sm[t + j * T];
    } else {
      const uint16_t* row = reinterpret_cast<const uint16_t*>(sm);
#pragma unroll
      for (int j = 0; j < E; ++j) v[j] = bf16_bits_to_float(row[t + j * T]);
    }
  } else {
#pragma unroll
    for (int j = 0; j < E; ++j) v[j] = 0.f;
  }
  if constexpr (LN && E >= 64) {
    // Many values per thread (no fused counterpart): the sum of squares of
    // the raw values runs as eight interleaved chains and is finished before
    // any gain is applied; the gain loads take their address from an opaque
    // zero computed from it, and then from each group's last product, 16
    // values at a time. Otherwise the compiler keeps every raw value alive for
    // the sum while it forms the gain products early, doubling the live values
    // (255 registers and spills). The products are the same whatever the schedule.
    float q8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int j = 0; j < E; ++j) q8[j & 7] = __fmaf_rn(v[j], v[j], q8[j & 7]);
    ssq = ((q8[0] + q8[1]) + (q8[2] + q8[3])) + ((q8[4] + q8[5]) + (q8[6] + q8[7]));
    if (gain) {
      uint32_t z;
      asm volatile("and.b32 %0, %1, 0;\n" : "=r"(z) : "r"(__float_as_uint(ssq)));
      const float* gp = gain + t + z;
#pragma unroll
      for (int j0 = 0; j0 < E; j0 += 16) {
        float g[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) g[i] = __ldg(gp + (j0 + i) * T);
#pragma unroll
        for (int i = 0; i < 16; ++i) v[j0 + i] = __fmul_rn(v[j0 + i], g[i]);
        asm volatile("and.b32 %0, %1, 0;\n" : "=r"(z) : "r"(__float_as_uint(v[j0 + 15])));
        gp += z;
      }
    }
  } else if constexpr (LN) {
#pragma unroll
    for (int j = 0; j < E; ++j) ssq = __fmaf_rn(v[j], v[j], ssq);
    if (gain) {
#pragma unroll
      for (int j = 0; j < E; ++j) v[j] = __fmul_rn(v[j], __ldg(gain + t + j * T));
    }
  }
  __syncthreads();   // the staged rows are consumed; the exchanges overwrite them
#pragma unroll
  for (int p = 0; p < P; ++p) {
    const int hi = LOG_K - p * G;
    const int lo = hi - G > 0 ? hi - G : 0;
    const int nb = hi - lo;        // bits processed in this pass (register bits 0..nb-1)
    if (p > 0) {
      // exchange: previous pass layout -> this pass layout
      const int hi_prev = LOG_K - (p - 1) * G;
      const int lo_prev = hi_prev - G > 0 ? hi_prev - G : 0;
#pragma unroll
      for (int j = 0; j < E; ++j) sm[pad<G, C::PADW>(pass_index<G>(t, j, lo_prev))] = v[j];
      __syncthreads();
      if (C::PADW == 4 && lo == 0) {
        // last pass: E consecutive values at t * (E + 4), 16-byte aligned
        const float4* src = reinterpret_cast<const float4*>(sm + t * (E + 4));
#pragma unroll
        for (int q = 0; q < E / 4; ++q) {
          const float4 f = src[q];
          v[4 * q] = f.x; v[4 * q + 1] = f.y; v[4 * q + 2] = f.z; v[4 * q + 3] = f.w;
        }
      } else {
#pragma unroll
        for (int j = 0; j < E; ++j) v[j] = sm[pad<G, C::PADW>(pass_index<G>(t, j, lo))];
      }
      if (p + 1 < P) __syncthreads();
    }
    butterflies<E>(v, nb);
  }
  // Normalisation 2^(-LOG_K/2) (times the RMSNorm factor with LN).
  {
    float nrm = __uint_as_float((uint32_t)(127 - LOG_K / 2) << 23);
    if (LOG_K & 1) nrm *= 0.70710678118654752f;
    if constexpr (LN) {
      const float tot = token_reduce_f<T, C::WARPS_PER_TOKEN, false>(ssq, red_f, token_sub);
      const float r = __fdiv_rn(1.f, __fsqrt_rn(__fadd_rn(__fdiv_rn(tot, (float)K), kRmsEps)));
      nrm = __fmul_rn(nrm, r);
    }
    quant_tail<E, T, C::WARPS_PER_TOKEN, MODE>(v, K, t, token_sub, active, m, red_f, red_i, codes,
                                               scales, csum, Xr, nrm);
  }
}

// Plain per-token quantiser (no Hadamard), K % 256 == 0, one token per CTA,
// thread t holds the E consecutive values [E*t, E*t + E).
template <int E, int MODE, bool LN = false>
__global__ void __launch_bounds__(1024) quant_rows_kernel(const uint16_t* __restrict__ X, int M, int K,
                                                          const float* __restrict__ gain,
                                                          int8_t* __restrict__ codes,
                                                          float* __restrict__ scales,
                                                          int32_t* __restrict__ csum) {
  __shared__ float red_f[32];
  __shared__ int red_i[32];
  const int t = threadIdx.x;
  const int T = K / E;
  const size_t m = blockIdx.x;
  const bool active = t < T;
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
  float v[E];
  if (active) {
    const uint4* src = reinterpret_cast<const uint4*>(X + m * (size_t)K + (size_t)E * t);
#pragma unroll
    for (int q = 0; q < E / 8; ++q) {
      const uint4 u = __ldg(src + q);
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        v[8 * q + 2 * i] = __uint_as_float(w[i] << 16);
        v[8 * q + 2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
      }
    }
  } else {
#pragma unroll
    for (int j = 0; j < E; ++j) v[j] = 0.f;
  }
  // block-wide reduction over all warps (inactive threads contribute 0)
  const int nw = blockDim.x >> 5;
  const int lane = t & 31, wid = t >> 5;
  if constexpr (LN) {
    float q = 0.f;
#pragma unroll
    for (int j = 0; j < E; ++j) q = __fmaf_rn(v[j], v[j], q);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) q += __shfl_xor_sync(0xffffffffu, q, off);
    if (lane == 0) red_f[wid] = q;
    __syncthreads();
    float tot = 0.f;
    for (int i = 0; i < nw; ++i) tot += red_f[i];
    __syncthreads();
    const float r = __fdiv_rn(1.f, __fsqrt_rn(__fadd_rn(__fdiv_rn(tot, (float)K), kRmsEps)));
#pragma unroll
    for (int j = 0; j < E; ++j) {
      const float gj = (gain && active) ? __ldg(gain + E * t + j) : 1.f;
      v[j] = __fmul_rn(__fmul_rn(v[j], gj), r);
    }
  }
  float part = 0.f;
  if (MODE == kModeInt4) {
#pragma unroll
    for (int j = 0; j < E; ++j) part += fabsf(v[j]);
  } else {
#pragma unroll
    for (int j = 0; j < E; ++j) part = fmaxf(part, fabsf(v[j]));
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float o = __shfl_xor_sync(0xffffffffu, part, off);
    part = (MODE == kModeInt4) ? part + o : fmaxf(part, o);
  }
  if (lane == 0) red_f[wid] = part;
  __syncthreads();
  float r = red_f[0];
  for (int i = 1; i < nw; ++i) r = (MODE == kModeInt4) ? r + red_f[i] : fmaxf(r, red_f[i]);
  float mult, scale;
  int lo, hi;
  if (MODE == kModeInt4) {
    const float beta = __fdiv_rn(r, (float)K);
    mult = __fdiv_rn(kSqrt7, __fadd_rn(beta, kEps));
    scale = __fdiv_rn(beta, kSqrt7);
    lo = -8; hi = 7;
  } else {
    mult = __fdiv_rn(127.f, __fadd_rn(r, kEps));
    scale = __fdiv_rn(r, 127.f);
    lo = -128; hi = 127;
  }
  int cs = 0;   // inactive threads hold zeros, whose codes are 0
  uint32_t packed[E / 4];
#pragma unroll
  for (int q = 0; q < E / 4; ++q) {
    packed[q] = MODE == kModeInt4
                    ? quant4<true>(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3], mult, (float)lo, (float)hi)
                    : quant4<false>(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3], mult, 0.f, 0.f);
    cs = code_sum4(packed[q], cs);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) cs += __shfl_xor_sync(0xffffffffu, cs, off);
  if (lane == 0) red_i[wid] = cs;
  __syncthreads();
  int tot = 0;
  for (int i = 0; i < nw; ++i) tot += red_i[i];
  if (active) {
    if constexpr (E >= 16) {
      uint4* dst = reinterpret_cast<uint4*>(codes + m * (size_t)K + (size_t)E * t);
#pragma unroll
      for (int q = 0; q < E / 16; ++q)
        dst[q] = make_uint4(packed[4 * q], packed[4 * q + 1], packed[4 * q + 2], packed[4 * q + 3]);
    } else {
      uint2* dst = reinterpret_cast<uint2*>(codes + m * (size_t)K + (size_t)E * t);
      dst[0] = make_uint2(packed[0], packed[1]);
    }
    if (t == 0) {
      scales[m] = scale;
      if (csum) csum[m] = tot;
    }
  }
}

// Sum of each row of an int8 code matrix (for hbl_gemm_codes).
__global__ void __launch_bounds__(256) code_rowsum_kernel(const int8_t* __restrict__ codes, int K,
                                                          int32_t* __restrict__ csum) {
  __shared__ int red[8];
  const size_t m = blockIdx.x;
  const uint32_t* row = reinterpret_cast<const uint32_t*>(codes + m * (size_t)K);
  int s = 0;
  for (int i = threadIdx.x; i < K / 4; i += blockDim.x) {
    const uint32_t w = __ldg(row + i);
    s += (int)(int8_t)(w & 0xff) + (int)(int8_t)((w >> 8) & 0xff) + (int)(int8_t)((w >> 16) & 0xff) +
         (int)(int8_t)(w >> 24);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    int tot = 0;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) tot += red[i];
    csum[m] = tot;
  }
}

}  // namespace hbl
