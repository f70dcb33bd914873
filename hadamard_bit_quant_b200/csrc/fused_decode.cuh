// Fused decode forward: online Hadamard, per-token quantiser, ternary x int8
// GEMM and dequant epilogue in ONE kernel, for 1..16 tokens.
//
// BitNet v2 architecture walkthrough, section 3.4 "H-BitLinear: The Composite
// Layer", Eq. 9 (with Eq. 3-6 for the transform, Eq. 7 / Eq. 8 for the
// quantiser): Y = dequant( Q_A( H x ) (x) T ).
//
// With a few tokens the forward is a pass over N*K/4 bytes of packed weights
// plus a chain of short dependent steps (transform, statistic, codes, MMA,
// epilogue). Two kernels cost two grid boundaries and an L2 round trip of the
// codes; this kernel keeps every intermediate on chip:
//   * one CTA per SM, grouped into clusters of CS CTAs (CS = 1, 2, 4, 8 or
//     16: the token count rounded up to a power of two, halved where such
//     clusters cannot be scheduled);
//   * a producer warp streams the weights of the CTA's 16-row groups through
//     a TMA ring ([16 rows][64 B] boxes, one per 256-k block) from the first
//     instruction on, before the kernel waits for
//     the grid that produced X (programmatic dependent launch);
//   * the 8 consumer warps of cluster rank r transform and quantise token
//     rows r*R .. r*R + R - 1, R = ceil(M / CS) <= 2 (256 threads per row,
//     E = K/256 values per thread, butterflies in registers, passes exchanged
//     through padded shared memory) into this CTA's shared memory: codes
//     row-contiguous, scale and per-warp code sums beside them. The rows are
//     then exchanged in one of two ways (flag 16):
//       - pushed: lane 0 of warp q sends the rows to cluster ranks q and
//         q + 8 (every rank but this one) with bulk copies (shared memory to
//         distributed shared memory, completing as transaction bytes on the
//         peer's mbarrier); each CTA waits on its own barrier for the M - R
//         rows it receives. Bound by the cluster's copy bandwidth (~30 B/cycle
//         into each CTA), so it pays at few tokens only;
//       - through L2: one bulk copy stores this CTA's rows into a global
//         scratch (the forward's workspace), a cluster barrier orders the
//         stores before the loads, and one bulk copy brings all M rows back
//         (every cluster computes the same rows, bit for bit, so clusters that
//         store to the same scratch store the same bytes).
//     Either way each CTA then holds all M x K codes;
//   * the consumers then run the m16n8k32 MMAs of their groups (weights as A,
//     u = t + 1 unpacked in registers; codes as B), batches of groups
//     interleaved for independent accumulator chains, add the 8 warps' partial
//     sums in shared memory, subtract the code sums and store bf16.
// Two cluster barriers. #1 (arrive at start, wait while X loads) makes sure
// every peer runs and has armed its barrier. #2: pushed, arrive once this
// CTA's rows have all landed and wait at exit, which keeps every CTA's shared
// memory alive until the copies out of it have completed; through L2, arrive
// once this CTA's rows are in the scratch and wait before loading the others'.
// Every mbarrier wait is bounded; a CTA that gives up sets the device error
// word, still takes part in both cluster barriers, and writes no output.
#pragma once
#include <cuda.h>
#include "hbl_common.cuh"
#include "fwht_quant.cuh"
#include "gemm_mma.cuh"

namespace hbl {
namespace fdec {

constexpr int kGroupRows = 16;
constexpr int kChunk = 2048;
constexpr int kConsumers = 8;
constexpr int kRowThreads = 32 * kConsumers;        // threads per token row
constexpr int kThreads = 32 * (kConsumers + 1);
constexpr int kStages = 8;
constexpr int kUnitBytes = kGroupRows * (kChunk / 4);   // 8 KB = 8 boxes of [16][64 B], one per 256-k block
constexpr int kMaxGroups = 8;
constexpr int kRowBatch = 2;                        // token rows transformed together
constexpr int kMaxTokens = 16;
constexpr int kMetaBytes = 48;                      // scale + 8 per-warp code sums, padded to 16 B
constexpr long long kSpinLimit = 4000000000ll;

__host__ __device__ constexpr int ilog2_c(int x) { return x <= 1 ? 0 : 1 + ilog2_c(x / 2); }

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
HBL_DEVINL void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];\n" ::"r"(
          su32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(su32(bar)), "r"(x), "r"(y)
      : "memory");
}
HBL_DEVINL void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];\n" ::"r"(
          su32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(su32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}
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
HBL_DEVINL uint32_t map_rank(uint32_t local_addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;\n" : "=r"(r) : "r"(local_addr), "r"(rank));
  return r;
}
// Bulk copy of `bytes` (multiple of 16) from this CTA's shared memory to a
// peer's (addresses from mapa), completing as transaction bytes on the
// peer's mbarrier.
HBL_DEVINL void bulk_to_peer(uint32_t dst, const void* src, uint32_t bytes, uint32_t peer_bar) {
  asm volatile("cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(dst),
               "r"(su32(src)), "r"(bytes), "r"(peer_bar)
               : "memory");
}
HBL_DEVINL void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory"); }
// Shared -> global bulk copy of `bytes` (16-byte aligned, multiple of 16),
// waited for in full (the bytes are written) before the call returns.
HBL_DEVINL void bulk_store_wait(void* dst, const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;\n" ::"l"(dst), "r"(su32(src)), "r"(bytes)
               : "memory");
}
HBL_DEVINL void bulk_commit_wait_all() {
  asm volatile("cp.async.bulk.commit_group;\n" ::: "memory");
  asm volatile("cp.async.bulk.wait_group 0;\n" ::: "memory");
}
// Global -> shared bulk copy completing as transaction bytes on a local mbarrier.
HBL_DEVINL void bulk_load_local(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(
                   su32(dst)),
               "l"(src), "r"(bytes), "r"(su32(bar))
               : "memory");
}
HBL_DEVINL void fence_proxy_async_global() { asm volatile("fence.proxy.async.global;\n" ::: "memory"); }

HBL_DEVINL void cluster_arrive_relaxed() { asm volatile("barrier.cluster.arrive.relaxed.aligned;\n" ::: "memory"); }
HBL_DEVINL void cluster_arrive_release() { asm volatile("barrier.cluster.arrive.release.aligned;\n" ::: "memory"); }
HBL_DEVINL void cluster_wait() { asm volatile("barrier.cluster.wait.acquire.aligned;\n" ::: "memory"); }
// Named barrier over the consumer warps only (the producer never joins it).
HBL_DEVINL void consumers_sync() { asm volatile("bar.sync 1, %0;\n" ::"n"(kRowThreads) : "memory"); }

template <int LOG_K, int MT>
struct Layout {
  static constexpr int K = 1 << LOG_K;
  static constexpr int E = K / kRowThreads;
  static constexpr int KPAD = K + K / E;
  static constexpr size_t kRing = (size_t)kStages * kUnitBytes;
  static constexpr size_t kCodes = (size_t)MT * K;           // K/128 boxes of [MT][128 B]
  static constexpr size_t kX = (size_t)kRowBatch * KPAD * 4;
  static constexpr size_t oCodes = kRing;
  static constexpr size_t oX = oCodes + kCodes;
  static constexpr size_t oMeta = oX + kX;                    // per token: scale, 8 code sums, pad (48 B)
  static constexpr size_t oRed = oMeta + kMaxTokens * kMetaBytes;   // float [kRowBatch * 2][kConsumers]
  static constexpr size_t oBars = oRed + kRowBatch * 2 * kConsumers * 4;
  static constexpr size_t kBytes = 1024 + oBars + (2 * kStages + 1) * 8 + 16;
  static_assert(kMaxGroups * kConsumers * kGroupRows * MT * 4 <= kRing, "reduction must fit in the ring");
};

// Byte offset of the 16-byte code chunk holding k = 16*c16 .. 16*c16+15 of
// token m: token rows are contiguous (K bytes each, so a row moves between
// CTAs as one bulk copy); within each 128-byte segment the eight 16-byte
// chunks are permuted by XOR with 2 * (m % 4). An MMA fragment read (8-byte
// loads) has each half-warp touch 4 tokens x 2 adjacent chunks; the
// permutation puts those 8 (token, chunk) pairs on 8 distinct chunk slots, so
// the read is free of bank conflicts.
HBL_DEVINL int code_swz(int m) { return (m & 3) << 1; }
template <int K>
HBL_DEVINL uint32_t code_off(int m, int c16) {
  return (uint32_t)(m * K + (c16 >> 3) * 128 + (((c16 & 7) ^ code_swz(m)) << 4));
}

// Sum (or max) over the 256 consumer threads of NR values at once (one
// barrier for all rows). Per row: butterfly within each warp, then warps
// 0..7 in order (the order of the quantiser kernels).
template <int NR, bool IS_MAX>
HBL_DEVINL void rows_reduce_n(float (&x)[NR], float* slot) {
#pragma unroll
  for (int r = 0; r < NR; ++r)
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float o = __shfl_xor_sync(0xffffffffu, x[r], off);
      x[r] = IS_MAX ? fmaxf(x[r], o) : x[r] + o;
    }
  if ((threadIdx.x & 31) == 0) {
#pragma unroll
    for (int r = 0; r < NR; ++r) slot[r * kConsumers + (threadIdx.x >> 5)] = x[r];
  }
  consumers_sync();
#pragma unroll
  for (int r = 0; r < NR; ++r) {
    float a = slot[r * kConsumers];
#pragma unroll
    for (int i = 1; i < kConsumers; ++i) a = IS_MAX ? fmaxf(a, slot[r * kConsumers + i]) : a + slot[r * kConsumers + i];
    x[r] = a;
  }
}

// Phase 1 for NR (1 or 2) token rows m0, m0 + 1: load, optional RMSNorm,
// optional transform, quantise, and write the codes, the scale and the
// per-warp code sums of each row into this CTA's shared memory.
template <int LOG_K, int MT, int NR>
HBL_DEVINL void rows_phase(const uint16_t* __restrict__ X, int m0, bool had, bool int8, bool ln,
                           const float* __restrict__ gain, float* xb, float* s_red, uint8_t* cbuf, uint32_t* meta,
                           bool wait1) {
  constexpr int K = 1 << LOG_K, E = K / kRowThreads, G = ilog2_c(E), P = (LOG_K + G - 1) / G, KPAD = K + K / E;
  constexpr int T = kRowThreads;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  float v[NR][E];
  float nrm[NR];
  // loads: the flag branches stay outside the unrolled loops so that every
  // load of a row is in flight at once; `wait1` runs the cluster barrier wait
  // while they are
  if (had) {
    uint32_t raw[NR][E];
#pragma unroll
    for (int r = 0; r < NR; ++r) {
      const uint16_t* xr = X + (size_t)(m0 + r) * K;
#pragma unroll
      for (int j = 0; j < E; ++j) raw[r][j] = __ldg(xr + t + j * T);
    }
    if (wait1) cluster_wait();
#pragma unroll
    for (int r = 0; r < NR; ++r)
#pragma unroll
      for (int j = 0; j < E; ++j) v[r][j] = __uint_as_float(raw[r][j] << 16);
  } else {
    uint4 w4[NR][E / 8];
#pragma unroll
    for (int r = 0; r < NR; ++r) {
      const uint4* src = reinterpret_cast<const uint4*>(X + (size_t)(m0 + r) * K + (size_t)E * t);
#pragma unroll
      for (int q = 0; q < E / 8; ++q) w4[r][q] = __ldg(src + q);
    }
    if (wait1) cluster_wait();
#pragma unroll
    for (int r = 0; r < NR; ++r)
#pragma unroll
      for (int q = 0; q < E / 8; ++q) {
        const uint32_t w[4] = {w4[r][q].x, w4[r][q].y, w4[r][q].z, w4[r][q].w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          v[r][8 * q + 2 * i] = __uint_as_float(w[i] << 16);
          v[r][8 * q + 2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
      }
  }
#pragma unroll
  for (int r = 0; r < NR; ++r) nrm[r] = 1.f;
  if (ln) {
    // RMSNorm: sum of squares of the raw row; the gain per channel (on the
    // pass-0 layout with the transform, on the final layout without); the
    // per-token factor folded into the transform's scale, or applied.
    float tot[NR];
#pragma unroll
    for (int r = 0; r < NR; ++r) {
      float ssq = 0.f;
#pragma unroll
      for (int j = 0; j < E; ++j) ssq = __fmaf_rn(v[r][j], v[r][j], ssq);
      tot[r] = ssq;
    }
    consumers_sync();   // the slots' previous readers are done
    rows_reduce_n<NR, false>(tot, s_red);
#pragma unroll
    for (int r = 0; r < NR; ++r) {
      const float rr = __fdiv_rn(1.f, __fsqrt_rn(__fadd_rn(__fdiv_rn(tot[r], (float)K), kRmsEps)));
      if (had) {
        if (gain) {
#pragma unroll
          for (int j = 0; j < E; ++j) v[r][j] = __fmul_rn(v[r][j], __ldg(gain + t + j * T));
        }
        nrm[r] = rr;
      } else if (gain) {
#pragma unroll
        for (int j = 0; j < E; ++j) v[r][j] = __fmul_rn(__fmul_rn(v[r][j], __ldg(gain + E * t + j)), rr);
      } else {
#pragma unroll
        for (int j = 0; j < E; ++j) v[r][j] = __fmul_rn(__fmul_rn(v[r][j], 1.f), rr);
      }
    }
  }
  if (had) {
#pragma unroll
    for (int p = 0; p < P; ++p) {
      const int hi = LOG_K - p * G;
      const int lo = hi - G > 0 ? hi - G : 0;
      if (p > 0) {
        const int hi_prev = LOG_K - (p - 1) * G;
        const int lo_prev = hi_prev - G > 0 ? hi_prev - G : 0;
        consumers_sync();   // the previous readers of xb are done
#pragma unroll
        for (int r = 0; r < NR; ++r)
#pragma unroll
          for (int j = 0; j < E; ++j) xb[r * KPAD + pad<G>(pass_index<G>(t, j, lo_prev))] = v[r][j];
        consumers_sync();
#pragma unroll
        for (int r = 0; r < NR; ++r)
#pragma unroll
          for (int j = 0; j < E; ++j) v[r][j] = xb[r * KPAD + pad<G>(pass_index<G>(t, j, lo))];
      }
#pragma unroll
      for (int r = 0; r < NR; ++r) butterflies<E>(v[r], hi - lo);
    }
    float sc = __uint_as_float((uint32_t)(127 - LOG_K / 2) << 23);
    if (LOG_K & 1) sc *= 0.70710678118654752f;
#pragma unroll
    for (int r = 0; r < NR; ++r) nrm[r] = __fmul_rn(sc, nrm[r]);
  }
  // thread t now holds elements E*t .. E*t+E-1 of each row: the statistic
  float stat[NR];
#pragma unroll
  for (int r = 0; r < NR; ++r) {
    float part = 0.f;
    if (!int8) {
#pragma unroll
      for (int j = 0; j < E; ++j) part += fabsf(v[r][j]);
    } else {
#pragma unroll
      for (int j = 0; j < E; ++j) part = fmaxf(part, fabsf(v[r][j]));
    }
    stat[r] = part;
  }
  consumers_sync();   // the slots' previous readers are done
  if (int8) rows_reduce_n<NR, true>(stat, s_red + 2 * kConsumers);
  else rows_reduce_n<NR, false>(stat, s_red + 2 * kConsumers);
#pragma unroll
  for (int r = 0; r < NR; ++r) {
    const int m = m0 + r;
    const float rs = __fmul_rn(stat[r], nrm[r]);
    float mult, scale;
    int lo, hi;
    if (!int8) {
      const float beta = __fdiv_rn(rs, (float)K);
      mult = __fdiv_rn(kSqrt7, __fadd_rn(beta, kEps));
      scale = __fdiv_rn(beta, kSqrt7);
      lo = -8; hi = 7;
    } else {
      mult = __fdiv_rn(127.f, __fadd_rn(rs, kEps));
      scale = __fdiv_rn(rs, 127.f);
      lo = -128; hi = 127;
    }
    mult = __fmul_rn(mult, nrm[r]);
    int csum = 0;
    uint32_t packed[E / 4];
    if (int8) {
#pragma unroll
      for (int q = 0; q < E / 4; ++q)
        packed[q] = quant4<false>(v[r][4 * q], v[r][4 * q + 1], v[r][4 * q + 2], v[r][4 * q + 3], mult, 0.f, 0.f);
    } else {
#pragma unroll
      for (int q = 0; q < E / 4; ++q)
        packed[q] = quant4<true>(v[r][4 * q], v[r][4 * q + 1], v[r][4 * q + 2], v[r][4 * q + 3], mult, (float)lo,
                                 (float)hi);
    }
#pragma unroll
    for (int q = 0; q < E / 4; ++q) csum = code_sum4(packed[q], csum);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) csum += __shfl_xor_sync(0xffffffffu, csum, off);
    if constexpr (E == 8) {
      *reinterpret_cast<uint2*>(cbuf + code_off<K>(m, t >> 1) + ((t & 1) << 3)) = make_uint2(packed[0], packed[1]);
    } else {
#pragma unroll
      for (int h = 0; h < E / 16; ++h)
        *reinterpret_cast<uint4*>(cbuf + code_off<K>(m, t * (E / 16) + h)) =
            make_uint4(packed[4 * h], packed[4 * h + 1], packed[4 * h + 2], packed[4 * h + 3]);
    }
    uint32_t* mrow = meta + m * (kMetaBytes / 4);
    if (lane == 0) mrow[1 + warp] = (uint32_t)csum;
    if (t == 0) mrow[0] = __float_as_uint(scale);
  }
}

// Phase 2 for a CTA that owns exactly NG groups: per 2048-k chunk, wait for
// all NG weight units, load every fragment, release the slots, then issue the
// chunk's MMAs q by q over all groups (2*NG independent accumulator chains;
// with one token tile, even and odd q accumulate separately). Codes are read
// from the resident row-major buffer. Ends by writing this warp's partial sums
// into shared memory (aliasing the ring) once every consumer is past its last
// unit: red[warp][group][token][row] (the epilogue's threads take consecutive
// rows of one token, so its reads are free of bank conflicts and its stores
// contiguous).
template <int NG, int TN, int K>
HBL_DEVINL bool fused_mma(uint8_t* ring, const uint8_t* cbuf, uint64_t* wfull, uint64_t* wempty, volatile int* abort,
                          int warp, int lane) {
  constexpr int MT = 8 * TN;
  constexpr int nchunks = K / kChunk;
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
    uint2 bf[TN][8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int box = c * (kChunk / 128) + 2 * warp + (q >> 2), cch = 2 * (q & 3) + (tig >> 1);
#pragma unroll
      for (int i = 0; i < TN; ++i) {
        const int m = 8 * i + g;
        bf[i][q] = *reinterpret_cast<const uint2*>(cbuf + m * K + box * 128 + ((cch ^ code_swz(m)) << 4) +
                                                   ((tig & 1) << 3));
      }
    }
    uint32_t A4[NG][4], B4[NG][4];
    // the NG unit barriers are probed back to back (their round trips overlap);
    // only a unit still in flight is waited for
    bool landed[NG];
#pragma unroll
    for (int b = 0; b < NG; ++b) {
      const int u = c * NG + b;
      landed[b] = mbar_test(&wfull[u % kStages], (uint32_t)(u / kStages) & 1u);
    }
#pragma unroll
    for (int b = 0; b < NG; ++b) {
      const int u = c * NG + b;
      const int s = u % kStages;
      if (!__all_sync(0xffffffffu, landed[b] || mbar_wait(&wfull[s], (uint32_t)(u / kStages) & 1u, abort))) ok = false;
      // block `warp` of the unit: box `warp`, [16 rows][64 B]; rows sit 64 B
      // apart, so the two rows a quarter-warp reads fall in different bank halves
      const uint8_t* wb = ring + (size_t)s * kUnitBytes + warp * (kGroupRows * 64);
      const uint4 pa = *reinterpret_cast<const uint4*>(wb + g * 64 + (tig << 4));
      const uint4 pb = *reinterpret_cast<const uint4*>(wb + (g + 8) * 64 + (tig << 4));
      A4[b][0] = pa.x; A4[b][1] = pa.y; A4[b][2] = pa.z; A4[b][3] = pa.w;
      B4[b][0] = pb.x; B4[b][1] = pb.y; B4[b][2] = pb.z; B4[b][3] = pb.w;
    }
    __syncwarp();
    if (lane == 0) {
#pragma unroll
      for (int b = 0; b < NG; ++b) mbar_arrive(&wempty[(c * NG + b) % kStages]);
    }
    if (!ok) break;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int w = q >> 1, jj = 2 * (q & 1);
#pragma unroll
      for (int b = 0; b < NG; ++b) {
        const uint32_t a[4] = {unpack_u8x4(A4[b][w], jj), unpack_u8x4(B4[b][w], jj), unpack_u8x4(A4[b][w], jj + 1),
                               unpack_u8x4(B4[b][w], jj + 1)};
#pragma unroll
        for (int i = 0; i < TN; ++i) mma_u8s8_16832(acc[b][SPLIT == 2 ? (q & 1) : i], a, bf[i][q].x, bf[i][q].y);
      }
    }
  }
  if constexpr (SPLIT == 2) {
#pragma unroll
    for (int a = 0; a < NG; ++a)
#pragma unroll
      for (int r = 0; r < 4; ++r) acc[a][0][r] += acc[a][1][r];
  }
  consumers_sync();   // every consumer is past its last unit: the ring may be reused
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

// flags: bit 0 use_hadamard, bit 1 INT8 (else INT4), bit 2 RMSNorm prologue,
// bit 3 map_w is the 3-D blocked view (one copy per unit; else 2-D [16][64 B] boxes).
template <int LOG_K, int TN>
__global__ void __launch_bounds__(kThreads, 1)
fused_decode_kernel(const __grid_constant__ CUtensorMap map_w, const uint16_t* __restrict__ X, int M, int N,
                    const float* __restrict__ gain, const float* __restrict__ alpha, int flags,
                    uint16_t* __restrict__ Y, uint8_t* __restrict__ xcodes, uint8_t* __restrict__ xmeta) {
  constexpr int MT = 8 * TN;
  using Lay = Layout<LOG_K, MT>;
  constexpr int nchunks = Lay::K / kChunk;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* ring = base;
  uint8_t* cbuf = base + Lay::oCodes;
  float* xb = reinterpret_cast<float*>(base + Lay::oX);
  uint32_t* meta = reinterpret_cast<uint32_t*>(base + Lay::oMeta);
  float* s_red = reinterpret_cast<float*>(base + Lay::oRed);
  uint64_t* wfull = reinterpret_cast<uint64_t*>(base + Lay::oBars);
  uint64_t* wempty = wfull + kStages;
  uint64_t* codes_full = wempty + kStages;   // the peers' rows have landed
  volatile int* abort = reinterpret_cast<volatile int*>(codes_full + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t crank = cluster_rank(), csize = cluster_size();
  const int groups = N / kGroupRows;
  const int Gd = gridDim.x;
  const int ng = (groups - (int)blockIdx.x + Gd - 1) / Gd;
  const int units = nchunks * ng;
  const bool w3d = (flags & 8) != 0;
  const bool l2x = (flags & 16) != 0;   // rows exchanged through L2 (else pushed to the peers)
  // token rows [m0, m0 + nr) are transformed and quantised by this CTA:
  // ceil(M / cluster size) rows each (at most kRowBatch, checked at launch)
  const int rpc = (M + (int)csize - 1) / (int)csize;
  const int m0 = (int)crank * rpc;
  const int nr = M - m0 < 0 ? 0 : (M - m0 > rpc ? rpc : M - m0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&wfull[s], 1);
      mbar_init(&wempty[s], kConsumers);
    }
    mbar_init(codes_full, 1);
    // codes (K bytes) + scale and code sums of every row this CTA receives:
    // from the peers, the other M - nr rows; from the scratch, all M
    if (csize > 1) mbar_expect_tx(codes_full, (uint32_t)((l2x ? M : M - nr) * (Lay::K + kMetaBytes)));
    *abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  __syncthreads();
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
  // #1: this CTA runs and its codes barrier is armed (peers may copy into it after #1)
  if (csize > 1) cluster_arrive_relaxed();

  if (warp == kConsumers) {
    // ----- producer: the weight ring (independent of the previous grid) -----
    int u = 0;
    auto issue_w = [&](int uu) {
      const int s = uu % kStages;
      const int c = uu / ng, gl = uu % ng;
      const int row0 = ((int)blockIdx.x + gl * Gd) * kGroupRows;
      mbar_expect_tx(&wfull[s], kUnitBytes);
      uint8_t* dst = ring + (size_t)s * kUnitBytes;
      if (w3d) {
        tma_load_3d(dst, &map_w, &wfull[s], 0, row0, c * (kChunk / kKBlock));   // 8 blocks x 16 rows x 64 B
      } else {
#pragma unroll
        for (int b = 0; b < 8; ++b)
          tma_load_2d(dst + b * (kGroupRows * 64), &map_w, &wfull[s], c * (kChunk / 4) + b * 64, row0);
      }
    };
    if (lane == 0)
      for (; u < units && u < kStages; ++u) issue_w(u);
    __syncwarp();
    if (csize > 1) {
      cluster_wait();             // #1
      cluster_arrive_relaxed();   // #2: the producer sends and stores no rows
    }
    if (lane == 0) {
      bool ok = true;
      for (; u < units && ok; ++u) {
        const int s = u % kStages;
        if (!mbar_wait(&wempty[s], (uint32_t)((u / kStages) - 1) & 1u, abort)) { ok = false; break; }
        issue_w(u);
      }
      // bounded drain of the copies issued last
      for (int q = (u > kStages ? u - kStages : 0); q < u; ++q) {
        const long long t0 = clock64();
        while (!mbar_try_wait(&wfull[q % kStages], (uint32_t)(q / kStages) & 1u) && clock64() - t0 < kSpinLimit) {
        }
      }
    }
    __syncwarp();
    if (csize > 1) cluster_wait();   // #2
  } else {
    // ----- consumers, phase 1: transform + quantise this CTA's token rows -----
    const bool had = (flags & 1) != 0, int8 = (flags & 2) != 0, ln = (flags & 4) != 0;
    asm volatile("griddepcontrol.wait;\n" ::: "memory");   // X is ready past this point
    const float a_w = __ldg(alpha);
    // cluster barrier #1 (every peer runs and has armed its codes barrier) is
    // waited while this CTA's X loads are in flight
    const bool wait1 = csize > 1;
    if (nr == 2) rows_phase<LOG_K, MT, 2>(X, m0, had, int8, ln, gain, xb, s_red, cbuf, meta, wait1);
    else if (nr == 1) rows_phase<LOG_K, MT, 1>(X, m0, had, int8, ln, gain, xb, s_red, cbuf, meta, wait1);
    else if (wait1) cluster_wait();
    fence_proxy_async_smem();   // the rows written here are read next by the bulk-copy engine
    consumers_sync();           // ... and by every consumer warp
    bool ok = true;
    if (csize > 1 && !l2x) {
      // lane 0 of warp w sends to peers w, w + 8 (all peers but this CTA)
      if (lane == 0 && nr > 0) {
        for (uint32_t q = (uint32_t)warp; q < csize; q += kConsumers) {
          if (q == crank) continue;
          const uint32_t bar = map_rank(su32(codes_full), q);
          const uint32_t cb_off = (uint32_t)m0 * Lay::K, mt_off = (uint32_t)m0 * kMetaBytes;
          bulk_to_peer(map_rank(su32(cbuf + cb_off), q), cbuf + cb_off, (uint32_t)nr * Lay::K, bar);
          bulk_to_peer(map_rank(su32(reinterpret_cast<uint8_t*>(meta) + mt_off), q),
                       reinterpret_cast<uint8_t*>(meta) + mt_off, (uint32_t)nr * kMetaBytes, bar);
        }
      }
      // the peers' rows
      ok = __all_sync(0xffffffffu, mbar_wait(codes_full, 0u, abort)) != 0;
      cluster_arrive_relaxed();   // #2: every row this CTA receives has landed
    } else if (csize > 1) {
      // this CTA's rows -> the scratch, written in full before barrier #2
      if (warp == 0 && lane == 0 && nr > 0) {
        const uint32_t cb_off = (uint32_t)m0 * Lay::K, mt_off = (uint32_t)m0 * kMetaBytes;
        bulk_store_wait(xcodes + cb_off, cbuf + cb_off, (uint32_t)nr * Lay::K);
        bulk_store_wait(xmeta + mt_off, reinterpret_cast<uint8_t*>(meta) + mt_off, (uint32_t)nr * kMetaBytes);
        bulk_commit_wait_all();
        fence_proxy_async_global();
      }
      __syncwarp();
      cluster_arrive_release();   // #2: this CTA's rows are in the scratch
      cluster_wait();
      // every row of the cluster is in the scratch: load all M of them (this
      // CTA's own rows come back unchanged)
      if (warp == 0 && lane == 0) {
        fence_proxy_async_global();
        bulk_load_local(cbuf, xcodes, (uint32_t)M * Lay::K, codes_full);
        bulk_load_local(meta, xmeta, (uint32_t)M * kMetaBytes, codes_full);
      }
      ok = __all_sync(0xffffffffu, mbar_wait(codes_full, 0u, abort)) != 0;
    }

    // ----- consumers, phase 2: MMAs over the weight ring -----
    switch (ok ? ng : 0) {
      case 1: ok = fused_mma<1, TN, Lay::K>(ring, cbuf, wfull, wempty, abort, warp, lane); break;
      case 2: ok = fused_mma<2, TN, Lay::K>(ring, cbuf, wfull, wempty, abort, warp, lane); break;
      case 3: ok = fused_mma<3, TN, Lay::K>(ring, cbuf, wfull, wempty, abort, warp, lane); break;
      case 4: ok = fused_mma<4, TN, Lay::K>(ring, cbuf, wfull, wempty, abort, warp, lane); break;
      case 5: ok = fused_mma<5, TN, Lay::K>(ring, cbuf, wfull, wempty, abort, warp, lane); break;
      case 6: ok = fused_mma<6, TN, Lay::K>(ring, cbuf, wfull, wempty, abort, warp, lane); break;
      case 7: ok = fused_mma<7, TN, Lay::K>(ring, cbuf, wfull, wempty, abort, warp, lane); break;
      case 8: ok = fused_mma<8, TN, Lay::K>(ring, cbuf, wfull, wempty, abort, warp, lane); break;
      default: consumers_sync(); break;   // no groups (or no codes): keep the barrier count
    }
    consumers_sync();
    if (ok && *abort == 0) {
      const int* red = reinterpret_cast<const int*>(ring);
      const int per_group = kGroupRows * MT;
      for (int e = threadIdx.x; e < ng * per_group; e += kRowThreads) {
        const int gl = e / per_group, rem = e % per_group;
        const int tok = rem / kGroupRows, row = rem % kGroupRows;
        const int n = ((int)blockIdx.x + gl * Gd) * kGroupRows + row;
        if (tok < M) {
          int s = 0;
#pragma unroll
          for (int w = 0; w < kConsumers; ++w) s += red[((w * kMaxGroups + gl) * MT + tok) * kGroupRows + row];
          const uint32_t* mrow = meta + tok * (kMetaBytes / 4);
          int cs = 0;
#pragma unroll
          for (int w = 0; w < kConsumers; ++w) cs += (int)mrow[1 + w];
          s -= cs;
          const float y = __fmul_rn(__fmul_rn((float)s, __uint_as_float(mrow[0])), a_w);
          Y[(size_t)tok * N + n] = float_to_bf16_bits(y);
        }
      }
    }
    // pushed: #2, every copy into every CTA of the cluster has landed, so the
    // rows this CTA sent have been read and its shared memory may be released
    if (csize > 1 && !l2x) cluster_wait();
  }
}

}  // namespace fdec
}  // namespace hbl
