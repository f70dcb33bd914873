// Shared helpers for the H-BitLinear kernels (sm_100a). Internal header of libhbl.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/hbl.h"

#define HBL_DEVINL __device__ __forceinline__

namespace hbl {

constexpr float kEps = 1e-5f;                  // eps of Eq. 1, 7 and 8 (reading: 1e-5)
constexpr float kSqrt7 = 2.6457513110645906f;  // anchor of Eq. 8
constexpr int kKBlock = 256;                   // K granule of the packed weight layout

// Device error word: bounded waits set it instead of spinning forever.
// Bit values are hbl_status codes.
__device__ unsigned int g_error_word = 0;

HBL_DEVINL void set_device_error(unsigned int code) { atomicOr(&g_error_word, 1u << code); }

HBL_DEVINL unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;\n" : "=l"(t));
  return t;
}

// Failure-detection check: an mbarrier that nothing will ever complete, waited
// on with the same bounded try_wait loop the pipelined kernels use, but with a
// limit of `timeout_ns`. On expiry the kernel records HBL_ERR_TIMEOUT in the
// device error word and returns normally.
__global__ void wait_timeout_selftest_kernel(unsigned long long timeout_ns, int* gave_up) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t a = (uint32_t)__cvta_generic_to_shared(&bar);
  if (threadIdx.x == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 2;\n" ::"r"(a) : "memory");   // needs 2 arrivals
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(a) : "memory");   // only 1 ever comes
  }
  __syncthreads();
  const unsigned long long t0 = global_ns();
  uint32_t ok = 0;
  while (true) {
    asm volatile("{\n.reg .pred p;\nmbarrier.try_wait.parity.shared::cta.b64 p, [%1], 0;\nselp.u32 %0, 1, 0, p;\n}\n"
                 : "=r"(ok)
                 : "r"(a)
                 : "memory");
    if (ok) break;
    if (global_ns() - t0 > timeout_ns) break;
  }
  if (!ok && threadIdx.x == 0) {
    set_device_error(HBL_ERR_TIMEOUT);
    if (gave_up) *gave_up = 1;
  }
}

// ---------------------------------------------------------------------------
// Packed weight layout (opaque to callers).
//
// Row-major over N; each row holds K/4 bytes in blocks of 256 k (64 bytes).
// Within a block, the 32-bit word at byte offset 16*tig + 4*w (tig, w in 0..3)
// holds, at bits 8*i + 2*j (i, j in 0..3), the 2-bit value u = t + 1 in
// {0, 1, 2} of the ternary weight t at
//     k = 64*w + 32*(j >> 1) + 8*tig + 4*(j & 1) + i.
// Extracting (word >> 2j) & 0x03030303 therefore yields four consecutive k as
// unsigned bytes, and the 16-byte segment tig of a block holds exactly the k
// that lane group tig of an m16n8k32 fragment needs (k = 32q + 8*tig + 0..7
// for q = 0..7). The GEMM computes sum c*u and subtracts sum_k c.
// ---------------------------------------------------------------------------
HBL_DEVINL int packed_k_of(int tig, int w, int j, int i) {
  return 64 * w + 32 * (j >> 1) + 8 * tig + 4 * (j & 1) + i;
}

HBL_DEVINL uint32_t unpack_u8x4(uint32_t word, int j) { return (word >> (2 * j)) & 0x03030303u; }

// bf16 bits -> fp32 (exact)
HBL_DEVINL float bf16_bits_to_float(uint16_t b) { return __uint_as_float(((uint32_t)b) << 16); }

// fp32 -> bf16 bits, round to nearest even
HBL_DEVINL uint16_t float_to_bf16_bits(float f) {
  __nv_bfloat16 h = __float2bfloat16_rn(f);
  return *reinterpret_cast<uint16_t*>(&h);
}

HBL_DEVINL int clampi(int v, int lo, int hi) { return v < lo ? lo : (v > hi ? hi : v); }

}  // namespace hbl
