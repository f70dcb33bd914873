// C ABI of libhbl: argument checks, workspace layout and kernel dispatch for the
// H-BitLinear forward (BitNet v2 architecture walkthrough, section 3.4, Eq. 9).
// All kernels live in the headers included below (one translation unit, so the
// device error word is shared).
#include <atomic>
#include <mutex>
#include <cstring>
#include <string>
#include <vector>

#include <cuda.h>

#include "hbl_common.cuh"
#include "pack.cuh"
#include "fwht_quant.cuh"
#include "gemm_mma.cuh"
#include "gemm_tc.cuh"
#include "gemm_tc2.cuh"
#include "gemm_decode.cuh"
#include "gemm_decode2.cuh"
#include "gemm_stream.cuh"
#include "fused_decode.cuh"
#include "qkv_quant.cuh"

namespace hbl {
namespace {

constexpr int kMaxDevices = 64;

struct DeviceState {
  bool probed = false;
  bool supported = false;
  int sm_count = 0;
  AbsSumAcc* abs_acc = nullptr;   // scratch of hbl_pack_weights
  void* ws = nullptr;             // workspace of hbl_forward
  size_t ws_bytes = 0;
};

std::mutex g_mu;
DeviceState g_dev[kMaxDevices];

// Per-kernel timing: CUDA events around each launch while enabled.
struct Profiler {
  struct Entry { std::string name; int launches = 0; double ms = 0.0; };
  struct Pending { int entry; cudaEvent_t a, b; };
  std::mutex mu;
  bool on = false;
  std::vector<Entry> entries;
  std::vector<Pending> pending;
  std::vector<cudaEvent_t> pool;

  cudaEvent_t take() {
    if (!pool.empty()) { cudaEvent_t e = pool.back(); pool.pop_back(); return e; }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
  }
  void flush() {
    for (auto& p : pending) {
      float ms = 0.f;
      if (cudaEventSynchronize(p.b) == cudaSuccess && cudaEventElapsedTime(&ms, p.a, p.b) == cudaSuccess) {
        entries[p.entry].launches += 1;
        entries[p.entry].ms += ms;
      }
      pool.push_back(p.a);
      pool.push_back(p.b);
    }
    pending.clear();
  }
};
Profiler g_prof;

// Returns a token for prof_end (-1 when timing is off).
int prof_begin(const char* name, cudaStream_t s) {
  if (!g_prof.on) return -1;
  std::lock_guard<std::mutex> lk(g_prof.mu);
  int idx = -1;
  for (size_t i = 0; i < g_prof.entries.size(); ++i)
    if (g_prof.entries[i].name == name) { idx = (int)i; break; }
  if (idx < 0) { g_prof.entries.push_back(Profiler::Entry{name, 0, 0.0}); idx = (int)g_prof.entries.size() - 1; }
  Profiler::Pending p{idx, g_prof.take(), g_prof.take()};
  cudaEventRecord(p.a, s);
  g_prof.pending.push_back(p);
  return (int)g_prof.pending.size() - 1;
}

void prof_end(int token, cudaStream_t s) {
  if (token < 0) return;
  std::lock_guard<std::mutex> lk(g_prof.mu);
  if (token < (int)g_prof.pending.size()) cudaEventRecord(g_prof.pending[token].b, s);
}

struct ProfScope {
  int tok;
  cudaStream_t s;
  ProfScope(const char* name, cudaStream_t st) : tok(prof_begin(name, st)), s(st) {}
  ~ProfScope() { prof_end(tok, s); }
};

int current_device(int* dev) {
  if (cudaGetDevice(dev) != cudaSuccess) return HBL_ERR_CUDA;
  if (*dev < 0 || *dev >= kMaxDevices) return HBL_ERR_UNSUPPORTED;
  return HBL_OK;
}

// Probe the device once: sm_100 only. Also raises the dynamic shared memory
// limit of the kernels that need more than 48 KB.
int ensure_device(DeviceState** out) {
  int dev = 0;
  int st = current_device(&dev);
  if (st) return st;
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceState& d = g_dev[dev];
  if (!d.probed) {
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return HBL_ERR_CUDA;
    d.supported = (prop.major == 10 && prop.minor == 0);
    d.sm_count = prop.multiProcessorCount;
    d.probed = true;
    if (d.supported) {
      {
        const int mx = 200 * 1024;
        cudaFuncSetAttribute(dec::gemm_decode_kernel<1, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, mx);
        cudaFuncSetAttribute(dec::gemm_decode_kernel<2, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, mx);
        cudaFuncSetAttribute(dec::gemm_decode_kernel<4, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, mx);
        cudaFuncSetAttribute(dec::gemm_decode_kernel<8, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, mx);
        cudaFuncSetAttribute(dec::gemm_decode_kernel<1, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, mx);
        cudaFuncSetAttribute(dec::gemm_decode_kernel<2, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, mx);
        cudaFuncSetAttribute(dec::gemm_decode_kernel<4, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, mx);
        cudaFuncSetAttribute(dec::gemm_decode_kernel<8, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, mx);
      }
      if (cudaGetLastError() != cudaSuccess) return HBL_ERR_CUDA;
    }
  }
  if (!d.supported) return HBL_ERR_UNSUPPORTED;
  *out = &d;
  return HBL_OK;
}

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
inline bool is_pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }
inline int ilog2(int x) { int r = 0; while ((1 << r) < x) ++r; return r; }
inline bool misaligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) != 0; }
inline int launch_status() { return cudaGetLastError() == cudaSuccess ? HBL_OK : HBL_ERR_CUDA; }

struct WsLayout {
  size_t codes, scales, csum, dacc, total;
};

WsLayout ws_layout(int M, int K, int N) {
  WsLayout L;
  size_t off = 0;
  L.codes = off; off = align_up(off + (size_t)M * K, 256);
  L.scales = off; off = align_up(off + (size_t)M * 4, 256);
  L.csum = off; off = align_up(off + (size_t)M * 4, 256);
  L.dacc = off; off = align_up(off + (size_t)M * N * 4, 256);
  L.total = off;
  return L;
}

int check_weight_shape(int N, int K) {
  if (N < 16 || N % 16 != 0) return HBL_ERR_SHAPE;
  if (K < kKBlock || K % kKBlock != 0) return HBL_ERR_SHAPE;
  if ((long long)N * K >= (1ll << 31)) return HBL_ERR_SHAPE;
  return HBL_OK;
}

int check_act_shape(int M, int K, int use_hadamard) {
  if (M < 0) return HBL_ERR_SHAPE;
  if (use_hadamard) {
    if (!is_pow2(K) || K < 256 || K > 32768) return HBL_ERR_SHAPE;
  } else {
    if (K < kKBlock || K % kKBlock != 0 || K > 65536) return HBL_ERR_SHAPE;
  }
  if ((long long)M * K >= (1ll << 40)) return HBL_ERR_SHAPE;
  return HBL_OK;
}

#ifndef HBL_USE_PDL
#define HBL_USE_PDL 1
#endif
constexpr bool kUsePdl = HBL_USE_PDL != 0;

// Launch with programmatic stream serialization: the kernel may start while
// the previous kernel in the stream drains; it must execute griddepcontrol.wait
// before touching anything that kernel writes.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = kUsePdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// Raise a kernel's dynamic shared memory limit once per device (needed above 48 KB).
// The limit recorded per (device, kernel) only ever grows.
template <typename F>
void ensure_smem_attr(F* func, size_t bytes) {
  if (bytes <= 48 * 1024) return;
  struct Entry { int dev; const void* fn; size_t bytes; };
  static std::mutex mu;
  static std::vector<Entry> done;
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lk(mu);
  for (auto& e : done) {
    if (e.dev == dev && e.fn == (const void*)func) {
      if (e.bytes >= bytes) return;
      cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
      e.bytes = bytes;
      return;
    }
  }
  cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  done.push_back(Entry{dev, (const void*)func, bytes});
}

// Arguments of one Hadamard(+quantise) launch.
struct FwhtArgs {
  const void* X;        // bf16 or fp32 rows
  int M;
  const float* gain;    // RMSNorm gain (LN only), may be null
  int8_t* codes;
  float* scales;
  int32_t* csum;
  float* Xr;            // fp32 output (kModeF32)
};

template <int LOG_K, int G, int MODE, bool IN_F32, bool LN>
void launch_fwht(const FwhtArgs& a, cudaStream_t s) {
  using C = FwhtCfg<LOG_K, G>;
  const int grid = (a.M + C::TPC - 1) / C::TPC;
  ensure_smem_attr(fwht_quant_kernel<LOG_K, G, MODE, IN_F32, LN>, C::SMEM);
  ProfScope ps("fwht_quant", s);
  launch_pdl(fwht_quant_kernel<LOG_K, G, MODE, IN_F32, LN>, dim3(grid), dim3(C::THREADS), C::SMEM, s, a.X, a.M,
             a.gain, a.codes, a.scales, a.csum, a.Xr);
}

constexpr int kLatencyTokens = 64;

// Few tokens: more threads per token for latency; many tokens: 32-128 values
// per thread for throughput. For K = 2048, 4096 and 8192 the few-token
// configuration is 256 threads per token (E = K/256), the same split and
// summation order as the fused decode kernel, so both produce the same bits.
template <int MODE, bool IN_F32 = false, bool LN = false>
int dispatch_fwht(const FwhtArgs& a, int K, cudaStream_t s) {
  if (a.M <= kLatencyTokens) {
    switch (ilog2(K)) {
      case 10: launch_fwht<10, 3, MODE, IN_F32, LN>(a, s); return launch_status();
      case 11: launch_fwht<11, 3, MODE, IN_F32, LN>(a, s); return launch_status();
      case 12: launch_fwht<12, 4, MODE, IN_F32, LN>(a, s); return launch_status();
      case 13: launch_fwht<13, 5, MODE, IN_F32, LN>(a, s); return launch_status();
      case 14: launch_fwht<14, 4, MODE, IN_F32, LN>(a, s); return launch_status();
      default: break;
    }
  }
  switch (ilog2(K)) {
    case 8: launch_fwht<8, 4, MODE, IN_F32, LN>(a, s); break;
    case 9: launch_fwht<9, 5, MODE, IN_F32, LN>(a, s); break;
    case 10: launch_fwht<10, 5, MODE, IN_F32, LN>(a, s); break;
    case 11: launch_fwht<11, 6, MODE, IN_F32, LN>(a, s); break;
    case 12: launch_fwht<12, 6, MODE, IN_F32, LN>(a, s); break;
    case 13: launch_fwht<13, 7, MODE, IN_F32, LN>(a, s); break;
    case 14: launch_fwht<14, 7, MODE, IN_F32, LN>(a, s); break;
    case 15: launch_fwht<15, 5, MODE, IN_F32, LN>(a, s); break;
    default: return HBL_ERR_SHAPE;
  }
  return launch_status();
}

template <int MODE, bool LN>
int dispatch_rows(const uint16_t* X, int M, int K, const float* gain, int8_t* codes, float* scales,
                  int32_t* csum, cudaStream_t s) {
  auto blocks = [](int T) { return (T + 31) / 32 * 32; };
  ProfScope ps("quant_rows", s);
  // K = 2048, 4096, 8192: 256 threads with K/256 values each, the split of the fused decode kernel
  if (K <= 2048)
    launch_pdl(quant_rows_kernel<8, MODE, LN>, dim3(M), dim3(blocks(K / 8)), 0, s, X, M, K, gain, codes, scales,
               csum);
  else if (K <= 4096)
    launch_pdl(quant_rows_kernel<16, MODE, LN>, dim3(M), dim3(blocks(K / 16)), 0, s, X, M, K, gain, codes, scales,
               csum);
  else if (K <= 8192)
    launch_pdl(quant_rows_kernel<32, MODE, LN>, dim3(M), dim3(blocks(K / 32)), 0, s, X, M, K, gain, codes, scales,
               csum);
  else if (K <= 16384)
    launch_pdl(quant_rows_kernel<16, MODE, LN>, dim3(M), dim3(blocks(K / 16)), 0, s, X, M, K, gain, codes, scales,
               csum);
  else if (K <= 32768)
    launch_pdl(quant_rows_kernel<32, MODE, LN>, dim3(M), dim3(blocks(K / 32)), 0, s, X, M, K, gain, codes, scales,
               csum);
  else
    launch_pdl(quant_rows_kernel<64, MODE, LN>, dim3(M), dim3(blocks(K / 64)), 0, s, X, M, K, gain, codes, scales,
               csum);
  return launch_status();
}

// Optional RMSNorm (ln), optional Hadamard, then the per-token quantiser.
int run_quantize(const uint16_t* X, int M, int K, int act_bits, int use_hadamard, int8_t* codes,
                 float* scales, int32_t* csum, cudaStream_t s, bool ln = false, const float* gain = nullptr) {
  const FwhtArgs a{X, M, gain, codes, scales, csum, nullptr};
  if (use_hadamard) {
    if (ln)
      return act_bits == 4 ? dispatch_fwht<kModeInt4, false, true>(a, K, s)
                           : dispatch_fwht<kModeInt8, false, true>(a, K, s);
    return act_bits == 4 ? dispatch_fwht<kModeInt4>(a, K, s) : dispatch_fwht<kModeInt8>(a, K, s);
  }
  if (ln)
    return act_bits == 4 ? dispatch_rows<kModeInt4, true>(X, M, K, gain, codes, scales, csum, s)
                         : dispatch_rows<kModeInt8, true>(X, M, K, gain, codes, scales, csum, s);
  return act_bits == 4 ? dispatch_rows<kModeInt4, false>(X, M, K, nullptr, codes, scales, csum, s)
                       : dispatch_rows<kModeInt8, false>(X, M, K, nullptr, codes, scales, csum, s);
}

// D = sum c*u over K. Chooses the token tile and a split of K so that the grid
// covers the SMs at least twice; split partials are added atomically into a
// zeroed D.
int run_gemm(const int8_t* codes, int M, int K, int N, const uint8_t* Wpk, int32_t* D, int sm_count,
             cudaStream_t s) {
  const int nblk = K / kKBlock;
  const int TN = M <= 8 ? 1 : (M <= 16 ? 2 : (M <= 32 ? 4 : 8));
  const int MT = 8 * TN;
  const int gx = (N + kMmaRowsPerCta - 1) / kMmaRowsPerCta;
  const int gy = (M + MT - 1) / MT;
  const long long base = (long long)gx * gy;
  int splits = (int)((2LL * sm_count + base - 1) / base);
  if (splits > nblk) splits = nblk;
  if (splits < 1) splits = 1;
  const int kps = (nblk + splits - 1) / splits;
  splits = (nblk + kps - 1) / kps;
  const int atomic = splits > 1;
  if (atomic) {
    ProfScope pm("memset_acc", s);
    if (cudaMemsetAsync(D, 0, (size_t)M * N * 4, s) != cudaSuccess) return HBL_ERR_CUDA;
  }
  dim3 grid(gx, gy, splits);
  ProfScope ps("gemm_mma", s);
  const uint4* w = reinterpret_cast<const uint4*>(Wpk);
  switch (TN) {
    case 1: gemm_mma_kernel<1><<<grid, 128, 0, s>>>(codes, M, K, N, w, kps, D, atomic); break;
    case 2: gemm_mma_kernel<2><<<grid, 128, 0, s>>>(codes, M, K, N, w, kps, D, atomic); break;
    case 4: gemm_mma_kernel<4><<<grid, 128, 0, s>>>(codes, M, K, N, w, kps, D, atomic); break;
    default: gemm_mma_kernel<8><<<grid, 128, 0, s>>>(codes, M, K, N, w, kps, D, atomic); break;
  }
  return launch_status();
}

// ---------------------------------------------------------------------------
// tcgen05 path: tensor maps and launch
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Packed weights viewed as [K/256 blocks][N rows][64 B] (block stride 64 B, row
// stride K/4 B): one box of [8 blocks][box_rows rows][64 B] lands as eight
// consecutive [box_rows][64 B] tiles (the decode kernels' unit layout) in one
// TMA copy.
bool make_map_w_blocks(CUtensorMap* map, const void* Wpk, int N, int K, int box_rows = 16) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {64, (cuuint64_t)N, (cuuint64_t)K / 256};
  cuuint64_t strides[2] = {(cuuint64_t)K / 4, 64};
  cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 8};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(Wpk), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 2-D uint8 tensor map: rows x cols bytes, row stride `stride` bytes, box box_cols x box_rows,
// swizzle_bytes 0 (none), 64 or 128.
bool make_map_u8(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows, uint64_t stride,
                 uint32_t box_cols, uint32_t box_rows, int swizzle_bytes) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {stride};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swizzle_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                       : (swizzle_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_NONE),
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 0 auto, 1 warp-level mma.sync, 2 tcgen05 persistent (128 x 128 tiles), 3 decode without
// clusters or streaming, 4 tcgen05 one 128 x 256 tile per CTA (the default for M >= 128),
// 5 weight-streaming decode (the default for M <= 16 where it fits), 6 as 0 (the forward
// takes the fused single-kernel decode wherever it fits; 0 does the same).
// Every entry point reads it once and passes the value down, so one call never
// mixes two settings.
std::atomic<int> g_gemm_path{0};


// Persistent tcgen05 kernel (one CTA per SM, 128 x 128 tiles, double-buffered accumulator).
int run_gemm_tc2(const int8_t* codes, int M, int K, int N, const uint8_t* Wpk, const int32_t* csum,
                 const float* scales, const float* alpha, uint16_t* Y, int32_t* acc, int sm_count,
                 cudaStream_t s) {
  CUtensorMap mc, mw;
  if (!make_map_u8(&mc, codes, (uint64_t)K, (uint64_t)M, (uint64_t)K, 128, tc2::kToks, 128)) return HBL_ERR_CUDA;
  if (!make_map_u8(&mw, Wpk, (uint64_t)K / 4, (uint64_t)N, (uint64_t)K / 4, kKBlock / 4, tc2::kRows, 64))
    return HBL_ERR_CUDA;
  const int tiles = ((N + tc2::kRows - 1) / tc2::kRows) * ((M + tc2::kToks - 1) / tc2::kToks);
  const dim3 grid(tiles < sm_count ? tiles : sm_count);
  ProfScope ps("gemm_tc", s);
  if (Y) {
    ensure_smem_attr(tc2::gemm_tc2_kernel<true>, tc2::kSmemBytes);
    tc2::gemm_tc2_kernel<true><<<grid, tc2::kThreads, tc2::kSmemBytes, s>>>(mc, mw, M, K, N, csum, scales, alpha,
                                                                            Y, nullptr);
  } else {
    ensure_smem_attr(tc2::gemm_tc2_kernel<false>, tc2::kSmemBytes);
    tc2::gemm_tc2_kernel<false><<<grid, tc2::kThreads, tc2::kSmemBytes, s>>>(mc, mw, M, K, N, csum, nullptr,
                                                                             nullptr, nullptr, acc);
  }
  return launch_status();
}

// One-tile-per-CTA tcgen05 GEMM with 128 x 256 tiles (measured on B200 over
// prefill shapes: 256-token tiles beat 192 and 128 as the tile of a full wave,
// since a wider tile re-reads the weights less). When the tiles leave the last
// wave of CTAs at most half full, that wave's tiles are split into 128-token
// halves (twice the CTAs, each half as long), which shortens the wave instead
// of leaving SMs idle. bf16 output (Y != nullptr) or int32 output (acc).
int run_gemm_tc(const int8_t* codes, int M, int K, int N, const uint8_t* Wpk, const int32_t* csum,
                const float* scales, const float* alpha, uint16_t* Y, int32_t* acc, int sm_count, cudaStream_t s) {
  CUtensorMap mc, mch, mw;
  if (!make_map_u8(&mc, codes, (uint64_t)K, (uint64_t)M, (uint64_t)K, 128, (uint32_t)tc::kToks, 128))
    return HBL_ERR_CUDA;
  if (!make_map_u8(&mch, codes, (uint64_t)K, (uint64_t)M, (uint64_t)K, 128, (uint32_t)tc::kToks / 2, 128))
    return HBL_ERR_CUDA;
  if (!make_map_u8(&mw, Wpk, (uint64_t)K / 4, (uint64_t)N, (uint64_t)K / 4, kKBlock / 4, tc::kRows, 64))
    return HBL_ERR_CUDA;
  const int tiles = ((N + tc::kRows - 1) / tc::kRows) * ((M + tc::kToks - 1) / tc::kToks);
  const int tail = sm_count > 0 ? tiles % sm_count : 0;
  const int full = (tail > 0 && 2 * tail <= sm_count) ? tiles - tail : tiles;
  const dim3 grid((unsigned)(full + 2 * (tiles - full)));
  ProfScope ps("gemm_tc", s);
  if (Y) {
    ensure_smem_attr(tc::gemm_tc_kernel<true>, tc::kSmemBytes);
    tc::gemm_tc_kernel<true><<<grid, tc::kThreads, tc::kSmemBytes, s>>>(mc, mch, mw, M, K, N, full, csum, scales,
                                                                         alpha, Y, nullptr);
  } else {
    ensure_smem_attr(tc::gemm_tc_kernel<false>, tc::kSmemBytes);
    tc::gemm_tc_kernel<false><<<grid, tc::kThreads, tc::kSmemBytes, s>>>(mc, mch, mw, M, K, N, full, csum, nullptr,
                                                                          nullptr, nullptr, acc);
  }
  return launch_status();
}

// 3-D uint8 tensor map: dims {d0, d1, d2} bytes (d0 contiguous), byte strides {s1, s2}, box {b0, b1, b2}.
bool make_map_u8_3d(CUtensorMap* map, const void* base, const uint64_t (&dims)[3], const uint64_t (&strides)[2],
                    const uint32_t (&box)[3], int swizzle_bytes) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t d[3] = {dims[0], dims[1], dims[2]};
  cuuint64_t st[2] = {strides[0], strides[1]};
  cuuint32_t bx[3] = {box[0], box[1], box[2]};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), d, st, bx, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swizzle_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                       : (swizzle_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_NONE),
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool decode_path_fits(int M, int K) {
  return M <= kLatencyTokens && dec::smem_bytes(K, 8) <= 200 * 1024;
}

enum class GemmKind { Decode, Mma, Tc, Tc2 };

// Which GEMM kernel runs (after the quantiser). By size, from timings on B200
// over M in 1..4096 and K, N in 2048..16384:
//  * 1..16 tokens stream the weights (decode kernels);
//  * up to 32 tokens, and with N < 8192 up to 255 tokens (N <= 2048: up to
//    1023), the split-K warp-level kernel: it keeps every SM busy where the
//    tensor-core kernels would have few 128-row tiles;
//  * K >= 8192 with at least 256 tiles of 128 x 128: the tcgen05 kernel with
//    one 128 x 256 tile per CTA (half the weight re-reads of 128-token tiles);
//  * otherwise the persistent tcgen05 kernel (128 x 128 tiles, accumulator
//    double-buffered so the epilogue overlaps the next tile).
GemmKind choose_gemm(int M, int K, int N, int path) {
  switch (path) {
    case 1: return GemmKind::Mma;
    case 2: return GemmKind::Tc2;
    case 4: return GemmKind::Tc;
    default: break;
  }
  if (M <= 16 && decode_path_fits(M, K)) return GemmKind::Decode;
  if (M <= 32) return GemmKind::Mma;
  const long long tiles = (long long)((N + 127) / 128) * ((M + 127) / 128);
  if (K >= 8192 && tiles >= 256) return GemmKind::Tc;
  if (N >= 8192) return GemmKind::Tc2;
  if (M < 256 || (N <= 2048 && M < 1024)) return GemmKind::Mma;
  return GemmKind::Tc2;
}

#ifndef HBL_DECODE_MAX_CLUSTER
#define HBL_DECODE_MAX_CLUSTER 8
#endif
constexpr int kDecodeMaxCluster = HBL_DECODE_MAX_CLUSTER;

// Cluster K-split decode kernel: cluster size C (K slice KC = K / C) and shared memory.
bool decode2_config(int M, int K, int* C_out, int* KC_out, size_t* smem_out) {
  // measured on B200: below 9 tokens the one-CTA-per-16-rows kernel is faster
  if (M > kLatencyTokens || M <= 8 || K < 512) return false;
  const int MT = 8 * (M <= 8 ? 1 : (M <= 16 ? 2 : (M <= 32 ? 4 : 8)));
  for (int C = kDecodeMaxCluster; C >= 1; C >>= 1) {
    if (K % C) continue;
    const int KC = K / C;
    if (KC % 512) continue;
    const size_t sm = dec2::smem_bytes(KC, MT);
    if (sm <= 200 * 1024) {
      *C_out = C;
      *KC_out = KC;
      *smem_out = sm;
      return true;
    }
  }
  return false;
}

int run_gemm_decode2(const int8_t* codes, int M, int K, int N, const uint8_t* Wpk, const int32_t* csum,
                     const float* scales, const float* alpha, uint16_t* Y, int32_t* acc, cudaStream_t s) {
  int C = 0, KC = 0;
  size_t smem = 0;
  if (!decode2_config(M, K, &C, &KC, &smem)) return HBL_ERR_UNSUPPORTED;
  const int TN = M <= 8 ? 1 : (M <= 16 ? 2 : (M <= 32 ? 4 : 8));
  CUtensorMap mw, mc;
  if (!make_map_u8(&mw, Wpk, (uint64_t)K / 4, (uint64_t)N, (uint64_t)K / 4, 128, dec2::kRows, 128))
    return HBL_ERR_CUDA;
  if (!make_map_u8(&mc, codes, (uint64_t)K, (uint64_t)M, (uint64_t)K, 128, (uint32_t)(8 * TN), 128))
    return HBL_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(C, (N + dec2::kRows - 1) / dec2::kRows);
  cfg.blockDim = dim3(dec2::kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = kUsePdl ? 2 : 1;
  ProfScope ps("gemm_decode", s);
  cudaError_t e = cudaSuccess;
#define HBL_DEC2(TN_)                                                                                         \
  if (Y) {                                                                                                    \
    ensure_smem_attr(dec2::gemm_decode_cluster_kernel<TN_, true>, smem);                                      \
    e = cudaLaunchKernelEx(&cfg, dec2::gemm_decode_cluster_kernel<TN_, true>, mw, mc, csum, scales, alpha, M, K, \
                           N, KC, Y, (int32_t*)nullptr);                                                      \
  } else {                                                                                                    \
    ensure_smem_attr(dec2::gemm_decode_cluster_kernel<TN_, false>, smem);                                     \
    e = cudaLaunchKernelEx(&cfg, dec2::gemm_decode_cluster_kernel<TN_, false>, mw, mc, csum,                  \
                           (const float*)nullptr, (const float*)nullptr, M, K, N, KC, (uint16_t*)nullptr, acc); \
  }
  switch (TN) {
    case 1: HBL_DEC2(1); break;
    case 2: HBL_DEC2(2); break;
    case 4: HBL_DEC2(4); break;
    default: HBL_DEC2(8); break;
  }
#undef HBL_DEC2
  return e == cudaSuccess ? launch_status() : HBL_ERR_CUDA;
}

// Weight-streaming decode kernel: M <= 16, K % 2048 == 0, at most 8 row groups per CTA.
bool stream_fits(int M, int K, int N, int sm_count) {
  if (M < 1 || M > 16 || K % strm::kChunk != 0) return false;
  const int groups = N / strm::kGroupRows;
  const int G = groups < sm_count ? groups : sm_count;
  return G > 0 && groups <= strm::kMaxGroups * G;
}

// -1: the blocked weight view could not be encoded; the caller takes another decode kernel.
// reserve: SMs left to the kernel before it in the stream (the quantiser's one
// CTA per token), so that every CTA of this grid starts its weight prefetch at
// once instead of a few starting only after the quantiser's CTAs exit. Taken
// only where it leaves the largest number of row groups per CTA unchanged
// (measured on B200: M=1, K=N=16384 25.4 -> 24.0 us per forward; M=16,
// K=N=16384, where it would raise 7 groups per CTA to 8, 28.3 -> 30.7 us).
int run_gemm_stream(const int8_t* codes, int M, int K, int N, const uint8_t* Wpk, const int32_t* csum,
                    const float* scales, const float* alpha, uint16_t* Y, int32_t* acc, int sm_count,
                    cudaStream_t s, int reserve = 0) {
  const int TN = M <= 8 ? 1 : 2;
  CUtensorMap mw2, mw1, mc;
  if (!make_map_w_blocks(&mw2, Wpk, N, K, 32) || !make_map_w_blocks(&mw1, Wpk, N, K, 16)) return -1;
  // codes as [K/128 column tiles][M rows][128 B]; one box = one chunk of 2048 k
  if (!make_map_u8_3d(&mc, codes, {128, (uint64_t)M, (uint64_t)K / 128}, {(uint64_t)K, 128},
                      {128, (uint32_t)(8 * TN), (uint32_t)(strm::kChunk / 128)}, 128))
    return -1;
  const int groups = N / strm::kGroupRows;
  const int full_max = (groups + sm_count - 1) / sm_count;
  const bool take = reserve > 0 && reserve < sm_count &&
                    (groups + (sm_count - reserve) - 1) / (sm_count - reserve) == full_max;
  const int sms = take ? sm_count - reserve : sm_count;
  const dim3 grid(groups < sms ? groups : sms);
  ProfScope ps("gemm_decode", s);
  cudaError_t e;
#define HBL_STRM(TN_)                                                                                          \
  {                                                                                                            \
    const size_t sm = strm::Layout<8 * TN_>::kBytes;                                                           \
    if (Y) {                                                                                                   \
      ensure_smem_attr(strm::gemm_stream_kernel<TN_, true>, sm);                                               \
      e = launch_pdl(strm::gemm_stream_kernel<TN_, true>, grid, dim3(strm::kThreads), sm, s, mw2, mw1, mc,     \
                     csum, scales, alpha, M, K, N, Y, (int32_t*)nullptr);                                            \
    } else {                                                                                                   \
      ensure_smem_attr(strm::gemm_stream_kernel<TN_, false>, sm);                                              \
      e = launch_pdl(strm::gemm_stream_kernel<TN_, false>, grid, dim3(strm::kThreads), sm, s, mw2, mw1, mc,    \
                     csum, (const float*)nullptr, (const float*)nullptr, M, K, N, (uint16_t*)nullptr, acc);          \
    }                                                                                                          \
  }
  if (TN == 1) HBL_STRM(1) else HBL_STRM(2)
#undef HBL_STRM
  return e == cudaSuccess ? launch_status() : HBL_ERR_CUDA;
}

int run_gemm_decode(const int8_t* codes, int M, int K, int N, const uint8_t* Wpk, const int32_t* csum,
                    const float* scales, const float* alpha, uint16_t* Y, int32_t* acc, cudaStream_t s,
                    int sm_count, int path, int reserve = 0) {
  if ((path == 0 || path == 5 || path == 6) && stream_fits(M, K, N, sm_count)) {
    const int st = run_gemm_stream(codes, M, K, N, Wpk, csum, scales, alpha, Y, acc, sm_count, s, reserve);
    if (st >= 0) return st;
  }
  {
    int C, KC;
    size_t sm;
    if (path != 3 && decode2_config(M, K, &C, &KC, &sm))
      return run_gemm_decode2(codes, M, K, N, Wpk, csum, scales, alpha, Y, acc, s);
  }
  const int TN = M <= 8 ? 1 : (M <= 16 ? 2 : (M <= 32 ? 4 : 8));
  const dim3 grid((N + dec::kRows - 1) / dec::kRows);
  const size_t smem = dec::smem_bytes(K, TN);
  ProfScope ps("gemm_decode", s);
  cudaError_t e;
#define HBL_DEC(TN_)                                                                                           \
  e = Y ? launch_pdl(dec::gemm_decode_kernel<TN_, true>, grid, dim3(dec::kThreads), smem, s, codes, csum, scales, \
                     alpha, M, K, N, Wpk, Y, (int32_t*)nullptr)                                                 \
        : launch_pdl(dec::gemm_decode_kernel<TN_, false>, grid, dim3(dec::kThreads), smem, s, codes, csum,       \
                     (const float*)nullptr, (const float*)nullptr, M, K, N, Wpk, (uint16_t*)nullptr, acc)
  switch (TN) {
    case 1: HBL_DEC(1); break;
    case 2: HBL_DEC(2); break;
    case 4: HBL_DEC(4); break;
    default: HBL_DEC(8); break;
  }
#undef HBL_DEC
  return e == cudaSuccess ? launch_status() : HBL_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// Fused single-kernel decode forward (1..16 tokens, K in {2048, 4096, 8192}).
// ---------------------------------------------------------------------------
constexpr int kFusedNotApplicable = -1;
#ifndef HBL_FUSED_L2_CLUSTER
#define HBL_FUSED_L2_CLUSTER 16
#endif
constexpr int kFusedL2Cluster = HBL_FUSED_L2_CLUSTER;   // smallest cluster exchanging rows through L2

// Preferred cluster size of the fused decode kernel: one token row per CTA,
// i.e. M rounded up to a power of two (16-CTA clusters are non-portable and
// opted into at launch). Measured on B200 against two rows per CTA in half as
// many CTAs, it is faster at every token count (M=16: 9.9 -> 9.2 us). Where
// clusters of that size cannot be scheduled, or hold too few CTAs for the
// row groups, launch_fused halves it (each CTA then transforms ceil(M / size)
// rows, at most two).
int fused_cluster_size(int M) {
  int cs = 1;
  while (cs < M) cs <<= 1;
  return cs;
}

template <int LOG_K, int TN>
int launch_fused(const CUtensorMap& mw, const uint16_t* X, int M, int N, const float* gain, const float* alpha,
                 int flags, uint16_t* Y, uint8_t* xcodes, uint8_t* xmeta, int sm_count, cudaStream_t s) {
  auto* kern = fdec::fused_decode_kernel<LOG_K, TN>;
  const size_t smem = fdec::Layout<LOG_K, 8 * TN>::kBytes;
  ensure_smem_attr(kern, smem);
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.blockDim = dim3(fdec::kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = kUsePdl ? 2 : 1;
  // clusters of CS CTAs that fit at once (cached per device, kernel and cluster size)
  struct Entry { int dev; const void* fn; int cs; int clusters; };
  static std::mutex mu;
  static std::vector<Entry> known;
  int dev = 0;
  cudaGetDevice(&dev);
  auto clusters_of = [&](int CS) {
    std::lock_guard<std::mutex> lk(mu);
    for (auto& e : known)
      if (e.dev == dev && e.fn == (const void*)kern && e.cs == CS) return e.clusters;
    // clusters above 8 CTAs are opt-in (once per device and kernel, before the first launch)
    if (CS > 8) (void)cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    attr[0].val.clusterDim.x = (unsigned)CS;
    cfg.gridDim = dim3((unsigned)(sm_count / CS * CS));
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg) != cudaSuccess) {
      (void)cudaGetLastError();
      clusters = 0;
    }
    known.push_back(Entry{dev, (const void*)kern, CS, clusters});
    return clusters;
  };
  const int groups = N / fdec::kGroupRows;
  int CS = fused_cluster_size(M), grid = 0;
  for (;; CS /= 2) {
    if (CS * fdec::kRowBatch < M) return kFusedNotApplicable;   // at most two rows per CTA
    grid = clusters_of(CS) * CS;
    if (grid > sm_count / CS * CS) grid = sm_count / CS * CS;
    if (grid >= CS && groups <= fdec::kMaxGroups * grid) break;
    if (CS == 1) return kFusedNotApplicable;
  }
  attr[0].val.clusterDim.x = (unsigned)CS;
  cfg.gridDim = dim3((unsigned)grid);
  // rows exchanged through L2 in 16-CTA clusters (measured on B200, M=16:
  // 8.7 -> 7.1 us), pushed through distributed shared memory in smaller ones
  // (M=4: 5.0 us pushed, 5.4 us through L2)
  if (CS >= kFusedL2Cluster) flags |= 16;
  ProfScope ps("fused_decode", s);
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, mw, X, M, N, gain, alpha, flags, Y, xcodes, xmeta);
  return e == cudaSuccess ? launch_status() : HBL_ERR_CUDA;
}

bool fused_fits(int M, int K, int N) {
  if (M < 1 || M > fdec::kMaxTokens || N % fdec::kGroupRows != 0) return false;
  if (K != 2048 && K != 4096 && K != 8192) return false;
  const int MT = M <= 8 ? 8 : 16;
  return (long long)MT * K <= 65536;
}

// xcodes (M x K bytes) and xmeta (M x 48 bytes), 16-byte aligned: the global
// scratch through which the CTAs of a cluster exchange their token rows.
int run_fused_decode(const uint16_t* X, int M, int K, int N, const uint8_t* Wpk, const float* wscale, int act_bits,
                     int use_hadamard, bool ln, const float* gain, uint16_t* Y, uint8_t* xcodes, uint8_t* xmeta,
                     int sm_count, cudaStream_t s) {
  // [16 rows][64 B] tiles, unswizzled (the fused kernel's conflict-free fragment
  // reads): one 3-D copy per 8 KB unit where the driver accepts the blocked
  // view, else eight 2-D copies
  CUtensorMap mw;
  int flags = (use_hadamard ? 1 : 0) | (act_bits == 8 ? 2 : 0) | (ln ? 4 : 0);
  if (make_map_w_blocks(&mw, Wpk, N, K)) {
    flags |= 8;
  } else if (!make_map_u8(&mw, Wpk, (uint64_t)K / 4, (uint64_t)N, (uint64_t)K / 4, 64, fdec::kGroupRows, 0)) {
    return HBL_ERR_CUDA;
  }
  const bool tn1 = M <= 8;
  switch (K) {
    case 2048: return tn1 ? launch_fused<11, 1>(mw, X, M, N, gain, wscale, flags, Y, xcodes, xmeta, sm_count, s)
                          : launch_fused<11, 2>(mw, X, M, N, gain, wscale, flags, Y, xcodes, xmeta, sm_count, s);
    case 4096: return tn1 ? launch_fused<12, 1>(mw, X, M, N, gain, wscale, flags, Y, xcodes, xmeta, sm_count, s)
                          : launch_fused<12, 2>(mw, X, M, N, gain, wscale, flags, Y, xcodes, xmeta, sm_count, s);
    case 8192: return tn1 ? launch_fused<13, 1>(mw, X, M, N, gain, wscale, flags, Y, xcodes, xmeta, sm_count, s)
                          : kFusedNotApplicable;
    default: return kFusedNotApplicable;
  }
}

int forward_impl(const uint16_t* X, int M, int K, int N, const uint8_t* Wpk, const float* wscale,
                 int act_bits, int use_hadamard, uint16_t* Y, void* ws, size_t ws_bytes, cudaStream_t s,
                 DeviceState* d, bool ln = false, const float* gain = nullptr) {
  const WsLayout L = ws_layout(M, K, N);
  if (!ws || ws_bytes < L.total || (reinterpret_cast<uintptr_t>(ws) & 255u)) return HBL_ERR_WORKSPACE;
  char* base = static_cast<char*>(ws);
  int8_t* codes = reinterpret_cast<int8_t*>(base + L.codes);
  float* scales = reinterpret_cast<float*>(base + L.scales);
  int32_t* csum = reinterpret_cast<int32_t*>(base + L.csum);
  int32_t* D = reinterpret_cast<int32_t*>(base + L.dacc);
  const int path = g_gemm_path.load(std::memory_order_relaxed);
  if ((path == 0 || path == 6) && fused_fits(M, K, N)) {
    // the exchange scratch: the codes region (M x K) and the accumulator
    // region (M x N x 4 >= M x 48 bytes), neither used by the fused path otherwise
    static_assert(fdec::kMetaBytes <= 4 * fdec::kGroupRows, "row metadata fits the accumulator region");
    const int fs = run_fused_decode(X, M, K, N, Wpk, wscale, act_bits, use_hadamard, ln, gain, Y,
                                    reinterpret_cast<uint8_t*>(codes), reinterpret_cast<uint8_t*>(D), d->sm_count, s);
    if (fs != kFusedNotApplicable) return fs;
  }
  int st = run_quantize(X, M, K, act_bits, use_hadamard, codes, scales, csum, s, ln, gain);
  if (st) return st;
  switch (choose_gemm(M, K, N, path)) {
    case GemmKind::Tc2: return run_gemm_tc2(codes, M, K, N, Wpk, csum, scales, wscale, Y, nullptr, d->sm_count, s);
    case GemmKind::Tc: return run_gemm_tc(codes, M, K, N, Wpk, csum, scales, wscale, Y, nullptr, d->sm_count, s);
    case GemmKind::Decode:
      // the quantiser just launched runs one CTA per token on M SMs
      return run_gemm_decode(codes, M, K, N, Wpk, csum, scales, wscale, Y, nullptr, s, d->sm_count, path, M);
    case GemmKind::Mma: break;
  }
  st = run_gemm(codes, M, K, N, Wpk, D, d->sm_count, s);
  if (st) return st;
  const long long total8 = (long long)M * N / 8;
  ProfScope ps("dequant_store", s);
  dequant_store_kernel<<<(unsigned)((total8 + 255) / 256), 256, 0, s>>>(D, csum, scales, wscale, M, N, Y);
  return launch_status();
}

int check_forward_args(const uint16_t* X, int M, int K, int N, const uint8_t* Wpk, const float* wscale,
                       int act_bits, int use_hadamard, const uint16_t* Y) {
  if (act_bits != 4 && act_bits != 8) return HBL_ERR_INVALID_ARG;
  if (use_hadamard != 0 && use_hadamard != 1) return HBL_ERR_INVALID_ARG;
  int st = check_weight_shape(N, K);
  if (st) return st;
  st = check_act_shape(M, K, use_hadamard);
  if (st) return st;
  if (M > 0 && (!X || !Wpk || !wscale || !Y)) return HBL_ERR_INVALID_ARG;
  if (misaligned16(X) || misaligned16(Y) || misaligned16(Wpk)) return HBL_ERR_INVALID_ARG;
  return HBL_OK;
}

}  // namespace
}  // namespace hbl

using namespace hbl;

extern "C" {

const char* hbl_status_string(int status) {
  switch (status) {
    case HBL_OK: return "HBL_OK";
    case HBL_ERR_INVALID_ARG: return "HBL_ERR_INVALID_ARG";
    case HBL_ERR_SHAPE: return "HBL_ERR_SHAPE";
    case HBL_ERR_CUDA: return "HBL_ERR_CUDA";
    case HBL_ERR_ALLOC: return "HBL_ERR_ALLOC";
    case HBL_ERR_TIMEOUT: return "HBL_ERR_TIMEOUT";
    case HBL_ERR_UNSUPPORTED: return "HBL_ERR_UNSUPPORTED";
    case HBL_ERR_WORKSPACE: return "HBL_ERR_WORKSPACE";
    default: return "HBL_ERR_UNKNOWN";
  }
}

int hbl_version(void) { return 1; }

size_t hbl_packed_bytes(int N, int K) {
  if (N <= 0 || K <= 0) return 0;
  return (size_t)N * (size_t)K / 4;
}

int hbl_pack_weights(const float* W, int N, int K, uint8_t* Wpk, float* wscale, hbl_stream stream) {
  int st = check_weight_shape(N, K);
  if (st) return st;
  if (!W || !Wpk || !wscale) return HBL_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(Wpk) & 15u) return HBL_ERR_INVALID_ARG;
  DeviceState* d = nullptr;
  if ((st = ensure_device(&d))) return st;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!d->abs_acc && cudaMalloc(&d->abs_acc, sizeof(AbsSumAcc)) != cudaSuccess) {
      d->abs_acc = nullptr;
      return HBL_ERR_ALLOC;
    }
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(d->abs_acc, 0, sizeof(AbsSumAcc), s) != cudaSuccess) return HBL_ERR_CUDA;
  const long long n = (long long)N * K;
  int blocks = d->sm_count * 4;
  abs_sum_kernel<<<blocks, 256, 0, s>>>(W, n, d->abs_acc);
  alpha_finalize_kernel<<<1, 32, 0, s>>>(d->abs_acc, n, wscale);
  const long long words = n / 16;
  ternary_pack_kernel<<<(unsigned)((words + 255) / 256), 256, 0, s>>>(W, N, K, wscale,
                                                                      reinterpret_cast<uint32_t*>(Wpk));
  return launch_status();
}

int hbl_unpack_weights(const uint8_t* Wpk, int N, int K, int8_t* T, hbl_stream stream) {
  int st = check_weight_shape(N, K);
  if (st) return st;
  if (!Wpk || !T) return HBL_ERR_INVALID_ARG;
  DeviceState* d = nullptr;
  if ((st = ensure_device(&d))) return st;
  const long long words = (long long)N * K / 16;
  ternary_unpack_kernel<<<(unsigned)((words + 255) / 256), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<const uint32_t*>(Wpk), N, K, T);
  return launch_status();
}

size_t hbl_workspace_bytes(int M, int K, int N) {
  if (M < 0 || K <= 0 || N <= 0) return 0;
  return ws_layout(M, K, N).total;
}

int hbl_forward_ws(const hbl_bf16* X, int M, int K, int N, const uint8_t* Wpk, const float* wscale,
                   int act_bits, int use_hadamard, hbl_bf16* Y, void* ws, size_t ws_bytes, hbl_stream stream) {
  int st = check_forward_args(X, M, K, N, Wpk, wscale, act_bits, use_hadamard, Y);
  if (st || M == 0) return st;
  DeviceState* d = nullptr;
  if ((st = ensure_device(&d))) return st;
  return forward_impl(X, M, K, N, Wpk, wscale, act_bits, use_hadamard, Y, ws, ws_bytes,
                      reinterpret_cast<cudaStream_t>(stream), d);
}

int hbl_forward(const hbl_bf16* X, int M, int K, int N, const uint8_t* Wpk, const float* wscale, int act_bits,
                int use_hadamard, hbl_bf16* Y, hbl_stream stream) {
  int st = check_forward_args(X, M, K, N, Wpk, wscale, act_bits, use_hadamard, Y);
  if (st || M == 0) return st;
  DeviceState* d = nullptr;
  if ((st = ensure_device(&d))) return st;
  const size_t need = ws_layout(M, K, N).total;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (d->ws_bytes < need) {
      if (d->ws) {
        cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
        cudaFree(d->ws);
      }
      d->ws = nullptr;
      d->ws_bytes = 0;
      if (cudaMalloc(&d->ws, need) != cudaSuccess) return HBL_ERR_ALLOC;
      d->ws_bytes = need;
    }
  }
  return forward_impl(X, M, K, N, Wpk, wscale, act_bits, use_hadamard, Y, d->ws, d->ws_bytes,
                      reinterpret_cast<cudaStream_t>(stream), d);
}

int hbl_hadamard_f32(const hbl_bf16* X, int M, int K, float* Xr, hbl_stream stream) {
  int st = check_act_shape(M, K, 1);
  if (st || M == 0) return st;
  if (!X || !Xr) return HBL_ERR_INVALID_ARG;
  if (misaligned16(X) || misaligned16(Xr)) return HBL_ERR_INVALID_ARG;
  DeviceState* d = nullptr;
  if ((st = ensure_device(&d))) return st;
  return dispatch_fwht<kModeF32>(FwhtArgs{X, M, nullptr, nullptr, nullptr, nullptr, Xr}, K,
                                 reinterpret_cast<cudaStream_t>(stream));
}

int hbl_quantize(const hbl_bf16* X, int M, int K, int act_bits, int use_hadamard, int8_t* codes, float* scales,
                 int32_t* csum, hbl_stream stream) {
  if (act_bits != 4 && act_bits != 8) return HBL_ERR_INVALID_ARG;
  if (use_hadamard != 0 && use_hadamard != 1) return HBL_ERR_INVALID_ARG;
  int st = check_act_shape(M, K, use_hadamard);
  if (st || M == 0) return st;
  if (!X || !codes || !scales) return HBL_ERR_INVALID_ARG;
  if (misaligned16(X) || misaligned16(codes)) return HBL_ERR_INVALID_ARG;
  DeviceState* d = nullptr;
  if ((st = ensure_device(&d))) return st;
  return run_quantize(X, M, K, act_bits, use_hadamard, codes, scales, csum, reinterpret_cast<cudaStream_t>(stream));
}

int hbl_gemm_codes(const int8_t* codes, int M, int K, int N, const uint8_t* Wpk, int32_t* acc, hbl_stream stream) {
  int st = check_weight_shape(N, K);
  if (st) return st;
  if (M < 0) return HBL_ERR_SHAPE;
  if (M == 0) return HBL_OK;
  if (!codes || !Wpk || !acc) return HBL_ERR_INVALID_ARG;
  if (misaligned16(codes) || misaligned16(Wpk) || misaligned16(acc)) return HBL_ERR_INVALID_ARG;
  DeviceState* d = nullptr;
  if ((st = ensure_device(&d))) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // row sums go into the first M entries of a small library scratch
  int32_t* csum = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    const size_t need = align_up((size_t)M * 4, 256);
    if (d->ws_bytes < need) {
      if (d->ws) { cudaStreamSynchronize(s); cudaFree(d->ws); }
      d->ws = nullptr;
      d->ws_bytes = 0;
      if (cudaMalloc(&d->ws, need) != cudaSuccess) return HBL_ERR_ALLOC;
      d->ws_bytes = need;
    }
    csum = static_cast<int32_t*>(d->ws);
  }
  code_rowsum_kernel<<<M, 256, 0, s>>>(codes, K, csum);
  if ((st = launch_status())) return st;
  const int path = g_gemm_path.load(std::memory_order_relaxed);
  switch (choose_gemm(M, K, N, path)) {
    case GemmKind::Tc2: return run_gemm_tc2(codes, M, K, N, Wpk, csum, nullptr, nullptr, nullptr, acc, d->sm_count, s);
    case GemmKind::Tc: return run_gemm_tc(codes, M, K, N, Wpk, csum, nullptr, nullptr, nullptr, acc, d->sm_count, s);
    case GemmKind::Decode:
      return run_gemm_decode(codes, M, K, N, Wpk, csum, nullptr, nullptr, nullptr, acc, s, d->sm_count, path);
    case GemmKind::Mma: break;
  }
  if ((st = run_gemm(codes, M, K, N, Wpk, acc, d->sm_count, s))) return st;
  sub_rowsum_kernel<<<(unsigned)(((long long)M * N + 255) / 256), 256, 0, s>>>(acc, csum, M, N);
  return launch_status();
}

int hbl_forward_ln_ws(const hbl_bf16* X, int M, int K, int N, const float* gain, const uint8_t* Wpk,
                      const float* wscale, int act_bits, int use_hadamard, hbl_bf16* Y, void* ws, size_t ws_bytes,
                      hbl_stream stream) {
  int st = check_forward_args(X, M, K, N, Wpk, wscale, act_bits, use_hadamard, Y);
  if (st || M == 0) return st;
  if (misaligned16(gain)) return HBL_ERR_INVALID_ARG;
  DeviceState* d = nullptr;
  if ((st = ensure_device(&d))) return st;
  return forward_impl(X, M, K, N, Wpk, wscale, act_bits, use_hadamard, Y, ws, ws_bytes,
                      reinterpret_cast<cudaStream_t>(stream), d, true, gain);
}

int hbl_quantize_ln(const hbl_bf16* X, int M, int K, const float* gain, int act_bits, int use_hadamard,
                    int8_t* codes, float* scales, int32_t* csum, hbl_stream stream) {
  if (act_bits != 4 && act_bits != 8) return HBL_ERR_INVALID_ARG;
  if (use_hadamard != 0 && use_hadamard != 1) return HBL_ERR_INVALID_ARG;
  int st = check_act_shape(M, K, use_hadamard);
  if (st || M == 0) return st;
  if (!X || !codes || !scales) return HBL_ERR_INVALID_ARG;
  if (misaligned16(X) || misaligned16(codes) || misaligned16(gain)) return HBL_ERR_INVALID_ARG;
  DeviceState* d = nullptr;
  if ((st = ensure_device(&d))) return st;
  return run_quantize(X, M, K, act_bits, use_hadamard, codes, scales, csum, reinterpret_cast<cudaStream_t>(stream),
                      true, gain);
}

int hbl_hadamard_backward_f32(const float* dXr, int M, int K, float* dX, hbl_stream stream) {
  int st = check_act_shape(M, K, 1);
  if (st || M == 0) return st;
  if (!dXr || !dX) return HBL_ERR_INVALID_ARG;
  if (misaligned16(dXr) || misaligned16(dX)) return HBL_ERR_INVALID_ARG;
  DeviceState* d = nullptr;
  if ((st = ensure_device(&d))) return st;
  return dispatch_fwht<kModeF32, true, false>(FwhtArgs{dXr, M, nullptr, nullptr, nullptr, nullptr, dX}, K,
                                              reinterpret_cast<cudaStream_t>(stream));
}

int hbl_pack_weights_rotated(const float* W, int N, int K, uint8_t* Wpk, float* wscale, float* Wrot,
                             hbl_stream stream) {
  int st = check_weight_shape(N, K);
  if (st) return st;
  if ((st = check_act_shape(N, K, 1))) return st;
  if (!W || !Wpk || !wscale || !Wrot) return HBL_ERR_INVALID_ARG;
  if (misaligned16(W) || misaligned16(Wpk) || misaligned16(Wrot)) return HBL_ERR_INVALID_ARG;
  DeviceState* d = nullptr;
  if ((st = ensure_device(&d))) return st;
  // every weight row w becomes H w (W H^T), in fp32, then the usual ternarise + pack
  st = dispatch_fwht<kModeF32, true, false>(FwhtArgs{W, N, nullptr, nullptr, nullptr, nullptr, Wrot}, K,
                                            reinterpret_cast<cudaStream_t>(stream));
  if (st) return st;
  return hbl_pack_weights(Wrot, N, K, Wpk, wscale, stream);
}

int hbl_quantize_qkv(const hbl_bf16* X, int T, int H, int d, int bits, int bos_token, uint8_t* codes,
                     float* gamma, hbl_stream stream) {
  if (T < 0 || H < 1 || (d != 64 && d != 128 && d != 256)) return HBL_ERR_SHAPE;
  if ((long long)T * H >= (1ll << 31)) return HBL_ERR_SHAPE;
  if (bits < 2 || bits > 8 || bos_token >= T) return HBL_ERR_INVALID_ARG;
  if (T == 0) return HBL_OK;
  if (!X || !codes || !gamma) return HBL_ERR_INVALID_ARG;
  if (misaligned16(X) || misaligned16(codes)) return HBL_ERR_INVALID_ARG;
  DeviceState* dev = nullptr;
  int st = ensure_device(&dev);
  if (st) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int rows = T * H;
  const int per_cta = 8 * kQkvRowsPerWarp;
  const dim3 grid((rows + per_cta - 1) / per_cta);
  ProfScope ps("qkv_quant", s);
  if (d == 64) qkv_quant_kernel<2><<<grid, 256, 0, s>>>(X, rows, H, bits, bos_token, codes, gamma);
  else if (d == 128) qkv_quant_kernel<4><<<grid, 256, 0, s>>>(X, rows, H, bits, bos_token, codes, gamma);
  else qkv_quant_kernel<8><<<grid, 256, 0, s>>>(X, rows, H, bits, bos_token, codes, gamma);
  return launch_status();
}

int hbl_set_gemm_path(int path) {
  if (path < 0 || path > 6) return HBL_ERR_INVALID_ARG;
  g_gemm_path.store(path, std::memory_order_relaxed);
  return HBL_OK;
}

int hbl_profile_enable(int enable) {
  std::lock_guard<std::mutex> lk(g_prof.mu);
  g_prof.flush();
  if (enable) g_prof.entries.clear();
  g_prof.on = enable != 0;
  return HBL_OK;
}

int hbl_profile_count(void) {
  std::lock_guard<std::mutex> lk(g_prof.mu);
  g_prof.flush();
  return (int)g_prof.entries.size();
}

int hbl_profile_get(int i, char* name, int name_len, int* launches, double* total_ms) {
  std::lock_guard<std::mutex> lk(g_prof.mu);
  g_prof.flush();
  if (i < 0 || i >= (int)g_prof.entries.size()) return HBL_ERR_INVALID_ARG;
  const auto& e = g_prof.entries[i];
  if (name && name_len > 0) {
    std::strncpy(name, e.name.c_str(), (size_t)name_len - 1);
    name[name_len - 1] = 0;
  }
  if (launches) *launches = e.launches;
  if (total_ms) *total_ms = e.ms;
  return HBL_OK;
}

int hbl_selftest_wait_timeout(int timeout_us, int* gave_up, hbl_stream stream) {
  if (timeout_us < 1 || timeout_us > 10000000) return HBL_ERR_INVALID_ARG;
  DeviceState* d = nullptr;
  int st = ensure_device(&d);
  if (st) return st;
  wait_timeout_selftest_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      (unsigned long long)timeout_us * 1000ull, gave_up);
  return launch_status();
}

int hbl_get_device_error(hbl_stream stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return HBL_ERR_CUDA;
  unsigned int word = 0;
  if (cudaMemcpyFromSymbol(&word, g_error_word, sizeof(word)) != cudaSuccess) return HBL_ERR_CUDA;
  const unsigned int zero = 0;
  if (cudaMemcpyToSymbol(g_error_word, &zero, sizeof(zero)) != cudaSuccess) return HBL_ERR_CUDA;
  if (word & (1u << HBL_ERR_TIMEOUT)) return HBL_ERR_TIMEOUT;
  if (word & (1u << HBL_ERR_INVALID_ARG)) return HBL_ERR_INVALID_ARG;
  return word ? HBL_ERR_CUDA : HBL_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free forward: the workspace lives in a fixed device array that
// is part of the library image, so this entry point never allocates.
// ---------------------------------------------------------------------------
namespace hbl {
namespace {

constexpr size_t kNoAllocBytes = (size_t)8 << 20;  // 8 MiB, held on every device that loads the library

static __device__ __align__(256) unsigned char g_noalloc_ws[kNoAllocBytes];

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of g_noalloc_ws on the current device. The host-side name of
// the array is not a device address; it is looked up once per device, with
// that device current, and cached.
int noalloc_scratch(void** out) {
  int dev = 0;
  int st = current_device(&dev);
  if (st) return st;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_ws) != cudaSuccess || p == nullptr) return HBL_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return HBL_OK;
}

}  // namespace
}  // namespace hbl

extern "C" int hbl_forward_noalloc(const hbl_bf16* X, int M, int K, int N, const uint8_t* Wpk,
                                   const float* wscale, int act_bits, int use_hadamard, hbl_bf16* Y,
                                   hbl_stream stream) {
  int st = check_forward_args(X, M, K, N, Wpk, wscale, act_bits, use_hadamard, Y);
  if (st || M == 0) return st;
  if (ws_layout(M, K, N).total > kNoAllocBytes) return HBL_ERR_WORKSPACE;
  DeviceState* d = nullptr;
  if ((st = ensure_device(&d))) return st;
  void* ws = nullptr;
  if ((st = noalloc_scratch(&ws))) return st;
  return forward_impl(X, M, K, N, Wpk, wscale, act_bits, use_hadamard, Y, ws, kNoAllocBytes,
                      reinterpret_cast<cudaStream_t>(stream), d);
}
