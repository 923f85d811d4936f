// Shared device helpers of the CSA kernels (sm_100a): bf16 / FP8 / FP4 conversions through the
// hardware cvt instructions, warp reductions, launch-error plumbing.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include <atomic>

#include "csa.h"

namespace csa {

// Device-side error word (a bounded wait gave up).  Without relocatable device code every
// translation unit that includes this header holds its own copy; each copy's reader is registered at
// library load (below), and csa_device_status() reads and clears every registered copy.
static __device__ uint32_t g_csa_device_error = 0;

typedef cudaError_t (*DeviceErrorReader)(uint32_t* out);
// Library-wide list of the units' readers (abi.cu).
void register_device_error_reader(DeviceErrorReader f);

// Read and clear this unit's device error word (host side), OR-ing it into *out.
static inline cudaError_t take_device_error_here(uint32_t* out) {
  uint32_t v = 0, zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_csa_device_error, sizeof(v));
  if (e == cudaSuccess && v) e = cudaMemcpyToSymbol(g_csa_device_error, &zero, sizeof(zero));
  *out |= v;
  return e;
}

namespace {
const bool g_device_error_reader_registered = (register_device_error_reader(&take_device_error_here), true);
}  // namespace

// ----------------------------------------------------------------------------- host-side status

void set_last_cuda_error(cudaError_t e);

inline csa_status launch_status() {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_last_cuda_error(e);
    return CSA_ERR_CUDA;
  }
  return CSA_OK;
}

#define CSA_REQUIRE(cond) \
  do {                    \
    if (!(cond)) return CSA_ERR_INVALID; \
  } while (0)

#define CSA_SUPPORTED(cond) \
  do {                      \
    if (!(cond)) return CSA_ERR_UNSUPPORTED; \
  } while (0)

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Row of logical entry i of sequence b in a cache laid out by `m` (see csa_page_map); -1 if its page id
// is outside the pool (a caller error: the entry is then skipped, never addressed).
__host__ __device__ __forceinline__ long long page_row(const csa_page_map& m, int b, long long n_max, long long i) {
  if (m.table == nullptr) return (long long)b * n_max + i;
  const int pg = m.table[(long long)b * m.width + i / m.page_size];
  if (pg < 0 || pg >= m.n_pages) return -1;
  return (long long)pg * m.page_size + i % m.page_size;
}

// Host check of a page map: NULL table, or page_size % 128 == 0 and enough pages per sequence.
inline csa_status check_page_map(const csa_page_map& m, long long n_max) {
  if (m.table == nullptr) return CSA_OK;
  if (m.page_size <= 0 || m.page_size % 128 != 0 || m.width <= 0 || m.n_pages <= 0) return CSA_ERR_UNSUPPORTED;
  if ((long long)m.width * m.page_size < n_max) return CSA_ERR_INVALID;
  return CSA_OK;
}

// Rows a contiguous or paged cache array spans (the extent of its tensor map).
inline long long cache_rows(const csa_page_map& m, int B, long long n_max) {
  return m.table ? (long long)m.n_pages * m.page_size : (long long)B * n_max;
}

// A call of the attention has window rows: bf16 rows in win_kv, or FP8 rows in win_codes.
inline bool attn_has_window(const csa_attn_args* a) {
  return a->Wn > 0 && (a->win_format == CSA_WIN_FP8 ? a->win_codes != nullptr : a->win_kv != nullptr);
}

// ----------------------------------------------------------------- programmatic dependent launch
// The step kernels are launched so that they may start while the kernel before them in the stream is
// still finishing: each does its setup that touches no global memory, then pdl_wait() (the previous
// grid has completed and its writes are visible) before its first global read.  pdl_trigger() lets the
// next kernel start launching once every CTA of this one has begun.  Launched any other way, both are
// no-ops.  Under the early-start option some reads move ahead of the wait (the indexer's key tiles
// below the newest row, attention's window tiles); every grid still waits once before it completes, so
// a grid's completion implies its predecessor's.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
// L2 prefetch of one line: issued before pdl_wait() it fills the address translation (and L2) for reads
// right after the wait; L2 is coherent, so a line the previous kernel rewrites later is read fresh.
__device__ __forceinline__ void prefetch_l2(const void* p) { asm volatile("prefetch.global.L2 [%0];" ::"l"(p)); }

inline cudaLaunchConfig_t pdl_config(dim3 grid, dim3 block, size_t smem, cudaStream_t st, cudaLaunchAttribute* attr) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cfg;
}

template <typename... KArgs, typename... Args>
inline csa_status launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                             Args... args) {
  cudaLaunchAttribute attr[1];
  const cudaLaunchConfig_t cfg = pdl_config(grid, block, smem, st, attr);
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, args...);
  if (e != cudaSuccess) {
    set_last_cuda_error(e);
    return CSA_ERR_CUDA;
  }
  return launch_status();
}

// Raise a kernel's dynamic shared-memory limit once per device (the attribute is per device); later
// calls, including those made while a stream is being captured into a CUDA graph, skip the runtime call.
// Every kernel also asks for the largest shared-memory carveout: an SM runs CTAs of one carveout at a
// time, so a kernel that needs little shared memory would otherwise hold SMs in a small-carveout setting
// and keep the CTAs of the next kernel (launched early, programmatic dependent launch) off them until
// its own CTAs have left.
inline void set_smem_once(const void* func, int bytes, std::atomic<unsigned>& done) {
  int dev = 0;
  cudaGetDevice(&dev);
  const unsigned bit = 1u << (dev & 31);
  if (done.load(std::memory_order_acquire) & bit) return;
  if (bytes > 0) cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  cudaFuncSetAttribute(func, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
  done.fetch_or(bit, std::memory_order_acq_rel);
}

// ----------------------------------------------------------------------------- number formats

__device__ __forceinline__ float bf16_bits_to_f(uint32_t b) { return __uint_as_float(b << 16); }

__device__ __forceinline__ uint32_t f_to_bf16_bits(float f) {
  __nv_bfloat16 h = __float2bfloat16_rn(f);
  return (uint32_t)(*reinterpret_cast<uint16_t*>(&h));
}

// Two floats -> packed bf16x2 (lo in the low half), round to nearest even.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// fp32 -> E4M3 byte: round to nearest even, saturate to +-448, subnormals kept (PTX cvt ... satfinite).
__device__ __forceinline__ uint32_t f32_to_e4m3(float x) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(x));
  return r & 0xFFu;
}

// E4M3 byte -> float (exact).
__device__ __forceinline__ float e4m3_to_f32(uint32_t code) {
  uint32_t h2;
  uint16_t in = (uint16_t)(code & 0xFFu);
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(in));
  return __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu)));
}

// E4M3 byte -> f16x2 with the value in both halves (exact).
__device__ __forceinline__ uint32_t e4m3_to_h2_splat(uint32_t code) {
  uint32_t h2;
  uint16_t in = (uint16_t)((code & 0xFFu) * 0x0101u);
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(in));
  return h2;
}

// fp32 -> E2M1 nibble: round to nearest even, saturate to +-6; -0 is returned as +0.
__device__ __forceinline__ uint32_t f32_to_e2m1(float x) {
  uint32_t r;
  asm("{ .reg .b8 t; cvt.rn.satfinite.e2m1x2.f32 t, %1, %2; cvt.u32.u8 %0, t; }"
      : "=r"(r) : "f"(0.0f), "f"(x));
  r &= 0xFu;
  return (r & 0x7u) ? r : 0u;
}

// One byte of two E2M1 codes -> f16x2 (low nibble -> low half), exact.
__device__ __forceinline__ uint32_t e2m1x2_to_h2(uint32_t byte) {
  uint32_t h2;
  asm("{ .reg .b8 t; cvt.u8.u32 t, %1; cvt.rn.f16x2.e2m1x2 %0, t; }" : "=r"(h2) : "r"(byte & 0xFFu));
  return h2;
}

__device__ __forceinline__ uint32_t hmul2_bits(uint32_t a, uint32_t b) {
  __half2 r = __hmul2(*reinterpret_cast<__half2*>(&a), *reinterpret_cast<__half2*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}

// E2M1 value of a code: bits s|e1 e0|m, exponent bias 1; e = 0 is the subnormal 0.5*m.
__device__ __forceinline__ float e2m1_value(uint32_t code) {
  const uint32_t e = (code >> 1) & 3u, m = code & 1u;
  const float v = e ? ldexpf(1.0f + 0.5f * (float)m, (int)e - 1) : 0.5f * (float)m;
  return (code & 8u) ? -v : v;
}

// ----------------------------------------------------------------------------- warp helpers

__device__ __forceinline__ float warp_max(float v);

// FP4 pack of one 32-element block by one warp (lane e holds element e, an fp32 copy of a bf16):
//   s = E4M3_rne_satfinite(fp32(amax / fp32(6 g))); s == 0 -> all codes 0;
//   code_e = E2M1_rne_satfinite(fp32(x_e / fp32(s g))), -0 -> +0; element 2j in the low nibble of byte j.
// Writes the 16 code bytes at codes16 and the scale byte at *scale.
__device__ __forceinline__ void pack_block_warp(float x, float g, uint8_t* codes16, uint8_t* scale) {
  const int lane = threadIdx.x & 31;
  const float amax = warp_max(fabsf(x));
  const uint32_t s_code = f32_to_e4m3(__fdiv_rn(amax, 6.0f * g));
  const float s = e4m3_to_f32(s_code);
  uint32_t code = 0;
  if (s != 0.0f) code = f32_to_e2m1(__fdiv_rn(x, __fmul_rn(s, g)));
  const uint32_t pair = code | (__shfl_down_sync(0xffffffffu, code, 1) << 4);
  // bytes 4m..4m+3 gathered on lane 8m, one 32-bit store per 8 lanes
  const uint32_t b1 = __shfl_down_sync(0xffffffffu, pair, 2);
  const uint32_t b2 = __shfl_down_sync(0xffffffffu, pair, 4);
  const uint32_t b3 = __shfl_down_sync(0xffffffffu, pair, 6);
  if ((lane & 7) == 0)
    reinterpret_cast<uint32_t*>(codes16)[lane >> 3] = (pair & 0xFFu) | ((b1 & 0xFFu) << 8) | ((b2 & 0xFFu) << 16) | ((b3 & 0xFFu) << 24);
  if (lane == 0) *scale = (uint8_t)s_code;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Order-preserving map float -> uint32 (larger float -> larger key); -0 and +0 map to the same key.
__device__ __forceinline__ uint32_t float_order_key(float f) {
  f += 0.0f;  // -0 -> +0
  uint32_t b = __float_as_uint(f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

__device__ __forceinline__ float order_key_float(uint32_t k) {
  uint32_t b = (k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k;
  return __uint_as_float(b);
}

}  // namespace csa
