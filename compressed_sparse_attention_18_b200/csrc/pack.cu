// FP4 pack of compressed entries into a cache: E2M1 codes, one E4M3 scale per 32 elements, a per-tensor
// fp32 global scale, the RoPE slice copied as bf16.
// Sources: "DeepSeek-V4.1-Flash - Pushing the Limits of KV Cache Compression", §提案手法/アーキテクチャ,
// FP4 主 KV キャッシュ bullet (E2M1 main KV with E4M3 scale factors); "DeepSeek-V4: エージェントが実際に使える
// 100万トークンのコンテキスト", §ハイブリッド注意 storage paragraph (RoPE dims kept in BF16).
#include "csa_common.cuh"

namespace csa {

// One warp per cache row: every element of the row is loaded first (one memory latency per row),
// then each 32-block is packed by the whole warp (lane e = element e of the block).
__global__ void __launch_bounds__(256) pack_fp4_kernel(const uint16_t* __restrict__ src, int B, int n, int d,
                                                       int d_r, float g, const int32_t* __restrict__ row0,
                                                       int n_max, uint8_t* __restrict__ codes,
                                                       uint8_t* __restrict__ scales, uint16_t* __restrict__ rope,
                                                       const csa_page_map pm) {
  const int lane = threadIdx.x & 31;
  const int warps = blockDim.x >> 5;
  const long long total = (long long)B * n;
  const int d_n = d - d_r;
  const int S = d_n >> 5;
  const int S_pad = (S + 3) & ~3;
  for (long long row = (long long)blockIdx.x * warps + (threadIdx.x >> 5); row < total;
       row += (long long)gridDim.x * warps) {
    const int b = (int)(row / n);
    const int j = (int)(row % n);
    const long long dst = page_row(pm, b, n_max, (long long)(row0 ? row0[b] : 0) + j);
    if (dst < 0) continue;                       // a page outside the pool: nothing is written
    const uint16_t* s_row = src + row * d;
    uint8_t* c_row = codes + dst * (d_n >> 1);
    for (int blk0 = 0; blk0 < S; blk0 += 16) {
      float x[16];
#pragma unroll
      for (int u = 0; u < 16; ++u) x[u] = blk0 + u < S ? bf16_bits_to_f(s_row[(blk0 + u) * 32 + lane]) : 0.0f;
#pragma unroll
      for (int u = 0; u < 16; ++u)
        if (blk0 + u < S) pack_block_warp(x[u], g, c_row + (blk0 + u) * 16, scales + dst * S_pad + blk0 + u);
    }
    if (lane < S_pad - S) scales[dst * S_pad + S + lane] = 0;
    for (int e = lane; e < d_r; e += 32) rope[dst * d_r + e] = s_row[d_n + e];
  }
}

// FP8 window pack: one warp per (row, 64-channel block) of the first d_n channels, two elements per
// lane.  scale = fp32(amax / 448) (correctly rounded fp32 division, as the format fixes); code =
// E4M3_rne_satfinite(fp32(x / scale)) with -0 -> +0; a block with amax 0 gets scale 0 and codes 0.  The
// RoPE channels are copied.  Sources: "DeepSeek-V4.1-Flash - Pushing the Limits of KV Cache Compression",
// FP4 主 KV キャッシュ bullet (the sliding-window KV stays FP8); "DeepSeek-V4: エージェントが実際に使える100万トークン
// のコンテキスト", storage paragraph (FP8 KV with BF16 RoPE dims).
constexpr int FP8_WIN_BLOCK = 64;

__global__ void __launch_bounds__(256) pack_fp8_window_kernel(const uint16_t* __restrict__ src, int B, int n, int d,
                                                              int d_r, const int32_t* __restrict__ row0, int Wn,
                                                              uint8_t* __restrict__ codes, float* __restrict__ scales,
                                                              uint16_t* __restrict__ rope) {
  const int lane = threadIdx.x & 31;
  const int warps = blockDim.x >> 5;
  const int d_n = d - d_r;
  const int nb = d_n / FP8_WIN_BLOCK, nb_pad = (nb + 3) & ~3;
  const int units = nb + 1;                        // the blocks, then the RoPE copy and the scale padding
  const long long total = (long long)B * n * units;
  for (long long u = (long long)blockIdx.x * warps + (threadIdx.x >> 5); u < total; u += (long long)gridDim.x * warps) {
    const long long row = u / units;
    const int blk = (int)(u % units);
    const int b = (int)(row / n), j = (int)(row % n);
    const long long dst = (long long)b * Wn + (row0 ? row0[b] : 0) + j;
    const uint16_t* s_row = src + row * d;
    if (blk < nb) {
      const uint32_t pair = *reinterpret_cast<const uint32_t*>(s_row + blk * FP8_WIN_BLOCK + 2 * lane);
      const float x0 = bf16_bits_to_f(pair & 0xFFFFu), x1 = bf16_bits_to_f(pair >> 16);
      const float amax = warp_max(fmaxf(fabsf(x0), fabsf(x1)));
      const float sc = __fdiv_rn(amax, 448.0f);
      uint32_t c0 = 0, c1 = 0;
      if (sc > 0.0f) {
        c0 = f32_to_e4m3(__fdiv_rn(x0, sc));
        c1 = f32_to_e4m3(__fdiv_rn(x1, sc));
        if ((c0 & 0x7Fu) == 0) c0 = 0;              // -0 -> +0
        if ((c1 & 0x7Fu) == 0) c1 = 0;
      }
      reinterpret_cast<uint16_t*>(codes + dst * d_n + blk * FP8_WIN_BLOCK)[lane] = (uint16_t)(c0 | (c1 << 8));
      if (lane == 0) scales[dst * nb_pad + blk] = sc;
    } else {
      for (int e = lane; e < d_r; e += 32) rope[dst * d_r + e] = s_row[d_n + e];
      if (lane < nb_pad - nb) scales[dst * nb_pad + nb + lane] = 0.0f;
    }
  }
}

}  // namespace csa

using namespace csa;

extern "C" csa_status csa_pack_fp8_window(const csa_fp8_window_args* a, void* stream) {
  CSA_REQUIRE(a != nullptr && a->struct_size == sizeof(csa_fp8_window_args));
  CSA_REQUIRE(a->B >= 0 && a->n >= 0 && a->d > 0 && a->d_rope >= 0 && a->d_rope <= a->d);
  CSA_REQUIRE(a->Wn >= a->n);
  CSA_SUPPORTED((a->d - a->d_rope) % FP8_WIN_BLOCK == 0 && a->d_rope % 8 == 0);
  if ((long long)a->B * a->n == 0) return CSA_OK;
  CSA_REQUIRE(a->src && a->codes && a->scales && (a->d_rope == 0 || a->rope));
  CSA_SUPPORTED(((uintptr_t)a->src & 3) == 0 && ((uintptr_t)a->codes & 1) == 0);
  const long long units = (long long)a->B * a->n * ((a->d - a->d_rope) / FP8_WIN_BLOCK + 1);
  long long blocks = (units + 7) / 8;
  if (blocks > 148 * 16) blocks = 148 * 16;
  pack_fp8_window_kernel<<<(unsigned)blocks, 256, 0, (cudaStream_t)stream>>>(
      (const uint16_t*)a->src, a->B, a->n, a->d, a->d_rope, a->row0, a->Wn, a->codes, a->scales, (uint16_t*)a->rope);
  return launch_status();
}

extern "C" csa_status csa_pack_fp4(const csa_pack_args* a, void* stream) {
  CSA_REQUIRE(a != nullptr && a->struct_size == sizeof(csa_pack_args));
  CSA_REQUIRE(a->B >= 0 && a->n >= 0 && a->d > 0 && a->d_rope >= 0 && a->d_rope <= a->d);
  CSA_REQUIRE(a->n_max >= a->n);
  CSA_SUPPORTED((a->d - a->d_rope) % 32 == 0 && a->d_rope % 8 == 0);
  if ((long long)a->B * a->n == 0) return CSA_OK;
  CSA_REQUIRE(a->src && a->codes && a->scales && (a->d_rope == 0 || a->rope));
  CSA_REQUIRE(a->global_scale > 0.0f);
  {
    const csa_status pv = check_page_map(a->pages, a->n_max);
    if (pv != CSA_OK) return pv;
  }
  const long long rows = (long long)a->B * a->n;
  const int threads = 256;
  long long blocks = (rows + 7) / 8;
  if (blocks > 148 * 16) blocks = 148 * 16;
  pack_fp4_kernel<<<(unsigned)blocks, threads, 0, (cudaStream_t)stream>>>(
      (const uint16_t*)a->src, a->B, a->n, a->d, a->d_rope, a->global_scale, a->row0, a->n_max, a->codes,
      a->scales, (uint16_t*)a->rope, a->pages);
  return launch_status();
}
