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
                                                       uint8_t* __restrict__ scales, uint16_t* __restrict__ rope) {
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
    const long long dst = (long long)b * n_max + (row0 ? row0[b] : 0) + j;
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

}  // namespace csa

using namespace csa;

extern "C" csa_status csa_pack_fp4(const csa_pack_args* a, void* stream) {
  CSA_REQUIRE(a != nullptr && a->struct_size == sizeof(csa_pack_args));
  CSA_REQUIRE(a->B >= 0 && a->n >= 0 && a->d > 0 && a->d_rope >= 0 && a->d_rope <= a->d);
  CSA_REQUIRE(a->n_max >= a->n);
  CSA_SUPPORTED((a->d - a->d_rope) % 32 == 0 && a->d_rope % 8 == 0);
  if ((long long)a->B * a->n == 0) return CSA_OK;
  CSA_REQUIRE(a->src && a->codes && a->scales && (a->d_rope == 0 || a->rope));
  CSA_REQUIRE(a->global_scale > 0.0f);
  const long long rows = (long long)a->B * a->n;
  const int threads = 256;
  long long blocks = (rows + 7) / 8;
  if (blocks > 148 * 16) blocks = 148 * 16;
  pack_fp4_kernel<<<(unsigned)blocks, threads, 0, (cudaStream_t)stream>>>(
      (const uint16_t*)a->src, a->B, a->n, a->d, a->d_rope, a->global_scale, a->row0, a->n_max, a->codes,
      a->scales, (uint16_t*)a->rope);
  return launch_status();
}
