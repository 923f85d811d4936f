// FP4 pack of compressed entries into a cache: E2M1 codes, one E4M3 scale per 32 elements, a per-tensor
// fp32 global scale, the RoPE slice copied as bf16.
// Sources: "DeepSeek-V4.1-Flash - Pushing the Limits of KV Cache Compression", §提案手法/アーキテクチャ,
// FP4 主 KV キャッシュ bullet (E2M1 main KV with E4M3 scale factors); "DeepSeek-V4: エージェントが実際に使える
// 100万トークンのコンテキスト", §ハイブリッド注意 storage paragraph (RoPE dims kept in BF16).
#include "csa_common.cuh"

namespace csa {

// One warp per cache row: lane e holds element e of the current 32-block.
//   s = E4M3(fp32(amax / fp32(6 g))); s == 0 -> zero block; code = E2M1(fp32(x / fp32(s g))).
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
  const float six_g = 6.0f * g;
  for (long long row = (long long)blockIdx.x * warps + (threadIdx.x >> 5); row < total;
       row += (long long)gridDim.x * warps) {
    const int b = (int)(row / n);
    const int j = (int)(row % n);
    const long long dst = (long long)b * n_max + (row0 ? row0[b] : 0) + j;
    const uint16_t* s_row = src + row * d;
    uint8_t* c_row = codes + dst * (d_n >> 1);
    for (int blk = 0; blk < S; ++blk) {
      const float x = bf16_bits_to_f(s_row[blk * 32 + lane]);
      const float amax = warp_max(fabsf(x));
      const uint32_t s_code = f32_to_e4m3(__fdiv_rn(amax, six_g));
      const float s = e4m3_to_f32(s_code);
      uint32_t code = 0;
      if (s != 0.0f) code = f32_to_e2m1(__fdiv_rn(x, __fmul_rn(s, g)));
      const uint32_t hi = __shfl_down_sync(0xffffffffu, code, 1);
      if ((lane & 1) == 0) c_row[blk * 16 + (lane >> 1)] = (uint8_t)(code | (hi << 4));
      if (lane == 0) scales[dst * S_pad + blk] = (uint8_t)s_code;
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
