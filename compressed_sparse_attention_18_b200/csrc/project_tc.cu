// The compressor's two token projections on the 5th-generation tensor cores: C = x·W_kv and Z = x·W_g
// (bf16 in, fp32 accumulators in tensor memory, bf16 out), one launch for both.
// Sources: "DeepSeek-V4.1-Flash - Pushing the Limits of KV Cache Compression", CED bullet eq.(1) (the
// entry values C and the gate logits Z are separate linear maps of the hidden state); "DeepSeek-V4:
// エージェントが実際に使える100万トークンのコンテキスト", §ハイブリッド注意, Fig. 3 (the compressor these feed).
//
// Tile: 128 tokens (MMA M) x BN channels (MMA N = 256, or 128 for narrow heads) x 64 of d_model per
// pipeline stage (4 MMAs of K = 16).  Operands arrive by TMA with the 128-byte swizzle: x rows K-major,
// W rows as stored ([d_model][d], channels contiguous), which the MMA reads through an MN-major
// descriptor, so neither operand is transposed in memory.
// Warp roles (192 threads, persistent CTAs walking tiles t = blockIdx.x, blockIdx.x + gridDim.x, ...;
// consecutive tiles share their 128 x rows so those stay in L2 while both weights stream past):
//   warp 0      TMA producer (one thread) into a STAGES-deep ring;
//   warp 1      allocates tensor memory and issues the MMAs (one thread), two accumulator buffers so a
//               tile's epilogue overlaps the next tile's main loop;
//   warps 2..5  epilogue: each warp owns the 32 tokens of its tensor-memory lane quadrant, loads 32
//               columns at a time, rounds to bf16 and stores 64 contiguous bytes per token.
// Every wait is bounded; a wait that gives up records device error 1 and the kernel leaves.
#include "csa_common.cuh"
#include "sm100.cuh"

namespace csa {

using namespace sm100;

constexpr int PJ_BM = 128, PJ_BK = 64;
constexpr int PJ_THREADS = 192;

template <int BN>
struct PjCfg {
  static constexpr int STAGES = BN == 256 ? 4 : 6;
  static constexpr int A_BYTES = PJ_BM * PJ_BK * 2;       // 16 KB
  static constexpr int B_BYTES = PJ_BK * BN * 2;          // 32 KB (BN = 256)
  static constexpr uint32_t TMEM_COLS = 2 * BN;           // two accumulator buffers
};

template <int BN>
struct PjSmem {
  alignas(1024) uint8_t a[PjCfg<BN>::STAGES][PjCfg<BN>::A_BYTES];      // [token][64 x bf16], 128-byte swizzle
  alignas(1024) uint8_t b[PjCfg<BN>::STAGES][PjCfg<BN>::B_BYTES];      // [BN/64][64 k rows][64 ch bf16]
  alignas(8) uint64_t full[PjCfg<BN>::STAGES];
  alignas(8) uint64_t empty[PjCfg<BN>::STAGES];
  alignas(8) uint64_t acc_full[2];
  alignas(8) uint64_t acc_empty[2];
  alignas(8) uint64_t done;
  uint32_t tmem_base;
  uint32_t err;
};

struct PjParams {
  uint16_t* out0;   // C [M][N]
  uint16_t* out1;   // Z [M][N]
  int M, N, K;
  int n_tiles_n;    // N / BN
  int tiles;        // ceil(M / 128) * n_tiles_n * 2
};

template <int BN>
__global__ void __launch_bounds__(PJ_THREADS, 1) project_tc_kernel(const __grid_constant__ CUtensorMap xmap,
                                                                   const __grid_constant__ CUtensorMap w0map,
                                                                   const __grid_constant__ CUtensorMap w1map,
                                                                   const PjParams P) {
  using Cfg = PjCfg<BN>;
  constexpr int ST = Cfg::STAGES;
  extern __shared__ uint8_t smem_raw[];
  PjSmem<BN>& S = *reinterpret_cast<PjSmem<BN>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    S.err = 0;
    for (int s = 0; s < ST; ++s) { mbar_init(&S.full[s], 1); mbar_init(&S.empty[s], 1); }
    for (int a = 0; a < 2; ++a) { mbar_init(&S.acc_full[a], 1); mbar_init(&S.acc_empty[a], 4); }
    mbar_init(&S.done, 1);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&xmap);
    prefetch_tensormap(&w0map);
    prefetch_tensormap(&w1map);
  }
  if (warp == 1) { tmem_alloc(&S.tmem_base, Cfg::TMEM_COLS); tmem_relinquish(); }
  pdl_trigger();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = S.tmem_base;
  const int kb_n = (P.K + PJ_BK - 1) / PJ_BK;
  const int per_m = 2 * P.n_tiles_n;
  bool ok = true;

  if (warp == 0) {
    // ------------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      pdl_wait();                       // x may be written by the previous kernel
      int it = 0, issued = 0;
      for (int t = blockIdx.x; t < P.tiles && ok; t += gridDim.x) {
        const int m = t / per_m, rest = t % per_m, z = rest / P.n_tiles_n, n = rest % P.n_tiles_n;
        const CUtensorMap* wm = z ? &w1map : &w0map;
        for (int kb = 0; kb < kb_n; ++kb, ++it) {
          const int s = it % ST, f = it / ST;
          if (f > 0 && !mbar_wait(&S.empty[s], (f - 1) & 1)) { ok = false; break; }
          mbar_arrive_expect_tx(&S.full[s], Cfg::A_BYTES + Cfg::B_BYTES);
          tma_load_2d(S.a[s], &xmap, kb * PJ_BK, m * PJ_BM, &S.full[s]);
#pragma unroll
          for (int j = 0; j < BN / 64; ++j)
            tma_load_2d(S.b[s] + j * (PJ_BK * 128), wm, n * BN + 64 * j, kb * PJ_BK, &S.full[s]);
          ++issued;
        }
      }
      if (!ok) atomicOr(&S.err, 1u);
      // drain: the copies this thread issued complete before the CTA may leave
      for (int i = max(0, issued - ST); i < issued; ++i) mbar_wait(&S.full[i % ST], (i / ST) & 1, 1u << 16);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      pdl_wait();
      const uint32_t idesc = idesc_bf16(PJ_BM, BN, 0, 1);
      int it = 0, i = 0;
      for (int t = blockIdx.x; t < P.tiles && ok; t += gridDim.x, ++i) {
        const int a = i & 1, use = i >> 1;
        if (use > 0 && !mbar_wait(&S.acc_empty[a], (use - 1) & 1)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d = tbase + (uint32_t)(a * BN);
        for (int kb = 0; kb < kb_n; ++kb, ++it) {
          const int s = it % ST;
          if (!mbar_wait(&S.full[s], (it / ST) & 1)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_addr(S.a[s]), sb = smem_addr(S.b[s]);
#pragma unroll
          for (int kk = 0; kk < PJ_BK / 16; ++kk) {
            const uint64_t ad = smem_desc(sa + kk * 32, 16, 1024, LAYOUT_SW128);
            const uint64_t bd = smem_desc(sb + kk * 2048, PJ_BK * 128, 1024, LAYOUT_SW128);
            mma_bf16_ss(d, ad, bd, idesc, (kb | kk) != 0);
          }
          mma_commit(&S.empty[s]);
        }
        if (!ok) break;
        mma_commit(&S.acc_full[a]);
      }
      mma_commit(&S.done);
      if (!ok) atomicOr(&S.err, 1u);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const uint32_t lane_off = (uint32_t)(32 * q) << 16;
    int i = 0;
    for (int t = blockIdx.x; t < P.tiles && ok; t += gridDim.x, ++i) {
      const int m = t / per_m, rest = t % per_m, z = rest / P.n_tiles_n, n = rest % P.n_tiles_n;
      const int a = i & 1, use = i >> 1;
      if (!mbar_wait(&S.acc_full[a], use & 1)) { ok = false; break; }
      tc_fence_after();
      const int row = m * PJ_BM + 32 * q + lane;
      uint16_t* dst = (z ? P.out1 : P.out0) + (size_t)row * P.N + n * BN;
      uint32_t v[32];
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        tmem_ld_x32(tbase + lane_off + (uint32_t)(a * BN + 32 * c), v);
        tmem_wait_ld_x32(v);
        if (row < P.M) {
          uint4* o = reinterpret_cast<uint4*>(dst + 32 * c);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            o[j] = make_uint4(pack_bf16x2(__uint_as_float(v[8 * j + 0]), __uint_as_float(v[8 * j + 1])),
                              pack_bf16x2(__uint_as_float(v[8 * j + 2]), __uint_as_float(v[8 * j + 3])),
                              pack_bf16x2(__uint_as_float(v[8 * j + 4]), __uint_as_float(v[8 * j + 5])),
                              pack_bf16x2(__uint_as_float(v[8 * j + 6]), __uint_as_float(v[8 * j + 7])));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.acc_empty[a]);
    }
    if (!ok && lane == 0) atomicOr(&S.err, 1u);
  }
  __syncthreads();
  if (warp == 1) {
    // every MMA this CTA issued has completed before its tensor memory is released
    mbar_wait(&S.done, 0, 1u << 20);
    tc_fence_after();
    tmem_dealloc(tbase, Cfg::TMEM_COLS);
  }
  if (S.err && threadIdx.x == 0) atomicOr(&g_csa_device_error, 1u);
}

static bool encode_2d_bf16(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint32_t box_in,
                           uint32_t box_out) {
  const cuuint64_t gdim[2] = {inner, outer};
  const cuuint64_t gstride[1] = {inner * 2};
  const cuuint32_t box[2] = {box_in, box_out};
  const cuuint32_t estr[2] = {1, 1};
  return tensor_map_encoder()(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), gdim, gstride, box,
                              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BN>
static csa_status launch_projection(const void* x, const void* W0, const void* W1, void* C, void* Z, int M, int N,
                                    int K, cudaStream_t st) {
  CUtensorMap xm, w0m, w1m;
  if (!encode_2d_bf16(&xm, x, (uint64_t)K, (uint64_t)M, PJ_BK, PJ_BM) ||
      !encode_2d_bf16(&w0m, W0, (uint64_t)N, (uint64_t)K, 64, PJ_BK) ||
      !encode_2d_bf16(&w1m, W1, (uint64_t)N, (uint64_t)K, 64, PJ_BK))
    return CSA_ERR_CUDA;
  PjParams P{};
  P.out0 = (uint16_t*)C;
  P.out1 = (uint16_t*)Z;
  P.M = M;
  P.N = N;
  P.K = K;
  P.n_tiles_n = N / BN;
  P.tiles = ((M + PJ_BM - 1) / PJ_BM) * P.n_tiles_n * 2;
  int sms = 148;
  {
    int dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  }
  const int grid = P.tiles < sms ? P.tiles : sms;
  const int smem = (int)sizeof(PjSmem<BN>) + 1024;
  static std::atomic<unsigned> attr_done{0};
  set_smem_once((const void*)project_tc_kernel<BN>, smem, attr_done);
  return launch_pdl(project_tc_kernel<BN>, dim3(grid), dim3(PJ_THREADS), smem, st, xm, w0m, w1m, P);
}

// C = x·W0, Z = x·W1 for x [M][K], W [K][N], all bf16 row-major; N % 128 == 0, K % 8 == 0, every base
// 16-byte aligned (checked by the caller).
csa_status run_projection_tc(const void* x, const void* W0, const void* W1, void* C, void* Z, long long M, int N,
                             int K, cudaStream_t st) {
  if (tensor_map_encoder() == nullptr) return CSA_ERR_UNSUPPORTED;
  if (M > 0x7fffffffLL) return CSA_ERR_UNSUPPORTED;
  if (N % 256 == 0) return launch_projection<256>(x, W0, W1, C, Z, (int)M, N, K, st);
  return launch_projection<128>(x, W0, W1, C, Z, (int)M, N, K, st);
}

}  // namespace csa
