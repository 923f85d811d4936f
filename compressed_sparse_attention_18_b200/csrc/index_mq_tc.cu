// Lightning-indexer scores for many queries per sequence (chunked prefill, speculative decode) on the
// 5th-generation tensor cores (tcgen05, block-scaled FP4), with the causal visibility mask.
// Sources: "DeepSeek-V4: エージェントが実際に使える100万トークンのコンテキスト", §ハイブリッド注意, Fig. 3 (an FP4
// multi-head ReLU indexer scores every compressed entry a query can see); "DeepSeek-V4.1-Flash - Pushing
// the Limits of KV Cache Compression", FP4 主 KV キャッシュ bullet (E2M1 values with E4M3 scales).
//
// One CTA owns 16 queries of one sequence (MMA N = 16 queries x 8 indexer heads = 128 columns) and walks
// a range of 128-key tiles (MMA M).  Per tile two kind::mxf4nvf4 MMAs (K = 64 each, UE4M3 scales per 16
// elements; an E4M3 scale of a 32-block is written for both of its 16-element halves) form exactly
//   D[key][q][h] = sum_blk sq[q][h][blk] sk[key][blk] sum_{e in blk} e2m1(q_e) e2m1(k_e)
// in fp32; the epilogue applies s = sum_h w'[q][h] max(0, D) with w' = w g_q g_k and writes s for the
// keys the query sees (r key + r - 1 <= t, key < n_c); other columns of the row are left untouched.
//
// Warp roles (320 threads):
//   warp 0      TMA producer: 128 x 64 B FP4 key tile (64-byte swizzle) + the tile's 512 B of key scales;
//   warp 1      allocates tensor memory (512 columns) and issues the copies and MMAs (one thread);
//   warp 1      also lays each tile's key scales out for a tcgen05.cp into tensor memory;
//   warps 2..9  set-up: all ten warps FP4-quantise the 128 (query, head) rows (one thread per 32-element
//               block); then warps 2..5 write the query scale factors into their tensor-memory lane
//               quadrant; warps 2..9 read the accumulators (quadrant = warp % 4, queries
//               8 ((warp - 2) / 4) .. + 7), score and store.
// Tensor memory: NBUF accumulator buffers of 128 columns, NBUF x 8 key-scale columns, 8 query-scale
// columns.  Every wait is bounded; a wait that gives up records device error 1 and the kernel leaves.
#include "csa_common.cuh"
#include "sm100.cuh"

namespace csa {

using namespace sm100;

constexpr int MQ_QB = 16;                  // queries per CTA
constexpr int MQ_N = MQ_QB * 8;            // MMA N
constexpr int MQ_KEYS = 128;               // MMA M: keys per tile
constexpr int MQ_STAGES = 6;
constexpr int MQ_NBUF = 3, MQ_LAG = 2;
constexpr int MQ_EPI_WARPS = 8;
constexpr int MQ_THREADS = 64 + 32 * MQ_EPI_WARPS;
constexpr uint32_t MQ_TMEM_COLS = 512;
constexpr uint32_t MQ_COL_D = 0;                       // NBUF x 128
constexpr uint32_t MQ_COL_SFA = MQ_NBUF * 128;         // NBUF x (2 atoms x 4 columns)
constexpr uint32_t MQ_COL_SFB = MQ_COL_SFA + MQ_NBUF * 8;   // 2 atoms x 4 columns
static_assert(MQ_COL_SFB + 8 <= MQ_TMEM_COLS && MQ_LAG < MQ_NBUF, "tensor-memory plan");

struct MqSmem {
  alignas(1024) uint8_t codes[MQ_STAGES][MQ_KEYS * 64];
  alignas(1024) uint8_t qtile[MQ_N * 64];
  alignas(16) uint8_t sc[MQ_STAGES][MQ_KEYS * 4];
  alignas(16) uint32_t qsc[MQ_N];          // 4 E4M3 block scales of each (query, head) row
  alignas(16) uint32_t sfx[2][2][32][4];   // key scale factors in copy order, 2 slots: [atom][lane][col]
  alignas(16) float wq[MQ_N];
  int nvis[MQ_QB];
  alignas(8) uint64_t full[MQ_STAGES];
  alignas(8) uint64_t empty[MQ_STAGES];
  alignas(8) uint64_t sfa_full[MQ_NBUF];
  alignas(8) uint64_t acc_full[MQ_NBUF];
  alignas(8) uint64_t acc_empty[MQ_NBUF];
  alignas(8) uint64_t q_ready;
  alignas(8) uint64_t done;
  uint32_t tmem_base;
  uint32_t err;
};

struct MqParams {
  const uint16_t* q_I;      // [B][Nq][H_I][128] bf16
  const float* w;           // [B][Nq][H_I]
  const uint8_t* k_scales;  // [B][n_max][4]
  const int32_t* n_c;
  const int64_t* q_pos;     // [B][Nq]
  float* scores;            // [(b Nq + q) ld + key]
  long long ld;
  int Nq, n_max, ratio, H_I, splits;
  float g_q, gg;
  csa_page_map pm;          // key rows (table == NULL: contiguous [B][n_max])
};

__global__ void __launch_bounds__(MQ_THREADS, 1) index_mq_tc_kernel(const __grid_constant__ CUtensorMap kmap,
                                                                    const MqParams P) {
  extern __shared__ uint8_t smem_raw[];
  MqSmem& S = *reinterpret_cast<MqSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.z, q0 = blockIdx.y * MQ_QB;
  if (threadIdx.x == 0) {
    S.err = 0;
    for (int s = 0; s < MQ_STAGES; ++s) { mbar_init(&S.full[s], 1); mbar_init(&S.empty[s], 1); }
    for (int a = 0; a < MQ_NBUF; ++a) {
      mbar_init(&S.sfa_full[a], 4);
      mbar_init(&S.acc_full[a], 1);
      mbar_init(&S.acc_empty[a], MQ_EPI_WARPS);
    }
    mbar_init(&S.q_ready, 4);
    mbar_init(&S.done, 1);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) prefetch_tensormap(&kmap);
  if (warp == 1) { tmem_alloc(&S.tmem_base, MQ_TMEM_COLS); tmem_relinquish(); }
  pdl_trigger();
  pdl_wait();

  // visible keys of each query of the block; the CTA's key tiles cover the block's maximum
  const int ncb = min(P.n_c[b], P.n_max);
  if (threadIdx.x < MQ_QB) {
    const int q = q0 + threadIdx.x;
    long long nv = 0;
    if (q < P.Nq) {
      nv = (P.q_pos[(size_t)b * P.Nq + q] + 1) / P.ratio;
      if (nv > ncb) nv = ncb;
      if (nv < 0) nv = 0;
    }
    S.nvis[threadIdx.x] = (int)nv;
  }
  // FP4 quantisation of the block's (query, head) rows, one thread per 32-element block: the pack rule
  // s = E4M3(amax / 6 g_q), code = E2M1(x / (s g_q)); rows of absent queries / heads are zero
  for (int u = threadIdx.x; u < MQ_N * 4; u += MQ_THREADS) {
    const int n = u >> 2, blk = u & 3, j = n >> 3, h = n & 7, q = q0 + j;
    uint32_t words[4] = {0u, 0u, 0u, 0u};
    uint32_t s_code = 0;
    if (q < P.Nq && h < P.H_I) {
      const uint4* src = reinterpret_cast<const uint4*>(P.q_I + (((size_t)b * P.Nq + q) * P.H_I + h) * 128 + blk * 32);
      uint4 raw[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) raw[i] = __ldg(src + i);
      const uint32_t* r32 = reinterpret_cast<const uint32_t*>(raw);
      float amax = 0.0f;
#pragma unroll
      for (int i = 0; i < 16; ++i)
        amax = fmaxf(amax, fmaxf(fabsf(bf16_bits_to_f(r32[i] & 0xFFFFu)), fabsf(bf16_bits_to_f(r32[i] >> 16))));
      s_code = f32_to_e4m3(__fdiv_rn(amax, 6.0f * P.g_q));
      const float s = e4m3_to_f32(s_code);
      if (s != 0.0f) {
        const float sg = __fmul_rn(s, P.g_q);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const uint32_t lo = f32_to_e2m1(__fdiv_rn(bf16_bits_to_f(r32[i] & 0xFFFFu), sg));
          const uint32_t hi = f32_to_e2m1(__fdiv_rn(bf16_bits_to_f(r32[i] >> 16), sg));
          words[i >> 2] |= (lo | (hi << 4)) << (8 * (i & 3));
        }
      }
    }
    // 16 bytes of codes = 16-byte chunk `blk` of the row's 64 bytes, 64-byte swizzle
    *reinterpret_cast<uint4*>(&S.qtile[n * 64 + ((blk ^ ((n >> 1) & 3)) << 4)]) =
        make_uint4(words[0], words[1], words[2], words[3]);
    reinterpret_cast<uint8_t*>(&S.qsc[n])[blk] = (uint8_t)s_code;
  }
  for (int n = threadIdx.x; n < MQ_N; n += MQ_THREADS) {
    const int j = n >> 3, h = n & 7, q = q0 + j;
    S.wq[n] = (q < P.Nq && h < P.H_I) ? P.w[((size_t)b * P.Nq + q) * P.H_I + h] * P.gg : 0.0f;
  }
  fence_proxy_async_smem();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = S.tmem_base;
  int nv_max = 0;
#pragma unroll
  for (int j = 0; j < MQ_QB; ++j) nv_max = max(nv_max, S.nvis[j]);
  const int n_tiles = (nv_max + MQ_KEYS - 1) / MQ_KEYS;
  const int per = (n_tiles + P.splits - 1) / P.splits;
  const int t_begin = min(n_tiles, (int)blockIdx.x * per);
  const int ntile = min(n_tiles, t_begin + per) - t_begin;
  bool ok = true;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      const long long rows_total = (long long)gridDim.z * P.n_max;
      int issued = 0;
      for (int i = 0; i < ntile && ok; ++i) {
        const int s = i % MQ_STAGES, f = i / MQ_STAGES;
        if (f > 0 && !mbar_wait(&S.empty[s], (f - 1) & 1)) { ok = false; break; }
        const long long li = (long long)(t_begin + i) * MQ_KEYS;
        long long row;
        uint32_t sc_bytes;
        if (P.pm.table == nullptr) {
          row = (long long)b * P.n_max + li;
          long long nrow = rows_total - row;
          if (nrow > MQ_KEYS) nrow = MQ_KEYS;
          sc_bytes = (uint32_t)nrow * 4;                         // multiple of 16: n_max % 4 == 0
        } else {                                                 // a tile lies in one page
          row = page_row(P.pm, b, P.n_max, li);
          sc_bytes = row >= 0 ? MQ_KEYS * 4 : 0;
        }
        mbar_arrive_expect_tx(&S.full[s], sc_bytes ? MQ_KEYS * 64 + sc_bytes : 0);
        if (sc_bytes) {                                          // (an absent page: the tile is never scored)
          tma_load_2d(S.codes[s], &kmap, 0, (int)row, &S.full[s]);
          bulk_load(S.sc[s], P.k_scales + row * 4, sc_bytes, &S.full[s]);
        }
        ++issued;
      }
      if (!ok) atomicOr(&S.err, 1u);
      for (int i = max(0, issued - MQ_STAGES); i < issued; ++i)
        mbar_wait(&S.full[i % MQ_STAGES], (i / MQ_STAGES) & 1, 1u << 16);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    // The warp lays tile i's key scales out in copy order (atom k, lane L: the scales of keys L, L+32,
    // L+64, L+96 as UE4M3 x4, blocks 0,0,1,1 for k = 0 and 2,2,3,3 for k = 1); lane 0 copies them into
    // tensor memory and issues the MMAs (copies and MMAs run in issue order).
    const uint32_t idesc = idesc_mxf4_ue4m3(MQ_KEYS, MQ_N);
    const uint32_t qa = smem_addr(S.qtile);
    if (ntile > 0 && !mbar_wait(&S.q_ready, 0)) ok = false;
    ok = __all_sync(0xffffffffu, ok);
    for (int i = 0; i < ntile && ok; ++i) {
      const int s = i % MQ_STAGES, a = i % MQ_NBUF, use = i / MQ_NBUF;
      ok = __all_sync(0xffffffffu, mbar_wait(&S.full[s], (i / MQ_STAGES) & 1));
      // slot i & 1 was last copied for tile i - 2: that copy completed with tile i - 2's MMAs
      if (ok && i >= 2) ok = __all_sync(0xffffffffu, mbar_wait(&S.acc_full[(i - 2) % MQ_NBUF], ((i - 2) / MQ_NBUF) & 1));
      if (!ok) break;
      const int x = i & 1;
      {
        const uint32_t* sc = reinterpret_cast<const uint32_t*>(S.sc[s]);
        uint32_t v[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) v[c] = sc[lane + 32 * c];
        *reinterpret_cast<uint4*>(S.sfx[x][0][lane]) =
            make_uint4(__byte_perm(v[0], 0, 0x1100), __byte_perm(v[1], 0, 0x1100), __byte_perm(v[2], 0, 0x1100),
                       __byte_perm(v[3], 0, 0x1100));
        *reinterpret_cast<uint4*>(S.sfx[x][1][lane]) =
            make_uint4(__byte_perm(v[0], 0, 0x3322), __byte_perm(v[1], 0, 0x3322), __byte_perm(v[2], 0, 0x3322),
                       __byte_perm(v[3], 0, 0x3322));
        fence_proxy_async_smem();
      }
      __syncwarp();
      if (lane == 0 && use > 0 && !mbar_wait(&S.acc_empty[a], (use - 1) & 1)) ok = false;
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      if (lane == 0) {
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < 2; ++k)
          tmem_cp_32x128b_x4(tbase + MQ_COL_SFA + 8 * a + 4 * k, smem_desc(smem_addr(S.sfx[x][k]), 16, 128, LAYOUT_NONE));
        const uint32_t ca = smem_addr(S.codes[s]);
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const uint64_t ad = smem_desc(ca + 32 * k, 16, 512, LAYOUT_SW64);
          const uint64_t bd = smem_desc(qa + 32 * k, 16, 512, LAYOUT_SW64);
          mma_mxf4(tbase + MQ_COL_D + 128 * a, ad, bd, idesc, tbase + MQ_COL_SFA + 8 * a + 4 * k,
                   tbase + MQ_COL_SFB + 4 * k, k > 0);
        }
        mma_commit(&S.acc_full[a]);
        mma_commit(&S.empty[s]);
      }
      __syncwarp();
    }
    if (lane == 0) mma_commit(&S.done);
    if (!ok && lane == 0) atomicOr(&S.err, 1u);
    __syncwarp();
  } else {
    // ------------------------------------------------ query scale factors + epilogue
    const int q = warp & 3;                        // tensor-memory lane quadrant
    const int grp = (warp - 2) >> 2;               // queries 8 grp .. 8 grp + 7
    const bool sf_writer = grp == 0;
    const uint32_t lane_base = tbase + ((uint32_t)(32 * q) << 16);
    if (sf_writer) {
      // query scale factors: row n = lane + 32 c at lane `lane`, column c (atom k = 0) and 4 + c (k = 1)
      uint32_t v[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) v[c] = S.qsc[lane + 32 * c];
      tmem_st_x4(lane_base + MQ_COL_SFB + 0, __byte_perm(v[0], 0, 0x1100), __byte_perm(v[1], 0, 0x1100),
                 __byte_perm(v[2], 0, 0x1100), __byte_perm(v[3], 0, 0x1100));
      tmem_st_x4(lane_base + MQ_COL_SFB + 4, __byte_perm(v[0], 0, 0x3322), __byte_perm(v[1], 0, 0x3322),
                 __byte_perm(v[2], 0, 0x3322), __byte_perm(v[3], 0, 0x3322));
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.q_ready);
    }
    const float4* wq4 = reinterpret_cast<const float4*>(&S.wq[64 * grp]);
    int nvis[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) nvis[j] = S.nvis[8 * grp + j];
    uint32_t d[64];
    for (int e = 0; e < ntile && ok; ++e) {
      if (!mbar_wait(&S.acc_full[e % MQ_NBUF], (e / MQ_NBUF) & 1)) { ok = false; break; }
      tc_fence_after();
      const uint32_t col = MQ_COL_D + 128 * (e % MQ_NBUF) + 64 * grp;
      tmem_ld_x32(lane_base + col, d);
      tmem_ld_x32(lane_base + col + 32, d + 32);
      tmem_wait_ld_x32(d);
      tmem_wait_ld_x32(d + 32);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.acc_empty[e % MQ_NBUF]);
      const int key = (t_begin + e) * MQ_KEYS + 32 * q + lane;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float4 w0 = wq4[2 * j], w1 = wq4[2 * j + 1];
        const float wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
        float sc = 0.0f;
#pragma unroll
        for (int h = 0; h < 8; ++h) sc = fmaf(wv[h], fmaxf(__uint_as_float(d[8 * j + h]), 0.0f), sc);
        sc += 0.0f;
        if (key < nvis[j]) P.scores[((size_t)b * P.Nq + q0 + 8 * grp + j) * P.ld + key] = sc;
      }
    }
    if (!ok && lane == 0) atomicOr(&S.err, 1u);
  }
  __syncthreads();
  if (warp == 1) {
    mbar_wait(&S.done, 0, 1u << 20);
    tc_fence_after();
    tmem_dealloc(tbase, MQ_TMEM_COLS);
  }
  if (S.err && threadIdx.x == 0) atomicOr(&g_csa_device_error, 1u);
}

// Full-mode rows of several queries per sequence, d_I = 128.
bool index_mq_tc_eligible(const csa_index_args* a) {
  return a->cand == nullptr && a->Nq > 1 && a->d_I == 128 && a->H_I <= 8 && a->n_max % 4 == 0 && a->n_max > 0 &&
         cache_rows(a->k_pages, a->B, a->n_max) < 0x7fffffffLL &&
         (reinterpret_cast<uintptr_t>(a->k_codes) & 15) == 0 && (reinterpret_cast<uintptr_t>(a->k_scales) & 15) == 0 &&
         (reinterpret_cast<uintptr_t>(a->q_I) & 15) == 0 && tensor_map_encoder() != nullptr;
}

csa_status run_scores_mq_tc(const csa_index_args* a, float* scores, long long ld, cudaStream_t st) {
  CUtensorMap map;
  const cuuint64_t gdim[2] = {64, (cuuint64_t)cache_rows(a->k_pages, a->B, a->n_max)};
  const cuuint64_t gstride[1] = {64};
  const cuuint32_t box[2] = {64, MQ_KEYS};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = tensor_map_encoder()(&map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, (void*)a->k_codes, gdim, gstride, box, estr,
                                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return CSA_ERR_CUDA;
  MqParams P{};
  P.q_I = (const uint16_t*)a->q_I;
  P.w = a->w;
  P.k_scales = a->k_scales;
  P.n_c = a->n_c;
  P.q_pos = a->q_pos;
  P.scores = scores;
  P.ld = ld;
  P.Nq = a->Nq;
  P.n_max = a->n_max;
  P.ratio = a->ratio;
  P.H_I = a->H_I;
  P.g_q = a->g_q;
  P.gg = a->g_q * a->g_k;
  P.pm = a->k_pages;
  // key splits per query block: at most two waves of CTAs in all (one CTA per SM: the tensor memory),
  // rounded down so that few query blocks do not spill into a third, short wave; 2 while the query blocks
  // alone fill one to two waves; each CTA at least 8 key tiles
  const long long qblocks = (long long)a->B * ((a->Nq + MQ_QB - 1) / MQ_QB);
  const int tiles_row = (a->n_max + MQ_KEYS - 1) / MQ_KEYS;
  long long splits = (2 * 148) / qblocks;
  if (splits < 2 && qblocks < 2 * 148) splits = 2;
  if (splits > (tiles_row + 7) / 8) splits = (tiles_row + 7) / 8;
  if (splits < 1) splits = 1;
  P.splits = (int)splits;
  const int smem = (int)sizeof(MqSmem) + 1024;
  static std::atomic<unsigned> attr_done{0};
  set_smem_once((const void*)index_mq_tc_kernel, smem, attr_done);
  return launch_pdl(index_mq_tc_kernel, dim3(P.splits, (a->Nq + MQ_QB - 1) / MQ_QB, a->B), dim3(MQ_THREADS), smem, st,
                    map, P);
}

}  // namespace csa
