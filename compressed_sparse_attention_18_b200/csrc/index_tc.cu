// Lightning-indexer scores on the 5th-generation tensor cores (tcgen05, block-scaled FP4), for rows
// that score every visible key of one query (decode and the Full layer of cross-layer reuse).
// Sources: "DeepSeek-V4: エージェントが実際に使える100万トークンのコンテキスト", §ハイブリッド注意, Fig. 3 (an FP4
// multi-head ReLU indexer over the compressed entries); "DeepSeek-V4.1-Flash - Pushing the Limits of
// KV Cache Compression", FP4 主 KV キャッシュ bullet (E2M1 values with E4M3 scale factors).
//
// One tile = 256 keys = two MMA sub-tiles of 128 keys (M) x the 8 indexer heads of the query (N) x
// 128 elements (K, two K64 instructions of kind::mxf4nvf4 with UE4M3 scales per 16 elements; the
// key's E4M3 scale of each 32-block is written for both of its 16-element halves).  The tensor core
// forms exactly
//   D[key][h] = sum_blk sq[h][blk] * sk[key][blk] * sum_{e in blk} e2m1(q_e) e2m1(k_e)
// in fp32, i.e. the indexer's per-head dot product before the ReLU.  The epilogue applies
// s = sum_h w'[h] * max(0, D[key][h]) with w' = w * g_q * g_k.
//
// Warp roles (192 threads, persistent over a contiguous range of key tiles of one query row):
//   warp 0      TMA producer: 256 x 64 B FP4 code tile (2-D tensor map, 64-byte swizzle) and the
//               tile's 1 KB of key scales (bulk copy) into a STAGES-deep shared-memory ring;
//   warp 1      allocates tensor memory and issues the MMAs (one thread);
//   warps 2..5  write tile i's scale factors into tensor memory (tcgen05.st) while the accumulator of
//               tile i - LAG is being read (tcgen05.ld), then compute those scores, store them and
//               count them in the row histogram used by the top-k.
// Tensor memory holds a ring of NBUF tiles of scale factors and accumulators, so up to LAG MMAs are
// in flight behind the epilogue.  Every wait is bounded; on a timeout the kernel records device
// error 1 (csa_device_status) and leaves.
#include "csa_common.cuh"
#include "sm100.cuh"

namespace csa {

using namespace sm100;

constexpr int TC_STAGES = 3;
constexpr int TC_CTAS_PER_SM = 3;              // resident CTAs per SM (tensor memory, shared memory)
constexpr int TC_SUB = 128;                      // keys per MMA (M)
constexpr int TC_TILE = 2 * TC_SUB;              // keys per TMA box / pipeline step
constexpr int TC_CODE_BYTES = TC_TILE * 64;      // 256 keys x 128 FP4
constexpr int TC_SC_BYTES = TC_TILE * 4;         // 256 keys x 4 E4M3 scales
constexpr int TC_THREADS = 192;
constexpr int TC_NBUF = 3, TC_LAG = 2;
constexpr uint32_t TC_TMEM_COLS = 128;
constexpr uint32_t TC_COL_D = 0;                 // NBUF x (2 sub-tiles x 8 heads)
constexpr uint32_t TC_COL_SFA = 64;              // NBUF x (2 sub-tiles x 2 atoms x 4 columns)
constexpr uint32_t TC_COL_SFB = 112;             // 2 atoms x 4 columns
static_assert(TC_COL_D + 16 * TC_NBUF <= TC_COL_SFA && TC_COL_SFA + 16 * TC_NBUF <= TC_COL_SFB &&
              TC_COL_SFB + 8 <= TC_TMEM_COLS && TC_CTAS_PER_SM * TC_TMEM_COLS <= 512 && TC_LAG < TC_NBUF,
              "tensor-memory plan");
constexpr int TC_HIST_BINS = 4096, TC_HIST_SHIFT = 20;

// FUSED: the decode row is scored by a cluster of FT_CLUSTER CTAs that keep their scores in shared memory
// and select the row's top-k themselves (no score row in global memory, no separate top-k kernel).
constexpr int FT_CLUSTER = 8;
constexpr int FT_SCAP = 4096;                    // scores one CTA holds (16 tiles): rows up to 32768 keys
constexpr int FT_CAND = 4096;                    // boundary-bin candidates gathered in CTA 0 (its code stages)

template <bool FUSED>
struct TcSmemT {
  static constexpr int STAGES = FUSED ? 4 : TC_STAGES;   // fused: 2 CTAs per SM, 8 per row, 4 tiles in flight each
  alignas(1024) uint8_t codes[STAGES][TC_CODE_BYTES];
  alignas(1024) uint8_t qtile[8 * 64];
  alignas(16) uint8_t sc[STAGES][TC_SC_BYTES];
  alignas(16) uint32_t sfx[2][2][2][32][4];  // key scale factors in copy order, 2 slots: [sub-tile][atom][lane][col]
  uint32_t hist[TC_HIST_BINS];
  float scores[FUSED ? FT_SCAP : 1];             // fused: scores of this CTA's keys [key_lo, key_lo + nk)
  uint32_t gsl[FUSED ? TC_HIST_BINS / FT_CLUSTER : 1];   // fused: this CTA's slice of the row histogram
  uint32_t h256[FUSED ? 256 : 1];
  uint32_t stot, a_cnt, e_cnt, ctr0, ctr1, ctr2;
  uint32_t bc[8];
  float wq[8];
  uint8_t qsc[8][4];
  alignas(8) uint64_t full[STAGES];
  alignas(8) uint64_t empty[STAGES];
  alignas(8) uint64_t sfa_full[TC_NBUF];
  alignas(8) uint64_t acc_full[TC_NBUF];
  alignas(8) uint64_t acc_empty[TC_NBUF];
  alignas(8) uint64_t q_ready;              // query tile, its scale factors and weights are in place
  uint32_t tmem_base;
  uint32_t err;
};

struct TcParams {
  const uint16_t* q_I;      // [B][H_I][128] bf16 (Nq == 1)
  const float* w;           // [B][H_I]
  const uint8_t* k_scales;  // [B][n_max][4]
  const int32_t* n_c;
  const int64_t* q_pos;
  float* scores;            // [B][ld]
  uint32_t* hist;           // [B][4096] or null
  long long ld;
  int n_max, ratio, H_I, ctas_per_row;
  int early;                // read q_I, w, n_c, q_pos and key rows below n_c[b] - 1 before the wait
  float g_q, gg;
  csa_page_map pm;          // key rows (table == NULL: contiguous [B][n_max])
  int32_t* idx_out;         // fused: [B][k]
  float* scores_out;        // fused: [B][k] or null
  int k;
};

// FP4-quantise 32 elements held one per lane (pack rule, global scale g); returns this lane's code.
__device__ __forceinline__ uint32_t quant_lane(float x, float g, uint32_t* s_code_out) {
  const float amax = warp_max(fabsf(x));
  const uint32_t s_code = f32_to_e4m3(__fdiv_rn(amax, 6.0f * g));
  const float s = e4m3_to_f32(s_code);
  *s_code_out = s_code;
  return s != 0.0f ? f32_to_e2m1(__fdiv_rn(x, __fmul_rn(s, g))) : 0u;
}

template <class SM>
__device__ void fused_select(SM& S, const TcParams& P, int b, int n_vis, int key_lo, int nk, int span);

template <bool FUSED>
__global__ void __launch_bounds__(TC_THREADS, 1) index_score_tc_kernel(const __grid_constant__ CUtensorMap kmap,
                                                                       const TcParams P) {
  using SM = TcSmemT<FUSED>;
  constexpr int TC_STAGES = SM::STAGES;
  extern __shared__ uint8_t smem_raw[];
  SM& S = *reinterpret_cast<SM*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.y;
  // setup that reads no global memory, then wait for the previous kernel (it may append to the cache)
  if (threadIdx.x == 0) {
    S.err = 0;
    for (int s = 0; s < TC_STAGES; ++s) { mbar_init(&S.full[s], 1); mbar_init(&S.empty[s], 1); }
    for (int a = 0; a < TC_NBUF; ++a) {
      mbar_init(&S.sfa_full[a], 4);
      mbar_init(&S.acc_full[a], 1);
      mbar_init(&S.acc_empty[a], 4);
    }
    mbar_init(&S.q_ready, 4);
    fence_mbar_init();
    S.stot = 0; S.a_cnt = 0; S.e_cnt = 0; S.ctr0 = 0; S.ctr1 = 0; S.ctr2 = 0;
  }
  if (warp == 0 && lane == 0) prefetch_tensormap(&kmap);
  for (int i = threadIdx.x; i < TC_HIST_BINS; i += blockDim.x) S.hist[i] = 0;
  if (warp == 1) { tmem_alloc(&S.tmem_base, TC_TMEM_COLS); tmem_relinquish(); }
  pdl_trigger();
  if (!P.early) pdl_wait();
  // key tiles of this CTA
  long long nv = (P.q_pos[b] + 1) / P.ratio;
  const int ncb = min(P.n_c[b], P.n_max);
  // early start: the tiles below the one holding row n_c[b] - 1 (the entry the previous kernel may be
  // appending) are loaded before the wait (rows past a sequence's end that a tile also covers are never
  // scored)
  const int wait_tile = P.early ? (ncb - 1 >= 0 ? (ncb - 1) / TC_TILE : -1) : -1;
  if (nv > ncb) nv = ncb;
  if (nv < 0) nv = 0;
  const int n_vis = (int)nv;
  const int n_tiles = (n_vis + TC_TILE - 1) / TC_TILE;
  const int per = (n_tiles + P.ctas_per_row - 1) / P.ctas_per_row;
  const int t_begin = min(n_tiles, (int)blockIdx.x * per);
  const int t_end = min(n_tiles, t_begin + per);
  const int ntile = t_end - t_begin;

  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = S.tmem_base;
  bool ok = true;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      const long long rows_total = (long long)gridDim.y * P.n_max;
      // every key is read once per call: its lines go first when L2 needs room, so the stream does not
      // push out what the step reuses (the kernels' code, scores, ids, partials)
      const uint64_t stream_policy = l2_policy_evict_first();
      int issued = 0;
      bool waited = !P.early;
      for (int i = 0; i < ntile && ok; ++i) {
        const int s = i % TC_STAGES, f = i / TC_STAGES;
        if (!waited && t_begin + i >= wait_tile) { pdl_wait(); waited = true; }
        if (f > 0 && !mbar_wait(&S.empty[s], (f - 1) & 1)) { ok = false; break; }
        // two 128-row sub-tiles, each inside one page of a paged pool; rows past a sequence's end that a
        // tile also covers are never scored (a sub-tile of an absent page is left as it was)
        long long row[2];
        uint32_t sc_bytes[2], tx = 0;
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const long long li = (long long)(t_begin + i) * TC_TILE + u * TC_SUB;
          if (P.pm.table == nullptr) {
            row[u] = (long long)b * P.n_max + li;
            long long nrow = rows_total - row[u];
            if (nrow > TC_SUB) nrow = TC_SUB;
            if (nrow < 0) nrow = 0;
            sc_bytes[u] = (uint32_t)nrow * 4;                   // multiple of 16: n_max % 4 == 0
          } else {
            row[u] = li < P.n_max ? page_row(P.pm, b, P.n_max, li) : -1;
            sc_bytes[u] = row[u] >= 0 ? TC_SUB * 4 : 0;
          }
          if (sc_bytes[u] > 0) tx += TC_SUB * 64 + sc_bytes[u];
        }
        mbar_arrive_expect_tx(&S.full[s], tx);
#pragma unroll
        for (int u = 0; u < 2; ++u)
          if (sc_bytes[u] > 0) {
            tma_load_2d_hint(S.codes[s] + u * (TC_SUB * 64), &kmap, 0, (int)row[u], &S.full[s], stream_policy);
            bulk_load_hint(S.sc[s] + u * (TC_SUB * 4), P.k_scales + row[u] * 4, sc_bytes[u], &S.full[s],
                           stream_policy);
          }
        ++issued;
      }
      if (!ok) atomicOr(&S.err, 1u);
      // drain: wait (bounded) for the copies this thread issued before leaving
      for (int i = max(0, issued - TC_STAGES); i < issued; ++i)
        mbar_wait(&S.full[i % TC_STAGES], (i / TC_STAGES) & 1, 1u << 16);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    // The whole warp lays tile i's key scales out in copy order (sub-tile u, atom k, lane L: the scales
    // of keys L, L+32, L+64, L+96 as UE4M3 x4, blocks 0,0,1,1 for k = 0 and 2,2,3,3 for k = 1); lane 0
    // copies them into tensor memory and issues the MMAs (copies and MMAs run in issue order).
    const uint32_t idesc = idesc_mxf4_ue4m3(TC_SUB, 8);
    const uint32_t qa = smem_addr(S.qtile);
    if (ntile > 0 && !mbar_wait(&S.q_ready, 0)) ok = false;
    ok = __all_sync(0xffffffffu, ok);
    for (int i = 0; i < ntile && ok; ++i) {
      const int s = i % TC_STAGES, a = i % TC_NBUF, use = i / TC_NBUF;
      ok = __all_sync(0xffffffffu, mbar_wait(&S.full[s], (i / TC_STAGES) & 1));
      // slot i & 1 was last copied for tile i - 2: that copy completed with tile i - 2's MMAs
      if (ok && i >= 2) ok = __all_sync(0xffffffffu, mbar_wait(&S.acc_full[(i - 2) % TC_NBUF], ((i - 2) / TC_NBUF) & 1));
      if (!ok) break;
      const int x = i & 1;
      {
        const uint32_t* sc = reinterpret_cast<const uint32_t*>(S.sc[s]);
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          uint32_t v[4];
#pragma unroll
          for (int c = 0; c < 4; ++c) v[c] = sc[TC_SUB * u + 32 * c + lane];
          *reinterpret_cast<uint4*>(S.sfx[x][u][0][lane]) =
              make_uint4(__byte_perm(v[0], 0, 0x1100), __byte_perm(v[1], 0, 0x1100), __byte_perm(v[2], 0, 0x1100),
                         __byte_perm(v[3], 0, 0x1100));
          *reinterpret_cast<uint4*>(S.sfx[x][u][1][lane]) =
              make_uint4(__byte_perm(v[0], 0, 0x3322), __byte_perm(v[1], 0, 0x3322), __byte_perm(v[2], 0, 0x3322),
                         __byte_perm(v[3], 0, 0x3322));
        }
        fence_proxy_async_smem();
      }
      __syncwarp();
      if (lane == 0) {
        if (use > 0 && !mbar_wait(&S.acc_empty[a], (use - 1) & 1)) ok = false;
      }
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      if (lane == 0) {
        tc_fence_after();
#pragma unroll
        for (int u = 0; u < 2; ++u)
#pragma unroll
          for (int k = 0; k < 2; ++k)
            tmem_cp_32x128b_x4(tbase + TC_COL_SFA + 16 * a + 8 * u + 4 * k,
                               smem_desc(smem_addr(S.sfx[x][u][k]), 16, 128, LAYOUT_NONE));
        const uint32_t ca = smem_addr(S.codes[s]);
#pragma unroll
        for (int u = 0; u < 2; ++u)
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const uint64_t ad = smem_desc(ca + u * (TC_SUB * 64) + 32 * k, 16, 512, LAYOUT_SW64);
            const uint64_t bd = smem_desc(qa + 32 * k, 16, 512, LAYOUT_SW64);
            mma_mxf4(tbase + TC_COL_D + 16 * a + 8 * u, ad, bd, idesc, tbase + TC_COL_SFA + 16 * a + 8 * u + 4 * k,
                     tbase + TC_COL_SFB + 4 * k, k > 0);
          }
        mma_commit(&S.acc_full[a]);
        mma_commit(&S.empty[s]);
      }
      __syncwarp();
    }
    if (!ok && lane == 0) atomicOr(&S.err, 1u);
    __syncwarp();
  } else {
    // ------------------------------------------------------ query tile + epilogue
    const int q = warp & 3;                                      // tensor-memory lane quadrant
    const uint32_t lane_base = tbase + ((uint32_t)(32 * q) << 16);
    {
      // query: FP4 B tile (8 heads x 64 B, 64-byte swizzle), its scales and the head weights; warp
      // wg = warp - 2 takes heads 2wg, 2wg+1 (all eight loads issued before any use)
      const int wg = warp - 2;
      float x[2][4];
#pragma unroll
      for (int hh = 0; hh < 2; ++hh)
#pragma unroll
        for (int blk = 0; blk < 4; ++blk) {
          const int h = 2 * wg + hh;
          x[hh][blk] = h < P.H_I ? bf16_bits_to_f(P.q_I[((size_t)b * P.H_I + h) * 128 + blk * 32 + lane]) : 0.0f;
        }
      const float wv = (lane < 2 && 2 * wg + lane < P.H_I) ? P.w[(size_t)b * P.H_I + 2 * wg + lane] * P.gg : 0.0f;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int h = 2 * wg + hh;
#pragma unroll
        for (int blk = 0; blk < 4; ++blk) {
          uint32_t s_code = 0;
          const uint32_t code = quant_lane(x[hh][blk], P.g_q, &s_code);   // zero heads give code 0, scale 0
          const uint32_t pair = code | (__shfl_down_sync(0xffffffffu, code, 1) << 4);
          if ((lane & 1) == 0) {
            const int byte = blk * 16 + (lane >> 1);             // byte of the 64-byte row
            const int c = byte >> 4;
            S.qtile[h * 64 + ((c ^ ((h >> 1) & 3)) << 4) + (byte & 15)] = (uint8_t)pair;
          }
          if (lane == 0) S.qsc[h][blk] = (uint8_t)s_code;
        }
      }
      if (lane < 2) S.wq[2 * wg + lane] = wv;
      fence_proxy_async_smem();
      asm volatile("bar.sync 1, 128;" ::: "memory");             // the four epilogue warps
      // query scale factors: row h (< 8) at lane h of every quadrant, column j = 0
      uint32_t w0 = 0, w1 = 0;
      if (lane < 8) {
        const uint32_t v = *reinterpret_cast<const uint32_t*>(S.qsc[lane]);
        w0 = __byte_perm(v, 0, 0x1100);
        w1 = __byte_perm(v, 0, 0x3322);
      }
      tmem_st_x4(lane_base + TC_COL_SFB + 0, w0, 0, 0, 0);
      tmem_st_x4(lane_base + TC_COL_SFB + 4, w1, 0, 0, 0);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.q_ready);
    }
    float wq[8];
#pragma unroll
    for (int h = 0; h < 8; ++h) wq[h] = S.wq[h];
    float* srow = FUSED ? nullptr : P.scores + (size_t)b * P.ld;
    const int key_lo = t_begin * TC_TILE;
    uint32_t d[16];
    auto finish = [&](int i) {
      // d holds tile i's accumulators (issued by the caller): release them, then score
      tmem_wait_ld_x16(d);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.acc_empty[i % TC_NBUF]);
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int key = (t_begin + i) * TC_TILE + TC_SUB * u + 32 * q + lane;
        if (key < n_vis) {
          float sc = 0.f;
#pragma unroll
          for (int h = 0; h < 8; ++h) sc = fmaf(wq[h], fmaxf(__uint_as_float(d[8 * u + h]), 0.f), sc);
          sc += 0.0f;
          if constexpr (FUSED) {
            S.scores[key - key_lo] = sc;
            atomicAdd(&S.hist[float_order_key(sc) >> TC_HIST_SHIFT], 1u);
          } else {
            srow[key] = sc;
            if (P.hist) atomicAdd(&S.hist[float_order_key(sc) >> TC_HIST_SHIFT], 1u);
          }
        }
      }
    };
    for (int e = 0; e < ntile && ok; ++e) {
      if (!mbar_wait(&S.acc_full[e % TC_NBUF], (e / TC_NBUF) & 1)) { ok = false; break; }
      tc_fence_after();
      tmem_ld_x16(lane_base + TC_COL_D + 16 * (e % TC_NBUF), d);
      finish(e);
    }
    if (!ok && lane == 0) atomicOr(&S.err, 1u);
  }
  __syncthreads();
  if (P.early && threadIdx.x == 0) pdl_wait();   // this grid completes only after its predecessor
  if (S.err && threadIdx.x == 0) atomicOr(&g_csa_device_error, 1u);
  if constexpr (FUSED) {
    const int key_lo = t_begin * TC_TILE;
    fused_select(S, P, b, n_vis, key_lo, max(0, min(n_vis, t_end * TC_TILE) - key_lo), per * TC_TILE);
  } else if (P.hist && S.err == 0) {
    uint32_t* h = P.hist + (size_t)b * TC_HIST_BINS;
    for (int i = threadIdx.x; i < TC_HIST_BINS; i += blockDim.x) {
      const uint32_t c = S.hist[i];
      if (c) atomicAdd(&h[i], c);
    }
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, TC_TMEM_COLS);
  }
}

// ------------------------------------------------------------------------- fused top-k selection
// The CTAs of the row's cluster hold its scores; k_eff = min(k, n_vis) of them are selected by (score desc,
// key id asc) without leaving the chip:
//   1. the row histogram (top 12 bits of the order-preserving key, each CTA's own counts) is summed in
//      slices over the cluster, and every CTA finds the bin T holding the k_eff-th score;
//   2. each CTA writes its keys above T at slots from a prefix over the cluster's counts;
//   3. the keys in bin T: all of them when exactly needed, else they are gathered in CTA 0 (or, past
//      FT_CAND of them, read from the peers in place) and CTA 0 resolves them exactly by 8-bit digits of
//      the composite (order key, ~id) below the bin's bits.
// Every CTA executes every cluster barrier, whatever its own state.
struct FtCand {
  uint32_t key;
  int32_t id;
};

// Resolve `need` of the candidates get(j) (j < n; false = not a candidate) in CTA 0: composite v = key << 32 |
// ~id, all sharing the top 12 key bits; written at oi / os[base + ...] (S.ctr2 counts the slots used).
template <class SM, class Get>
__device__ void fused_resolve(SM& S, int n, uint32_t need, uint32_t base, Get get, int32_t* oi, float* os) {
  const uint32_t limit = base + need;                   // slots of this resolution: [base, base + need)
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint64_t prefix = 0, mask = 0;
  bool done = false;
  // digits of the 52 bits below the bin: [51:44] [43:36] [35:28] [27:20] [19:12] [11:4], then [3:0]
#pragma unroll 1
  for (int lv = 0; lv < 7 && !done; ++lv) {
    const int sh = lv < 6 ? 44 - 8 * lv : 0;
    const uint32_t dm = lv < 6 ? 255u : 15u;
    for (int i = tid; i < 256; i += blockDim.x) S.h256[i] = 0;
    __syncthreads();
    for (int j = tid; j < n; j += blockDim.x) {
      FtCand c;
      if (!get(j, c)) continue;
      const uint64_t v = ((uint64_t)c.key << 32) | (uint32_t)(0xFFFFFFFFu - (uint32_t)c.id);
      if ((v & mask) == prefix) atomicAdd(&S.h256[(uint32_t)(v >> sh) & dm], 1u);
    }
    __syncthreads();
    if (warp == 0) {
      // lane l owns digits 8 (31 - l) .. + 7, highest first
      uint32_t c[8], tot = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) { c[i] = S.h256[8 * (31 - lane) + 7 - i]; tot += c[i]; }
      uint32_t incl = tot;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      uint32_t acc = incl - tot;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (acc < need && acc + c[i] >= need) { S.bc[4] = 8 * (31 - lane) + 7 - i; S.bc[5] = acc; S.bc[6] = c[i]; }
        acc += c[i];
      }
    }
    __syncthreads();
    const uint32_t digit = S.bc[4], above = S.bc[5], cnt = S.bc[6];
    const uint64_t nprefix = prefix | ((uint64_t)digit << sh), nmask = mask | ((uint64_t)dm << sh);
    done = need == above + cnt;                          // every candidate of the threshold digit is taken
    for (int j = tid; j < n; j += blockDim.x) {
      FtCand c;
      if (!get(j, c)) continue;
      const uint64_t v = ((uint64_t)c.key << 32) | (uint32_t)(0xFFFFFFFFu - (uint32_t)c.id);
      if ((v & mask) != prefix) continue;
      const uint32_t dj = (uint32_t)(v >> sh) & dm;
      if (dj > digit || (done && dj == digit)) {
        const uint32_t slot = base + atomicAdd(&S.ctr2, 1u);
        if (slot < limit) {                             // (always, unless a bounded wait gave up upstream)
          oi[slot] = c.id;
          if (os) os[slot] = order_key_float(c.key);
        }
      }
    }
    need -= above;
    prefix = nprefix;
    mask = nmask;
    __syncthreads();
  }
}

// span = keys per CTA of the row (CTA r holds keys [r span, r span + span) of those visible)
template <class SM>
__device__ void fused_select(SM& S, const TcParams& P, int b, int n_vis, int key_lo, int nk, int span) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t rank = blockIdx.x, nr = gridDim.x;              // the cluster spans blockIdx.x
  const uint32_t K = (uint32_t)min(P.k, n_vis);
  int32_t* oi = P.idx_out + (size_t)b * P.k;
  float* os = P.scores_out ? P.scores_out + (size_t)b * P.k : nullptr;
  if (rank == 0)
    for (int j = (int)K + tid; j < P.k; j += blockDim.x) {
      oi[j] = -1;
      if (os) os[j] = -INFINITY;
    }
  constexpr int SL = TC_HIST_BINS / FT_CLUSTER;
  // (1) every CTA's histogram is complete
  cluster_sync_all();
  {
    uint32_t part = 0;
    for (int i = tid; i < SL; i += blockDim.x) {
      uint32_t v = 0;
      for (uint32_t r = 0; r < nr; ++r) v += ld_peer_u32(peer_addr(&S.hist[rank * SL + i], r));
      S.gsl[i] = v;
      part += v;
    }
    part = __reduce_add_sync(0xffffffffu, part);
    if (lane == 0 && part) atomicAdd(&S.stot, part);
  }
  // (2) the slices of the row histogram are complete
  cluster_sync_all();
  if (warp == 0 && K > 0) {
    // slice holding the K-th score (slices of higher bins on higher ranks), then its bin
    const uint32_t tot = lane < (int)nr ? ld_peer_u32(peer_addr(&S.stot, lane)) : 0u;
    uint32_t suf = tot;                                          // sum over ranks >= lane
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_down_sync(0xffffffffu, suf, o);
      if (lane + o < 32) suf += y;
    }
    const uint32_t above_s = suf - tot;
    const uint32_t hit = __ballot_sync(0xffffffffu, lane < (int)nr && above_s < K && K <= suf);
    const int sl = hit ? __ffs(hit) - 1 : 0;
    const uint32_t above_sl = __shfl_sync(0xffffffffu, above_s, sl);
    uint32_t bins[SL / 32], lt = 0;
#pragma unroll
    for (int i = 0; i < SL / 32; ++i) {
      bins[i] = ld_peer_u32(peer_addr(&S.gsl[(SL / 32) * lane + i], sl));
      lt += bins[i];
    }
    uint32_t lsuf = lt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_down_sync(0xffffffffu, lsuf, o);
      if (lane + o < 32) lsuf += y;
    }
    uint32_t acc = above_sl + lsuf - lt;
#pragma unroll
    for (int i = SL / 32 - 1; i >= 0; --i) {
      if (acc < K && acc + bins[i] >= K) {
        S.bc[0] = (uint32_t)(sl * SL + (SL / 32) * lane + i);
        S.bc[1] = acc;
        S.bc[2] = bins[i];
      }
      acc += bins[i];
    }
  }
  __syncthreads();
  const uint32_t T = S.bc[0], above = K > 0 ? S.bc[1] : 0u;
  // (3) this CTA's keys above T and in T
  if (K > 0) {
    uint32_t a = 0, e = 0;
    for (int i = tid; i < nk; i += blockDim.x) {
      const uint32_t bin = float_order_key(S.scores[i]) >> TC_HIST_SHIFT;
      a += bin > T;
      e += bin == T;
    }
    a = __reduce_add_sync(0xffffffffu, a);
    e = __reduce_add_sync(0xffffffffu, e);
    if (lane == 0) {
      if (a) atomicAdd(&S.a_cnt, a);
      if (e) atomicAdd(&S.e_cnt, e);
    }
  }
  cluster_sync_all();
  // (4) slots: prefix of the counts over lower ranks
  if (warp == 0) {
    const uint32_t a = lane < (int)nr ? ld_peer_u32(peer_addr(&S.a_cnt, lane)) : 0u;
    const uint32_t e = lane < (int)nr ? ld_peer_u32(peer_addr(&S.e_cnt, lane)) : 0u;
    uint32_t pa = a, pe = e;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t ya = __shfl_up_sync(0xffffffffu, pa, o), ye = __shfl_up_sync(0xffffffffu, pe, o);
      if (lane >= o) { pa += ya; pe += ye; }
    }
    const uint32_t E = __shfl_sync(0xffffffffu, pe, 31);
    if (lane == (int)rank) { S.bc[4] = pa - a; S.bc[5] = pe - e; }
    if (lane == 0) S.bc[6] = E;
  }
  __syncthreads();
  const uint32_t pa = S.bc[4], pe = S.bc[5], E = S.bc[6];
  const uint32_t need = K - above;
  const bool take_all = need == E;
  const bool gather = K > 0 && !take_all && E <= FT_CAND;
  FtCand* cand = reinterpret_cast<FtCand*>(&S.codes[0][0]);           // CTA 0's buffer (code stages are idle)
  static_assert(sizeof(S.codes) >= FT_CAND * sizeof(FtCand), "candidate buffer");
  if (K > 0) {
    for (int i = tid; i < nk; i += blockDim.x) {
      const float v = S.scores[i];
      const uint32_t key = float_order_key(v), bin = key >> TC_HIST_SHIFT;
      // (slot checks hold by construction; they keep a row whose streaming gave up inside its k slots)
      if (bin > T) {
        const uint32_t slot = pa + atomicAdd(&S.ctr0, 1u);
        if (slot < above) {
          oi[slot] = key_lo + i;
          if (os) os[slot] = v;
        }
      } else if (bin == T) {
        const uint32_t j = pe + atomicAdd(&S.ctr1, 1u);
        if (take_all) {
          if (above + j < K) {
            oi[above + j] = key_lo + i;
            if (os) os[above + j] = v;
          }
        } else if (gather && j < E) {
          st_peer_u32(peer_addr(&cand[j].key, 0), key);
          st_peer_u32(peer_addr(&cand[j].id, 0), (uint32_t)(key_lo + i));
        }
      }
    }
  }
  // (5) the boundary candidates are in CTA 0 (or in place)
  cluster_sync_all();
  if (rank == 0 && K > 0 && !take_all) {
    if (gather) {
      fused_resolve(S, (int)E, need, above, [&](int j, FtCand& c) { c = cand[j]; return true; }, oi, os);
    } else {
      // more candidates than the buffer: read them where they are (rank r holds keys r span + i), filtered
      // by bin T
      fused_resolve(S, (int)(nr * span), need, above, [&](int j, FtCand& c) {
        const uint32_t r = (uint32_t)j / (uint32_t)span, i = (uint32_t)j % (uint32_t)span;
        const uint32_t lo = r * (uint32_t)span;
        if (lo + i >= (uint32_t)n_vis) return false;
        const float v = __uint_as_float(ld_peer_u32(peer_addr(&S.scores[i], r)));
        c.key = float_order_key(v);
        c.id = (int32_t)(lo + i);
        return (c.key >> TC_HIST_SHIFT) == T;
      }, oi, os);
    }
  }
  // (6) the peers are done with this CTA's shared memory
  cluster_sync_all();
}

// --------------------------------------------------------------------------------------- host
namespace sm100 {
EncodeTiledFn tensor_map_encoder() {
  static std::atomic<EncodeTiledFn> fn{nullptr};
  EncodeTiledFn f = fn.load();
  if (!f) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qr) == cudaSuccess &&
        qr == cudaDriverEntryPointSuccess)
      f = (EncodeTiledFn)p;
    fn.store(f);
  }
  return f;
}
}  // namespace sm100

bool index_tc_eligible(const csa_index_args* a) {
  return a->cand == nullptr && a->Nq == 1 && a->d_I == 128 && a->H_I <= 8 && a->n_max % 4 == 0 && a->n_max > 0 &&
         cache_rows(a->k_pages, a->B, a->n_max) < 0x7fffffffLL &&
         (reinterpret_cast<uintptr_t>(a->k_codes) & 15) == 0 && (reinterpret_cast<uintptr_t>(a->k_scales) & 15) == 0 &&
         tensor_map_encoder() != nullptr;
}

static bool encode_key_map(const csa_index_args* a, CUtensorMap* map) {
  const cuuint64_t gdim[2] = {64, (cuuint64_t)cache_rows(a->k_pages, a->B, a->n_max)};
  const cuuint64_t gstride[1] = {64};
  const cuuint32_t box[2] = {64, TC_SUB};
  const cuuint32_t estr[2] = {1, 1};
  return tensor_map_encoder()(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, (void*)a->k_codes, gdim, gstride, box, estr,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static TcParams tc_params(const csa_index_args* a) {
  TcParams P{};
  P.q_I = (const uint16_t*)a->q_I;
  P.w = a->w;
  P.k_scales = a->k_scales;
  P.n_c = a->n_c;
  P.q_pos = a->q_pos;
  P.n_max = a->n_max;
  P.ratio = a->ratio;
  P.H_I = a->H_I;
  P.g_q = a->g_q;
  P.gg = a->g_q * a->g_k;
  P.pm = a->k_pages;
  P.early = (a->flags & CSA_EARLY_START) ? 1 : 0;
  return P;
}

csa_status run_scores_tc(const csa_index_args* a, float* scores, long long ld, uint32_t* hist, cudaStream_t st) {
  CUtensorMap map;
  if (!encode_key_map(a, &map)) return CSA_ERR_CUDA;
  TcParams P = tc_params(a);
  P.scores = scores;
  P.hist = hist;
  P.ld = ld;
  // TC_CTAS_PER_SM resident CTAs per SM: one wave, at most one per tile
  const int tiles_row = (a->n_max + TC_TILE - 1) / TC_TILE;
  int per_row = (TC_CTAS_PER_SM * 148) / a->B;
  if (per_row > tiles_row) per_row = tiles_row;
  if (per_row < 1) per_row = 1;
  P.ctas_per_row = per_row;
  const int smem = (int)sizeof(TcSmemT<false>) + 1024;
  static std::atomic<unsigned> attr_done{0};
  set_smem_once((const void*)index_score_tc_kernel<false>, smem, attr_done);
  return launch_pdl(index_score_tc_kernel<false>, dim3(per_row, a->B), dim3(TC_THREADS), smem, st, map, P);
}

// Fused decode indexer + top-k (CSA_ONCHIP_TOPK): single-query Full rows of at most FT_CLUSTER x FT_SCAP
// keys, no pool.
bool index_topk_fused_eligible(const csa_index_args* a) {
  return (a->flags & CSA_ONCHIP_TOPK) && index_tc_eligible(a) && a->pool_blocks == 0 && a->idx_out != nullptr &&
         a->n_max <= FT_CLUSTER * FT_SCAP && a->k >= 1 && a->k <= 4096;
}

csa_status run_index_topk_fused(const csa_index_args* a, cudaStream_t st) {
  CUtensorMap map;
  if (!encode_key_map(a, &map)) return CSA_ERR_CUDA;
  TcParams P = tc_params(a);
  P.idx_out = a->idx_out;
  P.scores_out = a->scores_out;
  P.k = a->k;
  P.ctas_per_row = FT_CLUSTER;
  static_assert(FT_CLUSTER * FT_SCAP >= FT_CLUSTER * TC_TILE && FT_SCAP % TC_TILE == 0, "tile split");
  const int smem = (int)sizeof(TcSmemT<true>) + 1024;
  static std::atomic<unsigned> attr_done{0};
  set_smem_once((const void*)index_score_tc_kernel<true>, smem, attr_done);
  cudaLaunchAttribute attr[2];
  cudaLaunchConfig_t cfg = pdl_config(dim3(FT_CLUSTER, a->B), dim3(TC_THREADS), (size_t)smem, st, attr);
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = FT_CLUSTER;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.numAttrs = 2;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, index_score_tc_kernel<true>, map, P);
  if (e != cudaSuccess) {
    set_last_cuda_error(e);
    return CSA_ERR_CUDA;
  }
  return launch_status();
}

}  // namespace csa
