// Attention on the 5th-generation tensor cores (tcgen05, bf16 in, fp32 accumulators in tensor memory), for
// rows with a 512-wide shared KV head (64-wide RoPE slice): one CTA takes one query (all heads) and `tpc`
// consecutive tiles of 128 keys of its key list [selected (or, dense, all visible) entries ‖ window rows],
// walked with an online softmax; the partials of a query's CTAs are merged by attn_merge_kernel.  Under
// the early start (CSA_EARLY_START) the split-0 CTAs come first in the grid and attend over the window
// tile before waiting for the kernel that writes the selected ids.
// Sources: "DeepSeek-V4: エージェントが実際に使える100万トークンのコンテキスト", §ハイブリッド注意, Fig. 3 (attention
// over the top-k compressed entries plus a sliding-window branch under one softmax; the 128x layer attends
// densely over all visible entries).
//
// Transposed formulation (the keys, not the <= 64 heads, fill the 128-row MMA):
//   S^T[key][h] = K[key][:] . Q[h][:]             M = 128 keys, N = 64 heads, K = 512 (32 MMAs, K-major)
//   P^T = exp2(S^T * scale*log2e - m_h)           per-head max / sum over the tile's keys: a 32-lane
//                                                 transpose-reduce in registers, then 4 warps through smem
//   O^T[dim][h] = sum_key K[key][dim] P^T[key][h] M = 4 x 128 dims, N = 64, K = 128 keys; the same K tile
//                                                 read through an MN-major descriptor (V = K)
// Tile assembly: Q and window rows arrive by TMA (3-D maps, 128-byte swizzle, rows outside the buffers read
// as zero); FP4 entries are gathered by id and dequantised by all 8 warps into the same swizzled layout.
// Partials (O / l in bf16, lse = ln l + m in fp32) per (query, CTA) go to the workspace; with one CTA per
// query it writes the bf16 output and lse itself.
#include <cstring>

#include "csa_common.cuh"
#include "sm100.cuh"

namespace csa {

using namespace sm100;

constexpr int TA_WORKERS = 256;           // warps 0-7: gather, softmax (4 lane quadrants x 2 head halves), epilogue
constexpr int TA_THREADS = TA_WORKERS + 32; // warp 8: barriers, tensor memory, TMA and MMA issue
constexpr int TA_KEYS = 128;
constexpr int TA_WBOX = 32;                // window rows per TMA box
constexpr uint32_t TA_TMEM_COLS = 512;
constexpr uint32_t TA_COL_S = 0;           // S^T: 64 columns
constexpr uint32_t TA_COL_O = 64;          // O^T: 4 x 64 columns
constexpr float TA_LOG2E = 1.4426950408889634f;
constexpr float TA_LN2 = 0.6931471805599453f;
constexpr int TA_MAX_CLUSTER = 8;          // portable cluster size: queries split over <= 8 CTAs merge in-cluster

struct TaSmem {
  alignas(1024) uint8_t K[8][TA_KEYS * 128];   // [dim block of 64][key][128 B], 128-byte swizzle
  alignas(1024) uint8_t Q[8][64 * 128];        // [dim block][head][128 B]
  alignas(1024) uint8_t P[TA_KEYS * 128];      // [key][64 heads bf16]
  float red_m[4][64], red_l[4][64];            // per lane-quadrant partial max / sum
  alignas(16) float m[64];                     // running max (log2 units)
  float l[64], fac[64];                        // running sum, this tile's rescale
  int32_t ids[TA_KEYS];                        // entry id of each entry row, -1 if absent
  // per dim block: Q landed, window boxes landed, gathered rows written
  alignas(8) uint64_t bar_q[8], bar_w[8], bar_k[8];
  uint64_t bar_s, bar_p, bar_o[4];
  uint32_t tmem_base;
  uint32_t err;
  int rescale;                                 // some head's running max moved: O and l are rescaled
  float cf[TA_MAX_CLUSTER][64];                // cluster merge: weight of each CTA's partial per head
  float cL[64];                                // cluster merge: 1 / total softmax sum per head
};

struct TaParams {
  int Nq, H, ratio, n_max, k, Wn, window, splits, hca;
  int rows;             // B * Nq
  int tpc;              // key tiles per CTA (a CTA walks tiles split*tpc .. split*tpc + tpc - 1 of its query)
  int cluster;          // the `splits` CTAs of a query form one thread-block cluster and merge their
                        // partials through distributed shared memory (no workspace partials, no merge kernel)
  int early_rows;       // > 0 (= rows): CTA i < early_rows is split 0 of query i; it walks the query's
                        // window tile before waiting for the previous kernel, then its entry tiles
  float g, scale_log2;
  const int64_t* q_pos;
  const uint8_t* codes;
  const uint8_t* scales;
  const uint16_t* rope;
  const int32_t* n_c;
  const int32_t* idx;
  const uint16_t* win;
  const int64_t* win_pos0;
  uint16_t* out;        // splits == 1
  float* lse;           // splits == 1 (may be null)
  uint16_t* part_o;     // [rows][splits][H][512] bf16 (splits = CTAs per query)
  float* part_lse;      // [rows][splits][H]
  int win_fp8;          // window rows are FP8 (codes / scales / rope below) instead of bf16 rows in `win`
  const uint8_t* wcodes;   // [B][Wn][448] E4M3
  const float* wscales;    // [B][Wn][8] fp32 (7 used)
  const uint16_t* wrope;   // [B][Wn][64] bf16
  csa_page_map pm;         // cache rows (table == NULL: contiguous [B][n_max])
};

__device__ __forceinline__ uint32_t sw128(int row, int chunk) { return (uint32_t)(row * 128 + ((chunk ^ (row & 7)) << 4)); }

__device__ __forceinline__ void cp16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(dst)), "l"(src));
}

// 2^x by the hardware approximation (one special-function instruction, relative error about 2^-22;
// results below 2^-126 flush to zero): P is rounded to bf16 right after, and l sums these same values.
__device__ __forceinline__ float ta_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t hmul2_bf16(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// Eight E2M1 codes (element e in bits 4e..4e+3 of w) times a bf16x2 scale splat -> four bf16x2 words
// (elements 2i, 2i+1 in word i).  Integer work only: the magnitudes index two byte tables of the bf16
// encodings of 0, 0.5, 1, 1.5, 2, 3, 4, 6 (prmt), the sign bits move to bits 15 / 31, and one bf16x2
// multiply applies the scale (E2M1 values are exact in bf16; the product is rounded once).
__device__ __forceinline__ uint4 e2m1x8_to_bf16_scaled(uint32_t w, uint32_t sc2) {
  constexpr uint32_t LO0 = 0xC0800000u, LO1 = 0xC0804000u;   // low bytes of the bf16 encodings, codes 0..7
  constexpr uint32_t HI0 = 0x3F3F3F00u, HI1 = 0x40404040u;   // high bytes
  const uint32_t m = w & 0x77777777u, mh = m >> 16;
  const uint32_t la = __byte_perm(LO0, LO1, m), ha = __byte_perm(HI0, HI1, m);
  const uint32_t lb = __byte_perm(LO0, LO1, mh), hb = __byte_perm(HI0, HI1, mh);
  const uint32_t x = w << 4;                                 // sign of element 2k at bit 7 of byte k
  uint4 o;
  o.x = hmul2_bf16(__byte_perm(la, ha, 0x5140) | (__byte_perm(x, w, 0x4400) & 0x80008000u), sc2);
  o.y = hmul2_bf16(__byte_perm(la, ha, 0x7362) | (__byte_perm(x, w, 0x5511) & 0x80008000u), sc2);
  o.z = hmul2_bf16(__byte_perm(lb, hb, 0x5140) | (__byte_perm(x, w, 0x6622) & 0x80008000u), sc2);
  o.w = hmul2_bf16(__byte_perm(lb, hb, 0x7362) | (__byte_perm(x, w, 0x7733) & 0x80008000u), sc2);
  return o;
}

// Two E4M3 codes (low byte first) times an fp32 scale -> packed bf16x2: exact E4M3 -> f16 conversion,
// the product rounded to fp32, then to bf16.
__device__ __forceinline__ uint32_t e4m3x2_to_bf16x2_scaled(uint32_t two, float sc) {
  uint32_t h2;
  const uint16_t in = (uint16_t)two;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(in));
  const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h2));
  return pack_bf16x2(f.x * sc, f.y * sc);
}

// 32 values per lane reduced across the warp's 32 lanes, transposed: on return lane l holds the reduction of
// value l over all lanes (31 shuffles, each halving the values a lane still carries).
template <bool kMax>
__device__ __forceinline__ float transpose_reduce32(float (&v)[32], int lane) {
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) {
    const bool up = (lane & s) != 0;
#pragma unroll
    for (int i = 0; i < s; ++i) {
      const float send = up ? v[i] : v[i + s];
      const float keep = up ? v[i + s] : v[i];
      const float got = __shfl_xor_sync(0xffffffffu, send, s);
      v[i] = kMax ? fmaxf(keep, got) : keep + got;
    }
  }
  return v[0];
}

__device__ __forceinline__ void tmem_st_x32(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};"
      ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]),
        "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]),
        "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

// Geometry of one 128-key tile of a query's key list [n_sel entries ‖ window rows].
struct TaTile {
  int key0, rs, rw, wa, we, zs;
  long long wrow_base;     // window buffer row of tile row r (r >= rs) is wrow_base + r
};
// FP8 window rows are gathered and dequantised by the workers (no TMA boxes: wa = we = rw).
__device__ __forceinline__ TaTile ta_tile(int key0, int n_sel, int n_list, long long wlo, long long p0, bool fp8) {
  TaTile g;
  g.key0 = key0;
  g.rs = min(max(n_sel - key0, 0), TA_KEYS);                        // rows [0, rs): entries
  g.rw = max(min(n_list - key0, TA_KEYS), 0);                       // rows [rs, rw): window, then empty
  g.wa = fp8 ? g.rw : (g.rs + TA_WBOX - 1) / TA_WBOX * TA_WBOX;      // window rows >= wa come by TMA boxes
  g.we = g.rw > g.wa ? (g.rw + TA_WBOX - 1) / TA_WBOX * TA_WBOX : g.wa;
  g.zs = g.rw > g.wa ? g.we : g.rw;                                  // rows >= zs are zero-filled
  g.wrow_base = (wlo - p0) + (long long)(key0 - n_sel);
  return g;
}

// Lazy rescaling: a head keeps its running max until a tile's max exceeds it by more than this (log2
// units), so probabilities stay <= 2^8 and O is rescaled in tensor memory only when a max jumps.
constexpr float TA_RESCALE_SLACK = 8.0f;

// W8: the window rows are FP8 (a separate instantiation keeps the bf16 path's code compact: each launch
// runs with a cold instruction cache)
template <bool W8>
__global__ void __launch_bounds__(TA_THREADS, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap wmap,
                   const TaParams P) {
  extern __shared__ uint8_t smem_raw[];
  TaSmem& S = *reinterpret_cast<TaSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // early window: the split-0 CTAs of all queries come first in the grid (they start during the previous
  // kernel and walk the window tile while it runs), then the other splits
  // (with a cluster per query the CTAs of a query are consecutive: rank = split)
  const bool early = P.early_rows > 0;
  const bool by_query = !early || P.cluster;
  const bool first_cta = early && (P.cluster ? (int)blockIdx.x % P.splits == 0 : (int)blockIdx.x < P.early_rows);
  const int jb = (int)blockIdx.x - P.early_rows;
  const int bq = by_query ? (int)blockIdx.x / P.splits : first_cta ? (int)blockIdx.x : jb / (P.splits - 1);
  const int split = by_query ? (int)blockIdx.x % P.splits : first_cta ? 0 : 1 + jb % (P.splits - 1);
  const int b = bq / P.Nq;
  // worker thread t owns tile row t/2 for the gather (its half of the row's FP4 blocks and RoPE slice)
  const int grow = (tid & (TA_WORKERS - 1)) >> 1, ghalf = tid & 1;
  // setup that reads no global memory, then wait for the previous kernel (it writes the selected ids)
  if (warp == 8) {
    if (lane == 0) {
      S.err = 0;
      for (int j = 0; j < 8; ++j) {
        mbar_init(&S.bar_q[j], 1);
        mbar_init(&S.bar_w[j], 1);
        mbar_init(&S.bar_k[j], TA_WORKERS / 32);
      }
      mbar_init(&S.bar_s, 1);
      mbar_init(&S.bar_p, TA_WORKERS / 32);
      for (int j = 0; j < 4; ++j) mbar_init(&S.bar_o[j], 1);
      fence_mbar_init();
      prefetch_tensormap(&qmap);
      prefetch_tensormap(&wmap);
    }
    __syncwarp();
    tmem_alloc(&S.tmem_base, TA_TMEM_COLS);
    tmem_relinquish();
  }
  if (tid < 64) { S.m[tid] = -INFINITY; S.l[tid] = 0.f; }
  if (tid == 0) S.rescale = 0;
  pdl_trigger();
  // before the wait: prefetch the query's selected ids and one line per 2 MB of the sequence's cache
  // arrays, so the reads right after it find their address translations (and the ids) warm
  if (!P.hca) {
    const int lines = (P.k * 4 + 127) / 128;
    for (int i = tid; i < lines; i += TA_THREADS) prefetch_l2(P.idx + (size_t)bq * P.k + i * 32);
  }
  if (P.pm.table == nullptr) {
    const size_t n_max = (size_t)P.n_max;
    const size_t cb = n_max * 224, sb = n_max * 16, rb = n_max * 128, pg = (size_t)1 << 21;
    const size_t nc = (cb + pg - 1) / pg, ns = (sb + pg - 1) / pg, nr = (rb + pg - 1) / pg;
    const int j = tid - 64;
    if (n_max > 0 && j >= 0 && (size_t)j < nc + ns + nr) {
      const uint8_t* base = (size_t)j < nc ? P.codes + (size_t)b * cb + (size_t)j * pg
                          : (size_t)j < nc + ns ? P.scales + (size_t)b * sb + ((size_t)j - nc) * pg
                                                : reinterpret_cast<const uint8_t*>(P.rope) + (size_t)b * rb +
                                                      ((size_t)j - nc - ns) * pg;
      prefetch_l2(base);
    }
  }
  // positions and lengths are inputs of the step: under the early start they are read before the wait
  long long tq = 0, p0 = 0;
  int ncb = 0;
  auto load_pos = [&]() {
    tq = P.q_pos[bq];
    ncb = min(P.n_c[b], P.n_max);
    if (P.Wn > 0) p0 = P.win_pos0[b];
  };
  if (early) load_pos();
  if (!first_cta) pdl_wait();                    // (a window tile reads only q, positions and the window)
  if (!early) load_pos();
  int n_sel = P.k;
  if (P.hca) {                                   // all visible entries: r*i + r - 1 <= t and i < n_c
    long long nv = (tq + 1) / P.ratio;
    n_sel = (int)max(0LL, min(nv, (long long)ncb));
  }
  long long wlo = 0, whi = -1;
  if (P.Wn > 0) {
    wlo = max(max(0LL, tq - P.window + 1), p0);
    whi = min(tq, p0 + P.Wn - 1);
  }
  const int n_list = n_sel + (whi >= wlo ? (int)(whi - wlo + 1) : 0);
  const size_t unit_ho = ((size_t)bq * P.splits + split) * P.H;
  // this CTA's tiles (block-uniform): up to tpc consecutive tiles of the key list from split*tpc; with the
  // early window the splits cover the entries only and split 0 takes the window tile first (n_sel is
  // then a multiple of the tile)
  const int base_key = split * P.tpc * TA_KEYS;
  const bool has_win = first_cta && n_list > n_sel;
  const int n_ent = max(0, min(P.tpc, ((early ? n_sel : n_list) - base_key + TA_KEYS - 1) / TA_KEYS));
  const int ntile = n_ent + (has_win ? 1 : 0);
  auto tile_key = [&](int t) -> int {
    return has_win ? (t == 0 ? n_sel : base_key + (t - 1) * TA_KEYS) : base_key + t * TA_KEYS;
  };
  if (first_cta && !has_win) pdl_wait();          // no window rows: the entry tiles need the ids now
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = S.tmem_base;

  if (ntile == 0 && !P.cluster) {               // nothing in this CTA's tiles: an empty partial
    if (P.splits > 1) {
      if (tid < P.H) P.part_lse[unit_ho + tid] = -INFINITY;
    } else {
      for (int i = tid; i < P.H * 256; i += TA_THREADS)
        reinterpret_cast<uint32_t*>(P.out + (size_t)bq * P.H * 512)[i] = 0u;
      if (P.lse && tid < P.H) P.lse[(size_t)bq * P.H + tid] = -INFINITY;
    }
    if (warp == 8) tmem_dealloc(tb, TA_TMEM_COLS);
    return;
  }

  if (ntile == 0) {
    // an empty member of a cluster: m = -inf, l = 0 (its staged O is never read)
  } else if (warp == 8) {
    // ------------------------------------------------------------------ control: TMA, then MMA issue
    if (lane == 0) {
      bool ok = true;
#pragma unroll 1
      for (int j = 0; j < 8; ++j) {
        mbar_arrive_expect_tx(&S.bar_q[j], 64 * 128);
        tma_load_3d(S.Q[j], &qmap, j * 64, 0, bq, &S.bar_q[j]);
      }
      const uint32_t ids = idesc_bf16(128, 64, 0, 0);
      const uint32_t ido = idesc_bf16(128, 64, 1, 1);
#pragma unroll 1
      for (int t = 0; t < ntile; ++t) {
        const TaTile g = ta_tile(tile_key(t), n_sel, n_list, wlo, p0, W8);
        const int nbox = (g.we - g.wa) / TA_WBOX;
        // window boxes overwrite the K tile: only once the previous tile's O MMAs have completed (S MMAs
        // of an entry tile are queued behind them directly)
        if (t > 0 && nbox > 0 && ok) ok = mbar_wait(&S.bar_o[3], (t - 1) & 1);
#pragma unroll 1
        for (int j = 0; j < 8; ++j) {
          mbar_arrive_expect_tx(&S.bar_w[j], (uint32_t)(nbox * TA_WBOX * 128));
          if (ok)
            for (int i = 0; i < nbox; ++i)
              tma_load_3d(&S.K[j][(g.wa + i * TA_WBOX) * 128], &wmap, j * 64,
                          (int)(g.wrow_base + g.wa + i * TA_WBOX), b, &S.bar_w[j]);
        }
        // S^T = K Q^T, dim block by dim block as the blocks land
#pragma unroll 1
        for (int j = 0; j < 8 && ok; ++j) {
          ok = (t > 0 || mbar_wait(&S.bar_q[j], 0)) && mbar_wait(&S.bar_w[j], t & 1) &&
               mbar_wait(&S.bar_k[j], t & 1);
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int s2 = 0; s2 < 4; ++s2) {
            const uint64_t a = smem_desc(smem_addr(S.K[j]) + s2 * 32, 16, 1024, 2);
            const uint64_t bd = smem_desc(smem_addr(S.Q[j]) + s2 * 32, 16, 1024, 2);
            mma_bf16_ss(tb + TA_COL_S, a, bd, ids, (j | s2) != 0);
          }
        }
        mma_commit(&S.bar_s);
        // O^T (+)= V^T P^T (the K tile read MN-major, P stored [key][head]); O accumulates across tiles
        ok = ok && mbar_wait(&S.bar_p, t & 1);
        if (ok) tc_fence_after();
#pragma unroll 1
        for (int mt = 0; mt < 4; ++mt) {
          if (ok) {
#pragma unroll
            for (int s2 = 0; s2 < 8; ++s2) {
              const uint64_t a = smem_desc(smem_addr(S.K[2 * mt]) + s2 * 2048, 16384, 1024, 2);
              const uint64_t bd = smem_desc(smem_addr(S.P) + s2 * 2048, 16384, 1024, 2);
              mma_bf16_ss(tb + TA_COL_O + 64 * mt, a, bd, ido, t > 0 || s2 > 0);
            }
          }
          mma_commit(&S.bar_o[mt]);
        }
      }
      if (!ok) atomicOr(&S.err, 1u);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------------------------- workers
    const int quad = warp & 3, hh = warp >> 2;
    const int key = 32 * quad + lane;
    const uint32_t lane_base = tb + ((uint32_t)(32 * quad) << 16);
    bool ok = true;
    // this thread's row of a tile: entry id and its FP4 blocks 2j + ghalf, scale row and RoPE quarter,
    // loaded one tile ahead (registers)
    // raw id of this thread's row of a tile (loaded one tile before it is used), then its check
    auto raw_id = [&](const TaTile& g) -> int {
      const int li = g.key0 + grow;
      if (grow >= g.rs) return -1;
      return P.hca ? li : (li < P.k ? P.idx[(size_t)bq * P.k + li] : -1);
    };
    auto check_id = [&](int v) -> int { return (v >= 0 && v < ncb) ? v : -1; };
    uint4 cv[7], sc16, rp[4];
    auto load_row = [&](int id) {
#pragma unroll
      for (int j = 0; j < 7; ++j) cv[j] = make_uint4(0, 0, 0, 0);
      sc16 = make_uint4(0, 0, 0, 0);
#pragma unroll
      for (int c = 0; c < 4; ++c) rp[c] = make_uint4(0, 0, 0, 0);
      const long long r = id >= 0 ? page_row(P.pm, b, P.n_max, id) : -1;   // row in the cache arrays
      if (r >= 0) {
        // the row's lines are requested from L2 first: a prefetch holds no L1 miss slot, and the 128 random
        // rows of a tile otherwise reach DRAM only as fast as the SM's outstanding misses drain
        if (ghalf == 0) {
          prefetch_l2(P.codes + (size_t)r * 224);
          prefetch_l2(P.codes + (size_t)r * 224 + 223);
          prefetch_l2(P.scales + (size_t)r * 16);
        } else {
          prefetch_l2(P.codes + (size_t)r * 224 + 112);
          prefetch_l2(P.rope + (size_t)r * 64);
        }
        const uint8_t* crow = P.codes + (size_t)r * 224 + ghalf * 16;
#pragma unroll
        for (int j = 0; j < 7; ++j) cv[j] = __ldg(reinterpret_cast<const uint4*>(crow + j * 32));
        sc16 = __ldg(reinterpret_cast<const uint4*>(P.scales + (size_t)r * 16));
        const uint4* rrow = reinterpret_cast<const uint4*>(P.rope + (size_t)r * 64) + ghalf * 4;
#pragma unroll
        for (int c = 0; c < 4; ++c) rp[c] = __ldg(rrow + c);
      }
    };
    // FP8 window row of a tile (rows [rs, rw)) in the same registers an entry row uses: codes of this
    // thread's 32 channels of 64-channel blocks 0-2 in cv[0..5], the 7 block scales in cv[6] (0-3) and
    // sc16 (4-6), the RoPE quarter in rp; blocks 3-6 are read into cv[0..6], sc16 during the gather.
    auto is_win8 = [&](const TaTile& gg) { return W8 && grow >= gg.rs && grow < gg.rw; };
    auto win8_ptr = [&](const TaTile& gg) -> const uint8_t* {
      return P.wcodes + ((size_t)b * P.Wn + (size_t)(gg.wrow_base + grow)) * 448 + ghalf * 32;
    };
    auto load_win8 = [&](const TaTile& gg) {
      const size_t wr = (size_t)b * P.Wn + (size_t)(gg.wrow_base + grow);
      const uint4* crow = reinterpret_cast<const uint4*>(win8_ptr(gg));
#pragma unroll
      for (int j = 0; j < 3; ++j) {
        cv[2 * j] = __ldg(crow + 4 * j);
        cv[2 * j + 1] = __ldg(crow + 4 * j + 1);
      }
      const uint4* srow = reinterpret_cast<const uint4*>(P.wscales + wr * 8);
      cv[6] = __ldg(srow);
      sc16 = __ldg(srow + 1);
      const uint4* rrow = reinterpret_cast<const uint4*>(P.wrope + wr * 64) + ghalf * 4;
#pragma unroll
      for (int c = 0; c < 4; ++c) rp[c] = __ldg(rrow + c);
    };
    TaTile g = ta_tile(tile_key(0), n_sel, n_list, wlo, p0, W8);
    int id = check_id(raw_id(g));                  // a window tile reads no id
    int id_next = ntile > 1 && !has_win ? raw_id(ta_tile(tile_key(1), n_sel, n_list, wlo, p0, W8)) : -1;
    load_row(id);
    if (is_win8(g)) load_win8(g);
#pragma unroll 1
    for (int t = 0; t < ntile; ++t) {
      // a tile of entry rows only can be refilled block by block as the previous tile's O MMAs release
      // them (O M-tile mt reads dim blocks 2mt, 2mt+1); any other tile waits for all of them first
      const bool pure = g.rs == TA_KEYS;
      if (t > 0 && !pure) {
#pragma unroll 1
        for (int mt = 0; mt < 4; ++mt) ok = mbar_wait(&S.bar_o[mt], (t - 1) & 1) && ok;
        tc_fence_after();
      }
      if (ghalf == 0) S.ids[grow] = id;
      if (!pure) {
        // window rows before the first TMA box, by asynchronous copies
        const int r_end = min(g.wa, g.rw);
        const int n = W8 ? 0 : (r_end > g.rs ? r_end - g.rs : 0) * 64;
        for (int i = tid; i < n; i += TA_WORKERS) {
          const int row = g.rs + (i >> 6), c = i & 63;
          const long long wr = g.wrow_base + row;
          cp16(&S.K[c >> 3][sw128(row, c & 7)], P.win + ((size_t)b * P.Wn + wr) * 512 + c * 8);
        }
        // empty rows
        for (int i = tid; i < (TA_KEYS - g.zs) * 64; i += TA_WORKERS) {
          const int row = g.zs + (i >> 6), c = i & 63;
          *reinterpret_cast<uint4*>(&S.K[c >> 3][sw128(row, c & 7)]) = make_uint4(0, 0, 0, 0);
        }
        asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
      }
      const bool win8_row = is_win8(g);
      float ws3 = 0.f, ws4 = 0.f, ws5 = 0.f, ws6 = 0.f;
      // dequantise dim block by dim block: bf16(e2m1 * bf16(e4m3 * g)); each block released to the MMA warp
#pragma unroll
      for (int j = 0; j < 7; ++j) {
        if (win8_row && j == 3) {
          // blocks 0-2 are done: keep scales 3-6, read the codes of blocks 3-6 into the same registers
          ws3 = __uint_as_float(cv[6].w);
          ws4 = __uint_as_float(sc16.x);
          ws5 = __uint_as_float(sc16.y);
          ws6 = __uint_as_float(sc16.z);
          const uint4* crow = reinterpret_cast<const uint4*>(win8_ptr(g));
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            cv[2 * i] = __ldg(crow + 4 * (3 + i));
            if (i < 3) cv[2 * i + 1] = __ldg(crow + 4 * (3 + i) + 1);
          }
          sc16 = __ldg(crow + 4 * 6 + 1);
        }
        if (t > 0 && pure && (j & 1) == 0) {
          ok = mbar_wait(&S.bar_o[j >> 1], (t - 1) & 1) && ok;
          tc_fence_after();
        }
        if (grow < g.rs) {
          const int part = 2 * j + ghalf;                  // word (2j + ghalf) / 4 of the scale row: j / 2
          const uint32_t word = (j >> 1) == 0 ? sc16.x : (j >> 1) == 1 ? sc16.y : (j >> 1) == 2 ? sc16.z : sc16.w;
          const uint32_t sb = f_to_bf16_bits(e4m3_to_f32((word >> ((part & 3) * 8)) & 0xFFu) * P.g);
          const uint32_t sc2 = sb | (sb << 16);
          const uint32_t w4[4] = {cv[j].x, cv[j].y, cv[j].z, cv[j].w};
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4)
            *reinterpret_cast<uint4*>(&S.K[j][sw128(grow, ghalf * 4 + q4)]) = e2m1x8_to_bf16_scaled(w4[q4], sc2);
        } else if (win8_row) {
          // FP8 window row: bf16(e4m3 * scale of the 64-channel block)
          const float sc = j == 0 ? __uint_as_float(cv[6].x) : j == 1 ? __uint_as_float(cv[6].y)
                         : j == 2 ? __uint_as_float(cv[6].z) : j == 3 ? ws3 : j == 4 ? ws4 : j == 5 ? ws5 : ws6;
          const uint4 c0 = j < 3 ? cv[2 * j] : cv[2 * (j - 3)];
          const uint4 c1 = j < 3 ? cv[2 * j + 1] : j < 6 ? cv[2 * (j - 3) + 1] : sc16;
          const uint32_t w8[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4)
            *reinterpret_cast<uint4*>(&S.K[j][sw128(grow, ghalf * 4 + q4)]) =
                make_uint4(e4m3x2_to_bf16x2_scaled(w8[2 * q4] & 0xFFFFu, sc), e4m3x2_to_bf16x2_scaled(w8[2 * q4] >> 16, sc),
                           e4m3x2_to_bf16x2_scaled(w8[2 * q4 + 1] & 0xFFFFu, sc),
                           e4m3x2_to_bf16x2_scaled(w8[2 * q4 + 1] >> 16, sc));
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.bar_k[j]);
      }
      if (t > 0 && pure) {
        ok = mbar_wait(&S.bar_o[3], (t - 1) & 1) && ok;
        tc_fence_after();
      }
      // RoPE slice (dim block 7) of the entry rows (and of FP8 window rows)
      if (grow < g.rs || win8_row) {
#pragma unroll
        for (int c = 0; c < 4; ++c) *reinterpret_cast<uint4*>(&S.K[7][sw128(grow, ghalf * 4 + c)]) = rp[c];
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.bar_k[7]);
      const TaTile gt = g;
      // next tile's row (its id arrived during this tile's gather), in flight during this tile's softmax
      // and MMAs; the id of the tile after it is requested now
      auto advance = [&]() {
        g = ta_tile(tile_key(t + 1), n_sel, n_list, wlo, p0, W8);
        id = check_id(id_next);
        load_row(id);
        if (is_win8(g)) load_win8(g);
        id_next = t + 2 < ntile ? raw_id(ta_tile(tile_key(t + 2), n_sel, n_list, wlo, p0, W8)) : -1;
      };
      // the window tile (split 0 under the early start) runs its softmax too before the wait; its
      // entry tile's ids and rows are read after it
      const bool win_first = has_win && t == 0;
      if (t + 1 < ntile && !win_first) advance();
      asm volatile("bar.sync 1, 256;" ::: "memory");   // workers only: ids visible to the softmax

      // ---- softmax of this tile: warp w reads lanes 32*(w%4).. (its keys) and head half w/4
      ok = mbar_wait(&S.bar_s, t & 1) && ok;
      tc_fence_after();
      // one 32-value array per thread: the scores for the max, reloaded from tensor memory for the
      // probabilities, which then feed the sum
      const bool valid = key < gt.rs ? (S.ids[key] >= 0) : (key < gt.rw);
      float red[32];
      {
        uint32_t sv[32];
        tmem_ld_x32(lane_base + TA_COL_S + hh * 32, sv);
        tmem_wait_ld_x32(sv);
#pragma unroll
        for (int j = 0; j < 32; ++j) red[j] = valid ? __uint_as_float(sv[j]) * P.scale_log2 : -INFINITY;
      }
      S.red_m[quad][hh * 32 + lane] = transpose_reduce32<true>(red, lane);
      asm volatile("bar.sync 1, 256;" ::: "memory");
      if (tid < 64) {
        const float mt = fmaxf(fmaxf(S.red_m[0][tid], S.red_m[1][tid]), fmaxf(S.red_m[2][tid], S.red_m[3][tid]));
        const float mo = S.m[tid];
        float mn = mo, f = 1.f;
        if (mt > mo + TA_RESCALE_SLACK || (mo == -INFINITY && mt > -INFINITY)) {
          mn = mt;
          f = mo == -INFINITY ? 0.f : exp2f(mo - mn);
        }
        S.m[tid] = mn;
        S.fac[tid] = f;
        S.l[tid] *= f;
        if (f != 1.f && t > 0) S.rescale = 1;
      }
      asm volatile("bar.sync 1, 256;" ::: "memory");
      if (t > 0 && S.rescale) {
        // a running max moved: scale the accumulated O^T columns of this thread's heads
#pragma unroll 1
        for (int mt = 0; mt < 4; ++mt) {
          uint32_t ov[32];
          tmem_ld_x32(lane_base + TA_COL_O + 64 * mt + hh * 32, ov);
          tmem_wait_ld_x32(ov);
#pragma unroll
          for (int j = 0; j < 32; ++j) ov[j] = __float_as_uint(__uint_as_float(ov[j]) * S.fac[hh * 32 + j]);
          tmem_st_x32(lane_base + TA_COL_O + 64 * mt + hh * 32, ov);
        }
        tmem_wait_st();
      }
      {
        uint32_t sv[32];
        tmem_ld_x32(lane_base + TA_COL_S + hh * 32, sv);
        tmem_wait_ld_x32(sv);
        uint32_t pk[16];
        float mh[32];
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
          const float4 v4 = *reinterpret_cast<const float4*>(&S.m[hh * 32 + j]);
          mh[j] = v4.x; mh[j + 1] = v4.y; mh[j + 2] = v4.z; mh[j + 3] = v4.w;
        }
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          const float m0 = mh[j], m1 = mh[j + 1];
          const float z0 = valid ? __uint_as_float(sv[j]) * P.scale_log2 : -INFINITY;
          const float z1 = valid ? __uint_as_float(sv[j + 1]) * P.scale_log2 : -INFINITY;
          const float p0f = m0 == -INFINITY ? 0.f : ta_exp2(z0 - m0);
          const float p1f = m1 == -INFINITY ? 0.f : ta_exp2(z1 - m1);
          red[j] = p0f;
          red[j + 1] = p1f;
          pk[j >> 1] = pack_bf16x2(p0f, p1f);
        }
#pragma unroll
        for (int c = 0; c < 4; ++c)
          *reinterpret_cast<uint4*>(&S.P[sw128(key, hh * 4 + c)]) =
              make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.bar_p);
      S.red_l[quad][hh * 32 + lane] = transpose_reduce32<false>(red, lane);
      asm volatile("bar.sync 1, 256;" ::: "memory");
      if (tid < 64) S.l[tid] += (S.red_l[0][tid] + S.red_l[1][tid]) + (S.red_l[2][tid] + S.red_l[3][tid]);
      if (tid == 0) S.rescale = 0;
      asm volatile("bar.sync 1, 256;" ::: "memory");
      if (win_first && t + 1 < ntile) {
        // from here on the ids and entries of the previous kernels
        pdl_wait();
        id_next = raw_id(ta_tile(tile_key(1), n_sel, n_list, wlo, p0, W8));
        advance();
      }
    }

    // ---- epilogue, M-tile by M-tile as the last O MMAs complete: lane = dim, columns = heads
    float il[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const float lj = S.l[hh * 32 + j];
      il[j] = lj > 0.f ? 1.f / lj : 0.f;
    }
    const int hmax = min(32, P.H - hh * 32);
    const int tl = ntile - 1;
    if (P.cluster) {
      // stage the unnormalised O (fp32, [head][512 dims]) over the K tile once every O MMA has read it
      ok = mbar_wait(&S.bar_o[3], tl & 1) && ok;
      tc_fence_after();
    }
    float* stage = reinterpret_cast<float*>(&S.K[0][0]);
#pragma unroll 1
    for (int mt = 0; mt < 4; ++mt) {
      if (!P.cluster) {
        ok = mbar_wait(&S.bar_o[mt], tl & 1) && ok;
        tc_fence_after();
      }
      uint32_t ov[32];
      tmem_ld_x32(lane_base + TA_COL_O + 64 * mt + hh * 32, ov);
      tmem_wait_ld_x32(ov);
      const int dim = 128 * mt + 32 * quad + lane;
      if (P.cluster) {
#pragma unroll
        for (int j = 0; j < 32; ++j) stage[(hh * 32 + j) * 512 + dim] = __uint_as_float(ov[j]);
      } else if (P.splits == 1) {
        uint16_t* o = P.out + ((size_t)bq * P.H + hh * 32) * 512 + dim;
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (j < hmax) o[(size_t)j * 512] = (uint16_t)f_to_bf16_bits(__uint_as_float(ov[j]) * il[j]);
      } else {
        uint16_t* o = P.part_o + (unit_ho + hh * 32) * 512 + dim;
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (j < hmax) o[(size_t)j * 512] = (uint16_t)f_to_bf16_bits(__uint_as_float(ov[j]) * il[j]);
      }
    }
    if (!ok && lane == 0) atomicOr(&S.err, 1u);
    if (tid < P.H && !P.cluster) {
      const float lh = S.l[tid];
      const float ls = lh > 0.f ? (S.m[tid] + log2f(lh)) * TA_LN2 : -INFINITY;
      if (P.splits == 1) {
        if (P.lse) P.lse[(size_t)bq * P.H + tid] = ls;
      } else {
        P.part_lse[unit_ho + tid] = ls;
      }
    }
    tc_fence_before();
  }
  if (first_cta && tid == 0) pdl_wait();         // the grid completes only after its predecessor
  if (P.cluster) {
    // ---- merge of the query's partials inside its cluster: every CTA's m, l (per head) and staged O
    // are visible after the barrier; CTA `split` writes dims [d0, d1) of the output
    cluster_sync_all();
    const int ns = P.splits;
    if (tid < 64) {
      float mr[TA_MAX_CLUSTER], lr[TA_MAX_CLUSTER], M = -INFINITY;
#pragma unroll
      for (int r = 0; r < TA_MAX_CLUSTER; ++r) {
        mr[r] = -INFINITY;
        lr[r] = 0.f;
        if (r < ns) {
          mr[r] = ld_peer_f32(peer_addr(&S.m[tid], r));
          lr[r] = ld_peer_f32(peer_addr(&S.l[tid], r));
          if (lr[r] > 0.f) M = fmaxf(M, mr[r]);
        }
      }
      float L = 0.f;
#pragma unroll
      for (int r = 0; r < TA_MAX_CLUSTER; ++r) {
        const float f = (r < ns && lr[r] > 0.f) ? exp2f(mr[r] - M) : 0.f;
        S.cf[r][tid] = f;
        L += f * lr[r];
      }
      S.cL[tid] = L > 0.f ? 1.f / L : 0.f;
      if (split == 0 && P.lse && tid < P.H) P.lse[(size_t)bq * P.H + tid] = L > 0.f ? (M + log2f(L)) * TA_LN2 : -INFINITY;
    }
    __syncthreads();
    const int per = ((512 + ns - 1) / ns + 3) & ~3;
    const int d0 = min(512, split * per), d1 = min(512, d0 + per);
    const int groups = (d1 - d0) >> 2;
    uint32_t base[TA_MAX_CLUSTER];
#pragma unroll
    for (int r = 0; r < TA_MAX_CLUSTER; ++r) base[r] = r < ns ? peer_addr(&S.K[0][0], r) : 0u;
    // two outputs per thread per round, all their peer loads issued before the first is used
    const int items = P.H * groups;
    for (int it0 = tid; it0 < items; it0 += 2 * TA_THREADS) {
      float4 v[2][TA_MAX_CLUSTER];
      int hs[2], ds[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int it = it0 + u * TA_THREADS;
        hs[u] = it < items ? it / groups : 0;
        ds[u] = d0 + 4 * (it < items ? it % groups : 0);
#pragma unroll
        for (int r = 0; r < TA_MAX_CLUSTER; ++r)
          v[u][r] = (it < items && r < ns && S.cf[r][hs[u]] != 0.f)
                        ? ld_peer_v4(base[r] + (uint32_t)((hs[u] * 512 + ds[u]) * 4))
                        : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        if (it0 + u * TA_THREADS >= items) continue;
        const int h = hs[u];
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int r = 0; r < TA_MAX_CLUSTER; ++r) {
          const float f = r < ns ? S.cf[r][h] : 0.f;
          acc.x = fmaf(f, v[u][r].x, acc.x); acc.y = fmaf(f, v[u][r].y, acc.y);
          acc.z = fmaf(f, v[u][r].z, acc.z); acc.w = fmaf(f, v[u][r].w, acc.w);
        }
        const float il = S.cL[h];
        uint2 o2;
        o2.x = pack_bf16x2(acc.x * il, acc.y * il);
        o2.y = pack_bf16x2(acc.z * il, acc.w * il);
        *reinterpret_cast<uint2*>(P.out + ((size_t)bq * P.H + h) * 512 + ds[u]) = o2;
      }
    }
    cluster_sync_all();                          // the peers have read this CTA's shared memory
  }
  __syncthreads();
  if (warp == 8) {
    if (S.err && lane == 0) atomicOr(&g_csa_device_error, 1u);
    tc_fence_after();
    tmem_dealloc(tb, TA_TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------------------------------
// Persistent variant, for many queries of several tiles each with one CTA per query (the chunked
// prefill's 4096 queries per chunk, multi-position decode): one CTA per SM takes the queries blockIdx.x,
// blockIdx.x + gridDim.x, ... one after another, each over all of its key tiles.  The tiles of its queries
// form one stream through the same barriers: the next query's Q is loaded by TMA as soon as the S MMAs of
// the current query's last tile have read Q, the next query's first tile is gathered as the current
// query's last O MMAs release the K tile, and the current query's epilogue runs while that tile's S MMAs
// do.  BF16 window rows only.

// A unit is split `split` of query bq (uid = bq * splits + split): tiles [split * tpc, split * tpc + tpc) of
// the query's key list.  Its positions and lengths are read one unit ahead (plain loads, used a tile or
// more later).
struct TaUnitRaw {
  int uid, nc;
  long long tq, wp0;
};
struct TaUnit {
  int uid, bq, split, b, n_sel, n_list, ncb;
  int t0, ntile;        // the unit's first tile of the query's list and its number of tiles
  int wofs;             // window buffer row of the first window key (wlo - win_pos0)
};

__device__ __forceinline__ TaUnitRaw ta_unit_load(const TaParams& P, int uid) {
  TaUnitRaw r;
  const int bq = uid / P.splits, b = bq / P.Nq;
  r.uid = uid;
  r.tq = P.q_pos[bq];
  r.nc = P.n_c[b];
  r.wp0 = P.Wn > 0 ? P.win_pos0[b] : 0;
  return r;
}

// The query's key list [n_sel entries ‖ window rows] (the per-query kernel's rule) and the unit's part.
__device__ __forceinline__ TaUnit ta_unit(const TaParams& P, const TaUnitRaw& r) {
  TaUnit u;
  u.uid = r.uid;
  u.bq = r.uid / P.splits;
  u.split = r.uid % P.splits;
  u.b = u.bq / P.Nq;
  u.ncb = min(r.nc, P.n_max);
  u.n_sel = P.k;
  if (P.hca) u.n_sel = (int)max(0LL, min((r.tq + 1) / P.ratio, (long long)u.ncb));
  long long wlo = 0, whi = -1;
  if (P.Wn > 0) {
    wlo = max(max(0LL, r.tq - P.window + 1), r.wp0);
    whi = min(r.tq, r.wp0 + P.Wn - 1);
  }
  u.wofs = whi >= wlo ? (int)(wlo - r.wp0) : 0;   // in [0, Wn) when the window is not empty
  u.n_list = u.n_sel + (whi >= wlo ? (int)(whi - wlo + 1) : 0);
  u.t0 = u.split * P.tpc;
  u.ntile = max(0, min(P.tpc, (u.n_list + TA_KEYS - 1) / TA_KEYS - u.t0));
  return u;
}

// Tile t of a unit (tile t0 + t of its query's key list).
__device__ __forceinline__ TaTile ta_tile_u(const TaUnit& u, int t) {
  return ta_tile((u.t0 + t) * TA_KEYS, u.n_sel, u.n_list, u.wofs, 0, false);
}

// The first unit with keys among units kk, kk+1, ... of this CTA (from `raw` if those are unit kk's
// positions), writing the outputs of the ones without keys with threads tid < nthreads: zero rows and
// lse = -inf, or an empty partial (lse = -inf) when queries are split; bq = -1 if there is none.
__device__ __forceinline__ TaUnit ta_next_unit(const TaParams& P, int kk, int nu, TaUnitRaw raw, int tid,
                                               int nthreads) {
  TaUnit uu{};
  uu.bq = -1;
#pragma unroll 1
  for (; kk < nu; ++kk) {
    const int uid = (int)blockIdx.x + kk * (int)gridDim.x;
    if (raw.uid != uid) raw = ta_unit_load(P, uid);
    uu = ta_unit(P, raw);
    if (uu.ntile > 0) return uu;
    if (P.splits > 1) {
      if (tid < P.H) P.part_lse[(size_t)uid * P.H + tid] = -INFINITY;
    } else {
      for (int i = tid; i < P.H * 256; i += nthreads)
        reinterpret_cast<uint32_t*>(P.out + (size_t)uu.bq * P.H * 512)[i] = 0u;
      if (P.lse && tid < P.H) P.lse[(size_t)uu.bq * P.H + tid] = -INFINITY;
    }
    uu.bq = -1;
  }
  return uu;
}

// Epilogue of a unit, by the 8 worker warps once its last O MMAs have completed (phase `par` of bar_o):
// O^T / l from tensor memory to bf16 rows [head][512], and lse, into the output (one unit per query) or
// the unit's partial (split queries, merged by the split-merge kernel); resets the running max and sum
// for the next unit.  Returns false if a wait gave up.
__device__ __forceinline__ bool ta_epilogue(TaSmem& S, const TaParams& P, int uid, uint32_t par, uint32_t lane_base,
                                            int hh, int quad, int lane, int tid) {
  bool ok = true;
  const bool part = P.splits > 1;
  uint16_t* orow = part ? P.part_o + (size_t)uid * P.H * 512 : P.out + (size_t)uid * P.H * 512;
  float* lrow = part ? P.part_lse + (size_t)uid * P.H : (P.lse ? P.lse + (size_t)uid * P.H : nullptr);
  if (tid < 64) {
    const float lh = S.l[tid];
    S.fac[tid] = lh > 0.f ? 1.f / lh : 0.f;
    if (tid < P.H && lrow) lrow[tid] = lh > 0.f ? (S.m[tid] + log2f(lh)) * TA_LN2 : -INFINITY;
    S.m[tid] = -INFINITY;
    S.l[tid] = 0.f;
  }
  asm volatile("bar.sync 1, 256;" ::: "memory");
  const int hmax = min(32, P.H - hh * 32);
#pragma unroll 1
  for (int mt = 0; mt < 4; ++mt) {
    ok = ok && mbar_wait(&S.bar_o[mt], par);
    tc_fence_after();
    uint32_t ov[32];
    tmem_ld_x32(lane_base + TA_COL_O + 64 * mt + hh * 32, ov);
    tmem_wait_ld_x32(ov);
    const int dim = 128 * mt + 32 * quad + lane;
    uint16_t* o = orow + (size_t)hh * 32 * 512 + dim;
#pragma unroll
    for (int j = 0; j < 32; j += 4) {
      const float4 il = *reinterpret_cast<const float4*>(&S.fac[hh * 32 + j]);
      if (j < hmax) o[(size_t)j * 512] = (uint16_t)f_to_bf16_bits(__uint_as_float(ov[j]) * il.x);
      if (j + 1 < hmax) o[(size_t)(j + 1) * 512] = (uint16_t)f_to_bf16_bits(__uint_as_float(ov[j + 1]) * il.y);
      if (j + 2 < hmax) o[(size_t)(j + 2) * 512] = (uint16_t)f_to_bf16_bits(__uint_as_float(ov[j + 2]) * il.z);
      if (j + 3 < hmax) o[(size_t)(j + 3) * 512] = (uint16_t)f_to_bf16_bits(__uint_as_float(ov[j + 3]) * il.w);
    }
  }
  tc_fence_before();
  asm volatile("bar.sync 1, 256;" ::: "memory");   // every worker has read fac (the softmax rewrites it)
  return ok;
}

__global__ void __launch_bounds__(TA_THREADS, 1)
    attn_tc_persist_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap wmap,
                           const TaParams P) {
  extern __shared__ uint8_t smem_raw[];
  TaSmem& S = *reinterpret_cast<TaSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int grow = (tid & (TA_WORKERS - 1)) >> 1, ghalf = tid & 1;
  // this CTA's units: its k-th is unit blockIdx.x + k * gridDim.x of the rows * splits
  const int n_units = P.rows * P.splits;
  const int nu = (int)blockIdx.x < n_units ? (n_units - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  auto unit_q = [&](int k) { return (int)blockIdx.x + k * (int)gridDim.x; };
  if (warp == 8) {
    if (lane == 0) {
      S.err = 0;
      for (int j = 0; j < 8; ++j) {
        mbar_init(&S.bar_q[j], 1);
        mbar_init(&S.bar_w[j], 1);
        mbar_init(&S.bar_k[j], TA_WORKERS / 32);
      }
      mbar_init(&S.bar_s, 1);
      mbar_init(&S.bar_p, TA_WORKERS / 32);
      for (int j = 0; j < 4; ++j) mbar_init(&S.bar_o[j], 1);
      fence_mbar_init();
      prefetch_tensormap(&qmap);
      prefetch_tensormap(&wmap);
    }
    __syncwarp();
    tmem_alloc(&S.tmem_base, TA_TMEM_COLS);
    tmem_relinquish();
  }
  if (tid < 64) { S.m[tid] = -INFINITY; S.l[tid] = 0.f; }
  if (tid == 0) S.rescale = 0;
  pdl_trigger();
  pdl_wait();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = S.tmem_base;

  if (warp == 8) {
    // ------------------------------------------------------------------ control: TMA, then MMA issue
    if (lane == 0) {
      bool ok = true;
      const uint32_t ids = idesc_bf16(128, 64, 0, 0);
      const uint32_t ido = idesc_bf16(128, 64, 1, 1);
      // descriptor bases (an offset below 256 KB adds to the 14-bit address field without a carry)
      const uint64_t kdesc = smem_desc(smem_addr(S.K[0]), 16, 1024, 2), qdesc = smem_desc(smem_addr(S.Q[0]), 16, 1024, 2);
      const uint64_t vdesc = smem_desc(smem_addr(S.K[0]), 16384, 1024, 2), pdesc = smem_desc(smem_addr(S.P), 16384, 1024, 2);
      auto load_q = [&](int bq) {
#pragma unroll 1
        for (int j = 0; j < 8; ++j) {
          mbar_arrive_expect_tx(&S.bar_q[j], 64 * 128);
          tma_load_3d(S.Q[j], &qmap, j * 64, 0, bq, &S.bar_q[j]);
        }
      };
      // first query with keys (a query without keys has no tiles: the workers write its output)
      int k = 0;
      TaUnit u{};
      for (; k < nu; ++k) {
        u = ta_unit(P, ta_unit_load(P, unit_q(k)));
        if (u.ntile > 0) break;
      }
      if (k < nu) load_q(u.bq);
      uint32_t f = 0, qk = 0;                  // tiles and queries with keys so far
#pragma unroll 1
      while (k < nu && ok) {
        const TaUnitRaw nraw = k + 1 < nu ? ta_unit_load(P, unit_q(k + 1)) : TaUnitRaw{};
#pragma unroll 1
        for (int t = 0; t < u.ntile && ok; ++t, ++f) {
          const TaTile g = ta_tile_u(u, t);
          const int nbox = (g.we - g.wa) / TA_WBOX;
          // window boxes overwrite the K tile: only once the previous tile's O MMAs have completed
          if (f > 0 && nbox > 0) ok = mbar_wait(&S.bar_o[3], (f - 1) & 1);
#pragma unroll 1
          for (int j = 0; j < 8; ++j) {
            mbar_arrive_expect_tx(&S.bar_w[j], (uint32_t)(nbox * TA_WBOX * 128));
            if (ok)
              for (int i = 0; i < nbox; ++i)
                tma_load_3d(&S.K[j][(g.wa + i * TA_WBOX) * 128], &wmap, j * 64,
                            (int)(g.wrow_base + g.wa + i * TA_WBOX), u.b, &S.bar_w[j]);
          }
          // S^T = K Q^T, dim block by dim block as the blocks land.  At N = 64 the tensor pipe keeps up with
          // one MMA per ~75 cycles only when they are issued back to back: the loops are unrolled, the
          // descriptors advance by adds, and a landed block costs a non-blocking test, not a wait.
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            if (ok && !((t > 0 || mbar_test(&S.bar_q[j], qk & 1)) && mbar_test(&S.bar_w[j], f & 1) &&
                        mbar_test(&S.bar_k[j], f & 1)))
              ok = (t > 0 || mbar_wait(&S.bar_q[j], qk & 1)) && mbar_wait(&S.bar_w[j], f & 1) &&
                   mbar_wait(&S.bar_k[j], f & 1);
            if (ok) {
              tc_fence_after();
#pragma unroll
              for (int s2 = 0; s2 < 4; ++s2)
                mma_bf16_ss(tb + TA_COL_S, kdesc + (uint64_t)((j * TA_KEYS * 128 + s2 * 32) >> 4),
                            qdesc + (uint64_t)((j * 64 * 128 + s2 * 32) >> 4), ids, (j | s2) != 0);
            }
          }
          mma_commit(&S.bar_s);
          if (t + 1 == u.ntile && k + 1 < nu && ok) {
            // the next query with keys; its Q replaces this one's once this tile's S MMAs have read it
            int kn = k + 1;
            TaUnit un = ta_unit(P, nraw);
            while (un.ntile == 0 && ++kn < nu) un = ta_unit(P, ta_unit_load(P, unit_q(kn)));
            if (kn < nu) {
              ok = mbar_wait(&S.bar_s, f & 1);
              if (ok) load_q(un.bq);
            }
          }
          // O^T (+)= V^T P^T; the first tile of a query starts its accumulator afresh (the previous
          // query's epilogue has read it: the workers arrive on bar_p only after that)
          ok = ok && mbar_wait(&S.bar_p, f & 1);
          if (ok) tc_fence_after();
#pragma unroll
          for (int mt = 0; mt < 4; ++mt) {
            if (ok) {
#pragma unroll
              for (int s2 = 0; s2 < 8; ++s2)
                mma_bf16_ss(tb + TA_COL_O + 64 * mt, vdesc + (uint64_t)((2 * mt * TA_KEYS * 128 + s2 * 2048) >> 4),
                            pdesc + (uint64_t)((s2 * 2048) >> 4), ido, t > 0 || s2 > 0);
            }
            mma_commit(&S.bar_o[mt]);
          }
        }
        ++qk;
        // advance to the next query with keys (the same scan as above)
        int kn = k + 1;
        TaUnit un{};
        if (kn < nu) {
          un = ta_unit(P, nraw);
          while (un.ntile == 0 && ++kn < nu) un = ta_unit(P, ta_unit_load(P, unit_q(kn)));
        }
        k = kn;
        u = un;
      }
      if (!ok) atomicOr(&S.err, 1u);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------------------------- workers
    const int quad = warp & 3, hh = warp >> 2;
    const int key = 32 * quad + lane;
    const uint32_t lane_base = tb + ((uint32_t)(32 * quad) << 16);
    bool ok = true;
    uint4 cv[7], sc16, rp[4];
    auto load_row = [&](int b, int id) {
#pragma unroll
      for (int j = 0; j < 7; ++j) cv[j] = make_uint4(0, 0, 0, 0);
      sc16 = make_uint4(0, 0, 0, 0);
#pragma unroll
      for (int c = 0; c < 4; ++c) rp[c] = make_uint4(0, 0, 0, 0);
      const long long r = id >= 0 ? page_row(P.pm, b, P.n_max, id) : -1;
      if (r >= 0) {
        const uint8_t* crow = P.codes + (size_t)r * 224 + ghalf * 16;
#pragma unroll
        for (int j = 0; j < 7; ++j) cv[j] = __ldg(reinterpret_cast<const uint4*>(crow + j * 32));
        sc16 = __ldg(reinterpret_cast<const uint4*>(P.scales + (size_t)r * 16));
        const uint4* rrow = reinterpret_cast<const uint4*>(P.rope + (size_t)r * 64) + ghalf * 4;
#pragma unroll
        for (int c = 0; c < 4; ++c) rp[c] = __ldg(rrow + c);
      }
    };
    auto raw_id = [&](const TaUnit& uu, const TaTile& gg) -> int {
      if (grow >= gg.rs) return -1;
      const int li = gg.key0 + grow;
      return P.hca ? li : (li < P.k ? P.idx[(size_t)uu.bq * P.k + li] : -1);
    };
    auto check_id = [&](const TaUnit& uu, int v) -> int { return (v >= 0 && v < uu.ncb) ? v : -1; };
    // the first query with keys at or after unit kk (from its raw positions, if they are those of unit
    // kk), writing the outputs of the ones without keys; bq = -1 if there is none
    auto next_unit = [&](int kk, TaUnitRaw raw) -> TaUnit {
      return ta_next_unit(P, kk, nu, raw, tid, TA_WORKERS);
    };
    auto unit_index = [&](const TaUnit& uu) { return uu.bq < 0 ? nu : (uu.uid - (int)blockIdx.x) / (int)gridDim.x; };
    auto epilogue = [&](int uid, uint32_t par) { ok = ta_epilogue(S, P, uid, par, lane_base, hh, quad, lane, tid) && ok; };

    TaUnit u = nu > 0 ? next_unit(0, ta_unit_load(P, unit_q(0))) : TaUnit{};
    if (nu == 0) u.bq = -1;
    int k = unit_index(u);
    int bq_done = -1;                           // unit (uid) awaiting its epilogue
    TaUnitRaw nraw{};
    nraw.uid = -1;
    if (k + 1 < nu) nraw = ta_unit_load(P, unit_q(k + 1));
    int id = -1;
    if (k < nu) {
      id = check_id(u, raw_id(u, ta_tile_u(u, 0)));
      load_row(u.b, id);
    }
    uint32_t f = 0;
    int t = 0;
#pragma unroll 1
    while (k < nu) {
      // the tile after this one (this query's next, or the next query's first): its id is read now and
      // its row after this tile's gather
      int kn = k, tn = t + 1;
      TaUnit un = u;
      if (tn == u.ntile) {
        un = next_unit(k + 1, nraw);
        kn = unit_index(un);
        tn = 0;
      }
      const bool more = kn < nu;
      const int raw_next = more ? raw_id(un, ta_tile_u(un, tn)) : -1;
      const TaTile g = ta_tile_u(u, t);

      // ---- gather: the K tile is refilled block by block as the previous tile's O MMAs release it
      const bool pure = g.rs == TA_KEYS;
      if (f > 0 && !pure) {
#pragma unroll 1
        for (int mt = 0; mt < 4; ++mt) ok = ok && mbar_wait(&S.bar_o[mt], (f - 1) & 1);
        tc_fence_after();
      }
      if (ghalf == 0) S.ids[grow] = id;
      if (!pure) {
        const int r_end = min(g.wa, g.rw);
        const int n = (r_end > g.rs ? r_end - g.rs : 0) * 64;
        for (int i = tid; i < n; i += TA_WORKERS) {
          const int row = g.rs + (i >> 6), c = i & 63;
          const long long wr = g.wrow_base + row;
          cp16(&S.K[c >> 3][sw128(row, c & 7)], P.win + ((size_t)u.b * P.Wn + wr) * 512 + c * 8);
        }
        for (int i = tid; i < (TA_KEYS - g.zs) * 64; i += TA_WORKERS) {
          const int row = g.zs + (i >> 6), c = i & 63;
          *reinterpret_cast<uint4*>(&S.K[c >> 3][sw128(row, c & 7)]) = make_uint4(0, 0, 0, 0);
        }
        asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
      }
#pragma unroll
      for (int j = 0; j < 7; ++j) {
        if (f > 0 && pure && (j & 1) == 0) {
          ok = ok && mbar_wait(&S.bar_o[j >> 1], (f - 1) & 1);
          tc_fence_after();
        }
        if (grow < g.rs) {
          const int part = 2 * j + ghalf;
          const uint32_t word = (j >> 1) == 0 ? sc16.x : (j >> 1) == 1 ? sc16.y : (j >> 1) == 2 ? sc16.z : sc16.w;
          const uint32_t sb = f_to_bf16_bits(e4m3_to_f32((word >> ((part & 3) * 8)) & 0xFFu) * P.g);
          const uint32_t sc2 = sb | (sb << 16);
          const uint32_t w4[4] = {cv[j].x, cv[j].y, cv[j].z, cv[j].w};
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4)
            *reinterpret_cast<uint4*>(&S.K[j][sw128(grow, ghalf * 4 + q4)]) = e2m1x8_to_bf16_scaled(w4[q4], sc2);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.bar_k[j]);
      }
      if (f > 0 && pure) {
        ok = ok && mbar_wait(&S.bar_o[3], (f - 1) & 1);
        tc_fence_after();
      }
      if (grow < g.rs) {
#pragma unroll
        for (int c = 0; c < 4; ++c) *reinterpret_cast<uint4*>(&S.K[7][sw128(grow, ghalf * 4 + c)]) = rp[c];
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.bar_k[7]);
      // the next tile's row, in flight during this tile's softmax and MMAs
      if (more) {
        id = check_id(un, raw_next);
        load_row(un.b, id);
      }
      // what the softmax needs of this tile; then the cursor moves on (one query's geometry stays live)
      const int rs_t = g.rs, rw_t = g.rw, t_cur = t;
      const int bq_ends = t + 1 == u.ntile ? u.uid : -1;
      k = kn;
      t = tn;
      u = un;
      asm volatile("bar.sync 1, 256;" ::: "memory");   // workers only: ids visible to the softmax

      // ---- the previous query's epilogue: its last O MMAs completed before this tile's gather
      if (bq_done >= 0) {
        epilogue(bq_done, (f - 1) & 1);
        bq_done = -1;
      }

      // ---- softmax of this tile (as in the per-query kernel)
      ok = ok && mbar_wait(&S.bar_s, f & 1);
      tc_fence_after();
      const bool valid = key < rs_t ? (S.ids[key] >= 0) : (key < rw_t);
      float red[32];
      {
        uint32_t sv[32];
        tmem_ld_x32(lane_base + TA_COL_S + hh * 32, sv);
        tmem_wait_ld_x32(sv);
#pragma unroll
        for (int j = 0; j < 32; ++j) red[j] = valid ? __uint_as_float(sv[j]) * P.scale_log2 : -INFINITY;
      }
      S.red_m[quad][hh * 32 + lane] = transpose_reduce32<true>(red, lane);
      asm volatile("bar.sync 1, 256;" ::: "memory");
      if (tid < 64) {
        const float mt = fmaxf(fmaxf(S.red_m[0][tid], S.red_m[1][tid]), fmaxf(S.red_m[2][tid], S.red_m[3][tid]));
        const float mo = S.m[tid];
        float mn = mo, fc = 1.f;
        if (mt > mo + TA_RESCALE_SLACK || (mo == -INFINITY && mt > -INFINITY)) {
          mn = mt;
          fc = mo == -INFINITY ? 0.f : exp2f(mo - mn);
        }
        S.m[tid] = mn;
        S.fac[tid] = fc;
        S.l[tid] *= fc;
        if (fc != 1.f && t_cur > 0) S.rescale = 1;
      }
      asm volatile("bar.sync 1, 256;" ::: "memory");
      if (t_cur > 0 && S.rescale) {
#pragma unroll 1
        for (int mt = 0; mt < 4; ++mt) {
          uint32_t ov[32];
          tmem_ld_x32(lane_base + TA_COL_O + 64 * mt + hh * 32, ov);
          tmem_wait_ld_x32(ov);
#pragma unroll
          for (int j = 0; j < 32; ++j) ov[j] = __float_as_uint(__uint_as_float(ov[j]) * S.fac[hh * 32 + j]);
          tmem_st_x32(lane_base + TA_COL_O + 64 * mt + hh * 32, ov);
        }
        tmem_wait_st();
      }
      {
        uint32_t sv[32];
        tmem_ld_x32(lane_base + TA_COL_S + hh * 32, sv);
        tmem_wait_ld_x32(sv);
        uint32_t pk[16];
        float mh[32];
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
          const float4 v4 = *reinterpret_cast<const float4*>(&S.m[hh * 32 + j]);
          mh[j] = v4.x; mh[j + 1] = v4.y; mh[j + 2] = v4.z; mh[j + 3] = v4.w;
        }
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          const float m0 = mh[j], m1 = mh[j + 1];
          const float z0 = valid ? __uint_as_float(sv[j]) * P.scale_log2 : -INFINITY;
          const float z1 = valid ? __uint_as_float(sv[j + 1]) * P.scale_log2 : -INFINITY;
          const float p0f = m0 == -INFINITY ? 0.f : ta_exp2(z0 - m0);
          const float p1f = m1 == -INFINITY ? 0.f : ta_exp2(z1 - m1);
          red[j] = p0f;
          red[j + 1] = p1f;
          pk[j >> 1] = pack_bf16x2(p0f, p1f);
        }
#pragma unroll
        for (int c = 0; c < 4; ++c)
          *reinterpret_cast<uint4*>(&S.P[sw128(key, hh * 4 + c)]) =
              make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.bar_p);
      S.red_l[quad][hh * 32 + lane] = transpose_reduce32<false>(red, lane);
      asm volatile("bar.sync 1, 256;" ::: "memory");
      if (tid < 64) S.l[tid] += (S.red_l[0][tid] + S.red_l[1][tid]) + (S.red_l[2][tid] + S.red_l[3][tid]);
      if (tid == 0) S.rescale = 0;
      asm volatile("bar.sync 1, 256;" ::: "memory");

      if (bq_ends >= 0) {
        bq_done = bq_ends;
        // positions of the query after the next one, read now and used when the next one ends
        nraw.uid = -1;
        if (k + 1 < nu) nraw = ta_unit_load(P, unit_q(k + 1));
      }
      ++f;
    }
    if (bq_done >= 0) epilogue(bq_done, (f - 1) & 1);
    if (!ok && lane == 0) atomicOr(&S.err, 1u);
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 8) {
    if (S.err && lane == 0) atomicOr(&g_csa_device_error, 1u);
    tc_fence_after();
    tmem_dealloc(tb, TA_TMEM_COLS);
  }
}

// Early window (CSA_EARLY_START): split 0 of each query, placed first in the grid, attends over the
// window tile before the step's index and top-k kernels have ended; possible when the window fills one
// tile right after the k entries (k a multiple of the tile, at most one tile of window).
bool attn_tc_early(const csa_attn_args* a, int hca) {
  const long long n_win = attn_has_window(a) ? (a->Wn < a->window ? a->Wn : a->window) : 0;
  return !hca && (a->flags & CSA_EARLY_START) && n_win > 0 && n_win <= TA_KEYS && a->k > 0 && a->k % TA_KEYS == 0;
}

// The persistent kernel (one CTA per SM walking units back to back) takes the plans with BF16 window rows,
// no early window and at least two tiles per SM on average; HCA (entries streamed from HBM in order) only
// with more queries than SMs, as the per-query kernel measured faster for few long HCA queries.
static bool attn_tc_persist_ok(const csa_attn_args* a, int hca, long long rows, long long tiles) {
  return (hca ? rows > 148 : rows * tiles >= 2 * 148) && rows <= 0x7fffffffLL && a->win_format == CSA_WIN_BF16 && !attn_tc_early(a, hca);
}

// Tiles per unit for the persistent kernel: units (query, split) are dealt to the CTAs in turn, so the
// plan that finishes first is found by adding up each CTA's units.  Costs in tile-times (≈ 6.9 µs): a unit
// its tiles plus an epilogue of TA_EPI_TILES; splitting adds the merge launch (TA_MERGE_TILES) and each
// unit's partial (H rows of 512 bf16) written and read back at the HBM rate (≈ 6 TB/s).  Queries enough
// to keep every CTA busy with whole queries stay unsplit.
constexpr double TA_EPI_TILES = 0.4, TA_MERGE_TILES = 0.5, TA_TILE_US = 6.9, TA_HBM_BYTES_PER_US = 6.0e6;
static int attn_tc_persist_tpc(long long rows, long long tiles, int H) {
  const double part_tiles = (double)H * 512 * 2 * 2 / (TA_HBM_BYTES_PER_US * TA_TILE_US);
  if (rows >= 4 * 148) return (int)tiles;
  double best = 1e300;
  long long best_tpc = tiles;
  const long long max_splits = tiles < 32 ? tiles : 32;
  for (long long sp = 1; sp <= max_splits; ++sp) {
    const long long tpc = (tiles + sp - 1) / sp, splits = (tiles + tpc - 1) / tpc;
    if (splits != sp || rows * splits > 0x7fffffffLL) continue;   // the same plan as a smaller split count
    const long long units = rows * splits, grid = units < 148 ? units : 148;
    double worst = 0.0;
    for (long long c = 0; c < grid; ++c) {
      double load = 0.0;
      for (long long uid = c; uid < units; uid += grid) {
        const long long sidx = uid % splits, nt = tiles - sidx * tpc < tpc ? tiles - sidx * tpc : tpc;
        load += (double)nt + TA_EPI_TILES;
      }
      if (load > worst) worst = load;
    }
    if (splits > 1) worst += TA_MERGE_TILES + (double)units * part_tiles;
    if (worst < best - 1e-9) {
      best = worst;
      best_tpc = tpc;
    }
  }
  return (int)best_tpc;
}

// Key tiles per query and the CTAs that share them.  Per-query kernel: one tile per CTA while the grid fits
// one wave of the 148 SMs, else enough tiles per CTA (walked in order, online softmax) to come back to one
// wave; with the early window the entry tiles alone are planned this way and split 0 also takes the window
// tile (first, while the previous kernel still runs).  Persistent kernel: see attn_tc_persist_tpc.
void attn_tc_plan(const csa_attn_args* a, int hca, int* splits, int* tpc) {
  const bool early = attn_tc_early(a, hca);
  const long long n_win = attn_has_window(a) ? (a->Wn < a->window ? a->Wn : a->window) : 0;
  const long long n = (hca ? a->n_max : a->k) + (early ? 0 : n_win);
  const long long tiles = n > 0 ? (n + TA_KEYS - 1) / TA_KEYS : 1;
  const long long rows = (long long)a->B * a->Nq;
  long long t;
  if (attn_tc_persist_ok(a, hca, rows, tiles)) {
    t = attn_tc_persist_tpc(rows, tiles, a->H);
  } else {
    t = (rows * tiles + 147) / 148;
    if (t < 1) t = 1;
    if (t > tiles) t = tiles;
  }
  *tpc = (int)t;
  *splits = (int)((tiles + t - 1) / t);
}

// The persistent kernel's plans (the same decision attn_tc_plan made).
bool attn_tc_persistent(const csa_attn_args* a, int hca, int splits) {
  (void)splits;
  const bool early = attn_tc_early(a, hca);
  const long long n_win = attn_has_window(a) ? (a->Wn < a->window ? a->Wn : a->window) : 0;
  const long long n = (hca ? a->n_max : a->k) + (early ? 0 : n_win);
  const long long tiles = n > 0 ? (n + TA_KEYS - 1) / TA_KEYS : 1;
  return attn_tc_persist_ok(a, hca, (long long)a->B * a->Nq, tiles);
}

// Queries split over 2..8 CTAs can merge inside a thread-block cluster (CSA_CLUSTER_MERGE: no workspace,
// no merge kernel).
bool attn_tc_cluster(int splits) { return splits >= 2 && splits <= TA_MAX_CLUSTER; }

bool attn_tc_eligible(const csa_attn_args* a, int hca, int max_splits) {
  int splits = 0, tpc = 0;
  attn_tc_plan(a, hca, &splits, &tpc);
  return a->d == 512 && a->d_rope == 64 && a->H <= 64 && splits >= 1 && splits <= max_splits &&
         ((uintptr_t)a->q & 15) == 0 && (a->n_max == 0 || (((uintptr_t)a->kv_codes & 15) == 0 &&
                                                           ((uintptr_t)a->kv_rope & 15) == 0)) &&
         (a->win_format == CSA_WIN_FP8
              ? (!attn_has_window(a) || ((((uintptr_t)a->win_codes | (uintptr_t)a->win_scales | (uintptr_t)a->win_rope) &
                                          15) == 0))
              : (!a->win_kv || a->Wn == 0 || ((uintptr_t)a->win_kv & 15) == 0)) &&
         tensor_map_encoder() != nullptr;
}

csa_status launch_attn_tc(const csa_attn_args* a, int hca, int splits, int tpc, uint16_t* part_o,
                          float* part_lse, cudaStream_t st) {
  const long long rows = (long long)a->B * a->Nq;
  CUtensorMap qmap, wmap;
  {
    const cuuint64_t gdim[3] = {512, (cuuint64_t)a->H, (cuuint64_t)rows};
    const cuuint64_t gstride[2] = {1024, (cuuint64_t)a->H * 1024};
    const cuuint32_t box[3] = {64, 64, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    if (tensor_map_encoder()(&qmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, (void*)a->q, gdim, gstride, box, estr,
                             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return CSA_ERR_CUDA;
  }
  const bool fp8 = a->win_format == CSA_WIN_FP8;
  const int Wn = attn_has_window(a) ? a->Wn : 0;
  if (Wn > 0 && !fp8) {
    const cuuint64_t gdim[3] = {512, (cuuint64_t)Wn, (cuuint64_t)a->B};
    const cuuint64_t gstride[2] = {1024, (cuuint64_t)Wn * 1024};
    const cuuint32_t box[3] = {64, TA_WBOX, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    if (tensor_map_encoder()(&wmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, (void*)a->win_kv, gdim, gstride, box, estr,
                             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return CSA_ERR_CUDA;
  } else {
    memset(&wmap, 0, sizeof(wmap));            // never read: no window rows
  }
  TaParams P{};
  P.Nq = a->Nq; P.H = a->H; P.ratio = a->ratio; P.n_max = a->n_max; P.k = hca ? 0 : a->k; P.rows = (int)rows;
  P.Wn = Wn; P.window = a->window; P.splits = splits; P.tpc = tpc; P.hca = hca; P.g = a->g_kv;
  P.early_rows = attn_tc_early(a, hca) ? (int)rows : 0;
  P.cluster = (attn_tc_cluster(splits) && (a->flags & CSA_CLUSTER_MERGE)) ? 1 : 0;
  const float scale = a->softmax_scale != 0.0f ? a->softmax_scale : 1.0f / sqrtf((float)a->d);
  P.scale_log2 = scale * TA_LOG2E;
  P.q_pos = a->q_pos; P.codes = a->kv_codes; P.scales = a->kv_scales;
  P.rope = (const uint16_t*)a->kv_rope; P.n_c = a->n_c; P.idx = hca ? nullptr : a->idx; P.win = (const uint16_t*)a->win_kv;
  P.win_pos0 = a->win_pos0; P.out = (uint16_t*)a->out; P.lse = a->lse; P.part_o = part_o; P.part_lse = part_lse;
  P.win_fp8 = fp8 ? 1 : 0;
  P.pm = a->kv_pages;
  if (fp8) {
    P.win = nullptr;
    P.wcodes = a->win_codes;
    P.wscales = a->win_scales;
    P.wrope = (const uint16_t*)a->win_rope;
  }
  const int smem = (int)sizeof(TaSmem) + 1024;
  if (attn_tc_persistent(a, hca, splits)) {
    // one persistent CTA per SM walks its units (query, split) back to back
    int sms = 148;
    {
      int dev = 0;
      if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    }
    static std::atomic<unsigned> attr_done_p{0};
    set_smem_once((const void*)attn_tc_persist_kernel, smem, attr_done_p);
    const long long units = rows * splits;
    const unsigned grid = (unsigned)(units < sms ? units : sms);
    return launch_pdl(attn_tc_persist_kernel, dim3(grid), dim3(TA_THREADS), (size_t)smem, st, qmap, wmap, P);
  }
  static std::atomic<unsigned> attr_done{0};
  static std::atomic<unsigned> attr_done8{0};
  auto* kfn = fp8 ? attn_tc_kernel<true> : attn_tc_kernel<false>;
  set_smem_once((const void*)kfn, smem, fp8 ? attr_done8 : attr_done);
  if (!P.cluster)
    return launch_pdl(kfn, dim3((unsigned)(rows * splits)), dim3(TA_THREADS), (size_t)smem, st, qmap, wmap, P);
  cudaLaunchAttribute attr[2];
  cudaLaunchConfig_t cfg = pdl_config(dim3((unsigned)(rows * splits)), dim3(TA_THREADS), (size_t)smem, st, attr);
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = (unsigned)splits;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.numAttrs = 2;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kfn, qmap, wmap, P);
  if (e != cudaSuccess) {
    set_last_cuda_error(e);
    return CSA_ERR_CUDA;
  }
  return launch_status();
}


}  // namespace csa
