// Lightning indexer (FP4 multi-head ReLU dot product), per-query top-k, Reindex over a candidate list,
// and the hierarchical candidate pool.
// Sources: "DeepSeek-V4: エージェントが実際に使える100万トークンのコンテキスト", §ハイブリッド注意, Fig. 3 (an FP4
// indexer with ReLU scores and several heads picks the top-k compressed blocks per query);
// "DeepSeek-V4.1-Flash - Pushing the Limits of KV Cache Compression", CSA2 bullet + Fig. 4 (Reindex
// re-scores the previous layer's keys with this layer's query) and the Hierarchical Sparse Indexer
// bullet + Fig. 5 (blocks of positions ranked by their best score form a candidate pool).
//
// Score of key i for query (b, t):
//   s = g_q g_k sum_h w_h max(0, sum_blk sq[h][blk] sk[i][blk] sum_{e in blk} q_e k_e)
// Computed on the tensor pipe with mma.sync m16n8k16 (f16 in, fp32 accumulate): A = 16 keys, each
// element the exact f16 product e2m1(k_e)*sk, B = the 8 indexer heads of one query, each element
// e2m1(q_e)*sq.  The products are exact; the fp32 sums over the 128 elements are the kernel's only
// rounding.  Each thread of a quad owns one 32-element scale block of its two key rows, so the key
// side needs one 128-bit load per row and one scale byte.
#include "csa_common.cuh"
#include "sm100.cuh"

namespace csa {

constexpr int IDX_HEADS = 8;           // MMA N: indexer heads, padded with zero heads
constexpr int IDX_WARPS = 4;
constexpr int IDX_TARGET_CTAS = 148 * 4;  // about one wave of resident CTAs
constexpr int IDX_QT = 32;             // max queries per CTA (query fragments staged in shared memory)
constexpr int TOPK_THREADS = 1024;
constexpr int TOPK_CHUNK = 32768;      // max row length held in shared memory (implicit ids)
constexpr int TOPK_CHUNK_IDS = 16384;  // max row length with explicit ids
constexpr int TOPK_SHORT = 8192;        // rows up to this length go to the 256-thread kernel
constexpr int HIST_BINS = 4096;        // score histogram: top 12 bits of the order-preserving key
constexpr int HIST_SHIFT = 20;

// ---------------------------------------------------------------------------- query quantisation
// One warp per (query, head) row of q_I: FP4 pack rule (global scale g_q), then the f16 products
// e2m1(q_e)*sq (exact in f16) written to the CTA's query tile; heads >= H_I are zero.
// w' = w * g_q * g_k (the global scales factor out of the ReLU: both are positive).
__device__ void quantize_query_tile(const uint16_t* __restrict__ qI, const float* __restrict__ w, int row0, int nq,
                                    int H_I, int d_I, float g_q, float gg, __half* s_q, float* s_w) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const float six_g = 6.0f * g_q;
  for (int rh = warp; rh < nq * IDX_HEADS; rh += nw) {
    const int qq = rh / IDX_HEADS, h = rh % IDX_HEADS;
    __half* dst = s_q + (size_t)rh * d_I;
    if (h >= H_I) {
      for (int e = lane; e < d_I; e += 32) dst[e] = __float2half(0.0f);
      if (lane == 0) s_w[rh] = 0.0f;
      continue;
    }
    const uint16_t* src = qI + ((size_t)(row0 + qq) * H_I + h) * d_I;
    for (int blk = 0; blk < d_I / 32; ++blk) {
      const float x = bf16_bits_to_f(src[blk * 32 + lane]);
      const float amax = warp_max(fabsf(x));
      const uint32_t s_code = f32_to_e4m3(__fdiv_rn(amax, six_g));
      const float sv = e4m3_to_f32(s_code);
      uint32_t code = 0;
      if (sv != 0.0f) code = f32_to_e2m1(__fdiv_rn(x, __fmul_rn(sv, g_q)));
      dst[blk * 32 + lane] = __float2half(e2m1_value(code) * sv);
    }
    if (lane == 0) s_w[rh] = w[(size_t)(row0 + qq) * H_I + h] * gg;
  }
}

// ------------------------------------------------------------------------------------- scoring
__device__ __forceinline__ void mma_f16(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <int DI>
struct KeyRow {
  // DI = 128: a thread holds one 32-element block (16 bytes); DI = 64: half a block (8 bytes).
  static constexpr int BYTES = DI == 128 ? 16 : 8;
  static constexpr int REGS = BYTES;  // one f16x2 per code byte
  uint32_t w[BYTES / 4];
};

template <int DI>
__device__ __forceinline__ void load_key(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales,
                                         long long key, bool valid, int t, KeyRow<DI>& raw, uint32_t& sc) {
  constexpr int S_PAD = ((DI / 32) + 3) & ~3;
  if (!valid) {
#pragma unroll
    for (int i = 0; i < KeyRow<DI>::BYTES / 4; ++i) raw.w[i] = 0;
    sc = 0;
    return;
  }
  const uint8_t* p = codes + (size_t)key * (DI / 2) + t * KeyRow<DI>::BYTES;
  if constexpr (DI == 128) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(p));
    raw.w[0] = v.x; raw.w[1] = v.y; raw.w[2] = v.z; raw.w[3] = v.w;
    sc = __ldg(scales + (size_t)key * S_PAD + t);
  } else {
    const uint2 v = __ldg(reinterpret_cast<const uint2*>(p));
    raw.w[0] = v.x; raw.w[1] = v.y;
    sc = __ldg(scales + (size_t)key * S_PAD + (t >> 1));
  }
}

template <int DI>
__device__ __forceinline__ void convert_key(const KeyRow<DI>& raw, uint32_t sc, uint32_t* a) {
  const uint32_t s2 = e4m3_to_h2_splat(sc);
#pragma unroll
  for (int i = 0; i < KeyRow<DI>::BYTES; ++i) a[i] = hmul2_bits(e2m1x2_to_h2(raw.w[i >> 2] >> ((i & 3) * 8)), s2);
}

// Grid: x = key range (4 warps x tpw tiles of 16 keys or candidates), y = query tile, z = sequence.
// cand != nullptr: Reindex mode, one query per CTA, keys gathered by id.  Dynamic shared memory holds
// the tile's query fragments [qt][IDX_HEADS][DI] f16.
template <int DI>
__global__ void __launch_bounds__(IDX_WARPS * 32) index_score_kernel(
    const uint16_t* __restrict__ q_I, const float* __restrict__ w, int H_I, float g_q, float gg, int Nq, int qt,
    const uint8_t* __restrict__ k_codes, const uint8_t* __restrict__ k_scales, int n_max,
    const int32_t* __restrict__ n_c, const int64_t* __restrict__ q_pos, int ratio,
    const int32_t* __restrict__ cand, int n_cand, float* __restrict__ scores, long long ld, int tpw,
    uint32_t* __restrict__ hist, const csa_page_map pm) {
  constexpr int STEPS = DI / 16;
  constexpr int BREGS = DI / 8;           // f16x2 registers of one head slice per thread
  constexpr int S_PAD = ((DI / 32) + 3) & ~3;
  extern __shared__ __align__(16) uint8_t s_dyn[];
  __half* s_q = reinterpret_cast<__half*>(s_dyn);          // [qt][IDX_HEADS][DI]
  // single-query CTAs may also count their scores in HIST_BINS bins (key >> HIST_SHIFT) for the top-k
  uint32_t* s_hist = reinterpret_cast<uint32_t*>(s_dyn + (size_t)qt * IDX_HEADS * DI * 2);
  __shared__ float s_w[IDX_QT][IDX_HEADS];
  __shared__ int s_nvis[IDX_QT];
  __shared__ long long s_t[IDX_QT];

  const int b = blockIdx.z;
  const int q0 = cand ? blockIdx.y : blockIdx.y * qt;
  const int nq = cand ? 1 : min(qt, Nq - q0);
  const int ncb = min(n_c[b], n_max);   // entries beyond the cache capacity do not exist
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int keys_per_cta = IDX_WARPS * tpw * 16;
  const int chunk0 = blockIdx.x * keys_per_cta;
  const int n_cols = cand ? n_cand : n_max;
  if (chunk0 >= n_cols) return;

  quantize_query_tile(q_I, w, b * Nq + q0, nq, H_I, DI, g_q, gg, s_q, &s_w[0][0]);
  if (hist)
    for (int i = tid; i < HIST_BINS; i += blockDim.x) s_hist[i] = 0;
  int max_vis = 0;
  for (int qq = 0; qq < nq; ++qq) {
    const long long tq = q_pos[(size_t)b * Nq + q0 + qq];
    long long nv = (tq + 1) / ratio;
    if (nv > ncb) nv = ncb;
    if (nv < 0) nv = 0;
    if (tid == 0) { s_nvis[qq] = (int)nv; s_t[qq] = tq; }
    max_vis = max(max_vis, (int)nv);
  }
  __syncthreads();
  if (!cand && chunk0 >= max_vis) return;

  const int chunk_end = min(n_cols, chunk0 + keys_per_cta);
  const int col_end = cand ? chunk_end : min(chunk_end, max_vis);
  const int32_t* cand_row = cand ? cand + ((size_t)b * Nq + q0) * n_cand : nullptr;
  const long long t0 = s_t[0];

  // key = the row of the key's codes / scales in the (contiguous or paged) cache arrays
  auto key_of = [&](int col, long long& key, bool& ok) {
    int id;
    if (cand_row) {
      id = col < col_end ? cand_row[col] : -1;
      ok = id >= 0 && id < ncb && (long long)ratio * id + ratio - 1 <= t0;
    } else {
      id = col;
      ok = col < col_end && col < ncb;
    }
    key = ok ? page_row(pm, b, n_max, id) : -1;
    ok = ok && key >= 0;
  };

  const int first_col = chunk0 + warp * tpw * 16;
  uint32_t bq0[BREGS];
  {
    const uint4* bq = reinterpret_cast<const uint4*>(s_q + (size_t)g * DI + t * (DI / 4));
#pragma unroll
    for (int i = 0; i < BREGS / 4; ++i) {
      const uint4 v = bq[i];
      bq0[4 * i] = v.x; bq0[4 * i + 1] = v.y; bq0[4 * i + 2] = v.z; bq0[4 * i + 3] = v.w;
    }
  }
  long long key[2][2];
  bool kval[2][2];
  KeyRow<DI> raw[2][2];
  uint32_t sc[2][2];
  // software pipeline: raw[cur] holds the tile being converted, raw[cur ^ 1] the next tile in flight
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    key_of(first_col + g + 8 * h, key[0][h], kval[0][h]);
    load_key<DI>(k_codes, k_scales, key[0][h], kval[0][h], t, raw[0][h], sc[0][h]);
  }
#pragma unroll 2
  for (int tile = 0; tile < tpw; ++tile) {
    const int cur = tile & 1;
    const int col0 = first_col + tile * 16;
    if (col0 >= col_end) break;
    if (tile + 1 < tpw) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        key_of(col0 + 16 + g + 8 * h, key[cur ^ 1][h], kval[cur ^ 1][h]);
        load_key<DI>(k_codes, k_scales, key[cur ^ 1][h], kval[cur ^ 1][h], t, raw[cur ^ 1][h], sc[cur ^ 1][h]);
      }
    }
    uint32_t a[2][KeyRow<DI>::REGS];
#pragma unroll
    for (int h = 0; h < 2; ++h) convert_key<DI>(raw[cur][h], sc[cur][h], a[h]);

    for (int qq = 0; qq < nq; ++qq) {
      // B fragment: head g, elements [t*DI/4 + 4s, +4) for k16 step s -> one contiguous slice
      // (decode: one query, fragments loaded once before the tile loop)
      uint32_t bfr[BREGS];
      if (nq == 1) {
#pragma unroll
        for (int i = 0; i < BREGS; ++i) bfr[i] = bq0[i];
      } else {
        const uint4* bq = reinterpret_cast<const uint4*>(s_q + ((size_t)qq * IDX_HEADS + g) * DI + t * (DI / 4));
#pragma unroll
        for (int i = 0; i < BREGS / 4; ++i) {
          const uint4 v = bq[i];
          bfr[4 * i] = v.x; bfr[4 * i + 1] = v.y; bfr[4 * i + 2] = v.z; bfr[4 * i + 3] = v.w;
        }
      }
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int s = 0; s < STEPS; ++s) {
        const uint32_t af[4] = {a[0][2 * s], a[1][2 * s], a[0][2 * s + 1], a[1][2 * s + 1]};
        mma_f16(acc, af, bfr[2 * s], bfr[2 * s + 1]);
      }
      const float w0 = s_w[qq][2 * t], w1 = s_w[qq][2 * t + 1];
      float r0 = w0 * fmaxf(acc[0], 0.f) + w1 * fmaxf(acc[1], 0.f);
      float r1 = w0 * fmaxf(acc[2], 0.f) + w1 * fmaxf(acc[3], 0.f);
      r0 += __shfl_xor_sync(0xffffffffu, r0, 1);
      r0 += __shfl_xor_sync(0xffffffffu, r0, 2);
      r1 += __shfl_xor_sync(0xffffffffu, r1, 1);
      r1 += __shfl_xor_sync(0xffffffffu, r1, 2);
      if (t < 2) {
        const int col = col0 + g + 8 * t;
        const float v = (t ? r1 : r0) + 0.0f;
        float* row = scores + (size_t)(b * Nq + q0 + qq) * ld;
        bool counted = false;
        if (cand_row) {
          if (col < col_end) {
            const bool ok = t ? kval[cur][1] : kval[cur][0];
            row[col] = ok ? v : -INFINITY;
            counted = ok;
          }
        } else if (col < s_nvis[qq]) {
          row[col] = v;
          counted = true;
        }
        if (hist && counted) atomicAdd(&s_hist[float_order_key(v) >> HIST_SHIFT], 1u);
      }
    }
  }
  if (hist) {
    __syncthreads();
    uint32_t* h = hist + (size_t)(b * Nq + q0) * HIST_BINS;
    for (int i = tid; i < HIST_BINS; i += blockDim.x) {
      const uint32_t c = s_hist[i];
      if (c) atomicAdd(&h[i], c);
    }
  }
}

// ------------------------------------------------------------------------------------- top-k
// Block-wide selection over one row held in shared memory as order-preserving 32-bit keys.
// Total order: score desc, then key id asc, then position asc (ids repeat only in malformed
// candidate lists).  MSB-first radix passes with 8-bit digits find the threshold, then every element
// above it is emitted and the ties are taken in (id, position) order.

template <int NW>                           // warps of the block
struct TopkSmemT {
  uint32_t hist[256];
  uint32_t whist[NW][256];                  // per-warp histograms: contention only inside a warp
  uint32_t scan[NW];
  uint32_t bcast[4];
  uint32_t counter;
  uint32_t tie_taken;
};
using TopkSmem = TopkSmemT<TOPK_THREADS / 32>;

// Find the R-th largest value of key(j) over positions j < n with filt(j).  Returns the threshold
// key; *n_above = number of filtered elements with key > threshold.
template <class SM, class KeyF, class FiltF>
__device__ uint32_t radix_threshold(SM& sm, int n, uint32_t R, KeyF key, FiltF filt, uint32_t* n_above) {
  uint32_t prefix = 0, mask = 0, rem = R;
  for (int shift = 24; shift >= 0; shift -= 8) {
    const int nw = blockDim.x >> 5, wid = threadIdx.x >> 5;
    if (n <= 8192) {
      // few candidates: one block-wide histogram
      for (int i = threadIdx.x; i < 256; i += blockDim.x) sm.hist[i] = 0;
      __syncthreads();
      for (int j = threadIdx.x; j < n; j += blockDim.x) {
        if (!filt(j)) continue;
        const uint32_t k = key(j);
        if ((k & mask) == prefix) atomicAdd(&sm.hist[(k >> shift) & 255u], 1u);
      }
      __syncthreads();
    } else {
      for (int i = threadIdx.x; i < nw * 256; i += blockDim.x) (&sm.whist[0][0])[i] = 0;
      __syncthreads();
      // per-warp histograms: scores cluster in a few bins, so a block-wide histogram serialises
      uint32_t* wh = sm.whist[wid];
      for (int j = threadIdx.x; j < n; j += blockDim.x) {
        if (!filt(j)) continue;
        const uint32_t k = key(j);
        if ((k & mask) == prefix) atomicAdd(&wh[(k >> shift) & 255u], 1u);
      }
      __syncthreads();
      for (int i = threadIdx.x; i < 256; i += blockDim.x) {
        uint32_t c = 0;
        for (int w = 0; w < nw; ++w) c += sm.whist[w][i];
        sm.hist[i] = c;
      }
      __syncthreads();
    }
    if (threadIdx.x < 32) {
      // suffix sums over 256 bins: lane l owns bins [8l, 8l+8)
      const int l = threadIdx.x;
      uint32_t loc[8], tot = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) { loc[i] = sm.hist[8 * l + i]; tot += loc[i]; }
      // exclusive suffix over lanes: sum of totals of lanes > l
      uint32_t suf = tot;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_down_sync(0xffffffffu, suf, o);
        if (l + o < 32) suf += v;
      }
      uint32_t above = suf - tot;  // elements in bins of higher lanes
      int found = -1;
      uint32_t found_above = 0;
      for (int i = 7; i >= 0; --i) {
        if (found < 0 && above + loc[i] >= rem && above < rem) { found = 8 * l + i; found_above = above; }
        above += loc[i];
      }
      if (found >= 0) { sm.bcast[0] = (uint32_t)found; sm.bcast[1] = found_above; }
    }
    __syncthreads();
    const uint32_t digit = sm.bcast[0];
    rem -= sm.bcast[1];
    prefix |= digit << shift;
    mask |= 255u << shift;
    __syncthreads();
  }
  *n_above = R - rem;
  return prefix;
}

// Exclusive block scan of one value per thread; returns the prefix, *total = sum.
template <class SM>
__device__ uint32_t block_exclusive_scan(SM& sm, uint32_t v, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sm.scan[warp] = x;
  __syncthreads();
  if (warp == 0) {
    const int nw = blockDim.x >> 5;
    uint32_t s = lane < nw ? sm.scan[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    if (lane < nw) sm.scan[lane] = s;
  }
  __syncthreads();
  const uint32_t base = warp ? sm.scan[warp - 1] : 0;
  *total = sm.scan[(blockDim.x >> 5) - 1];
  __syncthreads();
  return base + x - v;
}

// One CTA per row.  Row r: scores at in_scores + r*in_ld, length len (from lens[r] or the visibility
// rule), ids from in_ids (explicit) or id = id_base + position.  Writes k slots of out_idx /
// out_scores at row r (stride k_out).
// Per-row state of the long-row histogram selection: scores emitted above the boundary bin, boundary-bin
// scores parked, CTAs finished, and whether the row was resolved (else the tournament selects it).
struct LongRowState {
  uint32_t up, at, done, ok;
};

struct TopkRowArgs {
  const float* in_scores;
  const int32_t* in_ids;
  long long in_ld;
  int n_cols;              // columns available in this call's rows
  int col_base;            // first column of the row segment (tournament chunks)
  const int64_t* q_pos;    // when lens come from visibility (may be null)
  const int32_t* n_c;
  int ratio, Nq, rows_per_seg;
  int k;
  int32_t* out_idx;
  float* out_scores;
  long long out_ld;
  const LongRowState* skip;   // rows whose state says resolved are left alone (null: none)
  int early;                  // histogram rows: q_pos and n_c are read before the wait (CSA_EARLY_START)
};


// Select the K largest of keys[0..len) (0 = not a candidate; nvalid candidates in all) by (key desc,
// id asc), writing ids / scores to oi[base + slot], os[base + slot] in unspecified order.  Candidates
// with equal key and equal id (a repeated id) are interchangeable: any of them gives the same output.
template <class SM, class IdF>
__device__ void select_in_smem(SM& sm, const uint32_t* keys, int len, uint32_t K, uint32_t nvalid, IdF idof,
                               int32_t* oi, float* os, uint32_t base) {
  auto valid = [&](int j) { return keys[j] != 0u; };
  uint32_t T1 = 0, above1 = 0, T2 = 0xFFFFFFFFu, need_pos = 0;
  bool all_ties = true;
  if (K > 0 && K < nvalid) {
    T1 = radix_threshold(sm, len, K, [&](int j) { return keys[j]; }, valid, &above1);
    const uint32_t need = K - above1;
    uint32_t tl = 0;
    for (int j = threadIdx.x; j < len; j += blockDim.x) tl += (keys[j] == T1);
    uint32_t nties;
    block_exclusive_scan(sm, tl, &nties);
    if (nties > need) {
      all_ties = false;
      uint32_t above2;
      T2 = radix_threshold(sm, len, need, [&](int j) { return ~idof(j); },
                           [&](int j) { return keys[j] == T1; }, &above2);
      need_pos = need - above2;
    }
  }
  if (threadIdx.x == 0) { sm.counter = 0; sm.tie_taken = 0; }
  __syncthreads();
  for (int j = threadIdx.x; j < len; j += blockDim.x) {
    const uint32_t kj = keys[j];
    if (kj == 0u) continue;
    bool take;
    if (K >= nvalid) take = true;
    else if (kj > T1) take = true;
    else if (kj < T1) take = false;
    else if (all_ties) take = true;
    else {
      const uint32_t k2 = ~idof(j);
      if (k2 > T2) take = true;
      else if (k2 < T2) take = false;
      else take = atomicAdd(&sm.tie_taken, 1u) < need_pos;
    }
    if (take) {
      const uint32_t slot = base + atomicAdd(&sm.counter, 1u);
      oi[slot] = (int32_t)idof(j);
      if (os) os[slot] = order_key_float(kj);
    }
  }
  __syncthreads();
}

// Load one row segment into shared memory as order-preserving keys (0 = not a candidate) and, with
// explicit ids, the ids; returns the number of candidates.  8 independent loads in flight per thread.
template <class SM>
__device__ uint32_t load_row_keys(SM& sm, const float* __restrict__ src, const int32_t* __restrict__ isrc,
                                  int len, uint32_t* keys, int32_t* ids) {
  uint32_t nvalid_loc = 0;
  constexpr int U = 8;
  for (int j0 = threadIdx.x; j0 < len; j0 += U * blockDim.x) {
    float v[U];
    int32_t id[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int j = j0 + u * blockDim.x;
      v[u] = j < len ? src[j] : -INFINITY;
      id[u] = (isrc && j < len) ? isrc[j] : 0;
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int j = j0 + u * blockDim.x;
      if (j >= len) continue;
      const bool ok = v[u] > -INFINITY && id[u] >= 0;
      keys[j] = ok ? float_order_key(v[u]) : 0u;
      if (isrc) ids[j] = id[u];
      nvalid_loc += ok;
    }
  }
  uint32_t nvalid;
  block_exclusive_scan(sm, nvalid_loc, &nvalid);
  return nvalid;
}

// THREADS x one row segment of at most CAP scores (CAP ids after them for explicit-id rows): the full
// 1024-thread kernel for segments up to 32768 scores, a 256-thread one with row-sized shared memory
// (several CTAs per SM) for rows of at most 8192 (multi-query prefill rows, candidate lists).
template <int THREADS, int CAP>
__global__ void __launch_bounds__(THREADS) topk_kernel(TopkRowArgs A) {
  extern __shared__ __align__(16) uint32_t s_keys[];
  __shared__ TopkSmemT<THREADS / 32> sm;
  const int seg = blockIdx.x;                  // segment (chunk) of the row
  const int row = blockIdx.y;
  pdl_trigger();
  pdl_wait();                                  // scores (and the long-row pass's flags) come from the previous kernel
  if (A.skip && A.skip[row].ok) return;        // selected by the long-row histogram pass
  const int col0 = A.col_base + seg * A.rows_per_seg;
  int len = min(A.rows_per_seg, A.n_cols - col0);
  if (A.q_pos) {
    const int b = row / A.Nq;
    long long nv = (A.q_pos[row] + 1) / A.ratio;
    if (nv > A.n_c[b]) nv = A.n_c[b];
    len = (int)max(0LL, min((long long)len, nv - col0));
  }
  if (len < 0) len = 0;
  uint32_t* keys = s_keys;
  int32_t* ids = reinterpret_cast<int32_t*>(s_keys + (A.in_ids ? CAP : 0));
  const float* src = A.in_scores + row * A.in_ld + col0;
  const int32_t* isrc = A.in_ids ? A.in_ids + row * A.in_ld + col0 : nullptr;
  const uint32_t nvalid = load_row_keys(sm, src, isrc, len, keys, ids);
  const int out_seg = blockIdx.x;
  int32_t* oi = A.out_idx + row * A.out_ld + (long long)out_seg * A.k;
  float* os = A.out_scores ? A.out_scores + row * A.out_ld + (long long)out_seg * A.k : nullptr;
  const uint32_t K = min((uint32_t)A.k, nvalid);
  auto idof = [&](int j) -> uint32_t { return isrc ? (uint32_t)ids[j] : (uint32_t)(A.col_base + seg * A.rows_per_seg + j); };

  select_in_smem(sm, keys, len, K, nvalid, idof, oi, os, 0u);
  for (int s = (int)K + threadIdx.x; s < A.k; s += blockDim.x) {
    oi[s] = -1;
    if (os) os[s] = -INFINITY;
  }
}


// Exact selection of the `need` best of n <= 64 candidates (key desc, id asc, position asc) by the whole
// block: warp w ranks candidates w, w + #warps, ... (its lanes split the comparisons; a candidate's rank is
// the number of candidates that beat it) and writes the winners at oi/os[base + rank].  Every thread of
// the block calls it.
__device__ void block_rank_select(const uint32_t* keys, const int32_t* ids, int n, uint32_t need, int32_t* oi,
                                  float* os, uint32_t base) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  for (int i = warp; i < n; i += nw) {
    const uint32_t ki = keys[i];
    const int32_t ii = ids[i];
    uint32_t beat = 0;
    for (int j = lane; j < n; j += 32) {
      const uint32_t kj = keys[j];
      const int32_t ij = ids[j];
      beat += (kj > ki) || (kj == ki && (ij < ii || (ij == ii && j < i)));
    }
    const uint32_t rank = __reduce_add_sync(0xffffffffu, beat);
    if (lane == 0 && rank < need) {
      oi[base + rank] = ii;
      if (os) os[base + rank] = order_key_float(ki);
    }
  }
}

// Histogram-guided selection for one row (decode / Reindex rows, and the hierarchical pool's block scores):
// the kernel before it has counted the row's scores in 4096 bins of the top 12 bits of their
// order-preserving keys.  The bin holding the K-th largest score is found from the histogram; one pass over
// the row (bit masks in registers) emits every score in a higher bin, at slots from one block scan, and
// collects the boundary bin's scores.  The block resolves those on the remaining key bits (digit levels,
// then a rank over all warps).  If the boundary bin overflows the candidate buffer the row is selected by
// the full path instead.
constexpr int TOPK_HIST_PER_THREAD = TOPK_CHUNK / TOPK_THREADS;   // 32 scores per thread, 8 x float4
constexpr int TOPK_RANK_MAX = 64;
constexpr int TOPK_HIST_CAND = 4096;     // boundary-bin candidates held in shared memory

// Bin T (of HIST_BINS, thread t owning bins 4(T-1-t)..+3 counted from the top) holding the R-th largest
// element given per-bin counts; returns {T, count above T, count in T} in sm.bcast[0..2] (zeros if R == 0
// or R > total).  *total receives the number of counted elements.
// (hv: the four bins 4*owner .. 4*owner+3 this thread loaded, owner = blockDim.x - 1 - threadIdx.x)
__device__ void hist_find_bin_v(TopkSmem& sm, const uint4 hv, uint32_t R, uint32_t* total) {
  const int owner = (int)blockDim.x - 1 - (int)threadIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const uint32_t mine = hv.x + hv.y + hv.z + hv.w;
  // counts above this thread's bins: an inclusive scan inside the warp (threads in order of descending
  // bins), then every warp scans the warp totals itself (two barriers in all)
  uint32_t x = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sm.scan[warp] = x;
  __syncthreads();
  const uint32_t wt = lane < nw ? sm.scan[lane] : 0u;
  uint32_t wi = wt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, wi, o);
    if (lane >= o) wi += y;
  }
  const uint32_t wbase = __shfl_sync(0xffffffffu, wi - wt, warp);
  const uint32_t tot = __shfl_sync(0xffffffffu, wi, nw - 1);
  *total = tot;
  const uint32_t above_me = wbase + x - mine;
  const uint32_t K = min(R, tot);
  if (K > 0 && above_me < K && K <= above_me + mine) {       // exactly one thread holds the K-th count
    const uint32_t c[4] = {hv.w, hv.z, hv.y, hv.x};
    uint32_t acc = above_me;
    for (int i = 0; i < 4; ++i) {
      if (acc + c[i] >= K) {
        sm.bcast[0] = (uint32_t)(owner * 4 + 3 - i);
        sm.bcast[1] = acc;
        sm.bcast[2] = c[i];
        break;
      }
      acc += c[i];
    }
  }
  if (K == 0 && threadIdx.x == 0) { sm.bcast[0] = 0; sm.bcast[1] = 0; sm.bcast[2] = 0; }
  __syncthreads();
}

__device__ void hist_find_bin(TopkSmem& sm, const uint32_t* bins, uint32_t R, uint32_t* total) {
  const int owner = (int)blockDim.x - 1 - (int)threadIdx.x;
  hist_find_bin_v(sm, reinterpret_cast<const uint4*>(bins)[owner], R, total);
}

// The `need` best of the nT boundary-bin candidates (keys, ids in shared memory) by (key desc, id asc),
// written at oi/os[above ..]: all of them when they are exactly needed, by rank for a few, else by 8-bit
// digit levels.  Block-wide (every thread of the block calls it); s_cnt: two words of shared memory.
__device__ void resolve_boundary(TopkSmem& sm, uint32_t* ckeys, int32_t* cids, uint32_t nT, uint32_t need,
                                 uint32_t above, int32_t* oi, float* os, uint32_t* s_cnt) {
  if (need == nT) {
    for (int j = threadIdx.x; j < (int)nT; j += blockDim.x) {
      oi[above + j] = cids[j];
      if (os) os[above + j] = order_key_float(ckeys[j]);
    }
  } else if (nT <= (uint32_t)TOPK_RANK_MAX) {
    block_rank_select(ckeys, cids, (int)nT, need, oi, os, above);
  } else {
    // boundary bin: 8-bit digits of the remaining key bits (19..12, 11..4, 3..0), one 256-bin histogram
    // per level scanned by one warp, until at most TOPK_RANK_MAX candidates share the threshold prefix;
    // those go by rank (key, id, position), all of them by the block radix path if that never happens
    uint32_t* h2 = &sm.whist[0][0];                                // 256 bins
    uint32_t* k2 = &sm.whist[1][0];                                // TOPK_RANK_MAX keys, then ids
    int32_t* i2 = reinterpret_cast<int32_t*>(&sm.whist[1][TOPK_RANK_MAX]);
    uint32_t pref = 0, pmask = 0, rem = need, base_out = above, n_in = nT;
    bool ranked = false;
#pragma unroll 1
    for (int level = 0; level < 3 && !ranked; ++level) {
      const int sh = level == 0 ? 12 : level == 1 ? 4 : 0;
      const uint32_t dm = level == 2 ? 15u : 255u;
      if (threadIdx.x < 256) h2[threadIdx.x] = 0;
      if (threadIdx.x == 0) { s_cnt[0] = 0; s_cnt[1] = 0; }
      __syncthreads();
      for (int j = threadIdx.x; j < (int)nT; j += blockDim.x) {
        const uint32_t k = ckeys[j] & 0xFFFFFu;
        if ((k & pmask) == pref) atomicAdd(&h2[(k >> sh) & dm], 1u);
      }
      __syncthreads();
      if (threadIdx.x < 32) {
        // lane l owns digits 8(31-l) .. 8(31-l)+7, highest first
        const int lane = threadIdx.x;
        uint32_t c[8], tot = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) { c[i] = h2[8 * (31 - lane) + 7 - i]; tot += c[i]; }
        uint32_t incl = tot;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        uint32_t acc = incl - tot;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (acc < rem && acc + c[i] >= rem) {
            sm.bcast[0] = 8 * (31 - lane) + 7 - i;
            sm.bcast[1] = acc;
            sm.bcast[2] = c[i];
          }
          acc += c[i];
        }
      }
      __syncthreads();
      const uint32_t digit = sm.bcast[0], above2 = sm.bcast[1], n2 = sm.bcast[2];
      const uint32_t npref = pref | (digit << sh), nmask = pmask | (dm << sh);
      // write the candidates in a higher digit; keep the threshold digit's few for ranking (slots from one
      // shared counter per warp and kind: lanes take theirs from the ballot below them)
      const int lane = threadIdx.x & 31;
      for (int j0 = 0; j0 + (int)(threadIdx.x & ~31u) < (int)nT; j0 += blockDim.x) {
        const int j = j0 + (int)threadIdx.x;
        bool up = false, at = false;
        uint32_t kj = 0;
        int32_t ij = 0;
        if (j < (int)nT) {
          kj = ckeys[j];
          ij = cids[j];
          const uint32_t k = kj & 0xFFFFFu;
          if ((k & pmask) == pref) {
            const uint32_t dj = (k >> sh) & dm;
            up = dj > digit;
            at = dj == digit && n2 <= (uint32_t)TOPK_RANK_MAX;
          }
        }
        const uint32_t bu = __ballot_sync(0xffffffffu, up), ba = __ballot_sync(0xffffffffu, at);
        uint32_t su = 0, sa = 0;
        if (lane == 0) {
          if (bu) su = atomicAdd(&s_cnt[0], (uint32_t)__popc(bu));
          if (ba) sa = atomicAdd(&s_cnt[1], (uint32_t)__popc(ba));
        }
        su = __shfl_sync(0xffffffffu, su, 0);
        sa = __shfl_sync(0xffffffffu, sa, 0);
        const uint32_t below = (1u << lane) - 1u;
        if (up) {
          const uint32_t slot = base_out + su + (uint32_t)__popc(bu & below);
          oi[slot] = ij;
          if (os) os[slot] = order_key_float(kj);
        } else if (at) {
          const uint32_t slot = sa + (uint32_t)__popc(ba & below);
          k2[slot] = kj;
          i2[slot] = ij;
        }
      }
      __syncthreads();
      base_out += above2;
      rem -= above2;
      pref = npref;
      pmask = nmask;
      n_in = n2;
      if (n2 <= (uint32_t)TOPK_RANK_MAX) {
        block_rank_select(k2, i2, (int)n2, rem, oi, os, base_out);
        ranked = true;
      }
    }
    if (!ranked) {
      // more than TOPK_RANK_MAX candidates with one full key: exact selection among them
      for (int j = threadIdx.x; j < (int)nT; j += blockDim.x)
        if ((ckeys[j] & 0xFFFFFu) != pref) ckeys[j] = 0u;
      __syncthreads();
      auto idof = [&](int j) -> uint32_t { return (uint32_t)cids[j]; };
      select_in_smem(sm, ckeys, (int)nT, rem, n_in, idof, oi, os, base_out);
    }
  }
}

__global__ void __launch_bounds__(TOPK_THREADS) topk_hist_kernel(TopkRowArgs A, uint32_t* __restrict__ hist) {
  // dynamic shared memory: the row [TOPK_CHUNK] (scores, or scores | ids for explicit-id rows), then the
  // boundary-bin candidates: keys [TOPK_HIST_CAND] | ids [TOPK_HIST_CAND]
  extern __shared__ __align__(16) uint32_t s_topk[];
  __shared__ __align__(16) TopkSmem sm;
  __shared__ __align__(8) uint64_t row_bar;
  __shared__ uint32_t s_cnt[2];
  static_assert(TOPK_HIST_PER_THREAD * TOPK_THREADS == TOPK_CHUNK && TOPK_HIST_PER_THREAD % 4 == 0 &&
                TOPK_HIST_PER_THREAD <= 32, "row split");
  static_assert(sizeof(TopkSmem::whist) >= HIST_BINS * 4, "second-level histogram in the per-warp histograms");
  const int row = blockIdx.y;
  pdl_trigger();
  if (threadIdx.x < 4 && A.n_cols > 0) {       // warm translations: the row's ends, its histogram, its output
    const float* r0 = A.in_scores + row * A.in_ld;
    const void* pf[4] = {r0, r0 + (A.n_cols - 1), hist ? (const void*)(hist + (size_t)row * HIST_BINS) : r0,
                         A.out_idx ? (const void*)(A.out_idx + row * A.out_ld) : r0};
    prefetch_l2(pf[threadIdx.x]);
  }
  // the row's visible length: under the early start the positions (inputs of the step that no kernel of
  // it writes) are read before the wait, so the row's copy can be issued the moment the scores are final
  auto row_len = [&]() -> int {
    int n = min(A.rows_per_seg, A.n_cols);
    if (A.q_pos) {
      const int b = row / A.Nq;
      long long nv = (A.q_pos[row] + 1) / A.ratio;
      if (nv > A.n_c[b]) nv = A.n_c[b];
      n = (int)max(0LL, min((long long)n, nv));
    }
    return max(n, 0);
  };
  int len = A.early ? row_len() : 0;
  if (threadIdx.x == 0) {
    sm100::mbar_init(&row_bar, 1);
    sm100::fence_mbar_init();
  }
  pdl_wait();                                  // scores and histogram come from the previous kernel
  if (!A.early) len = row_len();
  int32_t* oi = A.out_idx + row * A.out_ld;
  float* os = A.out_scores ? A.out_scores + row * A.out_ld : nullptr;
  const float* src = A.in_scores + row * A.in_ld;
  const int32_t* isrc = A.in_ids ? A.in_ids + row * A.in_ld : nullptr;
  float* s_row = reinterpret_cast<float*>(s_topk);
  int32_t* s_rid = reinterpret_cast<int32_t*>(s_topk + TOPK_CHUNK_IDS);   // explicit ids (len <= TOPK_CHUNK_IDS)
  uint32_t* ckeys = s_topk + TOPK_CHUNK;
  int32_t* cids = reinterpret_cast<int32_t*>(s_topk + TOPK_CHUNK + TOPK_HIST_CAND);

  // the row's histogram first (16 KB, each thread its four bins), so those loads do not queue behind the
  // row's copy; then the row into shared memory: one bulk copy when aligned, else plain loads
  const uint4 hv = reinterpret_cast<const uint4*>(hist + (size_t)row * HIST_BINS)[blockDim.x - 1 - threadIdx.x];
  __syncthreads();
  const uint32_t bytes = (uint32_t)len * 4u;
  const bool bulk = len > 0 && (len & 3) == 0 && (reinterpret_cast<uintptr_t>(src) & 15) == 0 &&
                    (!isrc || (reinterpret_cast<uintptr_t>(isrc) & 15) == 0);
  if (bulk && threadIdx.x == 0) {
    sm100::mbar_arrive_expect_tx(&row_bar, bytes * (isrc ? 2u : 1u));
    for (uint32_t off = 0; off < bytes; off += 32768u) {
      const uint32_t n = min(32768u, bytes - off);
      sm100::bulk_load(reinterpret_cast<uint8_t*>(s_row) + off, reinterpret_cast<const uint8_t*>(src) + off, n, &row_bar);
      if (isrc)
        sm100::bulk_load(reinterpret_cast<uint8_t*>(s_rid) + off, reinterpret_cast<const uint8_t*>(isrc) + off, n,
                         &row_bar);
    }
  } else if (!bulk) {
    for (int j = threadIdx.x; j < len; j += blockDim.x) {
      s_row[j] = src[j];
      if (isrc) s_rid[j] = isrc[j];
    }
  }
  uint32_t nvalid;
  hist_find_bin_v(sm, hv, (uint32_t)A.k, &nvalid);                             // overlaps the copy
  // the row's histogram is consumed: leave it zero for the next scoring call (each thread clears the
  // four bins it read)
  reinterpret_cast<uint4*>(hist + (size_t)row * HIST_BINS)[blockDim.x - 1 - threadIdx.x] = make_uint4(0, 0, 0, 0);
  const uint32_t K = min((uint32_t)A.k, nvalid);
  const uint32_t Tbin = sm.bcast[0], above = sm.bcast[1], nT = sm.bcast[2];
  const uint32_t need = K - above;
  if (bulk && !sm100::mbar_wait(&row_bar, 0)) atomicOr(&g_csa_device_error, 1u);
  // (plain loads: hist_find_bin's barriers have ordered them)
  bool done = false;
  if (K > 0) {
    // one pass: bit masks "above the boundary bin" / "in it" over this thread's 32 scores, one block scan
    // of the packed counts (above < 2^16, at <= 2^15) gives every thread its output slots
    // the boundary bin as a float interval [lo, hi]: two compares per score (float order = key order)
    const float lo = order_key_float(Tbin << HIST_SHIFT);
    const float hi = order_key_float((Tbin << HIST_SHIFT) | ((1u << HIST_SHIFT) - 1u));
    const bool fast = !isrc && Tbin > 0;                          // no ids; -inf lies below the bin
    uint32_t m_up = 0, m_at = 0;
    if (fast) {
      // one compare per score (at or above the bin: about k of the row), then the few set bits are split
      // into above the bin / in it
      uint32_t m_ge = 0;
#pragma unroll
      for (int i = 0; i < TOPK_HIST_PER_THREAD / 4; ++i) {
        const int j0 = 4 * (threadIdx.x + TOPK_THREADS * i);
        float4 f4 = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
        if (j0 + 3 < len) {
          f4 = *reinterpret_cast<const float4*>(s_row + j0);
        } else if (j0 < len) {
          f4.x = s_row[j0];
          if (j0 + 1 < len) f4.y = s_row[j0 + 1];
          if (j0 + 2 < len) f4.z = s_row[j0 + 2];
        }
        m_ge |= ((uint32_t)(f4.x >= lo) | ((uint32_t)(f4.y >= lo) << 1) | ((uint32_t)(f4.z >= lo) << 2) |
                 ((uint32_t)(f4.w >= lo) << 3)) << (4 * i);
      }
      for (uint32_t mk = m_ge; mk; mk &= mk - 1u) {
        const int e = __ffs(mk) - 1;
        if (s_row[4 * (threadIdx.x + TOPK_THREADS * (e >> 2)) + (e & 3)] > hi) m_up |= 1u << e;
      }
      m_at = m_ge & ~m_up;
    } else {
#pragma unroll 1
      for (int i = 0; i < TOPK_HIST_PER_THREAD / 4; ++i) {
        const int j0 = 4 * (threadIdx.x + TOPK_THREADS * i);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const float v = j0 + c < len ? s_row[j0 + c] : -INFINITY;
          const bool ok = v > -INFINITY && (!isrc || s_rid[j0 + c] >= 0);
          const uint32_t bin = float_order_key(v) >> HIST_SHIFT;
          if (ok && bin > Tbin) m_up |= 1u << (4 * i + c);
          if (ok && bin == Tbin) m_at |= 1u << (4 * i + c);
        }
      }
    }
    uint32_t tot;
    const uint32_t pre = block_exclusive_scan(sm, (uint32_t)__popc(m_up) | ((uint32_t)__popc(m_at) << 16), &tot);
    if ((tot & 0xFFFFu) == above && (tot >> 16) == nT && nT <= (uint32_t)TOPK_HIST_CAND) {
      uint32_t su = pre & 0xFFFFu, sa = pre >> 16;
      uint32_t mk = m_up | m_at;
#pragma unroll 1
      while (mk) {
        const int e = __ffs(mk) - 1;
        mk &= mk - 1u;
        const int j = 4 * (threadIdx.x + TOPK_THREADS * (e >> 2)) + (e & 3);
        const float v = s_row[j];
        const int32_t id = isrc ? s_rid[j] : j;
        if ((m_up >> e) & 1u) {
          oi[su] = id;
          if (os) os[su] = v + 0.0f;
          ++su;
        } else {
          ckeys[sa] = float_order_key(v);
          cids[sa] = id;
          ++sa;
        }
      }
      done = true;
    }
  }
  // every thread takes the same branch: `done` depends only on block-uniform values
  if (done) {
    __syncthreads();
    resolve_boundary(sm, ckeys, cids, nT, need, above, oi, os, s_cnt);
  } else if (K > 0) {
    // inconsistent counts or a boundary bin larger than the candidate buffer: the whole row, in place
    __syncthreads();
    uint32_t* keys = s_topk;
    uint32_t nv_loc = 0;
    for (int j = threadIdx.x; j < len; j += blockDim.x) {
      const float v = s_row[j];
      const bool ok = v > -INFINITY && (!isrc || s_rid[j] >= 0);
      keys[j] = ok ? float_order_key(v) : 0u;
      nv_loc += ok;
    }
    uint32_t nv2;
    block_exclusive_scan(sm, nv_loc, &nv2);
    auto idof2 = [&](int j) -> uint32_t { return isrc ? (uint32_t)s_rid[j] : (uint32_t)j; };
    select_in_smem(sm, keys, len, min((uint32_t)A.k, nv2), nv2, idof2, oi, os, 0u);
  }
  for (int s2 = (int)K + threadIdx.x; s2 < A.k; s2 += blockDim.x) {
    oi[s2] = -1;
    if (os) os[s2] = -INFINITY;
  }
}

// Long rows (several TOPK_CHUNK segments) with the row histogram of the scorer: CTA (seg, row) reads its
// segment once, emits every score above the boundary bin at a slot from the row's counter and parks the
// boundary-bin scores in the row's buffer (warp-aggregated atomics); the row's last CTA checks the counts
// against the histogram, resolves the boundary bin and marks the row resolved.  Counts that disagree (a
// stale histogram) or a boundary bin larger than the buffer leave the row to the tournament kernels that
// follow, which skip resolved rows.  The last CTA clears the histogram row.
__global__ void __launch_bounds__(TOPK_THREADS) topk_long_kernel(TopkRowArgs A, uint32_t* __restrict__ hist,
                                                                 LongRowState* __restrict__ state,
                                                                 uint32_t* __restrict__ cand) {
  extern __shared__ __align__(16) uint32_t s_lc[];   // boundary-bin keys [TOPK_HIST_CAND] | ids [TOPK_HIST_CAND]
  __shared__ __align__(16) TopkSmem sm;
  __shared__ uint32_t s_cnt[2];
  __shared__ uint32_t s_last;
  const int seg = blockIdx.x, row = blockIdx.y;
  pdl_trigger();
  pdl_wait();                                  // scores and histogram come from the previous kernel
  int len = A.n_cols;
  if (A.q_pos) {
    const int b = row / A.Nq;
    long long nv = (A.q_pos[row] + 1) / A.ratio;
    if (nv > A.n_c[b]) nv = A.n_c[b];
    len = (int)max(0LL, min((long long)len, nv));
  }
  uint32_t* hrow = hist + (size_t)row * HIST_BINS;
  uint32_t nvalid;
  hist_find_bin(sm, hrow, (uint32_t)A.k, &nvalid);
  const uint32_t K = min((uint32_t)A.k, nvalid);
  const uint32_t T = sm.bcast[0], above = sm.bcast[1], nT = sm.bcast[2];
  LongRowState& rs = state[row];
  uint32_t* ck = cand + (size_t)row * 2 * TOPK_HIST_CAND;
  int32_t* ci = reinterpret_cast<int32_t*>(ck + TOPK_HIST_CAND);
  int32_t* oi = A.out_idx + row * A.out_ld;
  float* os = A.out_scores ? A.out_scores + row * A.out_ld : nullptr;
  const float* src = A.in_scores + row * A.in_ld;
  const int c0 = seg * TOPK_CHUNK, c1 = min(len, c0 + TOPK_CHUNK);
  if (K > 0) {
    // this CTA's 32 scores per thread as bit masks (above the boundary bin / in it), one block scan, then one
    // reservation per CTA in the row's counters (not one dependent atomic per warp and hit)
    const bool vec = (reinterpret_cast<uintptr_t>(src) & 15) == 0;   // block-uniform
    uint32_t m_up = 0, m_at = 0;
#pragma unroll
    for (int i = 0; i < TOPK_HIST_PER_THREAD / 4; ++i) {
      const int j0 = c0 + 4 * (threadIdx.x + TOPK_THREADS * i);
      float f[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
      if (vec && j0 + 3 < c1) {
        const float4 f4 = *reinterpret_cast<const float4*>(src + j0);
        f[0] = f4.x; f[1] = f4.y; f[2] = f4.z; f[3] = f4.w;
      } else {
#pragma unroll
        for (int c = 0; c < 4; ++c)
          if (j0 + c < c1) f[c] = src[j0 + c];
      }
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const uint32_t bin = float_order_key(f[c]) >> HIST_SHIFT;
        const bool valid = f[c] > -INFINITY;
        if (valid && bin > T) m_up |= 1u << (4 * i + c);
        if (valid && bin == T) m_at |= 1u << (4 * i + c);
      }
    }
    uint32_t tot;
    const uint32_t pre = block_exclusive_scan(sm, (uint32_t)__popc(m_up) | ((uint32_t)__popc(m_at) << 16), &tot);
    if (threadIdx.x == 0) {
      s_cnt[0] = (tot & 0xFFFFu) ? atomicAdd(&rs.up, tot & 0xFFFFu) : 0u;
      s_cnt[1] = (tot >> 16) ? atomicAdd(&rs.at, tot >> 16) : 0u;
    }
    __syncthreads();
    uint32_t su = s_cnt[0] + (pre & 0xFFFFu), sa = s_cnt[1] + (pre >> 16);
#pragma unroll 1
    for (uint32_t mk = m_up | m_at; mk; mk &= mk - 1u) {
      const int e = __ffs(mk) - 1;
      const int j = c0 + 4 * (threadIdx.x + TOPK_THREADS * (e >> 2)) + (e & 3);
      const float v = src[j];
      if ((m_up >> e) & 1u) {
        if (su < above) {
          oi[su] = j;
          if (os) os[su] = v + 0.0f;
        }
        ++su;
      } else {
        if (sa < (uint32_t)TOPK_HIST_CAND) {
          ck[sa] = float_order_key(v);
          ci[sa] = j;
        }
        ++sa;
      }
    }
  }
  // the last CTA of the row resolves it
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    s_last = atomicAdd(&rs.done, 1u) == gridDim.x - 1 ? 1u : 0u;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  const uint32_t n_up = *reinterpret_cast<volatile uint32_t*>(&rs.up);
  const uint32_t n_at = *reinterpret_cast<volatile uint32_t*>(&rs.at);
  const bool good = K == 0 || (n_up == above && n_at == nT && nT <= (uint32_t)TOPK_HIST_CAND);
  if (good && K > 0) {
    uint32_t* ckeys = s_lc;
    int32_t* cids = reinterpret_cast<int32_t*>(s_lc + TOPK_HIST_CAND);
    for (int c = threadIdx.x; c < (int)nT; c += blockDim.x) {
      ckeys[c] = *reinterpret_cast<volatile uint32_t*>(ck + c);
      cids[c] = *reinterpret_cast<volatile int32_t*>(ci + c);
    }
    __syncthreads();
    resolve_boundary(sm, ckeys, cids, nT, K - above, above, oi, os, s_cnt);
  }
  if (good)
    for (int s2 = (int)K + threadIdx.x; s2 < A.k; s2 += blockDim.x) {
      oi[s2] = -1;
      if (os) os[s2] = -INFINITY;
    }
  // every CTA of the row has read the histogram (it counted itself done afterwards): clear it
  reinterpret_cast<uint4*>(hrow)[threadIdx.x] = make_uint4(0, 0, 0, 0);
  if (threadIdx.x == 0) rs.ok = good ? 1u : 0u;
}

// ------------------------------------------------------------------------- hierarchical pool
// Block scores of the hierarchical pool (max over the visible keys of each block of G) and their row
// histogram (top 12 bits of the order-preserving key; blocks without a visible key are -inf and not
// counted), so the pool's top blocks are selected like a decode row.  CTA: BM_THREADS threads x
// BM_PER_THREAD blocks of one row; its histogram is added to the row's (zero on entry).
constexpr int BM_THREADS = 1024, BM_PER_THREAD = 4;
__global__ void __launch_bounds__(BM_THREADS) block_max_kernel(const float* __restrict__ scores, long long ld,
                                                               int n_cols, const int64_t* __restrict__ q_pos,
                                                               const int32_t* __restrict__ n_c, int ratio, int Nq,
                                                               int G, int nblk, float* __restrict__ bs,
                                                               uint32_t* __restrict__ bhist) {
  __shared__ uint32_t h[HIST_BINS];
  const int row = blockIdx.y;
  for (int i = threadIdx.x; i < HIST_BINS; i += blockDim.x) h[i] = 0;
  long long nv = (q_pos[row] + 1) / ratio;
  if (nv > n_c[row / Nq]) nv = n_c[row / Nq];
  if (nv > n_cols) nv = n_cols;
  __syncthreads();
#pragma unroll
  for (int u = 0; u < BM_PER_THREAD; ++u) {
    const int j = (blockIdx.x * BM_PER_THREAD + u) * BM_THREADS + threadIdx.x;
    if (j >= nblk) break;
    float m = -INFINITY;
    for (int e = 0; e < G; ++e) {
      const long long i = (long long)j * G + e;
      if (i < nv) m = fmaxf(m, scores[row * ld + i]);
    }
    bs[(long long)row * nblk + j] = m;
    if (m > -INFINITY) atomicAdd(&h[float_order_key(m) >> HIST_SHIFT], 1u);
  }
  __syncthreads();
  uint32_t* hr = bhist + (size_t)row * HIST_BINS;
  for (int i = threadIdx.x; i < HIST_BINS; i += blockDim.x)
    if (h[i]) atomicAdd(&hr[i], h[i]);
}

// Row histograms for score rows no scorer counted (multi-query rows): the visible scores of a row (j <
// n_vis(t)) in HIST_BINS bins of the top 12 bits of their order-preserving keys, added to the row's
// histogram (zero on entry).  CTA: RH_THREADS threads x RH_PER_THREAD scores of one row.
constexpr int RH_THREADS = 1024, RH_PER_THREAD = 4;
__global__ void __launch_bounds__(RH_THREADS) row_hist_kernel(const float* __restrict__ scores, long long ld,
                                                              int n_cols, const int64_t* __restrict__ q_pos,
                                                              const int32_t* __restrict__ n_c, int ratio, int Nq,
                                                              uint32_t* __restrict__ hist) {
  __shared__ uint32_t h[HIST_BINS];
  const int row = blockIdx.y;
  for (int i = threadIdx.x; i < HIST_BINS; i += blockDim.x) h[i] = 0;
  long long nv = (q_pos[row] + 1) / ratio;
  if (nv > n_c[row / Nq]) nv = n_c[row / Nq];
  if (nv > n_cols) nv = n_cols;
  __syncthreads();
#pragma unroll
  for (int u = 0; u < RH_PER_THREAD; ++u) {
    const long long j = ((long long)blockIdx.x * RH_PER_THREAD + u) * RH_THREADS + threadIdx.x;
    if (j < nv) {
      const float v = scores[row * ld + j];
      if (v > -INFINITY) atomicAdd(&h[float_order_key(v) >> HIST_SHIFT], 1u);
    }
  }
  __syncthreads();
  uint32_t* hr = hist + (size_t)row * HIST_BINS;
  for (int i = threadIdx.x; i < HIST_BINS; i += blockDim.x)
    if (h[i]) atomicAdd(&hr[i], h[i]);
}

__global__ void pool_expand_kernel(const int32_t* __restrict__ blk, int P, int G, const float* __restrict__ scores,
                                   long long ld, int n_cols, const int64_t* __restrict__ q_pos,
                                   const int32_t* __restrict__ n_c, int ratio, int Nq, int32_t* __restrict__ pool) {
  const int row = blockIdx.y;
  const int s = blockIdx.x * blockDim.x + threadIdx.x;
  if (s >= P * G) return;
  long long nv = (q_pos[row] + 1) / ratio;
  if (nv > n_c[row / Nq]) nv = n_c[row / Nq];
  if (nv > n_cols) nv = n_cols;
  const int b = blk[(long long)row * P + s / G];
  int out = -1;
  if (b >= 0) {
    const long long i = (long long)b * G + s % G;
    if (i < nv && scores[row * ld + i] > -INFINITY) out = (int)i;
  }
  pool[(long long)row * P * G + s] = out;
}

// tensor-core scoring of single-query Full rows (index_tc.cu) and of multi-query Full rows (index_mq_tc.cu)
bool index_tc_eligible(const csa_index_args* a);
csa_status run_scores_tc(const csa_index_args* a, float* scores, long long ld, uint32_t* hist, cudaStream_t st);
bool index_mq_tc_eligible(const csa_index_args* a);
csa_status run_scores_mq_tc(const csa_index_args* a, float* scores, long long ld, cudaStream_t st);
// fused decode indexer + top-k in one cluster per row (index_tc.cu)
bool index_topk_fused_eligible(const csa_index_args* a);
csa_status run_index_topk_fused(const csa_index_args* a, cudaStream_t st);

// ------------------------------------------------------------------------------ orchestration
struct IndexPlan {
  int rows, n_cols, segs, seg_len;
  bool hist;   // single-query rows: histogram-guided selection (long rows: segment CTAs + tournament fallback)
  bool mq_hist;  // multi-query rows longer than TOPK_SHORT: a row-histogram pass, then the same selection
  size_t off_scores, off_tidx, off_tsc, off_bs, off_bidx, off_bhist, off_mqhist, off_lstate, off_lcand, off_hist,
      sel_total, total;
};

static bool one_query_per_cta(const csa_index_args* a) { return a->cand != nullptr || a->Nq == 1; }

// Workspace of the selection step (tournament buffers, pool block scores); the fused entry point
// places the score matrix in front of it.
static IndexPlan plan_index(const csa_index_args* a) {
  IndexPlan p{};
  p.rows = a->B * a->Nq;
  p.n_cols = a->cand ? a->n_cand : a->n_max;
  const int cap = TOPK_CHUNK;
  p.segs = (p.n_cols + cap - 1) / cap;
  if (p.segs < 1) p.segs = 1;
  p.seg_len = p.segs == 1 ? p.n_cols : cap;
  size_t o = 0;
  if (p.segs > 1) {
    p.off_tidx = o; o = align_up(o + (size_t)p.rows * p.segs * a->k * 4, 256);
    p.off_tsc = o;  o = align_up(o + (size_t)p.rows * p.segs * a->k * 4, 256);
  }
  if (p.segs > 1 && one_query_per_cta(a)) {
    p.off_lstate = o; o = align_up(o + (size_t)p.rows * sizeof(LongRowState), 256);
    p.off_lcand = o;  o = align_up(o + (size_t)p.rows * 2 * TOPK_HIST_CAND * 4, 256);
  }
  if (a->pool_blocks > 0) {
    const int G = a->pool_block_size;
    const int nblk = (p.n_cols + G - 1) / G;
    p.off_bs = o;   o = align_up(o + (size_t)p.rows * nblk * 4, 256);
    p.off_bidx = o; o = align_up(o + (size_t)p.rows * a->pool_blocks * 4, 256);
    p.off_bhist = o; o = align_up(o + (size_t)p.rows * HIST_BINS * 4, 256);
  }
  p.mq_hist = !one_query_per_cta(a) && p.segs == 1 && p.seg_len > TOPK_SHORT;
  if (p.mq_hist) {
    p.off_mqhist = o; o = align_up(o + (size_t)p.rows * HIST_BINS * 4, 256);
  }
  p.sel_total = o;
  p.off_scores = o;
  o = align_up(o + (size_t)p.rows * p.n_cols * 4, 256);
  p.hist = one_query_per_cta(a);
  p.off_hist = o;
  if (p.hist) o = align_up(o + (size_t)p.rows * HIST_BINS * 4, 256);
  p.total = o;
  return p;
}

// ptrs = false (workspace-size queries): shapes, flags and the page map only; the buffers may not exist yet
static csa_status validate_index(const csa_index_args* a, bool need_select, bool ptrs = true) {
  CSA_REQUIRE(a != nullptr && a->struct_size == sizeof(csa_index_args));
  CSA_REQUIRE(a->B >= 0 && a->Nq >= 0 && a->H_I >= 1 && a->ratio >= 1 && a->k >= 1 && a->n_max >= 0);
  CSA_SUPPORTED(a->d_I == 64 || a->d_I == 128);
  CSA_SUPPORTED(a->H_I <= IDX_HEADS && a->k <= 4096);
  CSA_REQUIRE(a->g_q > 0.0f && a->g_k > 0.0f);
  if (a->cand) {
    CSA_REQUIRE(a->n_cand >= 1);
    CSA_SUPPORTED(a->n_cand <= TOPK_CHUNK_IDS && a->pool_blocks == 0);
  }
  {
    const int n_cols = a->cand ? a->n_cand : a->n_max;
    const int segs = (n_cols + TOPK_CHUNK - 1) / TOPK_CHUNK;
    if (segs > 1) CSA_SUPPORTED((long long)segs * a->k <= TOPK_CHUNK_IDS);
  }
  if (a->pool_blocks > 0) {
    CSA_REQUIRE(a->pool_block_size >= 1 && (a->pool_out != nullptr || !ptrs));
    const int nblk = (a->n_max + a->pool_block_size - 1) / a->pool_block_size;
    CSA_SUPPORTED(nblk <= TOPK_CHUNK && a->pool_blocks <= 4096);
  }
  {
    const csa_status pv = check_page_map(a->k_pages, a->n_max);
    if (pv != CSA_OK) return pv;
  }
  if ((long long)a->B * a->Nq == 0 || !ptrs) return CSA_OK;
  CSA_REQUIRE(a->n_c && a->q_pos);
  if (need_select) CSA_REQUIRE(a->idx_out != nullptr);
  else CSA_REQUIRE(a->q_I && a->w && a->k_codes && a->k_scales);
  return CSA_OK;
}

// clear_hist: the histogram is this call's own scratch (fused entry points); a caller's histogram
// (csa_index_scores) is added into as it stands: zero at first use, and csa_topk clears each row it reads.
static csa_status run_scores(const csa_index_args* a, float* scores, long long ld, uint32_t* hist, bool clear_hist,
                             cudaStream_t st) {
  const int n_cols = a->cand ? a->n_cand : a->n_max;
  if (!one_query_per_cta(a)) hist = nullptr;
  if (hist && clear_hist) {
    cudaError_t e = cudaMemsetAsync(hist, 0, (size_t)a->B * a->Nq * HIST_BINS * 4, st);
    if (e != cudaSuccess) { set_last_cuda_error(e); return CSA_ERR_CUDA; }
  }
  if (index_tc_eligible(a)) return run_scores_tc(a, scores, ld, hist, st);
  if (index_mq_tc_eligible(a)) return run_scores_mq_tc(a, scores, ld, st);
  const int qt = a->cand ? 1 : (a->Nq < IDX_QT ? a->Nq : IDX_QT);
  const long long qtiles = (long long)a->B * (a->cand ? a->Nq : (a->Nq + qt - 1) / qt);
  // key range per CTA: enough CTAs for about one wave, at least one 16-key tile per warp
  long long per_seq = IDX_TARGET_CTAS / (qtiles > 0 ? qtiles : 1);
  if (per_seq < 1) per_seq = 1;
  long long tpw = (n_cols + IDX_WARPS * 16 * per_seq - 1) / (IDX_WARPS * 16 * per_seq);
  if (tpw < 1) tpw = 1;
  const long long kpc = IDX_WARPS * 16 * tpw;
  dim3 grid((unsigned)((n_cols + kpc - 1) / kpc), a->cand ? a->Nq : (a->Nq + qt - 1) / qt, a->B);
  if (n_cols == 0) return CSA_OK;
  const int smem = qt * IDX_HEADS * a->d_I * 2 + (hist ? HIST_BINS * 4 : 0);
  const float gg = a->g_q * a->g_k;
  static std::atomic<unsigned> attr128{0}, attr64{0};
  if (a->d_I == 128) {
    set_smem_once((const void*)index_score_kernel<128>, IDX_QT * IDX_HEADS * 128 * 2 + HIST_BINS * 4, attr128);
    index_score_kernel<128><<<grid, IDX_WARPS * 32, smem, st>>>(
        (const uint16_t*)a->q_I, a->w, a->H_I, a->g_q, gg, a->Nq, qt, a->k_codes, a->k_scales, a->n_max, a->n_c,
        a->q_pos, a->ratio, a->cand, a->n_cand, scores, ld, (int)tpw, hist, a->k_pages);
  } else {
    set_smem_once((const void*)index_score_kernel<64>, IDX_QT * IDX_HEADS * 64 * 2 + HIST_BINS * 4, attr64);
    index_score_kernel<64><<<grid, IDX_WARPS * 32, smem, st>>>(
        (const uint16_t*)a->q_I, a->w, a->H_I, a->g_q, gg, a->Nq, qt, a->k_codes, a->k_scales, a->n_max, a->n_c,
        a->q_pos, a->ratio, a->cand, a->n_cand, scores, ld, (int)tpw, hist, a->k_pages);
  }
  return launch_status();
}

constexpr int TOPK_SHORT_THREADS = 256;

static csa_status launch_topk(TopkRowArgs ta, int rows, int segs, bool ids, cudaStream_t st) {
  static_assert(TOPK_CHUNK_IDS * 8 == TOPK_CHUNK * 4, "one shared-memory size for both row kinds");
  dim3 grid(segs, rows);
  if (segs == 1 && ta.rows_per_seg <= TOPK_SHORT) {
    // shared memory sized to the row: keys of rows_per_seg columns (explicit ids follow at TOPK_SHORT)
    const size_t smem = ids ? (size_t)TOPK_SHORT * 8 : align_up((size_t)ta.rows_per_seg, 4) * 4;
    static std::atomic<unsigned> attr_s{0};
    set_smem_once((const void*)topk_kernel<TOPK_SHORT_THREADS, TOPK_SHORT>, TOPK_SHORT * 8, attr_s);
    return launch_pdl(topk_kernel<TOPK_SHORT_THREADS, TOPK_SHORT>, grid, dim3(TOPK_SHORT_THREADS), smem, st, ta);
  }
  const size_t smem = (size_t)TOPK_CHUNK * 4;
  static std::atomic<unsigned> attr_done{0};
  set_smem_once((const void*)topk_kernel<TOPK_THREADS, TOPK_CHUNK_IDS>, (int)smem, attr_done);
  return launch_pdl(topk_kernel<TOPK_THREADS, TOPK_CHUNK_IDS>, grid, dim3(TOPK_THREADS), smem, st, ta);
}

static csa_status run_select(const csa_index_args* a, const IndexPlan& p, const float* scores, long long ld,
                             const uint32_t* hist, uint8_t* w8, cudaStream_t st) {
  TopkRowArgs ta{};
  ta.in_scores = scores;
  ta.in_ids = a->cand;
  ta.in_ld = ld;
  ta.n_cols = p.n_cols;
  ta.col_base = 0;
  ta.q_pos = a->cand ? nullptr : a->q_pos;
  ta.n_c = a->n_c;
  ta.ratio = a->ratio;
  ta.Nq = a->Nq;
  ta.rows_per_seg = p.seg_len;
  ta.k = a->k;
  ta.early = (a->flags & CSA_EARLY_START) ? 1 : 0;
  if (a->cand) CSA_SUPPORTED(ld == a->n_cand);   // explicit ids are read with the score row stride
  if (p.segs == 1 && hist != nullptr && p.hist) {
    ta.out_idx = a->idx_out;
    ta.out_scores = a->scores_out;
    ta.out_ld = a->k;
    static std::atomic<unsigned> attr_h{0};
    const int smem_h = (TOPK_CHUNK + 2 * TOPK_HIST_CAND) * 4;
    set_smem_once((const void*)topk_hist_kernel, smem_h, attr_h);
    csa_status s = launch_pdl(topk_hist_kernel, dim3(1, p.rows), dim3(TOPK_THREADS), (size_t)smem_h, st, ta,
                              const_cast<uint32_t*>(hist));
    if (s != CSA_OK) return s;
  } else if (p.segs == 1 && p.mq_hist) {
    // multi-query rows: their histograms first (visible scores only), then the histogram-guided selection
    ta.out_idx = a->idx_out;
    ta.out_scores = a->scores_out;
    ta.out_ld = a->k;
    ta.early = 0;
    uint32_t* mh = (uint32_t*)(w8 + p.off_mqhist);
    const cudaError_t e = cudaMemsetAsync(mh, 0, (size_t)p.rows * HIST_BINS * 4, st);
    if (e != cudaSuccess) {
      set_last_cuda_error(e);
      return CSA_ERR_CUDA;
    }
    const int per_cta = RH_THREADS * RH_PER_THREAD;
    row_hist_kernel<<<dim3((p.n_cols + per_cta - 1) / per_cta, p.rows), RH_THREADS, 0, st>>>(
        scores, ld, p.n_cols, a->q_pos, a->n_c, a->ratio, a->Nq, mh);
    csa_status s = launch_status();
    if (s != CSA_OK) return s;
    static std::atomic<unsigned> attr_m{0};
    const int smem_h = (TOPK_CHUNK + 2 * TOPK_HIST_CAND) * 4;
    set_smem_once((const void*)topk_hist_kernel, smem_h, attr_m);
    s = launch_pdl(topk_hist_kernel, dim3(1, p.rows), dim3(TOPK_THREADS), (size_t)smem_h, st, ta, mh);
    if (s != CSA_OK) return s;
  } else if (p.segs == 1) {
    ta.out_idx = a->idx_out;
    ta.out_scores = a->scores_out;
    ta.out_ld = a->k;
    csa_status s = launch_topk(ta, p.rows, 1, a->cand != nullptr, st);
    if (s != CSA_OK) return s;
  } else {
    const LongRowState* skip = nullptr;
    if (hist != nullptr && p.hist) {
      // histogram pass over the segments; rows it cannot resolve go through the tournament below
      LongRowState* lst = (LongRowState*)(w8 + p.off_lstate);
      const cudaError_t e = cudaMemsetAsync(lst, 0, (size_t)p.rows * sizeof(LongRowState), st);
      if (e != cudaSuccess) {
        set_last_cuda_error(e);
        return CSA_ERR_CUDA;
      }
      TopkRowArgs tl = ta;
      tl.out_idx = a->idx_out;
      tl.out_scores = a->scores_out;
      tl.out_ld = a->k;
      static std::atomic<unsigned> attr_l{0};
      const int smem_l = 2 * TOPK_HIST_CAND * 4;
      set_smem_once((const void*)topk_long_kernel, smem_l, attr_l);
      csa_status s = launch_pdl(topk_long_kernel, dim3(p.segs, p.rows), dim3(TOPK_THREADS), (size_t)smem_l, st, tl,
                                const_cast<uint32_t*>(hist), lst, (uint32_t*)(w8 + p.off_lcand));
      if (s != CSA_OK) return s;
      skip = lst;
    }
    ta.skip = skip;
    int32_t* tidx = (int32_t*)(w8 + p.off_tidx);
    float* tsc = (float*)(w8 + p.off_tsc);
    ta.out_idx = tidx;
    ta.out_scores = tsc;
    ta.out_ld = (long long)p.segs * a->k;
    csa_status s = launch_topk(ta, p.rows, p.segs, false, st);
    if (s != CSA_OK) return s;
    TopkRowArgs tb{};
    tb.in_scores = tsc;
    tb.in_ids = tidx;
    tb.in_ld = (long long)p.segs * a->k;
    tb.n_cols = p.segs * a->k;
    tb.rows_per_seg = p.segs * a->k;
    tb.k = a->k;
    tb.out_idx = a->idx_out;
    tb.out_scores = a->scores_out;
    tb.out_ld = a->k;
    tb.skip = skip;
    CSA_SUPPORTED(tb.n_cols <= TOPK_CHUNK_IDS);
    s = launch_topk(tb, p.rows, 1, true, st);
    if (s != CSA_OK) return s;
  }
  if (a->pool_blocks > 0) {
    const int G = a->pool_block_size;
    const int nblk = (p.n_cols + G - 1) / G;
    float* bs = (float*)(w8 + p.off_bs);
    int32_t* bidx = (int32_t*)(w8 + p.off_bidx);
    uint32_t* bhist = (uint32_t*)(w8 + p.off_bhist);
    cudaError_t e = cudaMemsetAsync(bhist, 0, (size_t)p.rows * HIST_BINS * 4, st);
    if (e != cudaSuccess) {
      set_last_cuda_error(e);
      return CSA_ERR_CUDA;
    }
    const int per_cta = BM_THREADS * BM_PER_THREAD;
    block_max_kernel<<<dim3((nblk + per_cta - 1) / per_cta, p.rows), BM_THREADS, 0, st>>>(
        scores, ld, p.n_cols, a->q_pos, a->n_c, a->ratio, a->Nq, G, nblk, bs, bhist);
    csa_status s = launch_status();
    if (s != CSA_OK) return s;
    // the top blocks by (block score desc, block id asc): the histogram-guided row selection
    TopkRowArgs tc{};
    tc.in_scores = bs;
    tc.in_ld = nblk;
    tc.n_cols = nblk;
    tc.rows_per_seg = nblk;
    tc.k = a->pool_blocks;
    tc.out_idx = bidx;
    tc.out_ld = a->pool_blocks;
    static std::atomic<unsigned> attr_p{0};
    const int smem_h = (TOPK_CHUNK + 2 * TOPK_HIST_CAND) * 4;
    set_smem_once((const void*)topk_hist_kernel, smem_h, attr_p);
    s = launch_pdl(topk_hist_kernel, dim3(1, p.rows), dim3(TOPK_THREADS), (size_t)smem_h, st, tc, bhist);
    if (s != CSA_OK) return s;
    const int PG = a->pool_blocks * G;
    pool_expand_kernel<<<dim3((PG + 255) / 256, p.rows), 256, 0, st>>>(bidx, a->pool_blocks, G, scores, ld,
                                                                        p.n_cols, a->q_pos, a->n_c, a->ratio, a->Nq,
                                                                        a->pool_out);
    s = launch_status();
    if (s != CSA_OK) return s;
  }
  return CSA_OK;
}

// ------------------------------------------------------------------ allocation-free variant
// Scratch for csa_index_topk_noalloc: a file-scope device array, present in every GPU that loads
// this library for the life of the process.  Host code cannot use the symbol as a pointer (it is a
// host-side stand-in); its device address is looked up once per device with that device current.
static __device__ __align__(256) uint8_t g_noalloc_scratch[CSA_NOALLOC_SCRATCH_BYTES];
constexpr int NOALLOC_MAX_DEVICES = 64;
static std::atomic<uintptr_t> g_noalloc_ptr[NOALLOC_MAX_DEVICES];

static csa_status noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) { set_last_cuda_error(e); return CSA_ERR_CUDA; }
  if (dev < 0 || dev >= NOALLOC_MAX_DEVICES) return CSA_ERR_UNSUPPORTED;
  uintptr_t p = g_noalloc_ptr[dev].load(std::memory_order_acquire);
  if (p == 0) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess || ptr == nullptr) {
      set_last_cuda_error(e != cudaSuccess ? e : cudaErrorInvalidSymbol);
      return CSA_ERR_CUDA;
    }
    p = (uintptr_t)ptr;
    g_noalloc_ptr[dev].store(p, std::memory_order_release);
  }
  *out = (void*)p;
  return CSA_OK;
}

// ------------------------------------------------------------------ device error path check
// One thread waits on an mbarrier that nothing arrives on, with the given poll limit, exactly as the
// pipelines' bounded waits do; when the wait gives up it records device error 1, as they do.
__global__ void error_path_check_kernel(uint32_t polls) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x != 0) return;
  sm100::mbar_init(&bar, 1);
  sm100::fence_mbar_init();
  if (!sm100::mbar_wait(&bar, 0, polls)) atomicOr(&g_csa_device_error, 1u);
}

}  // namespace csa

using namespace csa;

extern "C" csa_status csa_check_error_path(uint32_t polls, void* stream) {
  CSA_REQUIRE(polls >= 1 && polls <= (1u << 20));
  error_path_check_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(polls);
  return launch_status();
}

extern "C" csa_status csa_index_topk_noalloc(const csa_index_args* a, void* stream) {
  csa_status v = validate_index(a, true);
  if (v != CSA_OK) return v;
  v = validate_index(a, false);
  if (v != CSA_OK) return v;
  const IndexPlan p = plan_index(a);
  if (p.rows == 0) return CSA_OK;
  if (p.total > CSA_NOALLOC_SCRATCH_BYTES) return CSA_ERR_WORKSPACE;   // before any CUDA call
  void* ws = nullptr;
  v = noalloc_scratch(&ws);
  if (v != CSA_OK) return v;
  // Nothing in the scratch needs to start at zero: every byte a call reads was written earlier in
  // the same call (scores of the visible columns, the tournament's k slots per segment, pool buffers).
  cudaStream_t st = (cudaStream_t)stream;
  uint8_t* w8 = (uint8_t*)ws;
  float* scores = (float*)(w8 + p.off_scores);
  uint32_t* hist = p.hist ? (uint32_t*)(w8 + p.off_hist) : nullptr;
  csa_status s = run_scores(a, scores, p.n_cols, hist, true, st);
  if (s != CSA_OK) return s;
  return run_select(a, p, scores, p.n_cols, hist, w8, st);
}

extern "C" csa_status csa_index_scores(const csa_index_args* a, float* scores, int64_t ld, void* stream) {
  csa_status v = validate_index(a, false);
  if (v != CSA_OK) return v;
  if ((long long)a->B * a->Nq == 0) return CSA_OK;
  const int n_cols = a->cand ? a->n_cand : a->n_max;
  CSA_REQUIRE(scores != nullptr && ld >= n_cols);
  return run_scores(a, scores, ld, a->hist, false, (cudaStream_t)stream);
}

extern "C" size_t csa_topk_workspace_size(const csa_index_args* a) {
  if (validate_index(a, true, false) != CSA_OK) return 0;
  return plan_index(a).sel_total;
}

extern "C" csa_status csa_topk(const csa_index_args* a, const float* scores, int64_t ld, void* ws, size_t ws_bytes,
                               void* stream) {
  csa_status v = validate_index(a, true);
  if (v != CSA_OK) return v;
  const IndexPlan p = plan_index(a);
  if (p.rows == 0) return CSA_OK;
  CSA_REQUIRE(scores != nullptr && ld >= p.n_cols);
  if (ws_bytes < p.sel_total) return CSA_ERR_WORKSPACE;
  CSA_REQUIRE(ws != nullptr || p.sel_total == 0);
  return run_select(a, p, scores, ld, a->hist, (uint8_t*)ws, (cudaStream_t)stream);
}

extern "C" size_t csa_index_topk_workspace_size(const csa_index_args* a) {
  if (validate_index(a, true, false) != CSA_OK) return 0;
  return plan_index(a).total;
}

extern "C" csa_status csa_index_topk(const csa_index_args* a, void* ws, size_t ws_bytes, void* stream) {
  csa_status v = validate_index(a, true);
  if (v != CSA_OK) return v;
  v = validate_index(a, false);
  if (v != CSA_OK) return v;
  const IndexPlan p = plan_index(a);
  if (p.rows == 0) return CSA_OK;
  if (index_topk_fused_eligible(a)) return run_index_topk_fused(a, (cudaStream_t)stream);   // no workspace used
  CSA_REQUIRE(ws != nullptr);
  if (ws_bytes < p.total) return CSA_ERR_WORKSPACE;
  cudaStream_t st = (cudaStream_t)stream;
  uint8_t* w8 = (uint8_t*)ws;
  float* scores = (float*)(w8 + p.off_scores);
  uint32_t* hist = p.hist ? (uint32_t*)(w8 + p.off_hist) : nullptr;
  csa_status s = run_scores(a, scores, p.n_cols, hist, true, st);
  if (s != CSA_OK) return s;
  return run_select(a, p, scores, p.n_cols, hist, w8, st);
}
