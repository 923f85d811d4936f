// Attention on the 5th-generation tensor cores (tcgen05, bf16 in, fp32 accumulators in tensor memory), for
// rows with a 512-wide shared KV head (64-wide RoPE slice): one CTA takes one query (all heads) and one tile
// of 128 keys of its key list [selected (or, dense, all visible) entries ‖ window rows]; the partials of a
// query's tiles are merged by attn_merge_kernel.
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
// Partial (O / l in bf16, lse = ln l + m in fp32) per (query, tile) go to the workspace; with one tile the
// CTA writes the bf16 output and lse itself.
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

struct TaSmem {
  alignas(1024) uint8_t K[8][TA_KEYS * 128];   // [dim block of 64][key][128 B], 128-byte swizzle
  alignas(1024) uint8_t Q[8][64 * 128];        // [dim block][head][128 B]
  alignas(1024) uint8_t P[TA_KEYS * 128];      // [key][64 heads bf16]
  float red_m[4][64], red_l[4][64];            // per lane-quadrant partial max / sum
  float m[64], inv_l[64], lse[64];
  int32_t ids[TA_KEYS];                        // entry id of each entry row, -1 if absent
  // per dim block: Q landed, window boxes landed, gathered rows written
  alignas(8) uint64_t bar_q[8], bar_w[8], bar_k[8];
  uint64_t bar_s, bar_p, bar_o[4];
  uint32_t tmem_base;
  uint32_t err;
};
struct TaParams {
  int Nq, H, ratio, n_max, k, Wn, window, splits, hca;
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
  uint16_t* part_o;     // [rows][splits][H][512] bf16
  float* part_lse;      // [rows][splits][H]
};

__device__ __forceinline__ uint32_t sw128(int row, int chunk) { return (uint32_t)(row * 128 + ((chunk ^ (row & 7)) << 4)); }

__device__ __forceinline__ void mma_bf16_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, bool acc) {
  asm volatile("{ .reg .pred p; setp.ne.b32 p, %4, 0;\n\ttcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p; }"
               ::"r"(d), "l"(a), "l"(b), "r"(idesc), "r"((uint32_t)acc) : "memory");
}
// kind::f16 instruction descriptor: bf16 A and B, fp32 accumulate; a_mn / b_mn select MN-major operands.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, int a_mn, int b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void cp16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(dst)), "l"(src));
}

__device__ __forceinline__ void tmem_ld_x32(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr) : "memory");
}
__device__ __forceinline__ void tmem_wait_ld_x32(uint32_t* r) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]),
                 "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]),
                 "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]),
                 "+r"(r[30]), "+r"(r[31])
               :: "memory");
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

__global__ void __launch_bounds__(TA_THREADS, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap wmap,
                   const TaParams P) {
  extern __shared__ uint8_t smem_raw[];
  TaSmem& S = *reinterpret_cast<TaSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bq = blockIdx.x / P.splits, split = blockIdx.x % P.splits;
  const int b = bq / P.Nq;
  const int key0 = split * TA_KEYS;
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
  pdl_trigger();
  pdl_wait();
  int id_raw = -1;
  if (!P.hca && tid < TA_WORKERS && key0 + grow < P.k) id_raw = P.idx[(size_t)bq * P.k + key0 + grow];
  const long long tq = P.q_pos[bq];
  const int ncb = min(P.n_c[b], P.n_max);
  int n_sel = P.k;
  if (P.hca) {                                   // all visible entries: r*i + r - 1 <= t and i < n_c
    long long nv = (tq + 1) / P.ratio;
    n_sel = (int)max(0LL, min(nv, (long long)ncb));
  }
  long long wlo = 0, whi = -1, p0 = 0;
  if (P.Wn > 0) {
    p0 = P.win_pos0[b];
    wlo = max(max(0LL, tq - P.window + 1), p0);
    whi = min(tq, p0 + P.Wn - 1);
  }
  const int n_list = n_sel + (whi >= wlo ? (int)(whi - wlo + 1) : 0);
  const size_t unit_ho = ((size_t)bq * P.splits + split) * P.H;
  // tile rows: [0, rs) entries, [rs, rw) window rows, [rw, 128) empty
  const int rs = min(max(n_sel - key0, 0), TA_KEYS);
  const int rw = max(min(n_list - key0, TA_KEYS), 0);
  const int wa = (rs + TA_WBOX - 1) / TA_WBOX * TA_WBOX;            // window rows >= wa come by TMA boxes
  const int we = rw > wa ? (rw + TA_WBOX - 1) / TA_WBOX * TA_WBOX : wa;
  const int zs = rw > wa ? we : rw;                                 // rows >= zs are zero-filled
  // window buffer row of tile row r (r >= rs)
  const long long wrow_base = (wlo - p0) + (long long)(key0 - n_sel);
  // entry ids of the tile rows for the softmax masks (the gather threads keep their own copies)
  if (tid < TA_WORKERS && ghalf == 0) {
    int id = -1;
    if (grow < rs) {
      const int v = P.hca ? key0 + grow : id_raw;
      if (v >= 0 && v < ncb) id = v;
    }
    S.ids[grow] = id;
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = S.tmem_base;

  if (key0 >= n_list) {                          // nothing in this tile: an empty partial
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

  if (warp == 8) {
    // ------------------------------------------------------------------ control: TMA, then MMA issue
    if (lane == 0) {
      const int nbox = (we - wa) / TA_WBOX;
#pragma unroll 1
      for (int j = 0; j < 8; ++j) {
        mbar_arrive_expect_tx(&S.bar_q[j], 64 * 128);
        tma_load_3d(S.Q[j], &qmap, j * 64, 0, bq, &S.bar_q[j]);
        mbar_arrive_expect_tx(&S.bar_w[j], (uint32_t)(nbox * TA_WBOX * 128));
        for (int i = 0; i < nbox; ++i)
          tma_load_3d(&S.K[j][(wa + i * TA_WBOX) * 128], &wmap, j * 64, (int)(wrow_base + wa + i * TA_WBOX), b,
                      &S.bar_w[j]);
      }
      bool ok = true;
      const uint32_t ids = idesc_bf16(128, 64, 0, 0);
#pragma unroll 1
      for (int j = 0; j < 8 && ok; ++j) {
        ok = mbar_wait(&S.bar_q[j], 0) && mbar_wait(&S.bar_w[j], 0) && mbar_wait(&S.bar_k[j], 0);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int s = 0; s < 4; ++s) {
          const uint64_t a = smem_desc(smem_addr(S.K[j]) + s * 32, 16, 1024, 2);
          const uint64_t bd = smem_desc(smem_addr(S.Q[j]) + s * 32, 16, 1024, 2);
          mma_bf16_ss(tb + TA_COL_S, a, bd, ids, (j | s) != 0);
        }
      }
      mma_commit(&S.bar_s);
      ok = ok && mbar_wait(&S.bar_p, 0);
      if (ok) tc_fence_after();
      const uint32_t ido = idesc_bf16(128, 64, 1, 1);
#pragma unroll 1
      for (int mt = 0; mt < 4; ++mt) {
        if (ok) {
#pragma unroll
          for (int s = 0; s < 8; ++s) {
            const uint64_t a = smem_desc(smem_addr(S.K[2 * mt]) + s * 2048, 16384, 1024, 2);
            const uint64_t bd = smem_desc(smem_addr(S.P) + s * 2048, 16384, 1024, 2);
            mma_bf16_ss(tb + TA_COL_O + 64 * mt, a, bd, ido, s > 0);
          }
        }
        mma_commit(&S.bar_o[mt]);
      }
      if (!ok) atomicOr(&S.err, 1u);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------------------------- workers
    const uint8_t* codes_b = P.codes + (size_t)b * P.n_max * 224;
    const uint8_t* scales_b = P.scales + (size_t)b * P.n_max * 16;
    const uint16_t* rope_b = P.rope + (size_t)b * P.n_max * 64;
    int id = -1;
    if (grow < rs) {
      const int v = P.hca ? key0 + grow : id_raw;
      if (v >= 0 && v < ncb) id = v;
    }
    // FP4 blocks 2j + ghalf (j = 0..6) of the row and its scale row; loads first
    uint4 cv[7];
    uint4 sc16 = make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int j = 0; j < 7; ++j) cv[j] = make_uint4(0, 0, 0, 0);
    if (id >= 0) {
      const uint8_t* crow = codes_b + (size_t)id * 224 + ghalf * 16;
#pragma unroll
      for (int j = 0; j < 7; ++j) cv[j] = __ldg(reinterpret_cast<const uint4*>(crow + j * 32));
      sc16 = __ldg(reinterpret_cast<const uint4*>(scales_b + (size_t)id * 16));
    }
    // RoPE slice (dim block 7): 4 x 16 B of the row per thread
    if (grow < rs) {
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int part = ghalf * 4 + c;
        uint8_t* dst = &S.K[7][sw128(grow, part)];
        if (id >= 0) cp16(dst, rope_b + (size_t)id * 64 + part * 8);
        else *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
      }
    }
    // window rows before the first TMA box, by asynchronous copies
    {
      const int r_end = min(wa, rw);
      const int n = (r_end > rs ? r_end - rs : 0) * 64;
      for (int i = tid; i < n; i += TA_WORKERS) {
        const int row = rs + (i >> 6), c = i & 63;
        const long long wr = wrow_base + row;
        cp16(&S.K[c >> 3][sw128(row, c & 7)], P.win + ((size_t)b * P.Wn + wr) * 512 + c * 8);
      }
    }
    // empty rows
    for (int i = tid; i < (TA_KEYS - zs) * 64; i += TA_WORKERS) {
      const int row = zs + (i >> 6), c = i & 63;
      *reinterpret_cast<uint4*>(&S.K[c >> 3][sw128(row, c & 7)]) = make_uint4(0, 0, 0, 0);
    }
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
    // dequantise dim block by dim block: bf16(e2m1 * bf16(e4m3 * g)); each block released to the MMA warp
    const uint32_t scw[4] = {sc16.x, sc16.y, sc16.z, sc16.w};
#pragma unroll
    for (int j = 0; j < 7; ++j) {
      if (grow < rs) {
        const int part = 2 * j + ghalf;
        const uint32_t sb = f_to_bf16_bits(e4m3_to_f32((scw[part >> 2] >> ((part & 3) * 8)) & 0xFFu) * P.g);
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
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(&S.bar_k[7]);
    asm volatile("bar.sync 1, 256;" ::: "memory");   // workers only: ids visible to the softmax

    // ---- softmax: warp w reads lanes 32*(w%4).. (its keys) and head half w/4
    const int quad = warp & 3, hh = warp >> 2;
    const int key = 32 * quad + lane;
    const uint32_t lane_base = tb + ((uint32_t)(32 * quad) << 16);
    bool ok = mbar_wait(&S.bar_s, 0);
    tc_fence_after();
    float z[32], red[32];
    {
      uint32_t sv[32];
      tmem_ld_x32(lane_base + TA_COL_S + hh * 32, sv);
      tmem_wait_ld_x32(sv);
      const bool valid = key < rs ? (S.ids[key] >= 0) : (key < rw);
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        z[j] = valid ? __uint_as_float(sv[j]) * P.scale_log2 : -INFINITY;
        red[j] = z[j];
      }
    }
    S.red_m[quad][hh * 32 + lane] = transpose_reduce32<true>(red, lane);
    asm volatile("bar.sync 1, 256;" ::: "memory");
    if (tid < 64) S.m[tid] = fmaxf(fmaxf(S.red_m[0][tid], S.red_m[1][tid]), fmaxf(S.red_m[2][tid], S.red_m[3][tid]));
    asm volatile("bar.sync 1, 256;" ::: "memory");
    {
      uint32_t pk[16];
#pragma unroll
      for (int j = 0; j < 32; j += 2) {
        const float m0 = S.m[hh * 32 + j], m1 = S.m[hh * 32 + j + 1];
        const float p0 = m0 == -INFINITY ? 0.f : exp2f(z[j] - m0);
        const float p1 = m1 == -INFINITY ? 0.f : exp2f(z[j + 1] - m1);
        red[j] = p0;
        red[j + 1] = p1;
        pk[j >> 1] = pack_bf16x2(p0, p1);
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
    if (tid < 64) {
      const float l = (S.red_l[0][tid] + S.red_l[1][tid]) + (S.red_l[2][tid] + S.red_l[3][tid]);
      S.inv_l[tid] = l > 0.f ? 1.f / l : 0.f;
      S.lse[tid] = l > 0.f ? (S.m[tid] + log2f(l)) * TA_LN2 : -INFINITY;
    }
    asm volatile("bar.sync 1, 256;" ::: "memory");

    // ---- epilogue, M-tile by M-tile as the O MMAs complete: lane = dim, columns = heads
    float il[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) il[j] = S.inv_l[hh * 32 + j];
    const int hmax = min(32, P.H - hh * 32);
#pragma unroll 1
    for (int mt = 0; mt < 4; ++mt) {
      ok = mbar_wait(&S.bar_o[mt], 0) && ok;
      tc_fence_after();
      uint32_t ov[32];
      tmem_ld_x32(lane_base + TA_COL_O + 64 * mt + hh * 32, ov);
      tmem_wait_ld_x32(ov);
      const int dim = 128 * mt + 32 * quad + lane;
      if (P.splits == 1) {
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
    if (tid < P.H) {
      if (P.splits == 1) {
        if (P.lse) P.lse[(size_t)bq * P.H + tid] = S.lse[tid];
      } else {
        P.part_lse[unit_ho + tid] = S.lse[tid];
      }
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 8) {
    if (S.err && lane == 0) atomicOr(&g_csa_device_error, 1u);
    tc_fence_after();
    tmem_dealloc(tb, TA_TMEM_COLS);
  }
}

int attn_tc_splits(const csa_attn_args* a, int hca) {
  const long long n_win = (a->win_kv && a->Wn > 0) ? (a->Wn < a->window ? a->Wn : a->window) : 0;
  const long long n = (hca ? a->n_max : a->k) + n_win;
  return (int)((n + TA_KEYS - 1) / TA_KEYS);
}

bool attn_tc_eligible(const csa_attn_args* a, int hca, int max_splits) {
  const int splits = attn_tc_splits(a, hca);
  return a->d == 512 && a->d_rope == 64 && a->H <= 64 && splits >= 1 && splits <= max_splits &&
         ((uintptr_t)a->q & 15) == 0 && (a->n_max == 0 || (((uintptr_t)a->kv_codes & 15) == 0 &&
                                                           ((uintptr_t)a->kv_rope & 15) == 0)) &&
         (!a->win_kv || a->Wn == 0 || ((uintptr_t)a->win_kv & 15) == 0) && tensor_map_encoder() != nullptr;
}

csa_status launch_attn_tc(const csa_attn_args* a, int hca, int splits, uint16_t* part_o, float* part_lse,
                          cudaStream_t st) {
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
  const int Wn = (a->win_kv && a->Wn > 0) ? a->Wn : 0;
  if (Wn > 0) {
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
  P.Nq = a->Nq; P.H = a->H; P.ratio = a->ratio; P.n_max = a->n_max; P.k = hca ? 0 : a->k;
  P.Wn = Wn; P.window = a->window; P.splits = splits; P.hca = hca; P.g = a->g_kv;
  const float scale = a->softmax_scale != 0.0f ? a->softmax_scale : 1.0f / sqrtf((float)a->d);
  P.scale_log2 = scale * TA_LOG2E;
  P.q_pos = a->q_pos; P.codes = a->kv_codes; P.scales = a->kv_scales;
  P.rope = (const uint16_t*)a->kv_rope; P.n_c = a->n_c; P.idx = hca ? nullptr : a->idx; P.win = (const uint16_t*)a->win_kv;
  P.win_pos0 = a->win_pos0; P.out = (uint16_t*)a->out; P.lse = a->lse; P.part_o = part_o; P.part_lse = part_lse;
  const int smem = (int)sizeof(TaSmem) + 1024;
  static std::atomic<unsigned> attr_done{0};
  set_smem_once((const void*)attn_tc_kernel, smem, attr_done);
  return launch_pdl(attn_tc_kernel, dim3((unsigned)(rows * splits)), dim3(TA_THREADS), (size_t)smem, st, qmap, wmap, P);
}

cudaError_t attn_take_device_error(uint32_t* out) { return take_device_error_here(out); }

}  // namespace csa
