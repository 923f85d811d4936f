// Decode attention on the 5th-generation tensor cores (tcgen05, bf16 in, fp32 in tensor memory), for
// CSA rows with a 512-wide shared KV head: one CTA takes one query (all heads) and one tile of 128 keys
// of its key list [selected entries ‖ window rows]; split partials are merged by attn_merge_kernel.
// Sources: "DeepSeek-V4: エージェントが実際に使える100万トークンのコンテキスト", §ハイブリッド注意, Fig. 3 (attention
// over the top-k compressed entries plus a sliding-window branch, one softmax).
//
// Transposed formulation (the keys, not the 64 heads, fill the 128-row MMA):
//   S^T[key][h] = K[key][:] . Q[h][:]          M = 128 keys, N = 64 heads, K = 512 (32 MMAs, K-major)
//   P^T = exp2(S^T * scale*log2e - m_h)        per-head max / sum over the 128 keys with redux.sync
//   O^T[dim][h] = sum_key K[key][dim] P^T[key][h]   M = 128 dims x 4, N = 64, K = 128 keys: the same K
//                                                   tile read through an MN-major descriptor (V = K)
// The FP4 entries are dequantised exactly into bf16 (E2M1 x E4M3 x g has at most 6 significant bits);
// window rows are copied.  Partial (O / l, lse = ln l + m) per (query, tile) go to the workspace.
#include "csa_common.cuh"
#include "sm100.cuh"

namespace csa {

using namespace sm100;

constexpr int TA_THREADS = 256;            // 8 warps gather; warps 0-3 softmax + epilogue; warp 4 MMA
constexpr int TA_KEYS = 128;
constexpr uint32_t TA_TMEM_COLS = 512;
constexpr uint32_t TA_COL_S = 0;           // S^T: 64 columns
constexpr uint32_t TA_COL_O = 64;          // O^T: 4 x 64 columns
constexpr float TA_LOG2E = 1.4426950408889634f;
constexpr float TA_LN2 = 0.6931471805599453f;

struct TaSmem {
  alignas(1024) uint8_t K[8][TA_KEYS * 128];   // [dim block of 64][key][128 B], 128-byte swizzle
  alignas(1024) uint8_t Q[8][64 * 128];        // [dim block][head][128 B]
  alignas(1024) uint8_t P[TA_KEYS * 128];      // [key][64 heads bf16]
  uint32_t red[4][64];                         // per-warp partial max / sums
  float m[64], inv_l[64], lse[64];
  int kind[TA_KEYS];                           // 0 absent, 1 FP4 entry, 2 window row
  alignas(8) uint64_t bar_s, bar_p, bar_o;
  uint32_t tmem_base;
  uint32_t err;
};

struct TaParams {
  int Nq, H, ratio, n_max, k, Wn, window, splits;
  float g, scale_log2;
  const uint16_t* q;
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
  float* part_o;        // [rows][splits][H][512]
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

__device__ __forceinline__ uint32_t redux_max_u32(uint32_t v) {
  uint32_t r;
  asm volatile("redux.sync.max.u32 %0, %1, 0xffffffff;" : "=r"(r) : "r"(v));
  return r;
}
__device__ __forceinline__ uint32_t redux_add_u32(uint32_t v) {
  uint32_t r;
  asm volatile("redux.sync.add.u32 %0, %1, 0xffffffff;" : "=r"(r) : "r"(v));
  return r;
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
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]),
                 "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]),
                 "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]),
                 "+r"(r[30]), "+r"(r[31])
               :: "memory");
}

__global__ void __launch_bounds__(TA_THREADS, 1) attn_tc_kernel(const TaParams P) {
  extern __shared__ uint8_t smem_raw[];
  TaSmem& S = *reinterpret_cast<TaSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int unit = blockIdx.x;
  const int bq = unit / P.splits, split = unit % P.splits;
  const int b = bq / P.Nq;
  const long long tq = P.q_pos[bq];
  const int ncb = min(P.n_c[b], P.n_max);
  const int n_sel = P.k;
  long long wlo = 0, whi = -1;
  if (P.win && P.Wn > 0) {
    const long long p0 = P.win_pos0[b];
    wlo = max(max(0LL, tq - P.window + 1), p0);
    whi = min(tq, p0 + P.Wn - 1);
  }
  const int n_list = n_sel + (whi >= wlo ? (int)(whi - wlo + 1) : 0);
  const int key0 = split * TA_KEYS;

  if (tid == 0) {
    S.err = 0;
    mbar_init(&S.bar_s, 1);
    mbar_init(&S.bar_p, 4);
    mbar_init(&S.bar_o, 1);
    fence_mbar_init();
  }
  if (warp == 4) { tmem_alloc(&S.tmem_base, TA_TMEM_COLS); tmem_relinquish(); }

  // ---- Q (rows >= H zero) into [dim block][head][128 B]
  const uint16_t* qsrc = P.q + (size_t)bq * P.H * 512;
  for (int i = tid; i < 64 * 64; i += TA_THREADS) {
    const int h = i >> 6, c = i & 63;
    uint8_t* dst = &S.Q[c >> 3][sw128(h, c & 7)];
    if (h < P.H) cp16(dst, qsrc + (size_t)h * 512 + c * 8);
    else *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
  }
  // ---- key tile: warp w fills rows 16w .. 16w+15
  const uint8_t* codes_b = P.codes + (size_t)b * P.n_max * 224;
  const uint8_t* scales_b = P.scales + (size_t)b * P.n_max * 16;
  const uint16_t* rope_b = P.rope + (size_t)b * P.n_max * 64;
  const int32_t* idx_row = P.idx + (size_t)bq * P.k;
  int kinds[16];
  long long srcs[16];
#pragma unroll
  for (int rr = 0; rr < 16; ++rr) {
    const int row = warp * 16 + rr;
    const int li = key0 + row;
    int kind = 0;
    long long src = 0;
    if (li < n_sel) {
      const int id = idx_row[li];
      if (id >= 0 && id < ncb) { kind = 1; src = id; }
    } else if (li < n_list) {
      kind = 2;
      src = (wlo + (li - n_sel)) - P.win_pos0[b];
    }
    kinds[rr] = kind;
    srcs[rr] = src;
  }
  // window rows and RoPE slices: asynchronous copies; FP4 blocks: loads first, then dequantise
  uint4 cv[16];
  uint32_t scv[16];
#pragma unroll
  for (int rr = 0; rr < 16; ++rr) {
    const int row = warp * 16 + rr;
    if (kinds[rr] == 2) {
      const uint16_t* wrow = P.win + ((size_t)b * P.Wn + srcs[rr]) * 512;
      cp16(&S.K[lane >> 3][sw128(row, lane & 7)], wrow + lane * 8);
      cp16(&S.K[(lane + 32) >> 3][sw128(row, (lane + 32) & 7)], wrow + (lane + 32) * 8);
    } else if (kinds[rr] == 1) {
      if (lane < 14) {
        cv[rr] = *reinterpret_cast<const uint4*>(codes_b + srcs[rr] * 224 + lane * 16);
        scv[rr] = scales_b[srcs[rr] * 16 + lane];
      } else if (lane >= 16 && lane < 24) {
        const int c = 56 + (lane - 16);
        cp16(&S.K[c >> 3][sw128(row, c & 7)], rope_b + srcs[rr] * 64 + (lane - 16) * 8);
      }
    } else {
      *reinterpret_cast<uint4*>(&S.K[lane >> 3][sw128(row, lane & 7)]) = make_uint4(0, 0, 0, 0);
      *reinterpret_cast<uint4*>(&S.K[(lane + 32) >> 3][sw128(row, (lane + 32) & 7)]) = make_uint4(0, 0, 0, 0);
    }
    if (lane == 0) S.kind[row] = kinds[rr];
  }
#pragma unroll
  for (int rr = 0; rr < 16; ++rr) {
    const int row = warp * 16 + rr;
    if (kinds[rr] == 1 && lane < 14) {
      const float sc = e4m3_to_f32(scv[rr]) * P.g;
      const uint32_t w4[4] = {cv[rr].x, cv[rr].y, cv[rr].z, cv[rr].w};
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        uint32_t o[4];
#pragma unroll
        for (int bb = 0; bb < 4; ++bb) {
          const uint32_t h = e2m1x2_to_h2(w4[q4] >> (bb * 8));
          const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h));
          o[bb] = pack_bf16x2(f.x * sc, f.y * sc);
        }
        const int c = lane * 4 + q4;                          // chunk of 8 dims
        *reinterpret_cast<uint4*>(&S.K[c >> 3][sw128(row, c & 7)]) = make_uint4(o[0], o[1], o[2], o[3]);
      }
    }
  }
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
  fence_proxy_async_smem();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = S.tmem_base;

  if (warp == 4) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t ids = idesc_bf16(128, 64, 0, 0);
      for (int s = 0; s < 32; ++s) {
        const uint64_t a = smem_desc(smem_addr(S.K[s >> 2]) + (s & 3) * 32, 16, 1024, 2);
        const uint64_t bd = smem_desc(smem_addr(S.Q[s >> 2]) + (s & 3) * 32, 16, 1024, 2);
        mma_bf16_ss(tb + TA_COL_S, a, bd, ids, s > 0);
      }
      mma_commit(&S.bar_s);
      bool ok = mbar_wait(&S.bar_p, 0);
      if (ok) {
        tc_fence_after();
        const uint32_t ido = idesc_bf16(128, 64, 1, 1);
        for (int mt = 0; mt < 4; ++mt)
          for (int s = 0; s < 8; ++s) {
            const uint64_t a = smem_desc(smem_addr(S.K[2 * mt]) + s * 2048, 16384, 1024, 2);
            const uint64_t bd = smem_desc(smem_addr(S.P) + s * 2048, 16384, 1024, 2);
            mma_bf16_ss(tb + TA_COL_O + 64 * mt, a, bd, ido, s > 0);
          }
      } else {
        atomicOr(&S.err, 1u);
      }
      mma_commit(&S.bar_o);
    }
    __syncwarp();
  } else if (warp < 4) {
    // ------------------------------------------------------- softmax over the tile's keys
    const uint32_t lane_base = tb + ((uint32_t)(32 * warp) << 16);
    const int key = 32 * warp + lane;
    bool ok = mbar_wait(&S.bar_s, 0);
    tc_fence_after();
    uint32_t sv[64];
    if (ok) {
      tmem_ld_x32(lane_base + TA_COL_S, sv);
      tmem_ld_x32(lane_base + TA_COL_S + 32, sv + 32);
    }
    const bool kv = ok && S.kind[key] != 0;
    // per-head max over the 128 keys: order-preserving integer keys, one redux per warp and head
#pragma unroll
    for (int h = 0; h < 64; ++h) {
      const float z = kv ? __uint_as_float(sv[h]) * P.scale_log2 : -INFINITY;
      sv[h] = __float_as_uint(z);
      const uint32_t mk = redux_max_u32(float_order_key(z));
      if (lane == (h & 31)) S.red[warp][h] = mk;
    }
    asm volatile("bar.sync 1, 128;" ::: "memory");
    if (tid < 64) {
      uint32_t mk = max(max(S.red[0][tid], S.red[1][tid]), max(S.red[2][tid], S.red[3][tid]));
      S.m[tid] = order_key_float(mk);
    }
    asm volatile("bar.sync 1, 128;" ::: "memory");
    // probabilities (bf16 into P), per-head sums as 2^-24 fixed point (32 keys < 2^29 per warp)
    uint32_t pk[32];
#pragma unroll
    for (int h = 0; h < 64; h += 2) {
      const float m0 = S.m[h], m1 = S.m[h + 1];
      const float p0 = (m0 == -INFINITY) ? 0.f : exp2f(__uint_as_float(sv[h]) - m0);
      const float p1 = (m1 == -INFINITY) ? 0.f : exp2f(__uint_as_float(sv[h + 1]) - m1);
      pk[h >> 1] = pack_bf16x2(p0, p1);
      const uint32_t s0 = redux_add_u32(__float2uint_rn(p0 * 16777216.0f));
      const uint32_t s1 = redux_add_u32(__float2uint_rn(p1 * 16777216.0f));
      if (lane == (h & 31)) S.red[warp][h] = s0;
      if (lane == ((h + 1) & 31)) S.red[warp][h + 1] = s1;
    }
#pragma unroll
    for (int c = 0; c < 8; ++c)
      *reinterpret_cast<uint4*>(&S.P[sw128(key, c)]) = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
    fence_proxy_async_smem();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&S.bar_p);
    asm volatile("bar.sync 1, 128;" ::: "memory");
    if (tid < 64) {
      const double tot = (double)S.red[0][tid] + S.red[1][tid] + S.red[2][tid] + S.red[3][tid];
      const float l = (float)(tot * (1.0 / 16777216.0));
      const float m = S.m[tid];
      S.inv_l[tid] = l > 0.f ? 1.f / l : 0.f;
      S.lse[tid] = l > 0.f ? (m + log2f(l)) * TA_LN2 : -INFINITY;
    }
    asm volatile("bar.sync 1, 128;" ::: "memory");
    // ------------------------------------------------------------------------- epilogue
    ok = ok && mbar_wait(&S.bar_o, 0);
    tc_fence_after();
    if (!ok && lane == 0) atomicOr(&S.err, 1u);
    if (ok) {
      for (int mt = 0; mt < 4; ++mt) {
        const int dim = 128 * mt + 32 * warp + lane;
        uint32_t ov[32];
        for (int hb = 0; hb < 64; hb += 32) {
          tmem_ld_x32(lane_base + TA_COL_O + 64 * mt + hb, ov);
          if (P.splits == 1) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int h = hb + j;
              if (h < P.H)
                P.out[((size_t)bq * P.H + h) * 512 + dim] =
                    (uint16_t)f_to_bf16_bits(__uint_as_float(ov[j]) * S.inv_l[h]);
            }
          } else {
            float* po = P.part_o + ((size_t)bq * P.splits + split) * P.H * 512 + dim;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int h = hb + j;
              if (h < P.H) po[(size_t)h * 512] = __uint_as_float(ov[j]) * S.inv_l[h];
            }
          }
        }
      }
      if (tid < P.H) {
        if (P.splits == 1) {
          if (P.lse) P.lse[(size_t)bq * P.H + tid] = S.lse[tid];
        } else {
          P.part_lse[((size_t)bq * P.splits + split) * P.H + tid] = S.lse[tid];
        }
      }
    }
    tc_fence_before();
  }
  __syncthreads();
  if (S.err && tid == 0) atomicOr(&g_csa_device_error, 1u);
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tb, TA_TMEM_COLS);
  }
}

bool attn_tc_eligible(const csa_attn_args* a, int hca, long long rows) {
  return !hca && a->d == 512 && a->d_rope == 64 && a->H <= 64 && rows < 148 && a->k + (a->win_kv ? a->Wn : 0) <= 4096 &&
         ((uintptr_t)a->q & 15) == 0 && ((uintptr_t)a->kv_codes & 15) == 0 && ((uintptr_t)a->kv_rope & 15) == 0 &&
         (!a->win_kv || ((uintptr_t)a->win_kv & 15) == 0);
}

int attn_tc_splits(const csa_attn_args* a) {
  const long long n_win = (a->win_kv && a->Wn > 0) ? (a->Wn < a->window ? a->Wn : a->window) : 0;
  const long long n = a->k + n_win;
  return (int)((n + TA_KEYS - 1) / TA_KEYS);
}

csa_status launch_attn_tc(const csa_attn_args* a, int splits, float* part_o, float* part_lse, cudaStream_t st) {
  TaParams P{};
  P.Nq = a->Nq; P.H = a->H; P.ratio = a->ratio; P.n_max = a->n_max; P.k = a->k;
  P.Wn = a->win_kv ? a->Wn : 0; P.window = a->window; P.splits = splits; P.g = a->g_kv;
  const float scale = a->softmax_scale != 0.0f ? a->softmax_scale : 1.0f / sqrtf((float)a->d);
  P.scale_log2 = scale * TA_LOG2E;
  P.q = (const uint16_t*)a->q; P.q_pos = a->q_pos; P.codes = a->kv_codes; P.scales = a->kv_scales;
  P.rope = (const uint16_t*)a->kv_rope; P.n_c = a->n_c; P.idx = a->idx; P.win = (const uint16_t*)a->win_kv;
  P.win_pos0 = a->win_pos0; P.out = (uint16_t*)a->out; P.lse = a->lse; P.part_o = part_o; P.part_lse = part_lse;
  const long long rows = (long long)a->B * a->Nq;
  const int smem = (int)sizeof(TaSmem) + 1024;
  static std::atomic<unsigned> attr_done{0};
  set_smem_once((const void*)attn_tc_kernel, smem, attr_done);
  attn_tc_kernel<<<(unsigned)(rows * splits), TA_THREADS, smem, st>>>(P);
  return launch_status();
}

cudaError_t attn_take_device_error(uint32_t* out) { return take_device_error_here(out); }

}  // namespace csa
