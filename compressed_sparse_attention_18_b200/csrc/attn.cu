// Attention over compressed entries plus the sliding window: CSA (the selected entries) and HCA
// (every visible entry).  One joint softmax per (query, head); one KV head shared by all query heads.
// Sources: "DeepSeek-V4: エージェントが実際に使える100万トークンのコンテキスト", §ハイブリッド注意, Fig. 3 (attention
// over the top-k compressed entries, with a sliding-window branch for the recent uncompressed tokens)
// and Fig. 4 (HCA: dense attention over the compressed stream, same window branch).
//
// Kernel: a CTA takes one query (all H heads, padded to 16-row groups) and a range of 64-key chunks
// of that query's key list [selected or visible entries ‖ window rows].  Per chunk: gather + dequantise
// the keys into shared memory as bf16 (E2M1 x E4M3 scale x g is exact in bf16), S = Q·K^T on the
// tensor pipe (mma.sync bf16, fp32 accumulate; the head dim is split over DS warps and the partial S
// tiles are summed through shared memory), online softmax in fp32 (exp2 with log2(e) folded into the
// scale), O += P·V with P in bf16.  Split-K partials (O, lse) are merged by a second kernel.
#include "csa_common.cuh"

namespace csa {

constexpr int AT_KC = 64;        // keys per chunk
constexpr int AT_WARPS = 8;
constexpr float LOG2E = 1.4426950408889634f;
constexpr float LN2 = 0.6931471805599453f;

__device__ __forceinline__ void ldsm4(uint32_t addr, uint32_t* r) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
__device__ __forceinline__ void ldsm4t(uint32_t addr, uint32_t* r) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
__device__ __forceinline__ void mma16816(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void cpa16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src));
}
__device__ __forceinline__ void cpa4(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src));
}
__device__ __forceinline__ void cpa_commit_wait_all() {
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

// Byte offset of 16-byte chunk `c` of row `r` in a [rows][D] bf16 tile, chunks XOR-swizzled by row.
template <int D>
__device__ __forceinline__ uint32_t swz(int r, int c) {
  return (uint32_t)(r * (D * 2) + ((c ^ (r & 7)) << 4));
}

struct AttnParams {
  int B, Nq, H, d_r, ratio, n_max, k, Wn, window, splits, chunks_per_split, hca;
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
  uint16_t* out;
  float* lse;
  float* part_o;    // [B*Nq][splits][H][D]
  float* part_lse;  // [B*Nq][splits][H]
  csa_page_map pm;         // cache rows (table == NULL: contiguous [B][n_max])
};

template <int D, int DS>
__global__ void __launch_bounds__(AT_WARPS * 32, 1) attn_kernel(AttnParams P) {
  constexpr int HG = AT_WARPS / DS;         // 16-row head groups
  constexpr int HP = HG * 16;               // padded heads
  constexpr int DSL = D / DS;               // head-dim slice of one warp
  constexpr int NT_O = DSL / 8;             // O n-tiles per warp
  constexpr int NT_S = AT_KC / 8;           // S n-tiles
  constexpr int CH = D / 8;                 // 16-byte chunks per row
  const int d_n = D - P.d_r;
  const int S_blocks = d_n / 32;
  const int S_pad = (S_blocks + 3) & ~3;

  constexpr int RAW_SC = (D - (D == 512 ? 64 : 32)) / 2;   // staging row: codes | scales (16) | rope
  constexpr int RAW_ROPE = RAW_SC + 16;
  constexpr int RAW = RAW_ROPE + (D == 512 ? 64 : 32) * 2;
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* sQ = smem;                                   // [HP][D] bf16
  uint8_t* sK = sQ + HP * D * 2;                        // [AT_KC][D] bf16
  float* sS = reinterpret_cast<float*>(sK + AT_KC * D * 2);  // [HG][DS][16][AT_KC]
  uint8_t* sRaw = reinterpret_cast<uint8_t*>(sS) + (DS > 1 ? HG * DS * 16 * AT_KC * 4 : 0);  // [AT_KC][RAW]
  __shared__ int s_valid[AT_KC];

  const int unit = blockIdx.x;
  const int bq = unit / P.splits, split = unit % P.splits;
  const int b = bq / P.Nq;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int hg = warp / DS, ds = warp % DS;
  const int g = lane >> 2, t = lane & 3;

  const long long tq = P.q_pos[bq];
  const int ncb = min(P.n_c[b], P.n_max);   // entries beyond the cache capacity do not exist
  int n_sel;
  if (P.hca) {
    long long nv = (tq + 1) / P.ratio;
    n_sel = (int)max(0LL, min((long long)ncb, nv));
  } else {
    n_sel = P.k;
  }
  long long wlo = 0, whi = -1;
  if (P.win && P.Wn > 0) {
    const long long p0 = P.win_pos0[b];
    wlo = max(max(0LL, tq - P.window + 1), p0);
    whi = min(tq, p0 + P.Wn - 1);
  }
  const int n_win = whi >= wlo ? (int)(whi - wlo + 1) : 0;
  const int n_list = n_sel + n_win;
  const int n_chunks = (n_list + AT_KC - 1) / AT_KC;
  const int c_begin = split * P.chunks_per_split;
  const int c_end = min(n_chunks, c_begin + P.chunks_per_split);

  // Q -> shared (rows >= H zero)
  const uint16_t* qsrc = P.q + (size_t)bq * P.H * D;
  const uint32_t sQa0 = (uint32_t)__cvta_generic_to_shared(sQ);
  for (int i = tid; i < HP * CH; i += blockDim.x) {
    const int r = i / CH, c = i % CH;
    if (r < P.H) cpa16(sQa0 + swz<D>(r, c), qsrc + (size_t)r * D + c * 8);
    else *reinterpret_cast<uint4*>(sQ + swz<D>(r, c)) = make_uint4(0, 0, 0, 0);
  }

  float o[NT_O][4];
#pragma unroll
  for (int j = 0; j < NT_O; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
  float m_r[2] = {-INFINITY, -INFINITY}, l_r[2] = {0.f, 0.f};

  const uint32_t sQa = (uint32_t)__cvta_generic_to_shared(sQ);
  const uint32_t sKa = (uint32_t)__cvta_generic_to_shared(sK);
  const int32_t* idx_row = P.idx ? P.idx + (size_t)bq * P.k : nullptr;

  for (int c = c_begin; c < c_end; ++c) {
    __syncthreads();  // previous chunk's K tile fully consumed
    // ---- gather, phase 1: asynchronous copies (raw FP4 rows -> staging, window rows -> K tile)
    const uint32_t sRawa = (uint32_t)__cvta_generic_to_shared(sRaw);
    for (int rr = 0; rr < AT_KC / AT_WARPS; ++rr) {
      const int row = warp * (AT_KC / AT_WARPS) + rr;
      const int li = c * AT_KC + row;
      int kind = 0;  // 0 invalid, 1 entry, 2 window
      long long src = 0;
      if (li < n_sel) {
        const int id = P.hca ? li : idx_row[li];
        if (id >= 0 && id < ncb) {
          src = page_row(P.pm, b, P.n_max, id);      // row in the (contiguous or paged) cache arrays
          kind = src >= 0 ? 1 : 0;
        }
      } else if (li < n_list) {
        kind = 2;
        src = (wlo + (li - n_sel)) - P.win_pos0[b];
      }
      if (kind == 1) {
        const uint32_t dst = sRawa + row * RAW;
        if (lane < d_n / 32) cpa16(dst + lane * 16, P.codes + src * (d_n / 2) + lane * 16);
        else if (lane >= 16 && lane < 16 + P.d_r / 8)
          cpa16(dst + RAW_ROPE + (lane - 16) * 16, P.rope + src * P.d_r + (lane - 16) * 8);
        else if (lane == 31)
          for (int q4 = 0; q4 < S_pad; q4 += 4) cpa4(dst + RAW_SC + q4, P.scales + src * S_pad + q4);
      } else if (kind == 2) {
        const uint16_t* wrow = P.win + ((size_t)b * P.Wn + src) * D;
        for (int cc = lane; cc < CH; cc += 32) cpa16(sKa + swz<D>(row, cc), wrow + cc * 8);
      } else {
        for (int cc = lane; cc < CH; cc += 32) *reinterpret_cast<uint4*>(sK + swz<D>(row, cc)) = make_uint4(0, 0, 0, 0);
      }
      if (lane == 0) s_valid[row] = kind;
    }
    cpa_commit_wait_all();
    __syncthreads();
    // ---- gather, phase 2: dequantise staged FP4 rows into the K tile (bf16, exact)
    for (int rr = 0; rr < AT_KC / AT_WARPS; ++rr) {
      const int row = warp * (AT_KC / AT_WARPS) + rr;
      if (s_valid[row] != 1) continue;
      const uint8_t* raw = sRaw + row * RAW;
      if (lane < d_n / 32) {
        const uint4 cv = *reinterpret_cast<const uint4*>(raw + lane * 16);
        const float sc = e4m3_to_f32(raw[RAW_SC + lane]) * P.g;
        const uint32_t w4[4] = {cv.x, cv.y, cv.z, cv.w};
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          uint32_t outw[4];
#pragma unroll
          for (int bb = 0; bb < 4; ++bb) {
            const uint32_t h = e2m1x2_to_h2(w4[q4] >> (bb * 8));
            const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h));
            outw[bb] = pack_bf16x2(f.x * sc, f.y * sc);
          }
          *reinterpret_cast<uint4*>(sK + swz<D>(row, lane * 4 + q4)) = make_uint4(outw[0], outw[1], outw[2], outw[3]);
        }
      } else if (lane >= 16 && lane < 16 + P.d_r / 8) {
        const int rc = lane - 16;
        *reinterpret_cast<uint4*>(sK + swz<D>(row, d_n / 8 + rc)) = *reinterpret_cast<const uint4*>(raw + RAW_ROPE + rc * 16);
      }
    }
    __syncthreads();

    // ---- S partial over this warp's head-dim slice
    float sacc[NT_S][4];
#pragma unroll
    for (int j = 0; j < NT_S; ++j) sacc[j][0] = sacc[j][1] = sacc[j][2] = sacc[j][3] = 0.f;
#pragma unroll 4
    for (int ks = 0; ks < DSL / 16; ++ks) {
      const int k0 = ds * DSL + ks * 16;
      uint32_t af[4];
      {
        const int r = hg * 16 + (lane & 15);
        const int cchunk = k0 / 8 + (lane >> 4);
        ldsm4(sQa + swz<D>(r, cchunk), af);
      }
#pragma unroll
      for (int j = 0; j < NT_S; j += 2) {
        uint32_t bf[4];
        const int mi = lane >> 3;
        const int key = j * 8 + (mi >> 1) * 8 + (lane & 7);
        const int cchunk = k0 / 8 + (mi & 1);
        ldsm4(sKa + swz<D>(key, cchunk), bf);
        mma16816(sacc[j], af, bf[0], bf[1]);
        mma16816(sacc[j + 1], af, bf[2], bf[3]);
      }
    }
    if (DS > 1) {
      float* mine = sS + ((size_t)(hg * DS + ds) * 16) * AT_KC;
#pragma unroll
      for (int j = 0; j < NT_S; ++j) {
        mine[g * AT_KC + j * 8 + 2 * t] = sacc[j][0];
        mine[g * AT_KC + j * 8 + 2 * t + 1] = sacc[j][1];
        mine[(g + 8) * AT_KC + j * 8 + 2 * t] = sacc[j][2];
        mine[(g + 8) * AT_KC + j * 8 + 2 * t + 1] = sacc[j][3];
      }
      __syncthreads();
#pragma unroll
      for (int od = 0; od < DS; ++od) {
        if (od == ds) continue;
        const float* other = sS + ((size_t)(hg * DS + od) * 16) * AT_KC;
#pragma unroll
        for (int j = 0; j < NT_S; ++j) {
          sacc[j][0] += other[g * AT_KC + j * 8 + 2 * t];
          sacc[j][1] += other[g * AT_KC + j * 8 + 2 * t + 1];
          sacc[j][2] += other[(g + 8) * AT_KC + j * 8 + 2 * t];
          sacc[j][3] += other[(g + 8) * AT_KC + j * 8 + 2 * t + 1];
        }
      }
    }
    // ---- online softmax (rows g and g + 8 of this head group)
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int j = 0; j < NT_S; ++j) {
      const bool v0 = s_valid[j * 8 + 2 * t] != 0, v1 = s_valid[j * 8 + 2 * t + 1] != 0;
      sacc[j][0] = v0 ? sacc[j][0] * P.scale_log2 : -INFINITY;
      sacc[j][1] = v1 ? sacc[j][1] * P.scale_log2 : -INFINITY;
      sacc[j][2] = v0 ? sacc[j][2] * P.scale_log2 : -INFINITY;
      sacc[j][3] = v1 ? sacc[j][3] * P.scale_log2 : -INFINITY;
      mx[0] = fmaxf(mx[0], fmaxf(sacc[j][0], sacc[j][1]));
      mx[1] = fmaxf(mx[1], fmaxf(sacc[j][2], sacc[j][3]));
    }
    float corr[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 1));
      mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 2));
      const float mnew = fmaxf(m_r[h], mx[h]);
      corr[h] = (mnew == -INFINITY) ? 1.f : exp2f(m_r[h] - mnew);
      m_r[h] = mnew;
    }
    float rs[2] = {0.f, 0.f};
#pragma unroll
    for (int j = 0; j < NT_S; ++j) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int h = e >> 1;
        const float p = (m_r[h] == -INFINITY) ? 0.f : exp2f(sacc[j][e] - m_r[h]);
        sacc[j][e] = p;
        rs[h] += p;
      }
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      rs[h] += __shfl_xor_sync(0xffffffffu, rs[h], 1);
      rs[h] += __shfl_xor_sync(0xffffffffu, rs[h], 2);
      l_r[h] = l_r[h] * corr[h] + rs[h];
    }
#pragma unroll
    for (int j = 0; j < NT_O; ++j) {
      o[j][0] *= corr[0]; o[j][1] *= corr[0];
      o[j][2] *= corr[1]; o[j][3] *= corr[1];
    }
    // ---- O += P · V over this warp's head-dim slice
#pragma unroll
    for (int kk = 0; kk < AT_KC / 16; ++kk) {
      uint32_t pa[4];
      pa[0] = pack_bf16x2(sacc[2 * kk][0], sacc[2 * kk][1]);
      pa[1] = pack_bf16x2(sacc[2 * kk][2], sacc[2 * kk][3]);
      pa[2] = pack_bf16x2(sacc[2 * kk + 1][0], sacc[2 * kk + 1][1]);
      pa[3] = pack_bf16x2(sacc[2 * kk + 1][2], sacc[2 * kk + 1][3]);
#pragma unroll
      for (int j = 0; j < NT_O; j += 2) {
        uint32_t bf[4];
        const int mi = lane >> 3;
        const int key = kk * 16 + (mi & 1) * 8 + (lane & 7);
        const int cchunk = (ds * DSL + j * 8) / 8 + (mi >> 1);
        ldsm4t(sKa + swz<D>(key, cchunk), bf);
        mma16816(o[j], pa, bf[0], bf[1]);
        mma16816(o[j + 1], pa, bf[2], bf[3]);
      }
    }
  }

  // ---- epilogue
  float inv_l[2], lse_r[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    inv_l[h] = l_r[h] > 0.f ? 1.f / l_r[h] : 0.f;
    lse_r[h] = l_r[h] > 0.f ? (m_r[h] + log2f(l_r[h])) * LN2 : -INFINITY;
  }
  const int rows[2] = {hg * 16 + g, hg * 16 + g + 8};
  if (P.splits == 1) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      if (rows[h] >= P.H) continue;
      uint16_t* orow = P.out + ((size_t)bq * P.H + rows[h]) * D + ds * DSL;
#pragma unroll
      for (int j = 0; j < NT_O; ++j)
        *reinterpret_cast<uint32_t*>(orow + j * 8 + 2 * t) =
            pack_bf16x2(o[j][2 * h] * inv_l[h], o[j][2 * h + 1] * inv_l[h]);
      if (P.lse && ds == 0 && t == 0) P.lse[(size_t)bq * P.H + rows[h]] = lse_r[h];
    }
  } else {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      if (rows[h] >= P.H) continue;
      float* orow = P.part_o + (((size_t)bq * P.splits + split) * P.H + rows[h]) * D + ds * DSL;
#pragma unroll
      for (int j = 0; j < NT_O; ++j)
        *reinterpret_cast<float2*>(orow + j * 8 + 2 * t) = make_float2(o[j][2 * h] * inv_l[h], o[j][2 * h + 1] * inv_l[h]);
      if (ds == 0 && t == 0) P.part_lse[((size_t)bq * P.splits + split) * P.H + rows[h]] = lse_r[h];
    }
  }
}

// Merge split partials: lse = log sum_s exp(lse_s); out = sum_s exp(lse_s - lse) O_s.
// One CTA per (query, head); each thread owns 4 consecutive output dims, the split weights are
// computed once per CTA in shared memory.
constexpr int MERGE_MAX_SPLITS = 128;
// Split merge: one warp per (query, head).  Lane l owns dims 16l .. 16l+15 (D = 512) or 4l .. 4l+3
// (D = 128); the split lse values and all partial loads of a chunk of splits (6 or 8) are issued
// together, so a merge of up to that many splits costs about one memory round trip.  Partials are fp32 (CUDA-core path) or bf16 (tensor-core path).
constexpr int MERGE_WARPS = 4;

// One split's partial for this lane's dims, held as loaded (bf16 pairs stay packed: 8 registers for 16
// dims) and widened to fp32 only where it is summed, so a chunk of splits in flight costs few registers.
template <typename PT, int DPL>
struct PartDims;
template <>
struct PartDims<uint16_t, 16> {
  uint4 a, b;
  __device__ __forceinline__ void load(const uint16_t* p) {
    a = *reinterpret_cast<const uint4*>(p);
    b = *reinterpret_cast<const uint4*>(p + 8);
  }
  __device__ __forceinline__ float get(int i) const {
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    return (i & 1) ? __uint_as_float(w[i >> 1] & 0xFFFF0000u) : __uint_as_float(w[i >> 1] << 16);
  }
};
template <>
struct PartDims<uint16_t, 4> {
  uint2 a;
  __device__ __forceinline__ void load(const uint16_t* p) { a = *reinterpret_cast<const uint2*>(p); }
  __device__ __forceinline__ float get(int i) const {
    const uint32_t w = i < 2 ? a.x : a.y;
    return (i & 1) ? __uint_as_float(w & 0xFFFF0000u) : __uint_as_float(w << 16);
  }
};
template <>
struct PartDims<float, 16> {
  float4 f[4];
  __device__ __forceinline__ void load(const float* p) {
#pragma unroll
    for (int i = 0; i < 4; ++i) f[i] = reinterpret_cast<const float4*>(p)[i];
  }
  __device__ __forceinline__ float get(int i) const {
    const float4 v = f[i >> 2];
    return (i & 3) == 0 ? v.x : (i & 3) == 1 ? v.y : (i & 3) == 2 ? v.z : v.w;
  }
};
template <>
struct PartDims<float, 4> {
  float4 f;
  __device__ __forceinline__ void load(const float* p) { f = *reinterpret_cast<const float4*>(p); }
  __device__ __forceinline__ float get(int i) const { return i == 0 ? f.x : i == 1 ? f.y : i == 2 ? f.z : f.w; }
};

// Inverse-RoPE epilogue on one (query, head) row held one lane-slice of DPL dims per lane (lane l: dims
// DPL l .. DPL l + DPL - 1): the RoPE channels (the last DR) sit on lanes L0 .. 31, the first half of each
// pair (m) HL lanes before its second half (m + DR/2); every lane of the warp must call it.
// (x1, x2) -> (x1 cos a + x2 sin a, -x1 sin a + x2 cos a), a = t theta^(-2m/DR): the angle in double,
// reduced by 2 pi (split in two parts) before the single-precision sin / cos.  Lane l computes the
// rotation of pair m = l mod DR/2 once, and the RoPE lanes fetch theirs by shuffles, so the warp spends
// one angle per lane rather than DPL per RoPE lane.
template <int D>
__device__ __forceinline__ void inverse_rope_lanes(float* y, int lane, long long t, float theta) {
  constexpr int DPL = D / 32, DR = D == 512 ? 64 : 32, L0 = (D - DR) / DPL, HL = DR / 2 / DPL;
  float pz[DPL];
#pragma unroll
  for (int i = 0; i < DPL; ++i) pz[i] = __shfl_xor_sync(0xffffffffu, y[i], HL);
  float sn_l, cs_l;
  {
    const int m = lane % (DR / 2);
    const double ang = (double)t * exp2(-2.0 * (double)m / DR * log2((double)theta));
    const double kk = rint(ang * 0.15915494309189535);             // 1 / (2 pi)
    double red = fma(-kk, 6.283185307179586, ang);                  // 2 pi, high part
    red = fma(-kk, 2.4492935982947064e-16, red);                    // 2 pi, low part
    sincosf((float)red, &sn_l, &cs_l);
  }
  const int jl = lane - L0;
  const bool first = jl < HL;
  const int m0 = ((jl >= 0 ? jl : 0) % HL) * DPL;
#pragma unroll
  for (int i = 0; i < DPL; ++i) {
    const float sn = __shfl_sync(0xffffffffu, sn_l, m0 + i);
    const float cs = __shfl_sync(0xffffffffu, cs_l, m0 + i);
    if (jl >= 0) {
      const float x1 = first ? y[i] : pz[i], x2 = first ? pz[i] : y[i];
      y[i] = first ? fmaf(x1, cs, x2 * sn) : fmaf(-x1, sn, x2 * cs);
    }
  }
}

template <typename PT, int D>
__global__ void __launch_bounds__(MERGE_WARPS * 32) attn_merge_kernel(const PT* __restrict__ part_o,
                                                                     const float* __restrict__ part_lse, int splits,
                                                                     int H, long long units, uint16_t* __restrict__ out,
                                                                     float* __restrict__ lse,
                                                                     const int64_t* __restrict__ q_pos, float rope_theta) {
  constexpr int DPL = D / 32;
  constexpr int MERGE_CHUNK = D == 512 ? 6 : 8;   // splits whose partials are in flight at once
  const int lane = threadIdx.x & 31;
  const long long unit = (long long)blockIdx.x * MERGE_WARPS + (threadIdx.x >> 5);
  // the kernel after the merge is launched only once every merge CTA has stored its rows (the trigger is
  // at the end): launched earlier, its CTAs crowd onto the few SMs the merge leaves free (in a decode step
  // the next compressor then holds three CTAs on an SM and keeps the indexer it runs beside off it)
  pdl_wait();
  if (unit >= units) return;
  const long long bq = unit / H;
  const int h = (int)(unit % H);
  float acc[DPL];
#pragma unroll
  for (int i = 0; i < DPL; ++i) acc[i] = 0.f;
  const PT* base = part_o + (bq * splits * H + h) * (long long)D + lane * DPL;
  const float* lrow = part_lse + bq * splits * H + h;
  float mx = -INFINITY, sum = 0.f;
  if (splits <= MERGE_CHUNK) {
    // one round: every lane loads all split lse values (broadcast) and its dims of every partial; empty
    // splits (lse = -inf, partial never written) are dropped by a select, never multiplied
    PartDims<PT, DPL> v[MERGE_CHUNK];
    float ls[MERGE_CHUNK];
#pragma unroll
    for (int c = 0; c < MERGE_CHUNK; ++c) {
      ls[c] = c < splits ? lrow[(long long)c * H] : -INFINITY;
      if (c < splits) v[c].load(base + (long long)c * H * D);
    }
#pragma unroll
    for (int c = 0; c < MERGE_CHUNK; ++c) mx = fmaxf(mx, ls[c]);
#pragma unroll
    for (int c = 0; c < MERGE_CHUNK; ++c) {
      const float w = (mx == -INFINITY || ls[c] == -INFINITY) ? 0.f : exp2f((ls[c] - mx) * LOG2E);
      sum += w;
      if (w != 0.f)
#pragma unroll
        for (int i = 0; i < DPL; ++i) acc[i] = fmaf(w, v[c].get(i), acc[i]);
    }
  } else {
    // max and weights of the split lse values (lanes hold splits s = lane, lane + 32, ...)
    for (int s = lane; s < splits; s += 32) mx = fmaxf(mx, lrow[(long long)s * H]);
    mx = warp_max(mx);
    for (int s = lane; s < splits; s += 32) {
      const float l = lrow[(long long)s * H];
      sum += (mx == -INFINITY || l == -INFINITY) ? 0.f : exp2f((l - mx) * LOG2E);
    }
    sum = warp_sum(sum);
    for (int s0 = 0; s0 < splits; s0 += MERGE_CHUNK) {
      PartDims<PT, DPL> v[MERGE_CHUNK];
      float wgt[MERGE_CHUNK];
#pragma unroll
      for (int c = 0; c < MERGE_CHUNK; ++c) {
        const int s = s0 + c;
        wgt[c] = 0.f;
        if (s < splits) {
          const float l = lrow[(long long)s * H];
          wgt[c] = (mx == -INFINITY || l == -INFINITY) ? 0.f : exp2f((l - mx) * LOG2E);
        }
        if (wgt[c] != 0.f) v[c].load(base + (long long)s * H * D);
      }
#pragma unroll
      for (int c = 0; c < MERGE_CHUNK; ++c)
        if (wgt[c] != 0.f)
#pragma unroll
          for (int i = 0; i < DPL; ++i) acc[i] = fmaf(wgt[c], v[c].get(i), acc[i]);
    }
  }
  const float inv = sum > 0.f ? 1.f / sum : 0.f;
#pragma unroll
  for (int i = 0; i < DPL; ++i) acc[i] *= inv;
  if (rope_theta != 0.f) inverse_rope_lanes<D>(acc, lane, q_pos[bq], rope_theta);
  uint16_t* o = out + (bq * H + h) * (long long)D + lane * DPL;
  uint32_t pk[DPL / 2];
#pragma unroll
  for (int i = 0; i < DPL / 2; ++i) pk[i] = pack_bf16x2(acc[2 * i], acc[2 * i + 1]);
  if (DPL == 16) {
    reinterpret_cast<uint4*>(o)[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    reinterpret_cast<uint4*>(o)[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
  } else {
    *reinterpret_cast<uint2*>(o) = make_uint2(pk[0], pk[1]);
  }
  if (lse && lane == 0) lse[bq * H + h] = sum > 0.f ? mx + logf(sum) : -INFINITY;
  pdl_trigger();
}

template <typename PT>
static csa_status launch_merge(const PT* po, const float* pl, int splits, int H, int D, long long rows, uint16_t* out,
                               float* lse, const int64_t* q_pos, float rope_theta, cudaStream_t st) {
  const long long units = rows * H;
  const unsigned grid = (unsigned)((units + MERGE_WARPS - 1) / MERGE_WARPS);
  static std::atomic<unsigned> attr512{0}, attr128{0};
  set_smem_once((const void*)attn_merge_kernel<PT, 512>, 0, attr512);
  set_smem_once((const void*)attn_merge_kernel<PT, 128>, 0, attr128);
  if (D == 512)
    return launch_pdl(attn_merge_kernel<PT, 512>, dim3(grid), dim3(MERGE_WARPS * 32), 0, st, po, pl, splits, H, units,
                      out, lse, q_pos, rope_theta);
  return launch_pdl(attn_merge_kernel<PT, 128>, dim3(grid), dim3(MERGE_WARPS * 32), 0, st, po, pl, splits, H, units,
                    out, lse, q_pos, rope_theta);
}

// Inverse-RoPE epilogue in place on a finished bf16 output (launches without split partials): one warp
// per (query, head), the same lane layout and rotation as the merge.
template <int D>
__global__ void __launch_bounds__(MERGE_WARPS * 32) out_rope_kernel(uint16_t* __restrict__ out, int H, long long units,
                                                                    const int64_t* __restrict__ q_pos, float rope_theta) {
  constexpr int DPL = D / 32;
  const int lane = threadIdx.x & 31;
  const long long unit = (long long)blockIdx.x * MERGE_WARPS + (threadIdx.x >> 5);
  pdl_trigger();
  pdl_wait();
  if (unit >= units) return;
  uint16_t* o = out + unit * (long long)D + lane * DPL;
  PartDims<uint16_t, DPL> raw;
  raw.load(o);
  float y[DPL];
#pragma unroll
  for (int i = 0; i < DPL; ++i) y[i] = raw.get(i);
  inverse_rope_lanes<D>(y, lane, q_pos[unit / H], rope_theta);
  uint32_t pk[DPL / 2];
#pragma unroll
  for (int i = 0; i < DPL / 2; ++i) pk[i] = pack_bf16x2(y[2 * i], y[2 * i + 1]);
  if (DPL == 16) {
    reinterpret_cast<uint4*>(o)[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    reinterpret_cast<uint4*>(o)[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
  } else {
    *reinterpret_cast<uint2*>(o) = make_uint2(pk[0], pk[1]);
  }
}

static csa_status launch_out_rope(uint16_t* out, int H, int D, long long rows, const int64_t* q_pos, float theta,
                                  cudaStream_t st) {
  const long long units = rows * H;
  const unsigned grid = (unsigned)((units + MERGE_WARPS - 1) / MERGE_WARPS);
  static std::atomic<unsigned> attr512{0}, attr128{0};
  set_smem_once((const void*)out_rope_kernel<512>, 0, attr512);
  set_smem_once((const void*)out_rope_kernel<128>, 0, attr128);
  if (D == 512) return launch_pdl(out_rope_kernel<512>, dim3(grid), dim3(MERGE_WARPS * 32), 0, st, out, H, units, q_pos, theta);
  return launch_pdl(out_rope_kernel<128>, dim3(grid), dim3(MERGE_WARPS * 32), 0, st, out, H, units, q_pos, theta);
}

// tensor-core decode path (attn_tc.cu)
void attn_tc_plan(const csa_attn_args* a, int hca, int* splits, int* tpc);
bool attn_tc_cluster(int splits);
csa_status launch_attn_tc(const csa_attn_args* a, int hca, int splits, int tpc, uint16_t* part_o, float* part_lse,
                          cudaStream_t st);

bool attn_tc_eligible(const csa_attn_args* a, int hca, int max_splits);

struct AttnPlan {
  int splits, cps, tpc;
  bool tc;
  size_t off_o, off_lse, total;
};

static AttnPlan plan_attn(const csa_attn_args* a, int hca) {
  AttnPlan p{};
  const long long rows_tc = (long long)a->B * a->Nq;
  if (attn_tc_eligible(a, hca, MERGE_MAX_SPLITS)) {
    p.tc = true;
    p.cps = 1;
    attn_tc_plan(a, hca, &p.splits, &p.tpc);
    size_t o = 0;
    const bool cluster = attn_tc_cluster(p.splits) && (a->flags & CSA_CLUSTER_MERGE);
    if (p.splits > 1 && !cluster) {                       // (a cluster merges its query's partials on chip)
      p.off_o = o;   o = align_up(o + (size_t)rows_tc * p.splits * a->H * a->d * 2, 256);
      p.off_lse = o; o = align_up(o + (size_t)rows_tc * p.splits * a->H * 4, 256);
    }
    p.total = o;
    return p;
  }
  const long long n_sel = hca ? a->n_max : a->k;
  const long long n_win = attn_has_window(a) ? (a->Wn < a->window ? a->Wn : a->window) : 0;
  const long long chunks = (n_sel + n_win + AT_KC - 1) / AT_KC;
  const long long rows = (long long)a->B * a->Nq;
  long long splits = rows >= 148 ? 1 : 148 / rows;
  if (splits > chunks) splits = chunks;
  if (splits > MERGE_MAX_SPLITS) splits = MERGE_MAX_SPLITS;
  if (splits < 1) splits = 1;
  p.cps = (int)((chunks + splits - 1) / splits);
  if (p.cps < 1) p.cps = 1;
  p.splits = (int)((chunks + p.cps - 1) / p.cps);
  if (p.splits < 1) p.splits = 1;
  size_t o = 0;
  if (p.splits > 1) {
    p.off_o = o;   o = align_up(o + (size_t)rows * p.splits * a->H * a->d * 4, 256);
    p.off_lse = o; o = align_up(o + (size_t)rows * p.splits * a->H * 4, 256);
  }
  p.total = o;
  return p;
}

// ptrs = false (workspace-size and kernel-count queries): shapes, flags and the page map only; the buffers
// may not exist yet
static csa_status validate_attn(const csa_attn_args* a, int hca, bool ptrs = true) {
  CSA_REQUIRE(a != nullptr && a->struct_size == sizeof(csa_attn_args));
  CSA_REQUIRE(a->B >= 0 && a->Nq >= 0 && a->H >= 1 && a->ratio >= 1 && a->n_max >= 0 && a->Wn >= 0 && a->window >= 1);
  CSA_SUPPORTED((a->d == 512 && a->d_rope == 64) || (a->d == 128 && a->d_rope == 32));
  CSA_SUPPORTED(a->H <= (a->d == 512 ? 64 : 16));
  CSA_REQUIRE(a->g_kv > 0.0f);
  CSA_REQUIRE(a->out_rope_theta >= 0.0f);        // (false for NaN too)
  CSA_REQUIRE(a->win_format == CSA_WIN_BF16 || a->win_format == CSA_WIN_FP8);
  if (!hca) CSA_REQUIRE(a->k >= 1);
  {
    const csa_status pv = check_page_map(a->kv_pages, a->n_max);
    if (pv != CSA_OK) return pv;
  }
  if ((long long)a->B * a->Nq == 0 || !ptrs) return CSA_OK;
  CSA_REQUIRE(a->q && a->q_pos && a->n_c && a->out);
  CSA_REQUIRE(a->n_max == 0 || (a->kv_codes && a->kv_scales && a->kv_rope));
  if (!hca) CSA_REQUIRE(a->idx != nullptr);
  if (a->Wn > 0 && a->win_format == CSA_WIN_BF16) CSA_REQUIRE(a->win_kv && a->win_pos0);
  if (a->Wn > 0 && a->win_format == CSA_WIN_FP8) {
    CSA_REQUIRE(a->win_codes && a->win_scales && a->win_rope && a->win_pos0);
    // FP8 window rows are read by the tensor-core path only (d = 512, 16-byte aligned rows)
    CSA_SUPPORTED(attn_tc_eligible(a, hca, MERGE_MAX_SPLITS));
  }
  return CSA_OK;
}

template <int D, int DS>
static csa_status launch_attn(const AttnParams& P, int units, cudaStream_t st) {
  constexpr int HG = AT_WARPS / DS;
  constexpr int RAW = (D - (D == 512 ? 64 : 32)) / 2 + 16 + (D == 512 ? 64 : 32) * 2;
  const size_t smem = (size_t)HG * 16 * D * 2 + (size_t)AT_KC * D * 2 + (DS > 1 ? (size_t)HG * DS * 16 * AT_KC * 4 : 0) +
                      (size_t)AT_KC * RAW;
  static std::atomic<unsigned> attr_done{0};
  set_smem_once((const void*)attn_kernel<D, DS>, (int)smem, attr_done);
  attn_kernel<D, DS><<<units, AT_WARPS * 32, smem, st>>>(P);
  return launch_status();
}

static csa_status run_attn(const csa_attn_args* a, void* ws, size_t ws_bytes, void* stream, int hca) {
  csa_status v = validate_attn(a, hca);
  if (v != CSA_OK) return v;
  const long long rows = (long long)a->B * a->Nq;
  if (rows == 0) return CSA_OK;
  const AttnPlan p = plan_attn(a, hca);
  if (ws_bytes < p.total) return CSA_ERR_WORKSPACE;
  CSA_REQUIRE(p.total == 0 || ws != nullptr);
  cudaStream_t st = (cudaStream_t)stream;
  if (p.tc) {
    const bool on_chip = p.splits == 1 || (attn_tc_cluster(p.splits) && (a->flags & CSA_CLUSTER_MERGE));
    uint16_t* po = !on_chip ? (uint16_t*)((uint8_t*)ws + p.off_o) : nullptr;
    float* pl = !on_chip ? (float*)((uint8_t*)ws + p.off_lse) : nullptr;
    csa_status s = launch_attn_tc(a, hca, p.splits, p.tpc, po, pl, st);
    if (s != CSA_OK) return s;
    const bool merged = on_chip;
    if (merged)
      return a->out_rope_theta != 0.0f
                 ? launch_out_rope((uint16_t*)a->out, a->H, a->d, rows, a->q_pos, a->out_rope_theta, st)
                 : CSA_OK;
    return launch_merge<uint16_t>(po, pl, p.splits, a->H, a->d, rows, (uint16_t*)a->out, a->lse, a->q_pos,
                                  a->out_rope_theta, st);
  }
  AttnParams P{};
  P.B = a->B; P.Nq = a->Nq; P.H = a->H; P.d_r = a->d_rope; P.ratio = a->ratio; P.n_max = a->n_max;
  P.k = a->k; P.Wn = a->win_kv ? a->Wn : 0; P.window = a->window; P.splits = p.splits;
  P.chunks_per_split = p.cps; P.hca = hca;
  P.g = a->g_kv;
  const float scale = a->softmax_scale != 0.0f ? a->softmax_scale : 1.0f / sqrtf((float)a->d);
  P.scale_log2 = scale * LOG2E;
  P.q = (const uint16_t*)a->q; P.q_pos = a->q_pos; P.codes = a->kv_codes; P.scales = a->kv_scales;
  P.rope = (const uint16_t*)a->kv_rope; P.n_c = a->n_c; P.idx = hca ? nullptr : a->idx; P.pm = a->kv_pages;
  P.win = (const uint16_t*)a->win_kv; P.win_pos0 = a->win_pos0; P.out = (uint16_t*)a->out; P.lse = a->lse;
  P.part_o = p.splits > 1 ? (float*)((uint8_t*)ws + p.off_o) : nullptr;
  P.part_lse = p.splits > 1 ? (float*)((uint8_t*)ws + p.off_lse) : nullptr;
  const int units = (int)(rows * p.splits);
  csa_status s;
  if (a->d == 512)
    s = launch_attn<512, 2>(P, units, st);
  else
    s = launch_attn<128, 8>(P, units, st);
  if (s != CSA_OK) return s;
  if (p.splits == 1)
    return a->out_rope_theta != 0.0f
               ? launch_out_rope((uint16_t*)a->out, a->H, a->d, rows, a->q_pos, a->out_rope_theta, st)
               : CSA_OK;
  return launch_merge<float>(P.part_o, P.part_lse, p.splits, a->H, a->d, rows, (uint16_t*)a->out, a->lse, a->q_pos,
                             a->out_rope_theta, st);
}

}  // namespace csa

using namespace csa;

extern "C" size_t csa_attn_workspace_size(const csa_attn_args* a, int hca) {
  if (validate_attn(a, hca, false) != CSA_OK) return 0;
  return plan_attn(a, hca).total;
}

extern "C" int csa_attn_kernel_count(const csa_attn_args* a, int hca) {
  if (validate_attn(a, hca, false) != CSA_OK) return -1;
  if ((long long)a->B * a->Nq == 0) return 0;
  const AttnPlan p = plan_attn(a, hca);
  const bool rope = a->out_rope_theta != 0.0f;
  if (p.tc) {
    const bool on_chip = p.splits == 1 || (attn_tc_cluster(p.splits) && (a->flags & CSA_CLUSTER_MERGE));
    return on_chip ? (rope ? 2 : 1) : 2;
  }
  return p.splits > 1 ? 2 : (rope ? 2 : 1);
}

extern "C" csa_status csa_sparse_attn(const csa_attn_args* a, void* ws, size_t ws_bytes, void* stream) {
  return run_attn(a, ws, ws_bytes, stream, 0);
}

extern "C" csa_status hca_dense_attn(const csa_attn_args* a, void* ws, size_t ws_bytes, void* stream) {
  return run_attn(a, ws, ws_bytes, stream, 1);
}
