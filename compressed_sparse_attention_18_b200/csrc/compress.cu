// Compressor: C = x·W_kv and Z = x·W_g (bf16 out), then per-channel softmax-gated pooling of
// non-overlapping groups of r tokens with a learned per-slot bias, RoPE on the pooled RoPE slice,
// and the indexer-key projection k_I = c·W_IK.
// Sources: "DeepSeek-V4: エージェントが実際に使える100万トークンのコンテキスト", §ハイブリッド注意, Fig. 3 (every 4
// tokens folded into one entry by softmax-gated pooling with a learned positional bias) and Fig. 4
// (128x for HCA); "DeepSeek-V4.1-Flash - Pushing the Limits of KV Cache Compression", CED bullet eq.(1)
// (entries C and gate logits Z are separate projections) and CSA2 bullet (no overlapping entries;
// indexer K projected from the main KV).
#include "csa_common.cuh"
#include "sm100.cuh"

namespace csa {

// The projections C = x·W_kv, Z = x·W_g run on the tensor cores (project_tc.cu).
csa_status run_projection_tc(const void* x, const void* W0, const void* W1, void* C, void* Z, long long M, int N,
                             int K, cudaStream_t st);

// --------------------------------------------------------------------------------------- pooling
// One CTA per (sequence, group of POOL_ENT entries, slice of OW indexer-key outputs).  Threads walk the
// d channels: per-channel softmax over the r slots of (Z + b_pos), weighted sum of C (all loads of a
// channel issued together when r <= 8; an online softmax streams longer groups); RoPE on the last d_r
// channels at the group-start position (the angle pos * theta^(-2m/d_r) and its reduction mod 2 pi in
// double, computed while the pooling loads are in flight; sin / cos of the reduced angle and the
// rotation in single precision); bf16 round; optionally the FP4 pack of c straight into the cache (slice
// 0 only); k_I[slice] = bf16(c · W_IK[:, slice]) with W_IK read from global memory (for short channel
// loops the slice is loaded into registers at kernel start), and its FP4 blocks packed into the cache.
constexpr int POOL_ENT = 4;
constexpr int POOL_THREADS = 256;
constexpr int POOL_WARPS = POOL_THREADS / 32;
constexpr int POOL_MAX_HALF = 32;   // RoPE pairs per row

struct PoolParams {
  const uint16_t* C;
  const uint16_t* Z;
  const float* b_pos;
  int T, d, d_r, r;
  float theta;
  const int64_t* pos0;
  const uint16_t* W_IK;
  int d_I;
  uint16_t* c_out;
  uint16_t* kI_out;
  csa_fp4_cache kv, ki;
  double inv_freq[POOL_MAX_HALF];   // theta^(-2m/d_r), m < d_r/2
};

__device__ __forceinline__ void pack_row_to_cache(const float* row, int d, int d_r, const csa_fp4_cache& cc, int b,
                                                  int entry) {
  const int d_n = d - d_r;
  const int S = d_n / 32, S_pad = (S + 3) & ~3;
  const long long dst = page_row(cc.pages, b, cc.n_max, (long long)(cc.row0 ? cc.row0[b] : 0) + entry);
  if (dst < 0) return;                          // a page outside the pool: nothing is written
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  for (int blk = warp; blk < S; blk += nw)
    pack_block_warp(row[blk * 32 + lane], cc.global_scale, cc.codes + dst * (d_n / 2) + blk * 16,
                    cc.scales + dst * S_pad + blk);
  if (threadIdx.x < S_pad - S) cc.scales[dst * S_pad + S + threadIdx.x] = 0;
  for (int e = threadIdx.x; e < d_r; e += blockDim.x)
    reinterpret_cast<uint16_t*>(cc.rope)[dst * d_r + e] = (uint16_t)(__float_as_uint(row[d_n + e]) >> 16);
}

__device__ __forceinline__ void fma8_bf16(float* acc, float p, const uint4& w) {
  const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    acc[2 * k] = fmaf(p, __uint_as_float(ww[k] << 16), acc[2 * k]);
    acc[2 * k + 1] = fmaf(p, __uint_as_float(ww[k] & 0xFFFF0000u), acc[2 * k + 1]);
  }
}

// OW: indexer-key outputs per CTA (32, 64 or 128); PRE: channels per thread when the W_IK slice is
// preloaded into registers (0: streamed).
template <int OW, int PRE, int ENT, int R>
__global__ void __launch_bounds__(POOL_THREADS) pool_kernel(PoolParams P) {
  constexpr int NOC = OW / 8;                       // 8-output chunks of the slice
  constexpr int NCHP = POOL_THREADS / NOC;          // channel phases
  // shared memory: pooled [ENT][d] fp32 | red [POOL_WARPS][ENT][OW] | k_I rows [ENT][OW]
  extern __shared__ __align__(128) float pooled[];
  const int b = blockIdx.y, z = blockIdx.z;
  const int d = P.d, d_r = P.d_r, r = R > 0 ? R : P.r, T = P.T, d_I = P.d_I;
  constexpr int RJ = R > 0 ? R : 8;                 // slots loaded per channel in the short-group path
  const int n_out = T / r;
  const int e0 = blockIdx.x * ENT;
  const int ne = min(ENT, n_out - e0);
  const int d_n = d - d_r;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int oc = tid % NOC, chp = tid / NOC;
  const int o_base = z * OW + oc * 8;
  // C, Z, the caches may come from the previous kernel.  Dependents are released only after the wait, so
  // when the next kernel starts, everything before this one on the stream has completed (the contract
  // that lets the indexer and the window tiles of attention start early in a decode step)
  pdl_wait();
  pdl_trigger();
  // W_IK slice into registers: before short groups (its latency overlaps their pooling), after long
  // ones (whose pooling needs the registers)
  uint4 wpre[PRE > 0 ? PRE : 1];
  auto load_w = [&]() {
    if (PRE > 0 && P.W_IK) {
#pragma unroll
      for (int i = 0; i < PRE; ++i) {
        const int ch = chp + NCHP * i;
        wpre[i] = ch < d ? __ldg(reinterpret_cast<const uint4*>(P.W_IK + (size_t)ch * d_I + o_base))
                         : make_uint4(0, 0, 0, 0);
      }
    }
  };
  const bool long_groups = R == 0 && r > 8;
  if (!long_groups) load_w();
  // RoPE angle of this thread's (entry, pair): pos * inv_freq and its reduction mod 2 pi in double, then
  // sin / cos of the reduced angle (|a| <= pi) in single precision
  const int half = d_r >> 1;
  const long long p0 = P.pos0 ? P.pos0[b] : 0;
  const bool rope_thread = P.theta != 0.0f && tid < ne * half;
  float rs_sn = 0.f, rs_cs = 1.f;
  auto rope_angle = [&]() {
    const int q = tid / half, mm = tid % half;
    const double ang = (double)(p0 + (long long)(e0 + q) * r) * P.inv_freq[mm];
    const double kk = rint(ang * 0.15915494309189535);              // 1 / (2 pi)
    double red = fma(-kk, 6.283185307179586, ang);                   // 2 pi, high part
    red = fma(-kk, 2.4492935982947064e-16, red);                     // 2 pi, low part
    sincosf((float)red, &rs_sn, &rs_cs);
  };
  const uint16_t* __restrict__ C = P.C;
  const uint16_t* __restrict__ Z = P.Z;
  const float* __restrict__ b_pos = P.b_pos;
  if (R > 0 || r <= 8) {
    // two channels per thread per round, all their loads issued before any arithmetic
    for (int i0 = tid; i0 < ne * d; i0 += 2 * POOL_THREADS) {
      float a[2][RJ], c[2][RJ];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int i = min(i0 + u * POOL_THREADS, ne * d - 1);
        const int q = i / d, ch = i % d;
        const size_t tok0 = (size_t)b * T + (size_t)(e0 + q) * r;
#pragma unroll
        for (int j = 0; j < RJ; ++j) {
          a[u][j] = j < r ? bf16_bits_to_f(Z[(tok0 + j) * d + ch]) + b_pos[(size_t)j * d + ch] : -INFINITY;
          c[u][j] = j < r ? bf16_bits_to_f(C[(tok0 + j) * d + ch]) : 0.f;
        }
      }
      if (i0 == tid && rope_thread) rope_angle();    // overlaps the loads of the first round
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int i = i0 + u * POOL_THREADS;
        if (i >= ne * d) continue;
        float m = a[u][0];
#pragma unroll
        for (int j = 1; j < RJ; ++j) m = fmaxf(m, a[u][j]);
        float l = 0.f, acc = 0.f;
#pragma unroll
        for (int j = 0; j < RJ; ++j) {
          const float p = j < r ? __expf(a[u][j] - m) : 0.f;
          l += p;
          acc = fmaf(p, c[u][j], acc);
        }
        pooled[i] = acc / l;
      }
    }
    if (ne * d <= tid && rope_thread) rope_angle();
  } else if (R == 0) {
    // long groups (r > 8): a thread owns 8 adjacent channels of one entry (16-byte loads of C and Z)
    // and one phase of the slots (j = ph, ph + split, ...); 4 slots per round with all their loads
    // issued together, an online softmax per channel, the phases merged by shuffles of adjacent lanes
    if (rope_thread) rope_angle();
    const int d8 = d >> 3, items = ne * d8;
    int split = 1;
    while (split < 16 && 2 * split <= r && 2 * split * items <= POOL_THREADS) split <<= 1;
    const int per = POOL_THREADS / split, ph = tid & (split - 1);
    for (int base = 0; base < items; base += per) {   // uniform trip count: every lane reaches the shuffles
      const int it = base + tid / split;
      const bool act = it < items;
      const int q = act ? it / d8 : 0, ch = act ? (it % d8) * 8 : 0;
      const size_t tok0 = (size_t)b * T + (size_t)(e0 + q) * r;
      float m[8], l[8], acc[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) { m[k] = -INFINITY; l[k] = 0.f; acc[k] = 0.f; }
      for (int j0 = act ? ph : r; j0 < r; j0 += 4 * split) {
        uint4 zv[4], cv[4];
        float4 b0[4], b1[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int j = min(j0 + u * split, r - 1);   // out-of-range slots re-read slot r-1, weight 0 below
          zv[u] = __ldg(reinterpret_cast<const uint4*>(Z + (tok0 + j) * d + ch));
          cv[u] = __ldg(reinterpret_cast<const uint4*>(C + (tok0 + j) * d + ch));
          b0[u] = __ldg(reinterpret_cast<const float4*>(b_pos + (size_t)j * d + ch));
          b1[u] = __ldg(reinterpret_cast<const float4*>(b_pos + (size_t)j * d + ch + 4));
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          float a[4], c[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const uint32_t zw = k < 2 ? zv[u].x : k < 4 ? zv[u].y : k < 6 ? zv[u].z : zv[u].w;
            const uint32_t cw = k < 2 ? cv[u].x : k < 4 ? cv[u].y : k < 6 ? cv[u].z : cv[u].w;
            const float4& bb = k < 4 ? b0[u] : b1[u];
            const float bk = (k & 3) == 0 ? bb.x : (k & 3) == 1 ? bb.y : (k & 3) == 2 ? bb.z : bb.w;
            const float zf = __uint_as_float((k & 1) ? (zw & 0xFFFF0000u) : (zw << 16));
            a[u] = j0 + u * split < r ? zf + bk : -INFINITY;
            c[u] = __uint_as_float((k & 1) ? (cw & 0xFFFF0000u) : (cw << 16));
          }
          const float mn = fmaxf(m[k], fmaxf(fmaxf(a[0], a[1]), fmaxf(a[2], a[3])));
          const float sc = m[k] == mn ? 1.f : __expf(m[k] - mn);
          float ls = l[k] * sc, as = acc[k] * sc;
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const float p = __expf(a[u] - mn);
            ls += p;
            as = fmaf(p, c[u], as);
          }
          m[k] = mn; l[k] = ls; acc[k] = as;
        }
      }
      for (int off = 1; off < split; off <<= 1)
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const float mo = __shfl_xor_sync(0xffffffffu, m[k], off);
          const float lo = __shfl_xor_sync(0xffffffffu, l[k], off);
          const float ao = __shfl_xor_sync(0xffffffffu, acc[k], off);
          const float mn = fmaxf(m[k], mo);
          const float s1 = m[k] == mn ? 1.f : __expf(m[k] - mn);
          const float s2 = mo == mn ? 1.f : __expf(mo - mn);
          l[k] = fmaf(l[k], s1, lo * s2);
          acc[k] = fmaf(acc[k], s1, ao * s2);
          m[k] = mn;
        }
      if (act && ph == 0) {
        float* dst = pooled + q * d + ch;
        *reinterpret_cast<float4*>(dst) = make_float4(acc[0] / l[0], acc[1] / l[1], acc[2] / l[2], acc[3] / l[3]);
        *reinterpret_cast<float4*>(dst + 4) = make_float4(acc[4] / l[4], acc[5] / l[5], acc[6] / l[6], acc[7] / l[7]);
      }
    }
  }
  if (long_groups) load_w();
  __syncthreads();
  if (rope_thread) {
    const int q = tid / half, mm = tid % half;
    float* row = pooled + q * d;
    const float x1 = row[d_n + mm], x2 = row[d_n + half + mm];
    row[d_n + mm] = fmaf(x1, rs_cs, -x2 * rs_sn);
    row[d_n + half + mm] = fmaf(x1, rs_sn, x2 * rs_cs);
  }
  __syncthreads();
  for (int i = tid; i < ne * d; i += POOL_THREADS) {
    const int q = i / d, ch = i % d;
    const uint32_t bits = f_to_bf16_bits(pooled[i]);
    if (P.c_out && z == 0) P.c_out[((size_t)b * n_out + e0 + q) * d + ch] = (uint16_t)bits;
    pooled[i] = bf16_bits_to_f(bits);
  }
  __syncthreads();
  if (P.kv.codes && z == 0)
    for (int q = 0; q < ne; ++q) pack_row_to_cache(pooled + q * d, d, d_r, P.kv, b, e0 + q);
  if (P.W_IK == nullptr) return;
  // k_I slice: thread (oc, chp) sums outputs o_base..o_base+7 over channels chp, chp + NCHP, ...
  float* red = pooled + ENT * d;               // [POOL_WARPS][ENT][OW]
  float* krow = red + POOL_WARPS * ENT * OW;   // [ENT][OW]
  float acc[ENT][8];
#pragma unroll
  for (int q = 0; q < ENT; ++q)
#pragma unroll
    for (int k = 0; k < 8; ++k) acc[q][k] = 0.f;
  if (PRE > 0) {
#pragma unroll
    for (int i = 0; i < PRE; ++i) {
      const int ch = chp + NCHP * i;
      if (ch < d)
#pragma unroll
        for (int q = 0; q < ENT; ++q)
          if (q < ne) fma8_bf16(acc[q], pooled[q * d + ch], wpre[i]);
    }
  } else {
#pragma unroll 4
    for (int ch = chp; ch < d; ch += NCHP) {
      const uint4 w = __ldg(reinterpret_cast<const uint4*>(P.W_IK + (size_t)ch * d_I + o_base));
#pragma unroll
      for (int q = 0; q < ENT; ++q)
        if (q < ne) fma8_bf16(acc[q], pooled[q * d + ch], w);
    }
  }
  // reduce over the channel phases: lanes NOC apart inside the warp, then the warps through smem
#pragma unroll
  for (int off = NOC; off < 32; off <<= 1)
#pragma unroll
    for (int q = 0; q < ENT; ++q)
#pragma unroll
      for (int k = 0; k < 8; ++k) acc[q][k] += __shfl_xor_sync(0xffffffffu, acc[q][k], off);
  if (lane < NOC)
#pragma unroll
    for (int q = 0; q < ENT; ++q)
#pragma unroll
      for (int k = 0; k < 8; ++k) red[(warp * ENT + q) * OW + oc * 8 + k] = acc[q][k];
  __syncthreads();
  for (int i = tid; i < ne * OW; i += POOL_THREADS) {
    const int q = i / OW, o = i % OW;
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < POOL_WARPS; ++w) v += red[(w * ENT + q) * OW + o];
    const uint32_t bits = f_to_bf16_bits(v);
    if (P.kI_out) P.kI_out[((size_t)b * n_out + e0 + q) * d_I + z * OW + o] = (uint16_t)bits;
    krow[q * OW + o] = bf16_bits_to_f(bits);
  }
  if (P.ki.codes) {
    __syncthreads();
    const csa_fp4_cache& cc = P.ki;
    const int S = d_I / 32, S_pad = (S + 3) & ~3;
    for (int t = warp; t < ne * (OW / 32); t += POOL_WARPS) {
      const int q = t / (OW / 32), blk = z * (OW / 32) + t % (OW / 32);
      const long long dst = page_row(cc.pages, b, cc.n_max, (long long)(cc.row0 ? cc.row0[b] : 0) + e0 + q);
      if (dst < 0) continue;
      pack_block_warp(krow[q * OW + (t % (OW / 32)) * 32 + lane], cc.global_scale, cc.codes + dst * (d_I / 2) + blk * 16,
                      cc.scales + dst * S_pad + blk);
      if (z == 0 && lane < S_pad - S) cc.scales[dst * S_pad + S + lane] = 0;
    }
  }
}

}  // namespace csa

using namespace csa;

extern "C" csa_status csa_compress(const csa_compress_args* a, void* stream) {
  CSA_REQUIRE(a != nullptr && a->struct_size == sizeof(csa_compress_args));
  CSA_REQUIRE(a->B >= 0 && a->T >= 0 && a->d > 0 && a->ratio >= 1 && a->d_rope >= 0 && a->d_rope <= a->d);
  CSA_REQUIRE(a->d_rope % 2 == 0 && a->d_index >= 0);
  CSA_SUPPORTED(a->d % 8 == 0);
  CSA_REQUIRE(a->C && a->Z && a->b_pos && (a->c_out || a->kv_pack.codes));
  CSA_REQUIRE(a->W_IK == nullptr || (a->kI_out && a->d_index > 0));
  cudaStream_t st = (cudaStream_t)stream;
  if (a->x) {
    CSA_REQUIRE(a->W_kv && a->W_g && a->d_model > 0);
    CSA_SUPPORTED(a->d % 128 == 0 && a->d_model % 8 == 0);
    CSA_SUPPORTED((((uintptr_t)a->x | (uintptr_t)a->W_kv | (uintptr_t)a->W_g | (uintptr_t)a->C | (uintptr_t)a->Z) &
                   15) == 0);
    const long long M = (long long)a->B * a->T;
    if (M > 0) {
      csa_status s = run_projection_tc(a->x, a->W_kv, a->W_g, a->C, a->Z, M, a->d, a->d_model, st);
      if (s != CSA_OK) return s;
    }
  }
  const int n_out = a->T / a->ratio;
  if (a->B == 0 || n_out == 0) return CSA_OK;
  if (a->W_IK) CSA_SUPPORTED(a->d_index == 64 || a->d_index == 128);
  if (a->kv_pack.codes) {
    CSA_REQUIRE(a->kv_pack.scales && (a->d_rope == 0 || a->kv_pack.rope) && a->kv_pack.global_scale > 0.0f);
    CSA_SUPPORTED((a->d - a->d_rope) % 32 == 0);
  }
  if (a->ki_pack.codes) CSA_REQUIRE(a->W_IK && a->ki_pack.scales && a->ki_pack.global_scale > 0.0f);
  for (const csa_fp4_cache* cc : {&a->kv_pack, &a->ki_pack})
    if (cc->codes) {
      const csa_status pv = check_page_map(cc->pages, cc->n_max);
      if (pv != CSA_OK) return pv;
    }
  if (a->W_IK) CSA_SUPPORTED(((uintptr_t)a->W_IK & 15) == 0);
  // groups longer than 8 slots are read 8 channels (16 bytes) at a time
  if (a->ratio > 8) CSA_SUPPORTED((((uintptr_t)a->C | (uintptr_t)a->Z | (uintptr_t)a->b_pos) & 15) == 0);
  if (a->W_IK) CSA_SUPPORTED((a->d_index * 2) % 16 == 0);
  CSA_SUPPORTED(POOL_ENT * (a->d_rope / 2) <= POOL_THREADS && a->d_rope / 2 <= POOL_MAX_HALF);
  // k_I output slices: enough CTAs for about one wave when there are few entry groups
  // one entry per CTA when each sequence completes a single group (decode), else POOL_ENT
  const int ent = n_out == 1 ? 1 : POOL_ENT;
  const long long groups = (long long)a->B * ((n_out + ent - 1) / ent);
  int OW = a->W_IK ? a->d_index : 32;
  while (a->W_IK && OW > 32 && groups * (a->d_index / OW) * 2 <= 148) OW >>= 1;
  const int nchp = POOL_THREADS / (OW / 8);
  const bool pre = a->W_IK && a->d <= 8 * nchp;
  const bool r4 = ent == 1 && a->ratio == 4;
  const size_t smem = (size_t)ent * a->d * sizeof(float) + (size_t)(POOL_WARPS + 1) * ent * OW * 4;
  CSA_SUPPORTED(smem <= 200 * 1024);
  PoolParams P{};
  P.C = (const uint16_t*)a->C; P.Z = (const uint16_t*)a->Z; P.b_pos = a->b_pos; P.T = a->T; P.d = a->d;
  P.d_r = a->d_rope; P.r = a->ratio; P.theta = a->rope_theta; P.pos0 = a->pos0; P.W_IK = (const uint16_t*)a->W_IK;
  P.d_I = a->d_index; P.c_out = (uint16_t*)a->c_out; P.kI_out = (uint16_t*)a->kI_out; P.kv = a->kv_pack;
  P.ki = a->ki_pack;
  for (int m = 0; m < a->d_rope / 2; ++m)
    P.inv_freq[m] = a->rope_theta != 0.0f ? pow((double)a->rope_theta, -2.0 * m / (double)a->d_rope) : 0.0;
  dim3 grid((n_out + ent - 1) / ent, a->B, a->W_IK ? a->d_index / OW : 1);
  // kernel variants: [OW 32/64/128][W_IK slice preloaded][one entry, ratio 4 | one entry | POOL_ENT entries]
  static const void* const table[3][2][3] = {
      {{(const void*)pool_kernel<32, 0, 1, 4>, (const void*)pool_kernel<32, 0, 1, 0>, (const void*)pool_kernel<32, 0, POOL_ENT, 0>},
       {(const void*)pool_kernel<32, 8, 1, 4>, (const void*)pool_kernel<32, 8, 1, 0>, (const void*)pool_kernel<32, 8, POOL_ENT, 0>}},
      {{(const void*)pool_kernel<64, 0, 1, 4>, (const void*)pool_kernel<64, 0, 1, 0>, (const void*)pool_kernel<64, 0, POOL_ENT, 0>},
       {(const void*)pool_kernel<64, 8, 1, 4>, (const void*)pool_kernel<64, 8, 1, 0>, (const void*)pool_kernel<64, 8, POOL_ENT, 0>}},
      {{(const void*)pool_kernel<128, 0, 1, 4>, (const void*)pool_kernel<128, 0, 1, 0>, (const void*)pool_kernel<128, 0, POOL_ENT, 0>},
       {(const void*)pool_kernel<128, 8, 1, 4>, (const void*)pool_kernel<128, 8, 1, 0>, (const void*)pool_kernel<128, 8, POOL_ENT, 0>}}};
  const int iow = OW == 32 ? 0 : OW == 64 ? 1 : 2, ivar = ent == 1 ? (r4 ? 0 : 1) : 2;
  const void* fn = table[iow][pre ? 1 : 0][ivar];
  static std::atomic<unsigned> attr_done[3][2][3];
  set_smem_once(fn, 200 * 1024, attr_done[iow][pre ? 1 : 0][ivar]);
  void* argv[] = {&P};
  cudaLaunchAttribute attr[1];
  const cudaLaunchConfig_t cfg = pdl_config(grid, dim3(POOL_THREADS), smem, st, attr);
  cudaError_t e = cudaLaunchKernelExC(&cfg, fn, argv);
  if (e != cudaSuccess) { set_last_cuda_error(e); return CSA_ERR_CUDA; }
  return launch_status();
}
