/*
 * csa.h — C ABI of the B200 (sm_100a) Compressed Sparse Attention layer over an FP4 KV cache.
 *
 * The layer (sources, by page title):
 *   [V4 blog]    "DeepSeek-V4: エージェントが実際に使える100万トークンのコンテキスト", §ハイブリッド注意：CSAとHCA,
 *                Fig. 3 (CSA: 4x softmax-gated compressor, FP4 ReLU "lightning" indexer, top-k, sliding window),
 *                Fig. 4 (HCA: 128x compressor, dense attention), storage paragraph (BF16 RoPE dims, FP4 indexer).
 *   [V4.1 notes] "DeepSeek-V4.1-Flash - Pushing the Limits of KV Cache Compression", §提案手法/アーキテクチャ:
 *                CED bullet eq.(1) (C, Z projections), CSA2 bullet + Fig. 4 (Full / Reindex / Reuse),
 *                Hierarchical Sparse Indexer bullet + Fig. 5, FP4 主 KV キャッシュ bullet.
 *
 * Conventions for every entry point:
 *   - Every pointer is caller-owned DEVICE memory (unless stated otherwise); the library allocates
 *     nothing.  Scratch comes from a caller workspace whose size the matching *_workspace_size() call
 *     returns for the same arguments (0 means none is needed; ws may then be NULL).  The size (and
 *     kernel-count) queries read the shapes, flags, page maps and the alignment of the input buffers
 *     given; output buffers may still be NULL then.
 *   - bf16 = IEEE bfloat16 stored as uint16; tensors are dense row-major with the shapes given.
 *   - Calls are asynchronous on `stream` (a cudaStream_t passed as void*; NULL = legacy default
 *     stream).  Argument errors are detected on the host before any launch and returned as
 *     CSA_ERR_INVALID / CSA_ERR_UNSUPPORTED / CSA_ERR_WORKSPACE; nothing is launched then.
 *     A launch failure returns CSA_ERR_CUDA.  No exception crosses the ABI.
 *   - Global mutable state: two device-side items only.  (1) The device error word that bounded waits
 *     set when they give up (one per device, read and cleared by csa_device_status).  (2) The static
 *     scratch array of csa_index_topk_noalloc (CSA_NOALLOC_SCRATCH_BYTES per device).  Host-side
 *     caches (tensor-map encoder, kernel attributes set once per device) hold no per-call data.
 *   - Arguments are passed as structs whose first field `struct_size` must equal sizeof(struct).
 *   - FP4 formats (E2M1 codes, one E4M3 scale per 32 elements, per-tensor fp32 global scale g):
 *       codes[n][d_n/2] u8 (element 2j in the low nibble of byte j), scales[n][S_pad] u8
 *       (S = d_n/32, S_pad = round_up(S, 4), pad bytes 0), rope[n][d_r] bf16.
 *       Dequantised element = e2m1(code) * e4m3(scale) * g.
 */
#ifndef CSA_H_
#define CSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum csa_status {
  CSA_OK = 0,
  CSA_ERR_INVALID = 1,      /* a NULL pointer, a bad size or a struct_size mismatch                    */
  CSA_ERR_UNSUPPORTED = 2,  /* a valid shape the library has no kernel for (e.g. d_I not 64/128)       */
  CSA_ERR_WORKSPACE = 3,    /* ws_bytes smaller than *_workspace_size() for the same arguments          */
  CSA_ERR_CUDA = 4,         /* a kernel launch or CUDA runtime call failed (see csa_last_cuda_error)   */
  CSA_ERR_DEVICE = 5        /* a device-side bounded wait gave up (csa_device_status)                  */
} csa_status;

/* Human-readable name of a status code (static string). */
const char* csa_status_string(int status);
/* Library version as 10000*major + 100*minor + patch. */
int csa_version(void);
/* The cudaError_t of the last CSA_ERR_CUDA returned on the calling host thread (0 if none). */
int csa_last_cuda_error(void);
/* Synchronises `stream`, then reports and clears the device-side error word of the current device
 * (every kernel of the library writes it):
 * CSA_ERR_DEVICE if a kernel gave up a bounded wait (a pipeline stalled; its outputs are incomplete),
 * CSA_OK otherwise, CSA_ERR_CUDA if the synchronisation itself failed. */
csa_status csa_device_status(void* stream);
/* Exercises the error path above without a fault: launches one thread that waits, `polls` times with
 * a short sleep between polls (1 <= polls <= 2^20, i.e. well under a second), on a barrier nothing
 * arrives on, then records device error 1 exactly as a stalled pipeline does.  The next
 * csa_device_status returns CSA_ERR_DEVICE (and clears the word).  No output; nothing else changes.
 * A library self-check, not part of the layer: the pages have no counterpart. */
csa_status csa_check_error_path(uint32_t polls, void* stream);

/* Overlap inside a decode step.  Every kernel of this library is launched with programmatic
 * dependent launch: it may become resident while the kernel before it on the stream still runs, and it
 * waits for that kernel to complete (and its writes to become visible) before it reads anything the
 * kernel could have written.  csa_compress's last kernel lets its dependents start only after all
 * work earlier on the stream has completed.
 * CSA_EARLY_START in `flags` (csa_index_args, csa_attn_args) lets a call do part of its work before
 * the kernels ahead of it in the step have completed:
 *   - csa_index_scores / csa_index_topk (Full mode, single query per row): scoring reads q_I, w, n_c,
 *     q_pos and the key rows [0, n_c[b] - 1) at once and writes scores and hist; only the 256-row
 *     tile that holds row n_c[b] - 1 waits.  Requires: the kernel just before the call is csa_compress,
 *     and that call writes none of these inputs except key rows >= n_c[b] - 1.
 *   - csa_topk / the selection of csa_index_topk (single-CTA histogram rows): reads n_c and q_pos before
 *     the scores are final, so the row's copy starts the moment they are.  Requires: the call follows
 *     csa_index_scores (csa_index_topk: its own scoring) of the same step, which follows csa_compress,
 *     and none of these calls writes n_c or q_pos.
 *   - csa_sparse_attn (k % 128 == 0, window <= 128): the window tile of every query runs in a CTA of
 *     its own that reads q, q_pos, n_c, win_kv, win_pos0 and writes its workspace partial at once; the
 *     CTAs over the selected entries wait as usual.  Requires: the step's earlier calls since
 *     csa_compress (csa_index_scores, csa_topk) write none of those inputs, and csa_compress is
 *     among them.
 * Paths that cannot use the flag ignore it.  Results are the same with and without it. */
#define CSA_EARLY_START 1u
/* CSA_CLUSTER_MERGE in csa_attn_args.flags: a query whose keys are split over 2..8 CTAs merges the
 * partial softmax results inside the CTAs' thread-block cluster (distributed shared memory; no workspace
 * partials, no merge kernel).  Without it the partials go through the workspace and a merge kernel,
 * which measured faster for the 128K decode step on B200 (the cluster's CTAs must be co-scheduled in one
 * GPC, and the merge adds code to a cold-instruction-cache kernel).  Results agree to rounding. */
#define CSA_CLUSTER_MERGE 2u
/* CSA_ONCHIP_TOPK in csa_index_args.flags (csa_index_topk, single-query Full rows of at most 32768 keys,
 * d_I = 128, no pool): score and select each row inside one thread-block cluster of 8 CTAs, the scores
 * never leaving shared memory.  Without it the scores go to the workspace with their histogram and a
 * top-k kernel selects them, which measured faster for the 128K decode step on B200 (more CTAs stream
 * the keys).  The selected sets are identical. */
#define CSA_ONCHIP_TOPK 4u

/* Paged caches ([V4.1 notes] §実装上の工夫: serving keeps the compressed KV in pages; the pages give no
 * layout, so this library fixes one).  A csa_page_map sends logical entry i of sequence b to row
 *   table[b * width + i / page_size] * page_size + i % page_size
 * of the arrays it accompanies, which are then pools [n_pages * page_size][...] instead of [B][n_max][...].
 * table == NULL means the contiguous layout (row = b * n_max + i).  page_size % 128 == 0, so every
 * 128-entry tile of the tensor-core kernels lies in one page; width * page_size >= n_max.  A page id
 * outside [0, n_pages) is a caller error: the kernels then neither read nor write outside the pool (such
 * a page is skipped), but results that depend on its entries are unspecified. */
typedef struct csa_page_map {
  const int32_t* table;    /* [B][width] device int32, or NULL */
  int32_t page_size;
  int32_t width;
  int32_t n_pages;
} csa_page_map;

/* ------------------------------------------------------------------------------------------------
 * csa_compress — the compressor ([V4 blog] Fig. 3 / Fig. 4; [V4.1 notes] eq.(1) and CSA2 bullet).
 *
 * Projection mode (x != NULL): C = bf16(x·W_kv), Z = bf16(x·W_g) are computed (tensor cores, fp32
 * accumulate) and written to the caller's C and Z buffers (C also serves as the token's window KV).
 * Pooling mode (x == NULL): C and Z are read.  Then, for every sequence b and entry i < T/ratio:
 *   c[b][i][ch] = sum_j softmax_j(Z[b][r i + j][ch] + b_pos[j][ch]) * C[b][r i + j][ch]
 * (one gate per channel, non-overlapping groups), RoPE on the last d_rope channels at position
 * pos0[b] + r i (half-split pairs, angle p * theta^(-2m/d_rope); rope_theta == 0 disables it),
 * rounded to bf16 into c_out; then k_I = bf16(c · W_IK) into kI_out when W_IK != NULL.
 * Trailing T % ratio tokens are ignored (the caller keeps them pending).
 * Fused append (decode): with kv_pack.codes / ki_pack.codes set, the same launch also packs c and k_I
 * into the FP4 caches exactly as csa_pack_fp4 would (then c_out / kI_out may be NULL).
 * Shapes: x[B][T][d_model], W_kv/W_g[d_model][d], C/Z[B][T][d], b_pos[ratio][d] fp32,
 *         W_IK[d][d_index], c_out[B][T/ratio][d], kI_out[B][T/ratio][d_index], pos0[B] int64 (NULL = 0).
 * Limits: d % 8 == 0, d_rope even and <= d, ratio >= 1; projection mode needs d % 128 == 0 and
 *         d_model % 32 == 0; ratio > 8 needs C, Z and b_pos 16-byte aligned (else CSA_ERR_UNSUPPORTED).
 *         No workspace.
 * ------------------------------------------------------------------------------------------------ */
/* An FP4 cache to append packed rows to (the layout csa_pack_fp4 writes): row i of sequence b goes to
 * cache row row0[b] + i.  codes == NULL means "no cache". */
typedef struct csa_fp4_cache {
  uint8_t* codes;          /* [B][n_max][d_n/2] */
  uint8_t* scales;         /* [B][n_max][S_pad] */
  void* rope;              /* [B][n_max][d_rope] bf16 (NULL when d_rope == 0) */
  const int32_t* row0;     /* [B] (NULL = 0) */
  int32_t n_max;
  float global_scale;
  csa_page_map pages;      /* paged pool (table == NULL: contiguous [B][n_max]) */
} csa_fp4_cache;

typedef struct csa_compress_args {
  uint32_t struct_size;
  int32_t B, T, d_model, d, d_rope, d_index, ratio;
  float rope_theta;
  const int64_t* pos0;
  const void* x;
  const void* W_kv;
  const void* W_g;
  void* C;
  void* Z;
  const float* b_pos;
  const void* W_IK;
  void* c_out;
  void* kI_out;
  csa_fp4_cache kv_pack;   /* optional: also FP4-pack each entry c into this cache (same bytes as csa_pack_fp4) */
  csa_fp4_cache ki_pack;   /* optional: also FP4-pack each indexer key k_I (d_rope = 0) into this cache */
} csa_compress_args;

csa_status csa_compress(const csa_compress_args* args, void* stream);

/* ------------------------------------------------------------------------------------------------
 * csa_pack_fp4 — FP4 pack of compressed entries into a cache ([V4.1 notes] FP4 主 KV キャッシュ bullet;
 * [V4 blog] storage paragraph: the RoPE slice stays BF16).
 *
 * For rows src[b][j] (j < n), written to cache row row0[b] + j of sequence b:
 *   per 32-block of the first d - d_rope channels: s = E4M3_rne_satfinite(fp32(amax / fp32(6 g)));
 *   s == 0 zeroes the block; else code_e = E2M1_rne_satfinite(fp32(x_e / fp32(s g))), -0 -> +0;
 *   the last d_rope channels are copied to rope.
 * Shapes: src[B][n][d] bf16; codes[B][n_max][(d-d_rope)/2]; scales[B][n_max][S_pad];
 *         rope[B][n_max][d_rope] bf16 (may be NULL iff d_rope == 0); row0[B] int32 (NULL = 0).
 * Limits: (d - d_rope) % 32 == 0, d_rope % 8 == 0, row0[b] + n <= n_max (not checked on the device:
 *         the caller owns the cache bookkeeping).  No workspace.
 * ------------------------------------------------------------------------------------------------ */
typedef struct csa_pack_args {
  uint32_t struct_size;
  int32_t B, n, d, d_rope, n_max;
  float global_scale;
  const void* src;
  const int32_t* row0;
  uint8_t* codes;
  uint8_t* scales;
  void* rope;
  csa_page_map pages;      /* paged pool (table == NULL: contiguous [B][n_max]) */
} csa_pack_args;

csa_status csa_pack_fp4(const csa_pack_args* args, void* stream);

/* ------------------------------------------------------------------------------------------------
 * csa_pack_fp8_window — FP8 pack of sliding-window KV rows ([V4.1 notes] FP4 主 KV キャッシュ bullet: the
 * window's uncompressed KV stays FP8; [V4 blog] storage paragraph: the RoPE channels stay BF16).
 *
 * The pages fix FP8 (E4M3) but not its scaling; this library uses one fp32 scale per 64 channels:
 * for rows src[b][j] (j < n), written to window row row0[b] + j of sequence b, per 64-block of the first
 * d - d_rope channels: scale = fp32(amax / 448) (correctly rounded fp32 division); scale == 0 zeroes the
 * block; else code_e = E4M3_rne_satfinite(fp32(x_e / scale)), -0 -> +0.  The last d_rope channels are
 * copied.  Dequantised element = e4m3(code) * scale.
 * Shapes: src[B][n][d] bf16; codes[B][Wn][d-d_rope] u8; scales[B][Wn][SW] fp32 with
 *         SW = round_up((d-d_rope)/64, 4) (pad entries 0); rope[B][Wn][d_rope] bf16; row0[B] int32 (NULL = 0).
 * Limits: (d - d_rope) % 64 == 0, d_rope % 8 == 0, row0[b] + n <= Wn (not checked on the device).
 *         No workspace.
 * ------------------------------------------------------------------------------------------------ */
typedef struct csa_fp8_window_args {
  uint32_t struct_size;
  int32_t B, n, d, d_rope, Wn;
  const void* src;
  const int32_t* row0;
  uint8_t* codes;
  float* scales;
  void* rope;
} csa_fp8_window_args;

csa_status csa_pack_fp8_window(const csa_fp8_window_args* args, void* stream);

/* ------------------------------------------------------------------------------------------------
 * csa_index_topk — lightning indexer scores + per-query top-k ([V4 blog] §ハイブリッド注意, Fig. 3;
 * Reindex mode and the hierarchical candidate pool: [V4.1 notes] CSA2 bullet Fig. 4, Fig. 5).
 *
 * q_I is quantised with the FP4 pack rule (global scale g_q).  For query (b, q) at t = q_pos[b][q]
 * and a visible key i (i < n_c[b], ratio*i + ratio - 1 <= t):
 *   s = g_q g_k sum_h w[b][q][h] * max(0, sum_blk sq[h][blk] sk[i][blk] P[h][i][blk]),
 *   P = E2M1 block dot product.  -0 is taken as +0.
 * Candidates: all visible keys (cand == NULL; Full mode) or cand[b][q][0..n_cand) (Reindex mode;
 * -1 entries and invisible ids are dropped).  Selected: the k_eff = min(k, #candidates) keys by
 * (score desc, key id asc), written to idx_out[b][q][0..k) in unspecified order, remaining slots -1;
 * scores_out (optional) gets the matching scores (-inf in padded slots).
 * Hierarchical pool (pool_blocks > 0, cand == NULL only): block score = max over the visible keys
 * of [G j, G j + G) (G = pool_block_size); the top pool_blocks blocks by (block score desc, block id
 * asc) are written to pool_out[b][q][0 .. pool_blocks*G) as G consecutive key ids per block (block
 * order unspecified; -1 for invisible keys and missing blocks).
 * Shapes: q_I[B][Nq][H_I][d_I] bf16, w[B][Nq][H_I] fp32, k_codes[B][n_max][d_I/2],
 *         k_scales[B][n_max][S_pad(d_I/32)], n_c[B] int32, q_pos[B][Nq] int64.
 * Limits: d_I in {64, 128}; H_I <= 8; 1 <= k <= 4096; with cand: n_cand <= 16384.
 * Workspace: csa_index_topk_workspace_size().
 * ------------------------------------------------------------------------------------------------ */
typedef struct csa_index_args {
  uint32_t struct_size;
  int32_t B, Nq, H_I, d_I, ratio, k, n_max;
  float g_q, g_k;
  const void* q_I;
  const float* w;
  const uint8_t* k_codes;
  const uint8_t* k_scales;
  const int32_t* n_c;
  const int64_t* q_pos;
  const int32_t* cand;
  int32_t n_cand;
  int32_t pool_blocks;
  int32_t pool_block_size;
  int32_t* pool_out;
  int32_t* idx_out;
  float* scores_out;
  uint32_t* hist;          /* optional, split calls only: [B*Nq][4096] score histogram that csa_index_scores
                              adds into (single-query rows: Nq == 1 or cand != NULL) and csa_topk uses to
                              find the k-th score's neighbourhood in one pass, leaving every row it read
                              zero again.  It must be zero before the first csa_index_scores call and
                              then hold the counts that call added.  Other counts cost time, not
                              correctness, while the histogram still counts at least k scores of a row
                              (csa_topk checks the counts at and above the k-th score's bin against the
                              scores and falls back to the full selection); a row whose histogram counts
                              fewer than k scores (e.g. one no scoring call filled) is taken to hold only
                              that many.  NULL = plain radix selection */
  uint32_t flags;          /* CSA_EARLY_START | CSA_ONCHIP_TOPK, or 0 */
  csa_page_map k_pages;    /* k_codes / k_scales as a paged pool (table == NULL: contiguous) */
} csa_index_args;

size_t csa_index_topk_workspace_size(const csa_index_args* args);
csa_status csa_index_topk(const csa_index_args* args, void* ws, size_t ws_bytes, void* stream);

/* csa_index_scores — the scoring half of csa_index_topk on its own ([V4 blog] §ハイブリッド注意: the
 * lightning indexer).  Writes scores[(b*Nq + q)*ld + j] fp32 for j < n_vis(t) = min(n_c[b],
 * floor((t+1)/ratio)) in Full mode, or for every j < n_cand in Reindex mode (-inf for dropped
 * candidates); other columns are left untouched.  ld >= n_max (Full) or >= n_cand (Reindex).
 * idx_out / scores_out / pool_out are ignored.  No workspace. */
csa_status csa_index_scores(const csa_index_args* args, float* scores, int64_t ld, void* stream);

/* csa_topk — the selection half of csa_index_topk ([V4 blog] Fig. 3: top-k per query; [V4.1 notes]
 * Fig. 5: hierarchical pool) over a score matrix laid out as csa_index_scores writes it, with the
 * same args (q_I, w, k_codes, k_scales may be NULL).  In Reindex mode ld must equal n_cand.
 * Workspace: csa_topk_workspace_size() (tournament buffers for rows longer than 32768, pool block scores
 * and their histograms, row histograms for multi-query rows longer than 8192 keys). */
size_t csa_topk_workspace_size(const csa_index_args* args);
csa_status csa_topk(const csa_index_args* args, const float* scores, int64_t ld, void* ws, size_t ws_bytes,
                    void* stream);

/* csa_index_topk_noalloc — csa_index_topk for callers that cannot allocate device memory: code that
 * runs where cudaMalloc is unavailable or forbidden (inside an allocator-free runtime or plugin
 * host, an embedded service with a fixed memory budget, or a caller that must not synchronise the
 * device the way cudaMalloc/cudaFree can).  The paper has no counterpart; this is a deployment
 * convenience of this library.  Same arguments, same results as csa_index_topk, no ws argument.
 * Its scratch is a static device array of CSA_NOALLOC_SCRATCH_BYTES that every GPU loading the
 * library holds until the process exits.  Problems needing more scratch than that (see
 * csa_index_topk_workspace_size) return CSA_ERR_WORKSPACE before any CUDA call.
 * The first call on each device looks up the array's device address (cudaGetSymbolAddress) with
 * that device current; make that first call before any stream capture.  All calls share the one
 * array: calls that overlap on the GPU (other streams, other host threads) race and must be
 * serialised by the caller.  It calls no cudaMalloc / cudaFree. */
#define CSA_NOALLOC_SCRATCH_BYTES (8u << 20)
csa_status csa_index_topk_noalloc(const csa_index_args* args, void* stream);

/* ------------------------------------------------------------------------------------------------
 * csa_sparse_attn / hca_dense_attn — softmax attention over compressed entries plus the sliding
 * window ([V4 blog] Fig. 3 for CSA: the selected entries; Fig. 4 for HCA: every visible entry).
 *
 * For query (b, q) at t = q_pos[b][q] with heads q[b][q][h][0..d):
 *   keys = values = the dequantised cache entries [e2m1*scale*g_kv over d - d_rope channels ‖ rope]
 *          for idx[b][q][j] in [0, n_c[b]) (csa_sparse_attn; other ids are skipped) or for every
 *          i < n_c[b] with ratio*i + ratio - 1 <= t (hca_dense_attn; idx ignored),
 *        ∪ window rows for tokens p in [max(0, t - window + 1), t] held by win_kv[b] at positions
 *          win_pos0[b] .. win_pos0[b] + Wn - 1 (absent positions are skipped).
 *   One joint softmax with logits softmax_scale * (q_h · K_j) (softmax_scale == 0 -> 1/sqrt(d)).
 *   out = bf16(sum_j p_j V_j); lse = ln sum_j exp(logit_j) (fp32; -inf and out = 0 for no keys).
 * Shapes: q/out[B][Nq][H][d] bf16, q_pos[B][Nq] int64, kv_codes[B][n_max][(d-d_rope)/2],
 *         kv_scales[B][n_max][S_pad], kv_rope[B][n_max][d_rope] bf16, n_c[B] int32,
 *         idx[B][Nq][k] int32, win_kv[B][Wn][d] bf16 (may be NULL with Wn = 0), win_pos0[B] int64,
 *         lse[B][Nq][H] fp32 (may be NULL).
 * Limits: d in {128, 512} with d_rope == 64 (d = 512) or 32 (d = 128); H <= 64.
 * Workspace: csa_attn_workspace_size() (split-K partials); `hca` selects the HCA key set.
 * csa_attn_kernel_count: how many kernels one call with these arguments launches (-1 if the arguments
 *   are invalid, 0 for an empty batch); no GPU work.
 * ------------------------------------------------------------------------------------------------ */
typedef struct csa_attn_args {
  uint32_t struct_size;
  int32_t B, Nq, H, d, d_rope, ratio, n_max, k, Wn, window;
  float g_kv, softmax_scale;
  const void* q;
  const int64_t* q_pos;
  const uint8_t* kv_codes;
  const uint8_t* kv_scales;
  const void* kv_rope;
  const int32_t* n_c;
  const int32_t* idx;
  const void* win_kv;
  const int64_t* win_pos0;
  void* out;
  float* lse;
  uint32_t flags;          /* CSA_EARLY_START | CSA_CLUSTER_MERGE, or 0 */
  /* Inverse-RoPE epilogue ([V4.1 notes] §実装上の工夫, inference kernels: the fused
     "RoPE-attention-RoPE-cast" kernel): nonzero rotates the last d_rope channels of out by the
     inverse of the query's RoPE, angle -t * out_rope_theta^(-2m/d_rope) for the half-split pair
     (m, m + d_rope/2), before the bf16 cast; the values' RoPE channels, rotated at their own positions,
     then come out relative to the query.  lse is unchanged.  0 = off. */
  float out_rope_theta;
  /* Window format ([V4.1 notes] FP4 主 KV キャッシュ bullet: the window KV stays FP8).  CSA_WIN_BF16: the
     window rows are win_kv (above).  CSA_WIN_FP8: they are the FP8 rows csa_pack_fp8_window writes,
     win_codes[B][Wn][d-d_rope], win_scales[B][Wn][SW] fp32, win_rope[B][Wn][d_rope] bf16 (win_kv is then
     ignored), dequantised as bf16(e4m3 * scale) before the tensor cores.  FP8 needs d = 512 (the
     tensor-core path) and 16-byte aligned buffers (else CSA_ERR_UNSUPPORTED). */
  uint32_t win_format;
  const uint8_t* win_codes;
  const float* win_scales;
  const void* win_rope;
  csa_page_map kv_pages;   /* kv_codes / kv_scales / kv_rope as a paged pool (table == NULL: contiguous) */
} csa_attn_args;

#define CSA_WIN_BF16 0u
#define CSA_WIN_FP8 1u

size_t csa_attn_workspace_size(const csa_attn_args* args, int hca);
int csa_attn_kernel_count(const csa_attn_args* args, int hca);
csa_status csa_sparse_attn(const csa_attn_args* args, void* ws, size_t ws_bytes, void* stream);
csa_status hca_dense_attn(const csa_attn_args* args, void* ws, size_t ws_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* CSA_H_ */
