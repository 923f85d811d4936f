"""CPU oracle for the Compressed Sparse Attention (CSA) layer over an FP4 KV cache.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline /
reference leg of ``bench.py`` may import or call this module.  The product path (the CUDA library
and its Python binding) never imports it and shares no code with it.

Plain, slow, obviously correct: numpy in float64 for every real-valued step, float32 only where the
format definition fixes an fp32 operation (the FP4 pack's scale and element divisions), no blocking,
fusion or reordering beyond what the definitions state.

Sources (page titles; section / figure / equation):
  [V4 blog]   "DeepSeek-V4: エージェントが実際に使える100万トークンのコンテキスト" — §ハイブリッド注意：CSAとHCA,
              Fig. 3 (CSA: compressor, lightning indexer, top-k, sliding window), Fig. 4 (HCA), and the
              storage paragraph after the layer-interleave paragraph (FP8 KV + BF16 RoPE dims, FP4 indexer).
  [V4.1 notes] "DeepSeek-V4.1-Flash - Pushing the Limits of KV Cache Compression" — §提案手法/アーキテクチャ:
              CED bullet eq.(1) (C, Z projections), CSA2 bullet + Fig. 4 (Full/Reindex/Reuse),
              Hierarchical Sparse Indexer bullet + Fig. 5, FP4 主 KV キャッシュ bullet.
Where the pages leave a step open, the reading taken is stated at the function that takes it; the
section tags S1-S8 below name the parts of the layer (compressor, pack, indexer, top-k, attention,
window, hierarchical pool, reuse).

Pinned by tests/test_oracle_*.py against closed forms, invariants, library routines (torch's FP8
cast, torch SDPA) and brute force on tiny inputs.  Parity of the end-to-end layer against the pages
themselves is unpinned: the pages print no worked example or output for CSA.
"""
from __future__ import annotations

import math

import numpy as np

# --------------------------------------------------------------------------------------------
# Binary floating-point formats (definitions: IEEE-754 style sign/exponent/mantissa; OCP FP8 E4M3
# and OCP MX E2M1 element encodings).  All values are carried as float64.
# --------------------------------------------------------------------------------------------

E2M1_MAGNITUDES = (0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)  # code 0..7; bit 3 = sign
E4M3_MAX = 448.0


def round_to_format(x, sig_bits: int, emin: int, max_finite: float | None, saturate: bool):
    """Round float64 ``x`` to the nearest value of a binary format with ``sig_bits`` significant bits
    (hidden bit included) and minimum normal exponent ``emin``; ties to even.  Subnormals keep the
    quantum 2^(emin - sig_bits + 1).  Values beyond ``max_finite`` saturate (``saturate``) or
    become inf."""
    x = np.asarray(x, dtype=np.float64)
    out = np.zeros_like(x)
    nz = x != 0
    ax = np.abs(x[nz])
    _, e = np.frexp(ax)              # ax = m * 2^e, 0.5 <= m < 1  -> leading bit exponent e-1
    lead = e.astype(np.int64) - 1
    qexp = np.maximum(lead, emin) - (sig_bits - 1)
    quantum = np.ldexp(1.0, qexp)
    r = np.rint(ax / quantum) * quantum   # np.rint: round half to even; exact scaling by 2^k
    if max_finite is not None:
        over = r > max_finite
        r = np.where(over, max_finite if saturate else np.inf, r)
    out[nz] = np.sign(x[nz]) * r
    return out


def bf16_round(x):
    """float64 -> nearest bfloat16 (8 significant bits, fp32 exponent range), RNE."""
    return round_to_format(x, 8, -126, None, False)


def fp32(x):
    return np.asarray(x, dtype=np.float32)


def e4m3_rne_satfinite(x):
    """Nearest E4M3 value (4 significant bits, emin -6, subnormal quantum 2^-9), saturating at 448."""
    return round_to_format(x, 4, -6, E4M3_MAX, True)


def e2m1_rne_satfinite(x):
    """Nearest E2M1 value (2 significant bits, emin 0, subnormal quantum 0.5), saturating at 6."""
    return round_to_format(x, 2, 0, 6.0, True)


def e4m3_encode(v):
    """Bit pattern of an exactly representable non-negative E4M3 value."""
    v = np.asarray(v, dtype=np.float64)
    code = np.zeros(v.shape, dtype=np.uint8)
    nz = v > 0
    _, e = np.frexp(v[nz])
    lead = e.astype(np.int64) - 1
    normal = lead >= -6
    mant_n = np.rint((v[nz] / np.ldexp(1.0, lead) - 1.0) * 8).astype(np.int64)
    mant_s = np.rint(v[nz] / 2.0 ** -9).astype(np.int64)
    c = np.where(normal, ((lead + 7) << 3) | mant_n, mant_s)
    code[nz] = c.astype(np.uint8)
    return code


def e4m3_decode(code):
    """Value of an E4M3 bit pattern (NaN for 0x7F / 0xFF)."""
    code = np.asarray(code, dtype=np.int64)
    s = np.where(code & 0x80, -1.0, 1.0)
    ex = (code >> 3) & 0xF
    m = code & 0x7
    val = np.where(ex == 0, m * 2.0 ** -9, np.ldexp(1.0 + m / 8.0, ex - 7))
    val = np.where((code & 0x7F) == 0x7F, np.nan, val)
    return s * val


def e2m1_encode(v):
    """Bit pattern of an exactly representable E2M1 value; -0 is written as +0 (code 0)."""
    v = np.asarray(v, dtype=np.float64)
    mags = np.array(E2M1_MAGNITUDES)
    mag_code = np.searchsorted(mags, np.abs(v))
    assert np.all(mags[mag_code] == np.abs(v)), "value not representable in E2M1"
    sign = (v < 0).astype(np.int64)
    return ((sign << 3) | mag_code).astype(np.uint8)


def e2m1_decode(code):
    code = np.asarray(code, dtype=np.int64)
    mags = np.array(E2M1_MAGNITUDES)
    return np.where(code & 0x8, -1.0, 1.0) * mags[code & 0x7]


# --------------------------------------------------------------------------------------------
# S2  FP4 pack  — [V4.1 notes] FP4 主 KV キャッシュ bullet; [V4 blog] storage paragraph
# --------------------------------------------------------------------------------------------

def scale_pad(n_blocks: int) -> int:
    return (n_blocks + 3) // 4 * 4


def pack_fp4(src, d_rope: int, g: float = 1.0):
    """Pack rows ``src[n, d]`` (bf16 values as float64): first ``d - d_rope`` channels to E2M1 with one
    E4M3 scale per 32 channels and the per-tensor fp32 global scale ``g``; last ``d_rope`` channels kept
    as bf16.  Returns (codes u8 [n, d_n/2], scales u8 [n, S_pad], rope float64 [n, d_rope]).

    Per 32-block: s = E4M3(fp32(amax / fp32(6 g))); an all-zero scale zeroes the block;
    code_e = E2M1(fp32(x_e / fp32(s g))), -0 written as +0."""
    src = np.asarray(src, dtype=np.float64)
    n, d = src.shape
    d_n = d - d_rope
    assert d_n % 32 == 0
    nb = d_n // 32
    blocks = src[:, :d_n].reshape(n, nb, 32)
    amax = np.max(np.abs(blocks), axis=2)                                   # exact (bf16 inputs)
    six_g = fp32(6.0) * fp32(g)
    s_f = fp32(amax) / six_g                                                # fp32 correctly rounded
    s = e4m3_rne_satfinite(s_f.astype(np.float64))
    den = (fp32(s) * fp32(g)).astype(np.float64)                            # fp32 product
    with np.errstate(divide="ignore", invalid="ignore"):
        q = (fp32(blocks) / fp32(den)[:, :, None]).astype(np.float64)      # fp32 correctly rounded
    q = np.where(s[:, :, None] == 0, 0.0, q)
    v = e2m1_rne_satfinite(q)
    v = np.where(v == 0, 0.0, v)                                            # -0 -> +0
    codes4 = e2m1_encode(v).reshape(n, d_n).astype(np.uint8)
    codes = (codes4[:, 0::2] | (codes4[:, 1::2] << 4)).astype(np.uint8)    # element 2j low nibble
    scales = np.zeros((n, scale_pad(nb)), dtype=np.uint8)
    scales[:, :nb] = e4m3_encode(s)
    rope = src[:, d_n:].copy()
    return codes, scales, rope


def unpack_codes(codes, d_n: int):
    """u8 [n, d_n/2] -> E2M1 codes [n, d_n] (element order)."""
    codes = np.asarray(codes, dtype=np.uint8)
    out = np.empty(codes.shape[:-1] + (d_n,), dtype=np.uint8)
    out[..., 0::2] = codes & 0xF
    out[..., 1::2] = codes >> 4
    return out


def dequant_fp4(codes, scales, d_n: int, g: float = 1.0):
    """x̂_e = e2m1(code_e) * e4m3(scale_block) * g   (exact in float64)."""
    nb = d_n // 32
    vals = e2m1_decode(unpack_codes(codes, d_n))
    s = e4m3_decode(np.asarray(scales)[..., :nb])
    return vals * np.repeat(s, 32, axis=-1) * float(np.float32(g))


# --------------------------------------------------------------------------------------------
# S6  FP8 window — [V4.1 notes] FP4 主 KV キャッシュ bullet (the sliding-window KV stays in FP8, being
#     more sensitive to quantisation); [V4 blog] storage paragraph (FP8 KV with the RoPE channels in
#     BF16).  The pages fix the element format, not its scaling: reading taken here, one fp32 scale per
#     64 channels of a row (the attention's 64-channel blocks), s = fp32(amax / 448), elements
#     E4M3 RNE with saturation, an all-zero block has scale 0 and codes 0; RoPE channels stay bf16.
# --------------------------------------------------------------------------------------------

FP8_WIN_BLOCK = 64


def pack_fp8_window(rows, d_rope: int):
    """Window rows [n, d] (bf16 values as float64) -> (codes u8 [n, d_n] E4M3 bit patterns, scales fp32
    [n, d_n / 64], rope float64 [n, d_rope])."""
    rows = np.asarray(rows, np.float64)
    n, d = rows.shape
    d_n = d - d_rope
    assert d_n % FP8_WIN_BLOCK == 0
    blocks = rows[:, :d_n].reshape(n, d_n // FP8_WIN_BLOCK, FP8_WIN_BLOCK)
    amax = np.abs(blocks).max(axis=-1)
    scale = (fp32(amax) / np.float32(E4M3_MAX)).astype(np.float32)          # fp32 division
    safe = np.where(scale > 0, scale, np.float32(1.0))
    q = (fp32(blocks) / safe[..., None]).astype(np.float32)                  # fp32 division
    v = e4m3_rne_satfinite(q.astype(np.float64))
    v = np.where(scale[..., None] > 0, v, 0.0)
    codes = e4m3_encode(np.abs(v)) | np.where(v < 0, 0x80, 0).astype(np.uint8)
    return codes.reshape(n, d_n).astype(np.uint8), scale, rows[:, d_n:].copy()


def dequant_fp8_window(codes, scales, rope):
    """Window rows [n, d] float64: e4m3(code) * scale of its 64-channel block, then the bf16 RoPE part."""
    codes = np.asarray(codes)
    n, d_n = codes.shape
    vals = e4m3_decode(codes).reshape(n, d_n // FP8_WIN_BLOCK, FP8_WIN_BLOCK)
    vals = vals * np.asarray(scales, np.float64)[..., None]
    return np.concatenate([vals.reshape(n, d_n), np.asarray(rope, np.float64)], axis=-1)


def paged_rows(pool, block_table, page: int, n: int):
    """Logical entries 0 .. n-1 of one sequence in a paged cache: entry i lives in slot i % page of the
    physical page block_table[i // page] of ``pool[n_pages, page, ...]`` (a reading for the paged cache:
    the pages name paged KV for serving but give no layout)."""
    pool = np.asarray(pool)
    table = np.asarray(block_table, np.int64)
    i = np.arange(n)
    return pool[table[i // page], i % page]


# --------------------------------------------------------------------------------------------
# S1  Compressor — [V4 blog] §ハイブリッド注意, Fig. 3 (4x softmax-gated pooling with a learned
#     positional bias) and Fig. 4 (128x for HCA); [V4.1 notes] CED bullet eq.(1) (C, Z are separate
#     projections of the hidden state) and CSA2 bullet (no overlapping entries; indexer K projected
#     from the main KV).
# --------------------------------------------------------------------------------------------

def project(x, W):
    """bf16(x · W) with a double accumulator.  x [..., d_m], W [d_m, d]."""
    return bf16_round(np.asarray(x, np.float64) @ np.asarray(W, np.float64))


def rope_rotate(v, pos, d_rope: int, theta: float):
    """Rotate the last ``d_rope`` channels of ``v[..., d]`` at positions ``pos[...]``: half-split pairs
    (m, m + d_rope/2), angle pos * theta^(-2m/d_rope)."""
    v = np.array(v, dtype=np.float64, copy=True)
    if theta == 0 or d_rope == 0:
        return v
    half = d_rope // 2
    m = np.arange(half, dtype=np.float64)
    inv_freq = theta ** (-2.0 * m / d_rope)
    ang = np.asarray(pos, dtype=np.float64)[..., None] * inv_freq
    cos, sin = np.cos(ang), np.sin(ang)
    d = v.shape[-1]
    x1 = v[..., d - d_rope:d - half].copy()
    x2 = v[..., d - half:].copy()
    v[..., d - d_rope:d - half] = x1 * cos - x2 * sin
    v[..., d - half:] = x1 * sin + x2 * cos
    return v


def compress_pool(C, Z, b_pos, r: int, d_rope: int = 0, theta: float = 0.0, pos0: int = 0):
    """Softmax-gated pooling of non-overlapping groups of ``r`` tokens, one gate per channel.

    C, Z [T, d] (bf16 values), b_pos [r, d].  For entry i, channel c:
        a_j = Z[r i + j, c] + b_pos[j, c];  w = softmax_j(a);  c_i = sum_j w_j C[r i + j, c]
    then RoPE on the last d_rope channels at position pos0 + r i, then one rounding to bf16.
    Returns c [T // r, d]."""
    C = np.asarray(C, np.float64)
    Z = np.asarray(Z, np.float64)
    T, d = C.shape
    n = T // r
    Cg = C[: n * r].reshape(n, r, d)
    a = Z[: n * r].reshape(n, r, d) + np.asarray(b_pos, np.float64)[None, :, :]
    a = a - a.max(axis=1, keepdims=True)
    e = np.exp(a)
    w = e / e.sum(axis=1, keepdims=True)
    pooled = (w * Cg).sum(axis=1)
    pos = pos0 + r * np.arange(n)
    pooled = rope_rotate(pooled, pos, d_rope, theta)
    return bf16_round(pooled)


def index_key(c, W_IK):
    """Indexer key k_I = bf16(c · W_IK) (CSA2: indexer K is a projection of the main KV)."""
    return project(c, W_IK)


def compress(x=None, W_kv=None, W_g=None, C=None, Z=None, *, b_pos, r, d_rope=0, theta=0.0, pos0=0,
             W_IK=None):
    """Full compressor for one sequence.  Projection mode (x, W_kv, W_g) or pooling mode (C, Z).
    Returns (c, k_I or None, C, Z)."""
    if x is not None:
        C = project(x, W_kv)
        Z = project(x, W_g)
    c = compress_pool(C, Z, b_pos, r, d_rope, theta, pos0)
    kI = index_key(c, W_IK) if W_IK is not None else None
    return c, kI, C, Z


# --------------------------------------------------------------------------------------------
# S3  Lightning indexer — [V4 blog] §ハイブリッド注意 (FP4, multi-head dot product with ReLU scores,
#     one score per compressed block per query)
# --------------------------------------------------------------------------------------------

def index_scores(qI, w, g_q, k_codes, k_scales, g_k, q_pos, n_c: int, r: int, keys=None):
    """Scores s(t, i) for one sequence.

    qI [Nq, H_I, d_I] bf16 values (quantized here with the FP4 pack, global scale g_q),
    w [Nq, H_I], index cache (k_codes [n, d_I/2], k_scales [n, S_pad], g_k).
    ``keys`` (optional) [Nq, m] key ids to score (-1 = empty); default all n cache rows.
    Returns (scores [Nq, m] float64 with -inf where not visible / empty, key ids [Nq, m]).

    P[h, i, b] = sum_{e in block b} q_e k_e over E2M1 values (exact);
    s = g_q g_k sum_h w_h max(0, sum_b sq[h,b] sk[i,b] P[h,i,b]);  -0 -> +0."""
    qI = np.asarray(qI, np.float64)
    Nq, H, dI = qI.shape
    nb = dI // 32
    qc, qs, _ = pack_fp4(qI.reshape(Nq * H, dI), 0, g_q)
    qv = e2m1_decode(unpack_codes(qc, dI)).reshape(Nq, H, nb, 32)
    sq = e4m3_decode(qs[:, :nb]).reshape(Nq, H, nb)
    n = np.asarray(k_codes).shape[0]
    kv = e2m1_decode(unpack_codes(k_codes, dI)).reshape(n, nb, 32)
    sk = e4m3_decode(np.asarray(k_scales)[:, :nb])
    if keys is None:
        keys = np.broadcast_to(np.arange(n), (Nq, n))
    keys = np.asarray(keys, np.int64)
    m = keys.shape[1]
    scores = np.full((Nq, m), -np.inf)
    gg = float(np.float32(g_q)) * float(np.float32(g_k))
    w = np.asarray(w, np.float64)
    for qi in range(Nq):
        ids = keys[qi]
        t = int(q_pos[qi])
        ok = (ids >= 0) & (ids < n_c) & (r * ids + r - 1 <= t)
        sel = ids[ok]
        P = np.einsum("hbe,ibe->hib", qv[qi], kv[sel])                      # exact block partials
        comb = np.einsum("hb,ib,hib->hi", sq[qi], sk[sel], P)
        s = gg * np.einsum("h,hi->i", w[qi], np.maximum(comb, 0.0))
        s = s + 0.0                                                          # -0 -> +0
        scores[qi, ok] = s
    return scores, keys


# --------------------------------------------------------------------------------------------
# S4  Top-k — [V4 blog] Fig. 3 (top-k compressed blocks per query)
# --------------------------------------------------------------------------------------------

def topk(scores, ids, k: int):
    """Per row: the k_eff = min(k, #finite) entries by (score desc, id asc); ids of those, padded with
    -1.  Returns (idx [Nq, k] int32 in that order, selected scores [Nq, k] with -inf padding)."""
    scores = np.asarray(scores, np.float64)
    ids = np.asarray(ids, np.int64)
    Nq = scores.shape[0]
    out = np.full((Nq, k), -1, dtype=np.int32)
    out_s = np.full((Nq, k), -np.inf)
    for qi in range(Nq):
        valid = np.isfinite(scores[qi])
        s = scores[qi][valid]
        i = ids[qi][valid]
        order = np.lexsort((i, -s))[:k]
        out[qi, : len(order)] = i[order]
        out_s[qi, : len(order)] = s[order]
    return out, out_s


# --------------------------------------------------------------------------------------------
# S7  Hierarchical pool — [V4.1 notes] Hierarchical Sparse Indexer bullet, Fig. 5
# --------------------------------------------------------------------------------------------

def hierarchical_pool(scores, n_blocks_keep: int, G: int = 8):
    """scores [Nq, n] over key ids 0..n-1 (-inf = not visible).  Block j = entries [G j, G j + G);
    block score = max over its visible entries.  Keep the top ``n_blocks_keep`` blocks by (block score
    desc, block id asc); the pool lists their entries (block by block, ascending inside a block), -1
    for entries that are not visible and for missing blocks.  Returns (pool [Nq, n_blocks_keep*G],
    kept block ids [Nq, n_blocks_keep] with -1 padding)."""
    scores = np.asarray(scores, np.float64)
    Nq, n = scores.shape
    nblk = (n + G - 1) // G
    padded = np.full((Nq, nblk * G), -np.inf)
    padded[:, :n] = scores
    bs = padded.reshape(Nq, nblk, G).max(axis=2)
    blk, _ = topk(bs, np.broadcast_to(np.arange(nblk), (Nq, nblk)), n_blocks_keep)
    pool = np.full((Nq, n_blocks_keep * G), -1, dtype=np.int32)
    for qi in range(Nq):
        for j, b in enumerate(blk[qi]):
            if b < 0:
                continue
            for e in range(G):
                i = b * G + e
                if i < n and np.isfinite(scores[qi, i]):
                    pool[qi, j * G + e] = i
    return pool, blk


# --------------------------------------------------------------------------------------------
# S5/S6  Attention over selected entries (or all visible entries: HCA) plus the sliding window —
#        [V4 blog] Fig. 3 (CSA: selected compressed entries ∪ window branch), Fig. 4 (HCA: dense over
#        the compressed stream, same window)
# --------------------------------------------------------------------------------------------

def entry_kv(codes, scales, rope, d_n: int, g: float):
    """Full d-dim key/value rows of the compressed cache: dequantized FP4 part ‖ bf16 RoPE part."""
    return np.concatenate([dequant_fp4(codes, scales, d_n, g), np.asarray(rope, np.float64)], axis=-1)


def window_rows(t: int, win_kv, win_pos0: int, W: int):
    """Rows of the window buffer holding tokens p in [max(0, t-W+1), t]."""
    Wn = win_kv.shape[0]
    lo = max(0, t - W + 1, win_pos0)
    hi = min(t, win_pos0 + Wn - 1)
    if hi < lo:
        return np.zeros((0, win_kv.shape[1]))
    return np.asarray(win_kv[lo - win_pos0: hi - win_pos0 + 1], np.float64)


def attention(q, q_pos, kv_rows, idx, n_c: int, win_kv, win_pos0: int, W: int, scale: float,
              round_out: bool = True, out_rope_theta: float = 0.0, d_rope: int = 0):
    """One sequence.  q [Nq, H, d] (bf16 values, already rotated); kv_rows [n, d] dequantized entries;
    idx [Nq, k] selected entry ids (entries < 0 or >= n_c skipped); window buffer win_kv [Wn, d] at
    positions win_pos0 ...  One joint softmax over selected ∪ window with logits scale·(q·K);
    K = V (one shared KV head).  Returns (out [Nq, H, d] (bf16-rounded unless round_out=False),
    lse [Nq, H] natural log, -inf for an empty set).
    out_rope_theta != 0: the "RoPE-attention-RoPE-cast" epilogue ([V4.1 notes] §実装上の工夫, inference
    kernels): before the bf16 cast the last d_rope channels of out are rotated back by the query's
    own RoPE (position -t), so the values' rotations come out relative to the query (a reading: the
    pages name the kernel, not its formula)."""
    q = np.asarray(q, np.float64)
    Nq, H, d = q.shape
    out = np.zeros((Nq, H, d))
    lse = np.full((Nq, H), -np.inf)
    for qi in range(Nq):
        ids = np.asarray(idx[qi], np.int64)
        ids = ids[(ids >= 0) & (ids < n_c)]
        K = np.concatenate([kv_rows[ids], window_rows(int(q_pos[qi]), win_kv, win_pos0, W)], axis=0)
        if K.shape[0] == 0:
            continue
        logits = scale * (q[qi] @ K.T)                                   # [H, m]
        mx = logits.max(axis=1, keepdims=True)
        e = np.exp(logits - mx)
        ssum = e.sum(axis=1, keepdims=True)
        lse[qi] = (mx + np.log(ssum))[:, 0]
        out[qi] = (e / ssum) @ K
        if out_rope_theta != 0.0 and d_rope:
            out[qi] = rope_rotate(out[qi], np.full(H, -float(q_pos[qi])), d_rope, out_rope_theta)
    if round_out:
        out = bf16_round(out)
    return out, lse


def hca_attention(q, q_pos, kv_rows, n_c: int, r: int, win_kv, win_pos0: int, W: int, scale: float,
                  round_out: bool = True, out_rope_theta: float = 0.0, d_rope: int = 0):
    """HCA: attention over every visible compressed entry (i < n_c, r i + r - 1 <= t) plus the window."""
    q_pos = np.asarray(q_pos, np.int64)
    Nq = q.shape[0]
    n_vis = [min(n_c, (int(t) + 1) // r) for t in q_pos]
    kmax = max(n_vis) if Nq else 0
    idx = np.full((Nq, max(kmax, 1)), -1, dtype=np.int64)
    for qi in range(Nq):
        idx[qi, : n_vis[qi]] = np.arange(n_vis[qi])
    return attention(q, q_pos, kv_rows, idx, n_c, win_kv, win_pos0, W, scale, round_out, out_rope_theta, d_rope)


def lse_merge(out1, lse1, out2, lse2):
    """Closed-form merge of two softmax-attention partials over disjoint key sets."""
    lse = np.logaddexp(lse1, lse2)
    a = np.exp(lse1 - lse)[..., None]
    b = np.exp(lse2 - lse)[..., None]
    return a * out1 + b * out2, lse
