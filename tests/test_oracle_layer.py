"""Pins for the oracle's compressor, indexer, top-k, attention and reuse paths, no GPU.

Each check ties the oracle to something it does not compute itself: closed forms (uniform / one-hot /
known gates, RoPE at position 0 and on unit vectors), library routines (torch matmul, torch SDPA),
brute force on tiny inputs (pairwise top-k ranks, per-element dot products), and invariants the
definitions fix (softmax rows sum to 1, LSE merge of disjoint key sets, k >= n -> dense)."""
import math
import os

import numpy as np
import pytest
import torch

from oracle import csa_oracle as O

GOLD = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng(1234)


def bf(x):
    return O.bf16_round(np.asarray(x, np.float64))


# ------------------------------------------------------------------------------------ compressor

def test_uniform_gate_is_mean_pooling():
    C = bf(rng.standard_normal((64, 40)))
    Z = np.tile(bf(rng.standard_normal((1, 40))), (64, 1))          # same logit in every slot
    c = O.compress_pool(C, Z, np.zeros((4, 40)), 4)
    assert np.array_equal(c, bf(C.reshape(16, 4, 40).mean(axis=1)))


def test_one_hot_gate_copies_a_token():
    C = bf(rng.standard_normal((32, 24)))
    Z = bf(rng.standard_normal((32, 24)))
    b = np.zeros((4, 24))
    b[2] = 1e4                                                        # slot 2 wins every channel
    c = O.compress_pool(C, Z, b, 4)
    assert np.array_equal(c, C[2::4])


def test_known_gate_weights():
    p = np.array([0.1, 0.2, 0.3, 0.4])
    C = bf(rng.standard_normal((8, 16)))
    b = np.tile(np.log(p)[:, None], (1, 16))
    c = O.compress_pool(C, np.zeros((8, 16)), b, 4)
    ref = bf(np.einsum("j,ijc->ic", p, C.reshape(2, 4, 16)))
    assert np.allclose(c, ref, rtol=2 ** -8, atol=0)


def test_gate_weights_sum_to_one_and_ratio_one_is_identity():
    C = np.full((128, 8), 0.75)
    Z = bf(rng.standard_normal((128, 8)) * 5)
    c = O.compress_pool(C, Z, bf(rng.standard_normal((128, 8))), 128)
    assert np.all(c == 0.75)
    C2 = bf(rng.standard_normal((16, 8)))
    assert np.array_equal(O.compress_pool(C2, Z[:16], np.zeros((1, 8)), 1), C2)


def test_rope_closed_forms():
    d, dr = 12, 8
    v = np.zeros((3, d))
    v[:, d - dr] = 1.0                                                # unit vector on pair m = 0
    v[:, d - dr + 1] = 1.0                                            # and on pair m = 1 (x1 part)
    pos = np.array([0, 5, 1000])
    out = O.rope_rotate(v, pos, dr, 10000.0)
    assert np.array_equal(out[0], v[0])                               # position 0: identity
    f1 = 10000.0 ** (-2.0 / dr)
    for i, p in enumerate(pos):
        assert math.isclose(out[i, d - dr], math.cos(p), abs_tol=1e-12)
        assert math.isclose(out[i, d - dr + dr // 2], math.sin(p), abs_tol=1e-12)
        assert math.isclose(out[i, d - dr + 1], math.cos(p * f1), abs_tol=1e-12)
        assert math.isclose(out[i, d - dr + dr // 2 + 1], math.sin(p * f1), abs_tol=1e-12)
    assert np.array_equal(out[:, : d - dr], v[:, : d - dr])           # nope part untouched
    w = rng.standard_normal((5, d))
    r5 = O.rope_rotate(w, np.arange(5) * 37, dr, 10000.0)
    n_in = w[:, d - dr: d - dr // 2] ** 2 + w[:, d - dr // 2:] ** 2
    n_out = r5[:, d - dr: d - dr // 2] ** 2 + r5[:, d - dr // 2:] ** 2
    assert np.allclose(n_in, n_out, rtol=1e-12)                       # pairs keep their norm


def test_compress_rope_position_is_group_start():
    C = bf(rng.standard_normal((16, 8)))
    Z = np.zeros((16, 8))
    c = O.compress_pool(C, Z, np.zeros((4, 8)), 4, d_rope=4, theta=10000.0, pos0=40)
    mean = C.reshape(4, 4, 8).mean(axis=1)
    ref = bf(O.rope_rotate(mean, 40 + 4 * np.arange(4), 4, 10000.0))
    assert np.array_equal(c, ref)


def test_projection_vs_torch_matmul():
    x = bf(rng.standard_normal((4, 7, 64)))
    W = bf(rng.standard_normal((64, 24)) / 8)
    ref = (torch.from_numpy(x) @ torch.from_numpy(W)).numpy()
    assert np.array_equal(O.project(x, W), bf(ref))
    c, kI, C, Z = O.compress(x[0], W, W, b_pos=np.zeros((4, 24)), r=4, W_IK=W[:24, :8])
    assert np.array_equal(C, Z) and kI.shape == (1, 8)


# --------------------------------------------------------------------------------------- indexer

def _pack(rows, g=1.0):
    return O.pack_fp4(rows, 0, g)


def test_index_single_head_positive_is_plain_dot():
    dI = 64
    q = bf(np.abs(rng.standard_normal((3, 1, dI))))
    k = bf(np.abs(rng.standard_normal((20, dI))))
    kc, ks, _ = _pack(k)
    s, _ = O.index_scores(q, np.ones((3, 1)), 1.0, kc, ks, 1.0, [10 ** 6] * 3, 20, 4)
    qc, qs, _ = _pack(q[:, 0])
    qd = O.dequant_fp4(qc, qs, dI)
    kd = O.dequant_fp4(kc, ks, dI)
    assert np.allclose(s, qd @ kd.T, rtol=1e-14, atol=0)


def test_index_brute_force_tiny():
    """Per-element loops over the dequantised values (a different route than block partials x scales)."""
    H, dI, n = 3, 64, 9
    q = bf(rng.standard_normal((2, H, dI)))
    k = bf(rng.standard_normal((n, dI)) * 2)
    w = rng.standard_normal((2, H))
    gq, gk = 0.5, 2.0
    kc, ks, _ = O.pack_fp4(k, 0, gk)
    pos = np.array([4 * 6 + 3, 4 * 9 - 1])
    s, _ = O.index_scores(q, w, gq, kc, ks, gk, pos, n, 4)
    qc, qs, _ = O.pack_fp4(q.reshape(-1, dI), 0, gq)
    qd = O.dequant_fp4(qc, qs, dI, gq).reshape(2, H, dI)
    kd = O.dequant_fp4(kc, ks, dI, gk)
    for a in range(2):
        for i in range(n):
            if 4 * i + 3 > pos[a]:
                assert s[a, i] == -np.inf
                continue
            tot = 0.0
            for h in range(H):
                dot = 0.0
                for e in range(dI):
                    dot += qd[a, h, e] * kd[i, e]
                tot += w[a, h] * max(dot, 0.0)
            assert math.isclose(s[a, i], tot, rel_tol=1e-12, abs_tol=1e-12)


def test_index_block_partials_exact_quarter_multiples():
    # unit scales and g = 1: the score of one head with w = 1 is an exact multiple of 0.25
    dI = 128
    qv = rng.choice([0.5, 1, 1.5, 2, 3, 4, -1, -0.5], size=(1, 1, dI))
    qv[..., ::32] = 6.0
    kv = rng.choice([0.5, 1, 1.5, 2, 3, 4, -2, -6], size=(16, dI))
    kv[:, ::32] = 6.0
    kc, ks, _ = _pack(kv)
    s, _ = O.index_scores(qv, np.ones((1, 1)), 1.0, kc, ks, 1.0, [10 ** 6], 16, 4)
    dots = np.maximum(kv @ qv[0, 0], 0)
    assert np.array_equal(s[0], dots) and np.all(np.mod(s[0] * 4, 1) == 0)


def test_index_linear_in_w_and_relu_per_head():
    H, dI, n = 4, 64, 32
    q = bf(rng.standard_normal((1, H, dI)))
    k = bf(rng.standard_normal((n, dI)))
    kc, ks, _ = _pack(k)
    w = rng.standard_normal((1, H))
    s1, _ = O.index_scores(q, w, 1.0, kc, ks, 1.0, [10 ** 6], n, 4)
    s2, _ = O.index_scores(q, -2.0 * w, 1.0, kc, ks, 1.0, [10 ** 6], n, 4)
    assert np.allclose(s2, -2.0 * s1, rtol=1e-14, atol=0)
    # one head only: s(q) + s(-q) = |q.k|  (ReLU(x) + ReLU(-x) = |x|)
    w1 = np.zeros((1, H)); w1[0, 1] = 1.0
    sp, _ = O.index_scores(q, w1, 1.0, kc, ks, 1.0, [10 ** 6], n, 4)
    sm, _ = O.index_scores(-q, w1, 1.0, kc, ks, 1.0, [10 ** 6], n, 4)
    qc, qs, _ = _pack(q[0])
    ref = np.abs(O.dequant_fp4(kc, ks, dI) @ O.dequant_fp4(qc, qs, dI)[1])
    assert np.allclose(sp[0] + sm[0], ref, rtol=1e-12, atol=1e-12)


def test_index_candidates_subset():
    H, dI, n = 2, 64, 40
    q = bf(rng.standard_normal((1, H, dI)))
    kc, ks, _ = _pack(bf(rng.standard_normal((n, dI))))
    w = np.ones((1, H))
    full, _ = O.index_scores(q, w, 1.0, kc, ks, 1.0, [4 * 30 + 3], n, 4)
    cand = np.array([[5, 39, -1, 0, 30, 31]])
    s, ids = O.index_scores(q, w, 1.0, kc, ks, 1.0, [4 * 30 + 3], n, 4, keys=cand)
    assert np.array_equal(ids, cand)
    for j, i in enumerate(cand[0]):
        assert s[0, j] == (full[0, i] if 0 <= i <= 30 else -np.inf)


# ----------------------------------------------------------------------------------------- top-k

def test_topk_brute_force_pairwise_rank():
    for trial in range(30):
        n = int(rng.integers(1, 40))
        k = int(rng.integers(1, 12))
        s = rng.choice([-1.0, 0.0, 0.5, 1.0, 2.0, -np.inf], size=(1, n))   # heavy ties
        ids = rng.permutation(n)[None, :] * 3
        idx, _ = O.topk(s, ids, k)
        chosen = set(int(i) for i in idx[0] if i >= 0)
        finite = [(s[0, j], ids[0, j]) for j in range(n) if np.isfinite(s[0, j])]
        for sc, i in finite:
            better = sum(1 for sc2, i2 in finite if sc2 > sc or (sc2 == sc and i2 < i))
            assert (better < k) == (int(i) in chosen)
        assert len(chosen) == min(k, len(finite))
        assert np.all(idx[0, len(chosen):] == -1)


def test_topk_signed_zero_ties_by_index():
    s = np.array([[0.0, -0.0, 0.0, -0.0, -1.0]])
    idx, _ = O.topk(s, np.arange(5)[None], 2)
    assert set(idx[0]) == {0, 1}


# ------------------------------------------------------------------------------------- attention

def _cache(n, d, dr, g=1.0):
    src = bf(rng.standard_normal((n, d)))
    codes, sc, rope = O.pack_fp4(src, dr, g)
    return O.entry_kv(codes, sc, rope, d - dr, g)


def test_attention_all_selected_equals_dense_sdpa():
    n, d, dr, H, W = 24, 64, 32, 4, 8
    kv = _cache(n, d, dr)
    win = bf(rng.standard_normal((W + 2, d)))
    t = 4 * n + 5
    q = bf(rng.standard_normal((1, H, d)))
    idx = rng.permutation(n)[None, :]
    scale = d ** -0.5
    out, lse = O.attention(q, [t], kv, idx, n, win, t - W - 1, W, scale, round_out=False)
    K = np.concatenate([kv, win[-W:]], axis=0)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q).transpose(0, 1)[None], torch.from_numpy(K)[None, None],
        torch.from_numpy(K)[None, None], scale=scale)[0].transpose(0, 1).numpy()
    assert np.allclose(out, ref, rtol=1e-12, atol=1e-12)
    lref = torch.logsumexp(torch.from_numpy(scale * q[0] @ K.T), dim=1).numpy()
    assert np.allclose(lse[0], lref, rtol=1e-12, atol=1e-12)


def test_attention_one_key_and_constant_values():
    d = 32
    kv = _cache(4, d, 0)
    q = bf(rng.standard_normal((1, 3, d)))
    out, _ = O.attention(q, [100], kv, np.array([[2, -1, 7]]), 4, np.zeros((0, d)), 0, 128, 0.3)
    assert np.array_equal(out[0], np.tile(kv[2], (3, 1)))          # one key (id 7 >= n_c skipped)
    const = np.tile(kv[1:2], (4, 1))
    out, _ = O.attention(q, [100], const, np.array([[0, 1, 2, 3]]), 4, np.tile(kv[1], (5, 1)), 96, 128,
                         0.3, round_out=False)
    assert np.allclose(out[0], np.tile(kv[1], (3, 1)), rtol=1e-14, atol=1e-14)   # rows sum to 1


def test_attention_inverse_rope_epilogue_closed_form():
    """One key (softmax weight 1): out is the key, whose RoPE pairs were stored rotated at its position
    p.  The epilogue rotates them back by the query position t, so pair m comes out as its raw value
    rotated by (p - t) * theta^(-2m/d_rope); the unit raw pair (1, 0) gives (cos, sin) of that angle."""
    d, d_r, theta = 12, 4, 10000.0
    f = [1.0, theta ** -0.5]                                   # theta^(-2m/d_r), m = 0, 1
    for p, t in ((900, 900), (901, 900), (37, 4095)):
        key = np.zeros(d)
        key[:8] = np.arange(1, 9)
        for m in range(2):                                     # raw pair (1, 0) stored rotated at p
            key[8 + m], key[10 + m] = math.cos(p * f[m]), math.sin(p * f[m])
        q = np.ones((1, 1, d))
        out, _ = O.attention(q, [t], key[None], np.array([[0]]), 1, np.zeros((0, d)), 0, 128, 0.1,
                             round_out=False, out_rope_theta=theta, d_rope=d_r)
        assert np.array_equal(out[0, 0, :8], key[:8])          # channels outside the RoPE slice untouched
        for m in range(2):
            a = (p - t) * f[m]
            assert abs(out[0, 0, 8 + m] - math.cos(a)) < 1e-9 and abs(out[0, 0, 10 + m] - math.sin(a)) < 1e-9
        off, _ = O.attention(q, [t], key[None], np.array([[0]]), 1, np.zeros((0, d)), 0, 128, 0.1, round_out=False)
        assert np.array_equal(off[0, 0], key)                  # theta = 0: no epilogue


def test_attention_lse_merge_of_disjoint_sets():
    n, d, H = 30, 64, 4
    kv = _cache(n, d, 32)
    q = bf(rng.standard_normal((1, H, d)))
    empty = np.zeros((0, d))
    a = np.array([[0, 3, 5, 8, 13]])
    b = np.array([[1, 2, 21, 29]])
    o1, l1 = O.attention(q, [999], kv, a, n, empty, 0, 128, 0.125, round_out=False)
    o2, l2 = O.attention(q, [999], kv, b, n, empty, 0, 128, 0.125, round_out=False)
    o, l = O.attention(q, [999], kv, np.concatenate([a, b], 1), n, empty, 0, 128, 0.125, round_out=False)
    om, lm = O.lse_merge(o1, l1, o2, l2)
    assert np.allclose(o, om, rtol=1e-12, atol=1e-13) and np.allclose(l, lm, rtol=1e-13, atol=0)


def test_attention_empty_set_and_window_bounds():
    d = 16
    win = bf(rng.standard_normal((300, d)))
    q = bf(rng.standard_normal((2, 2, d)))
    out, lse = O.attention(q, [50, 5], np.zeros((1, d)), np.full((2, 1), -1), 0,
                           np.zeros((0, d)), 0, 128, 1.0)
    assert np.all(out == 0) and np.all(lse == -np.inf)
    assert O.window_rows(5, win, 0, 128).shape[0] == 6                 # t + 1 tokens at the start
    assert O.window_rows(299, win, 0, 128).shape[0] == 128
    assert np.array_equal(O.window_rows(299, win, 0, 128), win[172:300])
    assert O.window_rows(299, win[100:], 100, 128).shape[0] == 128


def test_hca_equals_attention_over_all_visible():
    n, d, r = 40, 64, 128
    kv = _cache(n, d, 32)
    q = bf(rng.standard_normal((2, 4, d)))
    pos = np.array([128 * 17 + 5, 128 * 40 - 1])
    win = bf(rng.standard_normal((256, d)))
    oh, lh = O.hca_attention(q, pos, kv, n, r, win, pos[1] - 255, 128, 0.125)
    for a, t in enumerate(pos):
        nv = (t + 1) // r
        oa, la = O.attention(q[a:a + 1], [t], kv, np.arange(nv)[None], n, win, pos[1] - 255, 128, 0.125)
        assert np.array_equal(oh[a], oa[0]) and np.array_equal(lh[a], la[0])


# ----------------------------------------------------------------------------------------- reuse

def test_reindex_with_all_candidates_equals_full():
    H, dI, n, k = 8, 128, 300, 16
    q = bf(rng.standard_normal((2, H, dI)))
    w = rng.standard_normal((2, H))
    kc, ks, _ = _pack(bf(rng.standard_normal((n, dI))))
    pos = [4 * 200 + 3, 4 * 300 - 1]
    s, ids = O.index_scores(q, w, 1.0, kc, ks, 1.0, pos, n, 4)
    full, _ = O.topk(s, ids, k)
    cand = np.stack([rng.permutation(n), rng.permutation(n)])
    s2, ids2 = O.index_scores(q, w, 1.0, kc, ks, 1.0, pos, n, 4, keys=cand)
    re, _ = O.topk(s2, ids2, k)
    for a in range(2):
        assert set(full[a]) == set(re[a])


def test_hierarchical_pool_brute_force_and_cover_all():
    n, G = 70, 8
    s = rng.standard_normal((3, n))
    s[0, 50:] = -np.inf
    s[1, 3] = -np.inf
    pool, blk = O.hierarchical_pool(s, 4, G)
    for a in range(3):
        bs = [max([s[a, i] for i in range(b * G, min(n, b * G + G))]) for b in range((n + G - 1) // G)]
        order = sorted(range(len(bs)), key=lambda j: (-bs[j], j))
        assert list(blk[a]) == order[:4]
        for j, b in enumerate(blk[a]):
            for e in range(G):
                i = b * G + e
                want = i if (i < n and np.isfinite(s[a, i])) else -1
                assert pool[a, j * G + e] == want
    # a pool that keeps every block holds every visible entry: reindex over it = flat top-k
    pool, _ = O.hierarchical_pool(s, 9, G)
    for a in range(3):
        assert set(pool[a][pool[a] >= 0]) == set(np.flatnonzero(np.isfinite(s[a])))
        flat, _ = O.topk(s[a:a + 1], np.arange(n)[None], 10)
        sub = np.where(pool[a] >= 0, s[a][np.maximum(pool[a], 0)], -np.inf)[None]
        viap, _ = O.topk(sub, pool[a][None], 10)
        assert set(flat[0]) == set(viap[0])


def test_pool_size_from_the_pages():
    vals = {}
    for line in open(os.path.join(GOLD, "pages_numbers.txt")):
        if line.strip() and not line.startswith("#"):
            a, b = line.split()
            vals[a] = int(b)
    nb, G = vals["pool_blocks"], vals["pool_block_size"]
    n = nb * G * 2
    s = rng.standard_normal((1, n))
    pool, _ = O.hierarchical_pool(s, nb, G)
    assert pool.shape[1] == vals["pool_positions"] and np.all(pool >= 0)
    assert vals["csa_ratio"] == 4 and vals["hca_ratio"] == 128
