"""GPU parity of the chunked causal prefill (32768 tokens in 4096-token chunks, d_m = 4096, d = 512,
indexer 8 x 128 FP4, top-512): the compressor's projection GEMM and the multi-query indexer on the
tensor cores, at the real chunk shape, checked on sampled rows the oracle computes one by one (every
value of those rows) plus properties over every row; and small ragged cases checked everywhere."""
import numpy as np
import pytest
import torch

from csa_workloads import CFG3, gen, normal
from oracle import csa_oracle as O
from tests.cmp_utils import SCORE_RTOL, assert_close, check_topk_row, f64, np_u8

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _ulp_close(got, ref, what):
    rms = float(np.sqrt(np.mean(ref ** 2))) or 1.0
    assert_close(got, ref, 1e-3 * rms, 2.0 ** -7 * 1.01, what)


def _sample_rows(n, count, seed):
    rng = np.random.default_rng(seed)
    rows = set(rng.choice(n, size=min(count, n), replace=False).tolist()) | {0, n - 1, min(127, n - 1), min(128, n - 1)}
    return np.array(sorted(rows))


# ------------------------------------------------------------------------------ projection GEMM

def test_projection_cfg3_chunk(cuda_lib):
    """C = x W_kv, Z = x W_g for one 4096-token chunk at d_m = 4096, d = 512 (128 tiles of 128 x 256)."""
    csa = cuda_lib
    s = CFG3
    T = s.extra["chunk"]
    G = gen(30, DEV)
    x = normal((1, T, s.d_m), 1.0, G, DEV)
    W_kv = normal((s.d_m, s.d), s.d_m ** -0.5, G, DEV)
    W_g = normal((s.d_m, s.d), s.d_m ** -0.5, G, DEV)
    b_pos = normal((s.r, s.d), 0.1, G, DEV, torch.float32)
    c, _, C, Z = csa.compress(x=x, W_kv=W_kv, W_g=W_g, b_pos=b_pos, ratio=s.r, d_rope=s.d_r, rope_theta=10000.0)
    torch.cuda.synchronize()
    rows = _sample_rows(T, 96, 1)
    xs = f64(x[0, rows])
    _ulp_close(f64(C[0, rows]), O.project(xs, f64(W_kv)), "C sampled rows")
    _ulp_close(f64(Z[0, rows]), O.project(xs, f64(W_g)), "Z sampled rows")
    # every row: within a bf16 rounding of an fp32 product (property at full size)
    for got, W in ((C, W_kv), (Z, W_g)):
        ref = (x[0].float() @ W.float()).double()
        err = (got[0].double() - ref).abs()
        assert bool(torch.all(err <= 1e-3 + 2.0 ** -7 * 1.01 * ref.abs()))
    # the pooled entries of the chunk (same upstream bytes)
    for e in (0, 511, 1023):
        ref = O.compress_pool(f64(C[0, 4 * e:4 * e + 4]), f64(Z[0, 4 * e:4 * e + 4]), f64(b_pos), s.r, s.d_r,
                              10000.0, 4 * e)
        _ulp_close(f64(c[0, e:e + 1]), ref, f"pooled entry {e}")


@pytest.mark.parametrize("B,T,dm,d", [(2, 1000, 1000, 256), (1, 77, 512, 384), (3, 129, 64, 128)])
def test_projection_ragged(cuda_lib, B, T, dm, d):
    """Token counts off the 128-row tile, d_model off the 64-wide K step, N tiles of 128 and 256."""
    csa = cuda_lib
    G = gen(31)
    x = normal((B, T, dm), 1.0, G)
    W_kv = normal((dm, d), dm ** -0.5, G)
    W_g = normal((dm, d), dm ** -0.5, G)
    b_pos = torch.zeros((4, d), dtype=torch.float32)
    _, _, C, Z = csa.compress(x=x.to(DEV), W_kv=W_kv.to(DEV), W_g=W_g.to(DEV), b_pos=b_pos.to(DEV), ratio=4,
                              d_rope=0)
    torch.cuda.synchronize()
    for b in range(B):
        _ulp_close(f64(C[b]), O.project(f64(x[b]), f64(W_kv)), f"C b={b}")
        _ulp_close(f64(Z[b]), O.project(f64(x[b]), f64(W_g)), f"Z b={b}")


# ------------------------------------------------------------------------- multi-query indexer

def _mq_setup(csa, B, n_max, n_c, Nq, q_pos, H_I, seed, d_I=128):
    G = gen(seed, DEV)
    kI = normal((B, n_max, d_I), 1.0, G, DEV)
    qI = normal((B, Nq, H_I, d_I), 1.0, G, DEV)
    w = normal((B, Nq, H_I), H_I ** -0.5, G, DEV, torch.float32)
    kc = csa.PackedCache(B, n_max, d_I, 0, DEV)
    csa.pack_fp4(kI, kc)
    n_c_t = torch.tensor(n_c, dtype=torch.int32, device=DEV)
    q_pos_t = torch.as_tensor(np.asarray(q_pos, np.int64).reshape(B, Nq), device=DEV)
    return kc, qI, w, n_c_t, q_pos_t


def _check_score_rows(got_rows, s_ref, n_vis, what):
    for i in range(len(got_rows)):
        nv = int(n_vis[i])
        if nv == 0:
            continue
        ref = s_ref[i][:nv]
        assert np.all(np.isfinite(ref))
        rowmax = float(np.max(np.abs(ref)))
        assert_close(got_rows[i][:nv], ref, SCORE_RTOL * rowmax, SCORE_RTOL, f"{what} row {i}")


def test_index_multiquery_cfg3_last_chunk(cuda_lib):
    """The last 4096-query chunk of the 32K prefill: queries t = 28672 .. 32767 over all 8192 entries,
    causal (query t sees entries i with 4 i + 3 <= t).  Sampled rows: every score and the top-512 set
    against the oracle; every row: the columns past its visible range untouched, the rest finite."""
    csa = cuda_lib
    s = CFG3
    n = s.T // s.r
    Nq = s.extra["chunk"]
    t0 = s.T - Nq
    q_pos = np.arange(t0, s.T)
    kc, qI, w, n_c, qp = _mq_setup(csa, 1, n, [n], Nq, q_pos, s.H_I, seed=32)
    scores = torch.full((Nq, n), float("nan"), dtype=torch.float32, device=DEV)
    csa.index_scores(qI, w, kc, n_c, qp, scores, ratio=s.r)
    idx, _, _ = csa.index_topk(qI, w, kc, n_c, qp, ratio=s.r, k=s.k)
    torch.cuda.synchronize()
    n_vis = np.minimum((q_pos + 1) // s.r, n)
    # property over every row
    col = torch.arange(n, device=DEV)[None, :]
    vis = col < torch.as_tensor(n_vis, device=DEV)[:, None]
    assert bool(torch.all(torch.isfinite(scores[vis])))
    assert bool(torch.all(torch.isnan(scores[~vis])))
    assert bool(torch.all((idx >= 0).sum(-1) == s.k))
    # sampled rows against the oracle
    rows = _sample_rows(Nq, 24, 2)
    codes, scales = np_u8(kc.codes[0]), np_u8(kc.scales[0])
    s_ref, ids = O.index_scores(f64(qI[0, rows]), f64(w[0, rows]), 1.0, codes, scales, 1.0, q_pos[rows], n, s.r)
    got = scores[rows].cpu().numpy()
    _check_score_rows(got, s_ref, n_vis[rows], "cfg3 scores")
    gi = idx[0].cpu().numpy()
    for i, r in enumerate(rows):
        check_topk_row(gi[r], s_ref[i], ids[i], s.k, f"cfg3 top-k q={r}")


def test_index_multiquery_cfg3_first_chunk(cuda_lib):
    """Chunk 0: queries t = 0 .. 4095 over the chunk's own 1024 entries; the first queries see fewer
    than k entries (k_eff = visible count, the rest -1), t < 3 sees none."""
    csa = cuda_lib
    s = CFG3
    Nq = s.extra["chunk"]
    n = Nq // s.r
    q_pos = np.arange(0, Nq)
    kc, qI, w, n_c, qp = _mq_setup(csa, 1, n, [n], Nq, q_pos, s.H_I, seed=33)
    idx, sc, _ = csa.index_topk(qI, w, kc, n_c, qp, ratio=s.r, k=s.k, want_scores=True)
    torch.cuda.synchronize()
    n_vis = np.minimum((q_pos + 1) // s.r, n)
    cnt = (idx[0] >= 0).sum(-1).cpu().numpy()
    assert np.array_equal(cnt, np.minimum(n_vis, s.k))
    rows = np.array(sorted({0, 2, 3, 4, 100, 2046, 2047, 2048, 2051, 3000, 4095}))
    codes, scales = np_u8(kc.codes[0]), np_u8(kc.scales[0])
    s_ref, ids = O.index_scores(f64(qI[0, rows]), f64(w[0, rows]), 1.0, codes, scales, 1.0, q_pos[rows], n, s.r)
    gi = idx[0].cpu().numpy()
    for i, r in enumerate(rows):
        check_topk_row(gi[r], s_ref[i], ids[i], s.k, f"chunk 0 top-k q={r}")


@pytest.mark.parametrize("H_I", [8, 5])
def test_index_multiquery_ragged_everywhere(cuda_lib, H_I):
    """Two sequences, 37 queries (two 16-query blocks and a tail) at scattered positions (some before
    the first entry completes, some past n_c), n_c below n_max, fewer heads than 8: every score of
    every row against the oracle, every top-k set."""
    csa = cuda_lib
    B, n_max, Nq, k = 2, 1000, 37, 96
    n_c = [1000, 613]
    rng = np.random.default_rng(34)
    q_pos = rng.integers(0, 4 * 1100, size=(B, Nq))
    q_pos[0, :3] = [0, 2, 3]
    kc, qI, w, n_c_t, qp = _mq_setup(csa, B, n_max, n_c, Nq, q_pos, H_I, seed=35)
    scores = torch.full((B * Nq, n_max), float("nan"), dtype=torch.float32, device=DEV)
    csa.index_scores(qI, w, kc, n_c_t, qp, scores, ratio=4)
    idx, _, _ = csa.index_topk(qI, w, kc, n_c_t, qp, ratio=4, k=k)
    torch.cuda.synchronize()
    got = scores.view(B, Nq, n_max).cpu().numpy()
    for b in range(B):
        codes, scales = np_u8(kc.codes[b]), np_u8(kc.scales[b])
        s_ref, ids = O.index_scores(f64(qI[b]), f64(w[b]), 1.0, codes, scales, 1.0, q_pos[b], n_c[b], 4)
        n_vis = np.minimum((q_pos[b] + 1) // 4, n_c[b])
        _check_score_rows(got[b], s_ref, n_vis, f"b={b}")
        for q in range(Nq):
            assert np.all(np.isnan(got[b, q, n_vis[q]:])), f"b={b} q={q}: columns past the visible range written"
            check_topk_row(idx[b, q].cpu().numpy(), s_ref[q], ids[q], k, f"b={b} q={q}")


# ------------------------------------------------------------------- top-k of prefill-length rows

@pytest.mark.parametrize("n_equal", [8192, 1500, 40])
def test_topk_prefill_rows_with_ties(cuda_lib, n_equal):
    """Top-512 of rows of 8192 scores (the chunked prefill's rows, one CTA of 256 threads per row):
    n_equal scores share the value at the selection boundary, so the tie break (id ascending) decides:
    the whole row, 1500 or 40 of them.  Sets exactly as the oracle's (score desc, id asc); rows that see
    fewer than k entries pad with -1."""
    csa = cuda_lib
    rows, n, k = 6, 8192, 512
    rng = np.random.default_rng(80 + n_equal)
    sc = rng.standard_normal((rows, n)).astype(np.float32)
    for r in range(rows):
        perm = rng.permutation(n)
        top = perm[: k - 100]                       # clearly above the tie value
        tie = perm[k - 100: k - 100 + n_equal] if n_equal < n else perm
        sc[r, top] = 10.0 + rng.random(len(top)).astype(np.float32)
        sc[r, tie] = 3.0
        if n_equal == n:
            sc[r, :] = 3.0
    q_pos = np.full((1, rows), 4 * n - 1, np.int64)
    q_pos[0, -1] = 4 * 300 - 1                     # sees 300 entries only: k_eff = 300
    kc = csa.PackedCache(1, n, 128, 0, DEV)
    scores = torch.as_tensor(sc, device=DEV)
    n_c = torch.tensor([n], dtype=torch.int32, device=DEV)
    idx, _, _ = csa.topk(scores, kc, n_c, torch.as_tensor(q_pos, device=DEV), B=1, Nq=rows, ratio=4, k=k)
    torch.cuda.synchronize()
    got = idx[0].cpu().numpy()
    for r in range(rows):
        nv = min(n, (int(q_pos[0, r]) + 1) // 4)
        s = sc[r].astype(np.float64).copy()
        s[nv:] = -np.inf
        ref, _ = O.topk(s[None], np.arange(n)[None], k)
        assert set(got[r][got[r] >= 0].tolist()) == set(ref[0][ref[0] >= 0].tolist()), f"row {r}"
        assert np.all(got[r][min(k, nv):] == -1) and np.all(got[r][: min(k, nv)] >= 0), f"row {r} padding"
