"""GPU parity of the paged KV cache: the FP4 caches live in pools of pages with a block table per
sequence (entry i of sequence b in slot i % page of page table[b][i // page]); the tables are random
permutations of the pool's pages, so logical neighbours sit in unrelated pages.  Every writer (pack,
the compressor's fused append) and reader (indexer decode / multi-query / Reindex, top-k, tensor-core
and d = 128 attention, HCA) is checked against the oracle on the logical rows the oracle's paged_rows
reads back, including the 5-position speculative decode."""
import numpy as np
import pytest
import torch

from csa_workloads import gen, normal
from oracle import csa_oracle as O
from tests.cmp_utils import LSE_ATOL, LSE_RTOL, OUT_ATOL, OUT_RTOL, SCORE_RTOL, assert_close, check_topk_row, f64, np_u8

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _table(B, width, n_pages, seed):
    """A block table whose pages are a random permutation of the pool (plus spare pages unused)."""
    rng = np.random.default_rng(seed)
    perm = rng.permutation(n_pages)[: B * width]
    return torch.as_tensor(perm.reshape(B, width).astype(np.int32))


def _paged(csa, B, n_max, d, d_r, page, seed, spare=3, g=1.0):
    width = (n_max + page - 1) // page
    n_pages = B * width + spare
    table = _table(B, width, n_pages, seed)
    return csa.PagedCache(B, n_max, d, d_r, DEV, page, n_pages, table, g), table.numpy()


def _logical(cache, table, b, n):
    """Logical rows 0..n-1 of sequence b read back through the oracle's page mapping."""
    codes = O.paged_rows(np_u8(cache.codes).reshape(cache.n_pages, cache.page_size, -1), table[b], cache.page_size, n)
    scales = O.paged_rows(np_u8(cache.scales).reshape(cache.n_pages, cache.page_size, -1), table[b], cache.page_size, n)
    rope = None
    if cache.d_rope:
        rope = O.paged_rows(f64(cache.rope).reshape(cache.n_pages, cache.page_size, -1), table[b], cache.page_size, n)
    return codes, scales, rope


@pytest.mark.parametrize("page", [128, 256])
def test_paged_pack_bit_exact(cuda_lib, page):
    csa = cuda_lib
    B, n, d, d_r = 3, 700, 512, 64
    G = gen(50)
    src = normal((B, n, d), 1.0, G)
    cache, table = _paged(csa, B, n, d, d_r, page, seed=1)
    csa.pack_fp4(src.to(DEV), cache)
    torch.cuda.synchronize()
    for b in range(B):
        codes, scales, rope = O.pack_fp4(f64(src[b]), d_r, 1.0)
        gc, gs, gr = _logical(cache, table, b, n)
        assert np.array_equal(gc, codes) and np.array_equal(gs, scales), f"b={b}"
        assert np.array_equal(gr, f64(src[b, :, d - d_r:]))


def test_paged_compress_append(cuda_lib):
    """Pooling mode with the fused FP4 append of the new entries and their indexer keys into paged
    caches at per-sequence row offsets."""
    csa = cuda_lib
    B, r, d, d_r, dI = 2, 4, 512, 64, 128
    n_new, n_max, page = 37, 640, 128
    G = gen(51)
    C = normal((B, n_new * r, d), 1.0, G)
    Z = normal((B, n_new * r, d), 1.0, G)
    b_pos = normal((r, d), 0.1, G, dtype=torch.float32)
    W_IK = normal((d, dI), d ** -0.5, G)
    kv, tkv = _paged(csa, B, n_max, d, d_r, page, seed=2)
    ki, tki = _paged(csa, B, n_max, dI, 0, page, seed=3)
    row0 = torch.tensor([100, 300], dtype=torch.int32, device=DEV)
    c, kI, _, _ = csa.compress(C=C.to(DEV), Z=Z.to(DEV), b_pos=b_pos.to(DEV), ratio=r, d_rope=d_r, rope_theta=10000.0,
                               W_IK=W_IK.to(DEV), kv_cache=kv, ki_cache=ki, row0=row0)
    torch.cuda.synchronize()
    for b in range(B):
        r0 = int(row0[b])
        codes, scales, _ = O.pack_fp4(f64(c[b]), d_r, 1.0)
        gc, gs, _ = _logical(kv, tkv, b, r0 + n_new)
        assert np.array_equal(gc[r0:], codes) and np.array_equal(gs[r0:], scales), f"kv b={b}"
        kc, ks, _ = O.pack_fp4(f64(kI[b]), 0, 1.0)
        gc, gs, _ = _logical(ki, tki, b, r0 + n_new)
        assert np.array_equal(gc[r0:], kc) and np.array_equal(gs[r0:], ks), f"k_I b={b}"


@pytest.mark.parametrize("Nq,d_I,H_I,onchip", [(1, 128, 8, False), (1, 128, 8, True), (5, 128, 8, False),
                                               (3, 64, 4, False)])
def test_paged_index_topk(cuda_lib, Nq, d_I, H_I, onchip):
    """Decode (one query), speculative 5 positions, and the d_I = 64 path, over a paged index cache."""
    csa = cuda_lib
    B, n_max, page, k = 3, 3000, 256, 200
    n_c = [3000, 1777, 2500]
    G = gen(52 + Nq)
    kI = normal((B, n_max, d_I), 1.0, G)
    cache, table = _paged(csa, B, n_max, d_I, 0, page, seed=4 + Nq)
    csa.pack_fp4(kI.to(DEV), cache)
    qI = normal((B, Nq, H_I, d_I), 1.0, G)
    w = normal((B, Nq, H_I), H_I ** -0.5, G, dtype=torch.float32)
    q_pos = np.array([[4 * nc - Nq + j for j in range(Nq)] for nc in n_c], np.int64)
    q_pos[2] -= 1500                                           # sees fewer entries than it holds
    n_c_t = torch.tensor(n_c, dtype=torch.int32, device=DEV)
    qp = torch.as_tensor(q_pos, device=DEV)
    scores = torch.full((B * Nq, n_max), float("nan"), dtype=torch.float32, device=DEV)
    csa.index_scores(qI.to(DEV), w.to(DEV), cache, n_c_t, qp, scores, ratio=4)
    idx, _, _ = csa.index_topk(qI.to(DEV), w.to(DEV), cache, n_c_t, qp, ratio=4, k=k, onchip=onchip)
    torch.cuda.synchronize()
    got = scores.view(B, Nq, n_max).cpu().numpy()
    for b in range(B):
        codes, scales, _ = _logical(cache, table, b, n_max)
        s_ref, ids = O.index_scores(f64(qI[b]), f64(w[b]), 1.0, codes, scales, 1.0, q_pos[b], n_c[b], 4)
        for q in range(Nq):
            nv = min((q_pos[b, q] + 1) // 4, n_c[b])
            rowmax = float(np.max(np.abs(s_ref[q, :nv])))
            assert_close(got[b, q, :nv], s_ref[q, :nv], SCORE_RTOL * rowmax, SCORE_RTOL, f"scores b={b} q={q}")
            check_topk_row(idx[b, q].cpu().numpy(), s_ref[q], ids[q], k, f"top-k b={b} q={q}")


def test_paged_reindex_candidates(cuda_lib):
    csa = cuda_lib
    B, n_max, page, k, n_cand = 2, 2048, 128, 64, 300
    G = gen(55)
    kI = normal((B, n_max, 128), 1.0, G)
    cache, table = _paged(csa, B, n_max, 128, 0, page, seed=6)
    csa.pack_fp4(kI.to(DEV), cache)
    qI = normal((B, 1, 8, 128), 1.0, G)
    w = normal((B, 1, 8), 0.35, G, dtype=torch.float32)
    # distinct ids (a repeated id may legitimately be selected twice), some -1 and some past n_c
    cand = torch.stack([(torch.randperm(n_max + 10, generator=G)[:n_cand] - 5).view(1, n_cand)
                        for _ in range(B)]).to(torch.int32)
    n_c = [2048, 1500]
    q_pos = np.array([[4 * 2048 - 1], [4 * 1500 - 1]], np.int64)
    idx, _, _ = csa.index_topk(qI.to(DEV), w.to(DEV), cache, torch.tensor(n_c, dtype=torch.int32, device=DEV),
                               torch.as_tensor(q_pos, device=DEV), ratio=4, k=k, cand=cand.to(DEV))
    torch.cuda.synchronize()
    for b in range(B):
        codes, scales, _ = _logical(cache, table, b, n_max)
        s_ref, ids = O.index_scores(f64(qI[b]), f64(w[b]), 1.0, codes, scales, 1.0, q_pos[b], n_c[b], 4,
                                    keys=cand[b].numpy())
        check_topk_row(idx[b, 0].cpu().numpy(), s_ref[0], ids[0], k, f"reindex b={b}")


@pytest.mark.parametrize("case", ["decode", "speculative5", "hca", "d128"])
def test_paged_attention(cuda_lib, case):
    csa = cuda_lib
    if case == "d128":
        B, Nq, H, d, d_r, n_max, k, ratio = 2, 4, 8, 128, 32, 1024, 64, 4
    elif case == "hca":
        B, Nq, H, d, d_r, n_max, k, ratio = 2, 1, 64, 512, 64, 600, 0, 128
    else:
        B, Nq, H, d, d_r, n_max, k, ratio = 3, (5 if case == "speculative5" else 1), 64, 512, 64, 2048, 512, 4
    page = 128
    Wn = 128 + Nq - 1
    G = gen(56)
    kv = normal((B, n_max, d), 1.0, G)
    cache, table = _paged(csa, B, n_max, d, d_r, page, seed=7)
    csa.pack_fp4(kv.to(DEV), cache)
    q = normal((B, Nq, H, d), 1.0, G)
    win = normal((B, Wn, d), 1.0, G)
    n_c = [n_max, n_max - 300, n_max][:B]
    t_last = [ratio * nc - 1 for nc in n_c]
    q_pos = np.array([[t - Nq + 1 + j for j in range(Nq)] for t in t_last], np.int64)
    win_pos0 = [int(q_pos[b, 0]) - 127 for b in range(B)]
    n_c_t = torch.tensor(n_c, dtype=torch.int32, device=DEV)
    qp = torch.as_tensor(q_pos, device=DEV)
    wp0 = torch.tensor(win_pos0, dtype=torch.int64, device=DEV)
    if case == "hca":
        out, lse = csa.hca_attn(q.to(DEV), qp, cache, n_c_t, win.to(DEV), wp0, ratio=ratio)
        idx = None
    else:
        idx = torch.stack([torch.stack([torch.randperm(n_max + 40, generator=G)[:k] - 20 for _ in range(Nq)])
                           for _ in range(B)]).to(torch.int32)
        out, lse = csa.sparse_attn(q.to(DEV), qp, cache, n_c_t, idx.to(DEV), win.to(DEV), wp0, ratio=ratio)
    torch.cuda.synchronize()
    for b in range(B):
        codes, scales, rope = _logical(cache, table, b, n_max)
        rows = O.entry_kv(codes, scales, rope, d - d_r, 1.0)
        if case == "hca":
            o_ref, l_ref = O.hca_attention(f64(q[b]), q_pos[b], rows, n_c[b], ratio, f64(win[b]), win_pos0[b], 128,
                                           d ** -0.5)
        else:
            o_ref, l_ref = O.attention(f64(q[b]), q_pos[b], rows, idx[b].numpy(), n_c[b], f64(win[b]), win_pos0[b],
                                       128, d ** -0.5)
        assert_close(f64(out[b]), o_ref, OUT_ATOL, OUT_RTOL, f"{case} out b={b}")
        assert_close(lse[b].cpu().numpy(), l_ref, LSE_ATOL, LSE_RTOL, f"{case} lse b={b}")


def test_paged_map_rejected_when_malformed(cuda_lib):
    """Page sizes off the 128-entry tile and tables too narrow for n_max are refused on the host."""
    csa = cuda_lib
    G = gen(57, DEV)
    src = normal((1, 10, 128), 1.0, G, DEV)
    bad = csa.PagedCache(1, 200, 128, 0, DEV, 100, 4, torch.zeros((1, 2), dtype=torch.int32))
    with pytest.raises(csa.CSAError, match="UNSUPPORTED"):
        csa.pack_fp4(src, bad)
    narrow = csa.PagedCache(1, 300, 128, 0, DEV, 128, 4, torch.zeros((1, 2), dtype=torch.int32))
    with pytest.raises(csa.CSAError, match="INVALID"):
        csa.pack_fp4(src, narrow)
