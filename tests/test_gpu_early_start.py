"""Early start inside a decode step (CSA_EARLY_START): the indexer streams the key tiles below the
newest entry while the compressor that appends that entry still runs, and attention runs each query's
window tile while the top-k still runs.  The step must give the same bits as without the option, and
the newest entry must be scored from the bytes the compressor wrote in the same step."""
import numpy as np
import pytest
import torch

from csa_workloads import CFG2, decode_inputs
from oracle import csa_oracle as O
from tests.cmp_utils import SCORE_RTOL, LSE_ATOL, LSE_RTOL, OUT_ATOL, OUT_RTOL, assert_close, check_topk_row, f64, \
    np_u8

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _layer(n_c, B, inp, early, fused=False):
    from compressed_sparse_attention_18_b200.layer import CSADecodeLayer, LayerShape
    s = CFG2
    ls = LayerShape(B=B, n_max=(n_c + 7) // 8 * 8, r=s.r, H=s.H, d=s.d, d_r=s.d_r, H_I=s.H_I, d_I=s.d_I, k=s.k, W=s.W)
    L = CSADecodeLayer(ls, DEV, early_start=early, fused_index=fused)
    L.load_history(inp["kv_src"], inp["kI_src"], n_c)
    L.win.copy_(inp["win_kv"])
    return L


def _run(L, inp, steps=3):
    for _ in range(steps):            # repeated steps: the same appended entry, the histogram reused
        out, lse, idx = L.step(inp["C"], inp["Z"], inp["b_pos"], inp["W_IK"], inp["q"], inp["q_I"], inp["w"])
    torch.cuda.synchronize()
    return out.clone(), lse.clone(), idx.clone()


# n_c: newest entry inside a partial 256-row tile, first row of a tile, last row of a tile, in the third
# tile (the cache capacity is n_c rounded up to 8 rows, as the tensor-core scorer needs a multiple of 4)
# fused: the early layer selects with the fused indexer + top-k (scores kept on chip); its score row is
# then recomputed by a separate scoring call on the same cache bytes, which must give the same bits
@pytest.mark.parametrize("fused", [False, True], ids=["split", "fused"])
@pytest.mark.parametrize("n_c,B", [(4096 + 36, 16), (4096 + 1, 16), (4096, 16), (700, 24)])
def test_early_start_same_bits_and_fresh_newest_entry(cuda_lib, n_c, B, fused):
    s = CFG2
    csa = cuda_lib
    inp = decode_inputs(s, seed=11, device=DEV, n_c=n_c, B=B)
    La = _layer(n_c, B, inp, early=True, fused=fused)
    Lb = _layer(n_c, B, inp, early=False)
    oa, la, ia = _run(La, inp)
    ob, lb, ib = _run(Lb, inp)
    if fused:
        csa.index_scores(inp["q_I"], inp["w"], La.ki, La.n_c, La.q_pos, La.scores, ratio=s.r)
        torch.cuda.synchronize()
    # scores are bit-identical; selections compare as sets (their order is unspecified, and it decides
    # the order in which attention sums the entries, so the two layers' outputs agree to rounding)
    assert torch.equal(La.scores[:, :n_c], Lb.scores[:, :n_c])
    assert torch.equal(torch.sort(ia, dim=-1).values, torch.sort(ib, dim=-1).values)
    assert_close(f64(oa), f64(ob), OUT_ATOL, OUT_RTOL, "out early vs not")
    # on one selection: the early plan (split 0 walks the window tile, then its entry tile) is
    # deterministic and agrees with the stage-by-stage plan (window in a split of its own) to rounding
    o1, l1 = csa.sparse_attn(inp["q"], La.q_pos, La.kv, La.n_c, ia, La.win, La.win_pos0, ratio=s.r, window=s.W,
                             early_start=True)
    o2, l2 = csa.sparse_attn(inp["q"], La.q_pos, La.kv, La.n_c, ia, La.win, La.win_pos0, ratio=s.r, window=s.W,
                             early_start=False)
    torch.cuda.synchronize()
    assert torch.equal(o1, oa) and torch.equal(l1, la)
    assert_close(f64(o1), f64(o2), OUT_ATOL, OUT_RTOL, "out early vs stage-by-stage plan")
    assert_close(l1.cpu().numpy(), l2.cpu().numpy(), LSE_ATOL, LSE_RTOL, "lse early vs stage-by-stage plan")
    assert torch.equal(La.kv.codes, Lb.kv.codes) and torch.equal(La.ki.codes, Lb.ki.codes)
    assert int(La.hist.abs().sum()) == 0 and int(Lb.hist.abs().sum()) == 0   # the top-k left the histogram clean
    t = int(La.q_pos[0, 0])
    for b in (0, B - 1):
        codes, scales = np_u8(La.ki.codes[b, :n_c]), np_u8(La.ki.scales[b, :n_c])
        sc, ids = O.index_scores(f64(inp["q_I"][b, 0])[None], f64(inp["w"][b, 0])[None], 1.0, codes, scales, 1.0,
                                 [t], n_c, s.r)
        got = La.scores[b, :n_c].cpu().numpy().astype(np.float64)
        assert sc.shape[1] == n_c and np.all(np.isfinite(sc[0]))
        rowmax = np.max(np.abs(sc[0]))
        assert_close(got, sc[0], SCORE_RTOL * rowmax, SCORE_RTOL, f"scores b={b}")
        # the newest entry's score comes from the freshly appended key (a stale row would score 0)
        assert sc[0][n_c - 1] != 0.0
        assert abs(got[n_c - 1] - sc[0][n_c - 1]) <= SCORE_RTOL * (abs(sc[0][n_c - 1]) + rowmax)
        check_topk_row(ia[b, 0].cpu().numpy(), sc[0], ids[0], s.k, f"top-k b={b}")
        rows = O.entry_kv(np_u8(La.kv.codes[b, :n_c]), np_u8(La.kv.scales[b, :n_c]), f64(La.kv.rope[b, :n_c]),
                          s.d_n, 1.0)
        o_ref, l_ref = O.attention(f64(inp["q"][b]), [t], rows, ia[b].cpu().numpy(), n_c, f64(La.win[b]),
                                   t - s.W + 1, s.W, s.d ** -0.5)
        assert_close(f64(oa[b]), o_ref, OUT_ATOL, OUT_RTOL, f"out b={b}")
        assert_close(la[b].cpu().numpy(), l_ref, LSE_ATOL, LSE_RTOL, f"lse b={b}")


def test_early_start_window_ragged_and_absent(cuda_lib):
    """Window CTAs with a partial window (early positions: fewer than 128 window rows) and an early
    call whose window is absent (Wn = 0: the option is ignored)."""
    csa = cuda_lib
    s = CFG2
    B, n_c = 4, 700
    inp = decode_inputs(s, seed=12, device=DEV, n_c=n_c, B=B)
    kv = csa.PackedCache(B, n_c, s.d, s.d_r, DEV, 1.0)
    csa.pack_fp4(inp["kv_src"], kv)
    n_ct = torch.full((B,), n_c, dtype=torch.int32, device=DEV)
    t = torch.tensor([[40], [127], [200], [4 * n_c - 1]], dtype=torch.int64, device=DEV)
    win_pos0 = torch.clamp(t[:, 0] - s.W + 1, min=0)
    idx = torch.stack([torch.randperm(n_c - 1, device=DEV)[: s.k] for _ in range(B)]).view(B, 1, s.k).int()
    for early in (True, False):
        o1, l1 = csa.sparse_attn(inp["q"], t, kv, n_ct, idx, inp["win_kv"], win_pos0, ratio=s.r, window=s.W,
                                 early_start=early)
        o0, l0 = csa.sparse_attn(inp["q"], t, kv, n_ct, idx, None, None, ratio=s.r, window=s.W, early_start=early)
        torch.cuda.synchronize()
        for b in range(B):
            rows = O.entry_kv(np_u8(kv.codes[b]), np_u8(kv.scales[b]), f64(kv.rope[b]), s.d_n, 1.0)
            tb = int(t[b, 0])
            o_ref, l_ref = O.attention(f64(inp["q"][b]), [tb], rows, idx[b].cpu().numpy(), n_c,
                                       f64(inp["win_kv"][b]), int(win_pos0[b]), s.W, s.d ** -0.5)
            assert_close(f64(o1[b]), o_ref, OUT_ATOL, OUT_RTOL, f"out b={b} early={early}")
            assert_close(l1[b].cpu().numpy(), l_ref, LSE_ATOL, LSE_RTOL, f"lse b={b} early={early}")
            o_ref, l_ref = O.attention(f64(inp["q"][b]), [tb], rows, idx[b].cpu().numpy(), n_c,
                                       np.zeros((0, s.d)), 0, s.W, s.d ** -0.5)
            assert_close(f64(o0[b]), o_ref, OUT_ATOL, OUT_RTOL, f"out no window b={b} early={early}")


def test_topk_early_start_same_selection(cuda_lib):
    """csa_topk with CSA_EARLY_START reads each row's positions before its wait: on rows of different
    lengths and visibilities it selects exactly what the plain call selects (and leaves the histogram
    rows it read zero), the selection being the oracle's."""
    csa = cuda_lib
    from csa_workloads import gen, normal
    G = gen(31)
    B, n, k = 5, 9000, 512
    n_c = [9000, 513, 1, 4000, 8999]
    q_pos = [4 * 9000 - 1, 4 * 513 - 1, 3, 4 * 3000 + 1, 4 * 8999 - 1]
    kI = normal((B, n, 128), 1.0, G)
    qI = normal((B, 1, 8, 128), 1.0, G).to(DEV)
    w = normal((B, 1, 8), 8 ** -0.5, G, dtype=torch.float32).to(DEV)
    kc = csa.PackedCache(B, n, 128, 0, DEV, 1.0)
    csa.pack_fp4(kI.to(DEV), kc)
    n_c_t = torch.tensor(n_c, dtype=torch.int32, device=DEV)
    q_pos_t = torch.tensor(q_pos, dtype=torch.int64, device=DEV).view(B, 1)
    scores = torch.empty((B, n), dtype=torch.float32, device=DEV)
    h1 = torch.zeros((B, 4096), dtype=torch.int32, device=DEV)
    csa.index_scores(qI, w, kc, n_c_t, q_pos_t, scores, ratio=4, hist=h1, k=k)
    h2 = h1.clone()
    i1, _, _ = csa.topk(scores, kc, n_c_t, q_pos_t, B=B, Nq=1, ratio=4, k=k, hist=h1)
    i2, _, _ = csa.topk(scores, kc, n_c_t, q_pos_t, B=B, Nq=1, ratio=4, k=k, hist=h2, early_start=True)
    torch.cuda.synchronize()
    assert int(h1.abs().sum()) == 0 and int(h2.abs().sum()) == 0
    assert torch.equal(i1.sort(dim=-1).values, i2.sort(dim=-1).values)
    for b in range(B):
        codes, scales, _ = O.pack_fp4(f64(kI[b]), 0, 1.0)
        s_ref, ids = O.index_scores(f64(qI[b].cpu()), f64(w[b].cpu()), 1.0, codes, scales, 1.0,
                                    q_pos_t[b].cpu().numpy(), n_c[b], 4)
        check_topk_row(i2[b, 0].cpu().numpy(), s_ref[0], ids[0], k, f"early top-k b={b}")
