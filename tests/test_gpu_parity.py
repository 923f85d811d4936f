"""GPU parity: every stage of the CUDA path (through the C ABI) against the CPU oracle on the same
seeded inputs and the same upstream bytes, at sizes the oracle finishes in seconds that still span
several tiles and a ragged tail, plus the edge cases (empty / ragged / fully masked / ties / k >= n)."""
import numpy as np
import pytest
import torch

from csa_workloads import CFG1, gen, normal, small_layer_inputs
from oracle import csa_oracle as O
from tests.cmp_utils import (LSE_ATOL, LSE_RTOL, OUT_ATOL, OUT_RTOL, SCORE_RTOL, assert_close,
                             check_topk_row, f64, np_u8)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def bf16_bits(t):
    return t.detach().to("cpu").view(torch.int16).numpy()


# ------------------------------------------------------------------------------------------ pack

@pytest.mark.parametrize("d,d_r,g", [(512, 64, 1.0), (128, 32, 2.0 ** -4), (128, 0, 1.0), (64, 0, 0.5)])
def test_pack_bit_exact(cuda_lib, d, d_r, g):
    csa = cuda_lib
    B, n, n_max = 3, 37, 60
    G = gen(11)
    x = torch.randn((B, n, d), generator=G)
    x[0, 0] = 0.0                                        # all-zero row -> zero scales
    x[0, 1] *= 1e-7                                      # scales underflow toward E4M3 subnormals / zero
    x[0, 2] *= 1e4                                       # scales saturate at 448
    x[1, 3, :32] = torch.tensor(O.e2m1_decode(np.arange(32) % 16) * 0.75)   # exactly representable block
    x[2, 4, 1::2] = -1e-3                                # rounds to -0 -> +0
    src = x.to(torch.bfloat16)
    cache = csa.PackedCache(B, n_max, d, d_r, DEV, g)
    row0 = torch.tensor([0, 5, n_max - n], dtype=torch.int32, device=DEV)
    csa.pack_fp4(src.to(DEV), cache, row0)
    torch.cuda.synchronize()
    for b in range(B):
        codes, scales, rope = O.pack_fp4(f64(src[b]), d_r, g)
        r0 = int(row0[b])
        assert np.array_equal(np_u8(cache.codes[b, r0:r0 + n]), codes), f"codes b={b}"
        assert np.array_equal(np_u8(cache.scales[b, r0:r0 + n]), scales), f"scales b={b}"
        if d_r:
            assert np.array_equal(bf16_bits(cache.rope[b, r0:r0 + n]), bf16_bits(src[b, :, d - d_r:]))
    # rows outside [row0, row0 + n) untouched
    assert int(cache.codes[0, n:].abs().sum()) == 0


# ------------------------------------------------------------------------------------ compressor

def _ulp_close(got, ref, what):
    rms = float(np.sqrt(np.mean(ref ** 2))) or 1.0
    assert_close(got, ref, 1e-3 * rms, 2.0 ** -7 * 1.01, what)


def test_compress_projection_mode_cfg1(cuda_lib):
    csa = cuda_lib
    inp = small_layer_inputs(CFG1, seed=0)
    t = {k: v.to(DEV) for k, v in inp.items()}
    c, kI, C, Z = csa.compress(x=t["x"], W_kv=t["W_kv"], W_g=t["W_g"], b_pos=t["b_pos"], ratio=4,
                               d_rope=CFG1.d_r, rope_theta=10000.0, W_IK=t["W_IK"])
    torch.cuda.synchronize()
    x = f64(inp["x"][0])
    _ulp_close(f64(C[0]), O.project(x, f64(inp["W_kv"])), "C")
    _ulp_close(f64(Z[0]), O.project(x, f64(inp["W_g"])), "Z")
    # pooling and the index-key projection on the same upstream bytes
    c_ref = O.compress_pool(f64(C[0]), f64(Z[0]), f64(inp["b_pos"]), 4, CFG1.d_r, 10000.0, 0)
    _ulp_close(f64(c[0]), c_ref, "c")
    _ulp_close(f64(kI[0]), O.index_key(f64(c[0]), f64(inp["W_IK"])), "k_I")


@pytest.mark.parametrize("r,T,d,d_r,pos0", [(4, 4 * 97 + 3, 512, 64, 4 * 1000), (128, 128 * 9 + 17, 512, 64, 0),
                                            (1, 33, 128, 32, 7), (128, 128 + 5, 512, 64, 128 * 7),
                                            (16, 16 * 3 + 2, 128, 32, 0), (16, 16 + 3, 128, 32, 16 * 5)])
def test_compress_pooling_mode(cuda_lib, r, T, d, d_r, pos0):
    csa = cuda_lib
    G = gen(3)
    B = 2
    C = normal((B, T, d), 1.0, G)
    Z = normal((B, T, d), 1.0, G)
    b_pos = normal((r, d), 0.1, G, dtype=torch.float32)
    W_IK = normal((d, 128), d ** -0.5, G)
    p0 = torch.tensor([pos0, pos0 + 8 * r], dtype=torch.int64)
    n = T // r
    # fused FP4 append into caches at per-sequence row offsets (same bytes as csa_pack_fp4)
    kv = csa.PackedCache(B, n + 9, d, d_r, DEV, 0.5)
    ki = csa.PackedCache(B, n + 9, 128, 0, DEV)
    row0 = torch.tensor([0, 9], dtype=torch.int32, device=DEV)
    c, kI, _, _ = csa.compress(C=C.to(DEV), Z=Z.to(DEV), b_pos=b_pos.to(DEV), ratio=r, d_rope=d_r,
                               rope_theta=10000.0, pos0=p0.to(DEV), W_IK=W_IK.to(DEV), kv_cache=kv, ki_cache=ki,
                               row0=row0)
    torch.cuda.synchronize()
    for b in range(B):
        ref = O.compress_pool(f64(C[b]), f64(Z[b]), f64(b_pos), r, d_r, 10000.0, int(p0[b]))
        assert c.shape[1] == n
        _ulp_close(f64(c[b]), ref, f"c b={b}")
        _ulp_close(f64(kI[b]), O.index_key(f64(c[b]), f64(W_IK)), f"k_I b={b}")
        r0 = int(row0[b])
        codes, scales, rope = O.pack_fp4(f64(c[b]), d_r, 0.5)
        assert np.array_equal(np_u8(kv.codes[b, r0:r0 + n]), codes) and np.array_equal(np_u8(kv.scales[b, r0:r0 + n]), scales)
        assert np.array_equal(bf16_bits(kv.rope[b, r0:r0 + n]), bf16_bits(c[b, :, d - d_r:]))
        kc, ks, _ = O.pack_fp4(f64(kI[b]), 0, 1.0)
        assert np.array_equal(np_u8(ki.codes[b, r0:r0 + n]), kc) and np.array_equal(np_u8(ki.scales[b, r0:r0 + n]), ks)


# ---------------------------------------------------------------------------------------- indexer

def _index_case(csa, *, B, n_max, n_c, d_I, H_I, Nq, q_pos, k, g_q=1.0, g_k=1.0, key_std=1.0, seed=0,
                cand=None, pool_blocks=0, identical_keys=False, onchip=False):
    G = gen(seed)
    kI = normal((B, n_max, d_I), key_std, G)
    if identical_keys:
        kI[:] = kI[:, :1]
    qI = normal((B, Nq, H_I, d_I), 1.0, G)
    w = normal((B, Nq, H_I), H_I ** -0.5, G, dtype=torch.float32)
    kc = csa.PackedCache(B, n_max, d_I, 0, DEV, g_k)
    csa.pack_fp4(kI.to(DEV), kc)
    n_c_t = torch.tensor(n_c, dtype=torch.int32)
    q_pos_t = torch.tensor(q_pos, dtype=torch.int64).view(B, Nq)
    idx, sc, pool = csa.index_topk(qI.to(DEV), w.to(DEV), kc, n_c_t.to(DEV), q_pos_t.to(DEV), ratio=4, k=k, g_q=g_q,
                                   cand=cand.to(DEV) if cand is not None else None, pool_blocks=pool_blocks,
                                   want_scores=True, onchip=onchip)
    torch.cuda.synchronize()
    swaps = 0
    for b in range(B):
        codes, scales, _ = O.pack_fp4(f64(kI[b]), 0, g_k)
        assert np.array_equal(np_u8(kc.codes[b]), codes)
        keys = None if cand is None else cand[b].numpy()
        s_ref, ids = O.index_scores(f64(qI[b]), f64(w[b]), g_q, codes, scales, g_k, q_pos_t[b].numpy(), n_c[b], 4,
                                    keys=keys)
        gi = idx[b].cpu().numpy()
        gs = sc[b].cpu().numpy()
        for q in range(Nq):
            swaps += check_topk_row(gi[q], s_ref[q], ids[q], k, f"b={b} q={q}")
            # scores the kernel returns for its selection match the oracle's for the same ids
            score_of = dict(zip(ids[q].tolist(), s_ref[q].tolist()))
            sel = gi[q] >= 0
            ref = np.array([score_of[i] for i in gi[q][sel]])
            rowmax = np.max(np.abs(s_ref[q][np.isfinite(s_ref[q])])) if np.any(np.isfinite(s_ref[q])) else 0
            assert_close(gs[q][sel], ref, SCORE_RTOL * rowmax, SCORE_RTOL, f"scores b={b} q={q}")
            assert np.all(np.isneginf(gs[q][~sel]))
        if pool_blocks:
            pr, blk = O.hierarchical_pool(s_ref, pool_blocks, 8)
            gp = pool[b].cpu().numpy().reshape(Nq, pool_blocks, 8)
            for q in range(Nq):
                # each GPU block: 8 consecutive ids (or -1 where not visible); block set vs oracle's
                got_blocks = set()
                for j in range(pool_blocks):
                    row = gp[q, j]
                    ok = row[row >= 0]
                    if len(ok) == 0:
                        continue
                    bid = int(ok[0]) // 8
                    got_blocks.add(bid)
                    for e in range(8):
                        i = bid * 8 + e
                        want = i if (i < s_ref.shape[1] and np.isfinite(s_ref[q, i])) else -1
                        assert row[e] == want
                bscore = {int(bb): np.max(s_ref[q, bb * 8: bb * 8 + 8]) for bb in range(s_ref.shape[1] // 8 + 1)
                          if bb * 8 < s_ref.shape[1]}
                ids_b = np.array(sorted(bscore)); sc_b = np.array([bscore[i] for i in ids_b])
                gsel = np.array(sorted(got_blocks) + [-1] * (pool_blocks - len(got_blocks)))
                swaps += check_topk_row(gsel, sc_b, ids_b, pool_blocks, f"pool b={b} q={q}")
    return idx, swaps


def test_index_cfg1_small_layer(cuda_lib):
    q_pos = list(range(4080, 4096))
    _index_case(cuda_lib, B=1, n_max=1024, n_c=[1024], d_I=64, H_I=4, Nq=16, q_pos=q_pos, k=64,
                g_q=1.0, g_k=2.0 ** -4, key_std=0.03)


ONCHIP = pytest.mark.parametrize("onchip", [False, True], ids=["split", "onchip"])


@ONCHIP
def test_index_decode_ragged(cuda_lib, onchip):
    n_c = [4096, 1000, 37, 2048]
    q_pos = [4 * 4096 - 1, 4 * 1000 - 1, 4 * 37 - 1, 4 * 500 + 2]   # last: only 500 visible
    _index_case(cuda_lib, B=4, n_max=4096, n_c=n_c, d_I=128, H_I=8, Nq=1, q_pos=q_pos, k=512, seed=1, onchip=onchip)


def test_index_onchip_full_row_and_k_above_visible(cuda_lib):
    """The on-chip top-k at its largest row (32768 keys: 16 tiles per CTA of the cluster) and with
    k larger than the visible entries (slots past k_eff are -1)."""
    n = 32768
    _index_case(cuda_lib, B=2, n_max=n, n_c=[n, 300], d_I=128, H_I=8, Nq=1, q_pos=[4 * n - 1, 4 * 300 - 1],
                k=512, seed=13, onchip=True)


def test_index_prefill_causal_multi_query(cuda_lib):
    q_pos = list(range(1000, 1048))                       # 48 queries: one full 32-query tile + a tail
    _index_case(cuda_lib, B=1, n_max=512, n_c=[300], d_I=128, H_I=8, Nq=48, q_pos=q_pos, k=64, seed=2)


def test_index_multiquery_rows_histogram_pass(cuda_lib):
    """Multi-query rows longer than 8192 keys (speculative positions): the selection counts each row's
    visible scores in a histogram pass, then selects like a decode row.  Positions of one sequence see
    different prefixes (9000 to 20000 keys, some ending inside a 4096-score slice)."""
    q_pos = [4 * 20000 - 1, 4 * 12000 + 1, 4 * 9000 + 3, 4 * 15000 - 1, 4 * 10000, 4 * 14000 + 2]
    _index_case(cuda_lib, B=2, n_max=20000, n_c=[20000, 15000], d_I=128, H_I=8, Nq=3, q_pos=q_pos, k=512, seed=61)


def test_index_tournament_long_row(cuda_lib):
    n = 40000                                             # > one 32768-column top-k chunk
    _index_case(cuda_lib, B=2, n_max=n, n_c=[n, n - 123], d_I=128, H_I=8, Nq=1, q_pos=[4 * n - 1, 4 * n - 1],
                k=256, seed=3)


def test_index_long_rows_histogram_pass(cuda_lib):
    # rows of 3 and 4 top-k chunks: the histogram pass selects them (segment CTAs, the last one resolves
    # the boundary bin); the second row's visible length ends inside its third chunk
    n = 4 * 32768 - 100
    _index_case(cuda_lib, B=2, n_max=n, n_c=[n, 70000], d_I=128, H_I=8, Nq=1, q_pos=[4 * n - 1, 4 * 69000 + 1],
                k=2048, seed=10)


def test_index_long_row_boundary_overflow_falls_back(cuda_lib):
    # 70000 equal scores: the boundary bin holds more candidates than the row buffer, the tournament
    # selects the row instead; the smallest ids must win
    idx, swaps = _index_case(cuda_lib, B=1, n_max=70000, n_c=[70000], d_I=128, H_I=8, Nq=1, q_pos=[280000], k=10,
                             seed=11, identical_keys=True)
    assert swaps == 0 and sorted(idx[0, 0].tolist()) == list(range(10))


def test_topk_long_row_stale_histogram(cuda_lib):
    # split calls: the histogram is scored into twice before the top-k reads it (counts no longer match
    # the scores), so the long rows fall back to the tournament; the selection is still exact
    csa = cuda_lib
    G = gen(12)
    B, n, k = 2, 50000, 300
    kI = normal((B, n, 128), 1.0, G)
    qI = normal((B, 1, 8, 128), 1.0, G)
    w = normal((B, 1, 8), 8 ** -0.5, G, dtype=torch.float32)
    kc = csa.PackedCache(B, n, 128, 0, DEV, 1.0)
    csa.pack_fp4(kI.to(DEV), kc)
    n_c = torch.tensor([n, n - 5000], dtype=torch.int32, device=DEV)
    q_pos = torch.tensor([[4 * n - 1], [4 * (n - 5000) - 1]], dtype=torch.int64, device=DEV)
    scores = torch.empty((B, n), dtype=torch.float32, device=DEV)
    hist = torch.zeros((B, 4096), dtype=torch.int32, device=DEV)
    for _ in range(2):
        csa.index_scores(qI.to(DEV), w.to(DEV), kc, n_c, q_pos, scores, ratio=4, hist=hist, k=k)
    idx, sc, _ = csa.topk(scores, kc, n_c, q_pos, B=B, Nq=1, ratio=4, k=k, hist=hist, want_scores=True)
    torch.cuda.synchronize()
    assert int(hist.abs().sum()) == 0                     # the top-k left the histogram rows it read zero
    for b in range(B):
        codes, scales, _ = O.pack_fp4(f64(kI[b]), 0, 1.0)
        s_ref, ids = O.index_scores(f64(qI[b]), f64(w[b]), 1.0, codes, scales, 1.0, q_pos[b].cpu().numpy(),
                                    int(n_c[b]), 4)
        check_topk_row(idx[b, 0].cpu().numpy(), s_ref[0], ids[0], k, f"stale histogram b={b}")


def test_index_reindex_candidates(cuda_lib):
    G = gen(5)
    B, Nq, n_max, n_cand = 2, 2, 3000, 2048
    cand = torch.randint(-1, n_max + 50, (B, Nq, n_cand), generator=G, dtype=torch.int32)
    for b in range(B):
        for q in range(Nq):                               # distinct ids (a previous layer's selection)
            cand[b, q] = torch.randperm(n_max + 50, generator=G)[:n_cand].to(torch.int32) - 1
    _index_case(cuda_lib, B=B, n_max=n_max, n_c=[n_max, 2500], d_I=128, H_I=8, Nq=Nq,
                q_pos=[4 * n_max - 1, 4 * 2000, 4 * 2500 - 1, 4 * 100], k=512, seed=5, cand=cand)


def test_index_hierarchical_pool(cuda_lib):
    _index_case(cuda_lib, B=2, n_max=8192, n_c=[8192, 5000], d_I=128, H_I=8, Nq=1,
                q_pos=[4 * 8192 - 1, 4 * 4000 + 1], k=128, seed=6, pool_blocks=64)


@ONCHIP
def test_index_exact_ties_take_smallest_ids(cuda_lib, onchip):
    idx, swaps = _index_case(cuda_lib, B=1, n_max=64, n_c=[64], d_I=128, H_I=8, Nq=1, q_pos=[255], k=10, seed=7,
                             identical_keys=True, onchip=onchip)
    assert swaps == 0
    assert sorted(idx[0, 0].tolist()) == list(range(10))


@ONCHIP
def test_index_exact_ties_overflow_the_boundary_buffer(cuda_lib, onchip):
    # 20000 equal scores: the histogram's boundary bin holds more candidates than the selection buffer,
    # so the row takes the full selection path; the smallest ids must still win
    idx, swaps = _index_case(cuda_lib, B=1, n_max=20000, n_c=[20000], d_I=128, H_I=8, Nq=1, q_pos=[80000], k=10,
                             seed=9, identical_keys=True, onchip=onchip)
    assert swaps == 0 and sorted(idx[0, 0].tolist()) == list(range(10))


def test_index_k_larger_than_visible(cuda_lib):
    idx, _ = _index_case(cuda_lib, B=2, n_max=256, n_c=[256, 256], d_I=64, H_I=4, Nq=1, q_pos=[4 * 20 - 1, 2],
                         k=100, seed=8)
    assert sorted(idx[0, 0].tolist())[-20:] == list(range(20)) and (idx[0, 0] == -1).sum() == 80
    assert (idx[1, 0] == -1).all()                        # t = 2: nothing visible yet


# -------------------------------------------------------------------------------------- attention

def _attn_case(csa, *, B, Nq, H, d, d_r, n_max, n_c, q_pos, k=0, Wn=128, win_pos0=None, hca=False, ratio=4,
               seed=0, g=1.0, q_scale=1.0, rope_theta=0.0, win_fp8=False, early_start=False, cluster=False):
    """win_fp8: the window rows are FP8-packed on the GPU (csa_pack_fp8_window) and the oracle attends over
    its own FP8 pack of the same bf16 rows, dequantised (the pack itself is checked bit-exact elsewhere)."""
    G = gen(seed)
    kv = normal((B, n_max, d), 1.0, G)
    q = normal((B, Nq, H, d), q_scale, G)
    win = normal((B, Wn, d), 1.0, G) if Wn else None
    cache = csa.PackedCache(B, n_max, d, d_r, DEV, g)
    csa.pack_fp4(kv.to(DEV), cache)
    q_pos_t = torch.tensor(q_pos, dtype=torch.int64).view(B, Nq)
    if win_pos0 is None:
        win_pos0 = [int(q_pos_t[b].max()) - Wn + 1 for b in range(B)]
    wp0 = torch.tensor(win_pos0, dtype=torch.int64)
    n_c_t = torch.tensor(n_c, dtype=torch.int32)
    idx = None
    if not hca:
        idx = torch.empty((B, Nq, k), dtype=torch.int32)
        for b in range(B):
            for qq in range(Nq):
                perm = torch.randperm(n_max + 40, generator=G)[:k].to(torch.int32) - 20   # some < 0, some >= n_c
                idx[b, qq] = perm
    win_arg = win.to(DEV) if win is not None else None
    if win is not None and win_fp8:
        win_arg = csa.Fp8Window(B, Wn, d, d_r, DEV)
        csa.pack_fp8_window(win.to(DEV), win_arg)
    if hca:
        out, lse = csa.hca_attn(q.to(DEV), q_pos_t.to(DEV), cache, n_c_t.to(DEV), win_arg,
                                wp0.to(DEV) if win is not None else None, ratio=ratio, out_rope_theta=rope_theta)
    else:
        out, lse = csa.sparse_attn(q.to(DEV), q_pos_t.to(DEV), cache, n_c_t.to(DEV), idx.to(DEV), win_arg,
                                   wp0.to(DEV) if win is not None else None, ratio=ratio, out_rope_theta=rope_theta,
                                   early_start=early_start, cluster=cluster)
    torch.cuda.synchronize()
    scale = d ** -0.5
    for b in range(B):
        codes, scales, rope = O.pack_fp4(f64(kv[b]), d_r, g)
        rows = O.entry_kv(codes, scales, rope, d - d_r, g)
        wb = f64(win[b]) if win is not None else np.zeros((0, d))
        lse_extra = 0.0
        if win is not None and win_fp8:
            wc, ws, wr = O.pack_fp8_window(wb, d_r)
            wb = O.dequant_fp8_window(wc, ws, wr)
            # the kernel feeds bf16(e4m3 * scale) to the tensor cores: each window key element carries a
            # rounding of at most 2^-9 relative, so a window logit moves by at most
            # scale * 2^-9 * sum_e |q_e K_e|, and lse (1-Lipschitz in the logits) by at most the largest of those
            qa = np.abs(f64(q[b]))                                   # [Nq, H, d]
            lse_extra = scale * 2.0 ** -9 * float(np.max(qa @ np.abs(wb).T)) if len(wb) else 0.0
        if hca:
            o_ref, l_ref = O.hca_attention(f64(q[b]), q_pos_t[b].numpy(), rows, n_c[b], ratio, wb, win_pos0[b], 128,
                                           scale, out_rope_theta=rope_theta, d_rope=d_r)
        else:
            o_ref, l_ref = O.attention(f64(q[b]), q_pos_t[b].numpy(), rows, idx[b].numpy(), n_c[b], wb, win_pos0[b],
                                       128, scale, out_rope_theta=rope_theta, d_rope=d_r)
        assert_close(f64(out[b]), o_ref, OUT_ATOL, OUT_RTOL, f"out b={b}")
        assert_close(lse[b].cpu().numpy(), l_ref, LSE_ATOL + lse_extra, LSE_RTOL, f"lse b={b}")
    return out, lse


@pytest.mark.parametrize("k,Wn", [(512, 128), (64, 0)])   # split partials + merge; one tile, no merge
def test_attn_inverse_rope_epilogue(cuda_lib, k, Wn):
    n = 4096
    _attn_case(cuda_lib, B=2, Nq=1, H=64, d=512, d_r=64, n_max=n, n_c=[n, n - 7], q_pos=[4 * n - 1, 4 * n - 30],
               k=k, Wn=Wn, seed=31, rope_theta=10000.0)


def test_attn_inverse_rope_epilogue_d128_and_hca(cuda_lib):
    q_pos = list(range(4080, 4096))
    _attn_case(cuda_lib, B=1, Nq=16, H=8, d=128, d_r=32, n_max=1024, n_c=[1024], q_pos=q_pos, k=64, seed=32,
               rope_theta=10000.0)
    _attn_case(cuda_lib, B=2, Nq=1, H=64, d=512, d_r=64, n_max=300, n_c=[300, 150],
               q_pos=[128 * 300 - 1, 128 * 150 + 5], hca=True, ratio=128, seed=33, rope_theta=10000.0)


@pytest.mark.parametrize("B", [80, 300])   # a CTA per query; 300 > 148 queries: the persistent kernel
def test_attn_tiles_per_cta_with_rescale(cuda_lib, B):
    """Enough rows that each tensor-core CTA walks two 128-key tiles of its query; the second tile's
    entries have 4x the norm of the first's, so every head's running max jumps past the lazy-rescale
    slack and the accumulated O and l are rescaled before the second tile is added.  With 300 queries
    one persistent CTA per SM walks two or three queries back to back (the rescale flag and the running
    max and sum start afresh for each)."""
    csa = cuda_lib
    H, d, d_r, n_max, k = 64, 512, 64, 512, 256
    G = gen(21)
    kv = normal((B, n_max, d), 1.0, G)
    kv[:, n_max // 2:] *= 4.0
    q = normal((B, 1, H, d), 1.0, G)
    cache = csa.PackedCache(B, n_max, d, d_r, DEV, 1.0)
    csa.pack_fp4(kv.to(DEV), cache)
    t = 4 * n_max - 1
    q_pos = torch.full((B, 1), t, dtype=torch.int64)
    n_c = torch.full((B,), n_max, dtype=torch.int32)
    idx = torch.empty((B, 1, k), dtype=torch.int32)
    for b in range(B):
        lo = torch.randperm(n_max // 2, generator=G)[:k // 2]
        hi = torch.randperm(n_max // 2, generator=G)[:k // 2] + n_max // 2
        idx[b, 0] = torch.cat([lo, hi]).to(torch.int32)       # tile 0: small keys, tile 1: large keys
    out, lse = csa.sparse_attn(q.to(DEV), q_pos.to(DEV), cache, n_c.to(DEV), idx.to(DEV), None, None, ratio=4)
    torch.cuda.synchronize()
    scale = d ** -0.5
    for b in range(0, B, 7):
        codes, scales, rope = O.pack_fp4(f64(kv[b]), d_r, 1.0)
        rows = O.entry_kv(codes, scales, rope, d - d_r, 1.0)
        o_ref, l_ref = O.attention(f64(q[b]), q_pos[b].numpy(), rows, idx[b].numpy(), n_max, np.zeros((0, d)), 0,
                                   128, scale)
        # P enters the P.V product as bf16 (relative rounding <= 2^-9), so an output element can be off by
        # 2^-9 * max |v| over the query's keys; the absolute tolerance 1e-2 is that bound for unit-scale
        # entries (|v| <~ 5), and these entries are scaled by 4
        atol = max(OUT_ATOL, 2.0 ** -9 * float(np.max(np.abs(rows[idx[b, 0].numpy()]))))
        assert_close(f64(out[b]), o_ref, atol, OUT_RTOL, f"out b={b}")
        assert_close(lse[b].cpu().numpy(), l_ref, LSE_ATOL, LSE_RTOL, f"lse b={b}")


def test_attn_persistent_result_independent_of_unit_assignment(cuda_lib):
    """A query's result does not depend on which persistent CTA walked it or on the units before it (the
    running max and sum, the accumulator and Q are reset per unit): 300 queries in one call (2-3 units per
    CTA) against the same queries 150 per call (1-2 per CTA), bit for bit.  Three tiles per query (small
    entries, 4x entries forcing a rescale, then the window), ids with absent entries."""
    csa = cuda_lib
    B, H, d, d_r, n_max, k, Wn = 300, 64, 512, 64, 512, 256, 128
    G = gen(22)
    kv = normal((B, n_max, d), 1.0, G)
    kv[:, n_max // 2:] *= 4.0
    q = normal((B, 1, H, d), 1.0, G).to(DEV)
    win = normal((B, Wn, d), 1.0, G).to(DEV)
    t = 4 * n_max - 1
    q_pos = torch.full((B, 1), t, dtype=torch.int64, device=DEV)
    wp0 = torch.full((B,), t - Wn + 1, dtype=torch.int64, device=DEV)
    n_c = torch.full((B,), n_max, dtype=torch.int32, device=DEV)
    idx = torch.empty((B, 1, k), dtype=torch.int32)
    for b in range(B):
        lo = torch.randperm(n_max // 2, generator=G)[:k // 2]
        hi = torch.randperm(n_max // 2, generator=G)[:k // 2] + n_max // 2
        idx[b, 0] = torch.cat([lo, hi]).to(torch.int32)
    idx[::5, 0, ::7] = -1
    idx = idx.to(DEV)
    cache = csa.PackedCache(B, n_max, d, d_r, DEV, 1.0)
    csa.pack_fp4(kv.to(DEV), cache)
    out, lse = csa.sparse_attn(q, q_pos, cache, n_c, idx, win, wp0, ratio=4)
    for b0 in range(0, B, 150):
        sl = slice(b0, b0 + 150)
        sub = csa.PackedCache(150, n_max, d, d_r, DEV, 1.0)
        csa.pack_fp4(kv[sl].to(DEV), sub)
        o2, l2 = csa.sparse_attn(q[sl], q_pos[sl], sub, n_c[sl], idx[sl], win[sl].contiguous(), wp0[sl], ratio=4)
        torch.cuda.synchronize()
        assert torch.equal(o2, out[sl]), f"out of queries {b0}..{b0 + 149} differs between the two calls"
        assert torch.equal(l2, lse[sl]), f"lse of queries {b0}..{b0 + 149} differs between the two calls"


def test_attn_cfg1_shapes(cuda_lib):
    q_pos = list(range(4080, 4096))
    _attn_case(cuda_lib, B=1, Nq=16, H=8, d=128, d_r=32, n_max=1024, n_c=[1024], q_pos=q_pos, k=64, Wn=143,
               g=2.0 ** -4, seed=1)


def test_attn_cfg1_peaked_queries(cuda_lib):
    q_pos = list(range(4080, 4096))
    _attn_case(cuda_lib, B=1, Nq=16, H=8, d=128, d_r=32, n_max=1024, n_c=[1024], q_pos=q_pos, k=64, Wn=143,
               seed=2, q_scale=128 ** 0.5 / 4)


def test_attn_decode_d512(cuda_lib):
    n_c = [2048, 700, 2048]
    q_pos = [4 * 2048 - 1, 4 * 700 - 1, 4 * 1500 + 3]
    _attn_case(cuda_lib, B=3, Nq=1, H=64, d=512, d_r=64, n_max=2048, n_c=n_c, q_pos=q_pos, k=512, seed=3)


def test_attn_no_window_and_partial_window(cuda_lib):
    _attn_case(cuda_lib, B=2, Nq=1, H=64, d=512, d_r=64, n_max=600, n_c=[600, 600], q_pos=[2399, 2399], k=100,
               Wn=0, seed=4)
    # window buffer that starts after t - W + 1 (only part of the window held) and a query near the start
    _attn_case(cuda_lib, B=2, Nq=1, H=64, d=512, d_r=64, n_max=64, n_c=[64, 2], q_pos=[255, 9], k=64, Wn=50,
               win_pos0=[206, 0], seed=5)


def test_attn_many_queries_single_split(cuda_lib):
    q_pos = list(range(3000, 3000 + 150))                # >= 148 rows: the direct-write path
    _attn_case(cuda_lib, B=1, Nq=150, H=64, d=512, d_r=64, n_max=800, n_c=[800], q_pos=q_pos, k=64, Wn=300,
               seed=6)


def test_attn_persistent_ragged_queries(cuda_lib):
    """400 queries (more than the SMs, one CTA each): the persistent kernel walks 2-3 queries per CTA.
    Scattered positions against a 160-row window buffer give key lists of 3 or 4 tiles (window empty,
    partial or full), and the ids include absent (-1, out of range) entries."""
    rng = np.random.default_rng(50)
    B, Nq = 2, 200
    q_pos = np.sort(rng.integers(3000, 4000, size=(B, Nq)), axis=1)
    _attn_case(cuda_lib, B=B, Nq=Nq, H=64, d=512, d_r=64, n_max=1000, n_c=[1000, 800], q_pos=q_pos.ravel().tolist(),
               k=384, Wn=160, seed=52)


@pytest.mark.parametrize("Wn", [0, 128])
def test_attn_persistent_hca_variable_tiles(cuda_lib, Wn):
    """HCA over 400 queries: visible counts from 0 to 600 entries (0 to 5 tiles, plus the window).
    Without a window the queries before the first complete group have no keys at all; the persistent
    CTAs skip them between queries with keys (zero output, lse = -inf)."""
    rng = np.random.default_rng(53)
    B, Nq = 2, 200
    q_pos = rng.integers(0, 128 * 620, size=(B, Nq))
    q_pos[0, ::9] = rng.integers(0, 127, size=len(q_pos[0, ::9]))
    out, lse = _attn_case(cuda_lib, B=B, Nq=Nq, H=64, d=512, d_r=64, n_max=600, n_c=[600, 350],
                          q_pos=q_pos.ravel().tolist(), hca=True, ratio=128, Wn=Wn,
                          win_pos0=[int(q_pos[b].max()) - Wn + 1 for b in range(B)] if Wn else None, seed=54)
    if Wn == 0:
        empty = torch.as_tensor(q_pos < 127)
        assert bool(torch.all(out.cpu()[empty] == 0)) and bool(torch.all(torch.isneginf(lse.cpu()[empty])))


@pytest.mark.parametrize("Wn", [0, 128])
def test_attn_persistent_hca_split_units(cuda_lib, Wn):
    """HCA over 160 queries of up to 8-9 tiles (1024 entries, plus the window): more queries than SMs but
    few tiles each, so the persistent kernel deals (query, split) units of 2-3 tiles to the SMs and the
    merge combines them.  Visible counts from 0 to 1024 entries: units past a query's keys write empty
    partials, and a query without any keys comes out zero with lse = -inf."""
    rng = np.random.default_rng(55)
    B, Nq = 2, 80
    q_pos = rng.integers(0, 128 * 1100, size=(B, Nq))
    q_pos[0, ::7] = rng.integers(0, 127, size=len(q_pos[0, ::7]))
    out, lse = _attn_case(cuda_lib, B=B, Nq=Nq, H=64, d=512, d_r=64, n_max=1024, n_c=[1024, 700],
                          q_pos=q_pos.ravel().tolist(), hca=True, ratio=128, Wn=Wn,
                          win_pos0=[int(q_pos[b].max()) - Wn + 1 for b in range(B)] if Wn else None, seed=56)
    if Wn == 0:
        empty = torch.as_tensor(q_pos < 127)
        assert bool(torch.all(out.cpu()[empty] == 0)) and bool(torch.all(torch.isneginf(lse.cpu()[empty])))


@pytest.mark.parametrize("early_start", [False, True], ids=["plain", "early"])
def test_attn_workspace_reused_across_calls_and_plans(cuda_lib, early_start):
    """One caller workspace, sized by the size query before any output exists, serves repeated calls and
    calls of the other launch plan (early start or not) for the same queries: identical results every
    time, and against the oracle; the kernel-count query matches the plan (attention + split merge)."""
    csa = cuda_lib
    B, n = 6, 2048
    q_pos = [4 * n - 1 - 37 * b for b in range(B)]
    G = gen(71)
    kv = normal((B, n, 512), 1.0, G)
    q = normal((B, 1, 64, 512), 1.0, G).to(DEV)
    win = normal((B, 128, 512), 1.0, G).to(DEV)
    wp0 = torch.tensor([t - 127 for t in q_pos], dtype=torch.int64, device=DEV)
    qp = torch.tensor(q_pos, dtype=torch.int64, device=DEV).view(B, 1)
    n_c = torch.full((B,), n, dtype=torch.int32, device=DEV)
    # k = 384: 3 entry tiles (+ the window tile): 3 or 4 CTAs per query in both plans
    idx = torch.stack([torch.randperm(n, generator=G)[:384] for _ in range(B)]).view(B, 1, 384).to(torch.int32).to(DEV)
    cache = csa.PackedCache(B, n, 512, 64, DEV, 1.0)
    csa.pack_fp4(kv.to(DEV), cache)
    nbytes = max(csa.attn_workspace_size(q, qp, cache, n_c, idx, win, wp0, ratio=4, window=128, early_start=e)
                 for e in (False, True))
    assert nbytes > 0
    ws = torch.full((nbytes,), 0xA5, dtype=torch.uint8, device=DEV)
    assert csa.attn_kernel_count(q, qp, cache, n_c, idx, win, wp0, ratio=4, window=128,
                                 early_start=early_start) == 2
    outs = []
    for rep in range(3):
        # another plan (the other early-start setting) in between, on the same workspace
        csa.sparse_attn(q, qp, cache, n_c, idx, win, wp0, ratio=4, ws=ws, early_start=not early_start)
        out, lse = csa.sparse_attn(q, qp, cache, n_c, idx, win, wp0, ratio=4, ws=ws, early_start=early_start)
        torch.cuda.synchronize()
        outs.append((out.clone(), lse.clone()))
    assert all(torch.equal(o, outs[0][0]) and torch.equal(l, outs[0][1]) for o, l in outs[1:])
    scale = 512 ** -0.5
    for b in range(B):
        codes, scales, rope = O.pack_fp4(f64(kv[b]), 64, 1.0)
        rows = O.entry_kv(codes, scales, rope, 448, 1.0)
        o_ref, l_ref = O.attention(f64(q[b]), [q_pos[b]], rows, idx[b].cpu().numpy(), n, f64(win[b]), q_pos[b] - 127,
                                   128, scale)
        assert_close(f64(outs[0][0][b]), o_ref, OUT_ATOL, OUT_RTOL, f"out b={b}")
        assert_close(outs[0][1][b].cpu().numpy(), l_ref, LSE_ATOL, LSE_RTOL, f"lse b={b}")


@pytest.mark.parametrize("hca", [False, True], ids=["sparse", "hca"])
def test_attn_ctas_walking_many_tiles(cuda_lib, hca):
    """Few queries with long key lists (20 queries x 16-17 tiles): sparse, the persistent kernel walks units
    of a few tiles of one query each (units past a query's last tile write an empty partial); HCA, the
    per-query kernel's CTAs walk several tiles each; splits merged by the merge kernel, ragged last tiles
    and a partial window."""
    B, Nq, n = 5, 4, 2048
    rng = np.random.default_rng(90 + hca)
    q_pos = rng.integers(4 * 1500, 4 * n, size=(B, Nq))
    q_pos[0, 0] = 4 * n - 1
    kw = dict(hca=True, ratio=4) if hca else dict(k=1800)
    _attn_case(cuda_lib, B=B, Nq=Nq, H=64, d=512, d_r=64, n_max=n, n_c=[n, n - 37, 1700, n, 1999],
               q_pos=q_pos.ravel().tolist(), Wn=160, seed=91 + hca, **kw)


def test_attn_hca(cuda_lib):
    _attn_case(cuda_lib, B=2, Nq=1, H=64, d=512, d_r=64, n_max=300, n_c=[300, 300],
               q_pos=[128 * 300 - 1, 128 * 150 + 5], hca=True, ratio=128, seed=7)


def test_attn_hca_empty_set(cuda_lib):
    out, lse = _attn_case(cuda_lib, B=1, Nq=1, H=64, d=512, d_r=64, n_max=16, n_c=[0], q_pos=[100], hca=True,
                          ratio=128, Wn=0, seed=8)
    assert torch.all(out == 0) and torch.all(torch.isneginf(lse))


# ------------------------------------------------------------------------------------ FP8 window

@pytest.mark.parametrize("d,d_r", [(512, 64), (128, 0), (192, 64)])
def test_pack_fp8_window_bit_exact(cuda_lib, d, d_r):
    csa = cuda_lib
    B, n, Wn = 3, 45, 70
    G = gen(41)
    x = torch.randn((B, n, d), generator=G)
    x[0, 0] = 0.0                                        # all-zero row: scale 0, codes 0
    x[0, 1] *= 1e-30                                     # tiny scales (fp32 subnormal range)
    x[0, 2, :64] = torch.tensor(O.e4m3_decode(np.arange(64)) * 3.0)   # scaled E4M3 grid values
    x[1, 3] *= 3e4                                       # large rows
    x[2, 4, 1::2] = -1e-6                                # elements rounding to -0 -> +0
    x[2, 5, :64] = 0.0
    x[2, 5, 7] = -2.0                                    # one nonzero: its code is exactly -448
    src = x.to(torch.bfloat16)
    win = csa.Fp8Window(B, Wn, d, d_r, DEV)
    row0 = torch.tensor([0, 11, Wn - n], dtype=torch.int32, device=DEV)
    csa.pack_fp8_window(src.to(DEV), win, row0)
    torch.cuda.synchronize()
    nb = (d - d_r) // 64
    for b in range(B):
        codes, scales, rope = O.pack_fp8_window(f64(src[b]), d_r)
        r0 = int(row0[b])
        assert np.array_equal(np_u8(win.codes[b, r0:r0 + n]), codes), f"codes b={b}"
        got_s = win.scales[b, r0:r0 + n].cpu().numpy()
        assert np.array_equal(got_s[:, :nb].view(np.uint32), scales.astype(np.float32).view(np.uint32)), f"scales b={b}"
        assert np.all(got_s[:, nb:] == 0.0)
        if d_r:
            assert np.array_equal(bf16_bits(win.rope[b, r0:r0 + n]), bf16_bits(src[b, :, d - d_r:]))
    assert int(win.codes[0, n:].abs().sum()) == 0        # rows outside [row0, row0 + n) untouched


@pytest.mark.parametrize("early", [False, True])
def test_attn_fp8_window_decode(cuda_lib, early):
    n_c = [2048, 700, 2048, 1000]
    q_pos = [4 * 2048 - 1, 4 * 700 - 1, 4 * 1500 + 3, 4 * 1000 - 1]
    _attn_case(cuda_lib, B=4, Nq=1, H=64, d=512, d_r=64, n_max=2048, n_c=n_c, q_pos=q_pos, k=512, seed=42,
               win_fp8=True, early_start=early)


def test_attn_fp8_window_partial_multi_query_and_hca(cuda_lib):
    # a window buffer holding part of the window, a query near the start, several queries per sequence
    _attn_case(cuda_lib, B=2, Nq=1, H=64, d=512, d_r=64, n_max=64, n_c=[64, 2], q_pos=[255, 9], k=64, Wn=50,
               win_pos0=[206, 0], seed=43, win_fp8=True)
    q_pos = list(range(3000, 3000 + 37))
    _attn_case(cuda_lib, B=1, Nq=37, H=64, d=512, d_r=64, n_max=800, n_c=[800], q_pos=q_pos, k=200, Wn=300,
               seed=44, win_fp8=True)
    _attn_case(cuda_lib, B=2, Nq=1, H=64, d=512, d_r=64, n_max=300, n_c=[300, 300],
               q_pos=[128 * 300 - 1, 128 * 150 + 5], hca=True, ratio=128, seed=45, win_fp8=True)


@pytest.mark.parametrize("cluster", [True, False], ids=["cluster", "no_cluster"])
@pytest.mark.parametrize("k", [128, 384, 640, 896, 1024])
def test_attn_cluster_merge_sizes(cuda_lib, k, cluster):
    """Two decode queries whose key lists span 2, 4, 6, 8 and 9 tiles of 128 keys (k entries + the
    128-row window): with CSA_CLUSTER_MERGE 2..8 CTAs per query merge inside their thread-block cluster and
    9 go through the workspace partials and the merge kernel; without it 2..4 CTAs per query are merged
    by the query's last CTA and more by the merge kernel."""
    n = 4096
    _attn_case(cuda_lib, B=2, Nq=1, H=64, d=512, d_r=64, n_max=n, n_c=[n, n - 100], q_pos=[4 * n - 1, 4 * n - 401],
               k=k, seed=60 + k // 128, cluster=cluster)
