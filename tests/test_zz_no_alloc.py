"""csa_index_topk_noalloc: the indexer + top-k entry point for callers that cannot allocate device
memory (a runtime or plugin host that owns all device memory, a fixed-budget embedded service, or
code that must not trigger the implicit synchronisation of cudaMalloc/cudaFree).  Its scratch is a
static device array inside the library instead of a caller workspace.

Called through the C ABI (ctypes) and checked against csa_index_topk, the entry point with a caller
workspace, on two calls in a row with different queries (the shared array keeps the previous call's
contents, so the second call also checks that nothing stale leaks through).  The two run the same
kernels, so the selected sets and scores must agree exactly.  This file is collected last."""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _args(csa, q_I, w, kc, n_c, q_pos, k, idx, sc):
    B, Nq, H_I, d_I = q_I.shape
    return csa.IndexArgs(ctypes.sizeof(csa.IndexArgs), B, Nq, H_I, d_I, 4, k, kc.n_max, 1.0, kc.g, q_I.data_ptr(),
                         w.data_ptr(), kc.codes.data_ptr(), kc.scales.data_ptr(), n_c.data_ptr(), q_pos.data_ptr(),
                         None, 0, 0, 8, None, idx.data_ptr(), sc.data_ptr())


# (B, cache rows, n_c per sequence, last visible group per sequence): rows of one 32768-score segment
# (the single-CTA top-k), and a 70000-score row that the multi-segment top-k splits over several CTAs
# (its per-row state, candidate and tournament buffers all live in the shared static array)
CASES = [(4, 20000, [20000, 19993, 5000, 300], [19999, 19999, 4000, 299]),
         (1, 70000, [70000], [69999])]


@pytest.mark.parametrize("B,n,ncs,groups", CASES, ids=["one_segment", "multi_segment_70000"])
def test_noalloc_matches_workspace_entry_point(cuda_lib, B, n, ncs, groups):
    csa = cuda_lib
    lib = csa._lib
    torch.cuda.set_device(0)
    g = torch.Generator(device=DEV).manual_seed(21)
    d_I, H_I, k = 128, 8, 256
    kI = torch.randn((B, n, d_I), generator=g, device=DEV).to(torch.bfloat16)
    kc = csa.PackedCache(B, n, d_I, 0, DEV)
    csa.pack_fp4(kI, kc)
    n_c = torch.tensor(ncs, dtype=torch.int32, device=DEV)
    q_pos = torch.tensor([[4 * gi + 3] for gi in groups], dtype=torch.int64, device=DEV)
    if B == 4:
        q_pos[2, 0] = 4 * 4000 + 2                     # a query whose last group is still incomplete
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        q_I = torch.randn((B, 1, H_I, d_I), generator=g, device=DEV).to(torch.bfloat16)
        w = torch.randn((B, 1, H_I), generator=g, device=DEV) * 0.35
        idx_ref = torch.empty((B, 1, k), dtype=torch.int32, device=DEV)
        sc_ref = torch.empty((B, 1, k), dtype=torch.float32, device=DEV)
        a_ref = _args(csa, q_I, w, kc, n_c, q_pos, k, idx_ref, sc_ref)
        nbytes = lib.csa_index_topk_workspace_size(ctypes.byref(a_ref))
        assert 0 < nbytes <= (8 << 20)
        ws = torch.empty(nbytes, dtype=torch.uint8, device=DEV)
        assert lib.csa_index_topk(ctypes.byref(a_ref), ctypes.c_void_p(ws.data_ptr()), nbytes, stream) == 0
        idx = torch.full((B, 1, k), 7, dtype=torch.int32, device=DEV)
        sc = torch.zeros((B, 1, k), dtype=torch.float32, device=DEV)
        a = _args(csa, q_I, w, kc, n_c, q_pos, k, idx, sc)
        assert lib.csa_index_topk_noalloc(ctypes.byref(a), stream) == 0
        torch.cuda.synchronize()
        for b in range(B):
            r = idx_ref[b, 0].cpu().numpy()
            o = idx[b, 0].cpu().numpy()
            assert set(r.tolist()) == set(o.tolist()), f"call {call} b={b}"
            # same ids -> same scores (order of the slots is unspecified)
            rs = dict(zip(r.tolist(), sc_ref[b, 0].cpu().numpy().tolist()))
            os_ = dict(zip(o.tolist(), sc[b, 0].cpu().numpy().tolist()))
            assert all(rs[i] == os_[i] or (np.isneginf(rs[i]) and np.isneginf(os_[i])) for i in rs)
        if B == 4:
            assert (idx[3, 0] >= 0).sum() == min(k, 300)


def test_noalloc_rejects_problems_beyond_its_scratch(cuda_lib):
    csa = cuda_lib
    lib = csa._lib
    B, n, k = 64, 65536, 64                       # scores alone need 16 MB > the 8 MB array
    q_I = torch.zeros((B, 1, 8, 128), dtype=torch.bfloat16, device=DEV)
    w = torch.zeros((B, 1, 8), dtype=torch.float32, device=DEV)
    kc = csa.PackedCache(B, 16, 128, 0, DEV)
    kc.n_max = n                                  # sizes only: rejected before anything is launched
    n_c = torch.zeros((B,), dtype=torch.int32, device=DEV)
    q_pos = torch.zeros((B, 1), dtype=torch.int64, device=DEV)
    idx = torch.empty((B, 1, k), dtype=torch.int32, device=DEV)
    sc = torch.empty((B, 1, k), dtype=torch.float32, device=DEV)
    a = _args(csa, q_I, w, kc, n_c, q_pos, k, idx, sc)
    assert lib.csa_index_topk_workspace_size(ctypes.byref(a)) > (8 << 20)
    assert lib.csa_index_topk_noalloc(ctypes.byref(a), None) == 3     # CSA_ERR_WORKSPACE
