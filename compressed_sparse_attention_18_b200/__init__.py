"""Python binding of the B200 CSA library (libcsa_b200.so, C ABI in include/csa.h).

Argument marshalling only: every step runs in the CUDA kernels behind the C ABI.  torch supplies
device memory, streams and output/workspace allocation.  There is no CPU fallback: importing this
package fails loudly when the library has not been built, and every call requires CUDA tensors.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libcsa_b200.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python compressed_sparse_attention_18_b200/build.py` "
        "(nvcc, sm_100a).  There is no CPU fallback.")
_lib = ctypes.CDLL(LIB_PATH)

ENTRY_POINTS = ("csa_status_string", "csa_version", "csa_last_cuda_error", "csa_compress", "csa_pack_fp4",
                "csa_index_topk_workspace_size", "csa_index_topk", "csa_index_scores", "csa_topk_workspace_size",
                "csa_topk", "csa_attn_workspace_size", "csa_sparse_attn", "hca_dense_attn",
                "csa_index_topk_noalloc", "csa_device_status", "csa_check_error_path",
                "csa_pack_fp8_window", "csa_attn_kernel_count")
# (PagedCache: a paged pool + block table, accepted wherever a PackedCache is)

_u32, _i32, _f32, _vp = ctypes.c_uint32, ctypes.c_int32, ctypes.c_float, ctypes.c_void_p
CSA_EARLY_START = 1   # see csa.h: part of a call's work may start before the step's earlier kernels end
CSA_CLUSTER_MERGE = 2  # see csa.h: a query's split partials merge inside their thread-block cluster
CSA_ONCHIP_TOPK = 4   # see csa.h: decode rows scored and selected inside one cluster (scores stay on chip)


class PageMap(ctypes.Structure):
    _fields_ = [("table", _vp), ("page_size", _i32), ("width", _i32), ("n_pages", _i32)]


class Fp4Cache(ctypes.Structure):
    _fields_ = [("codes", _vp), ("scales", _vp), ("rope", _vp), ("row0", _vp), ("n_max", _i32),
                ("global_scale", _f32), ("pages", PageMap)]


class CompressArgs(ctypes.Structure):
    _fields_ = [("struct_size", _u32), ("B", _i32), ("T", _i32), ("d_model", _i32), ("d", _i32),
                ("d_rope", _i32), ("d_index", _i32), ("ratio", _i32), ("rope_theta", _f32), ("pos0", _vp),
                ("x", _vp), ("W_kv", _vp), ("W_g", _vp), ("C", _vp), ("Z", _vp), ("b_pos", _vp),
                ("W_IK", _vp), ("c_out", _vp), ("kI_out", _vp), ("kv_pack", Fp4Cache), ("ki_pack", Fp4Cache)]


class PackArgs(ctypes.Structure):
    _fields_ = [("struct_size", _u32), ("B", _i32), ("n", _i32), ("d", _i32), ("d_rope", _i32),
                ("n_max", _i32), ("global_scale", _f32), ("src", _vp), ("row0", _vp), ("codes", _vp),
                ("scales", _vp), ("rope", _vp), ("pages", PageMap)]


class IndexArgs(ctypes.Structure):
    _fields_ = [("struct_size", _u32), ("B", _i32), ("Nq", _i32), ("H_I", _i32), ("d_I", _i32),
                ("ratio", _i32), ("k", _i32), ("n_max", _i32), ("g_q", _f32), ("g_k", _f32), ("q_I", _vp),
                ("w", _vp), ("k_codes", _vp), ("k_scales", _vp), ("n_c", _vp), ("q_pos", _vp),
                ("cand", _vp), ("n_cand", _i32), ("pool_blocks", _i32), ("pool_block_size", _i32),
                ("pool_out", _vp), ("idx_out", _vp), ("scores_out", _vp), ("hist", _vp), ("flags", _u32), ("k_pages", PageMap)]


class AttnArgs(ctypes.Structure):
    _fields_ = [("struct_size", _u32), ("B", _i32), ("Nq", _i32), ("H", _i32), ("d", _i32), ("d_rope", _i32),
                ("ratio", _i32), ("n_max", _i32), ("k", _i32), ("Wn", _i32), ("window", _i32),
                ("g_kv", _f32), ("softmax_scale", _f32), ("q", _vp), ("q_pos", _vp), ("kv_codes", _vp),
                ("kv_scales", _vp), ("kv_rope", _vp), ("n_c", _vp), ("idx", _vp), ("win_kv", _vp),
                ("win_pos0", _vp), ("out", _vp), ("lse", _vp), ("flags", _u32), ("out_rope_theta", _f32),
                ("win_format", _u32), ("win_codes", _vp), ("win_scales", _vp), ("win_rope", _vp), ("kv_pages", PageMap)]


class Fp8WindowArgs(ctypes.Structure):
    _fields_ = [("struct_size", _u32), ("B", _i32), ("n", _i32), ("d", _i32), ("d_rope", _i32), ("Wn", _i32),
                ("src", _vp), ("row0", _vp), ("codes", _vp), ("scales", _vp), ("rope", _vp)]


_lib.csa_status_string.restype = ctypes.c_char_p
_lib.csa_status_string.argtypes = [ctypes.c_int]
_lib.csa_version.restype = ctypes.c_int
_lib.csa_last_cuda_error.restype = ctypes.c_int
_lib.csa_device_status.restype = ctypes.c_int
_lib.csa_device_status.argtypes = [_vp]
_lib.csa_check_error_path.restype = ctypes.c_int
_lib.csa_check_error_path.argtypes = [_u32, _vp]
for _name, _st in (("csa_compress", CompressArgs), ("csa_pack_fp4", PackArgs), ("csa_pack_fp8_window", Fp8WindowArgs)):
    getattr(_lib, _name).restype = ctypes.c_int
    getattr(_lib, _name).argtypes = [ctypes.POINTER(_st), _vp]
_lib.csa_index_topk_workspace_size.restype = ctypes.c_size_t
_lib.csa_index_topk_workspace_size.argtypes = [ctypes.POINTER(IndexArgs)]
_lib.csa_index_topk.restype = ctypes.c_int
_lib.csa_index_topk.argtypes = [ctypes.POINTER(IndexArgs), _vp, ctypes.c_size_t, _vp]
_lib.csa_index_topk_noalloc.restype = ctypes.c_int
_lib.csa_index_topk_noalloc.argtypes = [ctypes.POINTER(IndexArgs), _vp]
_lib.csa_index_scores.restype = ctypes.c_int
_lib.csa_index_scores.argtypes = [ctypes.POINTER(IndexArgs), _vp, ctypes.c_int64, _vp]
_lib.csa_topk_workspace_size.restype = ctypes.c_size_t
_lib.csa_topk_workspace_size.argtypes = [ctypes.POINTER(IndexArgs)]
_lib.csa_topk.restype = ctypes.c_int
_lib.csa_topk.argtypes = [ctypes.POINTER(IndexArgs), _vp, ctypes.c_int64, _vp, ctypes.c_size_t, _vp]
_lib.csa_attn_workspace_size.restype = ctypes.c_size_t
_lib.csa_attn_workspace_size.argtypes = [ctypes.POINTER(AttnArgs), ctypes.c_int]
_lib.csa_attn_kernel_count.restype = ctypes.c_int
_lib.csa_attn_kernel_count.argtypes = [ctypes.POINTER(AttnArgs), ctypes.c_int]
for _name in ("csa_sparse_attn", "hca_dense_attn"):
    getattr(_lib, _name).restype = ctypes.c_int
    getattr(_lib, _name).argtypes = [ctypes.POINTER(AttnArgs), _vp, ctypes.c_size_t, _vp]


class CSAError(RuntimeError):
    pass


def version() -> int:
    return _lib.csa_version()


def device_status(stream=None):
    """Synchronise and raise if a kernel recorded a device-side error (a bounded wait gave up)."""
    _check(_lib.csa_device_status(_stream(stream)), "device status")


def check_error_path(polls: int = 1000, stream=None):
    """Launch the library's error-path self-check: a bounded wait on a barrier nothing arrives on gives
    up after `polls` polls and records the device error that device_status() then reports."""
    _check(_lib.csa_check_error_path(int(polls), _stream(stream)), "check_error_path")


def _check(status: int, what: str):
    if status != 0:
        msg = _lib.csa_status_string(status).decode()
        if status == 4:
            msg += f" (cudaError {_lib.csa_last_cuda_error()})"
        raise CSAError(f"{what}: {msg}")


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise CSAError("tensor is not on a CUDA device (no CPU path)")
    if not t.is_contiguous():
        raise CSAError("tensor must be contiguous")
    return t.data_ptr()


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _ws(nbytes: int, device, ws=None, zero=False):
    if nbytes == 0:
        return None
    if ws is not None and ws.numel() * ws.element_size() >= nbytes:
        return ws
    return (torch.zeros if zero else torch.empty)(nbytes, dtype=torch.uint8, device=device)


# ------------------------------------------------------------------------------------------- API

def _page_map(cache):
    """The cache's csa_page_map (a NULL table for the contiguous layout)."""
    t = getattr(cache, "table", None)
    if t is None:
        return PageMap()
    return PageMap(_ptr(t), cache.page_size, t.shape[-1], cache.n_pages)


class PagedCache:
    """A paged FP4 cache: pools of n_pages pages x page_size entries (codes u8, scales u8, rope bf16) and a
    block table [B, width] int32; entry i of sequence b lives in slot i % page_size of page
    table[b, i // page_size] (csa_page_map).  Used wherever a PackedCache is."""

    def __init__(self, B, n_max, d, d_rope, device, page_size, n_pages, table, global_scale=1.0):
        d_n = d - d_rope
        s_pad = (d_n // 32 + 3) // 4 * 4
        rows = n_pages * page_size
        self.B, self.n_max, self.d, self.d_rope, self.g = B, n_max, d, d_rope, float(global_scale)
        self.page_size, self.n_pages = page_size, n_pages
        self.table = table.to(device=device, dtype=torch.int32).contiguous()
        self.codes = torch.zeros((rows, d_n // 2), dtype=torch.uint8, device=device)
        self.scales = torch.zeros((rows, s_pad), dtype=torch.uint8, device=device)
        self.rope = torch.zeros((rows, d_rope if d_rope else 0), dtype=torch.bfloat16, device=device)


def _fp4_target(cache, row0):
    if cache is None:
        return Fp4Cache()
    return Fp4Cache(_ptr(cache.codes), _ptr(cache.scales), _ptr(cache.rope) if cache.d_rope else None, _ptr(row0),
                    cache.n_max, cache.g, _page_map(cache))


def compress(*, b_pos, ratio, d_rope=0, rope_theta=0.0, pos0=None, x=None, W_kv=None, W_g=None, C=None, Z=None,
             W_IK=None, c_out=None, kI_out=None, kv_cache=None, ki_cache=None, row0=None, stream=None):
    """Compressor.  Projection mode (x [B,T,d_m], W_kv/W_g [d_m,d]) fills C, Z [B,T,d]; pooling mode
    reads C, Z.  kv_cache / ki_cache (PackedCache, rows row0[b] + i) also receive the FP4-packed entries
    and indexer keys from the same launch.  Returns (c [B,T//r,d], k_I [B,T//r,d_I] or None, C, Z)."""
    if x is not None:
        B, T, dm = x.shape
        d = W_kv.shape[1]
        if C is None:
            C = torch.empty((B, T, d), dtype=torch.bfloat16, device=x.device)
        if Z is None:
            Z = torch.empty((B, T, d), dtype=torch.bfloat16, device=x.device)
    else:
        B, T, d = C.shape
        dm = 0
    n = T // ratio
    dI = W_IK.shape[1] if W_IK is not None else 0
    if c_out is None:
        c_out = torch.empty((B, n, d), dtype=torch.bfloat16, device=C.device)
    if W_IK is not None and kI_out is None:
        kI_out = torch.empty((B, n, dI), dtype=torch.bfloat16, device=C.device)
    a = CompressArgs(ctypes.sizeof(CompressArgs), B, T, dm, d, d_rope, dI, ratio, rope_theta, _ptr(pos0),
                     _ptr(x), _ptr(W_kv), _ptr(W_g), _ptr(C), _ptr(Z), _ptr(b_pos), _ptr(W_IK), _ptr(c_out),
                     _ptr(kI_out) if W_IK is not None else None, _fp4_target(kv_cache, row0),
                     _fp4_target(ki_cache, row0))
    _check(_lib.csa_compress(ctypes.byref(a), _stream(stream)), "csa_compress")
    return c_out, (kI_out if W_IK is not None else None), C, Z


class PackedCache:
    """FP4 cache storage [B, n_max, ...]: codes u8, scales u8 (E4M3), rope bf16."""

    def __init__(self, B, n_max, d, d_rope, device, global_scale=1.0):
        d_n = d - d_rope
        s_pad = (d_n // 32 + 3) // 4 * 4
        self.B, self.n_max, self.d, self.d_rope, self.g = B, n_max, d, d_rope, float(global_scale)
        self.codes = torch.zeros((B, n_max, d_n // 2), dtype=torch.uint8, device=device)
        self.scales = torch.zeros((B, n_max, s_pad), dtype=torch.uint8, device=device)
        self.rope = torch.zeros((B, n_max, max(d_rope, 1) if d_rope else 0), dtype=torch.bfloat16, device=device)


def pack_fp4(src, cache: PackedCache, row0=None, stream=None):
    """Pack src [B, n, d] bf16 into cache rows row0[b] + j (row0 int32 [B] or None = 0)."""
    B, n, d = src.shape
    a = PackArgs(ctypes.sizeof(PackArgs), B, n, d, cache.d_rope, cache.n_max, cache.g, _ptr(src), _ptr(row0),
                 _ptr(cache.codes), _ptr(cache.scales), _ptr(cache.rope) if cache.d_rope else None,
                 _page_map(cache))
    _check(_lib.csa_pack_fp4(ctypes.byref(a), _stream(stream)), "csa_pack_fp4")
    return cache


def _index_args(q_I, w, kcache: PackedCache, n_c, q_pos, ratio, k, g_q, cand, pool_blocks, pool_block_size,
                pool_out, idx_out, scores_out):
    B, Nq, H_I, d_I = q_I.shape
    a = IndexArgs(ctypes.sizeof(IndexArgs), B, Nq, H_I, d_I, ratio, k, kcache.n_max, g_q, kcache.g, _ptr(q_I),
                  _ptr(w), _ptr(kcache.codes), _ptr(kcache.scales), _ptr(n_c), _ptr(q_pos), _ptr(cand),
                  cand.shape[-1] if cand is not None else 0, pool_blocks, pool_block_size, _ptr(pool_out),
                  _ptr(idx_out), _ptr(scores_out))
    a.k_pages = _page_map(kcache)
    return a


def index_topk(q_I, w, kcache: PackedCache, n_c, q_pos, *, ratio, k, g_q=1.0, cand=None, pool_blocks=0,
               pool_block_size=8, want_scores=False, idx_out=None, scores_out=None, pool_out=None, ws=None,
               early_start=False, onchip=False, stream=None):
    """Lightning indexer + top-k.  Returns (idx [B,Nq,k] int32, scores [B,Nq,k] or None, pool or None).
    onchip: CSA_ONCHIP_TOPK (decode rows scored and selected inside one cluster, scores never in HBM)."""
    B, Nq = q_I.shape[:2]
    dev = q_I.device
    if idx_out is None:
        idx_out = torch.empty((B, Nq, k), dtype=torch.int32, device=dev)
    if want_scores and scores_out is None:
        scores_out = torch.empty((B, Nq, k), dtype=torch.float32, device=dev)
    if pool_blocks and pool_out is None:
        pool_out = torch.empty((B, Nq, pool_blocks * pool_block_size), dtype=torch.int32, device=dev)
    a = _index_args(q_I, w, kcache, n_c, q_pos, ratio, k, g_q, cand, pool_blocks, pool_block_size, pool_out,
                    idx_out, scores_out)
    a.flags = (CSA_EARLY_START if early_start else 0) | (CSA_ONCHIP_TOPK if onchip else 0)
    nbytes = _lib.csa_index_topk_workspace_size(ctypes.byref(a))
    wbuf = _ws(nbytes, dev, ws)
    _check(_lib.csa_index_topk(ctypes.byref(a), _ptr(wbuf) if wbuf is not None else None, nbytes,
                               _stream(stream)), "csa_index_topk")
    return idx_out, scores_out, pool_out


def index_scores(q_I, w, kcache: PackedCache, n_c, q_pos, scores, *, ratio, g_q=1.0, cand=None, hist=None,
                 k=None, early_start=False, stream=None):
    """Lightning-indexer scores only, into scores [B*Nq, ld] fp32 (see csa_index_scores); hist
    ([B*Nq, 4096] uint32 as int32, optional, zero before first use) receives the score histogram for
    topk(), which leaves it zero again; k (optional) is recorded in the call's arguments.
    early_start: CSA_EARLY_START (only right after the compress call of the same decode step)."""
    a = _index_args(q_I, w, kcache, n_c, q_pos, ratio, k if k is not None else 1, g_q, cand, 0, 8, None, None, None)
    a.hist = _ptr(hist)
    a.flags = CSA_EARLY_START if early_start else 0
    _check(_lib.csa_index_scores(ctypes.byref(a), _ptr(scores), scores.shape[-1], _stream(stream)),
           "csa_index_scores")
    return scores


def topk(scores, kcache: PackedCache, n_c, q_pos, *, B, Nq, ratio, k, cand=None, pool_blocks=0, pool_block_size=8,
         want_scores=False, idx_out=None, scores_out=None, pool_out=None, hist=None, ws=None, early_start=False,
         stream=None):
    """Top-k (+ hierarchical pool) over a score matrix written by index_scores (see csa_topk).
    early_start: CSA_EARLY_START (only right after the index_scores call of the same decode step)."""
    dev = scores.device
    if idx_out is None:
        idx_out = torch.empty((B, Nq, k), dtype=torch.int32, device=dev)
    if want_scores and scores_out is None:
        scores_out = torch.empty((B, Nq, k), dtype=torch.float32, device=dev)
    if pool_blocks and pool_out is None:
        pool_out = torch.empty((B, Nq, pool_blocks * pool_block_size), dtype=torch.int32, device=dev)
    d_I = 2 * kcache.codes.shape[-1]
    a = IndexArgs(ctypes.sizeof(IndexArgs), B, Nq, 1, d_I, ratio, k, kcache.n_max, 1.0, kcache.g, None, None,
                  None, None, _ptr(n_c), _ptr(q_pos), _ptr(cand), cand.shape[-1] if cand is not None else 0,
                  pool_blocks, pool_block_size, _ptr(pool_out), _ptr(idx_out), _ptr(scores_out), _ptr(hist))
    a.flags = CSA_EARLY_START if early_start else 0
    nbytes = _lib.csa_topk_workspace_size(ctypes.byref(a))
    wbuf = _ws(nbytes, dev, ws)
    _check(_lib.csa_topk(ctypes.byref(a), _ptr(scores), scores.shape[-1], _ptr(wbuf) if wbuf is not None else None,
                         nbytes, _stream(stream)), "csa_topk")
    return idx_out, scores_out, pool_out


def topk_workspace_size(kcache, n_c, q_pos, *, B, Nq, ratio, k, cand=None, pool_blocks=0, pool_block_size=8):
    d_I = 2 * kcache.codes.shape[-1]
    a = IndexArgs(ctypes.sizeof(IndexArgs), B, Nq, 1, d_I, ratio, k, kcache.n_max, 1.0, kcache.g, None, None,
                  None, None, _ptr(n_c), _ptr(q_pos), _ptr(cand), cand.shape[-1] if cand is not None else 0,
                  pool_blocks, pool_block_size, 256 if pool_blocks else None, 256, None)
    return _lib.csa_topk_workspace_size(ctypes.byref(a))


def index_topk_workspace_size(q_I, w, kcache, n_c, q_pos, *, ratio, k, g_q=1.0, cand=None, pool_blocks=0,
                              pool_block_size=8):
    a = _index_args(q_I, w, kcache, n_c, q_pos, ratio, k, g_q, cand, pool_blocks, pool_block_size, None, None,
                    None)
    return _lib.csa_index_topk_workspace_size(ctypes.byref(a))


class Fp8Window:
    """FP8 sliding-window rows [B, Wn, d] as csa_pack_fp8_window writes them: E4M3 codes [B, Wn, d_n],
    fp32 scales per 64 channels [B, Wn, round_up(d_n / 64, 4)], RoPE channels bf16 [B, Wn, d_rope]."""

    def __init__(self, B, Wn, d, d_rope, device):
        d_n = d - d_rope
        self.B, self.Wn, self.d, self.d_rope = B, Wn, d, d_rope
        self.codes = torch.zeros((B, Wn, d_n), dtype=torch.uint8, device=device)
        self.scales = torch.zeros((B, Wn, (d_n // 64 + 3) // 4 * 4), dtype=torch.float32, device=device)
        self.rope = torch.zeros((B, Wn, d_rope), dtype=torch.bfloat16, device=device)

    @property
    def shape(self):
        return (self.B, self.Wn, self.d)


def pack_fp8_window(src, win: Fp8Window, row0=None, stream=None):
    """FP8-pack bf16 window rows src [B, n, d] into win rows row0[b] + j (csa_pack_fp8_window)."""
    B, n, d = src.shape
    a = Fp8WindowArgs(ctypes.sizeof(Fp8WindowArgs), B, n, d, win.d_rope, win.Wn, _ptr(src), _ptr(row0),
                      _ptr(win.codes), _ptr(win.scales), _ptr(win.rope) if win.d_rope else None)
    _check(_lib.csa_pack_fp8_window(ctypes.byref(a), _stream(stream)), "csa_pack_fp8_window")
# (PagedCache: a paged pool + block table, accepted wherever a PackedCache is)
    return win


def _attn_args(q, q_pos, cache: PackedCache, n_c, idx, win_kv, win_pos0, ratio, window, softmax_scale, out, lse):
    """win_kv: bf16 rows [B, Wn, d] or an Fp8Window."""
    B, Nq, H, d = q.shape
    k = idx.shape[-1] if idx is not None else 0
    Wn = win_kv.shape[1] if win_kv is not None else 0
    fp8 = isinstance(win_kv, Fp8Window)
    a = AttnArgs(ctypes.sizeof(AttnArgs), B, Nq, H, d, cache.d_rope, ratio, cache.n_max, k, Wn, window, cache.g,
                 softmax_scale, _ptr(q), _ptr(q_pos), _ptr(cache.codes), _ptr(cache.scales), _ptr(cache.rope),
                 _ptr(n_c), _ptr(idx), None if fp8 else _ptr(win_kv), _ptr(win_pos0), _ptr(out), _ptr(lse))
    if fp8:
        a.win_format = 1
        a.win_codes, a.win_scales, a.win_rope = _ptr(win_kv.codes), _ptr(win_kv.scales), _ptr(win_kv.rope)
    a.kv_pages = _page_map(cache)
    return a


def _attn(fn, hca, q, q_pos, cache, n_c, idx, win_kv, win_pos0, ratio, window, softmax_scale, out, lse, ws,
          stream, early_start=False, out_rope_theta=0.0, cluster=False):
    B, Nq, H, d = q.shape
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Nq, H), dtype=torch.float32, device=q.device)
    a = _attn_args(q, q_pos, cache, n_c, idx, win_kv, win_pos0, ratio, window, softmax_scale, out, lse)
    a.flags = (CSA_EARLY_START if early_start else 0) | (CSA_CLUSTER_MERGE if cluster else 0)
    a.out_rope_theta = out_rope_theta
    nbytes = _lib.csa_attn_workspace_size(ctypes.byref(a), hca)
    wbuf = _ws(nbytes, q.device, ws)
    _check(fn(ctypes.byref(a), _ptr(wbuf) if wbuf is not None else None, nbytes, _stream(stream)),
           "hca_dense_attn" if hca else "csa_sparse_attn")
    return out, lse


def sparse_attn(q, q_pos, cache: PackedCache, n_c, idx, win_kv=None, win_pos0=None, *, ratio=4, window=128,
                softmax_scale=0.0, out=None, lse=None, ws=None, early_start=False, out_rope_theta=0.0, cluster=False,
                stream=None):
    """CSA attention over the selected entries idx [B,Nq,k] plus the window.  Returns (out, lse).
    early_start: CSA_EARLY_START (window tiles start before the step's index and top-k kernels end;
    only inside a decode step that began with compress).  out_rope_theta: inverse-RoPE epilogue on the
    output's RoPE channels at the query position (0 = off).  cluster=True: CSA_CLUSTER_MERGE (split
    partials merged inside a thread-block cluster instead of through the workspace)."""
    return _attn(_lib.csa_sparse_attn, 0, q, q_pos, cache, n_c, idx, win_kv, win_pos0, ratio, window,
                 softmax_scale, out, lse, ws, stream, early_start, out_rope_theta, cluster)


def hca_attn(q, q_pos, cache: PackedCache, n_c, win_kv=None, win_pos0=None, *, ratio=128, window=128,
             softmax_scale=0.0, out=None, lse=None, ws=None, out_rope_theta=0.0, stream=None):
    """HCA attention over every visible entry plus the window.  Returns (out, lse)."""
    return _attn(_lib.hca_dense_attn, 1, q, q_pos, cache, n_c, None, win_kv, win_pos0, ratio, window,
                 softmax_scale, out, lse, ws, stream, out_rope_theta=out_rope_theta)


def attn_workspace_size(q, q_pos, cache, n_c, idx, win_kv, win_pos0, *, ratio, window, hca=False, early_start=False,
                        cluster=False):
    """Bytes of workspace one call with these arguments needs (csa_attn_workspace_size)."""
    a = _attn_args(q, q_pos, cache, n_c, idx, win_kv, win_pos0, ratio, window, 0.0, None, None)
    a.flags = (CSA_EARLY_START if early_start else 0) | (CSA_CLUSTER_MERGE if cluster else 0)
    return _lib.csa_attn_workspace_size(ctypes.byref(a), 1 if hca else 0)


def attn_kernel_count(q, q_pos, cache, n_c, idx, win_kv, win_pos0, *, ratio, window, hca=False, early_start=False,
                      cluster=False, out_rope_theta=0.0):
    """Kernels one attention call with these arguments launches (csa_attn_kernel_count)."""
    a = _attn_args(q, q_pos, cache, n_c, idx, win_kv, win_pos0, ratio, window, 0.0, None, None)
    a.flags = (CSA_EARLY_START if early_start else 0) | (CSA_CLUSTER_MERGE if cluster else 0)
    a.out_rope_theta = out_rope_theta
    return _lib.csa_attn_kernel_count(ctypes.byref(a), 1 if hca else 0)
