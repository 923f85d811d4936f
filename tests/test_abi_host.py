"""The C-ABI library loads and exports every entry point include/csa.h declares; host-side argument
validation returns the documented status codes without launching anything (no GPU needed)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "csa.h")


@pytest.fixture(scope="module")
def csa():
    import __graft_entry__
    __graft_entry__._build_module().build()
    import compressed_sparse_attention_18_b200 as m
    return m


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\*?\s+\**([a-z_0-9]+)\s*\(", text, flags=re.M)))


def test_every_declared_symbol_is_exported(csa):
    names = declared_functions()
    assert len(names) >= 10, names
    lib = ctypes.CDLL(csa.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), f"{n} declared in csa.h but not exported"
    assert set(csa.ENTRY_POINTS) <= set(names)


def test_status_strings_and_version(csa):
    lib = csa._lib
    assert lib.csa_status_string(0) == b"CSA_OK"
    assert lib.csa_status_string(3) == b"CSA_ERR_WORKSPACE"
    assert lib.csa_status_string(99) == b"CSA_ERR_UNKNOWN"
    assert csa.version() >= 100


def test_struct_sizes_match_the_header(csa):
    # the ctypes mirrors are the binding's only knowledge of the layout; a wrong struct_size is rejected
    a = csa.PackArgs(ctypes.sizeof(csa.PackArgs) + 4, 1, 1, 64, 0, 1, 1.0)
    assert csa._lib.csa_pack_fp4(ctypes.byref(a), None) == 1


def test_ctypes_mirrors_match_the_c_structs(csa, tmp_path):
    """sizeof of every argument struct as a C compiler sees include/csa.h == the binding's mirror."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "sz.c"
    src.write_text('#include <stdio.h>\n#include "csa.h"\nint main(void){printf("%zu %zu %zu %zu %zu %zu\\n",'
                   'sizeof(csa_compress_args),sizeof(csa_fp4_cache),sizeof(csa_pack_args),'
                   'sizeof(csa_index_args),sizeof(csa_attn_args),sizeof(csa_fp8_window_args));return 0;}\n')
    exe = tmp_path / "sz"
    subprocess.run([cc, "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    got = [int(v) for v in subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split()]
    want = [ctypes.sizeof(t) for t in (csa.CompressArgs, csa.Fp4Cache, csa.PackArgs, csa.IndexArgs, csa.AttnArgs,
                                       csa.Fp8WindowArgs)]
    assert got == want


def test_a_c_program_links_and_calls_the_abi(csa, tmp_path):
    """The ABI from plain C: a program compiled against include/csa.h and linked with the library gets
    the documented statuses for host-side argument errors and the workspace queries (no GPU needed)."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "use.c"
    src.write_text(r"""
#include <stdio.h>
#include <string.h>
#include "csa.h"
int main(void) {
  csa_pack_args p; memset(&p, 0, sizeof p);
  p.struct_size = sizeof p; p.B = 1; p.n = 1; p.d = 40; p.n_max = 1; p.global_scale = 1.0f;
  int s1 = csa_pack_fp4(&p, NULL);                       /* (d - d_rope) % 32 != 0 */
  p.struct_size = sizeof p + 4;
  int s2 = csa_pack_fp4(&p, NULL);                       /* struct_size mismatch */
  csa_attn_args a; memset(&a, 0, sizeof a);
  a.struct_size = sizeof a; a.B = 1; a.Nq = 1; a.H = 65; a.d = 512; a.d_rope = 64; a.ratio = 4;
  a.n_max = 16; a.k = 8; a.window = 128; a.g_kv = 1.0f;
  int s3 = csa_sparse_attn(&a, NULL, 0, NULL);           /* 65 heads: unsupported */
  csa_index_args i; memset(&i, 0, sizeof i);
  i.struct_size = sizeof i; i.B = 2; i.Nq = 1; i.H_I = 8; i.d_I = 128; i.ratio = 4; i.k = 16; i.n_max = 4096;
  i.g_q = 1.0f; i.g_k = 1.0f;
  size_t ws = csa_index_topk_workspace_size(&i);         /* shapes only: no buffer needed */
  i.k = 0;
  size_t ws_bad = csa_index_topk_workspace_size(&i);     /* k = 0: invalid, 0 */
  printf("%d %d %d %zu %s %d %zu\n", s1, s2, s3, ws, csa_status_string(s3), csa_version(), ws_bad);
  return 0;
}
""")
    exe = tmp_path / "use"
    libdir = os.path.dirname(csa.LIB_PATH)
    subprocess.run([cc, "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe), "-L", libdir,
                    "-l:" + os.path.basename(csa.LIB_PATH), "-Wl,-rpath," + libdir], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split()
    assert out[:3] == ["2", "1", "2"] and out[4] == "CSA_ERR_UNSUPPORTED"
    assert int(out[3]) >= 2 * 4096 * 4 and int(out[5]) == csa.version() and out[6] == "0"


def test_invalid_arguments_are_rejected_on_the_host(csa):
    lib = csa._lib
    # pack: d_n not a multiple of 32 -> unsupported; null pointers -> invalid
    a = csa.PackArgs(ctypes.sizeof(csa.PackArgs), 1, 4, 40, 0, 4, 1.0)
    assert lib.csa_pack_fp4(ctypes.byref(a), None) == 2
    a = csa.PackArgs(ctypes.sizeof(csa.PackArgs), 1, 4, 64, 0, 4, 1.0)
    assert lib.csa_pack_fp4(ctypes.byref(a), None) == 1
    a = csa.PackArgs(ctypes.sizeof(csa.PackArgs), 0, 4, 64, 0, 4, 1.0)
    assert lib.csa_pack_fp4(ctypes.byref(a), None) == 0          # empty batch: nothing to do
    assert lib.csa_pack_fp4(None, None) == 1
    # index: unsupported d_I, too many heads, bad k
    ia = csa.IndexArgs(ctypes.sizeof(csa.IndexArgs), 1, 1, 8, 96, 4, 8, 16, 1.0, 1.0)
    assert lib.csa_index_topk(ctypes.byref(ia), None, 0, None) == 2
    ia = csa.IndexArgs(ctypes.sizeof(csa.IndexArgs), 1, 1, 9, 128, 4, 8, 16, 1.0, 1.0)
    assert lib.csa_index_topk(ctypes.byref(ia), None, 0, None) == 2
    ia = csa.IndexArgs(ctypes.sizeof(csa.IndexArgs), 1, 1, 8, 128, 4, 0, 16, 1.0, 1.0)
    assert lib.csa_index_topk(ctypes.byref(ia), None, 0, None) == 1
    # index: valid shape, missing pointers -> invalid; workspace query works on the host
    ia = csa.IndexArgs(ctypes.sizeof(csa.IndexArgs), 2, 1, 8, 128, 4, 16, 4096, 1.0, 1.0)
    assert lib.csa_index_topk(ctypes.byref(ia), None, 0, None) == 1
    dummy = 256
    for f in ("q_I", "w", "k_codes", "k_scales", "n_c", "q_pos", "idx_out"):
        setattr(ia, f, dummy)
    ws = lib.csa_index_topk_workspace_size(ctypes.byref(ia))
    assert ws >= 2 * 4096 * 4                                      # materialised scores
    assert lib.csa_index_topk(ctypes.byref(ia), ctypes.c_void_p(dummy), ws - 1, None) == 3
    # attention: unsupported head dim / too many heads
    aa = csa.AttnArgs(ctypes.sizeof(csa.AttnArgs), 1, 1, 8, 256, 32, 4, 16, 8, 0, 128, 1.0, 0.0)
    assert lib.csa_sparse_attn(ctypes.byref(aa), None, 0, None) == 2
    aa = csa.AttnArgs(ctypes.sizeof(csa.AttnArgs), 1, 1, 65, 512, 64, 4, 16, 8, 0, 128, 1.0, 0.0)
    assert lib.hca_dense_attn(ctypes.byref(aa), None, 0, None) == 2
    aa = csa.AttnArgs(ctypes.sizeof(csa.AttnArgs), 1, 1, 64, 512, 64, 4, 16, 8, 0, 128, 1.0, 0.0)
    assert lib.csa_sparse_attn(ctypes.byref(aa), None, 0, None) == 1   # null q / idx
    for bad in (-1.0, float("nan")):                                   # inverse-RoPE base must be >= 0
        aa = csa.AttnArgs(ctypes.sizeof(csa.AttnArgs), 0, 1, 64, 512, 64, 4, 16, 8, 0, 128, 1.0, 0.0)
        aa.out_rope_theta = bad
        assert lib.csa_sparse_attn(ctypes.byref(aa), None, 0, None) == 1
        aa.out_rope_theta = 10000.0
        assert lib.csa_sparse_attn(ctypes.byref(aa), None, 0, None) == 0   # B = 0: nothing to do
    # paged caches: page sizes off the 128-entry tile, or a table too narrow for n_max, are refused
    a = csa.PackArgs(ctypes.sizeof(csa.PackArgs), 1, 4, 64, 0, 300, 1.0, 256, None, 256, 256, None)
    a.pages = csa.PageMap(256, 100, 3, 8)
    assert lib.csa_pack_fp4(ctypes.byref(a), None) == 2
    a.pages = csa.PageMap(256, 128, 2, 8)
    assert lib.csa_pack_fp4(ctypes.byref(a), None) == 1
    ia = csa.IndexArgs(ctypes.sizeof(csa.IndexArgs), 2, 1, 8, 128, 4, 16, 4096, 1.0, 1.0)
    ia.k_pages = csa.PageMap(256, 64, 64, 128)
    assert lib.csa_index_topk(ctypes.byref(ia), None, 0, None) == 2
    # FP8 window: an unknown format is invalid; FP8 on the d = 128 path is unsupported
    aa = csa.AttnArgs(ctypes.sizeof(csa.AttnArgs), 0, 1, 64, 512, 64, 4, 16, 8, 0, 128, 1.0, 0.0)
    aa.win_format = 7
    assert lib.csa_sparse_attn(ctypes.byref(aa), None, 0, None) == 1
    # error-path self-check: the poll count is checked before any launch
    assert lib.csa_check_error_path(0, None) == 1
    assert lib.csa_check_error_path((1 << 20) + 1, None) == 1
    # compress: bad ratio, projection mode with unsupported width
    ca = csa.CompressArgs(ctypes.sizeof(csa.CompressArgs), 1, 8, 64, 64, 0, 0, 0, 0.0)
    assert lib.csa_compress(ctypes.byref(ca), None) == 1


def test_workspace_sizes_scale_with_the_problem(csa):
    lib = csa._lib
    def attn_ws(B, k):
        a = csa.AttnArgs(ctypes.sizeof(csa.AttnArgs), B, 1, 64, 512, 64, 4, 32768, k, 128, 128, 1.0, 0.0)
        for f in ("q", "q_pos", "kv_codes", "kv_scales", "kv_rope", "n_c", "idx", "win_kv", "win_pos0", "out"):
            setattr(a, f, 256)
        return lib.csa_attn_workspace_size(ctypes.byref(a), 0)
    # (without a GPU driver the tensor-core path is not eligible: these are the d = 512 mma.sync plan's sizes;
    # on a B200 a decode query split over 2..4 CTAs keeps per-query counters and bf16 partials there)
    assert attn_ws(32, 512) > 0                                     # decode: split-K partials
    assert attn_ws(1024, 512) == 0                                  # enough queries: no split
    # a size query needs no output buffer (the workspace is sized before the outputs exist)
    a = csa.AttnArgs(ctypes.sizeof(csa.AttnArgs), 32, 1, 64, 512, 64, 4, 32768, 512, 128, 128, 1.0, 0.0)
    for f in ("q", "q_pos", "kv_codes", "kv_scales", "kv_rope", "n_c", "idx", "win_kv", "win_pos0"):
        setattr(a, f, 256)
    assert lib.csa_attn_workspace_size(ctypes.byref(a), 0) == attn_ws(32, 512)
    assert lib.csa_attn_kernel_count(ctypes.byref(a), 0) == 2
    ia = csa.IndexArgs(ctypes.sizeof(csa.IndexArgs), 32, 1, 8, 128, 4, 512, 32768, 1.0, 1.0)
    for f in ("q_I", "w", "k_codes", "k_scales", "n_c", "q_pos"):
        setattr(ia, f, 256)
    assert lib.csa_index_topk_workspace_size(ctypes.byref(ia)) > 0          # idx_out still NULL


def test_attn_kernel_count_host_checks(csa):
    """csa_attn_kernel_count: -1 for arguments the call would reject, 0 for an empty batch, else the
    launches of the plan (the mma.sync plan here: attention + merge when a query is split)."""
    lib = csa._lib

    def args(B, k, Wn=128):
        a = csa.AttnArgs(ctypes.sizeof(csa.AttnArgs), B, 1, 64, 512, 64, 4, 32768, k, Wn, 128, 1.0, 0.0)
        for f in ("q", "q_pos", "kv_codes", "kv_scales", "kv_rope", "n_c", "idx", "win_kv", "win_pos0", "out"):
            setattr(a, f, 256)
        return a
    assert lib.csa_attn_kernel_count(ctypes.byref(args(32, 0)), 0) == -1          # k = 0 for the CSA key set
    bad = args(32, 512)
    bad.struct_size = 4
    assert lib.csa_attn_kernel_count(ctypes.byref(bad), 0) == -1
    assert lib.csa_attn_kernel_count(ctypes.byref(args(0, 512)), 0) == 0
    assert lib.csa_attn_kernel_count(ctypes.byref(args(32, 512)), 0) == 2          # split queries: + merge
    assert lib.csa_attn_kernel_count(ctypes.byref(args(1024, 512)), 0) == 1        # one CTA per query
