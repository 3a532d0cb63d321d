"""The C-ABI library builds, loads and exports every entry point of include/bsa.h (CPU only).

No compute call is made; the argument checks exercised here return before any
CUDA call, so they run without a GPU.
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "bsa.h")


@pytest.fixture(scope="module")
def no_gpu():
    """The argument-check cases pass stand-in pointers (small integers): a case
    that got past the checks would reach CUDA with them.  Without a GPU that can
    only fail with an error code, so these cases run only where no GPU is visible."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("argument-check cases use stand-in pointers; they run where no GPU is visible")


@pytest.fixture(scope="module")
def lib():
    from block_sparse_attention_tokens_b200 import build, binding
    if not os.path.exists(binding._LIB_PATH):
        build.build()
    return binding.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(bsa_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_path(lib):
    names = declared_functions()
    for must in ("bsa_tile_permute", "bsa_tile_untile", "bsa_sta_mask", "bsa_radial_mask",
                 "bsa_nabla_mask", "bsa_mask_compact", "bsa_attn_fwd"):
        assert must in names


def test_every_declared_symbol_is_exported(lib):
    from block_sparse_attention_tokens_b200 import binding
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(declared_functions()) <= set(binding.EXPORTS) | {"bsa_status_string"}


def test_status_strings_and_version(lib):
    assert lib.bsa_status_string(0) == b"BSA_OK"
    assert lib.bsa_status_string(5) == b"BSA_ERR_TIMEOUT"
    assert lib.bsa_version() >= 100


def test_host_argument_validation_without_gpu(lib, no_gpu):
    # null pointers and bad shapes are rejected before anything touches CUDA
    assert lib.bsa_tile_permute(None, None, 1, 2, 2, 2, 1, 1, 1, 256, 8, 0, 0, None) == 1
    assert lib.bsa_sta_mask(1, 1, 1, 1, 1, 1, 0, None, None) == 1
    assert lib.bsa_radial_mask(10, 4, 4, None, None) == 1
    assert lib.bsa_mask_compact(None, 4, 4, None, None, None) == 1
    fake = ctypes.c_void_p(16)
    # unsupported head_dim / block sizes -> BSA_ERR_UNSUPPORTED
    # q k v B H nq nk d qkv_stride o_stride bq bk row_ptr col_idx list_heads scale o lse ws ws_bytes
    args = [fake, fake, fake, 1, 2, 256, 256, 96, 0, 0, 128, 128, fake, fake, 1, 0.0, fake, fake,
            fake, 1 << 20, None]
    assert lib.bsa_attn_fwd(*args) == 2
    args[7], args[10] = 128, 192
    assert lib.bsa_attn_fwd(*args) == 2
    # workspace too small -> BSA_ERR_WORKSPACE
    args[10] = 128
    args[19] = 16
    assert lib.bsa_attn_fwd(*args) == 3
    # list_heads must be 1 or batch*heads
    args[14] = 3
    assert lib.bsa_attn_fwd(*args) == 1
    # row strides: shorter than a row (2 heads x 128), or rows not 16-byte aligned
    args[14] = 1
    for i, val in ((8, 128), (8, 260), (9, 255)):
        bad = list(args)
        bad[i] = val
        assert lib.bsa_attn_fwd(*bad) == 1, (i, val)


def test_every_entry_rejects_bad_arguments_before_touching_cuda(lib, no_gpu):
    """Each case below is refused by the host-side checks, which run before any
    CUDA call: null pointers, unaligned pointers, unsupported head sizes and block
    sizes, inconsistent ranges, too small a workspace, overlapping buffers."""
    A = ctypes.c_void_p(16)          # 16-byte aligned stand-in; never dereferenced here
    U = ctypes.c_void_p(8)           # not 16-byte aligned
    INV, UNS, WS = 1, 2, 3
    # backward: q k v o dO lse B H nq nk d qkv_rs o_rs bq bk row_ptr col_idx list_heads scale
    #           dq dk dv ws ws_bytes
    bwd = [A, A, A, A, A, A, 1, 2, 256, 256, 128, 0, 0, 128, 128, A, A, 1, 0.0, A, A, A, A, 1 << 30,
           None]
    assert lib.bsa_attn_bwd(*([None] * 6 + bwd[6:15] + [None, None] + bwd[17:19] + [None] * 4
                               + bwd[23:])) == INV
    for i, val, rc in ((10, 96, UNS), (13, 192, UNS), (23, 16, WS), (17, 3, INV), (0, U, INV),
                       (22, U, INV), (11, 200, INV), (12, 260, INV)):
        args = list(bwd)
        args[i] = val
        assert lib.bsa_attn_bwd(*args) == rc, (i, val)
    # paged forward: q kp vp n_pool table ppb B H nq nk d bq bk row_ptr col_idx list_heads scale o lse ws ws_bytes
    paged = [A, A, A, 8, A, 4, 1, 2, 200, 500, 128, 128, 128, A, A, 2, 0.0, A, A, A, 1 << 30, None]
    args = list(paged)
    args[4] = None
    assert lib.bsa_attn_fwd_paged(*args) == INV                  # no page table
    args = list(paged)
    args[12] = 384
    assert lib.bsa_attn_fwd_paged(*args) == UNS                  # key block larger than a page
    args = list(paged)
    args[5] = 3
    assert lib.bsa_attn_fwd_paged(*args) == INV                  # 500 keys need 4 pages
    args = list(paged)
    args[6], args[15] = 2, 1
    assert lib.bsa_attn_fwd_paged(*args) == UNS                  # one shared list, two page tables
    # allocation-free forward: q k v B H nq nk d bq bk row_ptr col_idx list_heads scale o lse status
    # (the same checks, order and codes as bsa_attn_fwd come before the size check)
    na = [A, A, A, 1, 40, 453600, 453600, 128, 96, 128, A, A, 40, 0.0, A, A, A, None]
    assert lib.bsa_attn_fwd_noalloc(*na) == UNS                  # block 96, as bsa_attn_fwd
    na[8] = 128
    assert lib.bsa_attn_fwd_noalloc(*na) == WS                   # needs more than the fixed 8 MiB
    for i, val, rc in ((0, U, INV), (14, None, INV), (7, 96, UNS), (12, 3, INV), (10, None, INV)):
        args = list(na)
        args[i] = val
        assert lib.bsa_attn_fwd_noalloc(*args) == rc, (i, val)   # refused before the size
    # NABLA: select (qbar kbar B H QB KB d p scale kb_begin kb_end force base allowed mask near)
    sel = [A, A, 1, 2, 8, 8, 128, 0.9, 0.0, 0, 8, 0, None, None, A, None, None]
    for i, val, rc in ((7, 0.0, INV), (6, 96, UNS), (10, 9, INV), (9, 5, INV), (0, None, INV)):
        args = list(sel)
        args[i] = val
        if i == 9:
            args[10] = 4                                         # kb_begin > kb_end
        assert lib.bsa_nabla_select(*args) == rc, (i, val)
    # NABLA mask (q k B H nq nk d row_stride block p scale kb_begin kb_end force mask near ws
    #             ws_bytes)
    nm = [A, A, 1, 2, 1000, 1000, 128, 0, 64, 0.9, 0.0, 0, 16, 0, A, None, A, 1 << 30, None]
    for i, val, rc in ((8, 8, INV), (8, 72, INV), (17, 64, WS), (0, U, INV), (12, 17, INV),
                       (6, 32, UNS), (7, 250, INV), (7, 260, INV)):
        args = list(nm)
        args[i] = val
        assert lib.bsa_nabla_mask(*args) == rc, (i, val)
    # permutes: x y B T H W tT tH tW row_bytes n_pad x_stride y_stride (bytes)
    for f in (lib.bsa_tile_permute, lib.bsa_tile_untile):
        base = [A, ctypes.c_void_p(1 << 40), 1, 4, 8, 8, 4, 4, 4, 256, 256, 0, 0, None]
        for i, val in ((9, 8), (9, 24), (10, 255), (1, A), (0, U), (6, 0), (11, 128), (12, 264)):
            args = list(base)
            args[i] = val
            assert f(*args) == INV, (f, i, val)
    # fused permute + pooling: x y B T H W tT tH tW heads d n_pad block pooled x_rs y_rs
    pp = [A, ctypes.c_void_p(1 << 40), 1, 4, 8, 8, 4, 4, 4, 2, 128, 256, 64, A, 0, 0, None]
    for i, val in ((11, 250), (12, 96), (12, 2048), (10, 12), (1, A), (13, U), (14, 128),
                   (15, 260)):
        args = list(pp)
        args[i] = val
        assert lib.bsa_tile_permute_pool(*args) == INV, (i, val)
    # per-head slicing: x y B T H W shapes n_shapes choice heads d n_pad block pooled x_rs y_rs
    # status  (untile: y x B T H W shapes n_shapes choice heads d n_pad y_rs x_rs status)
    menu = (ctypes.c_int * 6)(4, 4, 4, 1, 8, 8)
    bad_menu = (ctypes.c_int * 6)(4, 4, 4, 1, 0, 8)
    Y = ctypes.c_void_p(1 << 40)
    sp = [A, Y, 1, 4, 8, 8, menu, 2, A, 2, 128, 256, 64, A, 0, 0, None, None]
    for i, val, rc in ((6, None, INV), (7, 0, INV), (7, 9, INV), (6, bad_menu, INV), (8, None, INV),
                       (8, ctypes.c_void_p(18), INV), (10, 12, INV), (10, 2048, UNS), (11, 255, INV), (12, 48, INV),
                       (12, 2048, INV), (13, U, INV), (14, 250, INV), (15, 260, INV), (1, A, INV)):
        args = list(sp)
        args[i] = val
        assert lib.bsa_scheme_permute(*args) == rc, (i, val)
    su = [A, Y, 1, 4, 8, 8, menu, 2, A, 2, 128, 256, 0, 0, None, None]
    for i, val, rc in ((6, None, INV), (7, 9, INV), (8, None, INV), (11, 255, INV),
                       (12, 250, INV), (13, 260, INV), (1, A, INV), (10, 2048, UNS)):
        args = list(su)
        args[i] = val
        assert lib.bsa_scheme_untile(*args) == rc, (i, val)
    # SICS: blocks (x B T H W tT tH tW heads d row_stride out) and scheme
    sb = [A, 1, 4, 8, 8, 4, 4, 4, 2, 128, 0, A, None]
    for i, val, rc in ((9, 96, UNS), (5, 300, UNS), (8, 200, UNS), (0, U, INV), (2, 0, INV),
                       (10, 128, INV), (10, 260, INV)):
        args = list(sb)
        args[i] = val
        assert lib.bsa_sics_blocks(*args) == rc, (i, val)
    shapes = (ctypes.c_int * 6)(4, 4, 4, 1, 8, 8)
    need = lib.bsa_sics_workspace_size(1, 2, 4, 8, 8, shapes, 2)
    assert need == 4 * 2 * 1 * 2 * (4 + 4)
    sch = [A, A, 1, 4, 8, 8, 2, 128, 0, shapes, 2, A, A, A, need, None]
    for i, val, rc in ((10, 0, INV), (10, 17, INV), (14, need - 4, WS), (1, U, INV),
                       (8, 200, INV)):
        args = list(sch)
        args[i] = val
        assert lib.bsa_sics_scheme(*args) == rc, (i, val)
    # paged cache: write (src B n_new H d first table ppb pool n_pool status)
    kw = [A, 1, 100, 2, 128, 0, A, 1, A, 4, None, None]
    for i, val, rc in ((0, None, INV), (4, 4, UNS), (5, 40, INV), (2, 0, INV), (8, U, INV)):
        args = list(kw)
        args[i] = val
        assert lib.bsa_kv_write(*args) == rc, (i, val)
    # block means (x table ppb B n_tokens H d block first n out out_blocks)
    bp = [A, A, 4, 1, 500, 2, 128, 64, 0, 8, A, 8, None]
    for i, val, rc in ((9, 9, INV), (6, 96, UNS), (2, 3, INV), (8, -1, INV), (10, None, INV)):
        args = list(bp)
        args[i] = val
        assert lib.bsa_block_pool(*args) == rc, (i, val)
    assert lib.bsa_kv_resident_blocks(None, 1, 4, 64, 8, A, None) == INV
    assert lib.bsa_kv_resident_blocks(A, 1, 4, 96, 8, A, None) == UNS
    # page scores (qbar kbar B H QB KB d scale kb_begin kb_end allowed block n_pages scores)
    ps = [A, A, 1, 2, 4, 16, 128, 0.1, 2, 12, None, 64, 8, A, None]
    for i, val, rc in ((6, 96, UNS), (9, 17, INV), (8, 13, INV), (11, 96, INV), (13, None, INV)):
        args = list(ps)
        args[i] = val
        assert lib.bsa_kv_page_scores(*args) == rc, (i, val)
    # keep/evict (scores B n_pages anchors recent_begin budget table ppb freed freed_count)
    kp = [A, 1, 40, 4, 32, 10, A, 40, A, A, None]
    for i, val, rc in ((3, 33, INV), (4, 41, INV), (7, 39, INV), (5, -1, INV), (8, None, INV)):
        args = list(kp)
        args[i] = val
        assert lib.bsa_kv_keep_pages(*args) == rc, (i, val)
    args = list(kp)
    args[2], args[3], args[4], args[7] = 9000, 0, 8193, 9000
    assert lib.bsa_kv_keep_pages(*args) == UNS                   # one CTA ranks <= 8192 pages
    args = list(kp)
    args[3] = args[4] = 10
    assert lib.bsa_kv_keep_pages(*args) == 0                     # no middle pages: nothing to do
    # status read-back and the bounded-wait self-test
    status = ctypes.c_int(0)
    assert lib.bsa_read_status(None, ctypes.byref(status), None) == INV
    assert lib.bsa_wait_selftest(None, 1000, None) == INV
    assert lib.bsa_wait_selftest(A, 0, None) == INV
    assert lib.bsa_wait_selftest(A, 20_000_000_000, None) == INV


def test_workspace_sizes(lib):
    ws = lib.bsa_attn_workspace_size(1, 24, 115200, 115200, 384, 384, 1)
    # status + counts + one 128-key tile entry per (q-block, k-block, k-tile)
    assert ws >= 300 * 300 * 3 * 4
    assert lib.bsa_attn_workspace_size(1, 1, 1, 1, 96, 128, 1) == 0
    assert lib.bsa_nabla_workspace_size(1, 40, 32760, 32760, 128, 64) == 256 + 4 * 40 * 128 * 1024


def declared_prototypes():
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    protos = {}
    for m in re.finditer(r"\b(bsa_[a-z0-9_]+)\s*\(([^)]*)\)\s*;", text):
        params = [p.strip() for p in m.group(2).split(",") if p.strip() and p.strip() != "void"]
        protos[m.group(1)] = params
    return protos


def test_binding_argument_counts_match_the_header(lib):
    protos = declared_prototypes()
    assert protos, "no prototypes parsed"
    for name, params in protos.items():
        f = getattr(lib, name)
        assert f.argtypes is not None, name
        assert len(f.argtypes) == len(params), (name, len(f.argtypes), len(params))


def test_header_compiles_as_c_and_links(tmp_path, lib, no_gpu):
    """A plain C program includes bsa.h, links libbsa.so and calls entry points whose
    argument checks run before any CUDA call (no GPU needed)."""
    import shutil
    import subprocess
    from block_sparse_attention_tokens_b200 import binding
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "use_bsa.c"
    src.write_text(r"""
#include <stdio.h>
#include "bsa.h"
int main(void) {
  if (bsa_version() < 200) return 1;
  if (bsa_sta_mask(1, 1, 1, 1, 1, 1, 0, NULL, NULL) != BSA_ERR_INVALID_ARG) return 2;
  if (bsa_attn_workspace_size(1, 1, 1, 1, 96, 128, 1) != 0) return 3;
  printf("%s\n", bsa_status_string(BSA_ERR_TIMEOUT));
  return 0;
}
""")
    exe = tmp_path / "use_bsa"
    lib_dir = os.path.dirname(binding._LIB_PATH)
    subprocess.run([gcc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    str(src), "-L", lib_dir, "-lbsa", f"-Wl,-rpath,{lib_dir}", "-o", str(exe)],
                   check=True, capture_output=True, text=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0, (out.returncode, out.stderr)
    assert out.stdout.strip() == "BSA_ERR_TIMEOUT"


def test_binding_fails_loudly_without_the_library(tmp_path):
    """A copy of the package with no libbsa.so: the first binding call raises
    ImportError; nothing falls back to another implementation."""
    import shutil
    import subprocess
    import sys
    pkg = os.path.join(ROOT, "block_sparse_attention_tokens_b200")
    dst = tmp_path / "block_sparse_attention_tokens_b200"
    shutil.copytree(pkg, dst, ignore=shutil.ignore_patterns("*.so", "csrc", "__pycache__"))
    code = ("from block_sparse_attention_tokens_b200 import binding, configs\n"
            "from block_sparse_attention_tokens_b200.pipeline import Plan\n"
            "for call in (lambda: binding.bsa_attn_workspace_size(1, 1, 128, 128, 128, 128, 1),\n"
            "             lambda: Plan(configs.get('sta_tiny'), 'cpu')):\n"
            "    try:\n"
            "        call()\n"
            "    except ImportError as e:\n"
            "        assert 'libbsa.so not found' in str(e)\n"
            "    else:\n"
            "        raise SystemExit('no error without the library')\n"
            "print('refused')\n")
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True,
                         cwd=str(tmp_path), env={**os.environ, "PYTHONPATH": str(tmp_path)})
    assert out.returncode == 0 and out.stdout.strip() == "refused", out.stderr[-2000:]
