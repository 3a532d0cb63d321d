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


def test_host_argument_validation_without_gpu(lib):
    # null pointers and bad shapes are rejected before anything touches CUDA
    assert lib.bsa_tile_permute(None, None, 1, 2, 2, 2, 1, 1, 1, 256, 8, None) == 1
    assert lib.bsa_sta_mask(1, 1, 1, 1, 1, 1, 0, None, None) == 1
    assert lib.bsa_radial_mask(10, 4, 4, None, None) == 1
    assert lib.bsa_mask_compact(None, 4, 4, None, None, None) == 1
    fake = ctypes.c_void_p(16)
    # unsupported head_dim / block sizes -> BSA_ERR_UNSUPPORTED
    args = [fake, fake, fake, 1, 2, 256, 256, 96, 128, 128, fake, fake, 1, 0.0, fake, fake, fake,
            1 << 20, None]
    assert lib.bsa_attn_fwd(*args) == 2
    args[7], args[8] = 128, 192
    assert lib.bsa_attn_fwd(*args) == 2
    # workspace too small -> BSA_ERR_WORKSPACE
    args[8] = 128
    args[17] = 16
    assert lib.bsa_attn_fwd(*args) == 3
    # list_heads must be 1 or batch*heads
    args[12] = 3
    assert lib.bsa_attn_fwd(*args) == 1


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


def test_header_compiles_as_c_and_links(tmp_path, lib):
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
  if (bsa_version() < 100) return 1;
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
