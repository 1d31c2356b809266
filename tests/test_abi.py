"""The C ABI library without a GPU: it loads, exports every entry point that
include/atom.h declares, and rejects bad arguments on the host before any CUDA
call (so these checks run on a machine with no GPU at all)."""
import ctypes as ct
import os
import re

import pytest

from w4a4_mixed_precision_b200 import atom

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "atom.h")

OK, INVALID, SHAPE, ALIGN, UNSUPPORTED = 0, 1, 2, 3, 4

# fake, never-dereferenced device addresses: aligned and misaligned
A16 = 0x10000
MIS = 0x10001


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(atom_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from w4a4_mixed_precision_b200 import build
    build.build()
    return atom.lib()


def test_header_declares_the_hot_path_entry_points():
    names = declared_functions()
    for required in ("atom_reorder_quant", "atom_quant_weights", "atom_w4a4_gemm",
                     "atom_w4a4_gemm_partials"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(declared_functions()) <= set(atom.SIGNATURES)


def test_status_strings_and_version(lib):
    for code, name in atom.STATUS.items():
        assert atom.atom_status_string(code) == name
    assert atom.atom_status_string(99) == "ATOM_ERR_UNKNOWN"
    assert atom.atom_version() >= 100
    assert atom.atom_gemm_workspace_bytes(8192, 28672, 8192) == 0


def quant(lib, x=A16, M=4, K=512, ld=512, idx=A16, n_out=128, group=128, q4=A16, q8=A16,
          sc=A16, fn="atom_reorder_quant"):
    return getattr(lib, fn)(x, M, K, ld, idx, n_out, group, q4, q8, sc, None)


@pytest.mark.parametrize("fn", ["atom_reorder_quant", "atom_quant_weights"])
@pytest.mark.parametrize("kw,expect", [
    (dict(K=500, ld=504), SHAPE),          # K not a multiple of 128
    (dict(K=128, ld=128), SHAPE),          # K < 256 (needs one INT4 group + the outlier group)
    (dict(K=65536, ld=65536), SHAPE),      # K above the staged-permutation limit
    (dict(ld=508), SHAPE),                 # ld < K
    (dict(ld=516), SHAPE),                 # ld not a multiple of 8 (16-byte rows)
    (dict(group=64), UNSUPPORTED),
    (dict(n_out=64), UNSUPPORTED),
    (dict(M=-1), INVALID),
    (dict(x=0), INVALID),
    (dict(idx=0), INVALID),
    (dict(q4=0), INVALID),
    (dict(sc=0), INVALID),
    (dict(x=MIS), ALIGN),
    (dict(q8=A16 + 8), ALIGN),
    (dict(sc=A16 + 2), ALIGN),
    (dict(M=0), OK),                       # empty input: nothing to do, nothing launched
])
def test_quantizer_host_validation(lib, fn, kw, expect):
    assert quant(lib, fn=fn, **kw) == expect


def gemm(lib, qa4=A16, qa8=A16, sa=A16, qw4=A16, qw8=A16, sw=A16, y=A16, M=16, N=256, K=512,
         n_out=128, group=128):
    return lib.atom_w4a4_gemm(qa4, qa8, sa, qw4, qw8, sw, y, M, N, K, n_out, group, None, 0, None)


@pytest.mark.parametrize("kw,expect", [
    (dict(K=384 + 64), SHAPE),
    (dict(N=260), SHAPE),                  # N must be a multiple of 8
    (dict(N=0), SHAPE),
    (dict(M=-3), INVALID),
    (dict(y=0), INVALID),
    (dict(sw=0), INVALID),
    (dict(qa4=MIS), ALIGN),
    (dict(y=A16 + 4), ALIGN),
    (dict(group=256), UNSUPPORTED),
    (dict(M=0), OK),
])
def test_gemm_host_validation(lib, kw, expect):
    assert gemm(lib, **kw) == expect


def test_partials_host_validation(lib):
    f = lib.atom_w4a4_gemm_partials
    args = [A16] * 6
    assert f(*args, 0, A16, 16, 256, 512, 128, 128, None) == INVALID      # no partials buffer
    assert f(*args, A16 + 4, None, 16, 256, 512, 128, 128, None) == ALIGN
    assert f(*args, A16, None, 16, 250, 512, 128, 128, None) == SHAPE
    assert f(*args, A16, None, 0, 256, 512, 128, 128, None) == OK


def test_python_binding_refuses_cpu_tensors(lib):
    import torch
    x = torch.zeros((4, 256), dtype=torch.float16)
    idx = torch.arange(128, dtype=torch.int32)
    with pytest.raises(ValueError):
        atom.atom_reorder_quant(x, idx)


def w8a8(lib, qa=A16, sa=A16, qw=A16, sw=A16, y=A16, M=256, N=256, K=256):
    return lib.atom_w8a8_gemm(qa, sa, qw, sw, y, M, N, K, None)


def test_w8a8_checks_arguments_on_the_host(lib):
    assert w8a8(lib, M=0) == OK
    assert w8a8(lib, N=0) == OK
    assert w8a8(lib, M=-1) == INVALID
    assert w8a8(lib, K=8) == SHAPE          # K below 16
    assert w8a8(lib, K=264) == SHAPE        # K % 16 != 0
    assert w8a8(lib, K=131072 + 16) == SHAPE   # the int32 sum could overflow
    assert w8a8(lib, N=260) == SHAPE        # N % 8 != 0
    assert w8a8(lib, qa=0) == INVALID
    assert w8a8(lib, y=0) == INVALID
    assert w8a8(lib, qa=MIS) == ALIGN
    assert w8a8(lib, qw=A16 + 8) == ALIGN
    assert w8a8(lib, sw=A16 + 4) == ALIGN   # sw is read as 16-byte vectors
    assert w8a8(lib, sa=MIS) == ALIGN


def test_kv_checks_arguments_on_the_host(lib):
    assert lib.atom_kv_quant(A16, 0, A16, A16, None) == OK
    assert lib.atom_kv_dequant(A16, A16, 0, A16, None) == OK
    assert lib.atom_kv_quant(A16, -1, A16, A16, None) == INVALID
    assert lib.atom_kv_quant(0, 4, A16, A16, None) == INVALID
    assert lib.atom_kv_dequant(A16, 0, 4, A16, None) == INVALID
    assert lib.atom_kv_quant(A16 + 8, 4, A16, A16, None) == ALIGN     # x: 16 bytes
    assert lib.atom_kv_quant(A16, 4, A16 + 4, A16, None) == ALIGN     # q4: 8 bytes
    assert lib.atom_kv_quant(A16, 4, A16, MIS, None) == ALIGN         # scales: 4 bytes
    assert lib.atom_kv_dequant(A16, A16, 4, A16 + 8, None) == ALIGN   # out: 16 bytes


def test_header_compiles_as_plain_c(tmp_path):
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "use_atom.c"
    src.write_text('#include "atom.h"\nint main(void) { return atom_status_string(ATOM_OK) == 0; }\n')
    r = subprocess.run([cc, "-std=c99", "-Wall", "-Werror", "-fsyntax-only", "-I",
                        os.path.join(ROOT, "include"), str(src)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


def gemm_quant(lib, M=16, N=256, K=512, n_out=128, group=128, qy4=A16, qy8=A16, sy=A16, qa4=A16):
    return lib.atom_w4a4_gemm_quant(qa4, A16, A16, A16, A16, A16, M, N, K, n_out, group,
                                    qy4, qy8, sy, None)


def test_quantizing_gemm_checks_arguments_on_the_host(lib):
    assert gemm_quant(lib, M=0) == OK
    assert gemm_quant(lib, N=200) == SHAPE            # not whole 128-column groups
    assert gemm_quant(lib, N=128) == SHAPE            # needs an INT4 group and the INT8 group
    assert gemm_quant(lib, N=32768 + 128) == SHAPE    # above the next layer's largest K
    assert gemm_quant(lib, qy4=0) == INVALID
    assert gemm_quant(lib, sy=0) == INVALID
    assert gemm_quant(lib, qy8=A16 + 8) == ALIGN
    assert gemm_quant(lib, sy=MIS) == ALIGN
    assert gemm_quant(lib, qa4=MIS) == ALIGN
    assert gemm_quant(lib, group=64) == UNSUPPORTED


def test_w4a8_entry_points_check_arguments_on_the_host(lib):
    q = lib.atom_reorder_quant_a8
    assert q(A16, 0, 512, 512, A16, 128, 128, A16, A16, None) == OK
    assert q(A16, 4, 500, 504, A16, 128, 128, A16, A16, None) == SHAPE
    assert q(A16, 4, 512, 512, A16, 128, 128, 0, A16, None) == INVALID
    assert q(A16, 4, 512, 512, A16, 128, 128, A16 + 8, A16, None) == ALIGN
    assert q(A16, 4, 512, 512, A16, 128, 64, A16, A16, None) == UNSUPPORTED
    g = lib.atom_w4a8_gemm
    args = [A16] * 5
    assert g(*args, A16, 0, 256, 512, 128, 128, None) == OK
    assert g(*args, 0, 16, 256, 512, 128, 128, None) == INVALID       # no y
    assert g(*args, A16, 16, 260, 512, 128, 128, None) == SHAPE       # N % 8 != 0
    assert g(MIS, *args[1:], A16, 16, 256, 512, 128, 128, None) == ALIGN
    assert g(*args, A16, 16, 256, 512, 64, 128, None) == UNSUPPORTED
    p = lib.atom_w4a8_gemm_partials
    assert p(*args, 0, A16, 16, 256, 512, 128, 128, None) == INVALID  # no partials buffer
    assert p(*args, A16 + 4, None, 16, 256, 512, 128, 128, None) == ALIGN


def test_timeout_aid_validates_its_limit_on_the_host(lib):
    """atom_debug_wait_timeout rejects a zero limit and one above the
    production 1 s before touching the device."""
    assert lib.atom_debug_wait_timeout(0, None) == INVALID
    assert lib.atom_debug_wait_timeout(2_000_000_000, None) == INVALID


def test_tiled_layout_entry_points_check_arguments_on_the_host(lib):
    assert lib.atom_tiled_weights_bytes(264, 1152) == 3 * 8 * 8192
    assert lib.atom_tiled_weights_bytes(0, 1152) == 0
    assert lib.atom_tiled_weights_bytes(264, 1000) == 0
    for fn in (lib.atom_pack_weights_tiled, lib.atom_unpack_weights_tiled):
        assert fn(A16, 0, 512, A16, None) == OK          # nothing to do
        assert fn(A16, -1, 512, A16, None) == INVALID
        assert fn(A16, 16, 500, A16, None) == SHAPE
        assert fn(A16, 16, 128, A16, None) == SHAPE
        assert fn(0, 16, 512, A16, None) == INVALID
        assert fn(A16, 16, 512, 0, None) == INVALID
        assert fn(MIS, 16, 512, A16, None) == ALIGN
        assert fn(A16, 16, 512, A16 + 8, None) == ALIGN
    g = lib.atom_w4a4_gemm_tiled
    args = [A16] * 6
    assert g(*args, A16, 0, 256, 512, 128, 128, None, 0, None) == OK
    assert g(*args, 0, 16, 256, 512, 128, 128, None, 0, None) == INVALID    # no y
    assert g(*args, A16, 16, 260, 512, 128, 128, None, 0, None) == SHAPE    # N % 8 != 0
    assert g(A16, A16, A16, MIS, A16, A16, A16, 16, 256, 512, 128, 128, None, 0, None) == ALIGN
    assert g(*args, A16, 16, 256, 512, 64, 128, None, 0, None) == UNSUPPORTED
