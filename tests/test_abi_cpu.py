"""The C-ABI library without a GPU: it loads, exports every function include/csa.h declares, sizes
workspaces, and rejects bad host arguments before touching the device."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "csa.h")


@pytest.fixture(scope="module")
def lib():
    from fp4_compressed_sparse_kv_b200 import build, csa
    build.build()
    return csa.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(csa_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ["csa_kv_pack_fp4", "csa_indexer_full", "csa_indexer_reindex", "csa_index_reuse",
              "csa_sparse_decode_attn", "csa_decode_layer", "csa_workspace_bytes",
              "csa_workspace_init", "csa_check_device_error", "csa_status_string"]:
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    from fp4_compressed_sparse_kv_b200 import csa
    out = subprocess.run(["nm", "-D", "--defined-only", csa.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\sT\s(csa_\w+)", out))
    for n in declared_functions():
        assert n in exported, n
        assert getattr(lib, n) is not None
    assert set(csa.EXPORTS) <= exported


def test_status_strings(lib):
    for s in range(7):
        assert lib.csa_status_string(s)
    assert lib.csa_status_string(3) == b"workspace too small"


def test_workspace_sizes(lib):
    f = lib.csa_workspace_bytes
    assert f(8, 64, 131072, 2048) > 0
    assert f(8, 64, 131072, 2048) >= f(8, 64, 131072, 512) >= f(8, 16, 131072, 512)
    assert f(1, 16, 4096, 64) > 256
    # invalid sizes give 0
    assert f(0, 64, 1000, 64) == 0
    assert f(1, 24, 1000, 64) == 0
    assert f(1, 64, 0, 64) == 0
    assert f(1, 64, 1 << 25, 64) == 0
    assert f(1, 64, 1000, 0) == 0
    assert f(1, 64, 1000, 8193) == 0


def test_bad_host_arguments_return_before_launch(lib):
    from fp4_compressed_sparse_kv_b200 import csa
    null = None
    # null layer / batch
    assert lib.csa_indexer_full(null, null, null, null, 64, null, null, null, 0, null) == 1
    assert lib.csa_sparse_decode_attn(null, null, null, 64, ctypes.c_float(0.1), null, null, 64, null,
                                      null, null, 0, null) == 1
    assert lib.csa_index_reuse(0, null, null, 1, null, null, 1, null, 0, null) == 1
    assert lib.csa_workspace_init(null, 256, null) == 1
    assert lib.csa_check_device_error(null, null, null) == 1
    # misaligned pointers are rejected too
    fake = ctypes.c_void_p(0x1000)
    odd = ctypes.c_void_p(0x1001)
    layer = csa.KVLayerC(0x1000, 0x1000, odd.value, 0x1000, 0x1000, 4, 1)
    assert lib.csa_kv_pack_fp4(ctypes.byref(layer), fake, fake, fake, null, 1, fake, 256, null) == 1
    # n == 0 is a no-op
    assert lib.csa_kv_pack_fp4(null, null, null, null, null, 0, null, 0, null) == 0


def test_screen_and_full_indexer_host_checks(lib):
    """Argument and workspace checks of the screened Full indexer happen on the host, before any
    launch: null or misaligned pointers, a bounds stride below ceil(max_seq_len / 8), and a workspace
    smaller than csa_workspace_bytes asks for."""
    from fp4_compressed_sparse_kv_b200 import csa
    null = None
    fake = ctypes.c_void_p(0x1000)
    lay = csa.KVLayerC(0x1000, 0x1000, 0x1000, 0x1000, 0x1000, 64, 1)
    bat = csa.BatchC(2, 0x1000, 0x1000, 64, 0x1000, 4096)   # B=2, max_seq_len 4,096: 512 blocks
    args = (ctypes.byref(lay), ctypes.byref(bat), fake, fake, fake, fake)
    assert lib.csa_indexer_screen_bounds(null, null, null, null, null, null, 512, null, 0, null) == 1
    assert lib.csa_indexer_screen_bounds(*args, 511, fake, 1 << 30, null) == 1       # stride too small
    odd = ctypes.c_void_p(0x1004)
    assert lib.csa_indexer_screen_bounds(ctypes.byref(lay), ctypes.byref(bat), fake, fake, odd, fake, 512, fake,
                                         1 << 30, null) == 1
    need = lib.csa_workspace_bytes(2, 16, 4096, 1)
    assert need > 0
    assert lib.csa_indexer_screen_bounds(*args, 512, fake, 256, null) == 3            # workspace too small
    assert lib.csa_indexer_full(ctypes.byref(lay), ctypes.byref(bat), fake, fake, 64, fake, fake, fake, 300,
                                null) == 3
    assert lib.csa_indexer_full(ctypes.byref(lay), ctypes.byref(bat), fake, fake, 0, fake, fake, fake, 1 << 30,
                                null) == 1                                               # k out of range


def test_binding_refuses_host_tensors():
    import torch
    from fp4_compressed_sparse_kv_b200 import csa
    with pytest.raises(ValueError):
        csa._ptr(torch.zeros(4), "x")


def test_persistent_record_sizes_and_host_checks(lib):
    import ctypes as C
    for n, want in [(0, 0), (1, 26624), (64, 26624), (65, 53248), (1 << 20, 16384 * 26624), (-1, 0)]:
        assert lib.csa_kv_record_bytes(n) == want
    ws = (C.c_uint8 * 272)()
    wsp = (C.addressof(ws) + 15) // 16 * 16
    # n = 0 is a no-op; a null layer or a negative n is refused before anything reaches the device
    assert lib.csa_kv_export(None, None, 0, None, None, 0, None) == 0
    assert lib.csa_kv_export(None, C.c_void_p(wsp), 64, C.c_void_p(wsp), C.c_void_p(wsp), 256, None) == 1
    assert lib.csa_kv_import(None, C.c_void_p(wsp), -5, C.c_void_p(wsp), C.c_void_p(wsp), 256, None) == 1
