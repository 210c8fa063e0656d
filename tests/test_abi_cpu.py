"""The C-ABI library builds, loads and exports what its header declares (CPU only).

No compute call is made here: these tests run where there is no GPU.
"""
import ctypes
import os
import subprocess

import pytest
import torch

import post_quantization_column_b200 as awq


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(awq.library_path()):
        from post_quantization_column_b200 import build
        build.build()
    return awq.library()


def test_header_declares_the_search_entry_points():
    names = awq.exported_functions()
    for required in ("awq_search", "awq_search_f32", "awq_search_ex", "awq_search_host", "awq_search_host_batch",
                     "awq_status_string"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    missing = [n for n in awq.exported_functions() if not hasattr(lib, n)]
    assert not missing, f"declared in the header but not exported: {missing}"
    out = subprocess.run(["nm", "-D", "--defined-only", awq.library_path()], capture_output=True, text=True)
    if out.returncode == 0:
        exported = {line.split()[-1] for line in out.stdout.splitlines() if " T " in line}
        assert set(awq.exported_functions()) <= exported


def test_status_strings_and_host_only_helpers(lib):
    assert awq.status_string(0) == "AWQ_OK"
    assert awq.status_string(6) == "AWQ_ERR_TIMEOUT"
    assert awq.status_string(99) == "AWQ_ERR_UNKNOWN"
    assert awq.tile_shape() == (128, 256)
    assert lib.awq_version() >= 1
    # 20 candidates + the reference copy of W, the tiled reference output, partials
    b = awq.workspace_bytes(4096, 4096, 4096, 128, 20)
    assert b >= 21 * 4096 * 4096 * 2 + 4096 * 4096 * 4
    assert awq.workspace_bytes(4096, 4096, 4100, 128, 20) == 0   # N % 8 != 0
    assert awq.workspace_bytes(4096, 4000, 4096, 128, 20) == 0   # K % group != 0


def test_argument_validation_happens_before_any_device_work(lib):
    # NULL pointers and bad shapes are rejected on the host; no CUDA call is reached
    null = ctypes.c_void_p(0)
    st = lib.awq_search(null, null, 16, 128, 64, 128, 20, null, null, null, null, null, null)
    assert st == 1
    assert b"NULL" in lib.awq_last_error_message()
    buf = ctypes.create_string_buffer(64)
    p = ctypes.cast(buf, ctypes.c_void_p)
    assert lib.awq_search(p, p, 16, 128, 60, 128, 20, p, p, p, p, null, null) == 2
    assert lib.awq_search(p, p, 16, 100, 64, 128, 20, p, p, p, p, null, null) == 2
    assert lib.awq_search(p, p, 16, 128, 64, 48, 20, p, p, p, p, null, null) == 1
    assert lib.awq_search(p, p, 16, 128, 64, 128, 0, p, p, p, p, null, null) == 1
    assert lib.awq_search(p, p, 0, 128, 64, 128, 20, p, p, p, p, null, null) == 2


def test_binding_rejects_host_tensors_for_the_device_entry_point():
    X = torch.zeros(4, 128, dtype=torch.bfloat16)
    W = torch.zeros(128, 8, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        awq.search(X, W)


def test_product_package_does_not_import_the_oracle():
    pkg = os.path.dirname(awq.__file__)
    for root, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(root, f), encoding="utf-8").read()
                assert "import oracle" not in text and "from oracle" not in text, f


def test_clip_token_sampling_matches_the_oracle_reading(lib):
    # the token count is host logic; the oracle's strided sample is the reading it follows
    import oracle.awq_clip as C
    for M in (1, 7, 511, 512, 513, 1023, 1024, 1500, 4096, 16384, 16385):
        for T in (1, 64, 512):
            assert awq.clip_token_count(M, T) == len(C.sample_tokens(M, T)), (M, T)
    assert lib.awq_clip_token_count(0, 512) == 0 and lib.awq_clip_token_count(16, 0) == 0


def test_clip_search_validation_happens_on_the_host(lib):
    null = ctypes.c_void_p(0)
    buf = ctypes.create_string_buffer(64)
    p = ctypes.cast(buf, ctypes.c_void_p)
    args = lambda **kw: [kw.get("X", p), p, 0, kw.get("s", p), 16, 128, 64, kw.get("group", 128),
                         kw.get("n_shrink", 10), kw.get("tokens", 512), kw.get("quantizer", 0), p, null, null,
                         p, p, p, null]
    assert lib.awq_clip_search(*args(X=null)) == 1
    assert lib.awq_clip_search(*args(s=null)) == 1
    assert lib.awq_clip_search(*args(n_shrink=0)) == 1
    assert lib.awq_clip_search(*args(n_shrink=21)) == 1
    assert lib.awq_clip_search(*args(tokens=0)) == 1
    assert lib.awq_clip_search(*args(group=48)) == 1
    assert b"group" in lib.awq_last_error_message()
    assert lib.awq_clip_search(*args(quantizer=2)) == 1
    assert b"quantizer" in lib.awq_last_error_message()


def test_plain_c_client_compiles_against_the_header(lib, tmp_path):
    """tests/c/awq_client.c (C99, -Wall -Werror) builds against include/awq_search.h and
    links with libawqsearch.so and the CUDA runtime: the boundary is usable from C."""
    from tests import c_client
    if not c_client.compiler() or not os.path.exists(os.path.join(c_client.CUDA, "include", "cuda_runtime_api.h")):
        pytest.skip("no C compiler or CUDA headers")
    exe = c_client.build(str(tmp_path))
    assert os.path.exists(exe)
