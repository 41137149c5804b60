"""The C-ABI library without a GPU: it loads, exports every entry point the header
declares, the header compiles as plain C, and the size query needs no device."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "w8a8.h")


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(w8a8_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    import block_wise_w8a8_b200.build as b
    b.build()
    return ctypes.CDLL(b.LIB)


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert len(names) >= 11, names
    for n in names:
        assert hasattr(lib, n), f"{n} declared in w8a8.h but not exported"


def test_only_declared_symbols_are_exported(lib):
    import block_wise_w8a8_b200.build as b
    out = subprocess.run(["nm", "-D", "--defined-only", b.LIB], capture_output=True, text=True,
                         check=True).stdout
    exported = sorted({line.split()[-1] for line in out.splitlines()
                       if line.split()[-1].startswith("w8a8_")})
    assert exported == _declared()


def test_header_is_plain_c(tmp_path):
    src = tmp_path / "t.c"
    src.write_text('#include "w8a8.h"\nint main(void){ w8a8_weight_t w = {0}; (void)w; '
                   'return (int)w8a8_linear_workspace_bytes(128, 128, 128) == 0; }\n')
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-fsyntax-only",
                    "-I", os.path.join(ROOT, "include"), str(src)], check=True)


def test_workspace_query_and_status_strings(lib):
    lib.w8a8_linear_workspace_bytes.restype = ctypes.c_size_t
    lib.w8a8_linear_workspace_bytes.argtypes = [ctypes.c_int64] * 3
    assert lib.w8a8_linear_workspace_bytes(256, 384, 128) == 256 * 384 + 2 * 3 * 4
    assert lib.w8a8_linear_workspace_bytes(1000, 2048, 8192) == 0      # guard: BF16 path
    assert lib.w8a8_linear_workspace_bytes(1024, 2000, 8192) == 0
    assert lib.w8a8_linear_workspace_bytes(128, 128, 100) == 0
    lib.w8a8_status_string.restype = ctypes.c_char_p
    assert lib.w8a8_status_string(0) == b"ok"
    assert lib.w8a8_status_string(5).startswith(b"workspace")


def test_host_linear_chunk_and_workspace_query(lib):
    """w8a8_linear_host's size queries: 4 MiB of x per chunk in whole 128-row steps, at
    least 128 rows, at most M; the workspace holds two x and two y chunks (each rounded up
    to 256 bytes) and the quantizer's workspace for one chunk."""
    lib.w8a8_linear_host_chunk_rows.restype = ctypes.c_int64
    lib.w8a8_linear_host_chunk_rows.argtypes = [ctypes.c_int64] * 2
    lib.w8a8_linear_host_workspace_bytes.restype = ctypes.c_size_t
    lib.w8a8_linear_host_workspace_bytes.argtypes = [ctypes.c_int64] * 4
    lib.w8a8_linear_workspace_bytes.restype = ctypes.c_size_t
    lib.w8a8_linear_workspace_bytes.argtypes = [ctypes.c_int64] * 3
    assert lib.w8a8_linear_host_chunk_rows(4096, 4096) == 512
    assert lib.w8a8_linear_host_chunk_rows(4096, 2048) == 1024
    assert lib.w8a8_linear_host_chunk_rows(4096, 3000) == 640      # 699 rows, down to 640
    assert lib.w8a8_linear_host_chunk_rows(4096, 65536) == 128     # at least 128
    assert lib.w8a8_linear_host_chunk_rows(300, 4096) == 300       # at most M
    r256 = lambda v: (v + 255) // 256 * 256
    for M, K, N, c in [(4096, 4096, 4096, 0), (1024, 2048, 8192, 384), (1000, 256, 384, 256)]:
        C = min(c or lib.w8a8_linear_host_chunk_rows(M, K), M)
        want = 2 * r256(C * K * 2) + 2 * r256(C * N * 2) + lib.w8a8_linear_workspace_bytes(C, K, N)
        assert lib.w8a8_linear_host_workspace_bytes(M, K, N, c) == want
    assert lib.w8a8_linear_host_workspace_bytes(0, 4096, 4096, 0) == 0


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    import block_wise_w8a8_b200 as w8
    monkeypatch.setattr(w8, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(w8, "_lib", None)
    with pytest.raises(RuntimeError):
        w8.lib()


def test_linear_host_binding_checks_its_input_first():
    """The binding refuses a non-CPU x (a meta tensor stands in for a device tensor here)
    and a non-BF16 x before it touches the weight or the library."""
    import torch

    import block_wise_w8a8_b200 as w8
    with pytest.raises(ValueError):
        w8.linear_host(torch.empty((128, 128), dtype=torch.bfloat16, device="meta"), None)
    with pytest.raises(TypeError):
        w8.linear_host(torch.zeros((128, 128), dtype=torch.float32), None)
    with pytest.raises(TypeError):
        w8.linear_host(torch.zeros((128, 256), dtype=torch.bfloat16)[:, ::2], None)
