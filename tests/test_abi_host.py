"""Host-side checks of the C ABI that need no GPU.

The library loads, exports every function include/qhl_stage.h declares, and
rejects bad arguments before touching the device.
"""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "qhl_stage.h")


@pytest.fixture(scope="module")
def qhl():
    from quantized_hybrid_layer_b200 import build as b
    b.build()
    import quantized_hybrid_layer_b200 as q
    return q


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"\b(stage_\w+|qhl_\w+)\s*\(", text)
    return sorted(set(names))


def declared_prototypes():
    """{name: parameter count} of every function prototype in the header."""
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    protos = {}
    for m in re.finditer(r"\b((?:stage|qhl)_\w+)\s*\(([^)]*)\)\s*;", text):
        params = " ".join(m.group(2).split())
        protos[m.group(1)] = 0 if params in ("", "void") else params.count(",") + 1
    return protos


def test_binding_signatures_match_the_header(qhl):
    protos = declared_prototypes()
    assert set(protos) == set(declared_functions())
    lib = qhl.lib()
    for name, n in protos.items():
        assert len(getattr(lib, name).argtypes) == n, name


def test_header_declares_the_four_calls_of_the_stage():
    names = declared_functions()
    for n in ("stage_load", "stage_forward", "stage_commit", "stage_rollback"):
        assert n in names


def test_library_exports_every_declared_symbol(qhl):
    names = declared_functions()
    assert set(names) == set(qhl.EXPORTS)
    lib = qhl.lib()
    for n in names:
        assert hasattr(lib, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", qhl.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\s[TW]\s(\w+)$", out, flags=re.M))
    assert set(names) <= exported


def test_packed_bytes_geometry(qhl):
    # Q4_0 item: 128 rows x 256 cols in 18432 bytes; Q8_0: 34816 bytes
    assert qhl.qhl_packed_bytes(2, 128, 256) == 18432
    assert qhl.qhl_packed_bytes(8, 128, 256) == 34816
    assert qhl.qhl_packed_bytes(2, 64, 256) == 18432                        # a short tile pads to 128 rows
    assert qhl.qhl_packed_bytes(2, 1024, 1024) == 8 * 4 * 18432
    assert qhl.qhl_packed_bytes(2, 10336, 5120) == 81 * 20 * 18432       # ragged rows pad to 128
    assert qhl.qhl_packed_bytes(2, 17408, 5120, paired=True) == 272 * 20 * 18432
    # packed bytes equal GGUF bytes whenever rows are a multiple of 128
    assert qhl.qhl_packed_bytes(2, 5120, 17408) == 5120 * 17408 // 32 * 18
    assert qhl.qhl_packed_bytes(8, 5120, 6144) == 5120 * 6144 // 32 * 34
    assert qhl.qhl_packed_bytes(2, 64, 100) == 0                            # cols % 256
    assert qhl.qhl_packed_bytes(3, 64, 256) == 0                            # unknown type


def test_bad_arguments_are_rejected_before_any_device_work(qhl):
    lib = qhl.lib()
    out = ctypes.c_void_p()
    cfg = qhl.StageConfig(5120, 17408, 16, 48, 128, 24, 4, 256, 64, 1e7, 1e-6, 4, 4352, 2)
    assert lib.stage_load(None, None, 0, 0, 4, None, ctypes.byref(out)) == -1
    assert lib.stage_load(ctypes.byref(cfg), None, 0, 2, 1, None, ctypes.byref(out)) == -1     # empty range
    bad = qhl.StageConfig(5120, 17408, 16, 48, 64, 24, 4, 256, 64, 1e7, 1e-6, 4, 4352, 2)    # dn_dim 64
    assert lib.stage_load(ctypes.byref(bad), None, 0, 0, 1, None, ctypes.byref(out)) == -6
    bad = qhl.StageConfig(5120, 17408, 16, 48, 128, 24, 4, 256, 64, 1e7, 1e-6, 4, 4352, 3)   # qtype
    assert lib.stage_load(ctypes.byref(bad), None, 0, 0, 1, None, ctypes.byref(out)) == -6
    bad = qhl.StageConfig(5000, 17408, 16, 48, 128, 24, 4, 256, 64, 1e7, 1e-6, 4, 4352, 2)   # hidden % 256
    assert lib.stage_load(ctypes.byref(bad), None, 0, 0, 1, None, ctypes.byref(out)) == -6
    assert out.value is None
    assert lib.stage_forward(None, None, 1, 0) == -1
    assert lib.stage_forward_f16(None, None, 1, 0) == -1
    assert lib.stage_forward_host(None, None, None, 1, 0) == -1
    assert lib.stage_commit(None, 0) == -1
    assert lib.stage_rollback(None) == -1
    assert lib.stage_committed_len(None) == -1
    assert lib.qhl_qgemv(2, 64, 256, None, None, 1, None, None) == -1
    assert b"bad argument" in lib.qhl_last_error()
    assert lib.qhl_qgemv(2, 64, 256, 16, 16, 17, 16, None) == -1          # n_tok > 16
    assert lib.qhl_deltanet_step(16, 47, 16, 1, 16, 16, 16, None) == -1   # Hv % Hk
    assert lib.qhl_repack(2, 64, 300, 16, None, 16, None) == -1           # cols % 256
    # pointers the kernels read as 16-byte vectors are checked before any device work
    assert lib.qhl_qgemv(2, 64, 256, 16 + 4, 16, 1, 16, None) == -1       # packed_dev misaligned
    assert b"aligned" in lib.qhl_last_error()
    assert lib.qhl_dequant(2, 64, 256, 16 + 8, 0, 0, 1, 16, None) == -1    # packed_dev misaligned
    assert b"aligned" in lib.qhl_last_error()
    assert lib.qhl_deltanet_step(16, 48, 16 + 4, 1, 16, 16, 16, None) == -1  # y_dev misaligned
    assert lib.qhl_deltanet_step(16, 48, 16, 1, 16, 16 + 8, 16, None) == -1  # snaps_dev misaligned
    assert b"aligned" in lib.qhl_last_error()
    lib.stage_free(None)                                                  # no-op


def test_missing_library_fails_loudly(monkeypatch, tmp_path, qhl):
    import importlib
    monkeypatch.setattr(qhl, "LIB_PATH", str(tmp_path / "absent.so"))
    monkeypatch.setattr(qhl, "_lib", None)
    with pytest.raises(ImportError):
        qhl.lib()


def test_binding_rejects_bad_buffers_before_calling_the_library(qhl):
    """The binding checks dtype, device, layout and shape itself, so a wrong
    buffer never reaches the C ABI (whose calls trust their sizes)."""
    import numpy as np
    import torch
    cfg = qhl.StageConfig(5120, 17408, 16, 48, 128, 24, 4, 256, 64, 1e7, 1e-6, 4, 4352, 2)
    st = qhl.Stage(0, cfg, 0, 4)                                # no handle: nothing is loaded
    with pytest.raises(ValueError):
        st.forward(torch.zeros(1, 5120), 0)                     # host tensor
    with pytest.raises(ValueError):
        st.forward_f16(torch.zeros(1, 5120, dtype=torch.float16), 0)
    with pytest.raises(ValueError):
        st.forward_host_buffers(np.zeros((1, 5120), np.float64), np.zeros((1, 5120), np.float32), 0)
    with pytest.raises(ValueError):
        st.forward_host_buffers(np.zeros((2, 5120), np.float32), np.zeros((1, 5120), np.float32), 0)
    with pytest.raises(ValueError):
        st.forward_host_buffers(np.zeros((1, 5120), np.float32), np.zeros((1, 10240), np.float32)[:, ::2], 0)
    K = np.zeros((4, 4352, 256), np.float16)
    with pytest.raises(ValueError):
        st.set_kv(3, K, K[:, :100])                             # V shorter than K
    with pytest.raises(ValueError):
        st.set_kv(3, K[:, :100], K[:, :100])                    # neither the cache's shape
