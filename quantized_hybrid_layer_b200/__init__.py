"""Python binding of the quantized hybrid layer-stage library (libqhl_stage.so).

Argument marshalling only: every step of the stage runs in the CUDA library
(``csrc/``), reached through the C ABI declared in ``include/qhl_stage.h``.
PyTorch supplies device memory and the CUDA stream.  There is no CPU fallback:
if the shared library is missing, importing the binding raises.

The names follow the C ABI: ``stage_load``, ``stage_forward``, ``stage_commit``,
``stage_rollback`` and friends, plus the kernel-level ``qhl_*`` calls.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libqhl_stage.so")

STAGE_Q4_0 = 2
STAGE_Q8_0 = 8
MAX_TOK = 16
PREFILL_EXACT, PREFILL_CHUNKED = 0, 1
PASS_KERNELS, PASS_PERSISTENT = 0, 1

STATUS = {
    0: "STAGE_OK", -1: "STAGE_E_ARG", -2: "STAGE_E_STATE", -3: "STAGE_E_OOM", -4: "STAGE_E_CUDA",
    -5: "STAGE_E_FORMAT", -6: "STAGE_E_UNSUPPORTED", -7: "STAGE_E_DEVICE",
}

#: every symbol include/qhl_stage.h declares
EXPORTS = (
    "stage_load", "stage_forward", "stage_forward_host", "stage_forward_f16", "stage_prefill", "stage_commit", "stage_rollback", "stage_reset", "stage_sync",
    "stage_committed_len", "stage_pending", "stage_get_dn_state", "stage_set_dn_state", "stage_get_kv",
    "stage_set_kv", "stage_set_kv_len", "stage_debug_dequant", "stage_set_pass_mode", "stage_pass_persistent",
    "stage_debug_inject",
    "stage_weight_bytes", "stage_last_error",
    "stage_free", "qhl_packed_bytes", "qhl_repack", "qhl_dequant", "qhl_qgemv", "qhl_deltanet_step",
    "qhl_qgemv_noalloc", "qhl_sync", "qhl_debug_inject", "qhl_last_error",
)


class StageError(RuntimeError):
    def __init__(self, code: int, message: str):
        super().__init__(f"{STATUS.get(code, code)}: {message}")
        self.code = code


class StageConfig(ctypes.Structure):
    _fields_ = [
        ("hidden", ctypes.c_int), ("ffn", ctypes.c_int),
        ("dn_k_heads", ctypes.c_int), ("dn_v_heads", ctypes.c_int), ("dn_dim", ctypes.c_int),
        ("att_q_heads", ctypes.c_int), ("att_kv_heads", ctypes.c_int), ("att_dim", ctypes.c_int),
        ("rope_dims", ctypes.c_int), ("rope_theta", ctypes.c_double), ("eps", ctypes.c_float),
        ("attn_every", ctypes.c_int), ("max_ctx", ctypes.c_int), ("qtype", ctypes.c_int),
    ]


class StageTensor(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char_p), ("data", ctypes.c_void_p), ("bytes", ctypes.c_size_t)]


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded CUDA library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python quantized_hybrid_layer_b200/build.py` (no CPU fallback exists)")
        L = ctypes.CDLL(LIB_PATH)
        vp, i, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        sig = {
            "stage_load": (i, [ctypes.POINTER(StageConfig), ctypes.POINTER(StageTensor), i, i, i, vp,
                               ctypes.POINTER(vp)]),
            "stage_forward": (i, [vp, vp, i, i]),
            "stage_forward_f16": (i, [vp, vp, i, i]),
            "stage_forward_host": (i, [vp, vp, vp, i, i]),
            "stage_prefill": (i, [vp, vp, i, i, i]),
            "stage_commit": (i, [vp, i]),
            "stage_rollback": (i, [vp]),
            "stage_reset": (i, [vp]),
            "stage_sync": (i, [vp]),
            "stage_committed_len": (i, [vp]),
            "stage_pending": (i, [vp]),
            "stage_get_dn_state": (i, [vp, i, vp, sz]),
            "stage_set_dn_state": (i, [vp, i, vp, sz]),
            "stage_get_kv": (i, [vp, i, vp, vp, sz]),
            "stage_set_kv": (i, [vp, i, vp, vp, sz]),
            "stage_set_kv_len": (i, [vp, i]),
            "stage_debug_dequant": (i, [vp, ctypes.c_char_p, i, vp, sz]),
            "stage_set_pass_mode": (i, [vp, i]),
            "stage_pass_persistent": (i, [vp, i]),
            "stage_debug_inject": (i, [vp, i, ctypes.c_uint]),
            "stage_weight_bytes": (sz, [vp]),
            "stage_last_error": (ctypes.c_char_p, [vp]),
            "stage_free": (None, [vp]),
            "qhl_packed_bytes": (sz, [i, i, i, i]),
            "qhl_repack": (i, [i, i, i, vp, vp, vp, vp]),
            "qhl_dequant": (i, [i, i, i, vp, i, i, i, vp, vp]),
            "qhl_qgemv": (i, [i, i, i, vp, vp, i, vp, vp]),
            "qhl_deltanet_step": (i, [i, i, vp, i, vp, vp, vp, vp]),
            "qhl_qgemv_noalloc": (i, [i, i, i, vp, vp, i, vp, vp]),
            "qhl_sync": (i, [vp]),
            "qhl_debug_inject": (i, [i, ctypes.c_uint]),
            "qhl_last_error": (ctypes.c_char_p, []),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _stream(stream) -> int | None:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return getattr(stream, "cuda_stream", stream)


def _ptr(t) -> int:
    return int(t.data_ptr())


def _check_hidden(hidden, dtype: str, width: int):
    """A forward's hidden buffer: contiguous CUDA tensor of `dtype`, [n_tok, width]."""
    if not (hidden.is_cuda and str(hidden.dtype) == f"torch.{dtype}" and hidden.is_contiguous()
            and hidden.dim() == 2 and hidden.shape[1] == width):
        raise ValueError(f"hidden must be a contiguous CUDA {dtype} tensor [n_tok, {width}], got "
                         f"{hidden.dtype} {tuple(hidden.shape)} on {hidden.device}")


def _host_ptr(x) -> int:
    return int(x.data_ptr()) if hasattr(x, "data_ptr") else int(x.ctypes.data)


def _check_host_hidden(x, width: int) -> int:
    """A host f32 [n_tok, width] C-contiguous buffer (numpy array or CPU torch tensor); returns n_tok."""
    if hasattr(x, "data_ptr"):
        ok = (not x.is_cuda and str(x.dtype) == "torch.float32" and x.is_contiguous() and x.dim() == 2
              and x.shape[1] == width)
    else:
        ok = (isinstance(x, np.ndarray) and x.dtype == np.float32 and x.flags.c_contiguous and x.ndim == 2
              and x.shape[1] == width)
    if not ok:
        raise ValueError(f"expected a host C-contiguous float32 [n_tok, {width}] buffer, got "
                         f"{type(x).__name__} {getattr(x, 'dtype', None)} {tuple(getattr(x, 'shape', ()))}")
    return int(x.shape[0])


def _check_qhl(rc: int):
    if rc != 0:
        raise StageError(rc, lib().qhl_last_error().decode())


def config_from_shape(shape, qtype: int, max_ctx: int) -> StageConfig:
    """Fill the C config from any object with the StageShape field names."""
    return StageConfig(shape.hidden, shape.ffn, shape.dn_k_heads, shape.dn_v_heads, shape.dn_dim,
                       shape.att_q_heads, shape.att_kv_heads, shape.att_dim, shape.rope_dims,
                       float(shape.rope_theta), float(shape.eps), shape.attn_every, int(max_ctx), int(qtype))


class Stage:
    """A loaded layer-stage (owns its device memory until ``free``)."""

    def __init__(self, handle: int, cfg: StageConfig, begin: int, end: int):
        self._h = ctypes.c_void_p(handle)
        self.cfg, self.begin, self.end = cfg, begin, end

    def _check(self, rc: int):
        if rc != 0:
            raise StageError(rc, lib().stage_last_error(self._h).decode())

    # the pass -------------------------------------------------------------
    def forward(self, hidden, pos: int):
        """hidden: contiguous CUDA float32 tensor [n_tok, hidden], updated in place."""
        _check_hidden(hidden, "float32", self.cfg.hidden)
        n = hidden.shape[0]
        self._check(lib().stage_forward(self._h, _ptr(hidden), n, pos))
        return hidden

    def forward_f16(self, hidden, pos: int):
        """hidden: contiguous CUDA float16 tensor [n_tok, hidden] (the wire format),
        updated in place with the pass's f32 result rounded to nearest even."""
        _check_hidden(hidden, "float16", self.cfg.hidden)
        n = hidden.shape[0]
        self._check(lib().stage_forward_f16(self._h, _ptr(hidden), n, pos))
        return hidden

    def forward_host_buffers(self, hidden_in, hidden_out, pos: int, sync: bool = True):
        """One C call from host memory: copy in, pass, copy out (stage_forward_host).
        hidden_in / hidden_out: host f32 [n_tok, hidden], C-contiguous numpy arrays or
        CPU torch tensors (page-locked for asynchronous copies); they may be the same
        buffer.  With sync=False the caller synchronises before reading hidden_out."""
        n = _check_host_hidden(hidden_in, self.cfg.hidden)
        if _check_host_hidden(hidden_out, self.cfg.hidden) != n:
            raise ValueError("hidden_in and hidden_out must hold the same number of tokens")
        self._check(lib().stage_forward_host(self._h, _host_ptr(hidden_in), _host_ptr(hidden_out), n, pos))
        if sync:
            self.sync()
        return hidden_out

    def prefill(self, hidden, pos: int, chunked: bool = False):
        """Prompt chunk, committed in the same call (stage_prefill): the exact
        token-by-token recurrence, or its chunked closed form."""
        _check_hidden(hidden, "float32", self.cfg.hidden)
        mode = PREFILL_CHUNKED if chunked else PREFILL_EXACT
        self._check(lib().stage_prefill(self._h, _ptr(hidden), hidden.shape[0], pos, mode))

    def commit(self, n_accepted: int):
        self._check(lib().stage_commit(self._h, n_accepted))

    def rollback(self):
        self._check(lib().stage_rollback(self._h))

    def reset(self):
        self._check(lib().stage_reset(self._h))

    def sync(self):
        self._check(lib().stage_sync(self._h))

    @property
    def committed_len(self) -> int:
        return lib().stage_committed_len(self._h)

    @property
    def pending(self) -> int:
        return lib().stage_pending(self._h)

    def set_pass_mode(self, mode: int):
        """PASS_KERNELS (one kernel per step, the default) or PASS_PERSISTENT
        (one cooperative kernel per forward pass where eligible)."""
        self._check(lib().stage_set_pass_mode(self._h, mode))

    def pass_persistent(self, n_tok: int) -> bool:
        """Whether an n_tok forward runs as the persistent kernel."""
        return lib().stage_pass_persistent(self._h, n_tok) == 1

    @property
    def last_error(self) -> str:
        """The stage's last error message (stage_last_error)."""
        return lib().stage_last_error(self._h).decode()

    def debug_inject(self, fault_item: int = -1, wait_limit: int = 0):
        """Failure injection for tests of the bounded waits (stage_debug_inject)."""
        self._check(lib().stage_debug_inject(self._h, fault_item, wait_limit))

    @property
    def weight_bytes(self) -> int:
        return int(lib().stage_weight_bytes(self._h))

    # state access ---------------------------------------------------------
    def get_dn_state(self, layer: int) -> np.ndarray:
        c = self.cfg
        out = np.empty((c.dn_v_heads, c.dn_dim, c.dn_dim), dtype=np.float32)
        self._check(lib().stage_get_dn_state(self._h, layer, out.ctypes.data, out.nbytes))
        return out

    def set_dn_state(self, layer: int, S: np.ndarray):
        S = np.ascontiguousarray(S, dtype=np.float32)
        self._check(lib().stage_set_dn_state(self._h, layer, S.ctypes.data, S.nbytes))

    def get_kv(self, layer: int):
        c = self.cfg
        K = np.empty((c.att_kv_heads, c.max_ctx, c.att_dim), dtype=np.float16)
        V = np.empty_like(K)
        self._check(lib().stage_get_kv(self._h, layer, K.ctypes.data, V.ctypes.data, K.nbytes))
        return K, V

    def set_kv(self, layer: int, K: np.ndarray, V: np.ndarray):
        c = self.cfg
        K = np.ascontiguousarray(K, dtype=np.float16)
        V = np.ascontiguousarray(V, dtype=np.float16)
        want = (c.att_kv_heads, c.max_ctx, c.att_dim)
        if K.shape != want or V.shape != want:
            raise ValueError(f"K and V must both be f16 {want}, got {K.shape} and {V.shape}")
        self._check(lib().stage_set_kv(self._h, layer, K.ctypes.data, V.ctypes.data, K.nbytes))

    def set_kv_len(self, n: int):
        self._check(lib().stage_set_kv_len(self._h, n))

    def debug_dequant(self, tensor: str, row: int, cols: int) -> np.ndarray:
        out = np.empty(cols, dtype=np.float32)
        self._check(lib().stage_debug_dequant(self._h, tensor.encode(), row, out.ctypes.data, out.size))
        return out

    def free(self):
        if self._h:
            lib().stage_free(self._h)
            self._h = ctypes.c_void_p(None)

    def __del__(self):
        try:
            self.free()
        except Exception:
            pass


def stage_load(cfg: StageConfig, tensors: dict, layer_begin: int, layer_end: int, stream=None) -> Stage:
    """Upload and repack host tensors {name: numpy array} for layers [layer_begin, layer_end)."""
    arrs = [(k.encode(), np.ascontiguousarray(v)) for k, v in tensors.items()]
    table = (StageTensor * len(arrs))(*[StageTensor(k, v.ctypes.data, v.nbytes) for k, v in arrs])
    out = ctypes.c_void_p()
    rc = lib().stage_load(ctypes.byref(cfg), table, len(arrs), layer_begin, layer_end, _stream(stream),
                          ctypes.byref(out))
    if rc != 0:
        raise StageError(rc, lib().qhl_last_error().decode())
    return Stage(out.value, cfg, layer_begin, layer_end)


def stage_forward(st: Stage, hidden, pos: int):
    return st.forward(hidden, pos)


def stage_forward_f16(st: Stage, hidden, pos: int):
    return st.forward_f16(hidden, pos)


def stage_commit(st: Stage, n_accepted: int):
    st.commit(n_accepted)


def stage_rollback(st: Stage):
    st.rollback()


def stage_free(st: Stage):
    st.free()


# ---------------------------------------------------------------------------
# kernel-level calls (torch CUDA tensors in, results written in place)

def qhl_packed_bytes(qtype: int, rows: int, cols: int, paired: bool = False) -> int:
    return int(lib().qhl_packed_bytes(qtype, rows, cols, 1 if paired else 0))


def qhl_repack(qtype: int, rows: int, cols: int, gguf, packed, gguf_b=None, stream=None):
    _check_qhl(lib().qhl_repack(qtype, rows, cols, _ptr(gguf), _ptr(gguf_b) if gguf_b is not None else None,
                                _ptr(packed), _stream(stream)))


def qhl_dequant(qtype: int, rows: int, cols: int, packed, row0: int, nrows: int, out, paired: bool = False,
                stream=None):
    _check_qhl(lib().qhl_dequant(qtype, rows, cols, _ptr(packed), 1 if paired else 0, row0, nrows, _ptr(out),
                                 _stream(stream)))


def qhl_qgemv(qtype: int, rows: int, cols: int, packed, x, y, stream=None):
    n = x.shape[0]
    _check_qhl(lib().qhl_qgemv(qtype, rows, cols, _ptr(packed), _ptr(x), n, _ptr(y), _stream(stream)))


def qhl_qgemv_noalloc(qtype: int, rows: int, cols: int, packed, x, y, stream=None):
    """qhl_qgemv for callers that cannot allocate device memory: its scratch is a
    fixed static device array, so the call allocates nothing (limits in qhl_stage.h)."""
    n = x.shape[0]
    _check_qhl(lib().qhl_qgemv_noalloc(qtype, rows, cols, _ptr(packed), _ptr(x), n, _ptr(y), _stream(stream)))


def qhl_deltanet_step(Hk: int, Hv: int, y, s_in, snaps, o, stream=None):
    n = y.shape[0]
    _check_qhl(lib().qhl_deltanet_step(Hk, Hv, _ptr(y), n, _ptr(s_in), _ptr(snaps), _ptr(o), _stream(stream)))


def qhl_sync(stream=None):
    """Wait for the stream; raise StageError(STAGE_E_DEVICE) if a qhl_qgemv /
    qhl_qgemv_noalloc kernel's bounded wait ran out since the last qhl_sync."""
    _check_qhl(lib().qhl_sync(_stream(stream)))


def qhl_debug_inject(fault_item: int = -1, wait_limit: int = 0):
    """Failure injection for tests of the qhl_qgemv error path (qhl_debug_inject)."""
    _check_qhl(lib().qhl_debug_inject(fault_item, wait_limit))
