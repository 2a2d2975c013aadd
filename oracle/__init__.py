"""Plain CPU oracle for the quantized hybrid layer-stage.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this package.  It
shares no code with the CUDA library (``quantized_hybrid_layer_b200``) and
neither imports the other; both take their inputs from ``synth``.

Every floating-point value is held in double precision, except the KV cache,
which the method stores as f16.  The quantised GEMV (dequantise + dot product)
runs in ``oracle_q.c`` (f64, plain loops); everything else is numpy f64 written
as the definitions read.  Where the pages leave a step open, the reading taken
is stated at the function.

Sources (page title, part of the page):

* "Unstable Legion: the peer-to-peer ChatGPT", "Splitting the workload" and
  "The runtime": a stage runs a contiguous range of layers, activation in,
  activation out, and holds the attention cache of those layers only.
* "ChatTorrent" README, "What it can run": the hybrid interleaves Gated
  DeltaNet (linear attention) layers and full-attention layers; the latter
  rotate part of each head (partial RoPE), normalise q and k per head and gate
  their output; blocks use RMSNorm and SwiGLU.
* "Peer-to-peer LLM inference in browser tabs, Qwen 3.8 27B" (SwarmLLM
  README): 27B hybrid Gated-DeltaNet + attention, GGUF Q4_0 with f16 block
  scales, 5,120-wide hidden state, drafts verified in one batched pass whose
  rejected tail is undone exactly in the recurrent state, so the speculative
  path gives what plain decoding gives.
* The update is the gated delta rule of the Gated DeltaNet paper, which the
  SwarmLLM README names among its prior work: ``S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T)
  + beta_t v_t k_t^T``, read out as ``o_t = S_t q_t``.
* Shapes: hidden 5,120 (SwarmLLM README diagram) and 64 layers (its peer
  split 0-21 / 22-42 / 43-63); FFN 17408, 16 key / 48 value heads of 128, 24 query / 4 KV heads
  of 256, RoPE on the first 64 dims with theta 1e7, eps 1e-6 and a 3:1
  DeltaNet:attention pattern are the defaults of ``synth.StageShape``.

Readings taken where the pages are silent:

* RMSNorm is ``x / sqrt(mean(x^2) + eps) * gamma`` with gamma applied as given.
* q, k of a DeltaNet key head are L2-normalised as ``x / sqrt(sum(x^2) + 1e-6)``.
* ``beta = sigmoid(b)``, ``alpha = exp(-softplus(a))``; value head h reads key
  head ``h // (Hv / Hk)``; ``o_t = S_t q_t`` after the update, with no scale,
  conv, norm or gate on o.
* Attention: per-head RMSNorm on q and k (shared gamma of length dh), then
  rotate-half RoPE on dims [0, rope_dims) pairing (i, i + rope_dims/2) with
  angle ``pos * theta^(-2i/rope_dims)``; scores ``q.k / sqrt(dh)``; query head j
  reads KV head ``j // (Hq / Hkv)``; output ``o * sigmoid(gate)`` element-wise.
* The in-projection row orders are those documented in ``synth``.
"""
from __future__ import annotations

import ctypes
import math

import numpy as np

from synth import Q4_0, Q8_0, QK, StageShape

from . import build as _build

_LIB = None


def lib() -> ctypes.CDLL:
    """Load (building on first use) the oracle's C part."""
    global _LIB
    if _LIB is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        L.orc_f16_to_f64.restype = ctypes.c_double
        L.orc_f16_to_f64.argtypes = [ctypes.c_uint16]
        L.orc_f16_array.restype = None
        L.orc_f16_array.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p]
        L.orc_dequant.restype = ctypes.c_int
        L.orc_dequant.argtypes = [ctypes.c_int, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p]
        L.orc_qgemv.restype = ctypes.c_int
        L.orc_qgemv.argtypes = [ctypes.c_int, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                                ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p]
        L.orc_threads.restype = ctypes.c_int
        L.orc_threads.argtypes = []
        _LIB = L
    return _LIB


def threads() -> int:
    """OpenMP threads the C part uses."""
    return int(lib().orc_threads())


# ----------------------------------------------------------------------------
# quantised weights
# ----------------------------------------------------------------------------

def _blocks_shape(qtype: int, blocks: np.ndarray):
    bb = {Q4_0: 18, Q8_0: 34}[qtype]
    assert blocks.dtype == np.uint8 and blocks.shape[-1] == bb and blocks.ndim == 3
    rows, nb = blocks.shape[0], blocks.shape[1]
    return rows, nb * QK


def f16_to_f64(bits: np.ndarray) -> np.ndarray:
    """IEEE binary16 bit patterns -> f64 values (decoder in oracle_q.c)."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    out = np.empty(b.shape, dtype=np.float64)
    lib().orc_f16_array(b.ctypes.data, b.size, out.ctypes.data)
    return out


def dequant(qtype: int, blocks: np.ndarray) -> np.ndarray:
    """GGUF Q4_0 / Q8_0 blocks [rows, cols/32, bytes] -> f64 [rows, cols] (exact)."""
    rows, cols = _blocks_shape(qtype, blocks)
    blocks = np.ascontiguousarray(blocks)
    out = np.empty((rows, cols), dtype=np.float64)
    rc = lib().orc_dequant(qtype, blocks.ctypes.data, rows, cols, out.ctypes.data)
    assert rc == 0
    return out


def qgemv(qtype: int, blocks: np.ndarray, x: np.ndarray) -> np.ndarray:
    """y = x W^T in f64; W in GGUF blocks [rows, cols/32, bytes], x [n, cols] -> y [n, rows]."""
    rows, cols = _blocks_shape(qtype, blocks)
    x = np.ascontiguousarray(np.atleast_2d(x), dtype=np.float64)
    assert x.shape[1] == cols
    n = x.shape[0]
    y = np.empty((n, rows), dtype=np.float64)
    rc = lib().orc_qgemv(qtype, np.ascontiguousarray(blocks).ctypes.data, rows, cols,
                         x.ctypes.data, n, y.ctypes.data)
    assert rc == 0
    return y


# ----------------------------------------------------------------------------
# element-wise maps and norms
# ----------------------------------------------------------------------------

def rmsnorm(x: np.ndarray, gamma: np.ndarray, eps: float) -> np.ndarray:
    """RMSNorm over the last axis: x / sqrt(mean(x^2) + eps) * gamma (ChatTorrent README, "What it can run")."""
    x = np.asarray(x, dtype=np.float64)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * np.asarray(gamma, dtype=np.float64)


def l2norm(x: np.ndarray, eps: float = 1e-6) -> np.ndarray:
    """x / sqrt(sum(x^2) + eps) over the last axis."""
    x = np.asarray(x, dtype=np.float64)
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps)


def sigmoid(x):
    return 1.0 / (1.0 + np.exp(-np.asarray(x, dtype=np.float64)))


def softplus(x):
    return np.logaddexp(0.0, np.asarray(x, dtype=np.float64))


def silu(x):
    x = np.asarray(x, dtype=np.float64)
    return x * sigmoid(x)


def rope(x: np.ndarray, pos: int, rope_dims: int, theta: float) -> np.ndarray:
    """Rotate-half RoPE on the first rope_dims dims of the last axis at position pos."""
    x = np.asarray(x, dtype=np.float64)
    half = rope_dims // 2
    i = np.arange(half, dtype=np.float64)
    ang = float(pos) * theta ** (-2.0 * i / rope_dims)
    c, s = np.cos(ang), np.sin(ang)
    out = x.copy()
    x1 = x[..., :half]
    x2 = x[..., half:rope_dims]
    out[..., :half] = x1 * c - x2 * s
    out[..., half:rope_dims] = x2 * c + x1 * s
    return out


# ----------------------------------------------------------------------------
# mixers, one token at a time
# ----------------------------------------------------------------------------

def deltanet_token(S: np.ndarray, q_raw, k_raw, v, b, a, shape: StageShape):
    """One gated-delta-rule step for every value head (Gated DeltaNet; ChatTorrent README, "What it can run").

    S is f64 [Hv, dv, dk].  Per value head h with key head g = h // (Hv/Hk):
    ``S <- alpha * S (I - beta k k^T) + beta v k^T`` and ``o = S q`` on the
    updated state, with q, k L2-normalised, beta = sigmoid(b),
    alpha = exp(-softplus(a)).  The identity matrix is materialised, as the
    rule is written.  Returns (S_new, o [Hv, dv]).
    """
    Hk, Hv, d = shape.dn_k_heads, shape.dn_v_heads, shape.dn_dim
    q = l2norm(np.reshape(q_raw, (Hk, d)))
    k = l2norm(np.reshape(k_raw, (Hk, d)))
    v = np.reshape(np.asarray(v, dtype=np.float64), (Hv, d))
    beta = sigmoid(np.reshape(b, (Hv,)))
    alpha = np.exp(-softplus(np.reshape(a, (Hv,))))
    rep = Hv // Hk
    eye = np.eye(d)
    S_new = np.empty_like(S, dtype=np.float64)
    o = np.empty((Hv, d), dtype=np.float64)
    for h in range(Hv):
        g = h // rep
        S_new[h] = alpha[h] * (S[h] @ (eye - beta[h] * np.outer(k[g], k[g]))) + beta[h] * np.outer(v[h], k[g])
        o[h] = S_new[h] @ q[g]
    return S_new, o


def deltanet_steps(S0: np.ndarray, q, k, v, b, a, shape: StageShape):
    """Run n tokens in sequence from S0; returns (o [n, Hv, dv], [S_0, S_1, ..., S_n])."""
    S = np.asarray(S0, dtype=np.float64)
    snaps = [S]
    outs = []
    for t in range(len(q)):
        S, o = deltanet_token(S, q[t], k[t], v[t], b[t], a[t], shape)
        snaps.append(S)
        outs.append(o)
    return np.stack(outs), snaps


def split_dn_in(y: np.ndarray, shape: StageShape):
    """Rows q | k | v | b | a of the DeltaNet in-projection output of one token."""
    Hk, Hv, d = shape.dn_k_heads, shape.dn_v_heads, shape.dn_dim
    o1 = Hk * d
    o2 = 2 * Hk * d
    o3 = o2 + Hv * d
    return y[:o1], y[o1:o2], y[o2:o3], y[o3:o3 + Hv], y[o3 + Hv:o3 + 2 * Hv]


def attention_token(y: np.ndarray, pos: int, K: np.ndarray, V: np.ndarray,
                    gq: np.ndarray, gk: np.ndarray, shape: StageShape) -> np.ndarray:
    """Full GQA attention for the token at absolute position ``pos`` (ChatTorrent README, "What it can run").

    y is the token's in-projection output (rows q | gate | k | v).  The token's
    k, v are QK-normed (k) and RoPE'd (k), rounded to f16 and written to cache
    row ``pos`` of K, V (f16 [Hkv, max_ctx, dh]); it then attends to rows
    0..pos.  Returns ``o * sigmoid(gate)`` flattened to [Hq*dh].
    """
    Hq, Hkv, dh = shape.att_q_heads, shape.att_kv_heads, shape.att_dim
    y = np.asarray(y, dtype=np.float64)
    q = y[:Hq * dh].reshape(Hq, dh)
    gate = y[Hq * dh:2 * Hq * dh].reshape(Hq, dh)
    off = 2 * Hq * dh
    k = y[off:off + Hkv * dh].reshape(Hkv, dh)
    v = y[off + Hkv * dh:off + 2 * Hkv * dh].reshape(Hkv, dh)
    q = rope(rmsnorm(q, gq, shape.eps), pos, shape.rope_dims, shape.rope_theta)
    k = rope(rmsnorm(k, gk, shape.eps), pos, shape.rope_dims, shape.rope_theta)
    K[:, pos, :] = k.astype(np.float16)
    V[:, pos, :] = v.astype(np.float16)
    rep = Hq // Hkv
    o = np.empty((Hq, dh), dtype=np.float64)
    for j in range(Hq):
        g = j // rep
        Kg = K[g, :pos + 1, :].astype(np.float64)
        Vg = V[g, :pos + 1, :].astype(np.float64)
        s = (Kg @ q[j]) / math.sqrt(dh)
        w = np.exp(s - np.max(s))
        w = w / np.sum(w)
        o[j] = w @ Vg
    return (o * sigmoid(gate)).reshape(-1)


# ----------------------------------------------------------------------------
# the stage
# ----------------------------------------------------------------------------

class OracleStage:
    """A contiguous layer range with its own recurrent states and KV caches.

    ``forward(h, pos)`` runs n tokens at positions pos .. pos+n-1 through every
    layer (layer by layer, tokens in order inside a layer) and leaves the pass
    pending; ``commit(j)`` keeps the first j tokens' effect on the DeltaNet
    states and the KV length, ``rollback()`` keeps none (SwarmLLM README:
    a batched verify pass whose rejected drafts leave no trace in the state).
    """

    def __init__(self, shape: StageShape, qtype: int, tensors: dict, begin: int, end: int, max_ctx: int):
        self.shape, self.qtype, self.t = shape, qtype, tensors
        self.begin, self.end, self.max_ctx = begin, end, max_ctx
        self.S = {}
        self.K, self.V = {}, {}
        for l in range(begin, end):
            if shape.is_attention(l):
                self.K[l] = np.zeros((shape.att_kv_heads, max_ctx, shape.att_dim), dtype=np.float16)
                self.V[l] = np.zeros_like(self.K[l])
            else:
                self.S[l] = np.zeros((shape.dn_v_heads, shape.dn_dim, shape.dn_dim), dtype=np.float64)
        self.kv_len = 0
        self.pending = None

    # state access -----------------------------------------------------------
    def set_dn_state(self, layer: int, S: np.ndarray):
        self.S[layer] = np.array(S, dtype=np.float64)

    def set_kv(self, layer: int, K: np.ndarray, V: np.ndarray):
        self.K[layer] = np.array(K, dtype=np.float16)
        self.V[layer] = np.array(V, dtype=np.float16)

    def set_kv_len(self, n: int):
        self.kv_len = int(n)

    # the pass ---------------------------------------------------------------
    def _w(self, layer, tag):
        return self.t[f"blk.{layer}.{tag}"]

    def forward(self, h: np.ndarray, pos: int) -> np.ndarray:
        if self.pending is not None:
            raise RuntimeError("a pass is pending; commit or roll back first")
        if pos != self.kv_len:
            raise ValueError("pos must equal the committed length")
        sh, qt = self.shape, self.qtype
        h = np.array(np.atleast_2d(h), dtype=np.float64)
        n = h.shape[0]
        if pos + n > self.max_ctx:
            raise ValueError("context overflow")
        snaps = {}
        for l in range(self.begin, self.end):
            x = rmsnorm(h, self._w(l, "norm1"), sh.eps)
            if sh.is_attention(l):
                y = qgemv(qt, self._w(l, "attn_in"), x)
                o = np.stack([attention_token(y[t], pos + t, self.K[l], self.V[l],
                                              self._w(l, "attn_q_norm"), self._w(l, "attn_k_norm"), sh)
                              for t in range(n)])
                h = h + qgemv(qt, self._w(l, "attn_out"), o)
            else:
                y = qgemv(qt, self._w(l, "dn_in"), x)
                S = self.S[l]
                seq = [S]
                outs = []
                for t in range(n):
                    q, k, v, b, a = split_dn_in(y[t], sh)
                    S, ot = deltanet_token(S, q, k, v, b, a, sh)
                    seq.append(S)
                    outs.append(ot.reshape(-1))
                snaps[l] = seq
                h = h + qgemv(qt, self._w(l, "dn_out"), np.stack(outs))
            x2 = rmsnorm(h, self._w(l, "norm2"), sh.eps)
            g = qgemv(qt, self._w(l, "ffn_gate"), x2)
            u = qgemv(qt, self._w(l, "ffn_up"), x2)
            h = h + qgemv(qt, self._w(l, "ffn_down"), silu(g) * u)
        self.pending = (pos, n, snaps)
        return h

    def commit(self, n_accepted: int):
        if self.pending is None:
            raise RuntimeError("no pending pass")
        pos, n, snaps = self.pending
        if not 0 <= n_accepted <= n:
            raise ValueError("n_accepted out of range")
        for l, seq in snaps.items():
            self.S[l] = seq[n_accepted]
        self.kv_len = pos + n_accepted
        self.pending = None

    def rollback(self):
        self.commit(0)

    def forward_sequential(self, h: np.ndarray, pos: int) -> np.ndarray:
        """The same tokens as plain decoding: one forward + commit(1) per token."""
        h = np.atleast_2d(h)
        out = []
        for t in range(h.shape[0]):
            out.append(self.forward(h[t:t + 1], pos + t)[0])
            self.commit(1)
        return np.stack(out)


def max_rel_err(got: np.ndarray, ref: np.ndarray) -> float:
    """max_i |got_i - ref_i| / max_i |ref_i| over one output vector (or matrix)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = float(np.max(np.abs(ref)))
    num = float(np.max(np.abs(got - ref)))
    if den == 0.0:
        return num
    return num / den
