"""Shared set-up for the GPU tests: the same seeded inputs for the CUDA stage
and for the oracle (each built from ``synth``; neither imports the other)."""
from __future__ import annotations

import numpy as np

import synth

TOL = 2e-3   # max relative error per output vector / per DeltaNet head state


def gemv_error_bound(qtype, W, x):
    """Per-output bound on |y_gpu - y| for y = x W^T, derived from the arithmetic.

    The CUDA GEMV carries x in block fixed point: per token and 32-column
    block, s = 2^(E - 21) with 2^E <= max |x| < 2^(E + 1), so an element is off
    by at most one unit s (half a unit from rounding; the codes never reach the
    clamp at 2^22).  Block sums over the integer codes are exact; turning a
    block's sums into f32 takes two roundings, adding it to the accumulator one
    more, and the stream-K and epilogue sums a few more, each at most 2^-24 of
    the magnitudes involved.  Bound per output:
        sum_j |W_j| s_j + (blocks + 8) 2^-23 sum_j |W_j| (|x_j| + s_j).
    """
    import oracle
    A = np.abs(oracle.dequant(qtype, W))                         # [rows, cols], exact
    x = np.atleast_2d(np.asarray(x, dtype=np.float32)).astype(np.float64)
    n, cols = x.shape
    m = np.abs(x).reshape(n, cols // 32, 32).max(axis=2)         # block maxima
    E = np.frexp(m)[1] - 1                                        # 2^E <= m < 2^(E+1)
    E = np.where(m > 0, np.maximum(E, -100), -100)
    step = np.repeat(np.ldexp(1.0, E - 21), 32, axis=1)          # [n, cols]
    return step @ A.T + (cols // 32 + 8) * 2.0 ** -23 * ((np.abs(x) + step) @ A.T)


def make_pair(shape, qtype, seed, begin, end, max_ctx, ctx, dn_std=0.01, with_oracle=True, tensors=None,
              stream=None):
    """A GPU stage and (optionally) an oracle stage over layers [begin, end) with
    DeltaNet states ~ N(0, dn_std), KV caches prefilled with ctx rows ~ N(0,1) f16
    and committed length ctx."""
    import quantized_hybrid_layer_b200 as q
    import oracle
    if tensors is None:
        tensors = synth.stage_tensors(shape, qtype, seed, begin, end)
    cfg = q.config_from_shape(shape, qtype, max_ctx)
    st = q.stage_load(cfg, tensors, begin, end, stream=stream)
    orc = oracle.OracleStage(shape, qtype, tensors, begin, end, max_ctx) if with_oracle else None
    for l in range(begin, end):
        if shape.is_attention(l):
            K, V = synth.kv_prefill(shape, seed, l, ctx, max_ctx)
            st.set_kv(l, K, V)
            if orc:
                orc.set_kv(l, K, V)
        else:
            S = synth.dn_state(shape, seed, l, dn_std)
            st.set_dn_state(l, S)
            if orc:
                orc.set_dn_state(l, S)
    st.set_kv_len(ctx)
    if orc:
        orc.set_kv_len(ctx)
    return st, orc, tensors


def rel_err_rows(got, ref):
    """max relative error of each row (one row = one token's hidden vector)."""
    import oracle
    got = np.atleast_2d(np.asarray(got, dtype=np.float64))
    ref = np.atleast_2d(np.asarray(ref, dtype=np.float64))
    return [oracle.max_rel_err(g, r) for g, r in zip(got, ref)]


def rel_err_heads(got, ref):
    """max relative error of each DeltaNet head state matrix."""
    import oracle
    return [oracle.max_rel_err(g, r) for g, r in zip(np.asarray(got), np.asarray(ref))]
