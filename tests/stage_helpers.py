"""Shared set-up for the GPU tests: the same seeded inputs for the CUDA stage
and for the oracle (each built from ``synth``; neither imports the other)."""
from __future__ import annotations

import numpy as np

import synth

TOL = 2e-3   # max relative error per output vector / per DeltaNet head state


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
