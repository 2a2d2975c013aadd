"""Parity of the full 64-layer stage (48 gated-DeltaNet + 16 attention layers,
hidden 5120, FFN 17408, Q4_0, seed 4) against the oracle, through the C ABI, in
the launch configuration `bench.py` times (one CUDA graph of kernels per
token, n_tok 1 from cached position 4096), and in its prefill configuration
(a 16-token chunk from position 0 through stage_prefill, chunked DeltaNet form).

The oracle computes every step on the host's cores (about 8 s per decoded
token): every element of each output hidden vector is compared, and the
DeltaNet state and new KV rows of the first and last layers of each kind.
Errors compound over 64 layers and over the recurrent state, so eight
consecutive committed decode steps are checked, not one.
"""
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest

import oracle
import synth
from synth import FULL, Q4_0
from stage_helpers import TOL, make_pair, rel_err_heads, rel_err_rows

pytestmark = pytest.mark.gpu

LAYERS = 64
CTX = 4096
MAX_CTX = CTX + 64
SEED = 4
DECODE_STEPS = 8
CHUNK = 16


def _run(st, h, pos):
    import torch
    x = torch.from_numpy(np.ascontiguousarray(h, dtype=np.float32)).cuda()
    st.forward(x, pos)
    torch.cuda.synchronize()
    st.sync()
    return x.cpu().numpy()


def test_64_layer_decode_steps_and_prefill_chunk_match_oracle():
    import torch
    assert torch.cuda.is_available(), "GPU test needs CUDA"
    tensors = {}
    with ThreadPoolExecutor(16) as ex:
        for t in ex.map(lambda l: synth.layer_tensors(FULL, Q4_0, SEED, l), range(LAYERS)):
            tensors.update(t)
    st, orc, _ = make_pair(FULL, Q4_0, SEED, 0, LAYERS, MAX_CTX, CTX, tensors=tensors)
    try:
        # plain decode: eight committed steps from context 4096
        for step in range(DECODE_STEPS):
            pos = CTX + step
            h = synth.hidden(FULL, SEED, 123 + step, 1)
            got = _run(st, h, pos)
            ref = orc.forward(h, pos)
            errs = rel_err_rows(got, ref)
            assert max(errs) <= TOL, (step, errs)
            st.commit(1)
            orc.commit(1)
        for l in (0, 62):                          # first and last DeltaNet layer
            assert max(rel_err_heads(st.get_dn_state(l), orc.S[l])) <= TOL, l
        for l in (3, 63):                          # first and last attention layer
            K, V = st.get_kv(l)
            for X, R in ((K, orc.K[l]), (V, orc.V[l])):
                for p in range(CTX, CTX + DECODE_STEPS):
                    assert max(rel_err_rows(X[:, p].astype(np.float64), R[:, p].astype(np.float64))) <= TOL
                assert np.array_equal(X[:, :CTX], R[:, :CTX])

        # prefill: a new sequence, one 16-token chunk from position 0 (zero
        # recurrent states, empty cache) through stage_prefill with the chunked
        # DeltaNet form (what bench.py times), against a fresh oracle stage
        # running the token-by-token recurrence
        st.reset()
        orc0 = oracle.OracleStage(FULL, Q4_0, tensors, 0, LAYERS, MAX_CTX)
        h = synth.hidden(FULL, SEED, 500, CHUNK)
        x = torch.from_numpy(np.ascontiguousarray(h, dtype=np.float32)).cuda()
        st.prefill(x, 0, chunked=True)
        torch.cuda.synchronize()
        st.sync()
        got = x.cpu().numpy()
        ref = orc0.forward(h, 0)
        errs = rel_err_rows(got, ref)
        assert max(errs) <= TOL, errs
        orc0.commit(CHUNK)
        assert st.committed_len == CHUNK and st.pending == 0
        for l in (0, 62):
            assert max(rel_err_heads(st.get_dn_state(l), orc0.S[l])) <= TOL, l
    finally:
        st.free()
