"""Parity of the full 64-layer stage (48 gated-DeltaNet + 16 attention layers,
hidden 5120, FFN 17408, Q4_0, seed 4) against the oracle, through the C ABI, in
the launch configuration `bench.py` times (one CUDA graph of kernels per
token, n_tok 1 from cached position 4096).

The oracle computes the whole step (about 8 s on the host's cores): every
element of the output hidden vector is compared, and the DeltaNet state and new
KV rows of the first and last layers of each kind.
"""
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest

import synth
from synth import FULL, Q4_0
from stage_helpers import TOL, make_pair, rel_err_heads, rel_err_rows

pytestmark = pytest.mark.gpu

LAYERS = 64
CTX = 4096
MAX_CTX = CTX + 64
SEED = 4


def test_64_layer_decode_step_matches_oracle():
    import torch
    assert torch.cuda.is_available(), "GPU test needs CUDA"
    import quantized_hybrid_layer_b200 as q
    tensors = {}
    with ThreadPoolExecutor(16) as ex:
        for t in ex.map(lambda l: synth.layer_tensors(FULL, Q4_0, SEED, l), range(LAYERS)):
            tensors.update(t)
    st, orc, _ = make_pair(FULL, Q4_0, SEED, 0, LAYERS, MAX_CTX, CTX, tensors=tensors)
    try:
        assert not st.pass_persistent(1)          # the default: the chain of kernels bench.py times
        h = synth.hidden(FULL, SEED, 123, 1)
        x = torch.from_numpy(np.ascontiguousarray(h, dtype=np.float32)).cuda()
        st.forward(x, CTX)
        torch.cuda.synchronize()
        st.sync()
        got = x.cpu().numpy()
        ref = orc.forward(h, CTX)
        errs = rel_err_rows(got, ref)
        assert max(errs) <= TOL, errs
        st.commit(1)
        orc.commit(1)
        for l in (0, 62):                          # first and last DeltaNet layer
            assert max(rel_err_heads(st.get_dn_state(l), orc.S[l])) <= TOL, l
        for l in (3, 63):                          # first and last attention layer
            K, V = st.get_kv(l)
            for X, R in ((K, orc.K[l]), (V, orc.V[l])):
                assert max(rel_err_rows(X[:, CTX].astype(np.float64), R[:, CTX].astype(np.float64))) <= TOL
                assert np.array_equal(X[:, :CTX], R[:, :CTX])
    finally:
        st.free()
