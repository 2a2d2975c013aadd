"""GPU parity of the whole layer-stage against the oracle, through the C ABI.

* one hybrid stage of 4 layers (DeltaNet, DeltaNet, DeltaNet, attention) at
  hidden 5120, Q4_0, n_tok 1 from cached position 4096 (seed 2),
* speculative verify passes of 4 and 16 tokens from position 4096 with a seeded
  accepted prefix, commit and rollback, Q4_0 and Q8_0 (seed 3): batched output
  bit-identical to sequential decoding, post-commit state bit-identical to the
  sequential state at that prefix, rollback restoring the state exactly,
* split equals whole (layers [0,4) = [0,2) then [2,4)),
* protocol and format errors leave the stage unchanged.
"""
import numpy as np
import pytest

import oracle
import synth
from synth import FULL, Q4_0, Q8_0
from stage_helpers import TOL, make_pair, rel_err_heads, rel_err_rows

pytestmark = pytest.mark.gpu

CTX = 4096
MAX_CTX = 4096 + 64


@pytest.fixture(scope="module")
def q():
    import torch
    assert torch.cuda.is_available(), "GPU test needs CUDA"
    import quantized_hybrid_layer_b200 as q
    return q


def run(st, h, pos):
    import torch
    x = torch.from_numpy(np.ascontiguousarray(h, dtype=np.float32)).cuda()
    st.forward(x, pos)
    torch.cuda.synchronize()
    st.sync()
    return x.cpu().numpy()


def dn_layers(begin, end):
    return [l for l in range(begin, end) if not FULL.is_attention(l)]


def attn_layers(begin, end):
    return [l for l in range(begin, end) if FULL.is_attention(l)]


@pytest.fixture(scope="module")
def stage3(q):
    st, orc, t = make_pair(FULL, Q4_0, 2, 0, 4, MAX_CTX, CTX)
    yield st, orc, t
    st.free()


def test_four_layer_stage_decode_matches_oracle(stage3):
    st, orc, _ = stage3
    for step in range(2):
        pos = CTX + step
        h = synth.hidden(FULL, 2, step, 1)
        got = run(st, h, pos)
        ref = orc.forward(h, pos)
        errs = rel_err_rows(got, ref)
        assert max(errs) <= TOL, errs
        st.commit(1)
        orc.commit(1)
        for l in dn_layers(0, 4):
            assert max(rel_err_heads(st.get_dn_state(l), orc.S[l])) <= TOL
        for l in attn_layers(0, 4):
            K, V = st.get_kv(l)
            for X, R in ((K, orc.K[l]), (V, orc.V[l])):
                # rows this run wrote: f16 of an f32 (GPU) vs f64 (oracle) value, so
                # they agree within the tolerance, not code for code
                for p in range(CTX, pos + 1):
                    assert max(rel_err_rows(X[:, p].astype(np.float64), R[:, p].astype(np.float64))) <= TOL
                assert np.array_equal(X[:, :CTX], R[:, :CTX])          # prefilled rows untouched
    assert st.committed_len == CTX + 2


def test_debug_dequant_of_stage_tensors_is_bit_exact(stage3):
    st, _, t = stage3
    H, F = FULL.hidden, FULL.ffn
    for name, rows, cols in (("blk.0.dn_in", FULL.dn_in_rows, H), ("blk.0.dn_out", H, FULL.dn_o),
                             ("blk.3.attn_in", FULL.attn_in_rows, H), ("blk.3.attn_out", H, FULL.attn_o),
                             ("blk.1.ffn_gate", F, H), ("blk.1.ffn_up", F, H), ("blk.2.ffn_down", H, F)):
        for row in (0, 1, rows // 2 + 3, rows - 1):
            got = st.debug_dequant(name, row, cols).astype(np.float64)
            ref = oracle.dequant(Q4_0, t[name][row:row + 1])[0]
            assert np.array_equal(got, ref), (name, row)


def _states(st, begin, end):
    return {l: st.get_dn_state(l) for l in dn_layers(begin, end)}


@pytest.mark.parametrize("qtype,n", [(Q4_0, 4), (Q4_0, 16), (Q8_0, 4)])
def test_verify_pass_commit_and_rollback(q, qtype, n):
    seed = 3
    st, orc, _ = make_pair(FULL, qtype, seed, 0, 4, MAX_CTX, CTX)
    try:
        h = synth.hidden(FULL, seed, 100 + n, n)
        S_init = _states(st, 0, 4)
        kv_init = {l: st.get_kv(l) for l in attn_layers(0, 4)}

        # batched verify pass, then rollback: everything back exactly
        out_b = run(st, h, CTX)
        assert st.pending == n
        st.rollback()
        assert st.committed_len == CTX and st.pending == 0
        for l, S in _states(st, 0, 4).items():
            assert np.array_equal(S, S_init[l])

        # the same tokens one at a time (plain decoding)
        seq_states = [S_init]
        out_s = []
        for t in range(n):
            out_s.append(run(st, h[t:t + 1], CTX + t)[0])
            st.commit(1)
            seq_states.append(_states(st, 0, 4))
        out_s = np.stack(out_s)
        assert np.array_equal(out_b, out_s), "batched verify differs from sequential decoding"
        kv_seq = {l: st.get_kv(l) for l in attn_layers(0, 4)}

        # back to the start, batched again, keep a seeded prefix
        for l, S in S_init.items():
            st.set_dn_state(l, S)
        for l, (K, V) in kv_init.items():
            st.set_kv(l, K, V)
        st.set_kv_len(CTX)
        out_b2 = run(st, h, CTX)
        assert np.array_equal(out_b2, out_b)
        j = synth.accepted_prefix(seed, n, n)
        st.commit(j)
        assert st.committed_len == CTX + j
        for l, S in _states(st, 0, 4).items():
            assert np.array_equal(S, seq_states[j][l]), (l, j)
        for l in attn_layers(0, 4):
            K, V = st.get_kv(l)
            assert np.array_equal(K[:, :CTX + j], kv_seq[l][0][:, :CTX + j])
            assert np.array_equal(V[:, :CTX + j], kv_seq[l][1][:, :CTX + j])

        # the oracle on the same verify pass
        ref = orc.forward(h, CTX)
        assert max(rel_err_rows(out_b, ref)) <= TOL
        orc.commit(j)
        for l in dn_layers(0, 4):
            assert max(rel_err_heads(st.get_dn_state(l), orc.S[l])) <= TOL

        # decoding continues from the committed prefix
        h2 = synth.hidden(FULL, seed, 200 + n, 1)
        got = run(st, h2, CTX + j)
        ref2 = orc.forward(h2, CTX + j)
        assert max(rel_err_rows(got, ref2)) <= TOL
    finally:
        st.free()


def test_split_stage_equals_whole(q):
    seed = 5
    t = synth.stage_tensors(FULL, Q4_0, seed, 0, 4)
    whole, _, _ = make_pair(FULL, Q4_0, seed, 0, 4, MAX_CTX, CTX, with_oracle=False, tensors=t)
    a, _, _ = make_pair(FULL, Q4_0, seed, 0, 2, MAX_CTX, CTX, with_oracle=False, tensors=t)
    b, _, _ = make_pair(FULL, Q4_0, seed, 2, 4, MAX_CTX, CTX, with_oracle=False, tensors=t)
    try:
        for n in (1, 3):
            h = synth.hidden(FULL, seed, n, n)
            out_w = run(whole, h, whole.committed_len)
            out_s = run(b, run(a, h, a.committed_len), b.committed_len)
            assert np.array_equal(out_w, out_s)
            for st in (whole, a, b):
                st.commit(n)
    finally:
        for st in (whole, a, b):
            st.free()


def test_protocol_errors_leave_state_unchanged(q, stage3):
    import torch
    st, _, _ = stage3
    pos = st.committed_len
    S = st.get_dn_state(0)
    x = torch.zeros((1, FULL.hidden), dtype=torch.float32, device="cuda")
    with pytest.raises(q.StageError) as e:
        st.forward(torch.zeros((17, FULL.hidden), dtype=torch.float32, device="cuda"), pos)
    assert e.value.code == -1
    with pytest.raises(q.StageError) as e:
        st.forward(x, pos + 1)
    assert e.value.code == -2
    with pytest.raises(q.StageError) as e:
        st.commit(0)
    assert e.value.code == -2
    st.forward(x, pos)
    with pytest.raises(q.StageError) as e:
        st.forward(x, pos)
    assert e.value.code == -2
    with pytest.raises(q.StageError) as e:
        st.commit(2)
    assert e.value.code == -1
    with pytest.raises(q.StageError) as e:
        st.get_dn_state(0)                      # refused while pending
    assert e.value.code == -2
    st.rollback()
    assert st.committed_len == pos
    assert np.array_equal(st.get_dn_state(0), S)
    with pytest.raises(q.StageError) as e:
        st.get_dn_state(3)                      # an attention layer
    assert e.value.code == -1
    with pytest.raises(q.StageError) as e:
        st.set_kv_len(MAX_CTX)
    assert e.value.code == -1
    with pytest.raises(q.StageError) as e:     # context overflow
        st.set_kv_len(MAX_CTX - 2)
        st.forward(torch.zeros((4, FULL.hidden), dtype=torch.float32, device="cuda"), MAX_CTX - 2)
    assert e.value.code == -1
    st.set_kv_len(pos)
    assert st.committed_len == pos


def test_load_rejects_missing_or_misshaped_tensors(q):
    t = synth.stage_tensors(FULL, Q4_0, 6, 3, 4)          # one attention layer
    cfg = q.config_from_shape(FULL, Q4_0, MAX_CTX)
    bad = dict(t)
    del bad["blk.3.attn_k_norm"]
    with pytest.raises(q.StageError) as e:
        q.stage_load(cfg, bad, 3, 4)
    assert e.value.code == -5 and "attn_k_norm" in str(e.value)
    bad = dict(t)
    bad["blk.3.ffn_down"] = bad["blk.3.ffn_down"][:-1]
    with pytest.raises(q.StageError) as e:
        q.stage_load(cfg, bad, 3, 4)
    assert e.value.code == -5
    st = q.stage_load(cfg, t, 3, 4)                         # an attention-only stage loads
    st.free()


@pytest.mark.parametrize("qtype,ns", [(Q4_0, (1, 2, 3, 4)), (Q8_0, (1, 3))])
def test_persistent_pass_equals_kernel_chain(q, qtype, ns):
    """The one-kernel persistent pass and the chain of per-step kernels run the
    same units with the same split: outputs and committed states are
    bit-identical."""
    import torch
    seed = 7
    st, _, _ = make_pair(FULL, qtype, seed, 0, 4, MAX_CTX, CTX, with_oracle=False)
    try:
        assert not st.pass_persistent(1)                      # the chain of kernels by default
        assert not st.pass_persistent(16)
        S0 = _states(st, 0, 4)
        kv0 = {l: st.get_kv(l) for l in attn_layers(0, 4)}
        for n in ns:
            st.set_pass_mode(q.PASS_PERSISTENT)
            assert st.pass_persistent(n), n
            h = synth.hidden(FULL, seed, n, n)
            res = {}
            for mode in (q.PASS_PERSISTENT, q.PASS_KERNELS):
                st.set_pass_mode(mode)
                out = run(st, h, CTX)
                st.commit(n)
                res[mode] = (out, _states(st, 0, 4), {l: st.get_kv(l) for l in attn_layers(0, 4)})
                for l, S in S0.items():                       # back to the starting state
                    st.set_dn_state(l, S)
                for l, (K, V) in kv0.items():
                    st.set_kv(l, K, V)
                st.set_kv_len(CTX)
            out_p, S_p, kv_p = res[q.PASS_PERSISTENT]
            out_k, S_k, kv_k = res[q.PASS_KERNELS]
            assert np.array_equal(out_p, out_k), n
            for l in S_p:
                assert np.array_equal(S_p[l], S_k[l]), (n, l)
            for l in kv_p:
                assert np.array_equal(kv_p[l][0], kv_k[l][0]) and np.array_equal(kv_p[l][1], kv_k[l][1]), (n, l)
        st.set_pass_mode(q.PASS_PERSISTENT)
        st.forward(torch.zeros((1, FULL.hidden), device="cuda"), CTX)
        with pytest.raises(q.StageError) as e:
            st.set_pass_mode(q.PASS_KERNELS)          # refused while a pass is pending
        assert e.value.code == -2
        st.rollback()
        with pytest.raises(q.StageError) as e:
            st.set_pass_mode(5)
        assert e.value.code == -1
    finally:
        st.free()


def test_persistent_pass_trace_shows_the_grid_barriers(q):
    """With tracing on, every CTA records each phase; no CTA starts a phase
    before every CTA has finished the previous one (the grid barrier)."""
    st, _, _ = make_pair(FULL, Q4_0, 8, 0, 4, MAX_CTX, CTX, with_oracle=False)
    try:
        with pytest.raises(q.StageError):
            st.get_trace()                                   # off by default
        st.set_pass_mode(q.PASS_PERSISTENT)
        st.set_trace(True)
        h = synth.hidden(FULL, 8, 0, 1)
        run(st, h, CTX)
        st.rollback()
        tr = st.get_trace().astype(np.int64)
        grid, n_phases, _ = tr.shape
        assert n_phases == 1 + 3 * 5 + 6                      # input, 3 DeltaNet layers, 1 attention layer
        assert (tr > 0).all()
        assert (tr[:, :, 1] >= tr[:, :, 0]).all()
        for ph in range(1, n_phases):
            assert tr[:, ph, 0].min() >= tr[:, ph - 1, 1].max(), ph
        st.set_trace(False)
        run(st, h, CTX)                                       # still runs without the trace buffer
        st.rollback()
    finally:
        st.free()


def test_zero_weight_stage_is_the_identity(q):
    """All quants at the Q4_0 zero point (nibble 8): every projection is 0, so
    each layer adds exact zeros and the stage returns its input bit for bit
    (a DeltaNet and an attention layer, a 3-token pass)."""
    seed = 9
    t = synth.stage_tensors(FULL, Q4_0, seed, 2, 4)
    for name, v in t.items():
        if v.dtype == np.uint8:                        # GGUF blocks: 2-byte scale + 16 bytes of nibbles
            b = v.reshape(v.shape[0], -1, 18).copy()
            b[:, :, 2:] = 0x88
            t[name] = b.reshape(v.shape)
    st, _, _ = make_pair(FULL, Q4_0, seed, 2, 4, MAX_CTX, CTX, with_oracle=False, tensors=t)
    try:
        h = synth.hidden(FULL, seed, 0, 3)
        out = run(st, h, CTX)
        assert np.array_equal(out, h.astype(np.float32))
        st.commit(3)
    finally:
        st.free()


@pytest.mark.parametrize("n", [1, 4])
def test_long_context_attention_layer_matches_oracle(q, n):
    """One attention layer at context 65536 (1025 chunks of 64 rows to split
    and combine), against the oracle."""
    seed = 10
    ctx = 65536
    st, orc, _ = make_pair(FULL, Q4_0, seed, 3, 4, ctx + 64, ctx)
    try:
        h = synth.hidden(FULL, seed, n, n)
        got = run(st, h, ctx)
        ref = orc.forward(h, ctx)
        assert max(rel_err_rows(got, ref)) <= TOL
        st.rollback()
    finally:
        st.free()


@pytest.mark.parametrize("n", [1, 5])
def test_f16_boundary_equals_the_f32_pass_rounded(q, stage3, n):
    """forward_f16 takes and returns the hidden state in binary16, the peers'
    wire format (10 KB per token at hidden 5120): its output is, bit for bit,
    the f32 pass on the same (f16-valued) input rounded to nearest even, and
    it leaves the same pending pass (rolled back here)."""
    import torch
    st, _, _ = stage3
    pos = st.committed_len
    h16 = synth.hidden(FULL, 11, 0, n).astype(np.float16)
    x16 = torch.from_numpy(h16.copy()).cuda()
    st.forward_f16(x16, pos)
    torch.cuda.synchronize()
    st.sync()
    got16 = x16.cpu().numpy()
    assert st.pending == n
    st.rollback()
    out32 = run(st, h16.astype(np.float32), pos)
    st.rollback()
    with np.errstate(over="ignore"):      # outputs beyond 65504 round to +-inf, on both sides
        want16 = out32.astype(np.float16)
    assert np.array_equal(got16.view(np.uint16), want16.view(np.uint16))
    assert st.committed_len == pos


def test_forward_from_host_buffers_equals_the_device_pass(q, stage3):
    """stage_forward_host (copy in, pass, copy out in one C call) gives the
    bits of stage_forward on a device buffer: pageable numpy buffers, and a
    page-locked torch buffer used in place."""
    import torch
    st, _, _ = stage3
    pos = st.committed_len
    h = synth.hidden(FULL, 12, 0, 3)
    out = np.empty_like(h)
    st.forward_host_buffers(h, out, pos)
    assert st.pending == 3
    st.rollback()
    ref = run(st, h, pos)
    st.rollback()
    assert np.array_equal(out, ref)
    hp = torch.from_numpy(h.copy()).pin_memory()
    st.forward_host_buffers(hp, hp, pos)
    st.rollback()
    assert np.array_equal(hp.numpy(), ref)
    assert st.committed_len == pos
