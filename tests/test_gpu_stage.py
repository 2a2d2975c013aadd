"""GPU parity of the whole layer-stage against the oracle, through the C ABI.

* one hybrid stage of 4 layers (DeltaNet, DeltaNet, DeltaNet, attention) at
  hidden 5120, Q4_0, n_tok 1 from cached position 4096 (seed 2),
* speculative verify passes of 4 and 16 tokens (and 5, 7, 13) from position
  4096 with a seeded accepted prefix, commit and rollback, Q4_0 and Q8_0
  (seed 3): batched output bit-identical to sequential decoding, post-commit
  state bit-identical to the sequential state at that prefix, rollback
  restoring the state exactly,
* split equals whole (layers [0,4) = [0,2) then [2,4)),
* the f16 boundary against the oracle and against the f32 pass,
* protocol and format errors leave the stage unchanged; a bounded wait that is
  made to run out is reported and the stage recovers.
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


# 4 and 16 draft tokens (config 4), Q8_0 at both, and the ragged counts 5, 7
# and 13 (a partial last attention group of 4, and 8-token MMA groups that a
# 16-token pass pads)
@pytest.mark.parametrize("qtype,n", [(Q4_0, 4), (Q4_0, 16), (Q8_0, 4), (Q8_0, 16), (Q4_0, 5), (Q4_0, 7),
                                     (Q4_0, 13)])
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


def test_f16_boundary_matches_the_oracle(q, stage3):
    """The wire form end to end against the oracle: the oracle runs the same
    layers on the f16 input values and its f64 output, rounded once to f16, is
    what the f16 entry must return within the tolerance (rounding to f16 adds
    at most 2^-11 relative, inside 2e-3)."""
    import torch
    st, orc, _ = stage3
    pos = st.committed_len
    h16 = synth.hidden(FULL, 14, 0, 2).astype(np.float16)
    x16 = torch.from_numpy(h16.copy()).cuda()
    st.forward_f16(x16, pos)
    torch.cuda.synchronize()
    st.sync()
    got = x16.cpu().numpy().astype(np.float64)
    st.rollback()
    ref = orc.forward(h16.astype(np.float64), pos)
    orc.rollback()
    # untrained weights grow the hidden state past the binary16 range: an
    # element whose true value is clearly beyond 65504 must come back as an
    # infinity of its sign, every other element within the tolerance of the
    # oracle, relative to the row's largest such element
    over = np.abs(ref) > 65504.0 * (1 + TOL)
    inside = np.abs(ref) < 65504.0 * (1 - TOL)
    assert np.all(np.isinf(got[over]) & (np.sign(got[over]) == np.sign(ref[over])))
    assert inside.any()
    for g, r, m in zip(got, ref, inside):
        if m.any():
            assert np.isfinite(g[m]).all()
            assert np.max(np.abs(g[m] - r[m])) / np.max(np.abs(r[m])) <= TOL
    assert st.committed_len == pos


def test_a_wait_that_runs_out_is_reported_and_the_stage_recovers(q):
    """Failure detection without a GPU fault.  stage_debug_inject makes CTA 0
    of the first in-projection skip one item's quants, with every GEMV wait
    capped at a few thousand iterations: that wait runs out, every kernel of
    the pass still finishes, stage_sync reports STAGE_E_DEVICE once, and after
    rollback, with injection off, the next pass gives the reference bits."""
    import torch
    seed = 13
    st, _, _ = make_pair(FULL, Q4_0, seed, 0, 4, MAX_CTX, CTX, with_oracle=False)
    try:
        h = synth.hidden(FULL, seed, 0, 2)
        ref = run(st, h, CTX)
        st.rollback()
        S0 = _states(st, 0, 4)
        st.debug_inject(fault_item=1, wait_limit=4096)
        x = torch.from_numpy(h.copy()).cuda()
        st.forward(x, CTX)
        with pytest.raises(q.StageError) as e:
            st.sync()
        assert e.value.code == -7                               # STAGE_E_DEVICE
        st.sync()                                               # reported once, then cleared
        st.rollback()
        for l, S in _states(st, 0, 4).items():                  # the committed state is untouched
            assert np.array_equal(S, S0[l])
        with pytest.raises(q.StageError) as e:
            st.debug_inject(fault_item=-2)
        assert e.value.code == -1
        st.debug_inject(-1, 0)
        out = run(st, h, CTX)
        assert np.array_equal(out, ref)
        st.rollback()
    finally:
        st.free()


def _prefill(st, h, pos, chunked):
    import torch
    x = torch.from_numpy(np.ascontiguousarray(h, dtype=np.float32)).cuda()
    st.prefill(x, pos, chunked=chunked)
    torch.cuda.synchronize()
    st.sync()
    return x.cpu().numpy()


@pytest.mark.parametrize("n", [5, 16])
def test_exact_prefill_equals_forward_and_commit(q, n):
    """stage_prefill(EXACT) keeps only each DeltaNet layer's final state but
    runs the same arithmetic: output, committed states and KV rows are those of
    stage_forward + stage_commit(n), bit for bit, and nothing is pending."""
    seed = 15
    st, _, _ = make_pair(FULL, Q4_0, seed, 0, 4, MAX_CTX, CTX, with_oracle=False)
    try:
        S0 = _states(st, 0, 4)
        kv0 = {l: st.get_kv(l) for l in attn_layers(0, 4)}
        h = synth.hidden(FULL, seed, n, n)
        ref = run(st, h, CTX)
        st.commit(n)
        S_ref = _states(st, 0, 4)
        kv_ref = {l: st.get_kv(l) for l in attn_layers(0, 4)}
        for l, S in S0.items():
            st.set_dn_state(l, S)
        for l, (K, V) in kv0.items():
            st.set_kv(l, K, V)
        st.set_kv_len(CTX)
        got = _prefill(st, h, CTX, chunked=False)
        assert np.array_equal(got, ref)
        assert st.committed_len == CTX + n and st.pending == 0
        for l, S in _states(st, 0, 4).items():
            assert np.array_equal(S, S_ref[l]), l
        for l in attn_layers(0, 4):
            K, V = st.get_kv(l)
            assert np.array_equal(K[:, :CTX + n], kv_ref[l][0][:, :CTX + n])
            assert np.array_equal(V[:, :CTX + n], kv_ref[l][1][:, :CTX + n])
        with pytest.raises(q.StageError) as e:
            _prefill(st, h, CTX, chunked=False)          # pos must be the committed length
        assert e.value.code == -2
    finally:
        st.free()


@pytest.mark.parametrize("qtype,n", [(Q4_0, 16), (Q8_0, 16), (Q4_0, 7)])
def test_chunked_prefill_matches_oracle(q, qtype, n):
    """stage_prefill(CHUNKED): the chunked closed form of the DeltaNet
    recurrence for a prompt chunk, against the oracle's token-by-token steps:
    every hidden vector, every DeltaNet head state and the new KV rows within
    the tolerance; decoding then continues from the committed chunk."""
    seed = 16
    st, orc, _ = make_pair(FULL, qtype, seed, 0, 4, MAX_CTX, CTX)
    try:
        h = synth.hidden(FULL, seed, 300 + n, n)
        got = _prefill(st, h, CTX, chunked=True)
        ref = orc.forward(h, CTX)
        orc.commit(n)
        assert max(rel_err_rows(got, ref)) <= TOL
        assert st.committed_len == CTX + n and st.pending == 0
        for l in dn_layers(0, 4):
            assert max(rel_err_heads(st.get_dn_state(l), orc.S[l])) <= TOL, l
        for l in attn_layers(0, 4):
            K, V = st.get_kv(l)
            for X, R in ((K, orc.K[l]), (V, orc.V[l])):
                for p in range(CTX, CTX + n):
                    assert max(rel_err_rows(X[:, p].astype(np.float64), R[:, p].astype(np.float64))) <= TOL
        h2 = synth.hidden(FULL, seed, 400 + n, 1)
        got2 = run(st, h2, CTX + n)
        assert max(rel_err_rows(got2, orc.forward(h2, CTX + n))) <= TOL
        st.rollback()
    finally:
        st.free()


@pytest.mark.parametrize("qtype,ns", [(Q4_0, (1, 2, 3, 4)), (Q8_0, (1, 3))])
def test_persistent_pass_equals_kernel_chain(q, qtype, ns):
    """The one-kernel persistent pass and the chain of per-step kernels run the
    same units with the same split: outputs, committed states and new KV rows
    are bit-identical."""
    import torch
    seed = 7
    st, _, _ = make_pair(FULL, qtype, seed, 0, 4, MAX_CTX, CTX, with_oracle=False)
    try:
        assert not st.pass_persistent(1)                      # the chain of kernels by default
        S0 = _states(st, 0, 4)
        kv0 = {l: st.get_kv(l) for l in attn_layers(0, 4)}
        for n in ns:
            h = synth.hidden(FULL, seed, n, n)
            res = {}
            for mode in (q.PASS_PERSISTENT, q.PASS_KERNELS):
                st.set_pass_mode(mode)
                assert st.pass_persistent(n) == (mode == q.PASS_PERSISTENT), (n, mode, st.last_error)
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
        assert not st.pass_persistent(16)                     # 16-token passes run as kernels
        st.forward(torch.zeros((1, FULL.hidden), device="cuda"), CTX)
        with pytest.raises(q.StageError) as e:
            st.set_pass_mode(q.PASS_KERNELS)                  # refused while a pass is pending
        assert e.value.code == -2
        st.rollback()
        with pytest.raises(q.StageError) as e:
            st.set_pass_mode(5)
        assert e.value.code == -1
        st.set_pass_mode(q.PASS_KERNELS)
    finally:
        st.free()
