"""Pins for the oracle: checks against what the pages and mathematics fix.

None of these re-call the oracle's own formula to check itself: they use
hand-derived fixtures, exact rational arithmetic, library routines for special
cases, closed forms and invariants, chosen so that a dropped term, a wrong sign
or index, or a transposed operand fails at least one of them.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
import synth
from synth import Q4_0, Q8_0, TINY

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


# ---------------------------------------------------------------- fixtures --

def _read_blocks(path):
    cases = []
    blk = None
    for line in open(path):
        line = line.strip()
        if line.startswith("block"):
            blk = bytes(int(v, 16) for v in line.split()[1:])
        elif line.startswith("values"):
            cases.append((blk, [Fraction(v) for v in line.split()[1:]]))
    return cases


@pytest.mark.parametrize("name,qtype", [("q4_0_block.txt", Q4_0), ("q8_0_block.txt", Q8_0)])
def test_dequant_golden_blocks(golden_dir, name, qtype):
    cases = _read_blocks(os.path.join(golden_dir, name))
    assert cases
    for blk, vals in cases:
        arr = np.frombuffer(blk, dtype=np.uint8).reshape(1, 1, -1)
        got = oracle.dequant(qtype, arr)[0]
        assert len(vals) == 32
        for g, v in zip(got, vals):
            assert Fraction(g) == v


def test_f16_decoder_matches_library_for_every_bit_pattern():
    bits = np.arange(65536, dtype=np.uint16)
    got = oracle.f16_to_f64(bits)
    ref = bits.view(np.float16).astype(np.float64)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    # the sign of zero is kept too
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan]))


def _dequant_by_bits(qtype, blocks):
    """A second, independent decoder: unpack bits with numpy, scale with numpy float16."""
    rows, nb, bb = blocks.shape
    d = blocks[:, :, 0:2].copy().view(np.float16)[..., 0].astype(np.float64)
    if qtype == Q4_0:
        bits = np.unpackbits(blocks[:, :, 2:], axis=-1, bitorder="little").reshape(rows, nb, 16, 8)
        weights = np.array([1, 2, 4, 8])
        lo = (bits[..., 0:4] * weights).sum(-1)
        hi = (bits[..., 4:8] * weights).sum(-1)
        q = np.concatenate([lo, hi], axis=-1) - 8
    else:
        q = blocks[:, :, 2:].view(np.int8).astype(np.int64)
    return (q * d[..., None]).reshape(rows, nb * 32)


@pytest.mark.parametrize("qtype", [Q4_0, Q8_0])
def test_dequant_matches_second_decoder(qtype):
    W = synth.qmatrix(qtype, synth.rng_for(11, 0, 1), 37, 96)
    assert np.array_equal(oracle.dequant(qtype, W), _dequant_by_bits(qtype, W))


@pytest.mark.parametrize("qtype", [Q4_0, Q8_0])
def test_qgemv_one_hot_selects_a_column(qtype):
    rows, cols = 48, 128
    W = synth.qmatrix(qtype, synth.rng_for(12, 0, 1), rows, cols)
    D = _dequant_by_bits(qtype, W)
    for c in (0, 17, 31, 32, 127):
        x = np.zeros((1, cols))
        x[0, c] = 1.0
        assert np.array_equal(oracle.qgemv(qtype, W, x)[0], D[:, c])


@pytest.mark.parametrize("qtype", [Q4_0, Q8_0])
def test_qgemv_against_exact_rationals(qtype):
    rows, cols, n = 5, 64, 3
    W = synth.qmatrix(qtype, synth.rng_for(13, 0, 1), rows, cols)
    x = synth.normal_f32(synth.rng_for(13, 0, 2), (n, cols)).astype(np.float64)
    y = oracle.qgemv(qtype, W, x)
    D = _dequant_by_bits(qtype, W)
    for t in range(n):
        for r in range(rows):
            exact = sum(Fraction(D[r, c]) * Fraction(x[t, c]) for c in range(cols))
            scale = sum(abs(Fraction(D[r, c]) * Fraction(x[t, c])) for c in range(cols))
            assert abs(Fraction(y[t, r]) - exact) <= scale * Fraction(cols, 2 ** 52)


# ------------------------------------------------------ element-wise maps --

def test_rmsnorm_constant_vector_closed_form():
    c, n, eps = 3.0, 64, 1e-6
    gamma = np.linspace(0.5, 1.5, n)
    got = oracle.rmsnorm(np.full((1, n), c), gamma, eps)[0]
    assert np.allclose(got, gamma * c / math.sqrt(c * c + eps), rtol=1e-15, atol=0)


def test_rmsnorm_scale_invariant_and_unit_rms():
    x = np.random.default_rng(1).standard_normal((2, 100)) * 1e3
    g = np.ones(100)
    a = oracle.rmsnorm(x, g, 1e-6)
    b = oracle.rmsnorm(7.0 * x, g, 1e-6)
    assert np.allclose(a, b, rtol=1e-12)
    assert np.allclose(np.sqrt(np.mean(a * a, axis=-1)), 1.0, rtol=1e-9)


def test_l2norm_unit_length_and_zero_safe():
    x = np.random.default_rng(2).standard_normal((3, 128))
    assert np.allclose(np.linalg.norm(oracle.l2norm(x), axis=-1), 1.0, rtol=1e-8)
    assert np.array_equal(oracle.l2norm(np.zeros((1, 8))), np.zeros((1, 8)))


def test_silu_sigmoid_softplus_closed_forms():
    assert oracle.silu(0.0) == 0.0
    assert oracle.sigmoid(0.0) == 0.5
    assert math.isclose(float(oracle.silu(1.0)), 1.0 / (1.0 + math.exp(-1.0)), rel_tol=1e-15)
    assert math.isclose(float(oracle.softplus(0.0)), math.log(2.0), rel_tol=1e-15)
    # alpha = exp(-softplus(a)) = 1 / (1 + e^a)
    for a in (-3.0, 0.0, 2.5):
        assert math.isclose(float(np.exp(-oracle.softplus(a))), 1.0 / (1.0 + math.exp(a)), rel_tol=1e-14)


# ------------------------------------------------------------------ RoPE --

def test_rope_identity_at_zero_and_norm_preserving():
    x = np.random.default_rng(3).standard_normal((4, 32))
    assert np.array_equal(oracle.rope(x, 0, 8, 1e4), x)
    y = oracle.rope(x, 1234, 8, 1e4)
    assert np.allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-13)
    assert np.array_equal(y[:, 8:], x[:, 8:])          # only the first rope_dims rotate


def test_rope_first_pair_closed_form():
    # frequency 0 has inv_freq 1: e_0 rotates to (cos p, sin p) in dims (0, half)
    x = np.zeros(16)
    x[0] = 1.0
    y = oracle.rope(x, 5, 8, 1e7)
    assert math.isclose(y[0], math.cos(5.0), abs_tol=1e-15)
    assert math.isclose(y[4], math.sin(5.0), abs_tol=1e-15)
    # last frequency: inv_freq = theta^(-2*3/8) on pair (3, 7)
    x = np.zeros(16)
    x[7] = 1.0
    y = oracle.rope(x, 100, 8, 1e4)
    ang = 100.0 * 1e4 ** (-6.0 / 8.0)
    assert math.isclose(y[3], -math.sin(ang), abs_tol=1e-14)
    assert math.isclose(y[7], math.cos(ang), abs_tol=1e-14)


def test_rope_scores_depend_only_on_relative_position():
    rng = np.random.default_rng(4)
    q, k = rng.standard_normal(32), rng.standard_normal(32)
    s1 = oracle.rope(q, 10, 16, 1e4) @ oracle.rope(k, 3, 16, 1e4)
    s2 = oracle.rope(q, 1010, 16, 1e4) @ oracle.rope(k, 1003, 16, 1e4)
    assert math.isclose(s1, s2, rel_tol=1e-10)


# -------------------------------------------------------------- DeltaNet --

def _dn_inputs(seed, sh=TINY):
    rng = np.random.default_rng(seed)
    S = rng.standard_normal((sh.dn_v_heads, sh.dn_dim, sh.dn_dim)) * 0.3
    q = rng.standard_normal((sh.dn_k_heads, sh.dn_dim))
    k = rng.standard_normal((sh.dn_k_heads, sh.dn_dim))
    v = rng.standard_normal((sh.dn_v_heads, sh.dn_dim))
    b = rng.standard_normal(sh.dn_v_heads)
    a = rng.standard_normal(sh.dn_v_heads)
    return S, q, k, v, b, a


def _unit(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def test_deltanet_rank_one_form():
    """S(I - b k k^T) = S - b (S k) k^T: the rank-one update equals the explicit one."""
    sh = TINY
    S, q, k, v, b, a = _dn_inputs(5)
    S1, o = oracle.deltanet_token(S, q, k, v, b, a, sh)
    kn = oracle.l2norm(k)
    beta = 1.0 / (1.0 + np.exp(-b))
    alpha = 1.0 / (1.0 + np.exp(a))
    rep = sh.dn_v_heads // sh.dn_k_heads
    for h in range(sh.dn_v_heads):
        kk = kn[h // rep]
        Sk = S[h] @ kk
        ref = alpha[h] * S[h] - alpha[h] * beta[h] * np.outer(Sk, kk) + beta[h] * np.outer(v[h], kk)
        assert np.allclose(S1[h], ref, rtol=1e-12, atol=1e-13)


def test_deltanet_invariants_along_and_across_k():
    """With |k| = 1: S_t k = alpha (1 - beta) S_{t-1} k + beta v; S_t u = alpha S_{t-1} u for u _|_ k."""
    sh = TINY
    S, q, k, v, b, a = _dn_inputs(6)
    S1, _ = oracle.deltanet_token(S, q, k, v, b, a, sh)
    kn = oracle.l2norm(k)
    beta = 1.0 / (1.0 + np.exp(-b))
    alpha = 1.0 / (1.0 + np.exp(a))
    rep = sh.dn_v_heads // sh.dn_k_heads
    rng = np.random.default_rng(7)
    for h in range(sh.dn_v_heads):
        kk = kn[h // rep]
        k2 = float(kk @ kk)                  # 1 up to the 1e-6 inside the norm
        lhs = S1[h] @ kk
        rhs = alpha[h] * (1.0 - beta[h] * k2) * (S[h] @ kk) + beta[h] * k2 * v[h]
        assert np.allclose(lhs, rhs, rtol=1e-11, atol=1e-12)
        u = rng.standard_normal(sh.dn_dim)
        u -= (u @ kk) / k2 * kk
        assert np.allclose(S1[h] @ u, alpha[h] * (S[h] @ u), rtol=1e-11, atol=1e-12)


def test_deltanet_beta_one_writes_v_along_k():
    sh = TINY
    S, q, k, v, b, a = _dn_inputs(8)
    b = np.full_like(b, 60.0)                 # sigmoid(60) == 1.0 in f64
    S1, _ = oracle.deltanet_token(S, q, k, v, b, a, sh)
    kn = _unit(k)
    rep = sh.dn_v_heads // sh.dn_k_heads
    for h in range(sh.dn_v_heads):
        assert np.allclose(S1[h] @ kn[h // rep], v[h], rtol=1e-6, atol=1e-6)


def test_deltanet_zero_state_single_step_readout_after_update():
    """From S0 = 0 one step gives o = beta v (k.q): the read-out uses the updated state."""
    sh = TINY
    S, q, k, v, b, a = _dn_inputs(9)
    S0 = np.zeros_like(S)
    _, o = oracle.deltanet_token(S0, q, k, v, b, a, sh)
    qn, kn = oracle.l2norm(q), oracle.l2norm(k)
    beta = 1.0 / (1.0 + np.exp(-b))
    rep = sh.dn_v_heads // sh.dn_k_heads
    for h in range(sh.dn_v_heads):
        g = h // rep
        assert np.allclose(o[h], beta[h] * v[h] * (kn[g] @ qn[g]), rtol=1e-12, atol=1e-14)


def test_deltanet_value_head_reads_key_head_h_div_rep():
    sh = TINY
    rep = sh.dn_v_heads // sh.dn_k_heads
    S0 = np.zeros((sh.dn_v_heads, sh.dn_dim, sh.dn_dim))
    q = np.zeros((sh.dn_k_heads, sh.dn_dim))
    k = np.zeros((sh.dn_k_heads, sh.dn_dim))
    for g in range(sh.dn_k_heads):
        q[g, g] = 1.0
        k[g, g] = 1.0                          # key head g points along axis g
    v = np.ones((sh.dn_v_heads, sh.dn_dim))
    b = np.full(sh.dn_v_heads, 60.0)
    a = np.zeros(sh.dn_v_heads)
    S1, o = oracle.deltanet_token(S0, q, k, v, b, a, sh)
    for h in range(sh.dn_v_heads):
        nz = np.nonzero(np.abs(S1[h]).sum(axis=0) > 0.5)[0]
        assert list(nz) == [h // rep]


def test_deltanet_alpha_decays_the_state():
    sh = TINY
    S, q, k, v, b, a = _dn_inputs(10)
    v = np.zeros_like(v)
    b = np.full_like(b, -60.0)                 # beta -> 0 (1e-26): only alpha acts
    S1, _ = oracle.deltanet_token(S, q, k, v, b, a, sh)
    alpha = 1.0 / (1.0 + np.exp(a))
    assert np.allclose(S1, alpha[:, None, None] * S, rtol=1e-12, atol=1e-20)


def test_deltanet_steps_snapshots_are_prefixes():
    sh = TINY
    S0, q, k, v, b, a = synth.deltanet_step_problem(sh, 1, 5)
    outs, snaps = oracle.deltanet_steps(S0, q, k, v, b, a, sh)
    for j in range(6):
        _, s2 = oracle.deltanet_steps(S0, q[:j], k[:j], v[:j], b[:j], a[:j], sh) if j else (None, [np.asarray(S0, np.float64)])
        assert np.array_equal(snaps[j], s2[-1])


# ------------------------------------------------------------- attention --

def _attn_y(rng, sh, q=None, gate=None, k=None, v=None):
    Hq, Hkv, dh = sh.att_q_heads, sh.att_kv_heads, sh.att_dim
    parts = [rng.standard_normal(Hq * dh) if q is None else q,
             rng.standard_normal(Hq * dh) if gate is None else gate,
             rng.standard_normal(Hkv * dh) if k is None else k,
             rng.standard_normal(Hkv * dh) if v is None else v]
    return np.concatenate(parts)


def test_attention_single_position_returns_gated_v():
    sh = TINY
    rng = np.random.default_rng(11)
    Hq, Hkv, dh = sh.att_q_heads, sh.att_kv_heads, sh.att_dim
    K = np.zeros((Hkv, 8, dh), np.float16)
    V = np.zeros_like(K)
    y = _attn_y(rng, sh, gate=np.zeros(Hq * dh))
    o = oracle.attention_token(y, 0, K, V, np.ones(dh), np.ones(dh), sh).reshape(Hq, dh)
    vv = y[2 * Hq * dh + Hkv * dh:].reshape(Hkv, dh).astype(np.float16).astype(np.float64)
    rep = Hq // Hkv
    for j in range(Hq):
        assert np.array_equal(o[j], 0.5 * vv[j // rep])     # sigmoid(0) = 1/2


def test_attention_equal_keys_average_values():
    sh = TINY
    rng = np.random.default_rng(12)
    Hq, Hkv, dh = sh.att_q_heads, sh.att_kv_heads, sh.att_dim
    ctx = 6
    K = np.zeros((Hkv, 16, dh), np.float16)
    V = np.zeros_like(K)
    y = _attn_y(rng, sh, gate=np.full(Hq * dh, 80.0))       # sigmoid(80) == 1
    # make the new key equal to the cached ones: store what the token will write
    kk = y[2 * Hq * dh:2 * Hq * dh + Hkv * dh].reshape(Hkv, dh)
    kk = oracle.rope(oracle.rmsnorm(kk, np.ones(dh), sh.eps), ctx, sh.rope_dims, sh.rope_theta).astype(np.float16)
    K[:, :ctx] = kk[:, None, :]
    V[:, :ctx] = rng.standard_normal((Hkv, ctx, dh)).astype(np.float16)
    o = oracle.attention_token(y, ctx, K, V, np.ones(dh), np.ones(dh), sh).reshape(Hq, dh)
    rep = Hq // Hkv
    for j in range(Hq):
        assert np.allclose(o[j], V[j // rep, :ctx + 1].astype(np.float64).mean(axis=0), rtol=1e-12, atol=1e-12)


def test_attention_two_keys_weight_ratio_is_exp_of_scaled_score_gap():
    """Two keys whose scores differ by D get weights in ratio exp(D / sqrt(dh))."""
    sh = TINY
    Hq, Hkv, dh = sh.att_q_heads, sh.att_kv_heads, sh.att_dim
    rng = np.random.default_rng(13)
    K = np.zeros((Hkv, 4, dh), np.float16)
    V = np.zeros_like(K)
    # cached key 0 is e_10 * 2, value e_0; the new token's key at pos 1 is 0-ish (value e_1)
    K[:, 0, 10] = 2.0
    V[:, 0, 0] = 1.0
    qv = np.zeros((Hq, dh))
    qv[:, 10] = 1.0                           # after QK-norm q becomes e_10 * sqrt(dh)
    kv_new = np.zeros((Hkv, dh))
    kv_new[:, 20] = 1e-3                      # normalised to e_20 * sqrt(dh): orthogonal to q
    vnew = np.zeros((Hkv, dh))
    vnew[:, 1] = 1.0
    y = _attn_y(rng, sh, q=qv.reshape(-1), gate=np.full(Hq * dh, 80.0), k=kv_new.reshape(-1), v=vnew.reshape(-1))
    # rope at position 1 rotates dims < rope_dims only; dims 10, 20 are beyond TINY's rope_dims
    assert sh.rope_dims <= 10
    o = oracle.attention_token(y, 1, K, V, np.ones(dh), np.ones(dh), sh).reshape(Hq, dh)
    q10 = 1.0 / math.sqrt(1.0 / dh + sh.eps)  # QK-norm of e_10 (eps inside the root)
    score_gap = 2.0 * q10                     # q.k0 - q.k1, with q.k1 = 0
    ratio = math.exp(score_gap / math.sqrt(dh))
    for j in range(Hq):
        assert math.isclose(o[j, 0] / o[j, 1], ratio, rel_tol=1e-12)
        assert math.isclose(o[j, 0] + o[j, 1], 1.0, rel_tol=1e-12)


def test_attention_writes_f16_cache_row_and_reads_kv_head_j_div_rep():
    sh = TINY
    Hq, Hkv, dh = sh.att_q_heads, sh.att_kv_heads, sh.att_dim
    rng = np.random.default_rng(14)
    K = rng.standard_normal((Hkv, 8, dh)).astype(np.float16)
    V = np.zeros_like(K)
    # every value row of KV head g (cached rows and the new one) is the constant g + 1,
    # so any softmax over head g's keys returns exactly g + 1
    vv = np.repeat(np.arange(1, Hkv + 1, dtype=np.float64)[:, None], dh, axis=1)
    V[:, :3] = vv[:, None, :].astype(np.float16)
    y = _attn_y(rng, sh, gate=np.full(Hq * dh, 80.0), v=vv.reshape(-1))
    o = oracle.attention_token(y, 3, K, V, np.ones(dh), np.ones(dh), sh).reshape(Hq, dh)
    assert np.array_equal(V[:, 3].astype(np.float64), vv)
    kk = y[2 * Hq * dh:2 * Hq * dh + Hkv * dh].reshape(Hkv, dh)
    kk = oracle.rope(oracle.rmsnorm(kk, np.ones(dh), sh.eps), 3, sh.rope_dims, sh.rope_theta)
    assert np.array_equal(K[:, 3], kk.astype(np.float16))
    rep = Hq // Hkv
    for j in range(Hq):
        assert np.allclose(o[j], j // rep + 1.0, rtol=1e-14)


# ----------------------------------------------------------------- stage --

def _tiny_stage(qtype=Q4_0, begin=0, end=4, seed=2, max_ctx=64, ctx=20):
    sh = TINY
    t = synth.stage_tensors(sh, qtype, seed, begin, end)
    st = oracle.OracleStage(sh, qtype, t, begin, end, max_ctx)
    for l in range(begin, end):
        if sh.is_attention(l):
            K, V = synth.kv_prefill(sh, seed, l, ctx, max_ctx)
            st.set_kv(l, K, V)
        else:
            st.set_dn_state(l, synth.dn_state(sh, seed, l, 0.3))
    st.set_kv_len(ctx)
    return st, t


def test_stage_with_zero_weights_is_identity():
    sh = TINY
    st, t = _tiny_stage()
    for name, arr in t.items():
        if arr.dtype == np.uint8:
            z = arr.copy()
            z[:, :, 2:] = 0x88                  # every nibble 8 -> weight 0
            t[name] = z
    h = synth.hidden(sh, 2, 0, 3).astype(np.float64)
    out = st.forward(h, 20)
    assert np.array_equal(out, h)


@pytest.mark.parametrize("qtype", [Q4_0, Q8_0])
def test_stage_batched_equals_sequential_and_commit_prefix(qtype):
    sh = TINY
    n = 5
    h = synth.hidden(sh, 3, 0, n).astype(np.float64)
    a, _ = _tiny_stage(qtype)
    b, _ = _tiny_stage(qtype)
    c, _ = _tiny_stage(qtype)
    out_b = a.forward(h, 20)
    out_s = b.forward_sequential(h, 20)
    assert np.allclose(out_b, out_s, rtol=1e-13, atol=0)
    j = 3
    a.commit(j)
    c.forward_sequential(h[:j], 20)
    assert a.kv_len == c.kv_len == 20 + j
    for l in a.S:
        assert np.allclose(a.S[l], c.S[l], rtol=1e-13, atol=1e-16)
    for l in a.K:
        assert np.array_equal(a.K[l][:, :a.kv_len], c.K[l][:, :c.kv_len])


def test_stage_rollback_restores_state_exactly():
    sh = TINY
    st, _ = _tiny_stage()
    before = {l: s.copy() for l, s in st.S.items()}
    kv_before = st.kv_len
    st.forward(synth.hidden(sh, 4, 0, 4).astype(np.float64), 20)
    st.rollback()
    assert st.kv_len == kv_before
    for l in before:
        assert np.array_equal(st.S[l], before[l])


def test_stage_split_equals_whole():
    """Layers [0,4) in one stage equal [0,2) then [2,4) with the hidden handed over."""
    sh = TINY
    h = synth.hidden(sh, 5, 0, 2).astype(np.float64)
    whole, _ = _tiny_stage(begin=0, end=4)
    first, _ = _tiny_stage(begin=0, end=2)
    second, _ = _tiny_stage(begin=2, end=4)
    out_w = whole.forward(h, 20)
    out_s = second.forward(first.forward(h, 20), 20)
    assert np.array_equal(out_w, out_s)


def test_stage_rejects_protocol_errors():
    sh = TINY
    st, _ = _tiny_stage()
    h = synth.hidden(sh, 6, 0, 1).astype(np.float64)
    with pytest.raises(ValueError):
        st.forward(h, 19)
    st.forward(h, 20)
    with pytest.raises(RuntimeError):
        st.forward(h, 21)
    with pytest.raises(ValueError):
        st.commit(2)
    st.commit(1)
    with pytest.raises(RuntimeError):
        st.commit(0)


def test_max_rel_err_definition():
    assert oracle.max_rel_err([1.0, 2.0], [1.0, 2.0]) == 0.0
    assert oracle.max_rel_err([1.0, 2.002], [1.0, 2.0]) == pytest.approx(1e-3)


# ------------------------------------------------- layer wiring, closed form --
# A constant hidden vector makes RMSNorm a closed form (c / sqrt(c^2 + eps) * gamma)
# and one-hot Q4_0 rows make every projection pick one scaled input, so a whole
# layer reduces to a few scalar formulas.  These pin the composition
# h += mixer(RMSNorm_1(h)); h += W_down(silu(W_gate x) * W_up x), x = RMSNorm_2(h)
# (ChatTorrent README, "What it can run"): a swapped norm weight, an FFN fed the
# un-normed h, gate and up exchanged, or a missing residual fails them.

def _onehot_q4(rows, cols, picks, scales):
    """GGUF Q4_0 blocks of a [rows, cols] matrix whose row r is scales[r] at
    column picks[r] and 0 elsewhere (nibble 9 = +1 unit there, 8 elsewhere)."""
    scales = np.ascontiguousarray(np.broadcast_to(np.asarray(scales, dtype=np.float16), (rows,)))
    W = np.empty((rows, cols // 32, 18), np.uint8)
    W[:, :, 0:2] = scales.view(np.uint8).reshape(rows, 1, 2)
    W[:, :, 2:] = 0x88
    for r, c in enumerate(picks):
        b, j = divmod(int(c), 32)
        byte = 2 + j % 16
        W[r, b, byte] = (W[r, b, byte] & 0xF0) | 0x09 if j < 16 else (W[r, b, byte] & 0x0F) | 0x90
    return W


def _zero_q4(W):
    Z = W.copy()
    Z[:, :, 2:] = 0x88
    return Z


def test_onehot_helper_dequantises_to_the_intended_matrix():
    W = _onehot_q4(3, 64, [0, 17, 63], [0.5, -1.5, 2.0])
    A = oracle.dequant(Q4_0, W)
    want = np.zeros((3, 64))
    want[0, 0], want[1, 17], want[2, 63] = 0.5, -1.5, 2.0
    assert np.array_equal(A, want)


def test_layer_wiring_ffn_reads_norm2_and_adds_to_h():
    sh = TINY
    H, F = sh.hidden, sh.ffn
    t = synth.stage_tensors(sh, Q4_0, 7, 0, 1)                    # layer 0: gated DeltaNet
    g1 = t["blk.0.norm1"].astype(np.float64)
    g2 = t["blk.0.norm2"].astype(np.float64)
    assert not np.allclose(g1, g2)
    rng = np.random.default_rng(70)
    cg, cu, cd = rng.integers(0, H, F), rng.integers(0, H, F), rng.integers(0, F, H)
    t["blk.0.dn_out"] = _zero_q4(t["blk.0.dn_out"])              # the mixer adds exact zeros
    t["blk.0.ffn_gate"] = _onehot_q4(F, H, cg, 0.75)
    t["blk.0.ffn_up"] = _onehot_q4(F, H, cu, -1.5)
    t["blk.0.ffn_down"] = _onehot_q4(H, F, cd, 0.5)
    st = oracle.OracleStage(sh, Q4_0, t, 0, 1, 8)
    st.set_dn_state(0, synth.dn_state(sh, 7, 0, 0.3))
    consts = np.array([1.7, -0.4])
    h = np.repeat(consts[:, None], H, axis=1)
    out = st.forward(h, 0)
    for i, c in enumerate(consts):
        x2 = c / np.sqrt(c * c + sh.eps) * g2
        g, u = 0.75 * x2[cg], -1.5 * x2[cu]
        f = g / (1.0 + np.exp(-g)) * u
        np.testing.assert_allclose(out[i], c + 0.5 * f[cd], rtol=1e-13, atol=1e-15)


def test_layer_wiring_attention_reads_norm1_and_adds_gated_v_to_h():
    """Attention layer at position 0: the softmax runs over one cached row (the
    token's own), so o = v as stored in the f16 cache, then o * sigmoid(gate)."""
    sh = TINY
    H = sh.hidden
    l = 3
    assert sh.is_attention(l)
    t = synth.stage_tensors(sh, Q4_0, 8, l, l + 1)
    g1 = t[f"blk.{l}.norm1"].astype(np.float64)
    Hq, Hkv, dh = sh.att_q_heads, sh.att_kv_heads, sh.att_dim
    rep = Hq // Hkv
    nq, nkv = Hq * dh, Hkv * dh
    rows = 2 * nq + 2 * nkv                                       # q | gate | k | v
    rng = np.random.default_rng(80)
    picks = rng.integers(0, H, rows)
    scales = np.full(rows, 0.5)
    scales[nq:2 * nq] = -0.75                                     # gate rows
    scales[2 * nq + nkv:] = 1.25                                  # v rows
    t[f"blk.{l}.attn_in"] = _onehot_q4(rows, H, picks, scales)
    co = rng.integers(0, nq, H)
    t[f"blk.{l}.attn_out"] = _onehot_q4(H, nq, co, 0.25)
    for tag in ("ffn_gate", "ffn_up", "ffn_down"):
        t[f"blk.{l}.{tag}"] = _zero_q4(t[f"blk.{l}.{tag}"])      # the FFN adds exact zeros
    st = oracle.OracleStage(sh, Q4_0, t, l, l + 1, 8)
    c = 0.9
    h = np.full((1, H), c)
    out = st.forward(h, 0)
    x1 = c / np.sqrt(c * c + sh.eps) * g1
    gate = -0.75 * x1[picks[nq:2 * nq]]
    v = 1.25 * x1[picks[2 * nq + nkv:]]                          # [Hkv * dh]
    v16 = v.astype(np.float16).astype(np.float64)                # the cache holds f16
    j = np.arange(nq)
    o = v16[(j // dh) // rep * dh + j % dh] / (1.0 + np.exp(-gate))
    np.testing.assert_allclose(out[0], c + 0.25 * o[co], rtol=1e-13, atol=1e-15)


def test_layer_wiring_deltanet_rows_maps_heads_and_readout():
    """One token through a gated-DeltaNet layer from a random state S0, with the
    FFN zeroed and one-hot in/out projections: per value head h (key head
    g = h // (Hv/Hk)), in the rank-one form of the update read out after it,
        o_h = alpha_h (S0_h q - beta_h (S0_h k)(k.q)) + beta_h v_h (k.q),
    q, k L2-normalised, beta = sigmoid(b), alpha = exp(-softplus(a)) = 1/(1+e^a),
    in-projection rows q | k | v | b | a."""
    sh = TINY
    H = sh.hidden
    Hk, Hv, d = sh.dn_k_heads, sh.dn_v_heads, sh.dn_dim
    rep = Hv // Hk
    t = synth.stage_tensors(sh, Q4_0, 9, 0, 1)
    g1 = t["blk.0.norm1"].astype(np.float64)
    rows = 2 * Hk * d + Hv * d + 2 * Hv
    rng = np.random.default_rng(90)
    picks = rng.integers(0, H, rows)
    scales = np.empty(rows)
    o_k, o_v, o_b = Hk * d, 2 * Hk * d, 2 * Hk * d + Hv * d
    scales[:o_k], scales[o_k:o_v], scales[o_v:o_b] = 0.5, -0.75, 1.25
    scales[o_b:o_b + Hv], scales[o_b + Hv:] = 0.5, -1.0
    t["blk.0.dn_in"] = _onehot_q4(rows, H, picks, scales)
    co = rng.integers(0, Hv * d, H)
    t["blk.0.dn_out"] = _onehot_q4(H, Hv * d, co, 0.25)
    for tag in ("ffn_gate", "ffn_up", "ffn_down"):
        t[f"blk.0.{tag}"] = _zero_q4(t[f"blk.0.{tag}"])
    S0 = synth.dn_state(sh, 9, 0, 0.3).astype(np.float64)        # [Hv, dv, dk]
    st = oracle.OracleStage(sh, Q4_0, t, 0, 1, 8)
    st.set_dn_state(0, S0.astype(np.float32))
    c = 1.3
    out = st.forward(np.full((1, H), c), 0)
    y = scales * (c / np.sqrt(c * c + sh.eps) * g1)[picks]        # the in-projection, row by row
    q = y[:o_k].reshape(Hk, d)
    k = y[o_k:o_v].reshape(Hk, d)
    v = y[o_v:o_b].reshape(Hv, d)
    b, a = y[o_b:o_b + Hv], y[o_b + Hv:]
    q = q / np.sqrt((q * q).sum(-1, keepdims=True) + 1e-6)
    k = k / np.sqrt((k * k).sum(-1, keepdims=True) + 1e-6)
    beta, alpha = 1.0 / (1.0 + np.exp(-b)), 1.0 / (1.0 + np.exp(a))
    S0 = S0.astype(np.float32).astype(np.float64)
    o = np.empty((Hv, d))
    for h in range(Hv):
        gq, gk = q[h // rep], k[h // rep]
        kq = gk @ gq
        o[h] = alpha[h] * (S0[h] @ gq - beta[h] * (S0[h] @ gk) * kq) + beta[h] * v[h] * kq
    np.testing.assert_allclose(out[0], c + 0.25 * o.reshape(-1)[co], rtol=1e-12, atol=1e-14)
