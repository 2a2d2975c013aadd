"""The seeded inputs follow the recipe the workload states (CPU).

Determinism and independence of the per-tensor streams, the documented
shapes and byte layouts, and the distributions: Q4_0 scales f16(|N(0,1)| 0.02)
with uniform nibbles, Q8_0 scales times 8/127 with int8 uniform on [-127, 127],
norm weights 1 + N(0, 0.02), hidden N(0, 1), DeltaNet state N(0, 0.01), KV
prefill N(0, 1) in f16 with the rows past the context left zero.
"""
import math

import numpy as np

import synth
from synth import FULL, Q4_0, Q8_0, TINY

HALF_NORMAL_MEAN = math.sqrt(2.0 / math.pi)   # E|N(0,1)|


def _scales(W):
    return W[:, :, 0:2].copy().view(np.float16)[..., 0].astype(np.float64)


def test_streams_are_deterministic_and_independent():
    a = synth.qmatrix(Q4_0, synth.rng_for(5, 3, 9), 64, 256)
    b = synth.qmatrix(Q4_0, synth.rng_for(5, 3, 9), 64, 256)
    c = synth.qmatrix(Q4_0, synth.rng_for(5, 4, 9), 64, 256)     # another layer
    d = synth.qmatrix(Q4_0, synth.rng_for(6, 3, 9), 64, 256)     # another seed
    assert np.array_equal(a, b)
    assert not np.array_equal(a, c) and not np.array_equal(a, d)
    # a subset of layers is generated exactly as inside the full range
    t_all = synth.stage_tensors(TINY, Q4_0, 2, 0, 4)
    t_sub = synth.stage_tensors(TINY, Q4_0, 2, 2, 3)
    for k, v in t_sub.items():
        assert np.array_equal(v, t_all[k])


def test_q4_0_scales_and_nibbles():
    W = synth.qmatrix(Q4_0, synth.rng_for(0, 0, synth.TAGS["gemv_w"]), 1024, 1024)
    assert W.shape == (1024, 32, 18) and W.dtype == np.uint8
    d = _scales(W)
    assert np.all(d >= 0) and np.all(np.isfinite(d))
    assert abs(d.mean() / (0.02 * HALF_NORMAL_MEAN) - 1) < 0.02
    q = W[:, :, 2:]
    nib = np.concatenate([(q & 0xF).ravel(), (q >> 4).ravel()])
    counts = np.bincount(nib, minlength=16)
    expect = nib.size / 16
    chi2 = float(((counts - expect) ** 2 / expect).sum())
    assert chi2 < 60.0                                             # 15 dof: p ~ 1e-7
    # weights (nibble - 8) * d have the magnitude of the model's Q4_0 layers
    assert abs(np.mean(nib) - 7.5) < 0.01


def test_q8_0_scales_and_codes():
    W = synth.qmatrix(Q8_0, synth.rng_for(0, 0, synth.TAGS["gemv_w"]), 512, 1024)
    assert W.shape == (512, 32, 34)
    d = _scales(W)
    assert abs(d.mean() / (0.02 * 8 / 127 * HALF_NORMAL_MEAN) - 1) < 0.03
    q = W[:, :, 2:].view(np.int8).astype(np.int64)
    assert q.min() == -127 and q.max() == 127                      # -128 never drawn
    assert abs(q.mean()) < 0.5
    assert abs(q.std() / math.sqrt((255 ** 2 - 1) / 12) - 1) < 0.01


def test_stage_tensor_shapes_and_norm_weights():
    t = synth.stage_tensors(FULL, Q4_0, 4, 2, 4)                   # layers 2 (DeltaNet) and 3 (attention)
    H, F = FULL.hidden, FULL.ffn
    assert t["blk.2.dn_in"].shape == (FULL.dn_in_rows, H // 32, 18)
    assert t["blk.2.dn_out"].shape == (H, FULL.dn_o // 32, 18)
    assert t["blk.3.attn_in"].shape == (FULL.attn_in_rows, H // 32, 18)
    assert t["blk.3.attn_out"].shape == (H, FULL.attn_o // 32, 18)
    for l in (2, 3):
        assert t[f"blk.{l}.ffn_gate"].shape == t[f"blk.{l}.ffn_up"].shape == (F, H // 32, 18)
        assert t[f"blk.{l}.ffn_down"].shape == (H, F // 32, 18)
    assert FULL.dn_in_rows == 2 * 16 * 128 + 48 * 128 + 2 * 48
    assert FULL.attn_in_rows == 2 * 24 * 256 + 2 * 4 * 256
    g = np.concatenate([t["blk.2.norm1"], t["blk.2.norm2"], t["blk.3.norm1"], t["blk.3.norm2"]]).astype(np.float64)
    assert t["blk.3.attn_q_norm"].shape == t["blk.3.attn_k_norm"].shape == (FULL.att_dim,)
    assert abs(g.mean() - 1.0) < 1e-3 and abs(g.std() / 0.02 - 1) < 0.05


def test_activations_states_and_kv_prefill():
    h = synth.hidden(FULL, 4, 0, 16)
    assert h.shape == (16, FULL.hidden) and h.dtype == np.float32
    assert abs(h.mean()) < 0.01 and abs(h.std() - 1) < 0.01
    S = synth.dn_state(FULL, 4, 0, 0.01)
    assert S.shape == (FULL.dn_v_heads, FULL.dn_dim, FULL.dn_dim) and S.dtype == np.float32
    assert abs(S.std() / 0.01 - 1) < 0.01
    K, V = synth.kv_prefill(FULL, 4, 3, 100, 160)
    assert K.shape == V.shape == (FULL.att_kv_heads, 160, FULL.att_dim) and K.dtype == np.float16
    assert not np.any(K[:, 100:]) and not np.any(V[:, 100:])
    assert abs(K[:, :100].astype(np.float64).std() - 1) < 0.05
    assert not np.array_equal(K[:, :100], V[:, :100])
