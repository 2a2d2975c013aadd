"""GPU parity of the single kernels against the oracle, through the C ABI.

* the quantised GEMV (single 1024x1024 Q4_0 GEMV at batch 1, seed 0; ragged
  shapes; every n_tok; the stage's full-size matrices on sampled rows),
* bit-exact dequantisation of repacked Q4_0 / Q8_0 weights,
* the gated-DeltaNet state step alone (48 value / 16 key heads of 128, S0 ~
  N(0, 0.01), n_tok 1 and 16, rollback to a seeded accepted prefix, seed 1).
"""
import numpy as np
import pytest

import oracle
import synth
from synth import FULL, Q4_0, Q8_0
from stage_helpers import TOL, gemv_error_bound, rel_err_heads, rel_err_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    import torch
    assert torch.cuda.is_available(), "GPU test needs CUDA"
    import quantized_hybrid_layer_b200 as q
    return q


def packed_on_gpu(q, qtype, W, W2=None):
    import torch
    rows, nb, _ = W.shape
    cols = nb * 32
    g = torch.from_numpy(np.ascontiguousarray(W).reshape(-1)).cuda()
    g2 = torch.from_numpy(np.ascontiguousarray(W2).reshape(-1)).cuda() if W2 is not None else None
    P = torch.empty(q.qhl_packed_bytes(qtype, rows, cols, paired=W2 is not None), dtype=torch.uint8, device="cuda")
    q.qhl_repack(qtype, rows, cols, g, P, gguf_b=g2)
    return P


def gemv_gpu(q, qtype, P, rows, cols, x):
    import torch
    xt = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()
    y = torch.empty((x.shape[0], rows), dtype=torch.float32, device="cuda")
    q.qhl_qgemv(qtype, rows, cols, P, xt, y)
    torch.cuda.synchronize()
    return y.cpu().numpy()


# ------------------------------------------------------------------ GEMV --

def test_single_q4_0_gemv_1024(q):
    W, x = synth.gemv_problem(0, 1024, 1024, 1)
    P = packed_on_gpu(q, Q4_0, W)
    y = gemv_gpu(q, Q4_0, P, 1024, 1024, x)
    ref = oracle.qgemv(Q4_0, W, x)
    err = rel_err_rows(y, ref)
    assert max(err) <= TOL, err
    assert np.all(np.abs(y - ref) <= gemv_error_bound(Q4_0, W, x))
    # x enters as block fixed point (step <= 2^-21 of the block max): the error
    # stays far inside the bound
    assert max(err) <= 2e-4


@pytest.mark.parametrize("qtype", [Q4_0, Q8_0])
@pytest.mark.parametrize("rows,cols", [(1, 256), (63, 512), (65, 256), (1000, 1280), (77, 5120)])
@pytest.mark.parametrize("n", [1, 3, 4, 16])
def test_gemv_ragged_shapes(q, qtype, rows, cols, n):
    W, x = synth.gemv_problem(5 + rows + cols, rows, cols, n, qtype)
    P = packed_on_gpu(q, qtype, W)
    y = gemv_gpu(q, qtype, P, rows, cols, x)
    ref = oracle.qgemv(qtype, W, x)
    assert max(rel_err_rows(y, ref)) <= TOL
    assert np.all(np.abs(y - ref) <= gemv_error_bound(qtype, W, x))


# (1500, 2304): one item per CTA; (4000, 5120): four or five items per CTA
# through the rings, with stream-K fix-ups
@pytest.mark.parametrize("qtype", [Q4_0, Q8_0])
@pytest.mark.parametrize("rows,cols", [(1500, 2304), (4000, 5120)])
def test_gemv_batched_is_bit_identical_to_single_tokens(q, qtype, rows, cols):
    W, x = synth.gemv_problem(21, rows, cols, 16, qtype)
    P = packed_on_gpu(q, qtype, W)
    # every n forms the same exact integer block sums on the tensor cores (MMA
    # N = 8 rows per token) and the same f32 updates, so every n equals the
    # single-token results
    for n in (16, 9, 8, 7, 5, 4, 3, 2):
        yb = gemv_gpu(q, qtype, P, rows, cols, x[:n])
        for t in range(n):
            y1 = gemv_gpu(q, qtype, P, rows, cols, x[t:t + 1])
            assert np.array_equal(yb[t], y1[0])


@pytest.mark.parametrize("rows,cols", [(FULL.dn_in_rows, FULL.hidden), (FULL.hidden, FULL.dn_o),
                                       (FULL.attn_in_rows, FULL.hidden), (FULL.ffn, FULL.hidden),
                                       (FULL.hidden, FULL.ffn)])
@pytest.mark.parametrize("n", [1, 16])
@pytest.mark.parametrize("qtype", [Q4_0, Q8_0])
def test_gemv_full_size_sampled_rows(q, rows, cols, n, qtype):
    W, x = synth.gemv_problem(31, rows, cols, n, qtype)
    P = packed_on_gpu(q, qtype, W)
    y = gemv_gpu(q, qtype, P, rows, cols, x)
    idx = np.sort(np.random.default_rng(rows + cols).choice(rows, size=min(rows, 192), replace=False))
    idx = np.unique(np.concatenate([idx, [0, rows - 1]]))
    ref = oracle.qgemv(qtype, W[idx], x)            # the oracle computes just these rows
    assert max(rel_err_rows(y[:, idx], ref)) <= TOL
    assert np.all(np.abs(y[:, idx] - ref) <= gemv_error_bound(qtype, W[idx], x))


# ------------------------------------------------------------- dequant --

@pytest.mark.parametrize("qtype", [Q4_0, Q8_0])
def test_dequant_bit_exact(q, qtype):
    import torch
    rows, cols = 130, 512
    W = synth.qmatrix(qtype, synth.rng_for(41, 0, 1), rows, cols)
    # plant edge scales: subnormal, zero, negative, largest finite
    W[0, :, 0:2] = np.frombuffer(np.array([0x0001], np.uint16).tobytes(), np.uint8)
    W[1, :, 0:2] = 0
    W[2, :, 0:2] = np.frombuffer(np.array([0xBC00], np.uint16).tobytes(), np.uint8)
    W[3, :, 0:2] = np.frombuffer(np.array([0x7BFF], np.uint16).tobytes(), np.uint8)
    P = packed_on_gpu(q, qtype, W)
    out = torch.empty((rows, cols), dtype=torch.float32, device="cuda")
    q.qhl_dequant(qtype, rows, cols, P, 0, rows, out)
    torch.cuda.synchronize()
    got = out.cpu().numpy().astype(np.float64)
    assert np.array_equal(got, oracle.dequant(qtype, W))


@pytest.mark.parametrize("qtype", [Q4_0, Q8_0])
def test_dequant_paired_gate_up_bit_exact(q, qtype):
    import torch
    F, H = 100, 256
    A = synth.qmatrix(qtype, synth.rng_for(42, 0, 1), F, H)
    B = synth.qmatrix(qtype, synth.rng_for(42, 0, 2), F, H)
    P = packed_on_gpu(q, qtype, A, B)
    out = torch.empty((2 * F, H), dtype=torch.float32, device="cuda")
    q.qhl_dequant(qtype, F, H, P, 0, 2 * F, out, paired=True)
    torch.cuda.synchronize()
    got = out.cpu().numpy().astype(np.float64)
    assert np.array_equal(got[:F], oracle.dequant(qtype, A))
    assert np.array_equal(got[F:], oracle.dequant(qtype, B))


# ------------------------------------------------------------ DeltaNet --

def _dn_y(q_, k_, v_, b_, a_):
    n = q_.shape[0]
    return np.concatenate([q_.reshape(n, -1), k_.reshape(n, -1), v_.reshape(n, -1), b_, a_], axis=1).astype(np.float32)


def _dn_gpu(q, S0, y):
    import torch
    sh = FULL
    n = y.shape[0]
    yt = torch.from_numpy(y).cuda()
    s_in = torch.from_numpy(np.ascontiguousarray(S0)).cuda()
    snaps = torch.empty((n, sh.dn_v_heads, sh.dn_dim, sh.dn_dim), dtype=torch.float32, device="cuda")
    o = torch.empty((n, sh.dn_v_heads * sh.dn_dim), dtype=torch.float32, device="cuda")
    q.qhl_deltanet_step(sh.dn_k_heads, sh.dn_v_heads, yt, s_in, snaps, o)
    torch.cuda.synchronize()
    return o.cpu().numpy(), snaps.cpu().numpy()


@pytest.mark.parametrize("n", [1, 16])
def test_deltanet_step_matches_oracle(q, n):
    sh = FULL
    S0, q_, k_, v_, b_, a_ = synth.deltanet_step_problem(sh, 1, n)
    o, snaps = _dn_gpu(q, S0, _dn_y(q_, k_, v_, b_, a_))
    o_ref, s_ref = oracle.deltanet_steps(S0, q_, k_, v_, b_, a_, sh)
    for t in range(n):
        assert max(rel_err_heads(o[t].reshape(sh.dn_v_heads, -1), o_ref[t])) <= TOL
        assert max(rel_err_heads(snaps[t], s_ref[t + 1])) <= TOL


def test_deltanet_batched_equals_sequential_and_rollback_prefix(q):
    sh = FULL
    n = 16
    S0, q_, k_, v_, b_, a_ = synth.deltanet_step_problem(sh, 1, n)
    y = _dn_y(q_, k_, v_, b_, a_)
    o_b, snaps_b = _dn_gpu(q, S0, y)
    S = S0
    seq = [S0]
    for t in range(n):
        o1, s1 = _dn_gpu(q, S, y[t:t + 1])
        assert np.array_equal(o1[0], o_b[t])
        S = s1[0]
        seq.append(S)
        assert np.array_equal(S, snaps_b[t])
    j = synth.accepted_prefix(1, 0, n)
    kept = S0 if j == 0 else snaps_b[j - 1]
    assert np.array_equal(kept, seq[j])


def test_qgemv_wait_that_runs_out_is_reported_by_qhl_sync(q):
    """qhl_debug_inject makes CTA 0 skip one item of the next qhl_qgemv calls
    with every wait capped short: the call returns, qhl_sync raises
    STAGE_E_DEVICE once (clearing the error word and the tile counters), and
    with injection off the next call gives the reference bits again."""
    import torch
    rows, cols = 1000, 5120
    W, x = synth.gemv_problem(71, rows, cols, 1)
    P = packed_on_gpu(q, Q4_0, W)
    ref = gemv_gpu(q, Q4_0, P, rows, cols, x)
    q.qhl_sync()
    try:
        q.qhl_debug_inject(0, 4096)
        gemv_gpu(q, Q4_0, P, rows, cols, x)
        with pytest.raises(q.StageError) as e:
            q.qhl_sync()
        assert e.value.code == -7
        q.qhl_sync()
    finally:
        q.qhl_debug_inject(-1, 0)
    assert np.array_equal(gemv_gpu(q, Q4_0, P, rows, cols, x), ref)
    q.qhl_sync()
