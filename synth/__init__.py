"""Seeded synthetic inputs for the quantized hybrid layer-stage.

This module is shared by the CUDA path (tests, bench) and by the oracle.  It
holds none of the method's arithmetic: it only draws random numbers with numpy's
PCG64 generator in a fixed, documented order and packs them into the byte
layouts the pages name (GGUF Q4_0 / Q8_0 blocks with binary16 scales, f32
activations and norm weights, f16 KV-cache rows).

Workload recipe (one stream per tensor, so any subset can be regenerated alone):

* Every tensor gets its own generator ``PCG64(SeedSequence(seed, spawn_key=key))``
  where ``key = (layer, tag)`` for weights and ``(layer, tag)`` / ``(step, tag)``
  for states and activations; ``seed`` is the workload seed (0 for the single
  GEMV, 1 for the DeltaNet step, 2 for the 4-layer stage, 3 for the verify
  pass, 4 for the 64-layer stage).
* Q4_0 matrix [rows, cols]: first ``rows*cols/32`` scale draws
  ``d = f16(|N(0,1)| * 0.02)`` (row-major over (row, block)), then
  ``rows*cols/32*16`` uniform random bytes (two uniform nibbles each).
* Q8_0 matrix: scale draws ``d = f16(|N(0,1)| * 0.02 * 8/127)``, then
  ``rows*cols`` int8 draws uniform on [-127, 127].  (Reading: the Q8_0 variant
  is the same model quantised to 8 bits, so a block's scale is the Q4_0 scale
  times 8/127, as a max-abs quantiser gives for 4-bit [-8, 7] vs 8-bit
  [-127, 127] codes; weights then have the Q4_0 magnitudes.)
* RMSNorm / QK-norm weights: ``1 + N(0, 0.02)`` in f32.
* Hidden states: ``N(0, 1)`` f32.  DeltaNet states: ``N(0, 0.01)`` f32.
  KV-cache prefill: ``N(0, 1)`` rounded to f16.
* ``N(0, s)`` always means standard deviation ``s``.

Layout conventions of the weight tensors handed to ``stage_load`` (names are
``blk.<layer>.<tag>``; row order inside the fused mixer in-projections):

* ``dn_in``   [2*Hk*dk + Hv*dv + 2*Hv, hidden]: rows q | k | v | b | a
* ``dn_out``  [hidden, Hv*dv]
* ``attn_in`` [2*Hq*dh + 2*Hkv*dh, hidden]:    rows q | gate | k | v
* ``attn_out`` [hidden, Hq*dh]
* ``ffn_gate``, ``ffn_up`` [ffn, hidden]; ``ffn_down`` [hidden, ffn]
* ``norm1``, ``norm2`` f32 [hidden]; ``attn_q_norm``, ``attn_k_norm`` f32 [dh]
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import numpy as np

QK = 32                      # weights per GGUF block (Q4_0 and Q8_0)
Q4_0 = 2                     # GGUF type ids
Q8_0 = 8
BLOCK_BYTES = {Q4_0: 18, Q8_0: 34}

# tensor tags (second element of a weight's spawn key)
TAGS = {
    "norm1": 1, "norm2": 2, "dn_in": 3, "dn_out": 4, "attn_in": 5,
    "attn_q_norm": 6, "attn_k_norm": 7, "attn_out": 8, "ffn_gate": 9,
    "ffn_up": 10, "ffn_down": 11,
    # states and activations
    "dn_state": 20, "kv_k": 21, "kv_v": 22, "hidden": 30,
    "gemv_w": 40, "gemv_x": 41,
    "step_q": 50, "step_k": 51, "step_v": 52, "step_b": 53, "step_a": 54,
    "step_s0": 55, "accept": 60,
}


@dataclass(frozen=True)
class StageShape:
    """Shapes of one hybrid decoder stack (the 27B-class hybrid by default)."""
    hidden: int = 5120
    ffn: int = 17408
    dn_k_heads: int = 16
    dn_v_heads: int = 48
    dn_dim: int = 128
    att_q_heads: int = 24
    att_kv_heads: int = 4
    att_dim: int = 256
    rope_dims: int = 64
    rope_theta: float = 1.0e7
    eps: float = 1.0e-6
    attn_every: int = 4      # layer i is full attention iff i % attn_every == attn_every - 1

    def is_attention(self, layer: int) -> bool:
        return layer % self.attn_every == self.attn_every - 1

    @property
    def dn_in_rows(self) -> int:
        return 2 * self.dn_k_heads * self.dn_dim + self.dn_v_heads * self.dn_dim + 2 * self.dn_v_heads

    @property
    def dn_o(self) -> int:
        return self.dn_v_heads * self.dn_dim

    @property
    def attn_in_rows(self) -> int:
        return 2 * self.att_q_heads * self.att_dim + 2 * self.att_kv_heads * self.att_dim

    @property
    def attn_o(self) -> int:
        return self.att_q_heads * self.att_dim


FULL = StageShape()
#: a small stack with the same structure, for CPU-only oracle tests
TINY = StageShape(hidden=256, ffn=512, dn_k_heads=2, dn_v_heads=6, dn_dim=16,
                  att_q_heads=4, att_kv_heads=2, att_dim=32, rope_dims=8,
                  rope_theta=1.0e4)


def rng_for(seed: int, *key: int) -> np.random.Generator:
    """Independent PCG64 stream for one tensor: SeedSequence(seed, spawn_key=key)."""
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(seed, spawn_key=tuple(int(k) for k in key))))


def _scales(rng: np.random.Generator, nblocks: int, scale: float = 0.02) -> np.ndarray:
    return (np.abs(rng.standard_normal(nblocks)) * scale).astype(np.float16)


def q4_0_matrix(rng: np.random.Generator, rows: int, cols: int) -> np.ndarray:
    """GGUF Q4_0 blocks, uint8 [rows, cols/32, 18]: binary16 d then 16 nibble bytes."""
    assert cols % QK == 0
    nb = cols // QK
    d = _scales(rng, rows * nb)
    qs = np.frombuffer(rng.bytes(rows * nb * 16), dtype=np.uint8)
    out = np.empty((rows, nb, 18), dtype=np.uint8)
    out[:, :, 0:2] = d.view(np.uint8).reshape(rows, nb, 2)
    out[:, :, 2:] = qs.reshape(rows, nb, 16)
    return out


def q8_0_matrix(rng: np.random.Generator, rows: int, cols: int) -> np.ndarray:
    """GGUF Q8_0 blocks, uint8 [rows, cols/32, 34]: binary16 d then 32 int8 in [-127, 127]."""
    assert cols % QK == 0
    nb = cols // QK
    d = _scales(rng, rows * nb, 0.02 * 8.0 / 127.0)
    qs = rng.integers(-127, 128, size=(rows, nb, 32), dtype=np.int8)
    out = np.empty((rows, nb, 34), dtype=np.uint8)
    out[:, :, 0:2] = d.view(np.uint8).reshape(rows, nb, 2)
    out[:, :, 2:] = qs.view(np.uint8)
    return out


def qmatrix(qtype: int, rng: np.random.Generator, rows: int, cols: int) -> np.ndarray:
    if qtype == Q4_0:
        return q4_0_matrix(rng, rows, cols)
    if qtype == Q8_0:
        return q8_0_matrix(rng, rows, cols)
    raise ValueError(f"unsupported qtype {qtype}")


def norm_weight(rng: np.random.Generator, n: int) -> np.ndarray:
    return (1.0 + 0.02 * rng.standard_normal(n)).astype(np.float32)


def normal_f32(rng: np.random.Generator, shape, std: float = 1.0) -> np.ndarray:
    return (std * rng.standard_normal(shape)).astype(np.float32)


def layer_tensors(shape: StageShape, qtype: int, seed: int, layer: int) -> dict:
    """All weight tensors of one decoder layer, keyed by ``blk.<layer>.<tag>``."""
    H, F = shape.hidden, shape.ffn
    t = {}

    def w(tag, rows, cols):
        t[f"blk.{layer}.{tag}"] = qmatrix(qtype, rng_for(seed, layer, TAGS[tag]), rows, cols)

    def g(tag, n):
        t[f"blk.{layer}.{tag}"] = norm_weight(rng_for(seed, layer, TAGS[tag]), n)

    g("norm1", H)
    if shape.is_attention(layer):
        w("attn_in", shape.attn_in_rows, H)
        g("attn_q_norm", shape.att_dim)
        g("attn_k_norm", shape.att_dim)
        w("attn_out", H, shape.attn_o)
    else:
        w("dn_in", shape.dn_in_rows, H)
        w("dn_out", H, shape.dn_o)
    g("norm2", H)
    w("ffn_gate", F, H)
    w("ffn_up", F, H)
    w("ffn_down", H, F)
    return t


def stage_tensors(shape: StageShape, qtype: int, seed: int, begin: int, end: int) -> dict:
    t = {}
    for layer in range(begin, end):
        t.update(layer_tensors(shape, qtype, seed, layer))
    return t


def dn_state(shape: StageShape, seed: int, layer: int, std: float = 0.01) -> np.ndarray:
    """Initial DeltaNet state of one layer, f32 [Hv, dv, dk] ~ N(0, std)."""
    return normal_f32(rng_for(seed, layer, TAGS["dn_state"]),
                      (shape.dn_v_heads, shape.dn_dim, shape.dn_dim), std)


def kv_prefill(shape: StageShape, seed: int, layer: int, ctx: int, max_ctx: int):
    """KV cache of one attention layer, f16 [Hkv, max_ctx, dh] each; rows < ctx ~ N(0,1), rest 0."""
    out = []
    for tag in ("kv_k", "kv_v"):
        c = np.zeros((shape.att_kv_heads, max_ctx, shape.att_dim), dtype=np.float16)
        rng = rng_for(seed, layer, TAGS[tag])
        c[:, :ctx, :] = rng.standard_normal((shape.att_kv_heads, ctx, shape.att_dim)).astype(np.float16)
        out.append(c)
    return out[0], out[1]


def hidden(shape: StageShape, seed: int, step: int, n_tok: int) -> np.ndarray:
    """Input hidden states for one pass, f32 [n_tok, hidden] ~ N(0, 1)."""
    return normal_f32(rng_for(seed, step, TAGS["hidden"]), (n_tok, shape.hidden))


def accepted_prefix(seed: int, step: int, n_tok: int) -> int:
    """Seeded accepted-draft length, uniform on 0..n_tok."""
    return int(rng_for(seed, step, TAGS["accept"]).integers(0, n_tok + 1))


def gemv_problem(seed: int, rows: int, cols: int, n_tok: int, qtype: int = Q4_0):
    """A single quantized GEMV: W [rows, cols] in GGUF blocks and x f32 [n_tok, cols]."""
    W = qmatrix(qtype, rng_for(seed, 0, TAGS["gemv_w"]), rows, cols)
    x = normal_f32(rng_for(seed, 0, TAGS["gemv_x"]), (n_tok, cols))
    return W, x


def deltanet_step_problem(shape: StageShape, seed: int, n_tok: int):
    """Raw per-token DeltaNet inputs for the state-step kernel alone.

    Returns S0 f32 [Hv, dv, dk] ~ N(0, 0.01) and, per token, raw q, k f32
    [n, Hk, dk], v f32 [n, Hv, dv], b, a f32 [n, Hv], all ~ N(0, 1).  The
    L2 normalisation of q, k and the maps b -> beta, a -> alpha belong to the
    method and are applied by the code under test.
    """
    Hk, Hv, d = shape.dn_k_heads, shape.dn_v_heads, shape.dn_dim
    S0 = normal_f32(rng_for(seed, 0, TAGS["step_s0"]), (Hv, d, d), 0.01)
    q = normal_f32(rng_for(seed, 0, TAGS["step_q"]), (n_tok, Hk, d))
    k = normal_f32(rng_for(seed, 0, TAGS["step_k"]), (n_tok, Hk, d))
    v = normal_f32(rng_for(seed, 0, TAGS["step_v"]), (n_tok, Hv, d))
    b = normal_f32(rng_for(seed, 0, TAGS["step_b"]), (n_tok, Hv))
    a = normal_f32(rng_for(seed, 0, TAGS["step_a"]), (n_tok, Hv))
    return S0, q, k, v, b, a


def with_layers(shape: StageShape, **kw) -> StageShape:
    return replace(shape, **kw)
