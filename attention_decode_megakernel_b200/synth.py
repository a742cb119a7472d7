"""Seeded synthetic inputs shared by the CUDA engine and the CPU oracle.

This module only draws numbers: model shapes, bf16 weight blobs, token
streams, isolated delta-step inputs and synthetic engine states.  It holds
none of the model's arithmetic (no norm, projection, recurrence or
attention), so that the oracle and the GPU path can both consume it without
sharing any computation.

Recipe (all draws use numpy's PCG64 generator, so the bytes are identical on
every machine):

* matrices, conv taps and the (tied) embedding: bf16 of N(0, 0.02^2) drawn in
  float32 and rounded to nearest-even;
* RMSNorm and gated-norm gains: exactly 1.0 (not drawn);
* A_log and dt_bias: float32 N(0, 0.02^2);
* tokens: uniform integers in [0, vocab);
* seeds: weights 0, prompt 1, draft tokens 2, isolated delta-step sweep 3.

The two model shapes are the ones the launch post's engine targets
("OS Megakernel that match M5 Max Tok/w at 2x the Throughput on RTX 3090",
the "Why nobody had done this yet?" paragraph: 24 layers, 18 DeltaNet + 6
full attention) plus a tiny 4-layer hybrid of the same family for fast
parity checks.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List

import numpy as np

SEED_WEIGHTS = 0
SEED_PROMPT = 1
SEED_DRAFTS = 2
SEED_SWEEP = 3

MAX_LAYERS = 64


@dataclasses.dataclass(frozen=True)
class ModelConfig:
    name: str
    layer_is_attn: tuple          # one bool per layer, True = full attention
    hidden: int
    vocab: int
    mlp: int
    dn_heads: int
    dn_dk: int
    dn_dv: int
    conv_k: int
    q_heads: int
    kv_heads: int
    head_dim: int
    rope_theta: float
    rms_eps: float = 1e-6
    max_ctx: int = 4096
    max_verify: int = 8

    @property
    def n_layers(self) -> int:
        return len(self.layer_is_attn)

    @property
    def n_dn(self) -> int:
        return sum(1 for a in self.layer_is_attn if not a)

    @property
    def n_attn(self) -> int:
        return sum(1 for a in self.layer_is_attn if a)

    @property
    def conv_channels(self) -> int:
        return 2 * self.dn_heads * self.dn_dk + self.dn_heads * self.dn_dv

    @property
    def in_proj_rows(self) -> int:
        # q, k, v, z, b, a
        return (2 * self.dn_heads * self.dn_dk + 2 * self.dn_heads * self.dn_dv
                + 2 * self.dn_heads)

    def with_ctx(self, max_ctx: int, max_verify: int | None = None) -> "ModelConfig":
        return dataclasses.replace(
            self, max_ctx=max_ctx,
            max_verify=self.max_verify if max_verify is None else max_verify)


def tiny_config(max_ctx: int = 256) -> ModelConfig:
    """4 layers [DN, DN, DN, Attn], hidden 256, vocab 4096."""
    return ModelConfig(
        name="tiny-hybrid-4L-h256", layer_is_attn=(False, False, False, True),
        hidden=256, vocab=4096, mlp=768, dn_heads=2, dn_dk=64, dn_dv=64,
        conv_k=4, q_heads=4, kv_heads=1, head_dim=64, rope_theta=1e4,
        rms_eps=1e-6, max_ctx=max_ctx, max_verify=8)


def hybrid_mid_config(max_ctx: int = 512) -> ModelConfig:
    """The 0.8B layer shapes in 4 layers [DN, DN, DN, Attn] with vocab 4096:
    full-width vectors and multi-chunk phases at a size the oracle runs fast."""
    return ModelConfig(
        name="hybrid-mid-4L-h1024", layer_is_attn=(False, False, False, True),
        hidden=1024, vocab=4096, mlp=3584, dn_heads=16, dn_dk=128, dn_dv=128,
        conv_k=4, q_heads=8, kv_heads=2, head_dim=256, rope_theta=1e7,
        rms_eps=1e-6, max_ctx=max_ctx, max_verify=8)


def hybrid_08b_config(max_ctx: int = 4096) -> ModelConfig:
    """24 layers (3 DN + 1 Attn) x 6, hidden 1024, vocab 151936, tied."""
    pattern = tuple([False, False, False, True] * 6)
    return ModelConfig(
        name="hybrid-0.8B-24L-h1024", layer_is_attn=pattern,
        hidden=1024, vocab=151936, mlp=3584, dn_heads=16, dn_dk=128,
        dn_dv=128, conv_k=4, q_heads=8, kv_heads=2, head_dim=256,
        rope_theta=1e7, rms_eps=1e-6, max_ctx=max_ctx, max_verify=8)


# --------------------------------------------------------------------------
# bf16 helpers (storage format only)
# --------------------------------------------------------------------------

def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (nearest-even); returns uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounding = ((u >> 16) & 1) + np.uint32(0x7FFF)
    return ((u + rounding) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


BF16_ONE = np.uint16(0x3F80)


# --------------------------------------------------------------------------
# weights
# --------------------------------------------------------------------------

def layer_tensor_shapes(cfg: ModelConfig, is_attn: bool) -> List[tuple]:
    """(name, shape, kind) in the canonical draw order of one layer.

    kind: 'w' = bf16 N(0,0.02), 'g' = bf16 gain fixed at 1, 'f' = f32 N(0,0.02).
    """
    H, I = cfg.hidden, cfg.mlp
    t = [("attn_norm", (H,), "g")]
    if is_attn:
        qd, kd = cfg.q_heads * cfg.head_dim, cfg.kv_heads * cfg.head_dim
        t += [("w_q", (qd, H), "w"), ("w_k", (kd, H), "w"),
              ("w_v", (kd, H), "w"), ("w_o", (H, qd), "w")]
    else:
        t += [("in_proj", (cfg.in_proj_rows, H), "w"),
              ("conv_w", (cfg.conv_channels, cfg.conv_k), "w"),
              ("A_log", (cfg.dn_heads,), "f"),
              ("dt_bias", (cfg.dn_heads,), "f"),
              ("out_norm", (cfg.dn_dv,), "g"),
              ("out_proj", (H, cfg.dn_heads * cfg.dn_dv), "w")]
    t += [("mlp_norm", (H,), "g"), ("w_gate", (I, H), "w"),
          ("w_up", (I, H), "w"), ("w_down", (H, I), "w")]
    return t


def _draw(rng: np.random.Generator, shape, kind: str) -> np.ndarray:
    n = int(np.prod(shape))
    if kind == "g":
        return np.full(shape, BF16_ONE, dtype=np.uint16)
    z = rng.standard_normal(n, dtype=np.float32)
    z *= np.float32(0.02)
    if kind == "f":
        return z.reshape(shape)
    return f32_to_bf16_bits(z).reshape(shape)


def make_weights(cfg: ModelConfig, seed: int = SEED_WEIGHTS) -> Dict:
    """Return {'embed', 'final_norm', 'layers': [dict per layer]}.

    bf16 tensors are uint16 arrays of bit patterns; A_log/dt_bias are float32.
    The embedding is tied: the LM head reads the same array.
    """
    rng = np.random.default_rng(seed)
    embed = _draw(rng, (cfg.vocab, cfg.hidden), "w")
    final_norm = _draw(rng, (cfg.hidden,), "g")
    layers = []
    for is_attn in cfg.layer_is_attn:
        d = {}
        for name, shape, kind in layer_tensor_shapes(cfg, is_attn):
            d[name] = _draw(rng, shape, kind)
        layers.append(d)
    return {"embed": embed, "final_norm": final_norm, "layers": layers}


def param_count(cfg: ModelConfig) -> int:
    n = cfg.vocab * cfg.hidden + cfg.hidden
    for is_attn in cfg.layer_is_attn:
        for _, shape, _ in layer_tensor_shapes(cfg, is_attn):
            n += int(np.prod(shape))
    return n


# --------------------------------------------------------------------------
# tokens
# --------------------------------------------------------------------------

def make_tokens(vocab: int, n: int, seed: int = SEED_PROMPT) -> np.ndarray:
    rng = np.random.default_rng(seed)
    return rng.integers(0, vocab, size=n, dtype=np.int64).astype(np.int32)


# --------------------------------------------------------------------------
# isolated gated delta-rule step sweep inputs
# --------------------------------------------------------------------------

def make_delta_sweep(B: int, steps: int, heads: int = 16, dk: int = 128,
                     dv: int = 128, seed: int = SEED_SWEEP) -> Dict:
    """Inputs of the isolated delta-step sweep.

    S0 ~ N(0, 0.1^2) float32 [B][heads][dv][dk]; per step q, k ~ N(0,1)
    scaled to unit length (input preparation, in float64) and then stored as
    bf16; v ~ N(0,1) bf16; beta ~ U(0,1); alpha ~ U(0.9, 1.0).
    """
    rng = np.random.default_rng(seed)
    S0 = (rng.standard_normal((B, heads, dv, dk), dtype=np.float32)
          * np.float32(0.1))

    def unit_rows(shape):
        z = rng.standard_normal(shape, dtype=np.float32).astype(np.float64)
        z /= np.sqrt((z * z).sum(axis=-1, keepdims=True))
        return f32_to_bf16_bits(z.astype(np.float32))

    q = unit_rows((steps, B, heads, dk))
    k = unit_rows((steps, B, heads, dk))
    v = f32_to_bf16_bits(rng.standard_normal((steps, B, heads, dv),
                                             dtype=np.float32))
    beta = rng.uniform(0.0, 1.0, size=(steps, B, heads)).astype(np.float32)
    alpha = rng.uniform(0.9, 1.0, size=(steps, B, heads)).astype(np.float32)
    return {"S0": S0, "q": q, "k": k, "v": v, "beta": beta, "alpha": alpha}


def make_delta_sequence(heads: int, T: int, dk: int = 128, alpha_lo: float = 0.3,
                        seed: int = SEED_SWEEP + 10) -> Dict:
    """Inputs of a whole-sequence gated delta rule (the prompt path's shape:
    one sequence, `heads` heads, T positions), all float32.

    S0 ~ N(0, 0.1^2) [heads][dk][dk]; q, k ~ N(0,1) scaled to unit length
    (input preparation, float64) [heads][T][dk]; v ~ N(0,1) [heads][T][dk];
    beta ~ U(0,1), alpha ~ U(alpha_lo, 1) [heads][T] (the 0.8B-shaped
    model's random weights give alpha near 0.5).
    """
    rng = np.random.default_rng(seed)
    S0 = rng.standard_normal((heads, dk, dk), dtype=np.float32) * np.float32(0.1)

    def unit_rows(shape):
        z = rng.standard_normal(shape, dtype=np.float32).astype(np.float64)
        z /= np.sqrt((z * z).sum(axis=-1, keepdims=True))
        return z.astype(np.float32)

    q = unit_rows((heads, T, dk))
    k = unit_rows((heads, T, dk))
    v = rng.standard_normal((heads, T, dk), dtype=np.float32)
    beta = rng.uniform(0.0, 1.0, size=(heads, T)).astype(np.float32)
    alpha = rng.uniform(alpha_lo, 1.0, size=(heads, T)).astype(np.float32)
    return {"S0": S0, "q": q, "k": k, "v": v, "beta": beta, "alpha": alpha}


# --------------------------------------------------------------------------
# synthetic engine state (long-context and verify parity without a long
# prompt through the oracle)
# --------------------------------------------------------------------------

def make_engine_state(cfg: ModelConfig, ctx: int, seed: int = 4) -> Dict:
    """A seeded state as if `ctx` tokens had been consumed.

    dn_state [n_dn][heads][dv][dk] f32 ~ N(0, 0.02^2);
    conv_state [n_dn][channels][conv_k-1] f32 ~ N(0, 0.5^2);
    k_cache / v_cache [n_attn][kv_heads][ctx][head_dim] bf16 ~ N(0, 0.5^2).
    """
    rng = np.random.default_rng(seed)
    dn = (rng.standard_normal((cfg.n_dn, cfg.dn_heads, cfg.dn_dv, cfg.dn_dk),
                              dtype=np.float32) * np.float32(0.02))
    conv = (rng.standard_normal((cfg.n_dn, cfg.conv_channels, cfg.conv_k - 1),
                                dtype=np.float32) * np.float32(0.5))
    shape = (cfg.n_attn, cfg.kv_heads, ctx, cfg.head_dim)
    kc = f32_to_bf16_bits(rng.standard_normal(shape, dtype=np.float32)
                          * np.float32(0.5))
    vc = f32_to_bf16_bits(rng.standard_normal(shape, dtype=np.float32)
                          * np.float32(0.5))
    return {"pos": ctx, "dn_state": dn, "conv_state": conv,
            "k_cache": kc, "v_cache": vc}
