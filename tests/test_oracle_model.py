"""Pins of the oracle's layer stack (CPU only).

Special cases whose outputs reduce to closed forms: zeroed exits make every
layer an identity on the residual stream; identity projections turn the MLP
and the attention layer into short formulas; a one-head DeltaNet with a
one-tap convolution has a two-step closed form.  Each case is built from
hand-chosen weights of a micro model.
"""
import dataclasses
import math

import numpy as np
import pytest

import oracle
from attention_decode_megakernel_b200 import synth

bf = synth.f32_to_bf16_bits


def f64(bits):
    return synth.bf16_bits_to_f32(bits).astype(np.float64)


def _micro_cfg(attn: bool, nkv=1, **kw):
    base = dict(name="micro", layer_is_attn=(attn,), hidden=4, vocab=8, mlp=4,
                dn_heads=1, dn_dk=2, dn_dv=2, conv_k=4, q_heads=2, kv_heads=nkv,
                head_dim=2, rope_theta=100.0, rms_eps=1e-6, max_ctx=16,
                max_verify=4)
    base.update(kw)
    return synth.ModelConfig(**base)


def _zeros_like_layer(cfg, is_attn):
    d = {}
    for name, shape, kind in synth.layer_tensor_shapes(cfg, is_attn):
        if kind == "g":
            d[name] = np.full(shape, synth.BF16_ONE, np.uint16)
        elif kind == "f":
            d[name] = np.zeros(shape, np.float32)
        else:
            d[name] = np.zeros(shape, np.uint16)
    return d


def _embed(cfg, rows):
    E = np.zeros((cfg.vocab, cfg.hidden), np.float32)
    for i, r in enumerate(rows):
        E[i] = r
    return bf(E)


# ------------------------------------------------------------------------

def test_zero_exits_make_every_layer_identity(tiny):
    cfg, w = tiny
    w = {"embed": w["embed"], "final_norm": w["final_norm"],
         "layers": [dict(d) for d in w["layers"]]}
    for d in w["layers"]:
        for name in ("out_proj", "w_o", "w_down"):
            if name in d:
                d[name] = np.zeros_like(d[name])
    m = oracle.OracleModel(cfg, w)
    E = f64(w["embed"])
    for tok in (5, 4095, 17):
        logits, hidden = m.step(tok, want_hidden=True)
        for l in range(cfg.n_layers):
            np.testing.assert_array_equal(hidden[l], E[tok])
        xn = oracle.rmsnorm(E[tok], w["final_norm"], eps=cfg.rms_eps)
        np.testing.assert_allclose(logits, E @ xn, rtol=1e-12, atol=1e-12)


def test_mlp_with_identity_projections():
    cfg = _micro_cfg(attn=False)
    layer = _zeros_like_layer(cfg, False)
    I4 = np.eye(4, dtype=np.float32)
    layer["w_gate"], layer["w_up"], layer["w_down"] = bf(I4), bf(2 * I4), bf(I4)
    x0 = np.array([0.5, -1.25, 2.0, 0.75], np.float32)
    w = {"embed": _embed(cfg, [x0]), "final_norm": np.full(4, synth.BF16_ONE, np.uint16),
         "layers": [layer]}
    m = oracle.OracleModel(cfg, w)
    _, hidden = m.step(0, want_logits=False, want_hidden=True)
    xn = oracle.rmsnorm(x0.astype(np.float64), eps=cfg.rms_eps)
    expect = x0 + np.array([oracle.silu(a) * 2 * a for a in xn])
    np.testing.assert_allclose(hidden[0], expect, rtol=1e-14)


@pytest.mark.parametrize("nkv", [1, 2, 4])
def test_attention_layer_two_positions_closed_form(nkv):
    """q_heads=4, head_dim=2, hidden 8, W_o = I.  At position 0 query head h
    returns the value of KV head h // (4 // nkv) (contiguous groups); at
    position 1 it mixes the two cached values with weight sigmoid(s1 - s0),
    s_j = RoPE(q,1).RoPE(k_j,j)/sqrt(2), the cache holding bf16-rounded keys
    and values."""
    nq, hd, H = 4, 2, 8
    cfg = _micro_cfg(attn=True, nkv=nkv, hidden=H, mlp=H, q_heads=nq)
    layer = _zeros_like_layer(cfg, True)
    rng = np.random.default_rng(0)
    Wq = rng.standard_normal((nq * hd, H)).astype(np.float32)
    Wk = rng.standard_normal((nkv * hd, H)).astype(np.float32)
    Wv = rng.standard_normal((nkv * hd, H)).astype(np.float32)
    layer["w_q"], layer["w_k"], layer["w_v"] = bf(Wq), bf(Wk), bf(Wv)
    layer["w_o"] = bf(np.eye(H, dtype=np.float32))
    x0 = np.array([1.0, -0.5, 0.25, 2.0, -1.0, 0.5, 0.75, -0.25], np.float32)
    x1 = np.array([-1.5, 0.5, 1.0, 0.125, 0.25, -2.0, 1.5, 0.5], np.float32)
    w = {"embed": _embed(cfg, [x0, x1]), "final_norm": np.full(H, synth.BF16_ONE, np.uint16),
         "layers": [layer]}
    m = oracle.OracleModel(cfg, w)
    Wq, Wk, Wv = f64(layer["w_q"]), f64(layer["w_k"]), f64(layer["w_v"])
    r = lambda v: np.array([oracle.bf16_value(oracle.bf16_round(a)) for a in v])
    group = lambda h: h // (nq // nkv)
    sl = lambda i: slice(hd * i, hd * i + hd)

    _, h0 = m.step(0, want_logits=False, want_hidden=True)
    xn0 = oracle.rmsnorm(x0.astype(np.float64), eps=cfg.rms_eps)
    v0 = r(Wv @ xn0)
    o0 = np.concatenate([v0[sl(group(h))] for h in range(nq)])
    np.testing.assert_allclose(h0[0], x0 + o0, rtol=1e-14, atol=1e-15)

    _, h1 = m.step(1, want_logits=False, want_hidden=True)
    xn1 = oracle.rmsnorm(x1.astype(np.float64), eps=cfg.rms_eps)
    q1, v1 = Wq @ xn1, r(Wv @ xn1)
    k0, k1 = Wk @ xn0, Wk @ xn1
    o1 = []
    for h in range(nq):
        g = group(h)
        qh = oracle.rope(q1[sl(h)], 1, cfg.rope_theta)
        kk0 = r(oracle.rope(k0[sl(g)], 0, cfg.rope_theta))
        kk1 = r(oracle.rope(k1[sl(g)], 1, cfg.rope_theta))
        s0, s1 = qh @ kk0 / math.sqrt(hd), qh @ kk1 / math.sqrt(hd)
        w1 = 1.0 / (1.0 + math.exp(-(s1 - s0)))
        o1.append(w1 * v1[sl(g)] + (1 - w1) * v0[sl(g)])
    np.testing.assert_allclose(h1[0], x1 + np.concatenate(o1), rtol=1e-13, atol=1e-14)


def test_deltanet_layer_two_steps_closed_form():
    """One head, dk=dv=2, conv taps (0,0,0,1) so the conv is SiLU of the
    current projection, out_norm = 1, out_proj = [I; 0].  With S_0 = 0:
      t=0: o_1 = b1 (k1.q1) v1
      t=1: o_2 = a2 b1 (k1.q2 - b2 (k1.k2)(k2.q2)) v1 + b2 (k2.q2) v2
    where q is L2-normalised (eps 1e-6 inside the root) and scaled by
    2^-1/2, k L2-normalised likewise,
    b = sigmoid(b-row), a = exp(-exp(A_log) softplus(a-row + dt_bias)).
    The layer output is out_proj (RMSNorm(o) * SiLU(z))."""
    cfg = _micro_cfg(attn=False)
    layer = _zeros_like_layer(cfg, False)
    rng = np.random.default_rng(1)
    P = rng.standard_normal((cfg.in_proj_rows, 4)).astype(np.float32)
    layer["in_proj"] = bf(P)
    conv = np.zeros((cfg.conv_channels, 4), np.float32)
    conv[:, 3] = 1.0
    layer["conv_w"] = bf(conv)
    layer["A_log"] = np.array([0.3], np.float32)
    layer["dt_bias"] = np.array([-0.2], np.float32)
    out = np.zeros((4, 2), np.float32)
    out[0, 0] = out[1, 1] = 1.0
    layer["out_proj"] = bf(out)
    x0 = np.array([1.0, -0.5, 0.25, 2.0], np.float32)
    x1 = np.array([-1.5, 0.5, 1.0, 0.125], np.float32)
    w = {"embed": _embed(cfg, [x0, x1]), "final_norm": np.full(4, synth.BF16_ONE, np.uint16),
         "layers": [layer]}
    m = oracle.OracleModel(cfg, w)
    P = f64(layer["in_proj"])

    def parts(x):
        u = P @ oracle.rmsnorm(x.astype(np.float64), eps=cfg.rms_eps)
        s = np.array([oracle.silu(a) for a in u[:6]])
        q = s[0:2] / math.sqrt(s[0:2] @ s[0:2] + 1e-6) / math.sqrt(2)
        k = s[2:4] / math.sqrt(s[2:4] @ s[2:4] + 1e-6)
        v = s[4:6]
        z = u[6:8]
        beta = oracle.sigmoid(u[8])
        alpha = math.exp(-math.exp(float(np.float32(0.3)))
                         * oracle.softplus(u[9] + float(np.float32(-0.2))))
        return q, k, v, z, beta, alpha

    def layer_out(o, z):
        g = oracle.rmsnorm(o, eps=cfg.rms_eps) * np.array([oracle.silu(a) for a in z])
        return np.array([g[0], g[1], 0.0, 0.0])

    q1, k1, v1, z1, b1, _ = parts(x0)
    q2, k2, v2, z2, b2, a2 = parts(x1)
    _, h = m.step(0, want_logits=False, want_hidden=True)
    o1 = b1 * (k1 @ q1) * v1
    np.testing.assert_allclose(h[0], x0 + layer_out(o1, z1), rtol=1e-12, atol=1e-14)
    _, h = m.step(1, want_logits=False, want_hidden=True)
    o2 = a2 * b1 * (k1 @ q2 - b2 * (k1 @ k2) * (k2 @ q2)) * v1 + b2 * (k2 @ q2) * v2
    np.testing.assert_allclose(h[0], x1 + layer_out(o2, z2), rtol=1e-12, atol=1e-14)
    dn, conv_state = m.get_state()
    np.testing.assert_allclose(dn[0, 0], a2 * (b1 * np.outer(v1, k1)) @ (
        np.eye(2) - b2 * np.outer(k2, k2)) + b2 * np.outer(v2, k2), rtol=1e-12, atol=1e-14)


def test_clone_and_state_roundtrip_are_exact(tiny):
    cfg, w = tiny
    toks = synth.make_tokens(cfg.vocab, 12, seed=synth.SEED_PROMPT)
    a = oracle.OracleModel(cfg, w)
    for t in toks[:6]:
        a.step(t, want_logits=False)
    b = a.clone()
    for t in toks[6:]:
        la, _ = a.step(t)
        lb, _ = b.step(t)
        np.testing.assert_array_equal(la, lb)
    st = synth.make_engine_state(cfg, ctx=40)
    a.set_state(st)
    assert a.pos == 40
    dn, conv = a.get_state()
    np.testing.assert_array_equal(dn, st["dn_state"].astype(np.float64))
    np.testing.assert_array_equal(conv, st["conv_state"].astype(np.float64))


def test_context_overflow_and_bad_token_rejected():
    cfg = synth.tiny_config(max_ctx=3)
    w = synth.make_weights(cfg)
    m = oracle.OracleModel(cfg, w)
    with pytest.raises(ValueError):
        m.step(cfg.vocab)
    for t in range(3):
        m.step(t, want_logits=False)
    with pytest.raises(ValueError):
        m.step(0)


def test_tiny_model_logits_are_finite_and_deterministic(tiny):
    cfg, w = tiny
    toks = synth.make_tokens(cfg.vocab, 8)
    outs = []
    for _ in range(2):
        m = oracle.OracleModel(cfg, w)
        outs.append(np.stack([m.step(t)[0] for t in toks]))
    np.testing.assert_array_equal(outs[0], outs[1])
    assert np.isfinite(outs[0]).all() and outs[0].std() > 0
