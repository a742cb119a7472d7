"""Pin of the oracle's layer wiring: a multi-layer hybrid stack brute-forced
in float64 NumPy (CPU only).

The launch post "OS Megakernel that match M5 Max Tok/w at 2x the
Throughput on RTX 3090" ("Why nobody had done this yet?") describes a stack
that alternates DeltaNet layers, each with its own recurrent state, and
full-attention layers, each with its own KV cache.  The single-layer pins of
test_oracle_model.py cannot see a mistake in how the oracle assigns state
and cache slots to layers (two DeltaNet layers sharing one state, two
attention layers sharing one cache, a layer reading its neighbour's conv
history).  Here a micro model with two layers of each kind, two DeltaNet
heads and large random weights on every path runs six positions through
the oracle and through an independent NumPy restatement written from the
definitions (Gated Delta Networks' gated delta rule with a short causal
conv; rotate-half RoPE; causal softmax attention with grouped KV heads;
SwiGLU; RMSNorm), keeping one state per layer in a dict keyed by the layer
index.  Logits, every layer's residual stream and every layer's recurrent
and conv state must agree to float64 rounding.  The same restatement with
the states of the two DeltaNet layers (or the caches of the two attention
layers) shared must disagree, which shows the comparison can see such a
mistake.
"""
import numpy as np
import pytest

import oracle
from attention_decode_megakernel_b200 import synth


def _cfg():
    return synth.ModelConfig(
        name="stack-micro", layer_is_attn=(False, True, False, True), hidden=8, vocab=11,
        mlp=6, dn_heads=2, dn_dk=2, dn_dv=2, conv_k=4, q_heads=2, kv_heads=1, head_dim=4,
        rope_theta=50.0, rms_eps=1e-6, max_ctx=16, max_verify=4)


def _weights(cfg, seed=123):
    """Random weights with scale 0.5 (so every layer changes the stream)."""
    rng = np.random.default_rng(seed)
    bf = synth.f32_to_bf16_bits

    def draw(shape, kind):
        z = rng.standard_normal(shape).astype(np.float32) * np.float32(0.5)
        if kind == "f":
            return z
        if kind == "g":
            return bf(np.float32(1.0) + z * np.float32(0.2))
        return bf(z)

    layers = []
    for is_attn in cfg.layer_is_attn:
        layers.append({name: draw(shape, kind)
                       for name, shape, kind in synth.layer_tensor_shapes(cfg, is_attn)})
    return {"embed": draw((cfg.vocab, cfg.hidden), "w"),
            "final_norm": draw((cfg.hidden,), "g"), "layers": layers}


def _f(bits):
    return synth.bf16_bits_to_f32(np.asarray(bits)).astype(np.float64)


def _bf16_round(x):
    """Nearest bf16 value (8 significant bits, ties to even) of float64 x."""
    m, e = np.frexp(np.asarray(x, np.float64))
    return np.ldexp(np.round(m * 256.0) / 256.0, e)


def _rms(x, g, eps):
    return x / np.sqrt(np.mean(x * x) + eps) * g


def _silu(x):
    return x / (1.0 + np.exp(-x))


def _rope(x, pos, theta):
    hd = x.size
    half = hd // 2
    i = np.arange(half, dtype=np.float64)
    ang = pos * theta ** (-2.0 * i / hd)
    c, s = np.cos(ang), np.sin(ang)
    a, b = x[:half], x[half:]
    return np.concatenate([a * c - b * s, b * c + a * s])


def numpy_stack(cfg, w, tokens, share_dn_state=False, share_kv=False):
    """Forward pass over `tokens`; returns per-position logits, per-position
    per-layer residual streams, and the final per-layer states."""
    H, nh, dk, dv = cfg.hidden, cfg.dn_heads, cfg.dn_dk, cfg.dn_dv
    nq, nkv, hd = cfg.q_heads, cfg.kv_heads, cfg.head_dim
    E = _f(w["embed"])
    S, hist, K, V = {}, {}, {}, {}
    for l, is_attn in enumerate(cfg.layer_is_attn):
        key_dn = 0 if share_dn_state else l
        key_kv = 0 if share_kv else l
        if not is_attn:
            S.setdefault(key_dn, np.zeros((nh, dv, dk)))
            hist.setdefault(key_dn, np.zeros((2 * nh * dk + nh * dv, cfg.conv_k - 1)))
        else:
            K.setdefault(key_kv, [])
            V.setdefault(key_kv, [])
    all_logits, all_hidden = [], []
    for pos, tok in enumerate(tokens):
        x = E[tok].copy()
        hidden = []
        for l, is_attn in enumerate(cfg.layer_is_attn):
            d = w["layers"][l]
            xn = _rms(x, _f(d["attn_norm"]), cfg.rms_eps)
            if not is_attn:
                key = 0 if share_dn_state else l
                p = _f(d["in_proj"]) @ xn
                nconv = 2 * nh * dk + nh * dv
                u, z = p[:nconv], p[nconv:nconv + nh * dv]
                b, a = p[nconv + nh * dv:nconv + nh * dv + nh], p[nconv + nh * dv + nh:]
                # causal conv over (u_{t-3}, u_{t-2}, u_{t-1}, u_t), then SiLU
                win = np.concatenate([hist[key], u[:, None]], axis=1)
                c = _silu(np.sum(_f(d["conv_w"]) * win, axis=1))
                hist[key] = win[:, 1:]
                q = c[:nh * dk].reshape(nh, dk)
                k = c[nh * dk:2 * nh * dk].reshape(nh, dk)
                v = c[2 * nh * dk:].reshape(nh, dv)
                o = np.zeros((nh, dv))
                for h in range(nh):
                    qh = q[h] / np.sqrt(np.sum(q[h] ** 2) + 1e-6) / np.sqrt(dk)
                    kh = k[h] / np.sqrt(np.sum(k[h] ** 2) + 1e-6)
                    beta = 1.0 / (1.0 + np.exp(-b[h]))
                    sp = np.log1p(np.exp(a[h] + d["dt_bias"][h]))
                    alpha = np.exp(-np.exp(np.float64(d["A_log"][h])) * sp)
                    # S_t = alpha S_{t-1} (I - beta k k^T) + beta v k^T ;  o_t = S_t q
                    Sh = S[key][h]
                    Sh = alpha * Sh @ (np.eye(dk) - beta * np.outer(kh, kh)) + beta * np.outer(v[h], kh)
                    S[key][h] = Sh
                    oh = Sh @ qh
                    o[h] = (oh / np.sqrt(np.mean(oh * oh) + cfg.rms_eps) * _f(d["out_norm"])
                            * _silu(z.reshape(nh, dv)[h]))
                x = x + _f(d["out_proj"]) @ o.reshape(-1)
            else:
                key = 0 if share_kv else l
                q = (_f(d["w_q"]) @ xn).reshape(nq, hd)
                k = (_f(d["w_k"]) @ xn).reshape(nkv, hd)
                v = (_f(d["w_v"]) @ xn).reshape(nkv, hd)
                K[key].append(_bf16_round(np.stack([_rope(k[g], pos, cfg.rope_theta)
                                                    for g in range(nkv)])))
                V[key].append(_bf16_round(v))
                Kc, Vc = np.stack(K[key]), np.stack(V[key])  # [t][nkv][hd]
                out = np.zeros((nq, hd))
                for h in range(nq):
                    g = h // (nq // nkv)
                    qr = _rope(q[h], pos, cfg.rope_theta)
                    s = Kc[:, g, :] @ qr / np.sqrt(hd)
                    pr = np.exp(s - s.max())
                    pr /= pr.sum()
                    out[h] = pr @ Vc[:, g, :]
                x = x + _f(d["w_o"]) @ out.reshape(-1)
            xn = _rms(x, _f(d["mlp_norm"]), cfg.rms_eps)
            hmid = _silu(_f(d["w_gate"]) @ xn) * (_f(d["w_up"]) @ xn)
            x = x + _f(d["w_down"]) @ hmid
            hidden.append(x.copy())
        all_hidden.append(np.stack(hidden))
        all_logits.append(E @ _rms(x, _f(w["final_norm"]), cfg.rms_eps))
    dn_layers = [l for l, a in enumerate(cfg.layer_is_attn) if not a]
    dn = np.stack([S[0 if share_dn_state else l] for l in dn_layers])
    conv = np.stack([hist[0 if share_dn_state else l] for l in dn_layers])
    return np.stack(all_logits), np.stack(all_hidden), dn, conv


@pytest.fixture(scope="module")
def stack():
    cfg = _cfg()
    w = _weights(cfg)
    tokens = [3, 7, 0, 10, 7, 5]
    m = oracle.OracleModel(cfg, w)
    logits, hidden = [], []
    for t in tokens:
        lg, hd = m.step(t, want_hidden=True)
        logits.append(lg)
        hidden.append(hd)
    dn, conv = m.get_state()
    return cfg, w, tokens, (np.stack(logits), np.stack(hidden), dn, conv)


def _rel(a, b):
    return float(np.abs(a - b).max() / max(np.abs(b).max(), 1e-300))


def test_stack_matches_numpy_restatement(stack):
    cfg, w, tokens, (lg, hd, dn, conv) = stack
    rl, rh, rdn, rconv = numpy_stack(cfg, w, tokens)
    assert _rel(lg, rl) < 1e-12
    assert _rel(hd, rh) < 1e-12
    assert _rel(dn, rdn) < 1e-12
    assert _rel(conv, rconv) < 1e-12
    # every layer changes the residual stream by a visible amount
    for l in range(1, cfg.n_layers):
        assert np.abs(hd[:, l] - hd[:, l - 1]).max() > 1e-2


@pytest.mark.parametrize("mutation", ["share_dn_state", "share_kv"])
def test_shared_slot_is_detected(stack, mutation):
    cfg, w, tokens, (lg, hd, dn, conv) = stack
    rl, rh, rdn, rconv = numpy_stack(cfg, w, tokens, **{mutation: True})
    assert _rel(lg, rl) > 1e-3
    assert _rel(hd, rh) > 1e-3
