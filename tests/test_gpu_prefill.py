"""GPU parity of the prompt (multi-token) path against the fp64 oracle.

Prompt processing is measured beside decode in the launch post ("OS
Megakernel that match M5 Max Tok/w at 2x the Throughput on RTX 3090",
results table, pp520).  The engine runs all but the last prompt position as
chunks (tensor-core GEMMs for the projections, a position-by-position scan
for the conv and the gated delta rule, causal attention over cache + chunk)
and the last position through the decode kernel.  The oracle consumes the
same prompt one token at a time; the last position's logits and per-layer
residual stream, and the recurrent state after the prompt, must agree under
the tolerances of tests/parity.py, and decoding must continue correctly from
the state the prompt path left.
"""
import numpy as np
import pytest

import oracle
from attention_decode_megakernel_b200 import synth

from parity import STATE_REL_L2, Tracker, rel_l2

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mk():
    import attention_decode_megakernel_b200 as m
    from attention_decode_megakernel_b200 import build
    build.build()
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return m


def _np(t):
    return t.detach().cpu().numpy()


def _split(x):
    """fp32 activations -> (hi, lo) bf16 bit patterns, the GEMM's operands."""
    hi = synth.f32_to_bf16_bits(x)
    lo = synth.f32_to_bf16_bits(x - synth.bf16_bits_to_f32(hi))
    return hi, lo


@pytest.mark.parametrize("n_out,T,K", [(200, 70, 192), (1024, 300, 1024), (520, 129, 3584)])
def test_tensor_core_gemm_against_oracle(mk, n_out, T, K):
    """C = X W^T with ragged row and token tails, against the oracle's GEMV
    of every token row (x = hi + lo exactly, in fp64)."""
    rng = np.random.default_rng(7)
    W = synth.f32_to_bf16_bits(rng.normal(0, 0.05, (n_out, K)).astype(np.float32))
    X = rng.normal(0, 1.0, (T, K)).astype(np.float32)
    hi, lo = _split(X)
    Xd = torch.from_numpy(np.concatenate([hi, lo]).view(np.int16)).cuda()
    Wd = torch.from_numpy(W.view(np.int16)).cuda()
    C = torch.full((T, n_out), float("nan"), dtype=torch.float32, device="cuda")
    mk.mk_debug_gemm(Wd, Xd, C)
    torch.cuda.synchronize()
    got = _np(C)
    x64 = synth.bf16_bits_to_f32(hi).astype(np.float64) + synth.bf16_bits_to_f32(lo)
    ref = np.stack([oracle.gemv(W, x64[t]) for t in range(T)])
    assert np.isfinite(got).all()
    # fp32 accumulation of exact bf16 products, plus the ~2^-17 relative
    # residual of the hi+lo split
    err = rel_l2(got, ref)
    assert err <= 2e-5, "GEMM rel-L2 %.3e" % err


def _prompt_vs_oracle(eng, orc, cfg, prompt, tr, state_tol=STATE_REL_L2):
    logits = torch.empty(cfg.vocab, dtype=torch.float32, device="cuda")
    eng.prefill(prompt, logits)
    ref = ref_h = None
    for t in prompt:
        ref, ref_h = orc.step(int(t), want_hidden=True)
    eng.sync()
    tr.logits(_np(logits), ref)
    tr.hidden(_np(eng.get_hidden()), ref_h)
    dn, conv, _, _ = eng.get_state()
    odn, oconv = orc.get_state()
    e_dn, e_conv = rel_l2(_np(dn), odn), rel_l2(_np(conv), oconv)
    assert e_dn <= state_tol, "DeltaNet state rel-L2 %.3e" % e_dn
    assert e_conv <= state_tol, "conv state rel-L2 %.3e" % e_conv
    assert eng.position == orc.pos
    return int(np.argmax(ref))


def _decode_on(eng, orc, cfg, tok, n, tr):
    logits = torch.empty(cfg.vocab, dtype=torch.float32, device="cuda")
    for _ in range(n):
        eng.decode_step(tok, logits)
        ref, ref_h = orc.step(tok, want_hidden=True)
        eng.sync()
        tr.logits(_np(logits), ref)
        tr.hidden(_np(eng.get_hidden()), ref_h)
        tok = int(np.argmax(ref))


def test_tiny_prompt_chunks_tiles_and_tails(mk):
    """Prompts of 300 then 170 positions (ragged 128-token tiles; the second
    starts mid-context, so conv history, DeltaNet state and the cache carry
    across calls), then greedy decode from the result."""
    cfg = synth.tiny_config(max_ctx=640)
    w = synth.make_weights(cfg)
    eng = mk.Engine(cfg, w)
    orc = oracle.OracleModel(cfg, w)
    tr = Tracker()
    toks = synth.make_tokens(cfg.vocab, 470)
    _prompt_vs_oracle(eng, orc, cfg, toks[:300], tr)
    nxt = _prompt_vs_oracle(eng, orc, cfg, toks[300:], tr)
    _decode_on(eng, orc, cfg, nxt, 8, tr)
    print(tr.finish())


def test_tiny_prompt_longer_than_one_chunk(mk):
    """1100 positions: more than one 1024-position chunk in a single call."""
    cfg = synth.tiny_config(max_ctx=1200)
    w = synth.make_weights(cfg)
    eng = mk.Engine(cfg, w)
    orc = oracle.OracleModel(cfg, w)
    tr = Tracker()
    nxt = _prompt_vs_oracle(eng, orc, cfg, synth.make_tokens(cfg.vocab, 1100), tr)
    _decode_on(eng, orc, cfg, nxt, 4, tr)
    print(tr.finish())


@pytest.mark.parametrize("n", [1, 2, 8, 9, 10])
def test_short_prompts_at_the_batch_threshold(mk, n):
    """Prompts at and around the length where the chunk path takes over."""
    cfg = synth.tiny_config(max_ctx=256)
    w = synth.make_weights(cfg)
    eng = mk.Engine(cfg, w)
    orc = oracle.OracleModel(cfg, w)
    tr = Tracker()
    nxt = _prompt_vs_oracle(eng, orc, cfg, synth.make_tokens(cfg.vocab, n), tr)
    _decode_on(eng, orc, cfg, nxt, 2, tr)
    print(tr.finish())


def test_mid_shapes_prompt(mk):
    """0.8B layer shapes (dk = dv = 128, head_dim 256, GQA 8:2), 4 layers,
    a 260-position prompt then 4 greedy steps."""
    cfg = synth.hybrid_mid_config(max_ctx=512)
    w = synth.make_weights(cfg)
    eng = mk.Engine(cfg, w)
    orc = oracle.OracleModel(cfg, w)
    tr = Tracker()
    nxt = _prompt_vs_oracle(eng, orc, cfg, synth.make_tokens(cfg.vocab, 260), tr)
    _decode_on(eng, orc, cfg, nxt, 4, tr)
    print(tr.finish())


@pytest.mark.slow
def test_08b_pp520(mk):
    """The full 24-layer model on the benchmark's 520-position prompt, then
    2 greedy steps."""
    cfg = synth.hybrid_08b_config(max_ctx=1024)
    w = synth.make_weights(cfg)
    eng = mk.Engine(cfg, w)
    orc = oracle.OracleModel(cfg, w)
    tr = Tracker()
    nxt = _prompt_vs_oracle(eng, orc, cfg, synth.make_tokens(cfg.vocab, 520), tr)
    _decode_on(eng, orc, cfg, nxt, 2, tr)
    print(tr.finish())
