"""GPU parity of the single-launch decode engine against the fp64 oracle.

Every call goes through the C ABI (libmk.so).  Teacher forcing: both sides
consume the same token stream (the oracle's greedy choices), and each step's
logits, per-layer residual stream and recurrent state are compared under the
tolerances of tests/parity.py.
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


@pytest.fixture(scope="module")
def big():
    cfg = synth.hybrid_08b_config(max_ctx=1024)
    return cfg, synth.make_weights(cfg)


def _np(t):
    return t.detach().cpu().numpy()


def _check_state(eng, orc, tol=STATE_REL_L2):
    dn, conv, _, _ = eng.get_state()
    odn, oconv = orc.get_state()
    e_dn = rel_l2(_np(dn), odn)
    e_conv = rel_l2(_np(conv), oconv)
    assert e_dn <= tol, "DeltaNet state rel-L2 %.3e" % e_dn
    assert e_conv <= tol, "conv state rel-L2 %.3e" % e_conv
    return e_dn, e_conv


def _teacher_forced(eng, orc, cfg, first_token, n_steps, tracker, check_hidden=True):
    """n_steps decode steps; returns the tokens fed."""
    logits = torch.empty(cfg.vocab, dtype=torch.float32, device="cuda")
    tok = int(first_token)
    fed = []
    for _ in range(n_steps):
        eng.decode_step(tok, logits)
        ref, ref_h = orc.step(tok, want_hidden=check_hidden)
        eng.sync()
        tracker.logits(_np(logits), ref)
        if check_hidden:
            tracker.hidden(_np(eng.get_hidden()), ref_h)
        fed.append(tok)
        tok = int(np.argmax(ref))
    return fed


def test_tiny_prompt_then_greedy_teacher_forced(mk):
    cfg = synth.tiny_config(max_ctx=256)
    w = synth.make_weights(cfg)
    eng = mk.Engine(cfg, w)
    orc = oracle.OracleModel(cfg, w)
    tr = Tracker()
    prompt = synth.make_tokens(cfg.vocab, 16)
    logits = torch.empty(cfg.vocab, dtype=torch.float32, device="cuda")
    for t in prompt:
        eng.decode_step(int(t), logits)
        ref, ref_h = orc.step(int(t), want_hidden=True)
        eng.sync()
        tr.logits(_np(logits), ref)
        tr.hidden(_np(eng.get_hidden()), ref_h)
    _check_state(eng, orc)
    _teacher_forced(eng, orc, cfg, int(np.argmax(ref)), 32, tr)
    _check_state(eng, orc)
    assert eng.position == 48 and orc.pos == 48
    print(tr.finish())


def test_mid_prompt_then_greedy_teacher_forced(mk):
    """0.8B layer shapes (4 layers): 100-token prompt (multi-split attention)
    then 16 greedy steps, every position compared."""
    cfg = synth.hybrid_mid_config(max_ctx=256)
    w = synth.make_weights(cfg)
    eng = mk.Engine(cfg, w)
    orc = oracle.OracleModel(cfg, w)
    tr = Tracker()
    prompt = synth.make_tokens(cfg.vocab, 100)
    logits = torch.empty(cfg.vocab, dtype=torch.float32, device="cuda")
    for t in prompt:
        eng.decode_step(int(t), logits)
        ref, ref_h = orc.step(int(t), want_hidden=True)
        eng.sync()
        tr.logits(_np(logits), ref)
        tr.hidden(_np(eng.get_hidden()), ref_h)
    _check_state(eng, orc)
    _teacher_forced(eng, orc, cfg, int(np.argmax(ref)), 16, tr)
    _check_state(eng, orc)
    print(tr.finish())


def test_tiny_prefill_matches_decode_loop(mk):
    cfg = synth.tiny_config(max_ctx=256)
    w = synth.make_weights(cfg)
    prompt = synth.make_tokens(cfg.vocab, 40)
    a = mk.Engine(cfg, w)
    la = torch.empty(cfg.vocab, dtype=torch.float32, device="cuda")
    a.prefill(prompt, la)
    orc = oracle.OracleModel(cfg, w)
    for t in prompt:
        ref, _ = orc.step(int(t))
    a.sync()
    tr = Tracker()
    tr.logits(_np(la), ref)
    _check_state(a, orc)


def test_08b_decode_after_state_load(mk, big):
    cfg, w = big
    st = synth.make_engine_state(cfg, ctx=520)
    eng = mk.Engine(cfg, w)
    dev = {k: (torch.from_numpy(v.view(np.int16) if v.dtype == np.uint16 else v).cuda()
               if isinstance(v, np.ndarray) else v) for k, v in st.items()}
    eng.set_state(dev)
    orc = oracle.OracleModel(cfg, w)
    orc.set_state(st)
    tr = Tracker()
    _teacher_forced(eng, orc, cfg, 1234, 4, tr)
    _check_state(eng, orc)
    print(tr.finish())


@pytest.mark.slow
def test_08b_decode_at_32k_context(mk):
    """Long-context shape: the attention layers' cache holds 32,768
    positions (a seeded synthetic state of that shape) and the attention
    split covers all of them; 2 teacher-forced steps against the oracle."""
    cfg = synth.hybrid_08b_config(max_ctx=32768 + 8)
    w = synth.make_weights(cfg)
    st = synth.make_engine_state(cfg, ctx=32768)
    eng = mk.Engine(cfg, w)
    dev = {k: (torch.from_numpy(v.view(np.int16) if v.dtype == np.uint16 else v).cuda()
               if isinstance(v, np.ndarray) else v) for k, v in st.items()}
    eng.set_state(dev)
    del dev
    orc = oracle.OracleModel(cfg, w)
    orc.set_state(st)
    del st
    tr = Tracker()
    _teacher_forced(eng, orc, cfg, 4321, 2, tr)
    _check_state(eng, orc)
    print(tr.finish())


def test_08b_prompt_then_decode(mk, big):
    cfg, w = big
    eng = mk.Engine(cfg, w)
    orc = oracle.OracleModel(cfg, w)
    prompt = synth.make_tokens(cfg.vocab, 6)
    logits = torch.empty(cfg.vocab, dtype=torch.float32, device="cuda")
    eng.prefill(prompt, logits)
    for t in prompt:
        ref, ref_h = orc.step(int(t), want_hidden=True)
    eng.sync()
    tr = Tracker()
    tr.logits(_np(logits), ref)
    tr.hidden(_np(eng.get_hidden()), ref_h)
    _teacher_forced(eng, orc, cfg, int(np.argmax(ref)), 3, tr)
    _check_state(eng, orc)
    print(tr.finish())


def test_generate_equals_decode_loop_bitwise(mk):
    cfg = synth.tiny_config(max_ctx=256)
    w = synth.make_weights(cfg)
    prompt = synth.make_tokens(cfg.vocab, 8)
    a, b = mk.Engine(cfg, w), mk.Engine(cfg, w)
    a.prefill(prompt)
    b.prefill(prompt)
    n = 20
    toks = torch.zeros(n, dtype=torch.int32, device="cuda")
    a.generate(int(prompt[-1]) ^ 1, n, toks)
    logits = torch.empty(cfg.vocab, dtype=torch.float32, device="cuda")
    tok, ref = int(prompt[-1]) ^ 1, []
    for _ in range(n):
        b.decode_step(tok, logits)
        tok = int(torch.argmax(logits).item())
        ref.append(tok)
    assert _np(toks).tolist() == ref
    assert a.last_argmax() == ref[-1]
    sa, sb = a.get_state()[0], b.get_state()[0]
    assert torch.equal(sa, sb)


@pytest.mark.parametrize("cfg_name,keep", [("tiny", 1), ("tiny", 3), ("tiny", 5), ("mid", 2)])
def test_verify_against_oracle_then_accept(mk, cfg_name, keep):
    """Speculative-verify shape: 5 tokens (1 accepted + 4 drafts) in one
    call.  Every position's logits must match the oracle stepping the same
    tokens; the current state must be untouched until mk_accept; after
    accepting `keep` positions the state equals the oracle's after those
    positions and decoding continues from it."""
    cfg = (synth.tiny_config(max_ctx=256) if cfg_name == "tiny"
           else synth.hybrid_mid_config(max_ctx=256))
    w = synth.make_weights(cfg)
    prompt = synth.make_tokens(cfg.vocab, 40)
    drafts = synth.make_tokens(cfg.vocab, 5, seed=synth.SEED_DRAFTS)
    eng = mk.Engine(cfg, w)
    orc = oracle.OracleModel(cfg, w)
    eng.prefill(prompt)
    for t in prompt:
        orc.step(int(t))
    before = [x.clone() for x in eng.get_state()[:2]]
    vl = torch.empty((5, cfg.vocab), dtype=torch.float32, device="cuda")
    eng.verify(drafts, vl)
    eng.sync()
    assert eng.position == 40
    after = eng.get_state()[:2]
    assert torch.equal(before[0], after[0]) and torch.equal(before[1], after[1])
    tr = Tracker()
    ref_orc = orc.clone()
    for j in range(5):
        ref, _ = ref_orc.step(int(drafts[j]))
        tr.logits(_np(vl[j]), ref)
    eng.accept(keep)
    assert eng.position == 40 + keep
    for j in range(keep):
        ref, _ = orc.step(int(drafts[j]))
    _check_state(eng, orc)
    _teacher_forced(eng, orc, cfg, int(np.argmax(ref)), 3, tr)
    print(tr.finish())


def test_verify_twice_and_cycle_buffers(mk):
    """Repeated verify/accept cycles: each verify first replays the
    positions the previous accept kept, then records its own; the state
    buffers rotate; the result tracks the oracle."""
    cfg = synth.tiny_config(max_ctx=256)
    w = synth.make_weights(cfg)
    eng = mk.Engine(cfg, w)
    orc = oracle.OracleModel(cfg, w)
    prompt = synth.make_tokens(cfg.vocab, 16)
    eng.prefill(prompt)
    for t in prompt:
        orc.step(int(t))
    rng = np.random.default_rng(11)
    tr = Tracker()
    vl = torch.empty((8, cfg.vocab), dtype=torch.float32, device="cuda")
    for it in range(6):
        n = int(rng.integers(1, 9))
        toks = rng.integers(0, cfg.vocab, n)
        eng.verify(toks, vl[:n])
        eng.sync()
        keep = int(rng.integers(1, n + 1))
        ref_orc = orc.clone()
        for j in range(n):
            ref, _ = ref_orc.step(int(toks[j]))
            tr.logits(_np(vl[j]), ref)
        eng.accept(keep)
        for j in range(keep):
            orc.step(int(toks[j]))
    _check_state(eng, orc)
    print(tr.finish())


def test_accepted_positions_replayed_by_every_kind_of_call(mk):
    """After mk_accept the kept positions are applied by whichever call reads
    the state next: a prompt chunk, a verify, a decode step or generate.
    Logits of every call track the oracle fed the same accepted tokens."""
    cfg = synth.tiny_config(max_ctx=256)
    w = synth.make_weights(cfg)
    eng = mk.Engine(cfg, w)
    orc = oracle.OracleModel(cfg, w)
    tr = Tracker()
    rng = np.random.default_rng(23)
    logits = torch.empty(cfg.vocab, dtype=torch.float32, device="cuda")
    vl = torch.empty((8, cfg.vocab), dtype=torch.float32, device="cuda")

    def verify_accept(n, keep):
        toks = rng.integers(0, cfg.vocab, n)
        eng.verify(toks, vl[:n])
        eng.sync()
        ref_orc = orc.clone()
        for j in range(n):
            ref, _ = ref_orc.step(int(toks[j]))
            tr.logits(_np(vl[j]), ref)
        eng.accept(keep)
        for j in range(keep):
            orc.step(int(toks[j]))

    prompt = synth.make_tokens(cfg.vocab, 16)
    eng.prefill(prompt)
    for t in prompt:
        orc.step(int(t))
    verify_accept(5, 2)
    more = rng.integers(0, cfg.vocab, 12)  # a prompt chunk reads the state next
    eng.prefill(more, logits)
    for t in more:
        ref, _ = orc.step(int(t))
    eng.sync()
    tr.logits(_np(logits), ref)
    verify_accept(6, 6)
    verify_accept(3, 1)  # a verify replays the 6 kept above
    tok = int(rng.integers(0, cfg.vocab))
    eng.decode_step(tok, logits)  # a decode step replays the 1 kept above
    ref, _ = orc.step(tok)
    eng.sync()
    tr.logits(_np(logits), ref)
    verify_accept(4, 3)
    n = 4
    toks = torch.zeros(n, dtype=torch.int32, device="cuda")
    lg = torch.empty((n, cfg.vocab), dtype=torch.float32, device="cuda")
    first = int(rng.integers(0, cfg.vocab))
    eng.generate(first, n, toks, lg)  # generate replays the 3 kept above
    eng.sync()
    fed = first
    for i in range(n):
        ref, _ = orc.step(fed)
        tr.logits(_np(lg[i]), ref)
        fed = int(_np(toks)[i])
    assert eng.position == orc.pos
    _check_state(eng, orc)
    print(tr.finish())


def test_engine_errors(mk):
    cfg = synth.tiny_config(max_ctx=4)
    w = synth.make_weights(cfg)
    eng = mk.Engine(cfg, w)
    with pytest.raises(mk.MkError) as e:
        eng.accept(1)
    assert e.value.code == mk.MK_ERR_STATE
    with pytest.raises(mk.MkError) as e:
        eng.decode_step(cfg.vocab)
    assert e.value.code == mk.MK_ERR_ARG
    eng.prefill([1, 2, 3, 4])
    with pytest.raises(mk.MkError) as e:
        eng.decode_step(5)
    assert e.value.code == mk.MK_ERR_CTX_OVERFLOW
    eng.reset()
    vl = torch.empty((9, cfg.vocab), dtype=torch.float32, device="cuda")
    with pytest.raises(mk.MkError) as e:
        eng.verify(list(range(9)), vl)
    assert e.value.code == mk.MK_ERR_ARG


def test_engine_edge_cases(mk):
    """Empty prompt, prompt past the cache, generate with no previous argmax,
    verify while one is pending, accept counts out of range."""
    cfg = synth.tiny_config(max_ctx=16)
    w = synth.make_weights(cfg)
    eng = mk.Engine(cfg, w)
    toks = torch.zeros(4, dtype=torch.int32, device="cuda")
    with pytest.raises(mk.MkError) as e:
        eng.generate(-1, 4, toks)  # no launch yet: no device argmax to feed
    assert e.value.code == mk.MK_ERR_STATE
    eng.prefill([])
    assert eng.position == 0
    with pytest.raises(mk.MkError) as e:
        eng.prefill(list(range(17)))
    assert e.value.code == mk.MK_ERR_CTX_OVERFLOW
    assert eng.position == 0
    vl = torch.empty((3, cfg.vocab), dtype=torch.float32, device="cuda")
    eng.verify([1, 2, 3], vl)
    with pytest.raises(mk.MkError) as e:
        eng.verify([1, 2, 3], vl)
    assert e.value.code == mk.MK_ERR_STATE
    with pytest.raises(mk.MkError) as e:
        eng.decode_step(1)
    assert e.value.code == mk.MK_ERR_STATE
    for bad in (0, 4):
        with pytest.raises(mk.MkError) as e:
            eng.accept(bad)
        assert e.value.code == mk.MK_ERR_ARG
    eng.accept(3)
    assert eng.position == 3
    eng.sync()


@pytest.mark.parametrize("phase", [1, 3, 9, 15, 16, 19, 20])
def test_wait_limit_reports_timeout_and_recovers(mk, phase):
    """A phase whose inputs wait for a tag nobody writes must give up after the
    wait limit, report MK_ERR_TIMEOUT and leave the context usable; mk_reset
    recovers the engine.  Tiny model phases (five per layer): 1 DeltaNet
    state update, 3 first MLP gate/up, 9 second layer's down projection,
    15 attention q|k|v projection, 16 attention, 19 attention layer's down
    projection, 20 LM head."""
    cfg = synth.tiny_config(max_ctx=64)
    w = synth.make_weights(cfg)
    eng = mk.Engine(cfg, w)
    eng.set_wait_limit(50_000_000, phase)  # 50 ms
    eng.decode_step(3)
    with pytest.raises(mk.MkError) as e:
        eng.sync()
    assert e.value.code == mk.MK_ERR_TIMEOUT
    eng.reset()
    eng.set_wait_limit(2_000_000_000, -1)  # default limit, no failing phase
    orc = oracle.OracleModel(cfg, w)
    tr = Tracker()
    _teacher_forced(eng, orc, cfg, 3, 3, tr)
