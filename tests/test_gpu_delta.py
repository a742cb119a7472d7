"""GPU parity of the isolated gated delta-rule step (batch sweep) against the
fp64 oracle, through the C ABI: B in {1, 8, 64} sequences x 16 heads,
dk = dv = 128, one launch per step.  Sampled (sequence, head) pairs are
replayed by the oracle over every step; the outputs at every step and the
final state must match within relative L2 1e-3."""
import numpy as np
import pytest

import oracle
from attention_decode_megakernel_b200 import synth

from parity import STATE_REL_L2, rel_l2

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


def _run(mk, B, steps, dk=128, heads=16):
    inp = synth.make_delta_sweep(B, steps, heads=heads, dk=dk, dv=dk)
    S = torch.from_numpy(inp["S0"]).cuda()
    q = torch.from_numpy(inp["q"].view(np.int16)).cuda()
    k = torch.from_numpy(inp["k"].view(np.int16)).cuda()
    v = torch.from_numpy(inp["v"].view(np.int16)).cuda()
    al = torch.from_numpy(inp["alpha"]).cuda()
    be = torch.from_numpy(inp["beta"]).cuda()
    o = torch.empty((steps, B, heads, dk), dtype=torch.float32, device="cuda")
    for t in range(steps):
        mk.mk_delta_step(S, q[t], k[t], v[t], al[t], be[t], o[t])
    torch.cuda.synchronize()
    return inp, S.cpu().numpy(), o.cpu().numpy()


def _oracle_pair(inp, b, h):
    f = lambda a: synth.bf16_bits_to_f32(a).astype(np.float64)
    S = inp["S0"][b, h].astype(np.float64).copy()
    o = oracle.delta_sequence(S, f(inp["q"][:, b, h]), f(inp["k"][:, b, h]),
                              f(inp["v"][:, b, h]), inp["alpha"][:, b, h].astype(np.float64),
                              inp["beta"][:, b, h].astype(np.float64))
    return S, o


@pytest.mark.parametrize("B,steps,pairs", [(1, 1024, 16), (8, 1024, 12), (64, 1024, 8)])
def test_delta_sweep_matches_oracle(mk, B, steps, pairs):
    inp, S, o = _run(mk, B, steps)
    rng = np.random.default_rng(B)
    picks = {(0, 0), (B - 1, 15)}
    while len(picks) < pairs:
        picks.add((int(rng.integers(B)), int(rng.integers(16))))
    for b, h in sorted(picks):
        S_ref, o_ref = _oracle_pair(inp, b, h)
        assert rel_l2(S[b, h], S_ref) <= STATE_REL_L2
        assert rel_l2(o[:, b, h], o_ref) <= STATE_REL_L2


def test_delta_step_dk64_and_edge_values(mk):
    # alpha = 1, beta = 0 keeps the state bit for bit; dk = 64 variant
    inp = synth.make_delta_sweep(2, 1, heads=3, dk=64, dv=64)
    S = torch.from_numpy(inp["S0"]).cuda()
    S0 = S.clone()
    q = torch.from_numpy(inp["q"][0].view(np.int16)).cuda()
    k = torch.from_numpy(inp["k"][0].view(np.int16)).cuda()
    v = torch.from_numpy(inp["v"][0].view(np.int16)).cuda()
    al = torch.ones((2, 3), dtype=torch.float32, device="cuda")
    be = torch.zeros((2, 3), dtype=torch.float32, device="cuda")
    o = torch.empty((2, 3, 64), dtype=torch.float32, device="cuda")
    mk.mk_delta_step(S, q, k, v, al, be, o)
    torch.cuda.synchronize()
    assert torch.equal(S, S0)
    qf = torch.from_numpy(synth.bf16_bits_to_f32(inp["q"][0])).cuda()
    ref = torch.einsum("bhij,bhj->bhi", S0.double(), qf.double())
    assert rel_l2(o.cpu().numpy(), ref.cpu().numpy()) < 1e-6
