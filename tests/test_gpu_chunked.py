"""GPU parity of the chunkwise-parallel gated delta rule (the prompt path's
form: chunks of 64 positions prepared independently, then one pass over the
chunks; "Gated Delta Networks", WY / UT representation) against the fp64
oracle's position-by-position recurrence, through the C ABI.

Every head's output at every position and the final state must match the
oracle within relative L2 1e-3 (the DeltaNet state tolerance), at the
0.8B-shaped model's head shape (16 heads, dk = dv = 128) and at lengths that
cover one position, exactly one chunk, a chunk plus one, a ragged tail and
the pp520 prompt (519 positions on the chunk path).
"""
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


def _gpu(mk, inp):
    dev = {k: torch.from_numpy(np.ascontiguousarray(v)).cuda() for k, v in inp.items()}
    S = dev["S0"].clone()
    heads, T, dk = inp["q"].shape
    o = torch.empty((heads, T, dk), dtype=torch.float32, device="cuda")
    mk.mk_delta_chunked(S, dev["q"], dev["k"], dev["v"], dev["alpha"], dev["beta"], o)
    torch.cuda.synchronize()
    return S.cpu().numpy(), o.cpu().numpy()


@pytest.mark.parametrize("T,dk", [(1, 128), (64, 128), (65, 128), (200, 128), (519, 128),
                                  (130, 64)])
def test_chunked_matches_sequential_oracle(mk, T, dk):
    heads = 16 if dk == 128 else 2
    inp = synth.make_delta_sequence(heads, T, dk)
    S, o = _gpu(mk, inp)
    for h in range(heads):
        Sr = inp["S0"][h].astype(np.float64)
        ref = oracle.delta_sequence(Sr, inp["q"][h], inp["k"][h], inp["v"][h],
                                    inp["alpha"][h], inp["beta"][h])
        e_o = rel_l2(o[h], ref)
        e_s = rel_l2(S[h], Sr)
        assert e_o <= STATE_REL_L2, "head %d outputs rel-L2 %.3e" % (h, e_o)
        assert e_s <= STATE_REL_L2, "head %d state rel-L2 %.3e" % (h, e_s)
        # every position, not only on average
        per_pos = np.linalg.norm(o[h] - ref, axis=1) / np.maximum(np.linalg.norm(ref, axis=1), 1e-30)
        assert per_pos.max() <= 1e-2, "head %d worst position rel err %.3e" % (h, per_pos.max())


def test_chunked_strong_decay_and_zero_beta(mk):
    """Edge gates: alpha near 0 in places (state almost reset) and beta = 0
    (no write) at every fourth position."""
    heads, T, dk = 4, 150, 128
    inp = synth.make_delta_sequence(heads, T, dk, alpha_lo=0.0, seed=99)
    inp["alpha"][:, ::7] = 1e-30
    inp["beta"][:, ::4] = 0.0
    S, o = _gpu(mk, inp)
    for h in range(heads):
        Sr = inp["S0"][h].astype(np.float64)
        ref = oracle.delta_sequence(Sr, inp["q"][h], inp["k"][h], inp["v"][h],
                                    inp["alpha"][h], inp["beta"][h])
        assert rel_l2(o[h], ref) <= STATE_REL_L2
        assert rel_l2(S[h], Sr) <= STATE_REL_L2


def test_chunked_rejects_bad_shapes(mk):
    S = torch.zeros((2, 96, 96), dtype=torch.float32, device="cuda")
    q = torch.zeros((2, 10, 96), dtype=torch.float32, device="cuda")
    al = torch.zeros((2, 10), dtype=torch.float32, device="cuda")
    with pytest.raises(mk.MkError):
        mk.mk_delta_chunked(S, q, q, q, al, al, q.clone())
