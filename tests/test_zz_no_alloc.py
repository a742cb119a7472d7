"""The allocation-free GEMM entry point (mk_debug_gemm_noalloc) against the
allocating one (mk_debug_gemm) on the same inputs, and against the fp64
oracle's matrix-vector product, through the C ABI.

The no-alloc entry point splits K over the SMs and sums the ranges from a
static device scratch array in a fixed order, so it agrees with the
single-range GEMM within fp32 rounding and is bitwise repeatable.  Collected
last (file name), it must pass alone and after every other test.
"""
import numpy as np
import pytest

from attention_decode_megakernel_b200 import synth

from parity import rel_l2

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


def _host_operands(n_out, T, K, seed):
    rng = np.random.default_rng(seed)
    W = synth.f32_to_bf16_bits(rng.normal(0, 0.05, (n_out, K)).astype(np.float32))
    X = rng.normal(0, 1.0, (T, K)).astype(np.float32)
    hi = synth.f32_to_bf16_bits(X)
    lo = synth.f32_to_bf16_bits(X - synth.bf16_bits_to_f32(hi))
    return W, hi, lo


def _operands(n_out, T, K, seed):
    W, hi, lo = _host_operands(n_out, T, K, seed)
    Wd = torch.from_numpy(W.view(np.int16)).cuda()
    Xd = torch.from_numpy(np.concatenate([hi, lo]).view(np.int16)).cuda()
    return Wd, Xd


@pytest.mark.parametrize("n_out,T,K", [(520, 5, 1024), (1024, 130, 2048)])
def test_noalloc_matches_oracle_gemv(mk, n_out, T, K):
    """Each output row against the oracle's fp64 W x of that position's
    activation (hi + lo, exact in float64)."""
    import oracle
    W, hi, lo = _host_operands(n_out, T, K, seed=7 * n_out + T)
    Wd = torch.from_numpy(W.view(np.int16)).cuda()
    Xd = torch.from_numpy(np.concatenate([hi, lo]).view(np.int16)).cuda()
    c = torch.full((T, n_out), float("nan"), dtype=torch.float32, device="cuda")
    mk.mk_debug_gemm_noalloc(Wd, Xd, c)
    torch.cuda.synchronize()
    got = c.cpu().numpy()
    x = (synth.bf16_bits_to_f32(hi).astype(np.float64)
         + synth.bf16_bits_to_f32(lo).astype(np.float64))
    ref = np.stack([oracle.gemv(W, x[t]) for t in range(T)])
    err = rel_l2(got, ref)
    assert err <= 2e-5, "no-alloc GEMM vs oracle rel-L2 %.3e" % err


@pytest.mark.parametrize("n_out,T,K", [(520, 5, 1024), (1024, 130, 2048), (200, 70, 192)])
def test_noalloc_matches_allocating_entry_twice(mk, n_out, T, K):
    Wd, Xd = _operands(n_out, T, K, seed=n_out + T)
    ref = torch.full((T, n_out), float("nan"), dtype=torch.float32, device="cuda")
    mk.mk_debug_gemm(Wd, Xd, ref)
    outs = []
    for _ in range(2):  # two calls in a row reuse the same static scratch
        c = torch.full((T, n_out), float("nan"), dtype=torch.float32, device="cuda")
        mk.mk_debug_gemm_noalloc(Wd, Xd, c)
        outs.append(c)
    torch.cuda.synchronize()
    r = ref.cpu().numpy()
    for c in outs:
        got = c.cpu().numpy()
        assert np.isfinite(got).all()
        err = rel_l2(got, r)
        assert err <= 2e-5, "no-alloc GEMM rel-L2 %.3e" % err
    assert torch.equal(outs[0], outs[1])


def test_noalloc_rejects_more_than_its_scratch(mk):
    n_out, T, K = 4096, 513, 64  # T * n_out > 2^21 floats
    Wd = torch.zeros((n_out, K), dtype=torch.int16, device="cuda")
    Xd = torch.zeros((2 * T, K), dtype=torch.int16, device="cuda")
    c = torch.zeros((T, n_out), dtype=torch.float32, device="cuda")
    with pytest.raises(mk.MkError) as ei:
        mk.mk_debug_gemm_noalloc(Wd, Xd, c)
    assert ei.value.code == mk.MK_ERR_ARG
