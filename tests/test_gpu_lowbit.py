"""GPU parity of the 4-bit weight path (mk_quantize_w4, mk_gemv_w4) with the
oracle's dequantising functions, through the C ABI.

Quantisation is integer work decided in fp32 on both sides: codes and scales
must match bit for bit.  The GEMV accumulates in fp32, so it is compared
with the oracle's fp64 product at rel-L2 1e-5.  Shapes span several row
blocks with ragged tails, every token count the kernel is built for, the
MLP width and the full tied LM head (sampled rows).
"""
import numpy as np
import pytest

import oracle
from attention_decode_megakernel_b200 import synth

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


def _quantize_on_gpu(mk, W_bits):
    rows, cols = W_bits.shape
    Wd = torch.from_numpy(W_bits.view(np.int16)).cuda()
    codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device="cuda")
    scales = torch.empty((rows, cols // 64), dtype=torch.float32, device="cuda")
    mk.quantize_w4(Wd, codes, scales)
    torch.cuda.synchronize()
    return codes, scales


def _rel_l2(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


@pytest.mark.parametrize("rows,cols", [(300, 1024), (77, 3584), (5, 64)])
def test_quantize_matches_oracle_bitwise(mk, rows, cols):
    rng = np.random.default_rng(rows + cols)
    w = rng.standard_normal((rows, cols), dtype=np.float32) * 0.02
    w[0, :64] = 0.0                      # an all-zero group
    w[-1, 64 % cols] = 0.0
    W = synth.f32_to_bf16_bits(w)
    codes, scales = _quantize_on_gpu(mk, W)
    oc, os_ = oracle.quantize_w4(W)
    assert np.array_equal(codes.cpu().numpy(), oc)
    assert np.array_equal(scales.cpu().numpy().view(np.uint32), os_.view(np.uint32))


@pytest.mark.parametrize("T", [1, 2, 3, 4, 5, 6, 7, 8])
@pytest.mark.parametrize("rows,cols", [(1000, 1024), (300, 3584), (17, 64)])
def test_gemv_w4_against_oracle(mk, T, rows, cols):
    rng = np.random.default_rng(1000 * T + rows)
    W = synth.f32_to_bf16_bits(rng.standard_normal((rows, cols), dtype=np.float32) * 0.02)
    codes, scales = _quantize_on_gpu(mk, W)
    x = rng.standard_normal((T, cols), dtype=np.float32)
    y = torch.full((T, rows), float("nan"), dtype=torch.float32, device="cuda")
    mk.gemv_w4(codes, scales, torch.from_numpy(x).cuda(), y)
    torch.cuda.synchronize()
    got = y.cpu().numpy()
    oc, os_ = codes.cpu().numpy(), scales.cpu().numpy()
    for t in range(T):
        want = oracle.gemv_w4(oc, os_, x[t].astype(np.float64))
        assert _rel_l2(got[t], want) <= 1e-5, (T, t)


def test_gemv_w4_full_lm_head_sampled_rows(mk):
    """The tied LM head of the 0.8B shape (151,936 x 1024), quantised on the
    GPU; 64 sampled rows of codes and 2 tokens of outputs against the oracle."""
    rows, cols = 151936, 1024
    rng = np.random.default_rng(11)
    W = synth.f32_to_bf16_bits(rng.standard_normal((rows, cols), dtype=np.float32) * 0.02)
    codes, scales = _quantize_on_gpu(mk, W)
    x = rng.standard_normal((2, cols), dtype=np.float32)
    y = torch.empty((2, rows), dtype=torch.float32, device="cuda")
    mk.gemv_w4(codes, scales, torch.from_numpy(x).cuda(), y)
    torch.cuda.synchronize()
    pick = np.concatenate([[0, 1, rows - 1], rng.choice(rows, 61, replace=False)])
    oc, os_ = oracle.quantize_w4(W[pick])
    assert np.array_equal(codes.cpu().numpy()[pick], oc)
    assert np.array_equal(scales.cpu().numpy()[pick], os_)
    got = y.cpu().numpy()[:, pick]
    for t in range(2):
        want = oracle.gemv_w4(oc, os_, x[t].astype(np.float64))
        assert _rel_l2(got[t], want) <= 1e-5


def test_w4_argument_errors(mk):
    codes = torch.zeros((4, 48), dtype=torch.uint8, device="cuda")
    scales = torch.zeros((4, 1), dtype=torch.float32, device="cuda")
    x = torch.zeros((1, 96), dtype=torch.float32, device="cuda")
    y = torch.zeros((1, 4), dtype=torch.float32, device="cuda")
    L = mk.lib()
    # cols not a multiple of 64
    assert L.mk_gemv_w4(codes.data_ptr(), scales.data_ptr(), x.data_ptr(), 1, 4, 96,
                        y.data_ptr(), None) == mk.MK_ERR_ARG
    assert L.mk_quantize_w4(codes.data_ptr(), 4, 96, codes.data_ptr(), scales.data_ptr(),
                            None) == mk.MK_ERR_ARG
    # token counts outside 1..8
    for T in (0, 9):
        assert L.mk_gemv_w4(codes.data_ptr(), scales.data_ptr(), x.data_ptr(), T, 4, 64,
                            y.data_ptr(), None) == mk.MK_ERR_ARG
