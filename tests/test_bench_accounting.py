"""The roofline numerators bench.py divides by, checked against the model's
shapes written out by hand (0.8B-shaped hybrid: 18 DeltaNet + 6 attention
layers, hidden 1024, vocab 151936, MLP 3584, 16 DeltaNet heads of 128,
8 query / 2 KV heads of 256)."""
import os
import sys

import pytest

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402
from attention_decode_megakernel_b200 import synth  # noqa: E402

H, V, I = 1024, 151936, 3584
NH, DK, DV = 16, 128, 128
NQ, NKV, HD = 8, 2, 256
CH = 2 * NH * DK + NH * DV            # conv channels q|k|v = 6144
RIN = CH + NH * DV + 2 * NH           # in-projection rows q|k|v|z|b|a = 8224
N_DN, N_ATT = 18, 6


def _layer_matrix_weights():
    mlp = 3 * I * H
    dn = RIN * H + H * NH * DV + mlp
    att = (NQ + 2 * NKV) * HD * H + H * NQ * HD + mlp
    return N_DN * dn + N_ATT * att


def test_decode_bytes_of_one_token():
    cfg = synth.hybrid_08b_config(max_ctx=1024)
    ctx = 520
    bf16, f32 = 2, 4
    small = (H + H) * bf16                                   # the two norm gains
    dn_small = CH * 4 * bf16 + 2 * NH * f32 + DV * bf16      # conv taps, A_log, dt_bias, out norm
    weights = (_layer_matrix_weights() * bf16 + N_DN * (small + dn_small) + N_ATT * small
               + V * H * bf16 + H * bf16)                    # tied head + final norm
    state = 2 * N_DN * NH * DV * DK * f32                    # read + write
    conv = 2 * N_DN * CH * 3 * f32
    kv = N_ATT * 2 * NKV * HD * bf16 * (ctx + 1)             # read ctx positions, write one
    logits = V * f32
    assert bench.decode_bytes(cfg, ctx) == weights + state + conv + kv + logits
    # the order of magnitude the measurements quote: 1.33 GB per token
    assert bench.decode_bytes(cfg, ctx) == pytest.approx(1.3304e9, rel=1e-3)


def test_prefill_flops_of_pp520():
    cfg = synth.hybrid_08b_config(max_ctx=1024)
    assert bench.matrix_params(cfg) == _layer_matrix_weights()
    flops = 2.0 * _layer_matrix_weights() * 520 + 2.0 * V * H
    assert flops == pytest.approx(504.744e9, rel=1e-5)


def test_verify_bytes_of_one_call():
    cfg = synth.hybrid_08b_config(max_ctx=4200)
    bf16, f32 = 2, 4
    ctx, n, replayed = 4096, 5, 1
    weights = bench.decode_bytes(cfg, 0) - 2 * N_DN * NH * DV * DK * f32 \
        - 2 * N_DN * CH * 3 * f32 - N_ATT * 2 * NKV * HD * bf16 - V * f32
    state = 2 * (N_DN * NH * DV * DK * f32 + N_DN * CH * 3 * f32)  # read + replayed write
    rec = N_DN * (NH * (DK + DV + 2) + CH) * f32                    # per position
    kv = N_ATT * 2 * NKV * HD * bf16 * (ctx + n)                    # read ctx, append n
    logits = n * V * f32
    assert bench.weight_bytes(cfg) == weights
    assert bench.verify_bytes(cfg, ctx, n, replayed) == \
        weights + state + (n + replayed) * rec + kv + logits
    # records are a few MB where 5 full state copies would be ~100 MB
    assert (n + replayed) * rec < 5e6
