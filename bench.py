#!/usr/bin/env python
"""Benchmark: batch-1 greedy decode (tg128) after a 520-token prompt (pp520)
on the 0.8B-shaped hybrid DeltaNet/attention model, synthetic bf16 weights.

One step = mk_reset + mk_prefill(520 prompt tokens) + mk_generate(128 greedy
tokens, device-resident loop).  `value` is decode tokens/s over all ranks
(replicas: one independent engine per GPU, no collective on the data path);
prefill tokens/s, the decode kernel's HBM roofline fraction, the
end-to-end number through host buffers and the CPU oracle baseline ride on
the same JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

PROMPT = 520
GEN = 128
# DRAM bytes (read + written) of one decode launch at context 520, from an ncu
# capture of the current decode kernel (dram__bytes_read.sum +
# dram__bytes_write.sum); None once the kernel changes.
DECODE_TRAFFIC_BYTES = 1340556000  # 1.311269 GB read + 29.286912 MB written
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
FALLBACK_BF16_TFLOPS_SUSTAINED = 1400.0


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=3)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-extras", action="store_true",
                   help="skip the long-context, verify, prefill-roofline and delta-sweep lines")
    p.add_argument("--mode", choices=["full", "kernel", "delta", "verify", "w4"], default="full",
                   help="small cases for profilers: kernel = W+K single decode launches "
                        "at context --ctx on a seeded synthetic state; delta = W+K "
                        "isolated delta steps at batch --batch; verify = W+K 5-token "
                        "verify calls at context 4096; w4 = the 4-bit weight GEMV at the "
                        "LM head's shape")
    p.add_argument("--ctx", type=int, default=520, help="context of --mode kernel")
    p.add_argument("--batch", type=int, default=8, help="sequences of --mode delta")
    return p.parse_args()


def run_kernel_mode(args):
    """W warm-up + K timed decode launches at context --ctx (one engine)."""
    import numpy as np
    import torch

    import attention_decode_megakernel_b200 as mk
    from attention_decode_megakernel_b200 import build, synth
    build.build()
    ctx = args.ctx
    cfg = synth.hybrid_08b_config(max_ctx=ctx + 64)
    w = synth.make_weights(cfg)
    eng = mk.Engine(cfg, w)
    st = synth.make_engine_state(cfg, ctx=ctx)
    dev = {k: (torch.from_numpy(v.view(np.int16) if v.dtype == np.uint16 else v).cuda()
               if isinstance(v, np.ndarray) else v) for k, v in st.items()}
    del st
    eng.set_state(dev)
    logits = torch.empty(cfg.vocab, dtype=torch.float32, device="cuda")
    for _ in range(args.warmup):
        eng.decode_step(1, logits)
    eng.sync()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(eng.stream)
    for _ in range(args.steps):
        eng.decode_step(1, logits)
    e1.record(eng.stream)
    eng.sync()
    ms = e0.elapsed_time(e1) / max(args.steps, 1)
    print(json.dumps({"mode": "kernel", "ctx": ctx, "launches": args.warmup + args.steps,
                      "ms_per_launch": ms,
                      "GBps": decode_bytes(cfg, ctx + args.warmup) / ms / 1e6}), flush=True)


def run_delta_mode(args):
    """W warm-up + K timed isolated delta steps, B = --batch sequences x 16
    heads, dk = dv = 128 (one launch per step)."""
    import torch

    import attention_decode_megakernel_b200 as mk
    from attention_decode_megakernel_b200 import build
    build.build()
    B, H, D = args.batch, 16, 128
    S = torch.randn(B, H, D, D, device="cuda") * 0.1
    q = torch.nn.functional.normalize(torch.randn(B, H, D, device="cuda"), dim=-1)
    k = torch.nn.functional.normalize(torch.randn(B, H, D, device="cuda"), dim=-1)
    q16, k16 = q.to(torch.bfloat16).view(torch.int16), k.to(torch.bfloat16).view(torch.int16)
    v16 = torch.randn(B, H, D, device="cuda").to(torch.bfloat16).view(torch.int16)
    be = torch.rand(B, H, device="cuda")
    al = 0.9 + 0.1 * torch.rand(B, H, device="cuda")
    o = torch.empty(B, H, D, device="cuda")
    for _ in range(args.warmup):
        mk.mk_delta_step(S, q16, k16, v16, al, be, o)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        mk.mk_delta_step(S, q16, k16, v16, al, be, o)
    e1.record()
    torch.cuda.synchronize()
    us = 1000.0 * e0.elapsed_time(e1) / max(args.steps, 1)
    sb = 2 * B * H * D * D * 4 + B * H * (3 * D * 2 + 8 + D * 4)
    print(json.dumps({"mode": "delta", "batch": B, "us_per_step": us, "bytes_per_step": sb,
                      "GBps": sb / us / 1e3}), flush=True)


def run_verify_mode(args):
    """W warm-up + K timed 5-token verify calls (accept 1 each) at context
    4096 of the 0.8B-shaped model on a seeded synthetic state."""
    import numpy as np
    import torch

    import attention_decode_megakernel_b200 as mk
    from attention_decode_megakernel_b200 import build, synth
    build.build()
    ctx = 4096
    cfg = synth.hybrid_08b_config(max_ctx=ctx + 64)
    w = synth.make_weights(cfg)
    eng = mk.Engine(cfg, w)
    st = synth.make_engine_state(cfg, ctx=ctx)
    eng.set_state({k: (torch.from_numpy(v.view(np.int16) if v.dtype == np.uint16 else v).cuda()
                       if isinstance(v, np.ndarray) else v) for k, v in st.items()})
    del st
    drafts = synth.make_tokens(cfg.vocab, 5 * (args.warmup + args.steps),
                               seed=synth.SEED_DRAFTS).reshape(-1, 5)
    vl = torch.empty((5, cfg.vocab), dtype=torch.float32, device="cuda")
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n0 = 0
    for i in range(args.warmup + args.steps):
        if i == args.warmup:
            eng.sync()
            n0 = eng.launch_count()
            e0.record(eng.stream)
        eng.verify(drafts[i], vl)
        eng.accept(1)
    e1.record(eng.stream)
    eng.sync()
    ms = e0.elapsed_time(e1) / max(args.steps, 1)
    print(json.dumps({"mode": "verify", "ctx": ctx, "calls": args.warmup + args.steps,
                      "ms_per_call": ms,
                      "launches_per_call": (eng.launch_count() - n0) / max(args.steps, 1)}),
          flush=True)


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, "fallback"


def sustained_tc_peak():
    """bf16 tensor throughput sustained under the power cap (the prompt path
    runs inside a seconds-long loop), else the burst figure."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["bf16_tflops_sustained"]), "measured sustained"
    except Exception:
        return FALLBACK_BF16_TFLOPS_SUSTAINED, "fallback sustained"


def weight_bytes(cfg):
    """Every weight once: the layers' tensors, the tied embedding (read as the
    LM head) and the final norm gain."""
    import numpy as np
    from attention_decode_megakernel_b200 import synth
    n = 0
    for is_attn in cfg.layer_is_attn:
        for _, shape, kind in synth.layer_tensor_shapes(cfg, is_attn):
            n += int(np.prod(shape)) * (4 if kind == "f" else 2)
    return n + cfg.vocab * cfg.hidden * 2 + cfg.hidden * 2


def state_bytes(cfg):
    """One read (or one write) of the DeltaNet state and the conv history."""
    return (cfg.n_dn * cfg.dn_heads * cfg.dn_dv * cfg.dn_dk * 4
            + cfg.n_dn * cfg.conv_channels * (cfg.conv_k - 1) * 4)


def kv_position_bytes(cfg):
    """K and V of one position in every attention layer (bf16)."""
    return cfg.n_attn * 2 * cfg.kv_heads * cfg.head_dim * 2


def decode_bytes(cfg, ctx):
    """Algorithmic HBM bytes of one decode launch at context `ctx` (the new
    token is position ctx): every weight once (tied embedding read as the LM
    head), DeltaNet state and conv history read + written, KV read of ctx
    positions + write of one, logits written."""
    return (weight_bytes(cfg) + 2 * state_bytes(cfg) + kv_position_bytes(cfg) * (ctx + 1)
            + cfg.vocab * 4)


def verify_bytes(cfg, ctx, n, replayed):
    """Algorithmic HBM bytes of one n-token verify call at context ctx whose
    previous accept kept `replayed` positions: every weight once; the state
    read once and, replayed, written once to the next buffer; n records
    written (per DeltaNet layer and position: key, value, alpha, beta and
    the conv inputs) and the replayed ones read; KV read over the context
    and n positions appended; n rows of logits."""
    rec = cfg.n_dn * (cfg.dn_heads * (cfg.dn_dk + cfg.dn_dv + 2) + cfg.conv_channels) * 4
    return (weight_bytes(cfg) + 2 * state_bytes(cfg) + (n + replayed) * rec
            + kv_position_bytes(cfg) * (ctx + n) + n * cfg.vocab * 4)


class Clocks:
    """nvidia-smi samples during the timed region (read-only)."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.p = None

    def start(self):
        try:
            self.p = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.Q,
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.p = None

    def stop(self):
        if self.p is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.p.terminate()
        try:
            self.p.wait(timeout=5)
        except Exception:
            self.p.kill()
        self.f.flush()
        self.f.seek(0)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.f.read().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        os.unlink(self.f.name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm)}


def oracle_decode_rate(cfg, w, budget_s=12.0, max_steps=64):
    """The fp64 oracle's decode tokens/s on this host at context 520 (state
    installed from the seeded synthetic generator), timed for ~budget_s."""
    import oracle
    from attention_decode_megakernel_b200 import synth
    m = oracle.OracleModel(cfg, w)
    m.set_state(synth.make_engine_state(cfg, ctx=PROMPT))
    tok, n, t0 = 1, 0, time.perf_counter()
    while n < max_steps:
        logits, _ = m.step(tok)
        tok = int(logits.argmax())
        n += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    return n / dt, n, dt, cores


def oracle_other_rates(cfg, w):
    """The oracle on the other configurations, on small bounded samples (a
    reported CPU baseline, not a target): prompt positions/s of the 0.8B
    model (8 positions from an empty state; the oracle has no batched prompt
    path, so this equals its decode rate at short context), verify calls/s
    (5 positions from a cloned state at context 520, the oracle's
    checkpoint = a clone) and gated delta steps/s for one sequence of
    16 heads x 128 x 128 (64 steps); the tiny model's decode tokens/s; the
    0.8B decode on a single thread (2 steps)."""
    import numpy as np
    import oracle
    from attention_decode_megakernel_b200 import synth
    out = {}
    m = oracle.OracleModel(cfg, w)
    toks = synth.make_tokens(cfg.vocab, 8)
    t0 = time.perf_counter()
    for t in toks:
        m.step(int(t), want_logits=False)
    out["prefill_positions_s"] = len(toks) / (time.perf_counter() - t0)
    m.set_state(synth.make_engine_state(cfg, ctx=PROMPT))
    drafts = synth.make_tokens(cfg.vocab, 5, seed=synth.SEED_DRAFTS)
    t0 = time.perf_counter()
    c = m.clone()
    for t in drafts:
        c.step(int(t))
    out["verify_calls_s"] = 1.0 / (time.perf_counter() - t0)
    sw = synth.make_delta_sweep(1, 64, heads=16, dk=128, dv=128)
    S = sw["S0"].astype(np.float64)
    q = synth.bf16_bits_to_f32(sw["q"]).astype(np.float64)
    k = synth.bf16_bits_to_f32(sw["k"]).astype(np.float64)
    v = synth.bf16_bits_to_f32(sw["v"]).astype(np.float64)
    t0 = time.perf_counter()
    for h in range(16):
        oracle.delta_sequence(S[0, h], q[:, 0, h], k[:, 0, h], v[:, 0, h],
                              sw["alpha"][:, 0, h].astype(np.float64),
                              sw["beta"][:, 0, h].astype(np.float64))
    out["delta_steps_s_B1"] = 64 / (time.perf_counter() - t0)
    # the tiny configuration's decode, and the 0.8B decode on one thread
    tcfg = synth.tiny_config(max_ctx=64)
    tm = oracle.OracleModel(tcfg, synth.make_weights(tcfg))
    t0 = time.perf_counter()
    for t in range(32):
        tm.step(t)
    out["tiny_decode_tok_s"] = 32 / (time.perf_counter() - t0)
    oracle.set_threads(1)
    try:
        m.set_state(synth.make_engine_state(cfg, ctx=PROMPT))
        t0 = time.perf_counter()
        for t in range(2):
            m.step(t + 1)
        out["decode_tok_s_1_thread"] = 2 / (time.perf_counter() - t0)
    finally:
        oracle.set_threads(0)
    return out


def run_reference(args, rank):
    """Reference arm: the CPU oracle as it stands, on the host cores."""
    if rank != 0:
        return
    from attention_decode_megakernel_b200 import synth
    cfg = synth.hybrid_08b_config(max_ctx=PROMPT + GEN + 8)
    w = synth.make_weights(cfg)
    import oracle
    m = oracle.OracleModel(cfg, w)
    st = synth.make_engine_state(cfg, ctx=PROMPT)
    per_step = 4
    times = []
    for i in range(args.warmup + args.steps):
        m.set_state(st)
        tok = 1
        t0 = time.perf_counter()
        for _ in range(per_step):
            logits, _ = m.step(tok)
            tok = int(logits.argmax())
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    total = sum(times)
    value = per_step * args.steps / total
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    sample = ("%d greedy decode steps per bench step of the 0.8B-shaped model at "
              "context 520 (seeded synthetic state), fp64 oracle" % per_step)
    line = {
        "impl": "reference", "metric": "batch-1 decode tok/s (tg128)", "value": value,
        "unit": "tok/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000 * total / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "hybrid-0.8B-24L-h1024 pp520+tg128 (decode at ctx 520)",
                   "prompt": PROMPT, "gen": GEN},
        "cpu_baseline": {"value": value, "unit": "tok/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tok/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def max_over_ranks(values, dist, device):
    """Each timing as the maximum over all ranks (the slowest replica sets
    the job's time); identity without a process group."""
    if dist is None:
        return [float(v) for v in values]
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def replica_rate(world, units_per_rank, max_ms):
    """Whole-job throughput of `world` independent replicas: every rank's
    units over the slowest rank's time."""
    return world * units_per_rank / (max_ms / 1000.0)


def matrix_params(cfg):
    """Weights of every projection matrix of the layer stack (no embedding)."""
    import numpy as np
    from attention_decode_megakernel_b200 import synth
    n = 0
    for is_attn in cfg.layer_is_attn:
        for name, shape, kind in synth.layer_tensor_shapes(cfg, is_attn):
            if len(shape) == 2 and shape[1] > 4:  # [out][in] matrices (not conv taps)
                n += int(np.prod(shape))
    return n


def state_to_device(torch, np, st):
    return {k: (torch.from_numpy(v.view(np.int16) if v.dtype == np.uint16 else v).cuda()
                if isinstance(v, np.ndarray) else v) for k, v in st.items()}


def w4_gemv_lines(mk, torch, hbm):
    """4-bit weight GEMV (mk_gemv_w4) at the tied LM head's shape (151,936 x
    1024) for 1 and 5 activation rows: three quantised copies used in turn,
    so each launch reads a matrix the one before did not (3 x 97 MB > the
    126 MB L2)."""
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    rows, cols = 151936, 1024
    g = torch.Generator(device="cuda").manual_seed(12)
    sets = []
    for _ in range(3):
        W = (torch.randn((rows, cols), generator=g, device="cuda") * 0.02).to(torch.bfloat16)
        codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device="cuda")
        scales = torch.empty((rows, cols // 64), dtype=torch.float32, device="cuda")
        mk.quantize_w4(W.view(torch.int16), codes, scales)
        sets.append((codes, scales))
        del W
    w4 = {}
    for T in (1, 5):
        x = torch.randn((T, cols), generator=g, device="cuda")
        y = torch.empty((T, rows), dtype=torch.float32, device="cuda")
        for i in range(6):
            mk.gemv_w4(sets[i % 3][0], sets[i % 3][1], x, y)
        torch.cuda.synchronize()
        n = 60
        e0.record()
        for i in range(n):
            mk.gemv_w4(sets[i % 3][0], sets[i % 3][1], x, y)
        e1.record()
        torch.cuda.synchronize()
        us = e0.elapsed_time(e1) * 1000.0 / n
        byts = rows * cols // 2 + rows * cols // 64 * 4 + T * cols * 4 + T * rows * 4
        w4["T%d" % T] = {"us_per_launch": us, "GBps": byts / us / 1e3,
                         "frac": byts / us / 1e3 / hbm, "bytes_per_launch": byts,
                         "bf16_equivalent_bytes": rows * cols * 2}
    del sets
    return w4


def extra_workloads(mk, synth, torch, np, prefill_ms_per_call, hbm, tc_peak, peak_kind):
    """The other configurations of the method, each timed on the device with
    CUDA events: long-context decode, 5-token verify, the prompt path's
    tensor-core roofline, the isolated delta-step sweep and the 4-bit weight
    GEMV."""
    out = {}
    # prompt path: algorithmic FLOPs of pp520 (every matrix once per position,
    # LM head for the last position only) over the measured prefill time
    cfg = synth.hybrid_08b_config(max_ctx=PROMPT + GEN + 8)
    flops = 2.0 * matrix_params(cfg) * PROMPT + 2.0 * cfg.vocab * cfg.hidden
    tf = flops / (prefill_ms_per_call / 1000.0) / 1e12
    tc_sus, sus_kind = sustained_tc_peak()
    out["prefill_pp520"] = {"tok_s": PROMPT / (prefill_ms_per_call / 1000.0),
                            "ms": prefill_ms_per_call, "gflop": flops / 1e9,
                            "roofline": {"bound": "tensor", "achieved": tf, "peak": tc_sus,
                                         "unit": "TFLOP/s", "frac": tf / tc_sus,
                                         "peak_kind": sus_kind, "burst_peak": tc_peak}}
    del cfg

    # long context: the attention layers' KV at 32768 positions (synthetic
    # state of that shape), then 32 greedy decode launches
    ctx = 32768
    cfg = synth.hybrid_08b_config(max_ctx=ctx + 64)
    w = synth.make_weights(cfg)
    eng = mk.Engine(cfg, w)
    dev = state_to_device(torch, np, synth.make_engine_state(cfg, ctx=ctx))
    eng.set_state(dev)
    toks = torch.zeros(32, dtype=torch.int32, device="cuda")
    eng.generate(1, 4, toks)
    eng.sync()
    eng.set_state(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(eng.stream)
    eng.generate(1, 32, toks)
    e1.record(eng.stream)
    eng.sync()
    ms = e0.elapsed_time(e1) / 32
    byts = sum(decode_bytes(cfg, ctx + i) for i in range(32)) / 32
    out["decode_ctx32k"] = {"tok_s": 1000.0 / ms, "ms_per_token": ms,
                            "roofline": {"bound": "hbm", "achieved": byts / ms / 1e6,
                                         "peak": hbm, "unit": "GB/s",
                                         "frac": byts / ms / 1e6 / hbm,
                                         "bytes_per_launch": byts}}
    eng.close()
    del eng, dev

    # speculative-verify shape: context 4096, 200 calls of 5 tokens (the
    # accepted token + 4 seeded drafts); draft j is kept while it equals the
    # greedy choice at position j-1
    ctx = 4096
    cfg = synth.hybrid_08b_config(max_ctx=ctx + 256)
    eng = mk.Engine(cfg, w)
    eng.set_state(state_to_device(torch, np, synth.make_engine_state(cfg, ctx=ctx)))
    drafts = synth.make_tokens(cfg.vocab, 4 * 220, seed=synth.SEED_DRAFTS).reshape(220, 4)
    vl = torch.empty((5, cfg.vocab), dtype=torch.float32, device="cuda")
    calls, kept, tok = 200, 0, 1
    for i in range(calls + 5):
        if i == 5:
            eng.sync()
            t0 = time.perf_counter()
            e0.record(eng.stream)
            kept = 0
        seq = np.concatenate([[tok], drafts[i % 220]]).astype(np.int32)
        eng.verify(seq, vl)
        am = torch.argmax(vl, dim=1).cpu().numpy()
        k = 1
        while k < 5 and seq[k] == am[k - 1]:
            k += 1
        eng.accept(k)
        kept += k
        tok = int(am[k - 1])
    e1.record(eng.stream)
    eng.sync()
    wall = time.perf_counter() - t0
    dev_ms = e0.elapsed_time(e1)
    # the context grows by the accepted positions: its mean over the calls
    vbytes = verify_bytes(cfg, ctx + kept / 2.0, 5, kept / calls)
    out["verify_5tok_ctx4096"] = {
        "calls_s": calls / (dev_ms / 1000.0), "ms_per_call": dev_ms / calls,
        "positions_s": 5 * calls / (dev_ms / 1000.0), "accepted_per_call": kept / calls,
        "wall_calls_s": calls / wall,
        "roofline": {"bound": "hbm", "achieved": vbytes / (dev_ms / calls) / 1e6, "peak": hbm,
                     "unit": "GB/s", "frac": vbytes / (dev_ms / calls) / 1e6 / hbm,
                     "bytes_per_call": vbytes}}
    eng.close()
    del eng, w

    # isolated gated delta-rule step: B sequences x 16 heads, dk = dv = 128,
    # 1024 sequential steps, one launch per step, the 1024 launches replayed
    # from one CUDA graph (the device time, not the host's launch rate)
    sweep = {}
    for B in (1, 8, 64):
        H, D, steps = 16, 128, 1024
        S = torch.randn(B, H, D, D, device="cuda") * 0.1
        q = torch.nn.functional.normalize(torch.randn(8, B, H, D, device="cuda"), dim=-1)
        k = torch.nn.functional.normalize(torch.randn(8, B, H, D, device="cuda"), dim=-1)
        q16, k16 = q.to(torch.bfloat16).view(torch.int16), k.to(torch.bfloat16).view(torch.int16)
        v16 = torch.randn(8, B, H, D, device="cuda").to(torch.bfloat16).view(torch.int16)
        be = torch.rand(8, B, H, device="cuda")
        al = 0.9 + 0.1 * torch.rand(8, B, H, device="cuda")
        o = torch.empty(B, H, D, device="cuda")
        for t in range(16):
            mk.mk_delta_step(S, q16[t % 8], k16[t % 8], v16[t % 8], al[t % 8], be[t % 8], o)
        torch.cuda.synchronize()
        cs = torch.cuda.Stream()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=cs):
            for t in range(steps):
                mk.mk_delta_step(S, q16[t % 8], k16[t % 8], v16[t % 8], al[t % 8], be[t % 8], o,
                                 stream=cs.cuda_stream)
        graph.replay()  # warm-up replay (replays run on the current stream)
        torch.cuda.synchronize()
        e0.record()
        graph.replay()
        e1.record()
        torch.cuda.synchronize()
        us = 1000.0 * e0.elapsed_time(e1) / steps
        del graph
        sb = 2 * B * H * D * D * 4 + B * H * (3 * D * 2 + 8 + D * 4)
        sweep["B%d" % B] = {"us_per_step": us, "state_GBps": sb / us / 1e3,
                            "frac": sb / us / 1e3 / hbm, "bytes_per_step": sb,
                            "launch": "CUDA graph of %d launches" % steps}
        del S, q, k, q16, k16, v16, be, al, o
    out["delta_sweep_dk128_h16"] = sweep

    out["gemv_w4_lmhead_151936x1024"] = w4_gemv_lines(mk, torch, hbm)
    return out


def main():
    args = parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank)
        return
    if args.mode == "delta":
        run_delta_mode(args)
        return
    if args.mode == "verify":
        run_verify_mode(args)
        return
    if args.mode == "w4":
        import torch
        import attention_decode_megakernel_b200 as mk
        from attention_decode_megakernel_b200 import build
        build.build()
        hbm, _, _ = peaks()
        print(json.dumps({"mode": "w4", "gemv_w4_lmhead_151936x1024":
                          w4_gemv_lines(mk, torch, hbm)}), flush=True)
        return
    if args.mode == "kernel":
        run_kernel_mode(args)
        return

    import numpy as np
    import torch

    import attention_decode_megakernel_b200 as mk
    from attention_decode_megakernel_b200 import build, synth

    build.build()
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))

    cfg = synth.hybrid_08b_config(max_ctx=PROMPT + GEN + 8)
    w = synth.make_weights(cfg)
    eng = mk.Engine(cfg, w)
    prompt = synth.make_tokens(cfg.vocab, PROMPT)
    toks = torch.zeros(GEN, dtype=torch.int32, device="cuda")
    stream = eng.stream

    def one_step(evs=None):
        eng.reset()
        if evs:
            evs[0].record(stream)
        eng.prefill(prompt)
        if evs:
            evs[1].record(stream)
        eng.generate(-1, GEN, toks)
        if evs:
            evs[2].record(stream)

    for _ in range(args.warmup):
        one_step()
    eng.sync()

    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    clk = Clocks(local)
    clk.start()
    launches0 = eng.launch_count()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    for k in range(args.steps):
        one_step(evs[k])
    torch.cuda.synchronize()
    eng.sync()
    launches = eng.launch_count() - launches0
    clocks = clk.stop()
    if dist:
        dist.barrier()
    prefill_ms = sum(e[0].elapsed_time(e[1]) for e in evs)
    decode_ms = sum(e[1].elapsed_time(e[2]) for e in evs)
    prefill_ms, decode_ms = max_over_ranks([prefill_ms, decode_ms], dist, "cuda")
    out_tokens = toks.cpu().numpy().tolist()

    # end to end through the public API with host buffers: the first token
    # comes from the host, the 128 generated tokens are read back into pinned
    # host memory, both inside the timed region
    host_toks = torch.zeros(GEN, dtype=torch.int32).pin_memory()
    e2e_times = []
    first = int(out_tokens[0])
    for _ in range(args.steps):
        eng.reset()
        eng.prefill(prompt)
        eng.sync()
        t0 = time.perf_counter()
        eng.generate(first, GEN, toks)
        host_toks.copy_(toks, non_blocking=True)
        stream.synchronize()
        e2e_times.append(time.perf_counter() - t0)
    e2e_s = max_over_ranks([sum(e2e_times)], dist, "cuda")[0]

    hbm, _, peak_kind = peaks()
    per_launch_s = decode_ms / 1000.0 / (GEN * args.steps)
    bytes_avg = sum(decode_bytes(cfg, PROMPT + i) for i in range(GEN)) / GEN
    achieved = bytes_avg / per_launch_s / 1e9
    value = replica_rate(world, GEN * args.steps, decode_ms)
    prefill_tps = world * PROMPT * args.steps / (prefill_ms / 1000.0)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, n, dt, cores = oracle_decode_rate(cfg, w)
        cpu = {"value": rate, "unit": "tok/s", "cores": cores, "kind": "oracle",
               "sample": "%d greedy decode steps of the 0.8B-shaped model at context 520 "
                         "(seeded synthetic state) in %.1f s, fp64 oracle" % (n, dt),
               "other_configs": oracle_other_rates(cfg, w)}

    extras = None
    if rank == 0 and world == 1 and not args.no_extras:
        eng_ms = prefill_ms / args.steps
        _, tc_peak, pk = peaks()
        extras = extra_workloads(mk, synth, torch, np, eng_ms, hbm, tc_peak, pk)

    line = {
        "metric": "batch-1 decode tok/s (tg128)", "value": value, "unit": "tok/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": (prefill_ms + decode_ms) / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "weights": "bf16",
        "data": "synthetic (seeded N(0,0.02) bf16 weights, uniform random prompt)",
        "config": {"workload": "hybrid-0.8B-24L-h1024 pp520+tg128", "prompt": PROMPT,
                   "gen": GEN, "batch": 1, "parallelism": "replicas" if world > 1 else "single",
                   "l2": "inputs larger than L2 (1.33 GB streamed per token vs 126 MB L2)"},
        "prefill_tok_s": prefill_tps,
        "decode_ms_per_token": per_launch_s * 1000.0,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                     "frac": achieved / hbm, "traffic": DECODE_TRAFFIC_BYTES, "peak_kind": peak_kind,
                     "kernel": "decode_kernel (one launch per token)",
                     "bytes_per_launch": bytes_avg},
        "e2e": {"value": world * GEN * args.steps / e2e_s, "unit": "tok/s",
                "h2d_bytes_per_step": 4, "d2h_bytes_per_step": GEN * 4},
        "gpu_launches": launches,
        "clocks": clocks,
        "cpu_baseline": cpu,
        "greedy_tokens_head": out_tokens[:8],
        "extras": extras,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    eng.close()
    if dist:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
