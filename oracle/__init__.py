"""ctypes binding of the fp64 CPU oracle (TEST INFRASTRUCTURE ONLY).

Only the tests, the smoke check and the benchmark's CPU-baseline leg import
this package.  It shares nothing with the CUDA engine except the seeded
inputs of ``attention_decode_megakernel_b200.synth``.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liboracle.so")
MAX_LAYERS = 64


def build(force: bool = False) -> str:
    """Compile oracle.c with gcc (strict IEEE: no fast-math)."""
    src = os.path.join(_HERE, "oracle.c")
    if (not force and os.path.exists(LIB_PATH)
            and os.path.getmtime(LIB_PATH) >= os.path.getmtime(src)
            and os.path.getmtime(LIB_PATH) >= os.path.getmtime(
                os.path.join(_HERE, "oracle.h"))):
        return LIB_PATH
    tmp = LIB_PATH + ".tmp.%d" % os.getpid()
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
           "-fno-fast-math", "-ffp-contract=off", src, "-o", tmp, "-lm"]
    subprocess.check_call(cmd)
    os.replace(tmp, LIB_PATH)
    return LIB_PATH


class OrcConfig(C.Structure):
    _fields_ = [("n_layers", C.c_int32),
                ("layer_is_attn", C.c_int32 * MAX_LAYERS),
                ("hidden", C.c_int32), ("vocab", C.c_int32), ("mlp", C.c_int32),
                ("dn_heads", C.c_int32), ("dn_dk", C.c_int32),
                ("dn_dv", C.c_int32), ("conv_k", C.c_int32),
                ("q_heads", C.c_int32), ("kv_heads", C.c_int32),
                ("head_dim", C.c_int32),
                ("rope_theta", C.c_double), ("rms_eps", C.c_double),
                ("max_ctx", C.c_int32)]


class OrcLayer(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in (
        "attn_norm", "in_proj", "conv_w", "A_log", "dt_bias", "out_norm",
        "out_proj", "w_q", "w_k", "w_v", "w_o", "mlp_norm", "w_gate", "w_up",
        "w_down")]


_lib = None
_D = C.POINTER(C.c_double)


def lib():
    global _lib
    if _lib is None:
        build()
        L = C.CDLL(LIB_PATH)
        L.orc_bf16_to_double.restype = C.c_double
        L.orc_bf16_to_double.argtypes = [C.c_uint16]
        L.orc_double_to_bf16.restype = C.c_uint16
        L.orc_double_to_bf16.argtypes = [C.c_double]
        for f in ("orc_sigmoid", "orc_softplus", "orc_silu"):
            getattr(L, f).restype = C.c_double
            getattr(L, f).argtypes = [C.c_double]
        L.orc_gemv.argtypes = [C.c_void_p, C.c_int, C.c_int, _D, _D]
        L.orc_quantize_w4.argtypes = [C.c_void_p, C.c_int, C.c_int, C.c_void_p, C.c_void_p]
        L.orc_dequantize_w4.argtypes = [C.c_void_p, C.c_void_p, C.c_int, C.c_int, _D]
        L.orc_gemv_w4.argtypes = [C.c_void_p, C.c_void_p, C.c_int, C.c_int, _D, _D]
        L.orc_set_threads.argtypes = [C.c_int]
        L.orc_set_threads.restype = None
        L.orc_rmsnorm.argtypes = [_D, C.c_void_p, C.c_int, C.c_double, _D]
        L.orc_l2norm.argtypes = [_D, C.c_int, C.c_double, _D]
        L.orc_causal_conv_step.argtypes = [C.c_int, C.c_int, C.c_void_p, _D, _D, _D]
        L.orc_gated_delta_step.argtypes = [C.c_int, C.c_int, _D, _D, _D, _D,
                                           C.c_double, C.c_double, _D]
        L.orc_delta_sequence.argtypes = [C.c_int, C.c_int, C.c_int, _D, _D, _D,
                                         _D, _D, _D, _D]
        L.orc_rope.argtypes = [_D, C.c_int, C.c_int, C.c_double]
        L.orc_softmax.argtypes = [_D, C.c_int, _D]
        L.orc_attention_head.argtypes = [_D, _D, _D, C.c_int, C.c_int, _D]
        L.orc_create.restype = C.c_void_p
        L.orc_create.argtypes = [C.POINTER(OrcConfig), C.POINTER(OrcLayer),
                                 C.c_void_p, C.c_void_p]
        L.orc_clone.restype = C.c_void_p
        L.orc_clone.argtypes = [C.c_void_p]
        L.orc_destroy.argtypes = [C.c_void_p]
        L.orc_reset.argtypes = [C.c_void_p]
        L.orc_pos.restype = C.c_int
        L.orc_pos.argtypes = [C.c_void_p]
        L.orc_step.restype = C.c_int
        L.orc_step.argtypes = [C.c_void_p, C.c_int, C.c_void_p, C.c_void_p]
        L.orc_get_state.argtypes = [C.c_void_p, C.c_void_p, C.c_void_p]
        L.orc_set_state.restype = C.c_int
        L.orc_set_state.argtypes = [C.c_void_p, C.c_int, C.c_void_p, C.c_void_p,
                                    C.c_void_p, C.c_void_p]
        _lib = L
    return _lib


def _dp(a: np.ndarray):
    assert a.dtype == np.float64 and a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(_D)


def _vp(a):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(C.c_void_p)


# ---- primitive wrappers (numpy in, numpy out) ----------------------------

def set_threads(n: int):
    """OpenMP threads for the oracle's GEMV rows (n <= 0: all cores)."""
    lib().orc_set_threads(int(n))


def sigmoid(x): return lib().orc_sigmoid(float(x))
def softplus(x): return lib().orc_softplus(float(x))
def silu(x): return lib().orc_silu(float(x))
def bf16_round(x): return lib().orc_double_to_bf16(float(x))
def bf16_value(b): return lib().orc_bf16_to_double(int(b))


def gemv(W_bits: np.ndarray, x: np.ndarray) -> np.ndarray:
    W_bits = np.ascontiguousarray(W_bits, dtype=np.uint16)
    x = np.ascontiguousarray(x, dtype=np.float64)
    y = np.zeros(W_bits.shape[0], np.float64)
    lib().orc_gemv(_vp(W_bits), W_bits.shape[0], W_bits.shape[1], _dp(x), _dp(y))
    return y


def quantize_w4(W_bits: np.ndarray):
    """4-bit group-wise codes (uint8 [rows][cols/2]) and scales (float32
    [rows][cols/64]) of a bf16 matrix given as uint16 bits."""
    W_bits = np.ascontiguousarray(W_bits, dtype=np.uint16)
    rows, cols = W_bits.shape
    if cols % 64:
        raise ValueError("cols must be a multiple of 64")
    codes = np.zeros((rows, cols // 2), dtype=np.uint8)
    scales = np.zeros((rows, cols // 64), dtype=np.float32)
    lib().orc_quantize_w4(_vp(W_bits), rows, cols, _vp(codes), _vp(scales))
    return codes, scales


def dequantize_w4(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.float32)
    rows, half = codes.shape
    Wd = np.zeros((rows, 2 * half), dtype=np.float64)
    lib().orc_dequantize_w4(_vp(codes), _vp(scales), rows, 2 * half, _dp(Wd))
    return Wd


def gemv_w4(codes: np.ndarray, scales: np.ndarray, x: np.ndarray) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.float32)
    rows, half = codes.shape
    x = np.ascontiguousarray(x, dtype=np.float64)
    y = np.zeros(rows, dtype=np.float64)
    lib().orc_gemv_w4(_vp(codes), _vp(scales), rows, 2 * half, _dp(x), _dp(y))
    return y


def rmsnorm(x, w_bits=None, eps=1e-6):
    x = np.ascontiguousarray(x, dtype=np.float64)
    y = np.zeros_like(x)
    wb = None if w_bits is None else np.ascontiguousarray(w_bits, dtype=np.uint16)
    lib().orc_rmsnorm(_dp(x), _vp(wb), x.size, eps, _dp(y))
    return y


def l2norm(x, eps=1e-6):
    x = np.ascontiguousarray(x, dtype=np.float64)
    y = np.zeros_like(x)
    lib().orc_l2norm(_dp(x), x.size, eps, _dp(y))
    return y


def conv_step(w_bits, state, u):
    """One causal-conv step; state [ch][K-1] is updated in place."""
    w_bits = np.ascontiguousarray(w_bits, dtype=np.uint16)
    ch, K = w_bits.shape
    assert state.dtype == np.float64 and state.shape == (ch, K - 1)
    u = np.ascontiguousarray(u, dtype=np.float64)
    out = np.zeros(ch, np.float64)
    lib().orc_causal_conv_step(ch, K, _vp(w_bits), _dp(state), _dp(u), _dp(out))
    return out


def delta_step(S, q, k, v, alpha, beta):
    """One gated delta step; S [dv][dk] float64 is updated in place."""
    dv, dk = S.shape
    q = np.ascontiguousarray(q, dtype=np.float64)
    k = np.ascontiguousarray(k, dtype=np.float64)
    v = np.ascontiguousarray(v, dtype=np.float64)
    o = np.zeros(dv, np.float64)
    lib().orc_gated_delta_step(dk, dv, _dp(S), _dp(q), _dp(k), _dp(v),
                               float(alpha), float(beta), _dp(o))
    return o


def delta_sequence(S, q, k, v, alpha, beta):
    """steps consecutive gated delta steps; S updated in place; returns o."""
    dv, dk = S.shape
    steps = q.shape[0]
    q = np.ascontiguousarray(q, dtype=np.float64)
    k = np.ascontiguousarray(k, dtype=np.float64)
    v = np.ascontiguousarray(v, dtype=np.float64)
    a = np.ascontiguousarray(alpha, dtype=np.float64)
    b = np.ascontiguousarray(beta, dtype=np.float64)
    o = np.zeros((steps, dv), np.float64)
    lib().orc_delta_sequence(dk, dv, steps, _dp(S), _dp(q), _dp(k), _dp(v),
                             _dp(a), _dp(b), _dp(o))
    return o


def rope(x, pos, theta):
    x = np.array(x, dtype=np.float64, copy=True)
    lib().orc_rope(_dp(x), x.size, int(pos), float(theta))
    return x


def softmax(s):
    s = np.ascontiguousarray(s, dtype=np.float64)
    p = np.zeros_like(s)
    lib().orc_softmax(_dp(s), s.size, _dp(p))
    return p


def attention_head(q, K, V):
    q = np.ascontiguousarray(q, dtype=np.float64)
    K = np.ascontiguousarray(K, dtype=np.float64)
    V = np.ascontiguousarray(V, dtype=np.float64)
    o = np.zeros(q.size, np.float64)
    lib().orc_attention_head(_dp(q), _dp(K), _dp(V), K.shape[0], q.size, _dp(o))
    return o


# ---- the model ------------------------------------------------------------

class OracleModel:
    """fp64 reference model over weights from ``synth.make_weights``."""

    def __init__(self, cfg, weights, _handle=None):
        self.cfg = cfg
        self.weights = weights          # keeps the numpy buffers alive
        L = lib()
        c = OrcConfig()
        c.n_layers = cfg.n_layers
        for i, a in enumerate(cfg.layer_is_attn):
            c.layer_is_attn[i] = 1 if a else 0
        c.hidden, c.vocab, c.mlp = cfg.hidden, cfg.vocab, cfg.mlp
        c.dn_heads, c.dn_dk, c.dn_dv, c.conv_k = (cfg.dn_heads, cfg.dn_dk,
                                                  cfg.dn_dv, cfg.conv_k)
        c.q_heads, c.kv_heads, c.head_dim = cfg.q_heads, cfg.kv_heads, cfg.head_dim
        c.rope_theta, c.rms_eps, c.max_ctx = cfg.rope_theta, cfg.rms_eps, cfg.max_ctx
        self._c = c
        layers = (OrcLayer * cfg.n_layers)()
        for i, d in enumerate(weights["layers"]):
            for name, _ in OrcLayer._fields_:
                if name in d:
                    setattr(layers[i], name, d[name].ctypes.data)
        self._layers = layers
        if _handle is None:
            _handle = L.orc_create(C.byref(c), layers, _vp(weights["embed"]),
                                   _vp(weights["final_norm"]))
            if not _handle:
                raise ValueError("oracle rejected the config")
        self._h = _handle

    def __del__(self):
        h = getattr(self, "_h", None)
        if h and _lib is not None:  # not during interpreter shutdown
            _lib.orc_destroy(h)
            self._h = None

    def clone(self) -> "OracleModel":
        h = lib().orc_clone(self._h)
        return OracleModel(self.cfg, self.weights, _handle=h)

    def reset(self):
        lib().orc_reset(self._h)

    @property
    def pos(self) -> int:
        return lib().orc_pos(self._h)

    def step(self, token: int, want_logits=True, want_hidden=False):
        cfg = self.cfg
        logits = np.zeros(cfg.vocab, np.float64) if want_logits else None
        hidden = (np.zeros((cfg.n_layers, cfg.hidden), np.float64)
                  if want_hidden else None)
        rc = lib().orc_step(self._h, int(token), _vp(logits), _vp(hidden))
        if rc != 0:
            raise ValueError("oracle step rejected (context full or bad token)")
        return logits, hidden

    def get_state(self):
        cfg = self.cfg
        dn = np.zeros((cfg.n_dn, cfg.dn_heads, cfg.dn_dv, cfg.dn_dk), np.float64)
        conv = np.zeros((cfg.n_dn, cfg.conv_channels, cfg.conv_k - 1), np.float64)
        lib().orc_get_state(self._h, _vp(dn), _vp(conv))
        return dn, conv

    def set_state(self, st):
        dn = np.ascontiguousarray(st["dn_state"], dtype=np.float32)
        conv = np.ascontiguousarray(st["conv_state"], dtype=np.float32)
        kc = np.ascontiguousarray(st["k_cache"], dtype=np.uint16)
        vc = np.ascontiguousarray(st["v_cache"], dtype=np.uint16)
        rc = lib().orc_set_state(self._h, int(st["pos"]), _vp(dn), _vp(conv),
                                 _vp(kc), _vp(vc))
        if rc != 0:
            raise ValueError("oracle rejected the state")
