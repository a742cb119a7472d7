"""Python binding of the single-launch decode engine (include/mk.h).

The functions below carry the C ABI's names and only marshal arguments:
every step of the forward pass runs in the CUDA kernels of ``libmk.so``.
PyTorch provides device memory and the current stream.  There is no CPU
fallback: without the built library every call raises.
"""
from __future__ import annotations

import ctypes as C
import os
import re
from typing import Dict, Optional

import numpy as np

from . import synth

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmk.so")
HEADER = os.path.join(os.path.dirname(_PKG), "include", "mk.h")
MAX_LAYERS = 64

MK_OK, MK_ERR_ARG, MK_ERR_CTX_OVERFLOW, MK_ERR_STATE = 0, 1, 2, 3
MK_ERR_LAUNCH, MK_ERR_TIMEOUT, MK_ERR_CUDA, MK_ERR_UNSUPPORTED = 4, 5, 6, 7
MK_ERR_RANGE = 8


class MkError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__("%s: %s (status %d)" % (what, mk_strerror(code), code))


class mk_config(C.Structure):
    _fields_ = [("n_layers", C.c_int32), ("layer_is_attn", C.c_uint8 * MAX_LAYERS),
                ("hidden", C.c_int32), ("vocab", C.c_int32), ("mlp", C.c_int32),
                ("dn_heads", C.c_int32), ("dn_dk", C.c_int32), ("dn_dv", C.c_int32),
                ("conv_k", C.c_int32), ("q_heads", C.c_int32), ("kv_heads", C.c_int32),
                ("head_dim", C.c_int32), ("rope_theta", C.c_float), ("rms_eps", C.c_float),
                ("max_ctx", C.c_int32), ("max_verify", C.c_int32)]


_LAYER_FIELDS = ("attn_norm", "in_proj", "conv_w", "A_log", "dt_bias", "out_norm",
                 "out_proj", "w_q", "w_k", "w_v", "w_o", "mlp_norm", "w_gate", "w_up",
                 "w_down")


class mk_layer_weights(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in _LAYER_FIELDS]


class mk_weights(C.Structure):
    _fields_ = [("embed", C.c_void_p), ("final_norm", C.c_void_p),
                ("layers", C.POINTER(mk_layer_weights))]


_lib = None


def lib():
    """Load libmk.so; raise if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("the CUDA engine library %s is not built; run "
                               "attention_decode_megakernel_b200.build.build()" % LIB_PATH)
        L = C.CDLL(LIB_PATH)
        vp, i32, i64, sz = C.c_void_p, C.c_int32, C.c_int64, C.c_size_t
        sig = {
            "mk_workspace_bytes": (sz, [C.POINTER(mk_config)]),
            "mk_create": (C.c_int, [C.POINTER(mk_config), C.POINTER(mk_weights), vp, sz, vp,
                                    C.POINTER(vp)]),
            "mk_destroy": (None, [vp]),
            "mk_reset": (C.c_int, [vp]),
            "mk_prefill": (C.c_int, [vp, vp, C.c_int, vp]),
            "mk_decode_step": (C.c_int, [vp, i32, vp]),
            "mk_generate": (C.c_int, [vp, i32, C.c_int, vp, vp]),
            "mk_verify": (C.c_int, [vp, vp, C.c_int, vp]),
            "mk_accept": (C.c_int, [vp, C.c_int]),
            "mk_position": (C.c_int, [vp]),
            "mk_sync": (C.c_int, [vp]),
            "mk_last_argmax": (i32, [vp]),
            "mk_set_state": (C.c_int, [vp, C.c_int, vp, vp, vp, vp]),
            "mk_get_state": (C.c_int, [vp, vp, vp, vp, vp]),
            "mk_get_hidden": (C.c_int, [vp, vp]),
            "mk_launch_count": (i64, [vp]),
            "mk_debug_set_wait_limit": (C.c_int, [vp, i64, C.c_int]),
            "mk_delta_step": (C.c_int, [vp, vp, vp, vp, vp, vp, vp, C.c_int, C.c_int,
                                        C.c_int, C.c_int, vp]),
            "mk_delta_chunked_ws_bytes": (sz, [C.c_int, C.c_int, C.c_int]),
            "mk_delta_chunked": (C.c_int, [vp, vp, vp, vp, vp, vp, vp, C.c_int, C.c_int,
                                           C.c_int, C.c_int, vp, sz, vp]),
            "mk_debug_gemm": (C.c_int, [vp, vp, vp, C.c_int, C.c_int, C.c_int, vp]),
            "mk_debug_gemm_noalloc": (C.c_int, [vp, vp, vp, C.c_int, C.c_int, C.c_int, vp]),
            "mk_quantize_w4": (C.c_int, [vp, C.c_int, C.c_int, vp, vp, vp]),
            "mk_gemv_w4": (C.c_int, [vp, vp, vp, C.c_int, C.c_int, C.c_int, vp, vp]),
            "mk_strerror": (C.c_char_p, [C.c_int]),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def header_symbols():
    """Names of the functions include/mk.h declares."""
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mk_[a-z_0-9]+)\s*\(", text)))


def mk_strerror(code: int) -> str:
    return lib().mk_strerror(int(code)).decode()


def _check(rc: int, what: str):
    if rc != MK_OK:
        raise MkError(rc, what)


def make_config(cfg: synth.ModelConfig) -> mk_config:
    c = mk_config()
    c.n_layers = cfg.n_layers
    for i, a in enumerate(cfg.layer_is_attn):
        c.layer_is_attn[i] = 1 if a else 0
    c.hidden, c.vocab, c.mlp = cfg.hidden, cfg.vocab, cfg.mlp
    c.dn_heads, c.dn_dk, c.dn_dv, c.conv_k = cfg.dn_heads, cfg.dn_dk, cfg.dn_dv, cfg.conv_k
    c.q_heads, c.kv_heads, c.head_dim = cfg.q_heads, cfg.kv_heads, cfg.head_dim
    c.rope_theta, c.rms_eps = cfg.rope_theta, cfg.rms_eps
    c.max_ctx, c.max_verify = cfg.max_ctx, cfg.max_verify
    return c


def mk_workspace_bytes(cfg: synth.ModelConfig) -> int:
    return int(lib().mk_workspace_bytes(C.byref(make_config(cfg))))


def _ptr(t) -> Optional[int]:
    return None if t is None else int(t.data_ptr())


def upload_weights(cfg: synth.ModelConfig, w: Dict, device="cuda"):
    """Pack the numpy weights into one device blob (128-byte aligned
    tensors) with a single host->device copy.  Returns (blob, offsets)."""
    import torch
    items = [("embed", w["embed"]), ("final_norm", w["final_norm"])]
    for l, d in enumerate(w["layers"]):
        for name in _LAYER_FIELDS:
            if name in d:
                items.append(("%d.%s" % (l, name), d[name]))
    offs, total = {}, 0
    for name, arr in items:
        offs[name] = total
        total += (arr.nbytes + 127) // 128 * 128
    blob = np.zeros(total, np.uint8)
    for name, arr in items:
        blob[offs[name]:offs[name] + arr.nbytes] = np.ascontiguousarray(arr).view(np.uint8).ravel()
    dev = torch.from_numpy(blob).to(device)
    return dev, offs


class Engine:
    """One engine over device-resident weights; every method is a C-ABI call."""

    def __init__(self, cfg: synth.ModelConfig, weights: Dict, device="cuda"):
        import torch
        self.cfg = cfg
        self.torch = torch
        self.blob, offs = upload_weights(cfg, weights, device)
        base = self.blob.data_ptr()
        self._layers = (mk_layer_weights * cfg.n_layers)()
        for l, d in enumerate(weights["layers"]):
            for name in _LAYER_FIELDS:
                key = "%d.%s" % (l, name)
                if key in offs:
                    setattr(self._layers[l], name, base + offs[key])
        self._w = mk_weights(base + offs["embed"], base + offs["final_norm"], self._layers)
        self._cfg = make_config(cfg)
        nbytes = int(lib().mk_workspace_bytes(C.byref(self._cfg)))
        if nbytes == 0:
            raise MkError(MK_ERR_ARG, "mk_workspace_bytes")
        self.ws = torch.empty(nbytes, dtype=torch.uint8, device=device)
        self.stream = torch.cuda.current_stream(self.ws.device)
        h = C.c_void_p()
        _check(lib().mk_create(C.byref(self._cfg), C.byref(self._w), self.ws.data_ptr(), nbytes,
                               self.stream.cuda_stream, C.byref(h)), "mk_create")
        self._h = h

    def close(self):
        if getattr(self, "_h", None):
            lib().mk_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # -- calls ----------------------------------------------------------------
    def reset(self):
        _check(lib().mk_reset(self._h), "mk_reset")

    @property
    def position(self) -> int:
        return lib().mk_position(self._h)

    def sync(self):
        _check(lib().mk_sync(self._h), "mk_sync")

    def prefill(self, tokens, logits=None):
        t = np.ascontiguousarray(tokens, dtype=np.int32)
        _check(lib().mk_prefill(self._h, t.ctypes.data, int(t.size), _ptr(logits)), "mk_prefill")

    def decode_step(self, token: int, logits=None):
        _check(lib().mk_decode_step(self._h, int(token), _ptr(logits)), "mk_decode_step")

    def generate(self, first_token: int, n: int, tokens_out, logits=None):
        _check(lib().mk_generate(self._h, int(first_token), int(n), _ptr(tokens_out),
                                 _ptr(logits)), "mk_generate")

    def verify(self, tokens, logits):
        t = np.ascontiguousarray(tokens, dtype=np.int32)
        _check(lib().mk_verify(self._h, t.ctypes.data, int(t.size), _ptr(logits)), "mk_verify")

    def accept(self, n_keep: int):
        _check(lib().mk_accept(self._h, int(n_keep)), "mk_accept")

    def last_argmax(self) -> int:
        return int(lib().mk_last_argmax(self._h))

    def launch_count(self) -> int:
        return int(lib().mk_launch_count(self._h))

    def set_wait_limit(self, ns: int, fail_phase: int = -1):
        _check(lib().mk_debug_set_wait_limit(self._h, int(ns), int(fail_phase)),
               "mk_debug_set_wait_limit")

    def set_state(self, st: Dict):
        """st: device tensors dn_state f32, conv_state f32, k_cache/v_cache
        (16-bit bf16 patterns), plus 'pos'."""
        _check(lib().mk_set_state(self._h, int(st["pos"]), _ptr(st["dn_state"]),
                                  _ptr(st["conv_state"]), _ptr(st.get("k_cache")),
                                  _ptr(st.get("v_cache"))), "mk_set_state")

    def get_state(self, with_kv=False):
        torch, cfg = self.torch, self.cfg
        dev = self.ws.device
        dn = torch.empty((cfg.n_dn, cfg.dn_heads, cfg.dn_dv, cfg.dn_dk), dtype=torch.float32,
                         device=dev)
        conv = torch.empty((cfg.n_dn, cfg.conv_channels, cfg.conv_k - 1), dtype=torch.float32,
                           device=dev)
        kc = vc = None
        if with_kv:
            shape = (cfg.n_attn, cfg.kv_heads, self.position, cfg.head_dim)
            kc = torch.empty(shape, dtype=torch.int16, device=dev)
            vc = torch.empty(shape, dtype=torch.int16, device=dev)
        _check(lib().mk_get_state(self._h, _ptr(dn), _ptr(conv), _ptr(kc), _ptr(vc)),
               "mk_get_state")
        return dn, conv, kc, vc

    def get_hidden(self):
        torch, cfg = self.torch, self.cfg
        h = torch.empty((cfg.n_layers, cfg.hidden), dtype=torch.float32, device=self.ws.device)
        _check(lib().mk_get_hidden(self._h, _ptr(h)), "mk_get_hidden")
        return h


def mk_delta_step(S, q, k, v, alpha, beta, o, stream=None):
    """Isolated gated delta step (in place on S) through the C ABI."""
    B, heads, dv, dk = S.shape
    st = stream if stream is not None else 0
    _check(lib().mk_delta_step(_ptr(S), _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta),
                               _ptr(o), int(B), int(heads), int(dk), int(dv), st),
           "mk_delta_step")


def mk_delta_chunked(S, q, k, v, alpha, beta, o, workspace=None, stream=None):
    """The gated delta rule over T positions in chunkwise form (in place on
    S [heads][dv][dk]); q, k [heads][T][dk], v and o [heads][T][dv], alpha,
    beta [heads][T], all float32 device tensors.  `workspace` (a device
    tensor) may be given; otherwise one is allocated with torch."""
    heads, dv, dk = S.shape
    T = q.shape[1]
    need = lib().mk_delta_chunked_ws_bytes(int(T), int(heads), int(dk))
    if need == 0:
        raise MkError(MK_ERR_ARG, "mk_delta_chunked_ws_bytes")
    if workspace is None:
        import torch
        workspace = torch.empty(need, dtype=torch.uint8, device=S.device)
    st = stream if stream is not None else 0
    _check(lib().mk_delta_chunked(_ptr(S), _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta),
                                  _ptr(o), int(T), int(heads), int(dk), int(dv), _ptr(workspace),
                                  int(workspace.numel() * workspace.element_size()), st),
           "mk_delta_chunked")


def mk_debug_gemm(W, X, Cout, stream=None):
    """C = X W^T on the prompt path's tensor-core GEMM (bf16 in, fp32 out)."""
    n_out, K = W.shape
    if X.numel() % (2 * K):
        raise ValueError("X must hold [2][T][K] bf16 (hi then lo operands)")
    T = X.numel() // (2 * K)
    if Cout.numel() != T * n_out:
        raise ValueError("C must hold [T][n_out] float32")
    st = stream if stream is not None else 0
    _check(lib().mk_debug_gemm(_ptr(W), _ptr(X), _ptr(Cout), int(n_out), int(T), int(K), st),
           "mk_debug_gemm")


def mk_debug_gemm_noalloc(W, X, Cout, stream=None):
    """mk_debug_gemm through the allocation-free entry point (static scratch)."""
    n_out, K = W.shape
    if X.numel() % (2 * K):
        raise ValueError("X must hold [2][T][K] bf16 (hi then lo operands)")
    T = X.numel() // (2 * K)
    if Cout.numel() != T * n_out:
        raise ValueError("C must hold [T][n_out] float32")
    st = stream if stream is not None else 0
    _check(lib().mk_debug_gemm_noalloc(_ptr(W), _ptr(X), _ptr(Cout), int(n_out), int(T), int(K),
                                       st), "mk_debug_gemm_noalloc")


def quantize_w4(W, codes, scales, stream=None):
    """4-bit group-wise quantisation of W (bf16 bits [rows][cols] as an int16
    device tensor) into codes (uint8 [rows][cols / 2]) and scales (float32
    [rows][cols / 64]), device tensors the caller provides."""
    rows, cols = W.shape
    if codes.numel() != rows * cols // 2 or scales.numel() != rows * cols // 64:
        raise ValueError("codes must hold [rows][cols/2] bytes, scales [rows][cols/64] floats")
    st = stream if stream is not None else 0
    _check(lib().mk_quantize_w4(_ptr(W), int(rows), int(cols), _ptr(codes), _ptr(scales), st),
           "mk_quantize_w4")


def gemv_w4(codes, scales, x, y, stream=None):
    """y [T][rows] = x [T][cols] times the dequantised 4-bit weights, transposed."""
    T, cols = x.shape
    rows = codes.numel() * 2 // cols
    if y.numel() != T * rows or scales.numel() != rows * cols // 64:
        raise ValueError("y must hold [T][rows] floats and scales [rows][cols/64]")
    st = stream if stream is not None else 0
    _check(lib().mk_gemv_w4(_ptr(codes), _ptr(scales), _ptr(x), int(T), int(rows), int(cols),
                            _ptr(y), st), "mk_gemv_w4")
