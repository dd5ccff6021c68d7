"""CPU oracle for the routed sigmoid top-k MoE FFN (TEST INFRASTRUCTURE).

Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's
``cpu_baseline`` / ``--impl reference`` legs may import this package.  The
product path (``mixture_experts_routed_sigmoid_b200``) never imports it, and
this package never imports the product path: they share only the seeded input
generator module ``moe_inputs``, which holds no arithmetic of the method.

The arithmetic lives in ``moe_oracle.c`` (plain C, f64 accumulation over
bf16-valued inputs, OpenMP over tokens).  This file builds it with gcc and
marshals numpy arrays through ctypes.  Sources followed (page title and item):

* mlx-native 0.13.0, ``src/ops/dense_matmul_id_auto.rs``: ``DenseMatmulIdShape``,
  input layouts, routing profiles, the Direct/Grouped dispatch pair.
* cortiq-engine 0.7.7, ``src/mimo_moe.rs``: module doc (top-8 sigmoid +
  selection-bias routing), ``Dynamic::run`` (combine weight ``p[e]/wsum``),
  ``tests::exact_moe`` (f64 reference), ``tests::rel`` (error metric).
* hf2q 0.1.1, ``eagle3/forward.rs``: SwiGLU MLP ``down(silu(gate(x))*up(x))``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "moe_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libmoe_oracle.so")
_lock = threading.Lock()
_default = None


def compile_source(src: str, out_path: str) -> str:
    """gcc a C source file into a shared library (IEEE f64, no fast-math)."""
    tmp = out_path + ".tmp%d" % os.getpid()
    subprocess.check_call(
        ["gcc", "-O2", "-fopenmp", "-fno-fast-math", "-ffp-contract=off", "-std=c11",
         "-shared", "-fPIC", "-o", tmp, src, "-lm"])
    os.replace(tmp, out_path)
    return out_path


def build(force: bool = False) -> str:
    """Compile ``libmoe_oracle.so`` next to its source if it is stale."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(SOURCE):
        compile_source(SOURCE, _LIB_PATH)
    return _LIB_PATH


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


class Oracle:
    """ctypes front of one build of the oracle library."""

    def __init__(self, lib_path: str):
        lib = ctypes.CDLL(lib_path)
        P = ctypes.c_void_p
        i32 = ctypes.c_int32
        lib.oracle_route.argtypes = [P, P, i32, i32, i32, P, P, P]
        lib.oracle_route.restype = None
        lib.oracle_router_logits.argtypes = [P, P, P, i32, i32, i32]
        lib.oracle_router_logits.restype = None
        lib.oracle_route_weights.argtypes = [P, P, i32, i32, i32, P]
        lib.oracle_route_weights.restype = None
        lib.oracle_expert_map.argtypes = [P, i32, i32, i32, P, P, P, P]
        lib.oracle_expert_map.restype = ctypes.c_int
        lib.oracle_matmul_id.argtypes = [P, P, P, P, i32, i32, i32, i32, i32, i32]
        lib.oracle_matmul_id.restype = None
        lib.oracle_ffn.argtypes = [P, P, P, P, P, P, P, i32, i32, i32, i32, i32, i32, i32, P, i32]
        lib.oracle_ffn.restype = None
        lib.oracle_ffn_shared.argtypes = [P] * 11 + [i32] * 6 + [i32, P, i32]
        lib.oracle_ffn_shared.restype = None
        lib.oracle_sigmoid_f32.argtypes = [ctypes.c_float]
        lib.oracle_sigmoid_f32.restype = ctypes.c_float
        self.lib = lib

    def sigmoid_f32(self, logit: float) -> float:
        """sigmoid in f64, rounded once to f32 (the routing score s)."""
        return float(self.lib.oracle_sigmoid_f32(ctypes.c_float(logit)))

    def route(self, logits: np.ndarray, bias: np.ndarray | None, top_k: int):
        """Sigmoid + selection-bias top-k routing.

        Returns ``(ids int32 [m, top_k], weights f32 [m, top_k], scores f32 [m, E])``.
        """
        logits = _c(logits, np.float32)
        m, n_experts = logits.shape
        b = None if bias is None else _c(bias, np.float32)
        ids = np.zeros((m, top_k), np.int32)
        weights = np.zeros((m, top_k), np.float32)
        scores = np.zeros((m, n_experts), np.float32)
        self.lib.oracle_route(_ptr(logits), None if b is None else _ptr(b), m, n_experts, top_k,
                              _ptr(ids), _ptr(weights), _ptr(scores))
        return ids, weights, scores

    def router_logits(self, x_bits: np.ndarray, W_bits: np.ndarray):
        """``x @ W_router.T`` in f64 over bf16 inputs: ``[m, hidden] x [E, hidden] -> [m, E]``."""
        x_bits = _c(x_bits, np.uint16)
        W_bits = _c(W_bits, np.uint16)
        m, hidden = x_bits.shape
        n_experts = W_bits.shape[0]
        assert W_bits.shape[1] == hidden
        out = np.zeros((m, n_experts), np.float64)
        self.lib.oracle_router_logits(_ptr(x_bits), _ptr(W_bits), _ptr(out), m, hidden, n_experts)
        return out

    def route_weights(self, logits: np.ndarray, ids: np.ndarray):
        """Combine weights ``s[ids[t,j]] / sum_j s[ids[t,j]]`` for caller-fixed ids."""
        logits = _c(logits, np.float32)
        ids = _c(ids, np.int32)
        m, n_experts = logits.shape
        top_k = ids.shape[1]
        weights = np.zeros((m, top_k), np.float32)
        self.lib.oracle_route_weights(_ptr(logits), _ptr(ids), m, n_experts, top_k, _ptr(weights))
        return weights

    def expert_map(self, ids: np.ndarray, n_experts: int):
        """Stable counting sort of routed rows by expert id.

        Returns ``(counts [E], offsets [E+1], perm [R], inv_perm [R])`` as int32.
        """
        ids = _c(ids, np.int32)
        m, top_k = ids.shape
        rows = m * top_k
        counts = np.zeros(n_experts, np.int32)
        offsets = np.zeros(n_experts + 1, np.int32)
        perm = np.zeros(rows, np.int32)
        inv = np.zeros(rows, np.int32)
        rc = self.lib.oracle_expert_map(_ptr(ids), m, top_k, n_experts, _ptr(counts),
                                        _ptr(offsets), _ptr(perm), _ptr(inv))
        if rc != 0:
            raise ValueError("expert id out of range")
        return counts, offsets, perm, inv

    def matmul_id(self, x_bits: np.ndarray, ids: np.ndarray, W_bits: np.ndarray, layout: int = 0):
        """``y[t, j] = W[ids[t, j]] @ x_row(t, j)`` in f64 over bf16 inputs.

        ``x_bits``: uint16 bf16 bits, ``[m, k]`` (layout 0) or ``[m, top_k, k]``
        (layout 1); ``W_bits``: uint16 ``[E, n, k]``.  Returns f64 ``[m, top_k, n]``.
        """
        ids = _c(ids, np.int32)
        m, top_k = ids.shape
        n_experts, n, k = W_bits.shape
        x_bits = _c(x_bits, np.uint16)
        W_bits = _c(W_bits, np.uint16)
        assert x_bits.shape[-1] == k
        y = np.zeros((m, top_k, n), np.float64)
        self.lib.oracle_matmul_id(_ptr(x_bits), _ptr(ids), _ptr(W_bits), _ptr(y), m, n, k, top_k,
                                  n_experts, layout)
        return y

    def ffn(self, x_bits, ids, weights, Wg_bits, Wu_bits, Wd_bits, layout: int = 0,
            tokens=None, act_mode: int = 0):
        """Routed SwiGLU MoE FFN in f64 for the given tokens (default: all).

        Returns f64 ``[len(tokens), hidden]``.
        """
        ids = _c(ids, np.int32)
        m, top_k = ids.shape
        n_experts, inter, hidden = Wg_bits.shape
        assert Wd_bits.shape == (n_experts, hidden, inter)
        weights = _c(weights, np.float32)
        args = [_c(x_bits, np.uint16), ids, weights, _c(Wg_bits, np.uint16),
                _c(Wu_bits, np.uint16), _c(Wd_bits, np.uint16)]
        tok = None if tokens is None else _c(tokens, np.int32)
        nt = m if tok is None else len(tok)
        y = np.zeros((nt, hidden), np.float64)
        self.lib.oracle_ffn(*[_ptr(a) for a in args], _ptr(y), m, hidden, inter, top_k,
                            n_experts, layout, act_mode, None if tok is None else _ptr(tok), nt)
        return y

    def ffn_shared(self, x_bits, ids, weights, Wg_bits, Wu_bits, Wd_bits, w_sh_bits,
                   Wsg_bits, Wsu_bits, Wsd_bits, tokens=None, act_mode: int = 0):
        """Routed FFN plus the sigmoid-gated shared expert, f64, for the given
        tokens (default: all); x is one row per token.  Returns ``[len(tokens), hidden]``."""
        ids = _c(ids, np.int32)
        m, top_k = ids.shape
        n_experts, inter, hidden = Wg_bits.shape
        inter_sh = Wsg_bits.shape[0]
        assert Wsg_bits.shape == Wsu_bits.shape == (inter_sh, hidden)
        assert Wsd_bits.shape == (hidden, inter_sh) and w_sh_bits.shape == (hidden,)
        args = [_c(x_bits, np.uint16), ids, _c(weights, np.float32), _c(Wg_bits, np.uint16),
                _c(Wu_bits, np.uint16), _c(Wd_bits, np.uint16), _c(w_sh_bits, np.uint16),
                _c(Wsg_bits, np.uint16), _c(Wsu_bits, np.uint16), _c(Wsd_bits, np.uint16)]
        tok = None if tokens is None else _c(tokens, np.int32)
        nt = m if tok is None else len(tok)
        y = np.zeros((nt, hidden), np.float64)
        self.lib.oracle_ffn_shared(*[_ptr(a) for a in args], _ptr(y), m, hidden, inter, inter_sh,
                                   top_k, n_experts, act_mode,
                                   None if tok is None else _ptr(tok), nt)
        return y

    @staticmethod
    def rel(a, b) -> float:
        """Error metric of cortiq-engine ``tests::rel``: ``max|a-b| / max|b|``."""
        a = np.asarray(a, np.float64)
        b = np.asarray(b, np.float64)
        d = np.abs(a - b)
        if np.isnan(d).any():
            return float("inf")
        return float(d.max(initial=0.0) / max(np.abs(b).max(initial=0.0), 1e-300))


def default() -> Oracle:
    global _default
    with _lock:
        if _default is None:
            _default = Oracle(build())
    return _default


def sigmoid_f32(logit):
    return default().sigmoid_f32(logit)


def route(logits, bias, top_k):
    return default().route(logits, bias, top_k)


def route_weights(logits, ids):
    return default().route_weights(logits, ids)


def router_logits(x_bits, W_bits):
    return default().router_logits(x_bits, W_bits)


def expert_map(ids, n_experts):
    return default().expert_map(ids, n_experts)


def matmul_id(x_bits, ids, W_bits, layout=0):
    return default().matmul_id(x_bits, ids, W_bits, layout)


def ffn(*args, **kwargs):
    return default().ffn(*args, **kwargs)


def ffn_shared(*args, **kwargs):
    return default().ffn_shared(*args, **kwargs)


rel = Oracle.rel
