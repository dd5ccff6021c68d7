"""Routed sigmoid top-k MoE FFN for one NVIDIA B200 (sm_100a).

Thin ctypes binding of the C-ABI library ``libmoe_b200.so`` (declared in
``include/moe_b200.h``).  Every step of the computation runs in the library's
CUDA kernels; this module only marshals torch tensors (device memory) and the
current CUDA stream into the C calls, and allocates outputs/workspaces with
torch when the caller does not pass them.  There is no CPU or PyTorch fallback:
if the library is missing or a call fails, an exception is raised.

Functions keep the C names:

* ``moe_route_topk(logits, bias, top_k)`` -> ``(ids, weights)``
* ``moe_router_topk(x, W_router, bias, top_k)`` -> ``(ids, weights, logits)``
* ``moe_route_weights(logits, ids)`` -> ``weights``
* ``moe_expert_map(ids, n_experts)`` -> ``(counts, offsets, perm, inv_perm)``
* ``moe_matmul_id(x, ids, W, layout=...)`` -> ``y [m, top_k, n]``
* ``moe_matmul_id_strided(x, ids, W_buf, expert_stride_bytes, n, k, n_experts)`` -> same,
  over a padded expert stack
* ``moe_ffn_forward(x, ids, weights, W_gate, W_up, W_down, layout=...)`` -> ``y [m, hidden]``
* ``moe_ffn_slots(x, ids, W_gate, W_up, W_down)`` -> unweighted per-slot rows ``[m, top_k, hidden]``
* ``moe_ffn_forward_shared(..., w_sh, W_sh_gate, W_sh_up, W_sh_down)`` -> the same plus the
  sigmoid-gated shared expert
* ``moe_ep_dispatch(x, ids, n_experts, n_ranks)`` / ``moe_ep_combine(d_back, weights, n_ranks, ws)``
  -> the device halves of an expert-parallel step (``ep.py`` drives the exchange)
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

SHARED_PER_TOKEN = 0
SLOTTED = 1

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")

STATUS = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARGUMENT", 2: "MOE_ERR_UNSUPPORTED_SHAPE",
          3: "MOE_ERR_WORKSPACE_TOO_SMALL", 4: "MOE_ERR_CUDA", 5: "MOE_ERR_DEVICE_TIMEOUT",
          6: "MOE_ERR_DEVICE_BAD_ID", 7: "MOE_ERR_DEVICE_RANGE"}

# Every exported symbol of include/moe_b200.h with its ctypes signature.
_P, _I32, _I64, _SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
SIGNATURES = {
    "moe_last_error": ([], ctypes.c_char_p),
    "moe_version": ([], ctypes.c_char_p),
    "moe_route_topk": ([_P, _P, _I32, _I32, _I32, _P, _P, _P, _P], ctypes.c_int),
    "moe_route_weights": ([_P, _P, _I32, _I32, _I32, _P, _P], ctypes.c_int),
    "moe_router_workspace": ([_I32, _I32, _I32], _SZ),
    "moe_router_topk": ([_P, _P, _P, _I32, _I32, _I32, _I32, _P, _P, _P, _P, _SZ, _P], ctypes.c_int),
    "moe_expert_map_workspace": ([_I32, _I32, _I32], _SZ),
    "moe_expert_map": ([_P, _I32, _I32, _I32, _P, _P, _P, _P, _P, _SZ, _P], ctypes.c_int),
    "moe_matmul_id_workspace": ([_I32, _I32, _I32, _I32, _I32, _I32], _SZ),
    "moe_matmul_id": ([_P, _P, _P, _P, _I32, _I32, _I32, _I32, _I32, _I32, _P, _SZ, _P],
                      ctypes.c_int),
    "moe_matmul_id_strided": ([_P, _P, _P, ctypes.c_uint64, _P, _I32, _I32, _I32, _I32, _I32, _I32,
                               _P, _SZ, _P], ctypes.c_int),
    "moe_ffn_workspace": ([_I32, _I32, _I32, _I32, _I32, _I32], _SZ),
    "moe_ffn_forward": ([_P, _P, _P, _P, _P, _P, _P, _I32, _I32, _I32, _I32, _I32, _I32, _P, _SZ,
                         _P], ctypes.c_int),
    "moe_ffn_slots": ([_P, _P, _P, _P, _P, _P, _I32, _I32, _I32, _I32, _I32, _I32, _P, _SZ, _P],
                      ctypes.c_int),
    "moe_ffn_shared_workspace": ([_I32, _I32, _I32, _I32, _I32, _I32], _SZ),
    "moe_ffn_forward_shared": ([_P] * 11 + [_I32] * 6 + [_P, _SZ, _P], ctypes.c_int),
    "moe_matmul_id_noalloc": ([_P, _P, _P, _P, _I32, _I32, _I32, _I32, _I32, _I32, _P],
                              ctypes.c_int),
    "moe_matmul_id_noalloc_status": ([_P], ctypes.c_int),
    "moe_ep_dispatch_workspace": ([_I32, _I32, _I32], _SZ),
    "moe_ep_dispatch": ([_P, _P, _I32, _I32, _I32, _I32, _I32, _I32, _P, _P, _P, _P, _SZ, _P],
                        ctypes.c_int),
    "moe_ep_combine": ([_P, _P, _P, _I32, _I32, _I32, _I32, _P, _SZ, _P], ctypes.c_int),
    "moe_set_stage_events": ([_P, _I32], ctypes.c_int),
    "moe_check_status": ([_P, _P], ctypes.c_int),
    "moe_clock_probe": ([_P, _I32, _P], ctypes.c_int),
    "moe_selftest_wait_timeout": ([_P, _I64, _P], ctypes.c_int),
}

_lock = threading.Lock()
_lib = None


class MoeError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS.get(status, status)}: {msg}")
        self.status = status


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the C-ABI library (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(path):
                raise RuntimeError(
                    f"{path} is missing: build it with "
                    "`python -m mixture_experts_routed_sigmoid_b200.build`")
            lib = ctypes.CDLL(path)
            for name, (args, res) in SIGNATURES.items():
                fn = getattr(lib, name)
                fn.argtypes = args
                fn.restype = res
            _lib = lib
    return _lib


def _check(status: int):
    if status != 0:
        raise MoeError(status, load_library().moe_last_error().decode())


def _stream(device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _ptr(t):
    return None if t is None else t.data_ptr()


def _require(t: torch.Tensor, name: str, dtype, device=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _workspace(nbytes: int, device) -> torch.Tensor:
    if nbytes == 0:
        raise MoeError(2, "shape rejected by the workspace query")
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def moe_route_topk(logits: torch.Tensor, bias: torch.Tensor | None, top_k: int,
                   ids: torch.Tensor | None = None, weights: torch.Tensor | None = None,
                   scores: torch.Tensor | None = None):
    """Sigmoid + selection-bias top-k routing; returns ``(ids, weights)``."""
    _require(logits, "logits", torch.float32)
    m, n_experts = logits.shape
    dev = logits.device
    if bias is not None:
        _require(bias, "bias", torch.float32, dev)
    if ids is None:
        ids = torch.empty((m, top_k), dtype=torch.int32, device=dev)
    if weights is None:
        weights = torch.empty((m, top_k), dtype=torch.float32, device=dev)
    _check(load_library().moe_route_topk(_ptr(logits), _ptr(bias), m, n_experts, top_k,
                                         _ptr(ids), _ptr(weights), _ptr(scores), _stream(dev)))
    return ids, weights


def moe_router_workspace(m: int, hidden: int, n_experts: int) -> int:
    return int(load_library().moe_router_workspace(m, hidden, n_experts))


def moe_router_topk(x: torch.Tensor, W_router: torch.Tensor, bias: torch.Tensor | None,
                    top_k: int, logits: torch.Tensor | None = None,
                    ids: torch.Tensor | None = None, weights: torch.Tensor | None = None,
                    ws: torch.Tensor | None = None):
    """Router projection ``x @ W_router.T`` then routing; returns ``(ids, weights, logits)``."""
    _require(x, "x", torch.bfloat16)
    dev = x.device
    _require(W_router, "W_router", torch.bfloat16, dev)
    if bias is not None:
        _require(bias, "bias", torch.float32, dev)
    m, hidden = x.shape
    n_experts = W_router.shape[0]
    if logits is None:
        logits = torch.empty((m, n_experts), dtype=torch.float32, device=dev)
    if ids is None:
        ids = torch.empty((m, top_k), dtype=torch.int32, device=dev)
    if weights is None:
        weights = torch.empty((m, top_k), dtype=torch.float32, device=dev)
    lib = load_library()
    if ws is None:
        ws = _workspace(int(lib.moe_router_workspace(m, hidden, n_experts)), dev)
    _check(lib.moe_router_topk(_ptr(x), _ptr(W_router), _ptr(bias), m, hidden, n_experts, top_k,
                               _ptr(logits), _ptr(ids), _ptr(weights), _ptr(ws), ws.numel(),
                               _stream(dev)))
    return ids, weights, logits


def moe_route_weights(logits: torch.Tensor, ids: torch.Tensor, weights: torch.Tensor | None = None):
    """Combine weights of caller-fixed ids."""
    _require(logits, "logits", torch.float32)
    _require(ids, "ids", torch.int32, logits.device)
    m, n_experts = logits.shape
    top_k = ids.shape[1]
    if weights is None:
        weights = torch.empty((m, top_k), dtype=torch.float32, device=logits.device)
    _check(load_library().moe_route_weights(_ptr(logits), _ptr(ids), m, n_experts, top_k,
                                            _ptr(weights), _stream(logits.device)))
    return weights


def moe_expert_map_workspace(m: int, top_k: int, n_experts: int) -> int:
    return int(load_library().moe_expert_map_workspace(m, top_k, n_experts))


def moe_expert_map(ids: torch.Tensor, n_experts: int, ws: torch.Tensor | None = None):
    """Per-expert counts, offsets and the stable expert-sorted permutation."""
    _require(ids, "ids", torch.int32)
    m, top_k = ids.shape
    dev = ids.device
    rows = m * top_k
    counts = torch.empty(n_experts, dtype=torch.int32, device=dev)
    offsets = torch.empty(n_experts + 1, dtype=torch.int32, device=dev)
    perm = torch.empty(rows, dtype=torch.int32, device=dev)
    inv = torch.empty(rows, dtype=torch.int32, device=dev)
    if ws is None:
        ws = _workspace(moe_expert_map_workspace(m, top_k, n_experts), dev)
    _check(load_library().moe_expert_map(_ptr(ids), m, top_k, n_experts, _ptr(counts),
                                         _ptr(offsets), _ptr(perm), _ptr(inv), _ptr(ws),
                                         ws.numel(), _stream(dev)))
    return counts, offsets, perm, inv


def moe_matmul_id_workspace(m, n, k, top_k, n_experts, layout=SHARED_PER_TOKEN) -> int:
    return int(load_library().moe_matmul_id_workspace(m, n, k, top_k, n_experts, layout))


def moe_matmul_id(x: torch.Tensor, ids: torch.Tensor, W: torch.Tensor,
                  layout: int = SHARED_PER_TOKEN, y: torch.Tensor | None = None,
                  ws: torch.Tensor | None = None):
    """``y[t, j] = W[ids[t, j]] @ x_row(t, j)``; returns f32 ``[m, top_k, n]``."""
    _require(x, "x", torch.bfloat16)
    dev = x.device
    _require(ids, "ids", torch.int32, dev)
    _require(W, "W", torch.bfloat16, dev)
    m, top_k = ids.shape
    n_experts, n, k = W.shape
    if y is None:
        y = torch.empty((m, top_k, n), dtype=torch.float32, device=dev)
    if ws is None:
        ws = _workspace(moe_matmul_id_workspace(m, n, k, top_k, n_experts, layout), dev)
    _check(load_library().moe_matmul_id(_ptr(x), _ptr(ids), _ptr(W), _ptr(y), m, n, k, top_k,
                                        n_experts, layout, _ptr(ws), ws.numel(), _stream(dev)))
    return y


def moe_matmul_id_strided(x: torch.Tensor, ids: torch.Tensor, W_buf: torch.Tensor,
                          expert_stride_bytes: int, n: int, k: int, n_experts: int,
                          layout: int = SHARED_PER_TOKEN, y: torch.Tensor | None = None,
                          ws: torch.Tensor | None = None):
    """``moe_matmul_id`` over a padded expert stack: expert ``e``'s ``[n, k]``
    bf16 matrix starts ``e * expert_stride_bytes`` bytes into the contiguous
    buffer ``W_buf`` (any dtype); returns f32 ``[m, top_k, n]``."""
    _require(x, "x", torch.bfloat16)
    dev = x.device
    _require(ids, "ids", torch.int32, dev)
    if not isinstance(W_buf, torch.Tensor) or not W_buf.is_cuda or W_buf.device != dev:
        raise ValueError(f"W_buf must be a CUDA tensor on {dev}")
    if not W_buf.is_contiguous():
        raise ValueError("W_buf must be contiguous")
    need = (n_experts - 1) * expert_stride_bytes + 2 * n * k
    have = W_buf.numel() * W_buf.element_size()
    if n_experts < 1 or have < need:
        raise ValueError(f"W_buf holds {have} bytes, the stack needs {need}")
    m, top_k = ids.shape
    if y is None:
        y = torch.empty((m, top_k, n), dtype=torch.float32, device=dev)
    if ws is None:
        ws = _workspace(moe_matmul_id_workspace(m, n, k, top_k, n_experts, layout), dev)
    _check(load_library().moe_matmul_id_strided(_ptr(x), _ptr(ids), _ptr(W_buf),
                                                expert_stride_bytes, _ptr(y), m, n, k, top_k,
                                                n_experts, layout, _ptr(ws), ws.numel(),
                                                _stream(dev)))
    return y


def moe_ffn_workspace(m, hidden, inter, top_k, n_experts, layout=SHARED_PER_TOKEN) -> int:
    return int(load_library().moe_ffn_workspace(m, hidden, inter, top_k, n_experts, layout))


def moe_ffn_forward(x: torch.Tensor, ids: torch.Tensor, weights: torch.Tensor,
                    W_gate: torch.Tensor, W_up: torch.Tensor, W_down: torch.Tensor,
                    layout: int = SHARED_PER_TOKEN, y: torch.Tensor | None = None,
                    ws: torch.Tensor | None = None):
    """Routed SwiGLU MoE FFN; returns f32 ``[m, hidden]``."""
    _require(x, "x", torch.bfloat16)
    dev = x.device
    _require(ids, "ids", torch.int32, dev)
    _require(weights, "weights", torch.float32, dev)
    for name, t in (("W_gate", W_gate), ("W_up", W_up), ("W_down", W_down)):
        _require(t, name, torch.bfloat16, dev)
    m, top_k = ids.shape
    n_experts, inter, hidden = W_gate.shape
    if y is None:
        y = torch.empty((m, hidden), dtype=torch.float32, device=dev)
    if ws is None:
        ws = _workspace(moe_ffn_workspace(m, hidden, inter, top_k, n_experts, layout), dev)
    _check(load_library().moe_ffn_forward(_ptr(x), _ptr(ids), _ptr(weights), _ptr(W_gate),
                                          _ptr(W_up), _ptr(W_down), _ptr(y), m, hidden, inter,
                                          top_k, n_experts, layout, _ptr(ws), ws.numel(),
                                          _stream(dev)))
    return y


def moe_check_status(ws: torch.Tensor) -> int:
    """Device status word of a workspace (synchronises the current stream)."""
    return int(load_library().moe_check_status(_ptr(ws), _stream(ws.device)))


def moe_ffn_slots(x: torch.Tensor, ids: torch.Tensor, W_gate: torch.Tensor, W_up: torch.Tensor,
                  W_down: torch.Tensor, layout: int = SHARED_PER_TOKEN,
                  d_slots: torch.Tensor | None = None, ws: torch.Tensor | None = None):
    """Unweighted per-slot down outputs before the combine; f32 ``[m, top_k, hidden]``."""
    _require(x, "x", torch.bfloat16)
    dev = x.device
    _require(ids, "ids", torch.int32, dev)
    for name, t in (("W_gate", W_gate), ("W_up", W_up), ("W_down", W_down)):
        _require(t, name, torch.bfloat16, dev)
    m, top_k = ids.shape
    n_experts, inter, hidden = W_gate.shape
    if d_slots is None:
        d_slots = torch.empty((m, top_k, hidden), dtype=torch.float32, device=dev)
    if ws is None:
        ws = _workspace(moe_ffn_workspace(m, hidden, inter, top_k, n_experts, layout), dev)
    _check(load_library().moe_ffn_slots(_ptr(x), _ptr(ids), _ptr(W_gate), _ptr(W_up), _ptr(W_down),
                                        _ptr(d_slots), m, hidden, inter, top_k, n_experts, layout,
                                        _ptr(ws), ws.numel(), _stream(dev)))
    return d_slots


def moe_ffn_shared_workspace(m, hidden, inter, inter_sh, top_k, n_experts) -> int:
    return int(load_library().moe_ffn_shared_workspace(m, hidden, inter, inter_sh, top_k,
                                                        n_experts))


def moe_ffn_forward_shared(x: torch.Tensor, ids: torch.Tensor, weights: torch.Tensor,
                           W_gate: torch.Tensor, W_up: torch.Tensor, W_down: torch.Tensor,
                           w_sh: torch.Tensor, W_sh_gate: torch.Tensor, W_sh_up: torch.Tensor,
                           W_sh_down: torch.Tensor, y: torch.Tensor | None = None,
                           ws: torch.Tensor | None = None):
    """Routed SwiGLU MoE FFN plus the sigmoid-gated shared expert; returns f32 ``[m, hidden]``."""
    _require(x, "x", torch.bfloat16)
    dev = x.device
    _require(ids, "ids", torch.int32, dev)
    _require(weights, "weights", torch.float32, dev)
    for name, t in (("W_gate", W_gate), ("W_up", W_up), ("W_down", W_down), ("w_sh", w_sh),
                    ("W_sh_gate", W_sh_gate), ("W_sh_up", W_sh_up), ("W_sh_down", W_sh_down)):
        _require(t, name, torch.bfloat16, dev)
    m, top_k = ids.shape
    n_experts, inter, hidden = W_gate.shape
    inter_sh = W_sh_gate.shape[0]
    if y is None:
        y = torch.empty((m, hidden), dtype=torch.float32, device=dev)
    if ws is None:
        ws = _workspace(moe_ffn_shared_workspace(m, hidden, inter, inter_sh, top_k, n_experts),
                        dev)
    _check(load_library().moe_ffn_forward_shared(
        _ptr(x), _ptr(ids), _ptr(weights), _ptr(W_gate), _ptr(W_up), _ptr(W_down), _ptr(w_sh),
        _ptr(W_sh_gate), _ptr(W_sh_up), _ptr(W_sh_down), _ptr(y), m, hidden, inter, inter_sh,
        top_k, n_experts, _ptr(ws), ws.numel(), _stream(dev)))
    return y


def moe_ep_dispatch_workspace(m: int, top_k: int, n_ranks: int) -> int:
    return int(load_library().moe_ep_dispatch_workspace(m, top_k, n_ranks))


def moe_ep_dispatch(x: torch.Tensor, ids: torch.Tensor, n_experts: int, n_ranks: int,
                    layout: int = SHARED_PER_TOKEN, send_x: torch.Tensor | None = None,
                    send_expert: torch.Tensor | None = None,
                    send_counts: torch.Tensor | None = None, ws: torch.Tensor | None = None):
    """Sort this rank's routed rows by owner rank and pack them for the
    all-to-all; returns ``(send_x [R, hidden] bf16, send_expert [R] int32,
    send_counts [n_ranks] int32 (device), ws)``.  Keep ``ws`` for
    :func:`moe_ep_combine` of the same step."""
    _require(x, "x", torch.bfloat16)
    dev = x.device
    _require(ids, "ids", torch.int32, dev)
    m, top_k = ids.shape
    hidden = x.shape[-1]
    rows = m * top_k
    if send_x is None:
        send_x = torch.empty((rows, hidden), dtype=torch.bfloat16, device=dev)
    if send_expert is None:
        send_expert = torch.empty(rows, dtype=torch.int32, device=dev)
    if send_counts is None:
        send_counts = torch.empty(n_ranks, dtype=torch.int32, device=dev)
    if ws is None:
        ws = _workspace(moe_ep_dispatch_workspace(m, top_k, n_ranks), dev)
    _check(load_library().moe_ep_dispatch(_ptr(x), _ptr(ids), m, hidden, top_k, n_experts,
                                          n_ranks, layout, _ptr(send_x), _ptr(send_expert),
                                          _ptr(send_counts), _ptr(ws), ws.numel(), _stream(dev)))
    return send_x, send_expert, send_counts, ws


def moe_ep_combine(d_back: torch.Tensor, weights: torch.Tensor, n_ranks: int, ws: torch.Tensor,
                   y: torch.Tensor | None = None):
    """Weighted slot-order combine of the rows returned by the owners
    (``d_back`` in this rank's send order); returns f32 ``[m, hidden]``."""
    _require(d_back, "d_back", torch.float32)
    dev = d_back.device
    _require(weights, "weights", torch.float32, dev)
    m, top_k = weights.shape
    hidden = d_back.shape[-1]
    if y is None:
        y = torch.empty((m, hidden), dtype=torch.float32, device=dev)
    _check(load_library().moe_ep_combine(_ptr(d_back), _ptr(weights), _ptr(y), m, hidden, top_k,
                                         n_ranks, _ptr(ws), ws.numel(), _stream(dev)))
    return y


def moe_set_stage_events(events, prerecord: bool = True) -> None:
    """Register torch.cuda.Event objects (>= 5) recorded between the stages of
    moe_ffn_forward / moe_matmul_id on this thread; None stops recording.
    With prerecord=False the events must already have been recorded once
    through torch (keeps extra records out of a timed region)."""
    lib = load_library()
    if events is None:
        _check(lib.moe_set_stage_events(None, 0))
        return
    # torch creates an event's handle at its first record() and only times
    # events it has recorded itself: record each once here, the library's
    # records then move them.
    if prerecord:
        for e in events:
            e.record()
    handles = (ctypes.c_void_p * len(events))(*[e.cuda_event for e in events])
    if not all(handles):
        raise RuntimeError("stage events have no CUDA handle")
    _check(lib.moe_set_stage_events(handles, len(events)))


def moe_clock_probe(out: torch.Tensor) -> None:
    """Enqueue a clock probe: ``out`` is an int64 CUDA tensor of shape
    ``[n_blocks, 3]`` filled with (SM id, SM cycle counter, global ns timer)."""
    _require(out, "out", torch.int64)
    _check(load_library().moe_clock_probe(_ptr(out), out.shape[0], _stream(out.device)))


def probe_clock_mhz(start: torch.Tensor, end: torch.Tensor):
    """Average SM clock (MHz) between two clock probes: the median over SMs
    seen by both of delta cycles / delta ns (host arithmetic on the probes)."""
    a = {int(r[0]): (int(r[1]), int(r[2])) for r in start.cpu().tolist()}
    rates = []
    for r in end.cpu().tolist():
        sm = int(r[0])
        if sm in a and int(r[2]) > a[sm][1]:
            rates.append((int(r[1]) - a[sm][0]) / (int(r[2]) - a[sm][1]) * 1e3)
    if not rates:
        return None
    rates.sort()
    return rates[len(rates) // 2]


def moe_selftest_wait_timeout(status_word: torch.Tensor, limit_ns: int) -> None:
    _require(status_word, "status_word", torch.int32)
    _check(load_library().moe_selftest_wait_timeout(_ptr(status_word), int(limit_ns),
                                                    _stream(status_word.device)))
