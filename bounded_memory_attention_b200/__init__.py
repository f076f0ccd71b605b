"""Python binding for librma, the RMA attention hot path on B200 (sm_100a).

Argument marshalling only: every step of decode, admit and prefill runs in
the CUDA kernels of ``librma.so``.  PyTorch provides device memory and
streams.  There is no CPU fallback: importing this package builds
``librma.so`` if it is missing or older than its sources (nvcc, sm_100a) and
fails if that is impossible.

The functions mirror the C ABI in ``include/rma.h`` (same names without the
``rma_`` prefix); see that header for the semantics, layouts and errors.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "librma.so")

STATUS_PENDING_OVERFLOW = 1
STATUS_NAN_SCORE = 2
STATUS_PREFILL_PENDING_OVERFLOW = 4
STATUS_BAD_COUNTERS = 8
STATUS_TIMEOUT = 16

KV_BF16 = 0
KV_FP8_E4M3 = 1

ERRORS = {0: "RMA_OK", -1: "RMA_ERR_INVALID_ARG", -2: "RMA_ERR_UNSUPPORTED", -3: "RMA_ERR_BUFFER_TOO_SMALL",
          -4: "RMA_ERR_CUDA", -5: "RMA_ERR_MISALIGNED"}


class _Config(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("n_layers", ctypes.c_int32), ("n_groups", ctypes.c_int32),
                ("q_per_group", ctypes.c_int32), ("head_dim", ctypes.c_int32), ("ring_slots", ctypes.c_int32),
                ("bank_slots", ctypes.c_int32), ("pend_slots", ctypes.c_int32), ("softmax_scale", ctypes.c_float),
                ("kv_format", ctypes.c_int32)]


class _Layout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_uint64) for n in (
        "total_bytes", "ring_k", "ring_v", "bank_k", "bank_v", "bank_score",
        "pend_k", "pend_v", "pend_score", "counters", "tickets", "status",
        "ring_k_exp", "ring_v_exp", "bank_k_exp", "bank_v_exp", "pend_k_exp", "pend_v_exp")]


def _load():
    from . import build as _build
    try:
        _build.build()          # no-op unless a source is newer than the library
    except Exception as ex:     # no nvcc, or a compile error: there is no fallback
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing and could not be built: {ex}") from ex
        raise ImportError(f"{LIB_PATH} is older than its sources and could not be rebuilt: {ex}") from ex
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32 = ctypes.c_void_p, ctypes.c_int
    cfgp = ctypes.POINTER(_Config)
    lib.rma_state_bytes.argtypes = [cfgp]
    lib.rma_state_bytes.restype = ctypes.c_size_t
    lib.rma_state_alloc.argtypes = [cfgp, vp, ctypes.c_size_t, vp, ctypes.POINTER(vp)]
    lib.rma_state_layout.argtypes = [vp, ctypes.POINTER(_Layout)]
    lib.rma_state_free.argtypes = [vp]
    lib.rma_state_free.restype = None
    lib.rma_workspace_bytes.argtypes = [vp, i32, ctypes.POINTER(ctypes.c_size_t)]
    lib.rma_set_decode_splits.argtypes = [vp, i32, i32]
    lib.rma_decode_step.argtypes = [vp, i32] + [vp] * 10 + [ctypes.c_size_t, vp]
    lib.rma_decode_step_noalloc.argtypes = [vp, i32] + [vp] * 9 + [vp]
    lib.rma_admit.argtypes = [vp, i32, i32, vp]
    lib.rma_prefill_block.argtypes = [vp, i32, i32] + [vp] * 10 + [ctypes.c_size_t, vp]
    lib.rma_get_status.argtypes = [vp, vp, ctypes.POINTER(ctypes.c_uint32)]
    lib.rma_state_quantize.argtypes = [vp, vp, vp]
    lib.rma_set_decode_overlap.argtypes = [vp, i32]
    lib.rma_strerror.argtypes = [i32]
    lib.rma_strerror.restype = ctypes.c_char_p
    lib.rma_last_error.argtypes = []
    lib.rma_last_error.restype = ctypes.c_char_p
    for f in ("rma_state_alloc", "rma_state_layout", "rma_workspace_bytes", "rma_set_decode_splits",
              "rma_decode_step", "rma_decode_step_noalloc", "rma_admit", "rma_prefill_block", "rma_get_status",
              "rma_state_quantize", "rma_set_decode_overlap"):
        getattr(lib, f).restype = ctypes.c_int
    return lib


lib = _load()


class RmaError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        msg = lib.rma_last_error().decode()
        super().__init__(f"{where}: {ERRORS.get(code, code)} ({msg})")


def _check(code: int, where: str) -> None:
    if code != 0:
        raise RmaError(code, where)


@dataclass
class Config:
    """RMA state dimensions; defaults are the pages' (4 groups, 1,023 + 1 window, 1,024 anchors, 256 pending).

    kv_format: KV_BF16 (the pages' storage) or KV_FP8_E4M3 (E4M3 codes with a power-of-two scale per row)."""
    batch: int = 1
    n_layers: int = 1
    n_groups: int = 4
    q_per_group: int = 4
    head_dim: int = 256
    ring_slots: int = 1023
    bank_slots: int = 1024
    pend_slots: int = 256
    softmax_scale: float = 1.0 / 16.0
    kv_format: int = KV_BF16

    def _c(self) -> _Config:
        return _Config(self.batch, self.n_layers, self.n_groups, self.q_per_group, self.head_dim,
                       self.ring_slots, self.bank_slots, self.pend_slots, self.softmax_scale, self.kv_format)

    @property
    def n_q_heads(self) -> int:
        return self.n_groups * self.q_per_group


def state_bytes(cfg: Config) -> int:
    c = cfg._c()
    return int(lib.rma_state_bytes(ctypes.byref(c)))


def _stream_handle(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t: torch.Tensor, dtype, numel: int, name: str) -> ctypes.c_void_p:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.numel() != numel:
        raise ValueError(f"{name} has {t.numel()} elements, expected {numel}")
    return ctypes.c_void_p(t.data_ptr())


class State:
    """A device state buffer (a torch uint8 tensor owned here) laid out by rma_state_alloc.

    Attributes ring_k, ring_v, bank_k, bank_v, bank_score, pend_k, pend_v,
    pend_score and counters are torch views into the buffer with the shapes
    listed in include/rma.h (counters [L, B, G, 4] = pos, bank_fill, pend_fill, 0).
    In an FP8 state the six K/V views are uint8 E4M3 codes, and ring_k_exp,
    ring_v_exp, bank_k_exp, bank_v_exp, pend_k_exp, pend_v_exp are int8 views
    [L, B, G, slots] of the rows' scale exponents (the padding to 16 slots is
    left out of the view).
    """

    def __init__(self, cfg: Config, device=None, stream=None, buffer: torch.Tensor = None):
        """Lay a state out over `buffer` (a CUDA uint8 tensor, 256-byte aligned, at least
        state_bytes(cfg) bytes, e.g. a view into a larger allocation), or over a fresh one."""
        self.cfg = cfg
        n = state_bytes(cfg)
        if n == 0:
            raise ValueError(f"invalid RMA config: {lib.rma_last_error().decode()}")
        if buffer is not None:
            if buffer.dtype != torch.uint8 or not buffer.is_cuda or not buffer.is_contiguous():
                raise TypeError("buffer must be a contiguous CUDA uint8 tensor")
            if buffer.numel() < n:
                raise ValueError(f"buffer holds {buffer.numel()} bytes, the state needs {n}")
            self.buffer = buffer[:n]
        else:
            device = torch.device(device if device is not None else "cuda")
            self.buffer = torch.empty(n + 256, dtype=torch.uint8, device=device)
            off = (-self.buffer.data_ptr()) % 256
            self.buffer = self.buffer[off:off + n]
        self._h = ctypes.c_void_p()
        c = cfg._c()
        _check(lib.rma_state_alloc(ctypes.byref(c), ctypes.c_void_p(self.buffer.data_ptr()), n,
                                   _stream_handle(stream), ctypes.byref(self._h)), "rma_state_alloc")
        lay = _Layout()
        _check(lib.rma_state_layout(self._h, ctypes.byref(lay)), "rma_state_layout")
        self.layout = {f: int(getattr(lay, f)) for f, _ in _Layout._fields_}
        L, B, G, D = cfg.n_layers, cfg.batch, cfg.n_groups, cfg.head_dim
        R, A, P = cfg.ring_slots, cfg.bank_slots, cfg.pend_slots

        def view(name, dtype, shape):
            nbytes = torch.tensor([], dtype=dtype).element_size()
            for s in shape:
                nbytes *= s
            o = self.layout[name]
            return self.buffer[o:o + nbytes].view(dtype).view(*shape)

        kv = torch.uint8 if cfg.kv_format == KV_FP8_E4M3 else torch.bfloat16
        self.ring_k = view("ring_k", kv, (L, B, G, R, D))
        self.ring_v = view("ring_v", kv, (L, B, G, R, D))
        self.bank_k = view("bank_k", kv, (L, B, G, A, D))
        self.bank_v = view("bank_v", kv, (L, B, G, A, D))
        self.bank_score = view("bank_score", torch.float32, (L, B, G, A))
        self.pend_k = view("pend_k", kv, (L, B, G, P, D))
        self.pend_v = view("pend_v", kv, (L, B, G, P, D))
        self.pend_score = view("pend_score", torch.float32, (L, B, G, P))
        self.counters = view("counters", torch.int32, (L, B, G, 4))
        if cfg.kv_format == KV_FP8_E4M3:
            for name, slots in (("ring_k_exp", R), ("ring_v_exp", R), ("bank_k_exp", A), ("bank_v_exp", A),
                                ("pend_k_exp", P), ("pend_v_exp", P)):
                padded = (slots + 15) // 16 * 16
                setattr(self, name, view(name, torch.int8, (L, B, G, padded))[..., :slots])

    @property
    def handle(self) -> ctypes.c_void_p:
        return self._h

    def workspace_bytes(self, n_tok: int) -> int:
        out = ctypes.c_size_t()
        _check(lib.rma_workspace_bytes(self._h, int(n_tok), ctypes.byref(out)), "rma_workspace_bytes")
        return int(out.value)

    def workspace(self, n_tok: int) -> torch.Tensor:
        """A fresh device workspace for calls with n_tok tokens (1 = decode)."""
        n = self.workspace_bytes(n_tok)
        w = torch.empty(n + 256, dtype=torch.uint8, device=self.buffer.device)
        off = (-w.data_ptr()) % 256
        return w[off:off + n]

    def close(self) -> None:
        if getattr(self, "_h", None) is not None and self._h.value:
            lib.rma_state_free(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def set_decode_splits(state: State, ring_splits: int, bank_splits: int) -> None:
    _check(lib.rma_set_decode_splits(state.handle, int(ring_splits), int(bank_splits)), "rma_set_decode_splits")


def set_decode_overlap(state: State, enable: bool) -> None:
    """rma_set_decode_overlap: decode calls stream their ring and bank while the previous decode
    call on the stream (another layer) finishes; see include/rma.h for the caller's side."""
    _check(lib.rma_set_decode_overlap(state.handle, 1 if enable else 0), "rma_set_decode_overlap")


def decode_step(state: State, layer: int, q, k_cur, v_cur, cand_k, cand_v, cand_score, w_g, b_g, out, ws,
                stream=None) -> torch.Tensor:
    """rma_decode_step on device tensors; returns ``out``."""
    c = state.cfg
    B, G, HQ, D = c.batch, c.n_groups, c.n_q_heads, c.head_dim
    bf, f32 = torch.bfloat16, torch.float32
    args = [_ptr(q, bf, B * HQ * D, "q"), _ptr(k_cur, bf, B * G * D, "k_cur"), _ptr(v_cur, bf, B * G * D, "v_cur"),
            _ptr(cand_k, bf, B * G * D, "cand_k"), _ptr(cand_v, bf, B * G * D, "cand_v"),
            _ptr(cand_score, f32, B * G, "cand_score"), _ptr(w_g, f32, HQ * D, "w_g"), _ptr(b_g, f32, HQ, "b_g"),
            _ptr(out, bf, B * HQ * D, "out")]
    if ws.dtype != torch.uint8 or not ws.is_cuda:
        raise TypeError("ws must be a CUDA uint8 tensor")
    _check(lib.rma_decode_step(state.handle, int(layer), *args, ctypes.c_void_p(ws.data_ptr()), ws.numel(),
                               _stream_handle(stream)), "rma_decode_step")
    return out


def decode_step_noalloc(state: State, layer: int, q, k_cur, v_cur, cand_k, cand_v, cand_score, w_g, b_g, out,
                        stream=None) -> torch.Tensor:
    """rma_decode_step_noalloc: a decode step for callers that cannot allocate device memory.

    Like ``decode_step`` but without a workspace: the library's built-in 32 MiB
    scratch per GPU holds the partials.  Calls that may overlap on the GPU
    share that scratch and must be ordered by the caller; the first call on a
    device should come before any stream capture.  Returns ``out``.
    """
    c = state.cfg
    B, G, HQ, D = c.batch, c.n_groups, c.n_q_heads, c.head_dim
    bf, f32 = torch.bfloat16, torch.float32
    args = [_ptr(q, bf, B * HQ * D, "q"), _ptr(k_cur, bf, B * G * D, "k_cur"), _ptr(v_cur, bf, B * G * D, "v_cur"),
            _ptr(cand_k, bf, B * G * D, "cand_k"), _ptr(cand_v, bf, B * G * D, "cand_v"),
            _ptr(cand_score, f32, B * G, "cand_score"), _ptr(w_g, f32, HQ * D, "w_g"), _ptr(b_g, f32, HQ, "b_g"),
            _ptr(out, bf, B * HQ * D, "out")]
    _check(lib.rma_decode_step_noalloc(state.handle, int(layer), *args, _stream_handle(stream)),
           "rma_decode_step_noalloc")
    return out


def admit(state: State, layer: int, force: bool = False, stream=None) -> None:
    """rma_admit."""
    _check(lib.rma_admit(state.handle, int(layer), 1 if force else 0, _stream_handle(stream)), "rma_admit")


def prefill_block(state: State, layer: int, q, k, v, cand_k, cand_v, cand_score, w_g, b_g, out, ws,
                  stream=None) -> torch.Tensor:
    """rma_prefill_block on device tensors (includes the forced admit); returns ``out``."""
    c = state.cfg
    B, G, HQ, D = c.batch, c.n_groups, c.n_q_heads, c.head_dim
    n = q.shape[1] if q.dim() == 4 else 0
    bf, f32 = torch.bfloat16, torch.float32
    args = [_ptr(q, bf, B * n * HQ * D, "q"), _ptr(k, bf, B * n * G * D, "k"), _ptr(v, bf, B * n * G * D, "v"),
            _ptr(cand_k, bf, B * n * G * D, "cand_k"), _ptr(cand_v, bf, B * n * G * D, "cand_v"),
            _ptr(cand_score, f32, B * n * G, "cand_score"), _ptr(w_g, f32, HQ * D, "w_g"),
            _ptr(b_g, f32, HQ, "b_g"), _ptr(out, bf, B * n * HQ * D, "out")]
    if ws.dtype != torch.uint8 or not ws.is_cuda:
        raise TypeError("ws must be a CUDA uint8 tensor")
    _check(lib.rma_prefill_block(state.handle, int(layer), int(n), *args, ctypes.c_void_p(ws.data_ptr()),
                                 ws.numel(), _stream_handle(stream)), "rma_prefill_block")
    return out


def state_quantize(dst: State, src: State, stream=None) -> None:
    """rma_state_quantize: every row of the BF16 state `src` quantised into the FP8 state `dst`."""
    _check(lib.rma_state_quantize(dst.handle, src.handle, _stream_handle(stream)), "rma_state_quantize")


def get_status(state: State, stream=None) -> int:
    """Wait for the stream, then read and clear the device status word (RMA_STATUS_* bits)."""
    flags = ctypes.c_uint32()
    _check(lib.rma_get_status(state.handle, _stream_handle(stream), ctypes.byref(flags)), "rma_get_status")
    return int(flags.value)
