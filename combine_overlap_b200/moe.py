"""Thin ctypes binding over libmoe_b200.so (the C ABI in include/moe.h).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  Tensors are torch CUDA tensors (PyTorch provides device memory and
streams); calls are issued on the current torch stream.  If the library is not
built this module raises at import -- there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")
HEADER = os.path.join(os.path.dirname(_HERE), "include", "moe.h")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is not built; run combine_overlap_b200.build.build() "
                      "(nvcc, sm_100a) first")

_lib = ctypes.CDLL(LIB_PATH)

MOE_OK, MOE_ERR_INVALID, MOE_ERR_UNSUPPORTED, MOE_ERR_CUDA, MOE_ERR_TIMEOUT, MOE_ERR_WORKSPACE = range(6)
MODE_SEQUENTIAL, MODE_OVERLAPPED = 0, 1
DBG_SKIP_FLAG_BAND = 0x1
SCHED_NO_JOIN = 0x2
SCHED_ONE_CTA = 0x4
DBG_TIMESTAMPS = 0x8
SCHED_GATHER_A = 0x10
SCHED_CTA_PAIR = 0x20
SCHED_B_PER_ATOM = 0x40
SCHED_FULL_TILES = 0x80
SCHED_WIDE_CTA = 0x100
DBG_IDENTITY_EXPERTS = 0x200
SCHED_INTERLEAVE = 0x400
SCHED_EVICT_FIRST = 0x800
SCHED_SIDE_COMBINE = 0x1000
SCHED_EXP_SILU = 0x4000
SCHED_GATHER_LSU = 0x8000


class MoEError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        self.cuda_error = last_cuda_error() if code == MOE_ERR_CUDA else 0
        detail = f"; {cuda_error_string(self.cuda_error)} (cudaError {self.cuda_error})" \
            if self.cuda_error else ""
        super().__init__(f"{what}: {status_string(code)} (code {code}){detail}")


class LayerArgs(ctypes.Structure):
    _fields_ = [
        ("T", ctypes.c_int), ("d", ctypes.c_int), ("f", ctypes.c_int), ("E", ctypes.c_int),
        ("k", ctypes.c_int),
        ("x", ctypes.c_void_p), ("logits", ctypes.c_void_p),
        ("W1", ctypes.c_void_p), ("W3", ctypes.c_void_p), ("W2", ctypes.c_void_p),
        ("out", ctypes.c_void_p),
        ("topk_idx", ctypes.c_void_p), ("topk_gate", ctypes.c_void_p),
        ("counts", ctypes.c_void_p), ("offsets", ctypes.c_void_p), ("perm", ctypes.c_void_p),
        ("consumer_sms", ctypes.c_int), ("mgb", ctypes.c_int), ("flags", ctypes.c_uint),
        ("timeout_us", ctypes.c_int),
        ("ev_ffn_begin", ctypes.c_void_p), ("ev_ffn_end", ctypes.c_void_p),
    ]


MAX_EP_RANKS = 8


class EpOwnerArgs(ctypes.Structure):
    _fields_ = [
        ("W", ctypes.c_int), ("rank", ctypes.c_int), ("N", ctypes.c_int), ("d", ctypes.c_int),
        ("f", ctypes.c_int), ("El", ctypes.c_int), ("k", ctypes.c_int),
        ("x_recv", ctypes.c_void_p), ("slot_recv", ctypes.c_void_p), ("recv_counts", ctypes.c_void_p),
        ("W1", ctypes.c_void_p), ("W3", ctypes.c_void_p), ("W2", ctypes.c_void_p),
        ("recv_base", ctypes.c_int * MAX_EP_RANKS),
        ("home_y", ctypes.c_void_p * MAX_EP_RANKS),
        ("home_arrive", ctypes.c_void_p * MAX_EP_RANKS),
        ("consumer_sms", ctypes.c_int), ("mgb", ctypes.c_int), ("flags", ctypes.c_uint),
        ("timeout_us", ctypes.c_int),
    ]


_P, _I, _S = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
_lib.moe_workspace_size.argtypes = [_I, _I, _I, _I, _I]
_lib.moe_workspace_size.restype = _S
_lib.moe_route.argtypes = [_P, _I, _I, _I, _P, _P, _P, _P, _S, _P]
_lib.moe_permute.argtypes = [_P, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _S, _P]
_lib.moe_grouped_ffn.argtypes = [_P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, ctypes.c_uint,
                                 _P, _S, _P]
_lib.moe_combine.argtypes = [_P, _P, _P, _I, _I, _I, _P, _P]
_lib.moe_layer_forward.argtypes = [ctypes.POINTER(LayerArgs), _I, _P, _S, _P]
_lib.moe_get_status.argtypes = [_P, _P, ctypes.POINTER(_I), ctypes.POINTER(_I)]
_lib.moe_status_string.argtypes = [_I]
_lib.moe_status_string.restype = ctypes.c_char_p
_lib.moe_num_sms.restype = _I
_lib.moe_tile_variant.argtypes = [_I, _I, _I, _I, ctypes.c_uint]
_lib.moe_tile_variant.restype = _I
_lib.moe_last_cuda_error.restype = _I
_lib.moe_cuda_error_string.argtypes = [_I]
_lib.moe_cuda_error_string.restype = ctypes.c_char_p
_lib.moe_debug_stamps.argtypes = [_P, _P, _P, _I, ctypes.POINTER(_I)]
_lib.moe_debug_stamps.restype = _I
_lib.moe_debug_band_stamps.argtypes = [_P, _P, _P, _I]
_lib.moe_debug_band_stamps.restype = _I
_lib.moe_debug_tokens_combined.argtypes = [_P, _I, _I, _I, _I, _I, _P, ctypes.POINTER(_I)]
_lib.moe_debug_tokens_combined.restype = _I
_lib.moe_permute_noalloc.argtypes = [_P, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P]
_lib.moe_permute_noalloc.restype = _I
_lib.moe_permute_noalloc_scratch_bytes.restype = _S
_lib.moe_ep_owner_workspace_size.argtypes = [_I, _I, _I, _I, _I]
_lib.moe_ep_owner_workspace_size.restype = _S
_lib.moe_ep_owner_forward.argtypes = [ctypes.POINTER(EpOwnerArgs), _I, _P, _S, _P]
_lib.moe_ep_home_combine.argtypes = [_P, _P, _P, _P, _I, _I, _I, _P, _P, _I, _P]
_lib.moe_ep_debug_plan.argtypes = [_P, _I, _I, _I, _I, _I, _P, _P, _I]
_lib.moe_ep_debug_plan.restype = _I
for _fn in ("moe_route", "moe_permute", "moe_grouped_ffn", "moe_combine", "moe_layer_forward",
            "moe_get_status", "moe_ep_owner_forward", "moe_ep_home_combine"):
    getattr(_lib, _fn).restype = _I


def declared_symbols() -> list[str]:
    """Function names declared in include/moe.h."""
    with open(HEADER) as fh:
        text = fh.read()
    return sorted(set(re.findall(r"^\s*(?:[\w\*]+\s+)+\**(moe_\w+)\s*\(", text, re.M)))


def status_string(code: int) -> str:
    return _lib.moe_status_string(int(code)).decode()


TILE_VARIANTS = {1: "128x256 per CTA", 2: "256x256 per CTA pair (cta_group::2)",
                 3: "256x256 per CTA (two 128-row MMAs)"}


def tile_variant(T: int, f: int, E: int, k: int, flags: int = 0) -> int:
    """The MMA tile variant the library picks for this shape and flags (1, 2, 3)."""
    return int(_lib.moe_tile_variant(T, f, E, k, int(flags)))


def last_cuda_error() -> int:
    """The cudaError_t value behind this thread's latest MOE_ERR_CUDA (0: none)."""
    return int(_lib.moe_last_cuda_error())


def cuda_error_string(code: int) -> str:
    return _lib.moe_cuda_error_string(int(code)).decode()


def _check(code: int, what: str):
    if code != MOE_OK:
        raise MoEError(code, what)


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _need(t: torch.Tensor, dtype, name: str):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _shape(t: torch.Tensor, shape: tuple, name: str):
    """The library sees pointers only: a tensor of another shape would be read or
    written out of bounds on the device, so sizes are checked here."""
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _weights(W1, W3, W2, d=None):
    """Checks W1, W3 [E][d][f] and W2 [E][f][d]; returns (E, d, f)."""
    for n, w in (("W1", W1), ("W3", W3), ("W2", W2)):
        _need(w, torch.bfloat16, n)
        if w.dim() != 3:
            raise ValueError(f"{n} must be 3-D, got shape {tuple(w.shape)}")
    E, dw, f = W1.shape
    if d is not None and dw != d:
        raise ValueError(f"W1 is [E][{dw}][f] but the rows have d = {d}")
    _shape(W3, (E, dw, f), "W3")
    _shape(W2, (E, f, dw), "W2")
    return E, dw, f


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def workspace_size(T: int, d: int, f: int, E: int, k: int) -> int:
    return int(_lib.moe_workspace_size(T, d, f, E, k))


def num_sms() -> int:
    return int(_lib.moe_num_sms())


def alloc_workspace(T, d, f, E, k, device="cuda") -> torch.Tensor:
    n = workspace_size(T, d, f, E, k)
    if n == 0:
        raise MoEError(MOE_ERR_UNSUPPORTED, "moe_workspace_size")
    return torch.empty(n, dtype=torch.uint8, device=device)


def route(logits: torch.Tensor, k: int, ws: torch.Tensor, counts: bool = False):
    _need(logits, torch.float32, "logits")
    T, E = logits.shape
    idx = torch.empty((T, k), dtype=torch.int32, device=logits.device)
    gate = torch.empty((T, k), dtype=torch.float32, device=logits.device)
    cnt = torch.empty(E, dtype=torch.int32, device=logits.device) if counts else None
    _check(_lib.moe_route(_ptr(logits), T, E, k, _ptr(idx), _ptr(gate), _ptr(cnt), _ptr(ws),
                          ws.numel(), _stream()), "moe_route")
    return (idx, gate, cnt) if counts else (idx, gate)


def permute(x: torch.Tensor, topk_idx: torch.Tensor, E: int, ws: torch.Tensor):
    _need(x, torch.bfloat16, "x")
    _need(topk_idx, torch.int32, "topk_idx")
    T, d = x.shape
    k = topk_idx.shape[1]
    _shape(topk_idx, (T, k), "topk_idx")
    dev = x.device
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    perm = torch.empty(T * k, dtype=torch.int32, device=dev)
    row_of = torch.empty(T * k, dtype=torch.int32, device=dev)
    x_perm = torch.empty((T * k, d), dtype=torch.bfloat16, device=dev)
    _check(_lib.moe_permute(_ptr(x), T, d, E, k, _ptr(topk_idx), _ptr(counts), _ptr(offsets),
                            _ptr(perm), _ptr(row_of), _ptr(x_perm), _ptr(ws), ws.numel(),
                            _stream()), "moe_permute")
    return counts, offsets, perm, row_of, x_perm


def permute_noalloc(x: torch.Tensor, topk_idx: torch.Tensor, E: int):
    """moe_permute without a workspace: the library's fixed scratch array is used
    instead (for callers that cannot allocate device memory; T <= 65536)."""
    _need(x, torch.bfloat16, "x")
    _need(topk_idx, torch.int32, "topk_idx")
    T, d = x.shape
    k = topk_idx.shape[1]
    _shape(topk_idx, (T, k), "topk_idx")
    dev = x.device
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    perm = torch.empty(T * k, dtype=torch.int32, device=dev)
    row_of = torch.empty(T * k, dtype=torch.int32, device=dev)
    x_perm = torch.empty((T * k, d), dtype=torch.bfloat16, device=dev)
    _check(_lib.moe_permute_noalloc(_ptr(x), T, d, E, k, _ptr(topk_idx), _ptr(counts),
                                    _ptr(offsets), _ptr(perm), _ptr(row_of), _ptr(x_perm),
                                    _stream()), "moe_permute_noalloc")
    return counts, offsets, perm, row_of, x_perm


def grouped_ffn(x_perm: torch.Tensor, offsets: torch.Tensor, W1, W3, W2, T: int, k: int,
                ws: torch.Tensor, want_h: bool = True, flags: int = 0):
    """x_perm: [T*k][d] bf16 (rows past offsets[E] unused); flags: SCHED_ONE_CTA,
    SCHED_CTA_PAIR, SCHED_B_PER_ATOM, SCHED_FULL_TILES."""
    _need(x_perm, torch.bfloat16, "x_perm")
    _need(offsets, torch.int32, "offsets")
    E, d, f = _weights(W1, W3, W2, x_perm.shape[1])
    _shape(x_perm, (T * k, d), "x_perm")
    _shape(offsets, (E + 1,), "offsets")
    dev = x_perm.device
    y = torch.empty((T * k, d), dtype=torch.bfloat16, device=dev)
    h = torch.empty((T * k, f), dtype=torch.bfloat16, device=dev) if want_h else None
    _check(_lib.moe_grouped_ffn(_ptr(x_perm), _ptr(offsets), T, d, f, E, k, _ptr(W1), _ptr(W3),
                                _ptr(W2), _ptr(h), _ptr(y), int(flags), _ptr(ws), ws.numel(),
                                _stream()),
           "moe_grouped_ffn")
    return h, y


def combine(y: torch.Tensor, row_of: torch.Tensor, topk_gate: torch.Tensor, out=None):
    _need(y, torch.bfloat16, "y")
    _need(row_of, torch.int32, "row_of")
    _need(topk_gate, torch.float32, "topk_gate")
    T, k = topk_gate.shape
    d = y.shape[1]
    _shape(y, (T * k, d), "y")
    _shape(row_of, (T * k,), "row_of")
    if out is None:
        out = torch.empty((T, d), dtype=torch.bfloat16, device=y.device)
    _need(out, torch.bfloat16, "out")
    _shape(out, (T, d), "out")
    _check(_lib.moe_combine(_ptr(y), _ptr(row_of), _ptr(topk_gate), T, d, k, _ptr(out), _stream()),
           "moe_combine")
    return out


def make_args(x, logits, W1, W3, W2, k, out, topk_idx=None, topk_gate=None, counts=None,
              offsets=None, perm=None, consumer_sms=0, mgb=1, flags=0, timeout_us=0,
              ev_begin=None, ev_end=None, d_ff=None) -> LayerArgs:
    T, d = x.shape
    E = logits.shape[1]
    f = W1.shape[2] if W1 is not None else d_ff
    wp = [0 if w is None else w.data_ptr() for w in (W1, W3, W2)]
    return LayerArgs(T, d, f, E, k, x.data_ptr(), logits.data_ptr(), *wp, out.data_ptr(),
                     *(0 if t is None else t.data_ptr() for t in (topk_idx, topk_gate, counts, offsets, perm)),
                     consumer_sms, mgb, flags, timeout_us,
                     None if ev_begin is None else ev_begin.cuda_event,
                     None if ev_end is None else ev_end.cuda_event)


def layer_forward(x, logits, W1, W3, W2, k, ws, mode=MODE_OVERLAPPED, out=None, outputs=False,
                  consumer_sms=0, mgb=1, flags=0, timeout_us=0, stream=None, ev_begin=None,
                  ev_end=None, d_ff=None):
    """One MoE layer.  Returns out, or (out, dict of routing outputs) if outputs.
    With flags DBG_IDENTITY_EXPERTS the weights may be None (then d_ff gives the
    FFN width the workspace was sized for)."""
    _need(x, torch.bfloat16, "x")
    _need(logits, torch.float32, "logits")
    T, d = x.shape
    if W1 is None and W3 is None and W2 is None and (flags & DBG_IDENTITY_EXPERTS):
        E, f = logits.shape[1], int(d_ff)
    else:
        E, _, f = _weights(W1, W3, W2, d)
    _shape(logits, (T, E), "logits")
    if ws.numel() < workspace_size(T, d, f, E, k):
        raise ValueError("workspace smaller than moe_workspace_size for this shape")
    dev = x.device
    if out is None:
        out = torch.empty((T, d), dtype=torch.bfloat16, device=dev)
    _need(out, torch.bfloat16, "out")
    _shape(out, (T, d), "out")
    extra = {}
    if outputs:
        extra = dict(topk_idx=torch.empty((T, k), dtype=torch.int32, device=dev),
                     topk_gate=torch.empty((T, k), dtype=torch.float32, device=dev),
                     counts=torch.empty(E, dtype=torch.int32, device=dev),
                     offsets=torch.empty(E + 1, dtype=torch.int32, device=dev),
                     perm=torch.empty(T * k, dtype=torch.int32, device=dev))
    # torch creates an event lazily and only times events it has seen recorded:
    # record them here first (this also creates them); the library records them
    # again at the FFN boundaries, and the last record is the one timed.
    s = stream if stream is not None else torch.cuda.current_stream()
    for ev in (ev_begin, ev_end):
        if ev is not None:
            ev.record(s)
    args = make_args(x, logits, W1, W3, W2, k, out, consumer_sms=consumer_sms, mgb=mgb,
                     flags=flags, timeout_us=timeout_us, ev_begin=ev_begin, ev_end=ev_end,
                     d_ff=f, **extra)

    _check(_lib.moe_layer_forward(ctypes.byref(args), int(mode), _ptr(ws), ws.numel(),
                                  _stream(stream)), "moe_layer_forward")
    return (out, extra) if outputs else out


def get_status(ws: torch.Tensor, stream=None):
    """(status code, consumer SMs used, row bands) of the last call on ws; syncs."""
    c = ctypes.c_int(0)
    nb = ctypes.c_int(0)
    code = _lib.moe_get_status(_ptr(ws), _stream(stream), ctypes.byref(c), ctypes.byref(nb))
    return int(code), int(c.value), int(nb.value)


def debug_stamps(ws: torch.Tensor, stream=None):
    """Per-CTA stamps of the last persistent launch run with DBG_TIMESTAMPS: a
    uint64 array [n_ctas][8] (start, GEMM1 queue drained, producer done,
    consumer done -- globaltimer ns -- GEMM1 tiles, GEMM2 tiles, consumer bands,
    cluster rank)."""
    import numpy as np
    out = np.zeros((256, 8), dtype=np.uint64)
    n = ctypes.c_int(0)
    _check(_lib.moe_debug_stamps(_ptr(ws), _stream(stream), out.ctypes.data_as(ctypes.c_void_p), 256,
                                 ctypes.byref(n)), "moe_debug_stamps")
    return out[:n.value]


def debug_band_stamps(ws: torch.Tensor, n_bands: int, stream=None):
    """Per consumed row band of the last DBG_TIMESTAMPS launch: [n][4] uint64 (ready
    ns, combined ns, tokens completed, consuming CTA)."""
    import numpy as np
    n = max(1, min(int(n_bands), 2048))
    out = np.zeros((n, 4), dtype=np.uint64)
    _check(_lib.moe_debug_band_stamps(_ptr(ws), _stream(stream), out.ctypes.data_as(ctypes.c_void_p), n),
           "moe_debug_band_stamps")
    return out


def debug_tokens_combined(ws: torch.Tensor, T: int, d: int, f: int, E: int, k: int, stream=None) -> int:
    """Tokens of the last overlapped call on ws (this shape) that the persistent
    kernel combined itself; the combine pass after it did the rest."""
    n = ctypes.c_int(0)
    _check(_lib.moe_debug_tokens_combined(_ptr(ws), T, d, f, E, k, _stream(stream), ctypes.byref(n)),
           "moe_debug_tokens_combined")
    return int(n.value)


class MoELayer:
    """Holds the weights and a workspace; forward() runs the layer."""

    def __init__(self, W1, W3, W2, k: int, max_tokens: int):
        self.W1, self.W3, self.W2, self.k = W1, W3, W2, k
        self.E, self.d, self.f = W1.shape
        self.max_tokens = max_tokens
        self.ws = alloc_workspace(max_tokens, self.d, self.f, self.E, k, W1.device)

    def forward(self, x, logits, mode=MODE_OVERLAPPED, **kw):
        if x.shape[0] > self.max_tokens:
            raise ValueError("more tokens than the workspace was sized for")
        return layer_forward(x, logits, self.W1, self.W3, self.W2, self.k, self.ws, mode, **kw)


# ---- expert parallelism: the fused return -----------------------------------
def ep_owner_workspace_size(N: int, d: int, f: int, El: int, W: int) -> int:
    return int(_lib.moe_ep_owner_workspace_size(N, d, f, El, W))


def ep_owner_forward(x_recv, slot_recv, recv_counts, W1, W3, W2, k: int, rank: int, recv_base,
                     home_y, home_arrive, ws, mode=MODE_OVERLAPPED, consumer_sms=0, mgb=1,
                     flags=0, timeout_us=0, stream=None):
    """The owner side of an expert-parallel layer (moe_ep_owner_forward): runs
    this rank's experts on the rows it received and returns every finished row
    band into its home rank's buffer (home_y[s], home_arrive[s], one per rank)."""
    _need(x_recv, torch.bfloat16, "x_recv")
    _need(slot_recv, torch.int32, "slot_recv")
    _need(recv_counts, torch.int32, "recv_counts")
    N, d = x_recv.shape
    El, _, f = _weights(W1, W3, W2, d)
    W = recv_counts.shape[0]
    _shape(recv_counts, (W, El), "recv_counts")
    _shape(slot_recv, (N,), "slot_recv")
    if not (1 <= W <= MAX_EP_RANKS) or len(home_y) != W or len(home_arrive) != W or len(recv_base) != W:
        raise ValueError("one home buffer, arrival array and receive base per rank")
    for s_, (y, a) in enumerate(zip(home_y, home_arrive)):
        _need(y, torch.bfloat16, f"home_y[{s_}]")
        _need(a, torch.int32, f"home_arrive[{s_}]")
        if y.shape[1] != d:
            raise ValueError(f"home_y[{s_}] rows must have d = {d}")
    if ws.numel() < ep_owner_workspace_size(N, d, f, El, W):
        raise ValueError("workspace smaller than moe_ep_owner_workspace_size")
    if N == 0:
        return   # nothing received: no band to compute or return
    a = EpOwnerArgs()
    a.W, a.rank, a.N, a.d, a.f, a.El, a.k = W, rank, N, d, f, El, k
    a.x_recv, a.slot_recv, a.recv_counts = x_recv.data_ptr(), slot_recv.data_ptr(), recv_counts.data_ptr()
    a.W1, a.W3, a.W2 = W1.data_ptr(), W3.data_ptr(), W2.data_ptr()
    for s_ in range(W):
        a.recv_base[s_] = int(recv_base[s_])
        a.home_y[s_] = home_y[s_].data_ptr()
        a.home_arrive[s_] = home_arrive[s_].data_ptr()
    a.consumer_sms, a.mgb, a.flags, a.timeout_us = consumer_sms, mgb, flags, timeout_us
    _check(_lib.moe_ep_owner_forward(ctypes.byref(a), int(mode), _ptr(ws), ws.numel(), _stream(stream)),
           "moe_ep_owner_forward")


def ep_home_combine(home_y, arrive, row_of, topk_gate, out=None, status=None, timeout_us=0,
                    stream=None):
    """The home side (moe_ep_home_combine): waits for each token's k returned
    rows, combines them and zeroes the arrival words.  Returns (out, status) with
    status a one-element int32 device tensor (0, or MOE_ERR_TIMEOUT)."""
    _need(home_y, torch.bfloat16, "home_y")
    _need(arrive, torch.int32, "arrive")
    _need(row_of, torch.int32, "row_of")
    _need(topk_gate, torch.float32, "topk_gate")
    T, k = topk_gate.shape
    d = home_y.shape[1]
    _shape(home_y, (T * k, d), "home_y")
    _shape(arrive, (T,), "arrive")
    _shape(row_of, (T * k,), "row_of")
    if out is None:
        out = torch.empty((T, d), dtype=torch.bfloat16, device=home_y.device)
    _shape(out, (T, d), "out")
    if status is None:
        status = torch.zeros(1, dtype=torch.int32, device=home_y.device)
    _check(_lib.moe_ep_home_combine(_ptr(home_y), _ptr(arrive), _ptr(row_of), _ptr(topk_gate), T, d, k,
                                    _ptr(out), _ptr(status), int(timeout_us), _stream(stream)),
           "moe_ep_home_combine")
    return out, status


def ep_band_dest(ws, N: int, d: int, f: int, El: int, W: int, n_bands: int, stream=None):
    """The combine plan of the last owner call on ws: [n_bands][2] int32 (home
    rank, home row of the band's first row), bands in schedule order."""
    import numpy as np
    out = np.zeros((max(1, n_bands), 2), dtype=np.int32)
    _check(_lib.moe_ep_debug_plan(_ptr(ws), N, d, f, El, W, _stream(stream),
                                  out.ctypes.data_as(ctypes.c_void_p), max(1, n_bands)),
           "moe_ep_debug_plan")
    return out[:n_bands]
