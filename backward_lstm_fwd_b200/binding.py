"""ctypes binding of liblstm.so (C ABI declared in include/liblstm.h).

Argument marshalling only: every step of the LSTM forward pass and BPTT runs
inside the library's CUDA kernels.  torch tensors are used for device memory
and for the current CUDA stream; nothing here computes on them.  When the
shared library is missing, every entry point raises -- there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "liblstm.so")

LSTM_OK = 0
LSTM_ERR_INVALID_ARG = 1
LSTM_ERR_UNSUPPORTED = 2
LSTM_ERR_WORKSPACE = 3
LSTM_ERR_CUDA = 4
LSTM_ERR_TIMEOUT = 5
LSTM_ERR_NOT_CORESIDENT = 6

ABI_VERSION = 103  # the liblstm.h this binding mirrors (100 * major + minor)
LSTM_F32 = 0
LSTM_BF16 = 1
LSTM_F16 = 2

EXPORTS = ("lstm_fwd_workspace_size", "lstm_bwd_workspace_size", "lstm_fwd_workspace_size_ex",
           "lstm_fwd_workspace_size_max", "lstm_fwd", "lstm_bwd",
           "lstm_fwd_ex", "lstm_bwd_ex", "lstm_stack_fwd_workspace_size",
           "lstm_stack_bwd_workspace_size", "lstm_stack_bwd_workspace_size_min",
           "lstm_stack_fwd", "lstm_stack_bwd",
           "lstm_status", "lstm_profile_begin", "lstm_profile_end", "lstm_launch_count",
           "lstm_strerror", "lstm_abi_version")

PHASES = ("input_proj", "fwd_recur", "bwd_recur", "dW", "db", "dx", "other")


class LstmError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: liblstm status {code} ({strerror(code)})")


class Dims(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int), ("B", ctypes.c_int), ("I", ctypes.c_int),
                ("H", ctypes.c_int), ("dtype", ctypes.c_int)]


LSTM_DIR_FORWARD, LSTM_DIR_REVERSE = 0, 1
LSTM_GATES_IFJO, LSTM_GATES_IJFO = 0, 1
GATE_ORDERS = {"ifjo": LSTM_GATES_IFJO, "ijfo": LSTM_GATES_IJFO}


class Options(ctypes.Structure):
    """lstm_options: the seq_length mask (device pointer or None), the
    direction (LSTM_DIR_FORWARD / LSTM_DIR_REVERSE) and the gate_order
    (LSTM_GATES_IFJO / LSTM_GATES_IJFO)."""
    _fields_ = [("seq_mask", ctypes.c_void_p), ("direction", ctypes.c_int),
                ("gate_order", ctypes.c_int)]


_lib = None


def load(path: str = LIB_PATH):
    """Load liblstm.so (raises if it has not been built)."""
    global _lib
    if _lib is not None and path == LIB_PATH:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"liblstm.so not found at {path}: build it with "
                           "`python -m backward_lstm_fwd_b200.build`")
    lib = ctypes.CDLL(path)
    vp, sz, ip = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
    dp = ctypes.POINTER(Dims)
    lib.lstm_fwd_workspace_size.argtypes = [dp]
    lib.lstm_fwd_workspace_size.restype = sz
    lib.lstm_bwd_workspace_size.argtypes = [dp]
    lib.lstm_bwd_workspace_size.restype = sz
    lib.lstm_fwd_workspace_size_max.argtypes = [dp]
    lib.lstm_fwd_workspace_size_max.restype = sz
    lib.lstm_fwd.argtypes = [dp] + [vp] * 10 + [vp, sz, vp]
    lib.lstm_fwd.restype = ip
    lib.lstm_bwd.argtypes = [dp] + [vp] * 15 + [vp, sz, vp]
    lib.lstm_bwd.restype = ip
    op = ctypes.POINTER(Options)
    lib.lstm_fwd_workspace_size_ex.argtypes = [dp, op]
    lib.lstm_fwd_workspace_size_ex.restype = sz
    lib.lstm_fwd_ex.argtypes = [dp, op] + [vp] * 10 + [vp, sz, vp]
    lib.lstm_fwd_ex.restype = ip
    lib.lstm_bwd_ex.argtypes = [dp, op] + [vp] * 15 + [vp, sz, vp]
    lib.lstm_bwd_ex.restype = ip
    pp = ctypes.POINTER(ctypes.c_void_p)  # host array of device pointers
    lib.lstm_stack_fwd_workspace_size.argtypes = [dp, ip]
    lib.lstm_stack_fwd_workspace_size.restype = sz
    lib.lstm_stack_bwd_workspace_size.argtypes = [dp, ip]
    lib.lstm_stack_bwd_workspace_size.restype = sz
    lib.lstm_stack_bwd_workspace_size_min.argtypes = [dp, ip]
    lib.lstm_stack_bwd_workspace_size_min.restype = sz
    lib.lstm_stack_fwd.argtypes = [dp, ip, op, vp, pp, pp] + [vp] * 7 + [vp, sz, vp]
    lib.lstm_stack_fwd.restype = ip
    lib.lstm_stack_bwd.argtypes = [dp, ip, op] + [vp] * 4 + [pp] + [vp] * 6 + [pp, pp] + \
        [vp] * 2 + [vp, sz, vp]
    lib.lstm_stack_bwd.restype = ip
    lib.lstm_status.argtypes = [vp, sz, vp]
    lib.lstm_status.restype = ip
    lib.lstm_strerror.argtypes = [ip]
    lib.lstm_strerror.restype = ctypes.c_char_p
    lib.lstm_abi_version.argtypes = []
    lib.lstm_abi_version.restype = ip
    lib.lstm_profile_begin.argtypes = []
    lib.lstm_profile_begin.restype = ip
    lib.lstm_profile_end.argtypes = [ctypes.POINTER(ctypes.c_double),
                                     ctypes.POINTER(ctypes.c_longlong)]
    lib.lstm_profile_end.restype = ip
    lib.lstm_launch_count.argtypes = []
    lib.lstm_launch_count.restype = ctypes.c_longlong
    lib.lstm_fwd_noalloc.argtypes = [dp] + [vp] * 10 + [vp]
    lib.lstm_fwd_noalloc.restype = ip
    lib.lstm_fwd_noalloc_status.argtypes = [vp]
    lib.lstm_fwd_noalloc_status.restype = ip
    ll = ctypes.c_longlong
    lib.lstm_test_tc_gemm.argtypes = [ip, ip, ip, vp, ll, ip, vp, ll, ip, vp, vp, ll, vp, sz, vp]
    lib.lstm_test_tc_gemm.restype = ip
    lib.lstm_test_set_wait_fault.argtypes = [ip, ll]
    lib.lstm_test_set_wait_fault.restype = ip
    lib.lstm_test_last_paths.argtypes = [ctypes.POINTER(ip), ctypes.POINTER(ip)]
    lib.lstm_test_last_paths.restype = ip
    lib.lstm_test_last_stack_chunks.argtypes = [ctypes.POINTER(ip), ctypes.POINTER(ip)]
    lib.lstm_test_last_stack_chunks.restype = ip
    lib.lstm_test_last_persist_split.argtypes = [ctypes.POINTER(ip), ctypes.POINTER(ip)]
    lib.lstm_test_last_persist_split.restype = ip
    lib.lstm_test_bwd_chunks.argtypes = [ip]
    lib.lstm_test_bwd_chunks.restype = ip
    lib.lstm_test_chunk_bound.argtypes = [ip, ip, ip]
    lib.lstm_test_chunk_bound.restype = ip
    v = lib.lstm_abi_version()
    if v // 100 != ABI_VERSION // 100 or v < ABI_VERSION:
        raise RuntimeError(f"{path}: ABI version {v}, this binding needs {ABI_VERSION} "
                           "(rebuild with `python -m backward_lstm_fwd_b200.build`)")
    if path == LIB_PATH:
        _lib = lib
    return lib


def strerror(code: int) -> str:
    try:
        return load().lstm_strerror(int(code)).decode()
    except RuntimeError:
        return "liblstm not loaded"


def dtype_code(dt: torch.dtype) -> int:
    if dt == torch.float32:
        return LSTM_F32
    if dt == torch.bfloat16:
        return LSTM_BF16
    if dt == torch.float16:
        return LSTM_F16
    raise ValueError(f"unsupported compute dtype {dt}")


def dims(T: int, B: int, I: int, H: int, dtype) -> Dims:
    code = dtype if isinstance(dtype, int) else dtype_code(dtype)
    return Dims(int(T), int(B), int(I), int(H), code)


def _p(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr() if t.numel() > 0 else None


def _stream(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def fwd_workspace_size(d: Dims, mask=None, reverse: bool = False, gate_order="ifjo") -> int:
    """Forward workspace bytes for the plan this call takes on the current
    device (lstm_fwd_workspace_size, or _ex with the call's options)."""
    if _plain(mask, reverse, gate_order):
        return int(load().lstm_fwd_workspace_size(ctypes.byref(d)))
    opt = _options(mask, reverse, gate_order)
    return int(load().lstm_fwd_workspace_size_ex(ctypes.byref(d), ctypes.byref(opt)))


def fwd_workspace_size_max(d: Dims) -> int:
    """Forward workspace bytes that cover every plan on every device."""
    return int(load().lstm_fwd_workspace_size_max(ctypes.byref(d)))


def bwd_workspace_size(d: Dims) -> int:
    return int(load().lstm_bwd_workspace_size(ctypes.byref(d)))


def _gate_order(gate_order) -> int:
    """"ifjo" / "ijfo" (the attribute's values) or the C constant itself."""
    return GATE_ORDERS[gate_order] if isinstance(gate_order, str) else int(gate_order)


def _options(mask, reverse, gate_order):
    return Options(_p(mask), LSTM_DIR_REVERSE if reverse else LSTM_DIR_FORWARD,
                   _gate_order(gate_order))


def _plain(mask, reverse, gate_order) -> bool:
    return mask is None and not reverse and _gate_order(gate_order) == LSTM_GATES_IFJO


def lstm_fwd(d: Dims, x, W, b, h0, c0, y, hT, cT, gates, cells, ws, ws_bytes=None,
             stream=None, check: bool = True, mask=None, reverse: bool = False,
             gate_order="ifjo") -> int:
    """Direct call of the C entry point lstm_fwd, or lstm_fwd_ex with a
    variable-length mask [T,B,H] (1 = real step, 0 = padding), the reverse
    direction and / or gate_order "ijfo" (device tensors or raw pointers)."""
    if ws_bytes is None:
        ws_bytes = ws.numel() * ws.element_size() if ws is not None else 0
    if _plain(mask, reverse, gate_order):
        rc = load().lstm_fwd(ctypes.byref(d), _p(x), _p(W), _p(b), _p(h0), _p(c0), _p(y),
                             _p(hT), _p(cT), _p(gates), _p(cells), _p(ws), ws_bytes,
                             _stream(stream))
    else:
        opt = _options(mask, reverse, gate_order)
        rc = load().lstm_fwd_ex(ctypes.byref(d), ctypes.byref(opt), _p(x), _p(W), _p(b), _p(h0),
                                _p(c0), _p(y), _p(hT), _p(cT), _p(gates), _p(cells), _p(ws),
                                ws_bytes, _stream(stream))
    if check and rc != LSTM_OK:
        raise LstmError(rc, "lstm_fwd")
    return rc


def lstm_bwd(d: Dims, dy, dhT, dcT, x, W, h0, c0, y, gates, cells, dx, dW, db, dh0, dc0, ws,
             ws_bytes=None, stream=None, check: bool = True, mask=None,
             reverse: bool = False, gate_order="ifjo") -> int:
    """Direct call of the C entry point lstm_bwd, or lstm_bwd_ex with the
    forward's mask, direction and gate_order (device tensors or raw pointers)."""
    if ws_bytes is None:
        ws_bytes = ws.numel() * ws.element_size() if ws is not None else 0
    if _plain(mask, reverse, gate_order):
        rc = load().lstm_bwd(ctypes.byref(d), _p(dy), _p(dhT), _p(dcT), _p(x), _p(W), _p(h0),
                             _p(c0), _p(y), _p(gates), _p(cells), _p(dx), _p(dW), _p(db),
                             _p(dh0), _p(dc0), _p(ws), ws_bytes, _stream(stream))
    else:
        opt = _options(mask, reverse, gate_order)
        rc = load().lstm_bwd_ex(ctypes.byref(d), ctypes.byref(opt), _p(dy), _p(dhT), _p(dcT),
                                _p(x), _p(W), _p(h0), _p(c0), _p(y), _p(gates), _p(cells),
                                _p(dx), _p(dW), _p(db), _p(dh0), _p(dc0), _p(ws), ws_bytes,
                                _stream(stream))
    if check and rc != LSTM_OK:
        raise LstmError(rc, "lstm_bwd")
    return rc


NOALLOC_SCRATCH_BYTES = 32 * 1024 * 1024


def _ptr_array(ts):
    """A host array of device pointers (None, a tensor or an int per entry);
    None for no array at all."""
    if ts is None:
        return None
    return (ctypes.c_void_p * len(ts))(*[_p(t) for t in ts])


def stack_fwd_workspace_size(d: Dims, L: int) -> int:
    return int(load().lstm_stack_fwd_workspace_size(ctypes.byref(d), int(L)))


def stack_bwd_workspace_size(d: Dims, L: int) -> int:
    return int(load().lstm_stack_bwd_workspace_size(ctypes.byref(d), int(L)))


def stack_bwd_workspace_size_min(d: Dims, L: int) -> int:
    """The smallest workspace lstm_stack_bwd accepts (layers one after another)."""
    return int(load().lstm_stack_bwd_workspace_size_min(ctypes.byref(d), int(L)))


def lstm_stack_fwd(d: Dims, L: int, x, Ws, bs, h0, c0, y, hT, cT, gates, cells, ws,
                   ws_bytes=None, stream=None, check: bool = True, mask=None,
                   reverse: bool = False, gate_order="ifjo") -> int:
    """Direct call of lstm_stack_fwd: Ws / bs are lists of L device tensors
    (bs may be None); the [L][...] arrays are single tensors."""
    if ws_bytes is None:
        ws_bytes = ws.numel() * ws.element_size() if ws is not None else 0
    opt = _options(mask, reverse, gate_order)
    Wa, ba = _ptr_array(Ws), _ptr_array(bs)
    rc = load().lstm_stack_fwd(ctypes.byref(d), int(L), ctypes.byref(opt), _p(x), Wa, ba, _p(h0),
                               _p(c0), _p(y), _p(hT), _p(cT), _p(gates), _p(cells), _p(ws),
                               ws_bytes, _stream(stream))
    if check and rc != LSTM_OK:
        raise LstmError(rc, "lstm_stack_fwd")
    return rc


def lstm_stack_bwd(d: Dims, L: int, dy, dhT, dcT, x, Ws, h0, c0, y, gates, cells, dx, dWs, dbs,
                   dh0, dc0, ws, ws_bytes=None, stream=None, check: bool = True, mask=None,
                   reverse: bool = False, gate_order="ifjo") -> int:
    """Direct call of lstm_stack_bwd: Ws, dWs and dbs are lists of L device
    tensors."""
    if ws_bytes is None:
        ws_bytes = ws.numel() * ws.element_size() if ws is not None else 0
    opt = _options(mask, reverse, gate_order)
    Wa, dWa, dba = _ptr_array(Ws), _ptr_array(dWs), _ptr_array(dbs)
    rc = load().lstm_stack_bwd(ctypes.byref(d), int(L), ctypes.byref(opt), _p(dy), _p(dhT),
                               _p(dcT), _p(x), Wa, _p(h0), _p(c0), _p(y), _p(gates), _p(cells),
                               _p(dx), dWa, dba, _p(dh0), _p(dc0), _p(ws), ws_bytes,
                               _stream(stream))
    if check and rc != LSTM_OK:
        raise LstmError(rc, "lstm_stack_bwd")
    return rc


def lstm_fwd_noalloc(d: Dims, x, W, b, h0, c0, y, hT, cT, gates, cells, stream=None,
                     check: bool = True) -> int:
    """Direct call of lstm_fwd_noalloc: lstm_fwd with the library's static
    device scratch instead of a caller workspace (for callers that may not
    allocate device memory)."""
    rc = load().lstm_fwd_noalloc(ctypes.byref(d), _p(x), _p(W), _p(b), _p(h0), _p(c0), _p(y),
                                 _p(hT), _p(cT), _p(gates), _p(cells), _stream(stream))
    if check and rc != LSTM_OK:
        raise LstmError(rc, "lstm_fwd_noalloc")
    return rc


def lstm_fwd_noalloc_status(stream=None) -> int:
    """Synchronise `stream`, then read and clear the status word of the static
    scratch lstm_fwd_noalloc uses on the current device."""
    return int(load().lstm_fwd_noalloc_status(_stream(stream)))


def lstm_status(ws, ws_bytes=None, stream=None) -> int:
    if ws_bytes is None:
        ws_bytes = ws.numel() * ws.element_size()
    return int(load().lstm_status(_p(ws), ws_bytes, _stream(stream)))


def profile_begin() -> None:
    load().lstm_profile_begin()


def profile_end():
    """Per-phase (device ms, kernel launches) since profile_begin()."""
    n = len(PHASES)
    ms = (ctypes.c_double * n)()
    la = (ctypes.c_longlong * n)()
    rc = load().lstm_profile_end(ms, la)
    if rc != LSTM_OK:
        raise LstmError(rc, "lstm_profile_end")
    return {p: (ms[i], la[i]) for i, p in enumerate(PHASES)}


def launch_count() -> int:
    return int(load().lstm_launch_count())


def test_tc_gemm(M, N, K, A, lda, a_mn_major, Bm, ldb, b_mn_major, bias, C, ldc, ws,
                 stream=None) -> int:
    """Test hook (include/liblstm_testing.h): C = A B^T (+ bias) on the tcgen05 core."""
    return int(load().lstm_test_tc_gemm(M, N, K, _p(A), lda, a_mn_major, _p(Bm), ldb, b_mn_major,
                                         _p(bias), _p(C), ldc, _p(ws),
                                         ws.numel() * ws.element_size(), _stream(stream)))


def test_set_wait_fault(skip_cta: int, wait_ns: int) -> None:
    """Test hook: CTA `skip_cta` of persistent launches never arrives (-1: off);
    device-side waits give up after wait_ns (<= 0: default 2 s)."""
    load().lstm_test_set_wait_fault(int(skip_cta), int(wait_ns))


def test_last_paths():
    """Test hook: (forward, backward) recurrent kernel of the last calls:
    0 per-step CUDA cores, 1 persistent K-resident, 2 persistent cluster."""
    f, b = ctypes.c_int(), ctypes.c_int()
    load().lstm_test_last_paths(ctypes.byref(f), ctypes.byref(b))
    return f.value, b.value


def test_last_stack_chunks():
    """Test hook: (forward, backward) chunks per layer of the last stack calls'
    layer wavefronts (0: layer after layer; -1: no such call yet)."""
    f, b = ctypes.c_int(), ctypes.c_int()
    load().lstm_test_last_stack_chunks(ctypes.byref(f), ctypes.byref(b))
    return f.value, b.value


def test_last_persist_split():
    """Test hook: (forward, backward) cluster size of the last persistent
    CUDA-core recurrences (0: none yet)."""
    f, b = ctypes.c_int(), ctypes.c_int()
    load().lstm_test_last_persist_split(ctypes.byref(f), ctypes.byref(b))
    return f.value, b.value


# ------------------------------------------------------------------ helpers
def empty_workspace(nbytes: int, device) -> torch.Tensor:
    """A byte tensor usable as workspace (torch's allocator returns 256-byte
    aligned blocks)."""
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


class State:
    """Outputs of one forward call (device tensors), kept for the backward."""

    def __init__(self, T, B, I, H, cd, device):
        self.dims = dims(T, B, I, H, cd)
        self.y = torch.empty((T, B, H), dtype=cd, device=device)
        self.hT = torch.empty((B, H), dtype=cd, device=device)
        self.cT = torch.empty((B, H), dtype=torch.float32, device=device)
        self.gates = torch.empty((T, B, 4 * H), dtype=cd, device=device)
        self.cells = torch.empty((T, B, H), dtype=torch.float32, device=device)


class Grads:
    def __init__(self, T, B, I, H, device):
        f = torch.float32
        self.dx = torch.empty((T, B, I), dtype=f, device=device)
        self.dW = torch.empty((4 * H, H + I), dtype=f, device=device)
        self.db = torch.empty((4 * H,), dtype=f, device=device)
        self.dh0 = torch.empty((B, H), dtype=f, device=device)
        self.dc0 = torch.empty((B, H), dtype=f, device=device)


def forward(x, W, b=None, h0=None, c0=None, ws=None, stream=None, mask=None,
            reverse: bool = False, gate_order="ifjo") -> State:
    """Allocate outputs and run lstm_fwd (lstm_fwd_ex with a mask, the
    reverse direction or gate_order "ijfo").  x [T,B,I], W [4H,H+I] and mask [T,B,H] share the
    compute dtype (float32 or bfloat16); c0 is float32."""
    T, B, I = x.shape
    H = W.shape[0] // 4
    st = State(T, B, I, H, x.dtype, x.device)
    if ws is None:
        ws = empty_workspace(fwd_workspace_size(st.dims, mask, reverse, gate_order), x.device)
    lstm_fwd(st.dims, x, W, b, h0, c0, st.y, st.hT, st.cT, st.gates, st.cells, ws, stream=stream,
             mask=mask, reverse=reverse, gate_order=gate_order)
    return st


def backward(st: State, x, W, h0=None, c0=None, dy=None, dhT=None, dcT=None, ws=None,
             stream=None, mask=None, reverse: bool = False, gate_order="ifjo") -> Grads:
    """Allocate gradients and run lstm_bwd on the saved state of forward()
    (lstm_bwd_ex with the forward's mask, direction and gate_order)."""
    T, B, I = x.shape
    H = W.shape[0] // 4
    g = Grads(T, B, I, H, x.device)
    if ws is None:
        ws = empty_workspace(bwd_workspace_size(st.dims), x.device)
    lstm_bwd(st.dims, dy, dhT, dcT, x, W, h0, c0, st.y, st.gates, st.cells, g.dx, g.dW, g.db,
             g.dh0, g.dc0, ws, stream=stream, mask=mask, reverse=reverse,
             gate_order=gate_order)
    return g


class StackState:
    """Outputs of one lstm_stack_fwd call: every layer's saved state."""

    def __init__(self, L, T, B, I, H, cd, device):
        self.L = L
        self.dims = dims(T, B, I, H, cd)
        self.y = torch.empty((L, T, B, H), dtype=cd, device=device)
        self.hT = torch.empty((L, B, H), dtype=cd, device=device)
        self.cT = torch.empty((L, B, H), dtype=torch.float32, device=device)
        self.gates = torch.empty((L, T, B, 4 * H), dtype=cd, device=device)
        self.cells = torch.empty((L, T, B, H), dtype=torch.float32, device=device)


class StackGrads:
    def __init__(self, L, T, B, I, H, device):
        f = torch.float32
        self.dx = torch.empty((T, B, I), dtype=f, device=device)
        self.dW = [torch.empty((4 * H, H + (I if l == 0 else H)), dtype=f, device=device)
                   for l in range(L)]
        self.db = [torch.empty((4 * H,), dtype=f, device=device) for _ in range(L)]
        self.dh0 = torch.empty((L, B, H), dtype=f, device=device)
        self.dc0 = torch.empty((L, B, H), dtype=f, device=device)


def forward_stack(x, Ws, bs=None, h0=None, c0=None, ws=None, stream=None, mask=None,
                  reverse: bool = False, gate_order="ifjo") -> StackState:
    """Allocate outputs and run lstm_stack_fwd.  x [T,B,I]; Ws[l] [4H, H+I_l];
    h0 [L,B,H] (compute dtype), c0 [L,B,H] float32."""
    T, B, I = x.shape
    L, H = len(Ws), Ws[0].shape[0] // 4
    st = StackState(L, T, B, I, H, x.dtype, x.device)
    if ws is None:
        ws = empty_workspace(stack_fwd_workspace_size(st.dims, L), x.device)
    lstm_stack_fwd(st.dims, L, x, Ws, bs, h0, c0, st.y, st.hT, st.cT, st.gates, st.cells, ws,
                   stream=stream, mask=mask, reverse=reverse, gate_order=gate_order)
    return st


def backward_stack(st: StackState, x, Ws, h0=None, c0=None, dy=None, dhT=None, dcT=None,
                   ws=None, stream=None, mask=None, reverse: bool = False,
                   gate_order="ifjo") -> StackGrads:
    """Allocate gradients and run lstm_stack_bwd on the saved state of
    forward_stack()."""
    T, B, I = x.shape
    L, H = len(Ws), Ws[0].shape[0] // 4
    g = StackGrads(L, T, B, I, H, x.device)
    if ws is None:
        ws = empty_workspace(stack_bwd_workspace_size(st.dims, L), x.device)
    lstm_stack_bwd(st.dims, L, dy, dhT, dcT, x, Ws, h0, c0, st.y, st.gates, st.cells, g.dx, g.dW,
                   g.db, g.dh0, g.dc0, ws, stream=stream, mask=mask, reverse=reverse,
                   gate_order=gate_order)
    return g
