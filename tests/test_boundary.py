"""The C ABI boundary, checked without a GPU: the library loads, exports every
function include/liblstm.h declares, sizes its workspaces, and rejects bad
arguments with a status code before it enqueues anything.  (Every rejected call
below returns before its first CUDA runtime call, so none needs a device.)"""
import ctypes
import os
import re

import pytest
import torch

from backward_lstm_fwd_b200 import build as lbuild
from backward_lstm_fwd_b200 import binding as L

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "liblstm.h")

FAKE = 0x10000  # a 16-byte aligned address that is never dereferenced


@pytest.fixture(scope="module")
def lib():
    lbuild.build()
    return L.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(lstm_\w+)\s*\(", text)))


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert set(names) >= set(L.EXPORTS)
    for n in names:
        assert hasattr(lib, n), f"{n} declared in liblstm.h but not exported"
    assert lib.lstm_abi_version() == L.ABI_VERSION == 103


def declared_arities():
    """{function: number of parameters} of every prototype in liblstm.h (the
    testing header's too)."""
    out = {}
    for h in (HEADER, HEADER.replace("liblstm.h", "liblstm_testing.h")):
        text = re.sub(r"/\*.*?\*/", "", open(h).read(), flags=re.S)
        for name, args in re.findall(r"\b(lstm_\w+)\s*\(([^;{]*?)\)\s*;", text, flags=re.S):
            args = args.strip()
            out[name] = 0 if args in ("", "void") else args.count(",") + 1
    return out


def test_binding_argument_counts_match_the_headers(lib):
    """Every prototype the binding types has as many ctypes argtypes as the
    header has parameters (drift between the two would pass garbage)."""
    arity = declared_arities()
    assert "lstm_stack_bwd" in arity and "lstm_test_tc_gemm" in arity
    for name, n in arity.items():
        argtypes = getattr(lib, name).argtypes
        assert argtypes is not None, name
        assert len(argtypes) == n, (name, len(argtypes), n)


def test_strerror(lib):
    for code in range(7):
        assert L.strerror(code)
    assert L.strerror(99) == "unknown status"


def test_workspace_sizes(lib):
    d = L.dims(256, 128, 1024, 1024, L.LSTM_BF16)
    fmax, bw = L.fwd_workspace_size_max(d), L.bwd_workspace_size(d)
    TB, G4 = 256 * 128, 4 * 1024
    assert fmax >= 256 + TB * G4 * 4 and fmax % 256 == 0
    assert bw >= 256 + TB * G4 * 2 and bw % 256 == 0
    # the plan-aware size: the control block alone (fused forward on a device
    # where it fits) or the whole layout; without a device, the whole layout
    fw = L.fwd_workspace_size(d)
    assert fw in (256, fmax)
    if not torch.cuda.is_available():
        assert fw == fmax
    mask_opt = L.Options(FAKE, L.LSTM_DIR_FORWARD, L.LSTM_GATES_IFJO)
    assert lib.lstm_fwd_workspace_size_ex(ctypes.byref(d), ctypes.byref(mask_opt)) in (256, fmax)
    assert lib.lstm_fwd_workspace_size_ex(ctypes.byref(d), None) == fw
    for q in (L.fwd_workspace_size, L.fwd_workspace_size_max):
        assert q(L.dims(-1, 2, 3, 4, 0)) == 0
        assert q(L.dims(0, 0, 0, 0, 0)) >= 256
    assert L.bwd_workspace_size(L.dims(1, 2, 3, 4, 7)) == 0
    # fp16 has bf16's layout (two-byte dG, W_h^T, per-group db partials)
    h = L.dims(256, 128, 1024, 1024, L.LSTM_F16)
    assert L.fwd_workspace_size_max(h) == fmax and L.bwd_workspace_size(h) == bw
    # fp32 keeps dG in fp32 and needs no W_h^T copy
    f = L.dims(256, 128, 1024, 1024, L.LSTM_F32)
    assert L.bwd_workspace_size(f) >= 256 + TB * G4 * 4


def fwd_args(d, **over):
    a = dict(x=FAKE, W=FAKE, b=None, h0=None, c0=None, y=FAKE, hT=FAKE, cT=FAKE, gates=FAKE,
             cells=FAKE, ws=FAKE, ws_bytes=L.fwd_workspace_size(d))
    a.update(over)
    return a


def call_fwd(d, **over):
    a = fwd_args(d, **over)
    return L.lstm_fwd(d, a["x"], a["W"], a["b"], a["h0"], a["c0"], a["y"], a["hT"], a["cT"],
                      a["gates"], a["cells"], a["ws"], ws_bytes=a["ws_bytes"], stream=0,
                      check=False)


def call_bwd(d, **over):
    a = dict(dy=None, dhT=None, dcT=None, x=FAKE, W=FAKE, h0=None, c0=None, y=FAKE, gates=FAKE,
             cells=FAKE, dx=FAKE, dW=FAKE, db=FAKE, dh0=FAKE, dc0=FAKE, ws=FAKE,
             ws_bytes=L.bwd_workspace_size(d))
    a.update(over)
    return L.lstm_bwd(d, a["dy"], a["dhT"], a["dcT"], a["x"], a["W"], a["h0"], a["c0"], a["y"],
                      a["gates"], a["cells"], a["dx"], a["dW"], a["db"], a["dh0"], a["dc0"],
                      a["ws"], ws_bytes=a["ws_bytes"], stream=0, check=False)


D = L.dims(4, 3, 5, 8, L.LSTM_F32)


@pytest.mark.parametrize("bad", [
    L.dims(-1, 3, 5, 8, 0), L.dims(4, -3, 5, 8, 0), L.dims(4, 3, -5, 8, 0),
    L.dims(4, 3, 5, -8, 0), L.dims(4, 3, 5, 8, 3), L.dims(4, 3, 5, 8, -1),
    L.dims(1 << 20, 1 << 12, 5, 8, 0),
    L.dims(1, 1, 5, 1 << 29, 0),
])
def test_bad_dims(lib, bad):
    assert call_fwd(bad, ws_bytes=1 << 30) == L.LSTM_ERR_INVALID_ARG
    assert call_bwd(bad, ws_bytes=1 << 30) == L.LSTM_ERR_INVALID_ARG


def test_unsupported_extent(lib):
    d = L.dims(1, 1, 5, 1 << 21, 0)
    assert call_fwd(d, ws_bytes=1 << 40) == L.LSTM_ERR_UNSUPPORTED
    assert call_bwd(d, ws_bytes=1 << 40) == L.LSTM_ERR_UNSUPPORTED


def test_null_dims_pointer(lib):
    rc = lib.lstm_fwd(None, *([None] * 10), None, 0, None)
    assert rc == L.LSTM_ERR_INVALID_ARG


@pytest.mark.parametrize("name", ["x", "W", "y", "hT", "cT", "gates", "cells"])
def test_fwd_required_pointer_null(lib, name):
    assert call_fwd(D, **{name: None}) == L.LSTM_ERR_INVALID_ARG


@pytest.mark.parametrize("name", ["x", "W", "b", "h0", "c0", "y", "hT", "cT", "gates", "cells"])
def test_fwd_misaligned_pointer(lib, name):
    assert call_fwd(D, **{name: FAKE + 4}) == L.LSTM_ERR_INVALID_ARG


@pytest.mark.parametrize("name", ["x", "W", "y", "gates", "cells", "dx", "dW", "db", "dh0", "dc0"])
def test_bwd_required_pointer_null(lib, name):
    assert call_bwd(D, **{name: None}) == L.LSTM_ERR_INVALID_ARG


@pytest.mark.parametrize("name", ["dy", "dhT", "dcT", "x", "W", "h0", "c0", "y", "gates",
                                  "cells", "dx", "dW", "db", "dh0", "dc0"])
def test_bwd_misaligned_pointer(lib, name):
    assert call_bwd(D, **{name: FAKE + 8}) == L.LSTM_ERR_INVALID_ARG


def test_workspace_errors(lib):
    need = L.fwd_workspace_size(D)
    assert call_fwd(D, ws=None) == L.LSTM_ERR_WORKSPACE
    assert call_fwd(D, ws_bytes=need - 1) == L.LSTM_ERR_WORKSPACE
    assert call_fwd(D, ws=FAKE + 16) == L.LSTM_ERR_WORKSPACE
    need = L.bwd_workspace_size(D)
    assert call_bwd(D, ws=None) == L.LSTM_ERR_WORKSPACE
    assert call_bwd(D, ws_bytes=need - 1) == L.LSTM_ERR_WORKSPACE
    assert call_bwd(D, ws=FAKE + 128) == L.LSTM_ERR_WORKSPACE


def test_empty_problem_needs_no_data_pointers(lib):
    # With T*B == 0 only the workspace is touched; the outputs hT/cT are
    # still required when B*H > 0.
    d = L.dims(0, 0, 5, 8, L.LSTM_F32)
    assert call_fwd(d, x=None, y=None, gates=None, cells=None, hT=None, cT=None,
                    ws=None) == L.LSTM_ERR_WORKSPACE
    d = L.dims(0, 3, 5, 8, L.LSTM_F32)
    assert call_fwd(d, x=None, y=None, gates=None, cells=None, hT=None) == L.LSTM_ERR_INVALID_ARG


def test_status_argument_checks(lib):
    assert lib.lstm_status(None, 256, None) == L.LSTM_ERR_INVALID_ARG
    assert lib.lstm_status(FAKE, 16, None) == L.LSTM_ERR_INVALID_ARG
    assert lib.lstm_status(FAKE + 16, 4096, None) == L.LSTM_ERR_INVALID_ARG


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(RuntimeError):
        L.load(str(tmp_path / "nope.so"))


@pytest.mark.parametrize("direction", [-1, 2, 7])
def test_unknown_direction_rejected(lib, direction):
    """lstm_fwd_ex / lstm_bwd_ex reject a direction other than LSTM_DIR_FORWARD /
    LSTM_DIR_REVERSE before anything is enqueued."""
    opt = L.Options(None, direction)
    a = fwd_args(D)
    rc = lib.lstm_fwd_ex(ctypes.byref(D), ctypes.byref(opt), a["x"], a["W"], a["b"], a["h0"],
                         a["c0"], a["y"], a["hT"], a["cT"], a["gates"], a["cells"], a["ws"],
                         a["ws_bytes"], None)
    assert rc == L.LSTM_ERR_INVALID_ARG
    rc = lib.lstm_bwd_ex(ctypes.byref(D), ctypes.byref(opt), None, None, None, FAKE, FAKE, None,
                         None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                         L.bwd_workspace_size(D), None)
    assert rc == L.LSTM_ERR_INVALID_ARG


@pytest.mark.parametrize("order", [-1, 2, 5])
def test_unknown_gate_order_rejected(lib, order):
    """lstm_fwd_ex / lstm_bwd_ex reject a gate_order other than LSTM_GATES_IFJO /
    LSTM_GATES_IJFO before anything is enqueued."""
    opt = L.Options(None, L.LSTM_DIR_FORWARD, order)
    a = fwd_args(D)
    rc = lib.lstm_fwd_ex(ctypes.byref(D), ctypes.byref(opt), a["x"], a["W"], a["b"], a["h0"],
                         a["c0"], a["y"], a["hT"], a["cT"], a["gates"], a["cells"], a["ws"],
                         a["ws_bytes"], None)
    assert rc == L.LSTM_ERR_INVALID_ARG
    rc = lib.lstm_bwd_ex(ctypes.byref(D), ctypes.byref(opt), None, None, None, FAKE, FAKE, None,
                         None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                         L.bwd_workspace_size(D), None)
    assert rc == L.LSTM_ERR_INVALID_ARG


def test_options_layout_matches_header():
    """The ctypes mirror of lstm_options has the C layout: a pointer, then the
    two ints (no padding between them)."""
    assert L.Options.seq_mask.offset == 0
    assert L.Options.direction.offset == ctypes.sizeof(ctypes.c_void_p)
    assert L.Options.gate_order.offset == ctypes.sizeof(ctypes.c_void_p) + 4
    assert ctypes.sizeof(L.Options) == ctypes.sizeof(ctypes.c_void_p) + 8


def test_misaligned_mask_rejected(lib):
    opt = L.Options(FAKE + 2, L.LSTM_DIR_FORWARD)
    a = fwd_args(D)
    rc = lib.lstm_fwd_ex(ctypes.byref(D), ctypes.byref(opt), a["x"], a["W"], a["b"], a["h0"],
                         a["c0"], a["y"], a["hT"], a["cT"], a["gates"], a["cells"], a["ws"],
                         a["ws_bytes"], None)
    assert rc == L.LSTM_ERR_INVALID_ARG


# ----------------------------------------------------------- stacked layers
DS = L.dims(4, 8, 16, 32, L.LSTM_BF16)


def call_stack_fwd(d, Lc, Ws=(FAKE, FAKE), bs=None, ws_bytes=None):
    if ws_bytes is None:
        ws_bytes = L.stack_fwd_workspace_size(d, max(Lc, 1))
    return L.lstm_stack_fwd(d, Lc, FAKE, None if Ws is None else list(Ws), bs, None, None, FAKE,
                            FAKE, FAKE, FAKE, FAKE, FAKE, ws_bytes=ws_bytes, stream=0,
                            check=False)


def call_stack_bwd(d, Lc, Ws=(FAKE, FAKE), dWs=(FAKE, FAKE), dbs=(FAKE, FAKE), ws_bytes=None):
    if ws_bytes is None:
        ws_bytes = L.stack_bwd_workspace_size(d, max(Lc, 1))
    return L.lstm_stack_bwd(d, Lc, FAKE, None, None, FAKE, None if Ws is None else list(Ws),
                            None, None, FAKE, FAKE, FAKE, FAKE,
                            None if dWs is None else list(dWs),
                            None if dbs is None else list(dbs), FAKE, FAKE, FAKE,
                            ws_bytes=ws_bytes, stream=0, check=False)


def test_stack_workspace_sizes(lib):
    one = L.bwd_workspace_size(DS)
    upper = L.bwd_workspace_size(L.dims(4, 8, 32, 32, L.LSTM_BF16))
    assert L.stack_fwd_workspace_size(DS, 1) == L.fwd_workspace_size_max(DS)
    assert L.stack_bwd_workspace_size(DS, 1) == one
    assert L.stack_bwd_workspace_size_min(DS, 1) == one
    # two layers, one after another: the larger layer's workspace plus dx
    # (float) and dy (bf16) of the upper layer, [T][B][H] each
    need = max(one, upper) + 4 * 8 * 32 * (4 + 2)
    assert L.stack_bwd_workspace_size_min(DS, 2) >= need
    # the layer wavefront: the control block and a workspace per layer, plus
    # those two buffers between each pair of layers
    for Lc in (2, 3):
        wave = 256 + Lc * max(one, upper) + (Lc - 1) * 4 * 8 * 32 * (4 + 2)
        assert L.stack_bwd_workspace_size(DS, Lc) >= wave
        assert L.stack_bwd_workspace_size(DS, Lc) > L.stack_bwd_workspace_size_min(DS, Lc)
    # float stacks run layer after layer only
    DF = L.dims(4, 8, 16, 32, L.LSTM_F32)
    assert L.stack_bwd_workspace_size(DF, 2) == L.stack_bwd_workspace_size_min(DF, 2)
    assert L.stack_bwd_workspace_size(DS, 0) == 0 and L.stack_fwd_workspace_size(DS, -1) == 0
    assert L.stack_bwd_workspace_size_min(DS, 0) == 0


@pytest.mark.parametrize("Lc", [0, -2])
def test_stack_layer_count_rejected(lib, Lc):
    assert call_stack_fwd(DS, Lc, ws_bytes=1 << 20) == L.LSTM_ERR_INVALID_ARG
    assert call_stack_bwd(DS, Lc, ws_bytes=1 << 20) == L.LSTM_ERR_INVALID_ARG


def test_stack_parameter_arrays_checked_before_any_layer(lib):
    """A missing or misaligned W / dW / db of any layer is reported before the
    first layer is enqueued."""
    assert call_stack_fwd(DS, 2, Ws=None) == L.LSTM_ERR_INVALID_ARG
    assert call_stack_fwd(DS, 2, Ws=(FAKE, None)) == L.LSTM_ERR_INVALID_ARG
    assert call_stack_fwd(DS, 2, Ws=(FAKE, FAKE + 2)) == L.LSTM_ERR_INVALID_ARG
    assert call_stack_fwd(DS, 2, bs=[None, FAKE + 4]) == L.LSTM_ERR_INVALID_ARG
    assert call_stack_bwd(DS, 2, dWs=(FAKE, None)) == L.LSTM_ERR_INVALID_ARG
    assert call_stack_bwd(DS, 2, dbs=None) == L.LSTM_ERR_INVALID_ARG
    assert call_stack_bwd(DS, 2, Ws=(None, FAKE)) == L.LSTM_ERR_INVALID_ARG


def test_stack_slices_must_align(lib):
    d = L.dims(4, 3, 16, 12, L.LSTM_BF16)  # B*H = 36: per-layer slices off 16 bytes
    assert call_stack_fwd(d, 2) == L.LSTM_ERR_UNSUPPORTED
    assert call_stack_bwd(d, 2) == L.LSTM_ERR_UNSUPPORTED


def test_stack_workspace_too_small(lib):
    need = L.stack_bwd_workspace_size_min(DS, 2)
    assert call_stack_bwd(DS, 2, ws_bytes=need - 1) == L.LSTM_ERR_WORKSPACE


def test_option_marshalling():
    """The binding's option struct: direction and gate_order constants, the
    attribute spellings, and when the plain entry points are used."""
    assert L._gate_order("ifjo") == L.LSTM_GATES_IFJO and L._gate_order("ijfo") == L.LSTM_GATES_IJFO
    assert L._gate_order(7) == 7  # raw values pass through (the library rejects them)
    with pytest.raises(KeyError):
        L._gate_order("iofj")
    o = L._options(None, True, "ijfo")
    assert o.seq_mask is None and o.direction == L.LSTM_DIR_REVERSE
    assert o.gate_order == L.LSTM_GATES_IJFO
    assert L._plain(None, False, "ifjo")
    assert not L._plain(None, True, "ifjo") and not L._plain(None, False, "ijfo")
    assert not L._plain(FAKE, False, "ifjo")


def test_dtype_codes():
    import torch
    assert L.dtype_code(torch.float32) == L.LSTM_F32
    assert L.dtype_code(torch.bfloat16) == L.LSTM_BF16
    assert L.dtype_code(torch.float16) == L.LSTM_F16
    with pytest.raises(ValueError):
        L.dtype_code(torch.float64)


def test_backward_chunking_host_logic(lib, monkeypatch):
    """The reverse-time chunks of the tensor-core backward (host logic, no
    GPU): min(6, T/16) chunks from T = 32 on, one below; boundaries strictly
    increasing from 0 to T; sizes shrinking geometrically, so that the last
    chunk (whose dW / dx GEMM runs alone) is the smallest."""
    monkeypatch.delenv("LSTM_BWD_CHUNKS", raising=False)
    assert lib.lstm_test_bwd_chunks(-1) == -1
    for T in list(range(0, 300)) + [1024, 4096]:
        n = lib.lstm_test_bwd_chunks(T)
        assert n == (min(6, T // 16) if T >= 32 else 1), T
        b = [lib.lstm_test_chunk_bound(T, n, c) for c in range(n + 1)]
        assert b[0] == 0 and b[-1] == T, (T, b)
        if T >= n:
            assert all(b[i + 1] > b[i] for i in range(n)), (T, b)
        sizes = [b[i + 1] - b[i] for i in range(n)]
        if n > 1 and T >= 64:
            assert sizes[-1] == min(sizes) and sizes[0] == max(sizes), (T, sizes)
    assert [lib.lstm_test_chunk_bound(256, 8, c) for c in range(9)] == \
        [0, 62, 111, 150, 182, 207, 227, 243, 256]
    assert lib.lstm_test_chunk_bound(10, 2, 3) == -1  # c > nch


def test_environment_switches_are_the_documented_ones():
    """Every environment variable the library reads is listed in
    liblstm_testing.h, and every listed one is read."""
    src = open(os.path.join(ROOT, "backward_lstm_fwd_b200", "csrc", "liblstm.cu")).read()
    read = set(re.findall(r'(?:getenv|env_is)\("([A-Z0-9_]+)"', src))
    hdr = open(HEADER.replace("liblstm.h", "liblstm_testing.h")).read()
    listed = set(re.findall(r"^ \*   (LSTM_[A-Z0-9_]+)=", hdr, flags=re.M))
    listed |= {"CUDA_INJECTION64_PATH", "NV_COMPUTE_PROFILER_PERFWORKS_DIR"}
    assert read == listed, (sorted(read), sorted(listed))


def test_backward_workspace_holds_the_split_k_partials(lib):
    """The CUDA-core dW splits its T*B rows into slabs when its 64 x 64 output
    tiles are too few to fill the device (the fp32 workload T=64, B=32, I=H=256:
    128 tiles, 3 slabs); the slabs' fp32 partial products live in the backward
    workspace, whose size does not depend on the device.  At the bench size
    the tiles fill the device and no such region is reserved."""
    small = L.dims(64, 32, 256, 256, L.LSTM_F32)
    TB, G4, K = 64 * 32, 4 * 256, 256 + 256
    need = 256 + TB * G4 * 4 + 3 * G4 * K * 4
    assert L.bwd_workspace_size(small) >= need
    # and not much more: the other regions (db chunks, delta c / h buffers) are small
    assert L.bwd_workspace_size(small) < need + 2 * G4 * K * 4
    big = L.dims(256, 128, 1024, 1024, L.LSTM_BF16)
    TB, G4, K = 256 * 128, 4096, 2048
    assert L.bwd_workspace_size(big) < 256 + TB * G4 * 2 + G4 * K * 4
