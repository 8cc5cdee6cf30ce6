"""Thin ctypes binding of libtwell.so (argument marshalling only).

Every function here has the name of the C entry point it calls and does no
arithmetic of its own: it checks that the tensors are contiguous CUDA tensors,
packs their device pointers and sizes, calls the library on the current torch
stream, and raises ``TwellError`` on a non-OK status.  The small ``Twell`` and
``Hybrid`` classes only allocate the caller-owned buffers of the two sparse
formats with torch.  If the library cannot be loaded the first call raises:
there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtwell.so")

TW_F32, TW_BF16 = 0, 1
STATUS = ["TW_OK", "TW_ERR_INVALID_ARG", "TW_ERR_UNSUPPORTED", "TW_ERR_ALIGNMENT",
          "TW_ERR_CUDA", "TW_ERR_SPILL_CAPACITY", "TW_ERR_BACKUP_CAPACITY",
          "TW_ERR_TIMEOUT", "TW_ERR_WORKSPACE"]
EXPORTS = ["twell_gate_gemm", "twell_fused_updown_workspace_size", "twell_fused_updown",
           "twell_fused_updown_noalloc", "twell_ffn_small_batch_workspace_size",
           "twell_ffn_small_batch", "twell_to_hybrid", "hybrid_ffn_forward_workspace_size",
           "hybrid_ffn_forward",
           "hybrid_ffn_backward_workspace_size", "hybrid_ffn_backward", "dense_ffn_forward",
           "dense_ffn_train_workspace_size", "dense_ffn_train_saved_bytes",
           "dense_ffn_train_forward", "dense_ffn_train_backward",
           "tw_test_withhold_next_gate_loads", "tw_measure_row_gather", "tw_measure_stream_read", "tw_status_string",
           "twell_version"]


class TwellError(RuntimeError):
    def __init__(self, fn, code):
        name = STATUS[code] if 0 <= code < len(STATUS) else str(code)
        super().__init__(f"{fn} returned {name}")
        self.code = code


class TwTwellC(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("F", ctypes.c_int32), ("W", ctypes.c_int32),
                ("C", ctypes.c_int32), ("dtype", ctypes.c_int), ("val", ctypes.c_void_p),
                ("idx", ctypes.c_void_p), ("cnt", ctypes.c_void_p),
                ("spill_ref", ctypes.c_void_p), ("spill_cap", ctypes.c_int32),
                ("spill_tk", ctypes.c_void_p), ("spill_val", ctypes.c_void_p),
                ("spill_n", ctypes.c_void_p)]


class TwHybridC(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("F", ctypes.c_int32), ("C_h", ctypes.c_int32),
                ("dtype", ctypes.c_int), ("ell_g", ctypes.c_void_p), ("ell_u", ctypes.c_void_p),
                ("ell_idx", ctypes.c_void_p), ("row_nnz", ctypes.c_void_p),
                ("row_slot", ctypes.c_void_p), ("backup_cap", ctypes.c_int32),
                ("backup_rows", ctypes.c_void_p), ("backup_g", ctypes.c_void_p),
                ("backup_u", ctypes.c_void_p), ("n_backup", ctypes.c_void_p)]


_lib = None


def lib():
    """Load libtwell.so once; raise if it is missing (no fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m activation_sparse_transformer_tma_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, st = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int
        PT, PH = ctypes.POINTER(TwTwellC), ctypes.POINTER(TwHybridC)
        L.twell_gate_gemm.argtypes = [vp, vp, i32, i32, i32, ctypes.c_int, PT, vp, vp, vp]
        L.twell_fused_updown_workspace_size.argtypes = [i32, i32]
        L.twell_fused_updown_workspace_size.restype = ctypes.c_size_t
        L.twell_fused_updown.argtypes = [vp, PT, vp, vp, i32, vp, ctypes.c_int, vp,
                                         ctypes.c_size_t, vp, vp]
        L.twell_fused_updown_noalloc.argtypes = [vp, PT, vp, vp, i32, vp, ctypes.c_int, vp, vp]
        L.twell_fused_updown_noalloc.restype = st
        L.twell_ffn_small_batch_workspace_size.argtypes = [i32, i32, i32]
        L.twell_ffn_small_batch_workspace_size.restype = ctypes.c_size_t
        L.twell_ffn_small_batch.argtypes = [vp, vp, vp, vp, i32, i32, i32, PT, vp, vp,
                                            ctypes.c_int, vp, ctypes.c_size_t, vp, vp]
        L.twell_to_hybrid.argtypes = [PT, PH, vp, vp]
        L.hybrid_ffn_forward_workspace_size.argtypes = [i32, i32]
        L.hybrid_ffn_forward_workspace_size.restype = ctypes.c_size_t
        L.hybrid_ffn_forward.argtypes = [vp, PH, vp, vp, i32, vp, ctypes.c_int, vp,
                                         ctypes.c_size_t, vp, vp]
        L.hybrid_ffn_backward_workspace_size.argtypes = [i32, i32, i32, i32, i32]
        L.hybrid_ffn_backward_workspace_size.restype = ctypes.c_size_t
        L.hybrid_ffn_backward.argtypes = [vp, vp, PH, vp, vp, vp, i32, ctypes.c_float, vp,
                                          ctypes.c_int, vp, vp, vp, vp, ctypes.c_size_t, vp, vp]
        L.dense_ffn_forward.argtypes = [vp, vp, vp, vp, i32, i32, i32, vp, vp, vp, vp]
        L.dense_ffn_train_workspace_size.argtypes = [i32, i32]
        L.dense_ffn_train_workspace_size.restype = ctypes.c_size_t
        L.dense_ffn_train_saved_bytes.argtypes = [i32, i32]
        L.dense_ffn_train_saved_bytes.restype = ctypes.c_size_t
        L.dense_ffn_train_forward.argtypes = [vp, vp, vp, vp, i32, i32, i32, vp, ctypes.c_size_t,
                                              vp, vp, vp]
        L.dense_ffn_train_backward.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, ctypes.c_float,
                                               vp, ctypes.c_size_t, vp, vp, vp, vp, vp, vp]
        L.tw_test_withhold_next_gate_loads.argtypes = [ctypes.c_uint64]
        L.tw_test_withhold_next_gate_loads.restype = None
        L.tw_measure_row_gather.argtypes = [vp, i32, i32, ctypes.c_int64, ctypes.c_uint32, vp,
                                            vp]
        L.tw_measure_row_gather.restype = st
        L.tw_measure_stream_read.argtypes = [vp, ctypes.c_int64, vp, vp]
        L.tw_measure_stream_read.restype = st
        L.tw_status_string.argtypes = [st]
        L.tw_status_string.restype = ctypes.c_char_p
        L.twell_version.restype = i32
        for name in ("twell_gate_gemm", "twell_fused_updown", "twell_ffn_small_batch",
                     "twell_to_hybrid",
                     "hybrid_ffn_forward", "hybrid_ffn_backward", "dense_ffn_forward",
                     "dense_ffn_train_forward", "dense_ffn_train_backward"):
            getattr(L, name).restype = st
        _lib = L
    return _lib


# ------------------------------------------------------------------ helpers --
def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return TW_BF16
    if t.dtype == torch.float32:
        return TW_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _torch_dtype(code: int):
    return torch.bfloat16 if code == TW_BF16 else torch.float32


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError("tensors passed to libtwell must be contiguous CUDA tensors")
    return t.data_ptr()


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _check(fn, code):
    if code != 0:
        raise TwellError(fn, code)


class Twell:
    """Caller-owned buffers of one TwELL tensor (tile-major, W = 128)."""

    def __init__(self, T, F, C, dtype=torch.bfloat16, spill_cap=None, device="cuda", W=128):
        K = F // W
        if spill_cap is None:
            spill_cap = max(1024, (K * T) // 16)
        self.T, self.F, self.W, self.C, self.spill_cap = T, F, W, C, spill_cap
        self.dtype = dtype
        self.val = torch.zeros((K, T, C), dtype=dtype, device=device) if C else None
        self.idx = torch.zeros((K, T, C), dtype=torch.uint8, device=device) if C else None
        self.cnt = torch.zeros((K, T), dtype=torch.uint8, device=device)
        self.spill_ref = torch.full((K, T), -1, dtype=torch.int32, device=device)
        self.spill_tk = torch.zeros((max(spill_cap, 1), 2), dtype=torch.int32, device=device)
        self.spill_val = torch.zeros((max(spill_cap, 1), W), dtype=dtype, device=device)
        self.spill_n = torch.zeros(1, dtype=torch.int32, device=device)

    def struct(self):
        return TwTwellC(self.T, self.F, self.W, self.C, _dt(self.spill_val), _ptr(self.val),
                        _ptr(self.idx), _ptr(self.cnt), _ptr(self.spill_ref), self.spill_cap,
                        _ptr(self.spill_tk), _ptr(self.spill_val), _ptr(self.spill_n))


class Hybrid:
    """Caller-owned buffers of one hybrid tensor (ELL part + dense backup rows)."""

    def __init__(self, T, F, C_h, dtype=torch.bfloat16, backup_cap=None, device="cuda"):
        if backup_cap is None:
            backup_cap = max(64, T // 8)
        self.T, self.F, self.C_h, self.backup_cap = T, F, C_h, backup_cap
        self.dtype = dtype
        self.ell_g = torch.zeros((T, C_h), dtype=dtype, device=device)
        self.ell_u = torch.zeros((T, C_h), dtype=dtype, device=device)
        self.ell_idx = torch.zeros((T, C_h), dtype=torch.int16, device=device)
        self.row_nnz = torch.zeros(T, dtype=torch.int32, device=device)
        self.row_slot = torch.zeros(T, dtype=torch.int32, device=device)
        self.backup_rows = torch.zeros(max(backup_cap, 1), dtype=torch.int32, device=device)
        self.backup_g = torch.zeros((max(backup_cap, 1), F), dtype=dtype, device=device)
        self.backup_u = torch.zeros((max(backup_cap, 1), F), dtype=dtype, device=device)
        self.n_backup = torch.zeros(1, dtype=torch.int32, device=device)

    def struct(self):
        e = self.ell_g if self.C_h else None
        return TwHybridC(self.T, self.F, self.C_h, _dt(self.backup_g), _ptr(e),
                         _ptr(self.ell_u if self.C_h else None),
                         _ptr(self.ell_idx if self.C_h else None), _ptr(self.row_nnz),
                         _ptr(self.row_slot), self.backup_cap, _ptr(self.backup_rows),
                         _ptr(self.backup_g), _ptr(self.backup_u), _ptr(self.n_backup))


# ------------------------------------------------------------- entry points --
def twell_gate_gemm(x, Wg_t, out: Twell, g_dense_dump=None, dev_status=None, stream=None):
    T, d = x.shape
    F = Wg_t.shape[0]
    s = out.struct()
    _check("twell_gate_gemm", lib().twell_gate_gemm(
        _ptr(x), _ptr(Wg_t), T, d, F, _dt(x), ctypes.byref(s), _ptr(g_dense_dump),
        _ptr(dev_status), _stream(stream)))


def twell_fused_updown_workspace_size(T, d):
    return int(lib().twell_fused_updown_workspace_size(T, d))


def fused_workspace(T, d, device="cuda"):
    """A caller-owned workspace tensor of the size twell_fused_updown needs."""
    return torch.empty(twell_fused_updown_workspace_size(T, d), dtype=torch.uint8, device=device)


def twell_fused_updown(x, g: Twell, Wu_t, Wd, y, ws, dev_status=None, stream=None):
    s = g.struct()
    _check("twell_fused_updown", lib().twell_fused_updown(
        _ptr(x), ctypes.byref(s), _ptr(Wu_t), _ptr(Wd), x.shape[1], _ptr(y), _dt(y), _ptr(ws),
        ws.numel() * ws.element_size(), _ptr(dev_status), _stream(stream)))


def twell_fused_updown_noalloc(x, g: Twell, Wu_t, Wd, y, dev_status=None, stream=None):
    """twell_fused_updown for callers that cannot allocate a workspace: the
    library uses its own fixed device array (see include/twell.h)."""
    s = g.struct()
    _check("twell_fused_updown_noalloc", lib().twell_fused_updown_noalloc(
        _ptr(x), ctypes.byref(s), _ptr(Wu_t), _ptr(Wd), x.shape[1], _ptr(y), _dt(y),
        _ptr(dev_status), _stream(stream)))


def twell_ffn_small_batch_workspace_size(T, d, F):
    return int(lib().twell_ffn_small_batch_workspace_size(T, d, F))


def small_batch_workspace(T, d, F, device="cuda"):
    """A zero-filled workspace for twell_ffn_small_batch (its barrier counters
    must start at zero; each call leaves them at zero)."""
    return torch.zeros(twell_ffn_small_batch_workspace_size(T, d, F), dtype=torch.uint8,
                       device=device)


def twell_ffn_small_batch(x, Wg_t, Wu_t, Wd, g: Twell, y, ws, g_dense_dump=None, dev_status=None,
                          stream=None):
    T, d = x.shape
    F = Wg_t.shape[0]
    s = g.struct()
    _check("twell_ffn_small_batch", lib().twell_ffn_small_batch(
        _ptr(x), _ptr(Wg_t), _ptr(Wu_t), _ptr(Wd), T, d, F, ctypes.byref(s), _ptr(g_dense_dump),
        _ptr(y), _dt(y), _ptr(ws), ws.numel() * ws.element_size(), _ptr(dev_status),
        _stream(stream)))


def twell_to_hybrid(g: Twell, out: Hybrid, dev_status=None, stream=None):
    sg, sh = g.struct(), out.struct()
    _check("twell_to_hybrid", lib().twell_to_hybrid(
        ctypes.byref(sg), ctypes.byref(sh), _ptr(dev_status), _stream(stream)))


def hybrid_ffn_forward_workspace_size(T, d):
    return int(lib().hybrid_ffn_forward_workspace_size(T, d))


def hybrid_ffn_forward(x, gu: Hybrid, Wu_t, Wd, y, ws=None, dev_status=None, stream=None):
    """ws: caller-owned workspace (hybrid_ffn_forward_workspace_size bytes);
    when None, one is allocated with torch for this call."""
    if ws is None:
        ws = torch.empty(hybrid_ffn_forward_workspace_size(x.shape[0], x.shape[1]),
                         dtype=torch.uint8, device=x.device)
    s = gu.struct()
    _check("hybrid_ffn_forward", lib().hybrid_ffn_forward(
        _ptr(x), ctypes.byref(s), _ptr(Wu_t), _ptr(Wd), x.shape[1], _ptr(y), _dt(y), _ptr(ws),
        ws.numel() * ws.element_size(), _ptr(dev_status), _stream(stream)))


def hybrid_ffn_backward_workspace_size(T, d, F, C_h, backup_cap):
    return int(lib().hybrid_ffn_backward_workspace_size(T, d, F, C_h, backup_cap))


def hybrid_ffn_backward(x, dy, gu: Hybrid, Wg_t, Wu_t, Wd, l1_lambda, dx, dWg_t, dWu_t, dWd, ws,
                        dev_status=None, stream=None):
    s = gu.struct()
    _check("hybrid_ffn_backward", lib().hybrid_ffn_backward(
        _ptr(x), _ptr(dy), ctypes.byref(s), _ptr(Wg_t), _ptr(Wu_t), _ptr(Wd), x.shape[1],
        float(l1_lambda), _ptr(dx), _dt(dx), _ptr(dWg_t), _ptr(dWu_t), _ptr(dWd), _ptr(ws),
        ws.numel() * ws.element_size(), _ptr(dev_status), _stream(stream)))


def dense_ffn_forward(x, Wg_t, Wu_t, Wd_dense, h_ws, y, dev_status=None, stream=None):
    T, d = x.shape
    F = Wg_t.shape[0]
    _check("dense_ffn_forward", lib().dense_ffn_forward(
        _ptr(x), _ptr(Wg_t), _ptr(Wu_t), _ptr(Wd_dense), T, d, F, _ptr(h_ws), _ptr(y),
        _ptr(dev_status), _stream(stream)))


def dense_ffn_train_workspace_size(T, F):
    return int(lib().dense_ffn_train_workspace_size(T, F))


def dense_ffn_train_saved_bytes(T, F):
    return int(lib().dense_ffn_train_saved_bytes(T, F))


def dense_train_workspace(T, F, device="cuda"):
    """A caller-owned workspace tensor for the dense training comparator."""
    return torch.empty(dense_ffn_train_workspace_size(T, F), dtype=torch.uint8, device=device)


def dense_ffn_train_forward(x, Wg_t, Wu_t, Wd, ws, y, dev_status=None, stream=None):
    T, d = x.shape
    F = Wg_t.shape[0]
    _check("dense_ffn_train_forward", lib().dense_ffn_train_forward(
        _ptr(x), _ptr(Wg_t), _ptr(Wu_t), _ptr(Wd), T, d, F, _ptr(ws),
        ws.numel() * ws.element_size(), _ptr(y), _ptr(dev_status), _stream(stream)))


def dense_ffn_train_backward(x, dy, Wg_t, Wu_t, Wd, l1_lambda, ws, dx, dWg_t, dWu_t, dWd,
                             dev_status=None, stream=None):
    T, d = x.shape
    F = Wg_t.shape[0]
    _check("dense_ffn_train_backward", lib().dense_ffn_train_backward(
        _ptr(x), _ptr(dy), _ptr(Wg_t), _ptr(Wu_t), _ptr(Wd), T, d, F, float(l1_lambda),
        _ptr(ws), ws.numel() * ws.element_size(), _ptr(dx), _ptr(dWg_t), _ptr(dWu_t), _ptr(dWd),
        _ptr(dev_status), _stream(stream)))


def dense_train_saved(ws, T, F):
    """Views of the g, u, h [T][F] bf16 tensors the training forward saved in ws."""
    part = (T * F * 2 + 255) // 256 * 256
    return [ws[i * part:i * part + T * F * 2].view(torch.bfloat16).view(T, F) for i in range(3)]


def status_bits(dev_status) -> list:
    """Names of the device-side conditions set in a status word tensor."""
    v = int(dev_status.item())
    return [STATUS[i] for i in range(len(STATUS)) if v & (1 << i)]


def measure_row_gather(mat, n_gathers, seed, checksum, stream=None):
    """Measurement aid (not part of the FFN): n_gathers scattered whole rows of
    the bf16 matrix mat [rows][d]; checksum (an int32 tensor, zeroed by the
    caller) receives the XOR of every 32-bit word read."""
    rows, d = mat.shape
    _check("tw_measure_row_gather", lib().tw_measure_row_gather(
        _ptr(mat), rows, d, int(n_gathers), int(seed) & 0xFFFFFFFF, _ptr(checksum), _stream(stream)))


def measure_stream_read(buf, checksum, stream=None):
    """Measurement aid (not part of the FFN): one launch that reads the whole
    device tensor buf front to back; checksum (an int32 tensor, zeroed by the
    caller) receives the XOR of every 32-bit word read."""
    _check("tw_measure_stream_read", lib().tw_measure_stream_read(
        _ptr(buf), buf.numel() * buf.element_size(), _ptr(checksum), _stream(stream)))
