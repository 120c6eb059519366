"""rope_add_rms_b200 -- Python binding of libnvnorm.so, the B200 fused row-normalisation library.

This module only marshals arguments: every step of every op runs in the CUDA kernels of
``libnvnorm.so`` (built from ``csrc/`` for sm_100a).  There is no fallback: if the library
is missing or a call fails, an exception is raised.  PyTorch supplies device memory and
the current stream.

The ``nv_*`` functions mirror the C entry points of ``include/nvnorm.h`` and write into
caller-provided output tensors.  ``rms_norm``, ``add_rms_norm``, ``layer_norm`` and
``norm_rope`` allocate their outputs and return them.
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "NvError", "Plan", "library", "library_path",
    "nv_rms_norm", "nv_add_rms_norm", "nv_add_rms_norm_host", "nv_allreduce_add_rms_norm",
    "nv_allreduce_add_rms_norm_peers", "nv_tp_publish", "ipc_export", "ipc_import", "ipc_close",
    "allreduce_add_rms_norm", "rope_llama3_freqs", "rope_yarn_freqs", "rope_suscaled_freqs",
    "nv_layer_norm", "nv_norm_rope",
    "nv_describe_plan",
    "nv_fault_count", "nv_selftest_bounded_wait", "nv_set_pointer_checks",
    "nv_rope", "rms_norm", "add_rms_norm", "layer_norm", "norm_rope", "norm_rope_into_cache",
    "rope", "nv_rms_norm_vjp", "nv_layer_norm_vjp", "nv_norm_vjp_workspace_size", "rms_norm_vjp",
    "layer_norm_vjp",
    "PATH_AUTO", "PATH_ROWS", "PATH_GENERIC", "PATH_STAGED", "PATH_RING", "PATH_SLOTS", "LAUNCH_DEFAULT",
    "LAUNCH_PLAIN",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_HERE, "libnvnorm.so")

NV_F32, NV_BF16, NV_F16 = 0, 1, 2
NV_OK, NV_ERR_INVALID_ARG, NV_ERR_UNSUPPORTED, NV_ERR_CUDA = 0, 1, 2, 3
PATH_AUTO, PATH_ROWS, PATH_GENERIC, PATH_STAGED, PATH_RING, PATH_SLOTS = 0, 1, 2, 3, 4, 5
LAUNCH_DEFAULT, LAUNCH_PLAIN = 0, 1

_DT = {torch.float32: NV_F32, torch.bfloat16: NV_BF16, torch.float16: NV_F16}


class NvError(RuntimeError):
    """A non-OK status from libnvnorm.so, with the library's message."""

    def __init__(self, fn: str, status: int, message: str):
        self.status = status
        self.message = message
        super().__init__(f"{fn}: {_status_name(status)}: {message}")


class Plan(ctypes.Structure):
    """nv_plan: kernel-variant selection (0 fields mean automatic)."""
    _fields_ = [("path", ctypes.c_int32), ("vec_per_thread", ctypes.c_int32),
                ("threads_per_row", ctypes.c_int32), ("rows_per_cta", ctypes.c_int32),
                ("ctas_per_sm", ctypes.c_int32), ("launch", ctypes.c_int32),
                ("stages", ctypes.c_int32)]

    def as_dict(self):
        return {k: getattr(self, k) for k, _ in self._fields_}


_lib = None


def library() -> ctypes.CDLL:
    """Load libnvnorm.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(library_path):
        raise ImportError(f"{library_path} is missing: build it with "
                          "`python -m rope_add_rms_b200.build` (nvcc, sm_100a)")
    lib = ctypes.CDLL(library_path)
    vp, i64, i32, f32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_float
    pp = ctypes.POINTER(Plan)
    sigs = {
        "nv_rms_norm": [vp, vp, vp, i64, i64, f32, i32, vp],
        "nv_add_rms_norm": [vp, vp, vp, vp, vp, i64, i64, f32, i32, vp],
        "nv_add_rms_norm_host": [vp, vp, vp, vp, vp, vp, vp, vp, vp, i64, i64, f32, i32, i64,
                                 vp],
        "nv_allreduce_add_rms_norm": [ctypes.POINTER(vp), i32, vp, vp, vp, vp, vp, i64, i64,
                                      f32, i32, vp],
        "nv_layer_norm": [vp, vp, vp, vp, i64, i64, f32, i32, vp],
        "nv_norm_rope": [vp, vp, vp, i64, i64, i64, i32, i32, f32, f32, i64, i32, f32, i32, vp],
        "nv_rms_norm_ex": [vp, vp, vp, i64, i64, f32, i32, vp, pp],
        "nv_add_rms_norm_ex": [vp, vp, vp, vp, vp, i64, i64, f32, i32, vp, pp],
        "nv_layer_norm_ex": [vp, vp, vp, vp, i64, i64, f32, i32, vp, pp],
        "nv_norm_rope_ex": [vp, vp, vp, i64, i64, i64, i32, i32, f32, f32, i64, i32, f32, i32,
                            vp, pp],
        "nv_describe_plan": [i32, i64, i64, i32, pp],
        "nv_rope": [vp, vp, vp, vp, i64, i64, i64, i64, i32, i32, f32, f32, i64, i32, i32, f32, i32,
                    vp],
        "nv_rope_ex": [vp, vp, vp, vp, i64, i64, i64, i64, i32, i32, f32, f32, i64, i32, i32, f32,
                       i32, vp, pp],
    }
    for name, args in sigs.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = ctypes.c_int
    lib.nv_status_string.argtypes = [ctypes.c_int]
    lib.nv_status_string.restype = ctypes.c_char_p
    lib.nv_last_error.argtypes = []
    lib.nv_last_error.restype = ctypes.c_char_p
    lib.nv_version.argtypes = []
    lib.nv_version.restype = ctypes.c_int32
    lib.nv_set_pointer_checks.argtypes = [ctypes.c_int32, ctypes.POINTER(ctypes.c_int32)]
    lib.nv_set_pointer_checks.restype = ctypes.c_int
    lib.nv_fault_count.argtypes = [ctypes.POINTER(ctypes.c_uint32), ctypes.c_int32]
    lib.nv_fault_count.restype = ctypes.c_int
    lib.nv_selftest_bounded_wait.argtypes = [ctypes.c_int32, ctypes.c_void_p]
    lib.nv_selftest_bounded_wait.restype = ctypes.c_int
    sz = ctypes.c_size_t
    lib.nv_rms_norm_vjp.argtypes = [vp, vp, vp, vp, vp, vp, sz, i64, i64, f32, i32, vp]
    lib.nv_rms_norm_vjp.restype = ctypes.c_int
    lib.nv_layer_norm_vjp.argtypes = [vp, vp, vp, vp, vp, vp, vp, sz, i64, i64, f32, i32, vp]
    lib.nv_layer_norm_vjp.restype = ctypes.c_int
    lib.nv_allreduce_add_rms_norm_peers.argtypes = [ctypes.POINTER(vp), i32, vp, vp, vp, vp, vp,
                                                    i64, i64, f32, i32, vp, i64, vp]
    lib.nv_allreduce_add_rms_norm_peers.restype = ctypes.c_int
    lib.nv_tp_publish.argtypes = [ctypes.POINTER(vp), i32, i32, i64, vp]
    lib.nv_tp_publish.restype = ctypes.c_int
    u64 = ctypes.c_uint64
    lib.nv_ipc_export.argtypes = [vp, vp, ctypes.POINTER(u64)]
    lib.nv_ipc_export.restype = ctypes.c_int
    lib.nv_ipc_import.argtypes = [vp, u64, ctypes.POINTER(vp)]
    lib.nv_ipc_import.restype = ctypes.c_int
    lib.nv_ipc_close.argtypes = [vp, u64]
    lib.nv_ipc_close.restype = ctypes.c_int
    lib.nv_rms_norm_vjp_static.argtypes = [vp, vp, vp, vp, vp, i64, i64, f32, i32, vp]
    lib.nv_rms_norm_vjp_static.restype = ctypes.c_int
    lib.nv_rope_llama3_freqs.argtypes = [i32, f32, f32, f32, f32, i64, vp]
    lib.nv_rope_llama3_freqs.restype = ctypes.c_int
    lib.nv_rope_yarn_freqs.argtypes = [i32, f32, f32, i64, f32, f32, vp, vp]
    lib.nv_rope_yarn_freqs.restype = ctypes.c_int
    lib.nv_rope_suscaled_freqs.argtypes = [i32, f32, vp, vp, i64, i64, i64, vp, vp]
    lib.nv_rope_suscaled_freqs.restype = ctypes.c_int
    lib.nv_norm_vjp_workspace_size.argtypes = [i32, i64, i64]
    lib.nv_norm_vjp_workspace_size.restype = sz
    _lib = lib
    return lib


def _status_name(status: int) -> str:
    return library().nv_status_string(status).decode()


def _check(fn: str, status: int):
    if status != NV_OK:
        raise NvError(fn, status, library().nv_last_error().decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _dtype(*ts):
    dts = {t.dtype for t in ts if t is not None}
    if len(dts) != 1:
        raise TypeError(f"all tensors must share one dtype, got {sorted(map(str, dts))}")
    dt = dts.pop()
    if dt not in _DT:
        raise TypeError(f"unsupported dtype {dt}")
    return _DT[dt]


def _rows_D(x):
    if not x.is_contiguous():
        raise ValueError("tensors must be contiguous (row-major, last axis contiguous)")
    D = x.shape[-1] if x.dim() else 1
    return (x.numel() // D if D else 0), D


def _plan(plan):
    if plan is None:
        return None
    if isinstance(plan, dict):
        plan = Plan(**plan)
    return ctypes.byref(plan)


# ---- C-ABI mirrors (outputs provided by the caller) ------------------------------------

def nv_rms_norm(x, w, y, eps, stream=None, plan=None):
    rows, D = _rows_D(x)
    lib = library()
    args = (_ptr(x), _ptr(w), _ptr(y), rows, D, eps, _dtype(x, w, y), _stream(stream))
    st = lib.nv_rms_norm(*args) if plan is None else lib.nv_rms_norm_ex(*args, _plan(plan))
    _check("nv_rms_norm", st)


def nv_add_rms_norm(x, r, w, y, h, eps, stream=None, plan=None):
    rows, D = _rows_D(x)
    lib = library()
    args = (_ptr(x), _ptr(r), _ptr(w), _ptr(y), _ptr(h), rows, D, eps, _dtype(x, r, w, y, h),
            _stream(stream))
    st = lib.nv_add_rms_norm(*args) if plan is None else lib.nv_add_rms_norm_ex(*args, _plan(plan))
    _check("nv_add_rms_norm", st)


def nv_add_rms_norm_host(x_host, r_host, w, y_host, h_host, x_dev, r_dev, y_dev, h_dev, eps,
                         chunk_rows=0, stream=None):
    """add_rms_norm on rows in page-locked host tensors (``pin_memory()``), staged through
    the caller's device tensors; copies in, compute and copies out pipelined over row
    chunks.  Asynchronous like the other calls (synchronise ``stream`` to read y_host)."""
    rows, D = _rows_D(x_host)
    for t in (x_host, r_host, y_host, h_host):
        if t.is_cuda:
            raise ValueError("x_host, r_host, y_host and h_host must be host tensors")
    lib = library()
    st = lib.nv_add_rms_norm_host(_ptr(x_host), _ptr(r_host), _ptr(w), _ptr(y_host),
                                  _ptr(h_host), _ptr(x_dev), _ptr(r_dev), _ptr(y_dev),
                                  _ptr(h_dev), rows, D, eps,
                                  _dtype(x_host, r_host, w, y_host, h_host, x_dev, r_dev,
                                         y_dev, h_dev), chunk_rows, _stream(stream))
    _check("nv_add_rms_norm_host", st)


def rope_llama3_freqs(dims, base=500000.0, factor=32.0, low_freq_factor=1.0,
                      high_freq_factor=4.0, original_max_position=8192):
    """Llama 3 scaled RoPE frequencies theta_i (i < dims/2) as a float32 host tensor, for
    ``nv_rope(..., freqs=...)`` after ``.cuda()``."""
    out = torch.empty(dims // 2, dtype=torch.float32)
    st = library().nv_rope_llama3_freqs(dims, base, factor, low_freq_factor, high_freq_factor,
                                        original_max_position, ctypes.c_void_p(out.data_ptr()))
    _check("nv_rope_llama3_freqs", st)
    return out


def rope_yarn_freqs(dims, base=10000.0, factor=4.0, original_max_position=4096, alpha=1.0,
                    beta=32.0):
    """YaRN scaled RoPE frequencies (a float32 host tensor of dims/2, for
    ``nv_rope(..., freqs=...)`` after ``.cuda()``) and its temperature factor mscale, which
    the caller applies (attention logits times mscale**2)."""
    out = torch.empty(dims // 2, dtype=torch.float32)
    m = ctypes.c_float(0.0)
    st = library().nv_rope_yarn_freqs(dims, base, factor, original_max_position, alpha, beta,
                                      ctypes.c_void_p(out.data_ptr()), ctypes.byref(m))
    _check("nv_rope_yarn_freqs", st)
    return out, m.value


def rope_suscaled_freqs(dims, short_factors, long_factors, seq_len, base=10000.0,
                        max_position=131072, original_max_position=4096):
    """SuScaled (LongRoPE) RoPE frequencies (a float32 host tensor of dims/2, for
    ``nv_rope(..., freqs=...)`` after ``.cuda()``): the long factors when seq_len exceeds
    the original context, else the short ones; and the attention factor mscale, which the
    caller applies to q and k."""
    sf = torch.as_tensor(short_factors, dtype=torch.float32).contiguous()
    lf = torch.as_tensor(long_factors, dtype=torch.float32).contiguous()
    if sf.numel() != dims // 2 or lf.numel() != dims // 2:
        raise ValueError("short_factors and long_factors must hold dims / 2 values")
    out = torch.empty(dims // 2, dtype=torch.float32)
    m = ctypes.c_float(0.0)
    st = library().nv_rope_suscaled_freqs(dims, base, ctypes.c_void_p(sf.data_ptr()),
                                          ctypes.c_void_p(lf.data_ptr()), seq_len, max_position,
                                          original_max_position, ctypes.c_void_p(out.data_ptr()),
                                          ctypes.byref(m))
    _check("nv_rope_suscaled_freqs", st)
    return out, m.value


def nv_allreduce_add_rms_norm(parts, r, w, y, h, eps, x_out=None, stream=None):
    """x = sum(parts) (in order, in double, rounded once), h = x + r, y = RmsNorm(h) * w.
    ``parts`` are device tensors shaped like r (this GPU's, or peers' mapped buffers)."""
    rows, D = _rows_D(r)
    table = (ctypes.c_void_p * len(parts))(*[t.data_ptr() for t in parts])
    lib = library()
    st = lib.nv_allreduce_add_rms_norm(table, len(parts), _ptr(r), _ptr(w), _ptr(y), _ptr(h),
                                       _ptr(x_out), rows, D, eps,
                                       _dtype(*parts, r, w, y, h, x_out), _stream(stream))
    _check("nv_allreduce_add_rms_norm", st)


def nv_allreduce_add_rms_norm_peers(part_ptrs, r, w, y, h, eps, flags, epoch, x_out=None,
                                    stream=None):
    """The one-shot form: ``part_ptrs`` are device addresses (ints) of every rank's partial,
    shaped and typed like r (this rank's own buffer and peers' mapped ones, rank order);
    waits on the device until every slot of ``flags`` (an int64 device tensor, one slot per
    rank) reaches ``epoch``, then computes as nv_allreduce_add_rms_norm."""
    rows, D = _rows_D(r)
    table = (ctypes.c_void_p * len(part_ptrs))(*[int(p) for p in part_ptrs])
    st = library().nv_allreduce_add_rms_norm_peers(
        table, len(part_ptrs), _ptr(r), _ptr(w), _ptr(y), _ptr(h), _ptr(x_out), rows, D, eps,
        _dtype(r, w, y, h, x_out), _ptr(flags), epoch, _stream(stream))
    _check("nv_allreduce_add_rms_norm_peers", st)


def nv_tp_publish(flag_ptrs, rank, epoch, stream=None):
    """Store ``epoch`` into slot ``rank`` of every rank's flag array (device addresses, rank
    order) once the work queued before on the stream is complete."""
    table = (ctypes.c_void_p * len(flag_ptrs))(*[int(p) for p in flag_ptrs])
    _check("nv_tp_publish", library().nv_tp_publish(table, len(flag_ptrs), rank, epoch,
                                                     _stream(stream)))


IPC_HANDLE_BYTES = 64


def ipc_export(t):
    """(handle bytes, offset) that another process of this node passes to ipc_import to map
    the device memory of tensor ``t``."""
    buf = ctypes.create_string_buffer(IPC_HANDLE_BYTES)
    off = ctypes.c_uint64(0)
    _check("nv_ipc_export", library().nv_ipc_export(ctypes.c_void_p(t.data_ptr()), buf,
                                                    ctypes.byref(off)))
    return buf.raw, off.value


def ipc_import(handle, offset):
    """Device address, in this process, of the memory another process exported."""
    if len(handle) != IPC_HANDLE_BYTES:
        raise ValueError("an IPC handle is 64 bytes")
    out = ctypes.c_void_p(0)
    _check("nv_ipc_import", library().nv_ipc_import(ctypes.create_string_buffer(handle, 64),
                                                    offset, ctypes.byref(out)))
    return out.value


def ipc_close(ptr, offset):
    _check("nv_ipc_close", library().nv_ipc_close(ctypes.c_void_p(ptr), offset))


def allreduce_add_rms_norm(parts, r, w, eps=1e-5):
    """Allocating form: returns (y, h, x) for device tensors."""
    y, h, x = torch.empty_like(r), torch.empty_like(r), torch.empty_like(r)
    nv_allreduce_add_rms_norm(parts, r, w, y, h, eps, x_out=x)
    return y, h, x


def nv_layer_norm(x, w, b, y, eps, stream=None, plan=None):
    rows, D = _rows_D(x)
    lib = library()
    args = (_ptr(x), _ptr(w), _ptr(b), _ptr(y), rows, D, eps, _dtype(x, w, b, y), _stream(stream))
    st = lib.nv_layer_norm(*args) if plan is None else lib.nv_layer_norm_ex(*args, _plan(plan))
    _check("nv_layer_norm", st)


def nv_norm_rope(x, w, y, L, dims, traditional, base, scale, offset, normalize, eps,
                 stream=None, plan=None):
    rows, D = _rows_D(x)
    lib = library()
    args = (_ptr(x), _ptr(w), _ptr(y), rows, L, D, dims, int(bool(traditional)), base, scale,
            offset, int(bool(normalize)), eps, _dtype(x, w, y), _stream(stream))
    st = lib.nv_norm_rope(*args) if plan is None else lib.nv_norm_rope_ex(*args, _plan(plan))
    _check("nv_norm_rope", st)


def nv_rope(x, w, y, L, dims, traditional, base, scale, offset, normalize, eps, freqs=None,
            forward=True, y_len=0, stream=None, plan=None):
    """General NormRope / Rope (cache output when y_len > 0, explicit float32 freqs,
    forward=False for the inverse rotation); x is [rows, D] with rows = B*H*L."""
    rows, D = _rows_D(x)
    if freqs is not None and freqs.dtype != torch.float32:
        raise TypeError("freqs must be float32")
    lib = library()
    args = (_ptr(x), _ptr(w), _ptr(freqs), _ptr(y), rows, L, y_len, D, dims,
            int(bool(traditional)), base, scale, offset, int(bool(forward)), int(bool(normalize)),
            eps, _dtype(x, w, y), _stream(stream))
    st = lib.nv_rope(*args) if plan is None else lib.nv_rope_ex(*args, _plan(plan))
    _check("nv_rope", st)


def nv_describe_plan(op: str, rows: int, D: int, dtype) -> dict:
    """The kernel variant the library picks for op on [rows, D] (16-byte aligned data)."""
    ops = {"rms_norm": 0, "add_rms_norm": 1, "layer_norm": 2, "norm_rope": 3}
    p = Plan()
    _check("nv_describe_plan", library().nv_describe_plan(ops[op], rows, D, _DT[dtype],
                                                           ctypes.byref(p)))
    return p.as_dict()


def nv_set_pointer_checks(enabled: bool) -> bool:
    """Turn the per-pointer driver queries of every call on or off (process-wide); returns
    the former setting.  Off is for callers that vouch for their pointers."""
    prev = ctypes.c_int32(0)
    _check("nv_set_pointer_checks", library().nv_set_pointer_checks(int(bool(enabled)),
                                                                     ctypes.byref(prev)))
    return bool(prev.value)


def nv_fault_count(reset: bool = False) -> int:
    """Bounded device waits that ran out on the current device (synchronises it)."""
    c = ctypes.c_uint32(0)
    _check("nv_fault_count", library().nv_fault_count(ctypes.byref(c), int(bool(reset))))
    return c.value


def nv_selftest_bounded_wait(ctas: int = 1, stream=None):
    """Launch `ctas` CTAs whose device-side bounded waits run out (about one second);
    each counts one fault in nv_fault_count.  A check of the failure path."""
    _check("nv_selftest_bounded_wait", library().nv_selftest_bounded_wait(int(ctas), _stream(stream)))


def nv_norm_vjp_workspace_size(op: str, rows: int, D: int) -> int:
    """Bytes of workspace the vjp column sums need (op 'rms_norm' or 'layer_norm')."""
    return library().nv_norm_vjp_workspace_size({"rms_norm": 0, "layer_norm": 2}[op], rows, D)


def _workspace(op, x, need, workspace):
    if not need:
        return None, 0
    rows, D = _rows_D(x)
    n = nv_norm_vjp_workspace_size(op, rows, D)
    if workspace is None:
        workspace = torch.empty(max(n, 1), dtype=torch.uint8, device=x.device)
    return workspace, workspace.numel() * workspace.element_size()


def nv_rms_norm_vjp(x, w, g, dx, dw, eps, workspace=None, stream=None):
    """Gradients of rms_norm: dx, and dw (exactly when w is given)."""
    rows, D = _rows_D(x)
    ws, nbytes = _workspace("rms_norm", x, dw is not None, workspace)
    _check("nv_rms_norm_vjp", library().nv_rms_norm_vjp(
        _ptr(x), _ptr(w), _ptr(g), _ptr(dx), _ptr(dw), _ptr(ws), nbytes, rows, D, eps,
        _dtype(x, w, g, dx, dw), _stream(stream)))


def nv_layer_norm_vjp(x, w, g, dx, dw, db, eps, workspace=None, stream=None):
    """Gradients of layer_norm: dx, dw (exactly when w is given), db (or None)."""
    rows, D = _rows_D(x)
    ws, nbytes = _workspace("layer_norm", x, dw is not None or db is not None, workspace)
    _check("nv_layer_norm_vjp", library().nv_layer_norm_vjp(
        _ptr(x), _ptr(w), _ptr(g), _ptr(dx), _ptr(dw), _ptr(db), _ptr(ws), nbytes, rows, D, eps,
        _dtype(x, w, g, dx, dw, db), _stream(stream)))


# ---- allocating wrappers ---------------------------------------------------------------

def rms_norm(x, w=None, eps=1e-5, stream=None):
    """y = x / sqrt(mean(x^2) + eps) * w over the last axis."""
    y = torch.empty_like(x)
    nv_rms_norm(x, w, y, eps, stream)
    return y


def add_rms_norm(x, r, w=None, eps=1e-5, stream=None):
    """(y, h): h = x + r (rounded to x's dtype), y = rms_norm(h, w, eps)."""
    y = torch.empty_like(x)
    h = torch.empty_like(x)
    nv_add_rms_norm(x, r, w, y, h, eps, stream)
    return y, h


def layer_norm(x, w=None, b=None, eps=1e-5, stream=None):
    """y = (x - mean) / sqrt(var + eps) * w + b over the last axis."""
    y = torch.empty_like(x)
    nv_layer_norm(x, w, b, y, eps, stream)
    return y


def norm_rope_into_cache(x, cache, w=None, dims=None, traditional=False, base=10000.0,
                         scale=1.0, offset=0, eps=1e-6, freqs=None, stream=None):
    """Normalise (eps None: skip) and rotate x [..., L, D]; write row l into
    cache [..., Lc, D] at row offset + l (the cache form of NormRope)."""
    L, D = x.shape[-2], x.shape[-1]
    normalize = eps is not None
    nv_rope(x, w, cache, L, D if dims is None else dims, traditional, base, scale, offset,
            normalize, eps if normalize else 0.0, freqs=freqs, y_len=cache.shape[-2],
            stream=stream)
    return cache


def rope(x, dims=None, traditional=False, base=10000.0, scale=1.0, offset=0, freqs=None,
         forward=True, stream=None):
    """Plain rotary embedding of x [..., L, D] (forward=False: the inverse rotation)."""
    L, D = x.shape[-2], x.shape[-1]
    y = torch.empty_like(x)
    nv_rope(x, None, y, L, D if dims is None else dims, traditional, base, scale, offset, False,
            0.0, freqs=freqs, forward=forward, stream=stream)
    return y


def norm_rope(x, w=None, dims=None, traditional=False, base=10000.0, scale=1.0, offset=0,
              eps=1e-6, stream=None):
    """RMS-normalise each row of x [..., L, D] (eps None: skip), then rotate its first dims
    features at positions offset + l (l the index on the second-to-last axis)."""
    if x.dim() < 2:
        raise ValueError("x must be [..., L, D]")
    L, D = x.shape[-2], x.shape[-1]
    y = torch.empty_like(x)
    normalize = eps is not None
    nv_norm_rope(x, w, y, L, D if dims is None else dims, traditional, base, scale, offset,
                 normalize, eps if normalize else 0.0, stream)
    return y


def rms_norm_vjp(x, w, g, eps=1e-5, stream=None):
    """(dx, dw) of rms_norm for upstream gradient g; dw is None when w is None."""
    dx = torch.empty_like(x)
    dw = None if w is None else torch.empty_like(w)
    nv_rms_norm_vjp(x, w, g, dx, dw, eps, stream=stream)
    return dx, dw


def layer_norm_vjp(x, w, g, eps=1e-5, with_db=True, stream=None):
    """(dx, dw, db) of layer_norm for upstream gradient g; dw None when w is None."""
    dx = torch.empty_like(x)
    dw = None if w is None else torch.empty_like(w)
    db = torch.empty(x.shape[-1], dtype=x.dtype, device=x.device) if with_db else None
    nv_layer_norm_vjp(x, w, g, dx, dw, db, eps, stream=stream)
    return dx, dw, db
