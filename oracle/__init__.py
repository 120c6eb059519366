"""fp64 CPU oracle for the fused row-normalisation ops -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may
import this package.  The product library (``rope_add_rms_b200``) never imports it and
shares no code with it; the one module both sides use is the seeded input generator
``rope_add_rms_b200.synth``, which does no normalisation arithmetic.

The arithmetic lives in ``oracle.c`` (plain C, double precision, one row at a time,
the definitions of docs.rs nuvec-core 0.5.0 "Enum FastOp" -- RmsNorm, AddRmsNorm,
LayerNorm, Rope, NormRope -- and of the miniVLLM "Layers" page, LayerNorm section, for
the residual return).  This wrapper only marshals numpy arrays and spreads row ranges
over threads (ctypes releases the GIL during each call).

Arrays: bfloat16 data travels as raw ``uint16`` bit patterns, float32 as ``float32``.
Normalised outputs come back unrounded as ``float64``; ``round_bf16`` rounds them once,
to nearest with ties to even.  Every function here is pinned by
``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from concurrent.futures import ThreadPoolExecutor

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(HERE, "oracle.c")
LIBRARY = os.path.join(HERE, "liboracle.so")

F32 = 0
BF16 = 1

CFLAGS = ["-O2", "-ffp-contract=off", "-fno-fast-math", "-fexcess-precision=standard",
          "-std=c11", "-fPIC", "-shared"]


def compile_oracle(src: str, out: str) -> str:
    """Compile one C source of the oracle into a shared library (gcc)."""
    tmp = out + f".tmp{os.getpid()}"
    subprocess.run(["gcc", *CFLAGS, "-o", tmp, src, "-lm"], check=True)
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    """Compile oracle.c to liboracle.so next to it unless it is up to date."""
    if force or not os.path.exists(LIBRARY) or \
            os.path.getmtime(LIBRARY) < os.path.getmtime(SOURCE):
        compile_oracle(SOURCE, LIBRARY)
    return LIBRARY


def default_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _io(a, name):
    """Check an I/O array; return (C-contiguous array, element-type code)."""
    a = np.asarray(a)
    if a.dtype == np.uint16:
        dt = BF16
    elif a.dtype == np.float32:
        dt = F32
    else:
        raise TypeError(f"{name}: expected uint16 (bfloat16 bits) or float32, got {a.dtype}")
    return np.ascontiguousarray(a), dt


def _chunks(rows, threads):
    n = max(1, min(threads or default_threads(), rows)) if rows else 1
    bounds = np.linspace(0, rows, n + 1).astype(np.int64)
    return [(int(bounds[i]), int(bounds[i + 1])) for i in range(n)]


def bf16_to_f64(bits) -> np.ndarray:
    """Exact widening of bfloat16 bit patterns."""
    bits = np.asarray(bits, dtype=np.uint16)
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


class Oracle:
    """The oracle's entry points over one compiled copy of the C source."""

    def __init__(self, path: str):
        lib = ctypes.CDLL(path)
        i64, f32, i32, vp = ctypes.c_int64, ctypes.c_float, ctypes.c_int, ctypes.c_void_p
        lib.oracle_bf16_from_f64.argtypes = [ctypes.c_double]
        lib.oracle_bf16_from_f64.restype = ctypes.c_uint16
        lib.oracle_round_bf16.argtypes = [vp, vp, i64]
        lib.oracle_round_bf16.restype = None
        lib.oracle_rms_norm.argtypes = [vp, vp, vp, i64, i64, i64, f32, i32]
        lib.oracle_add_rms_norm.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, f32, i32]
        f64 = ctypes.c_double
        lib.oracle_llama3_freqs.argtypes = [i64, f64, f64, f64, f64, f64, vp]
        lib.oracle_yarn_freqs.argtypes = [i64, f64, f64, f64, f64, f64, vp, vp]
        lib.oracle_suscaled_freqs.argtypes = [i64, f64, vp, vp, f64, f64, f64, vp, vp]
        lib.oracle_allreduce_add_rms_norm.argtypes = [vp, i32, vp, vp, vp, vp, vp, i64, i64, i64,
                                                      f32, i32]
        lib.oracle_layer_norm.argtypes = [vp, vp, vp, vp, i64, i64, i64, f32, i32]
        lib.oracle_rope_f64.argtypes = [vp, vp, i64, i64, i64, i64, i64, i32, f32, f32, i64, i32]
        lib.oracle_norm_rope.argtypes = [vp, vp, vp, i64, i64, i64, i64, i64, i32, f32, f32,
                                         i64, i32, f32, i32]
        lib.oracle_rope_ex.argtypes = [vp, vp, vp, vp, i64, i64, i64, i64, i64, i64, i32, f32, f32,
                                       i64, i32, i32, f32, i32]
        lib.oracle_rms_norm_vjp.argtypes = [vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, f32, i32]
        lib.oracle_layer_norm_vjp.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i64, i64, i64,
                                              f32, i32]
        for name in ("oracle_rms_norm", "oracle_add_rms_norm", "oracle_layer_norm",
                     "oracle_rope_f64", "oracle_norm_rope", "oracle_rope_ex",
                     "oracle_rms_norm_vjp", "oracle_layer_norm_vjp"):
            getattr(lib, name).restype = ctypes.c_int
        self.lib = lib
        self.path = path
        self.last_threads = 1

    def _run(self, fn, rows, threads):
        chunks = _chunks(rows, threads)
        if len(chunks) == 1:
            rcs = [fn(*chunks[0])]
        else:
            with ThreadPoolExecutor(len(chunks)) as ex:
                rcs = list(ex.map(lambda c: fn(*c), chunks))
        if any(rc != 0 for rc in rcs):
            raise MemoryError("oracle: row buffer allocation failed")
        self.last_threads = len(chunks)

    def round_bf16(self, v) -> np.ndarray:
        """Round float64 values to bfloat16 bit patterns (nearest, ties to even, once)."""
        v = np.ascontiguousarray(v, dtype=np.float64)
        out = np.empty(v.shape, np.uint16)
        self.lib.oracle_round_bf16(_ptr(v), _ptr(out), v.size)
        return out

    def rms_norm(self, x, w, eps, threads=None):
        """y = x / sqrt(mean(x^2) + eps) * w per row of x [rows, D]; w None means 1."""
        x, dt = _io(x, "x")
        rows, D = x.shape
        w = None if w is None else _io(w, "w")[0]
        y = np.empty((rows, D), np.float64)
        self._run(lambda a, b: self.lib.oracle_rms_norm(_ptr(x), _ptr(w), _ptr(y), a, b, D, eps,
                                                        dt), rows, threads)
        return y

    def add_rms_norm(self, x, r, w, eps, threads=None):
        """(y, h): h = x + r in binary32 rounded once to the I/O type, y = RmsNorm(h)."""
        x, dt = _io(x, "x")
        r = _io(r, "r")[0]
        rows, D = x.shape
        w = None if w is None else _io(w, "w")[0]
        y = np.empty((rows, D), np.float64)
        h = np.empty((rows, D), x.dtype)
        self._run(lambda a, b: self.lib.oracle_add_rms_norm(_ptr(x), _ptr(r), _ptr(w), _ptr(y),
                                                            _ptr(h), a, b, D, eps, dt),
                  rows, threads)
        return y, h

    def llama3_freqs(self, dims, base, factor, low_freq_factor, high_freq_factor, orig):
        """Llama 3 NTK-by-parts scaled frequencies theta_i, i < dims/2 (float64)."""
        out = np.empty(dims // 2, np.float64)
        if self.lib.oracle_llama3_freqs(dims, base, factor, low_freq_factor, high_freq_factor,
                                        orig, _ptr(out)) != 0:
            raise ValueError("arguments outside the Llama 3 scaling's domain")
        return out

    def yarn_freqs(self, dims, base, s, L, alpha=1.0, beta=32.0):
        """(frequencies h(theta_d), d < dims/2, float64; temperature factor sqrt(1/t)) of
        YaRN with extension factor s over original context length L."""
        out = np.empty(dims // 2, np.float64)
        mscale = ctypes.c_double(0.0)
        if self.lib.oracle_yarn_freqs(dims, base, s, L, alpha, beta, _ptr(out),
                                      ctypes.byref(mscale)) != 0:
            raise ValueError("arguments outside YaRN's domain")
        return out, mscale.value

    def suscaled_freqs(self, dims, base, short_factors, long_factors, seq_len, max_pos, orig):
        """(frequencies theta_i / lambda_i, i < dims/2, float64; attention factor) of the
        LongRoPE / SuScaled scaling: lambda the long factors when seq_len exceeds the
        original context orig, else the short ones."""
        sf = np.ascontiguousarray(short_factors, np.float64)
        lf = np.ascontiguousarray(long_factors, np.float64)
        if sf.shape != (dims // 2,) or lf.shape != (dims // 2,):
            raise ValueError("factor lists must hold dims / 2 values")
        out = np.empty(dims // 2, np.float64)
        mscale = ctypes.c_double(0.0)
        if self.lib.oracle_suscaled_freqs(dims, base, _ptr(sf), _ptr(lf), seq_len, max_pos, orig,
                                          _ptr(out), ctypes.byref(mscale)) != 0:
            raise ValueError("arguments outside the SuScaled scaling's domain")
        return out, mscale.value

    def allreduce_add_rms_norm(self, parts, r, w, eps, threads=None):
        """(y, h, x): x = the sum of the partial tensors (in order, in double) rounded once
        to the I/O type, then add_rms_norm(x, r)."""
        ps = [_io(p, "part") for p in parts]
        if not ps:
            raise ValueError("at least one partial tensor")
        dt = ps[0][1]
        ps = [p for p, _ in ps]
        r = _io(r, "r")[0]
        rows, D = r.shape
        if any(p.shape != (rows, D) or p.dtype != r.dtype for p in ps):
            raise ValueError("partial tensors must match r in shape and dtype")
        w = None if w is None else _io(w, "w")[0]
        y = np.empty((rows, D), np.float64)
        h = np.empty((rows, D), r.dtype)
        x = np.empty((rows, D), r.dtype)
        table = (ctypes.c_void_p * len(ps))(*[p.ctypes.data for p in ps])
        self._run(lambda a, b: self.lib.oracle_allreduce_add_rms_norm(
            ctypes.cast(table, ctypes.c_void_p), len(ps), _ptr(r), _ptr(w), _ptr(y), _ptr(x),
            _ptr(h), a, b, D, eps, dt), rows, threads)
        return y, h, x

    def layer_norm(self, x, w, b, eps, threads=None):
        """y = (x - mean) / sqrt(var + eps) * w + b per row; w None means 1, b None 0."""
        x, dt = _io(x, "x")
        rows, D = x.shape
        w = None if w is None else _io(w, "w")[0]
        b = None if b is None else _io(b, "b")[0]
        y = np.empty((rows, D), np.float64)
        self._run(lambda a, c: self.lib.oracle_layer_norm(_ptr(x), _ptr(w), _ptr(b), _ptr(y), a,
                                                          c, D, eps, dt), rows, threads)
        return y

    def rope_f64(self, x, L, dims, traditional, base, scale, offset, forward=True, threads=None):
        """Rope of float64 rows x [rows, D]; row k is at position offset + (k mod L)."""
        x = np.ascontiguousarray(x, dtype=np.float64)
        rows, D = x.shape
        y = np.empty_like(x)
        self._run(lambda a, b: self.lib.oracle_rope_f64(_ptr(x), _ptr(y), a, b, L, D, dims,
                                                        int(traditional), base, scale, offset,
                                                        int(forward)), rows, threads)
        return y

    def norm_rope(self, x, w, L, dims, traditional, base, scale, offset, normalize, eps,
                  threads=None):
        """NormRope of x [rows, D] (rows = B*H*L, row k at l = k mod L)."""
        x, dt = _io(x, "x")
        rows, D = x.shape
        w = None if w is None else _io(w, "w")[0]
        y = np.empty((rows, D), np.float64)
        self._run(lambda a, b: self.lib.oracle_norm_rope(_ptr(x), _ptr(w), _ptr(y), a, b, L, D,
                                                         dims, int(traditional), base, scale,
                                                         offset, int(normalize), eps, dt),
                  rows, threads)
        return y


    def rope_ex(self, x, w, L, dims, traditional, base, scale, offset, normalize, eps,
                forward=True, freqs=None, y=None, y_len=0, threads=None):
        """General NormRope / Rope: freqs (dims/2 values) replace base^(-2i/dims);
        forward=False rotates back; y_len > 0 writes rows into the float64 cache y
        [rows/L * y_len, D] at positions offset + l (other cache rows untouched)."""
        x, dt = _io(x, "x")
        rows, D = x.shape
        w = None if w is None else _io(w, "w")[0]
        f = None if freqs is None else np.ascontiguousarray(freqs, dtype=np.float64)
        if y_len:
            assert y is not None and y.dtype == np.float64 and y.flags.c_contiguous
            assert y.shape == (rows // L * y_len, D)
        else:
            y = np.empty((rows, D), np.float64)
        self._run(lambda a, b: self.lib.oracle_rope_ex(
            _ptr(x), _ptr(w), _ptr(f), _ptr(y), a, b, L, y_len, D, dims, int(traditional), base,
            scale, offset, int(forward), int(normalize), eps, dt), rows, threads)
        return y


    def _vjp(self, fn, nsums, x, g, w, threads):
        x, dt = _io(x, "x")
        g = _io(g, "g")[0]
        rows, D = x.shape
        w = None if w is None else _io(w, "w")[0]
        dx = np.empty((rows, D), np.float64)
        mdx = np.empty((rows, D), np.float64)
        chunks = _chunks(rows, threads)
        parts = [np.zeros((2 * nsums, D), np.float64) for _ in chunks]

        def one(i):
            a, b = chunks[i]
            p = parts[i]
            return fn(x, w, g, dx, mdx, p, a, b, D, dt)

        if len(chunks) == 1:
            rcs = [one(0)]
        else:
            with ThreadPoolExecutor(len(chunks)) as ex:
                rcs = list(ex.map(one, range(len(chunks))))
        if any(rc != 0 for rc in rcs):
            raise MemoryError("oracle: row buffer allocation failed")
        self.last_threads = len(chunks)
        tot = np.zeros((2 * nsums, D), np.float64)
        for p in parts:            # chunk order: a fixed summation order
            tot += p
        return dx, mdx, tot

    def rms_norm_vjp(self, x, w, g, eps, threads=None):
        """RmsNormVjp: (dx, dw or None, mag_dx, mag_dw) -- mag_* are the magnitude sums
        bounding a float32 evaluation's rounding error."""
        def fn(x, w, g, dx, mdx, p, a, b, D, dt):
            return self.lib.oracle_rms_norm_vjp(_ptr(x), _ptr(w), _ptr(g), _ptr(dx), _ptr(p[0]),
                                                _ptr(mdx), _ptr(p[1]), a, b, D, eps, dt)
        dx, mdx, tot = self._vjp(fn, 1, x, g, w, threads)
        return dx, (tot[0] if w is not None else None), mdx, tot[1]

    def layer_norm_vjp(self, x, w, g, eps, threads=None):
        """LayerNormVjp: (dx, dw, db, mag_dx, mag_dw, mag_db); dw is None without w."""
        def fn(x, w, g, dx, mdx, p, a, b, D, dt):
            return self.lib.oracle_layer_norm_vjp(_ptr(x), _ptr(w), _ptr(g), _ptr(dx), _ptr(p[0]),
                                                  _ptr(p[1]), _ptr(mdx), _ptr(p[2]), _ptr(p[3]),
                                                  a, b, D, eps, dt)
        dx, mdx, tot = self._vjp(fn, 2, x, g, w, threads)
        return dx, (tot[0] if w is not None else None), tot[1], mdx, tot[2], tot[3]


_default = None


def get() -> Oracle:
    """The oracle built from oracle.c (compiled on first use if needed)."""
    global _default
    if _default is None:
        _default = Oracle(build())
    return _default


def round_bf16(v):
    return get().round_bf16(v)


def rms_norm(x, w, eps, threads=None):
    return get().rms_norm(x, w, eps, threads)


def add_rms_norm(x, r, w, eps, threads=None):
    return get().add_rms_norm(x, r, w, eps, threads)


def llama3_freqs(dims, base, factor, low_freq_factor, high_freq_factor, orig):
    return get().llama3_freqs(dims, base, factor, low_freq_factor, high_freq_factor, orig)


def yarn_freqs(dims, base, s, L, alpha=1.0, beta=32.0):
    return get().yarn_freqs(dims, base, s, L, alpha, beta)


def suscaled_freqs(dims, base, short_factors, long_factors, seq_len, max_pos, orig):
    return get().suscaled_freqs(dims, base, short_factors, long_factors, seq_len, max_pos, orig)


def allreduce_add_rms_norm(parts, r, w, eps, threads=None):
    return get().allreduce_add_rms_norm(parts, r, w, eps, threads)


def layer_norm(x, w, b, eps, threads=None):
    return get().layer_norm(x, w, b, eps, threads)


def rope_f64(x, L, dims, traditional, base, scale, offset, forward=True, threads=None):
    return get().rope_f64(x, L, dims, traditional, base, scale, offset, forward, threads)


def norm_rope(x, w, L, dims, traditional, base, scale, offset, normalize, eps, threads=None):
    return get().norm_rope(x, w, L, dims, traditional, base, scale, offset, normalize, eps,
                           threads)


def rope_ex(x, w, L, dims, traditional, base, scale, offset, normalize, eps, forward=True,
            freqs=None, y=None, y_len=0, threads=None):
    return get().rope_ex(x, w, L, dims, traditional, base, scale, offset, normalize, eps,
                         forward, freqs, y, y_len, threads)


def rms_norm_vjp(x, w, g, eps, threads=None):
    return get().rms_norm_vjp(x, w, g, eps, threads)


def layer_norm_vjp(x, w, g, eps, threads=None):
    return get().layer_norm_vjp(x, w, g, eps, threads)
