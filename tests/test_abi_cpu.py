"""The C ABI on a machine without a GPU: symbols, status strings, host-side validation.

Every call here fails (or returns NV_OK for rows == 0) before the library touches the
CUDA runtime, so nothing is launched.
"""
import ctypes
import math
import os
import re
import subprocess

import pytest

import rope_add_rms_b200 as nv

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "nvnorm.h")

OK, INVALID, UNSUPPORTED = nv.NV_OK, nv.NV_ERR_INVALID_ARG, nv.NV_ERR_UNSUPPORTED
BF16, F32, F16 = nv.NV_BF16, nv.NV_F32, nv.NV_F16
FAKE = ctypes.c_void_p(0x10000)     # never dereferenced: validation stops first


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*NV_API\s+(?:const\s+)?\w+\*?\s+(nv_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for fn in ("nv_rms_norm", "nv_add_rms_norm", "nv_layer_norm", "nv_norm_rope",
               "nv_status_string", "nv_last_error"):
        assert fn in names


def test_library_exports_every_declared_symbol():
    out = subprocess.run(["nm", "-D", "--defined-only", nv.library_path], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    missing = [f for f in declared_functions() if f not in exported]
    assert not missing, f"declared but not exported: {missing}"
    lib = nv.library()
    for f in declared_functions():
        getattr(lib, f)
    # nothing else leaks out of the library (hidden visibility)
    ours = {s for s in exported if s.startswith("nv_")}
    assert ours == set(declared_functions())


def test_status_strings_and_version():
    lib = nv.library()
    assert lib.nv_status_string(0) == b"NV_OK"
    assert lib.nv_status_string(1) == b"NV_ERR_INVALID_ARG"
    assert lib.nv_status_string(2) == b"NV_ERR_UNSUPPORTED"
    assert lib.nv_status_string(3) == b"NV_ERR_CUDA"
    assert lib.nv_status_string(99) == b"NV_STATUS_UNKNOWN"
    assert lib.nv_version() >= 100


def rms(x=FAKE, w=None, y=FAKE, rows=4, D=8, eps=1e-5, dt=BF16):
    return nv.library().nv_rms_norm(x, w, y, rows, D, eps, dt, None)


def add(x=FAKE, r=FAKE, w=None, y=FAKE, h=ctypes.c_void_p(0x20000), rows=4, D=8, eps=1e-5,
        dt=BF16):
    return nv.library().nv_add_rms_norm(x, r, w, y, h, rows, D, eps, dt, None)


def layer(x=FAKE, w=None, b=None, y=FAKE, rows=4, D=8, eps=1e-5, dt=BF16):
    return nv.library().nv_layer_norm(x, w, b, y, rows, D, eps, dt, None)


def rope(x=FAKE, w=None, y=FAKE, rows=8, L=4, D=8, dims=8, trad=0, base=10000.0, scale=1.0,
         offset=0, normalize=1, eps=1e-6, dt=BF16):
    return nv.library().nv_norm_rope(x, w, y, rows, L, D, dims, trad, base, scale, offset,
                                     normalize, eps, dt, None)


def rope_general(x=FAKE, w=None, freqs=None, y=FAKE, rows=8, L=4, y_len=0, D=8, dims=8, trad=0,
                 base=10000.0, scale=1.0, offset=0, forward=1, normalize=1, eps=1e-6, dt=BF16):
    return nv.library().nv_rope(x, w, freqs, y, rows, L, y_len, D, dims, trad, base, scale, offset,
                                forward, normalize, eps, dt, None)


def vjp(op="rms", x=FAKE, w=None, g=FAKE, dx=FAKE, dw=None, db=None, ws=None, ws_bytes=0, rows=4,
        D=64, eps=1e-5, dt=BF16):
    lib = nv.library()
    if op == "rms":
        return lib.nv_rms_norm_vjp(x, w, g, dx, dw, ws, ws_bytes, rows, D, eps, dt, None)
    return lib.nv_layer_norm_vjp(x, w, g, dx, dw, db, ws, ws_bytes, rows, D, eps, dt, None)


def vjp_static(x=FAKE, w=None, g=FAKE, dx=FAKE, dw=None, rows=4, D=64, eps=1e-5, dt=BF16):
    return nv.library().nv_rms_norm_vjp_static(x, w, g, dx, dw, rows, D, eps, dt, None)


def allreduce(parts=(FAKE, FAKE), n=None, r=FAKE, w=None, y=FAKE, h=ctypes.c_void_p(0x20000),
              x_out=None, rows=4, D=8, eps=1e-5, dt=BF16):
    table = None if parts is None else (ctypes.c_void_p * max(len(parts), 1))(*parts)
    return nv.library().nv_allreduce_add_rms_norm(table, len(parts or ()) if n is None else n,
                                                  r, w, y, h, x_out, rows, D, eps, dt, None)


def host_add(x=FAKE, r=FAKE, y=FAKE, h=ctypes.c_void_p(0x20000), rows=4, D=8, chunk=0):
    return nv.library().nv_add_rms_norm_host(x, r, None, y, h, FAKE, FAKE, FAKE, FAKE, rows, D,
                                             1e-5, BF16, chunk, None)


def last_error():
    return nv.library().nv_last_error().decode()


@pytest.mark.parametrize("call, status, words", [
    (lambda: rms(dt=7), INVALID, "dtype"),
    (lambda: rms(dt=F16), UNSUPPORTED, "F16"),
    (lambda: rms(rows=-1), INVALID, "rows"),
    (lambda: rms(D=0), INVALID, "D"),
    (lambda: rms(eps=-1e-5), INVALID, "eps"),
    (lambda: rms(eps=math.nan), INVALID, "eps"),
    (lambda: rms(eps=math.inf), INVALID, "eps"),
    (lambda: rms(x=None), INVALID, "x is NULL"),
    (lambda: rms(y=None), INVALID, "y is NULL"),
    (lambda: rms(rows=2 ** 62, D=2 ** 20), INVALID, "overflows"),
    (lambda: add(r=None), INVALID, "r is NULL"),
    (lambda: add(h=None), INVALID, "h is NULL"),
    (lambda: add(h=FAKE), INVALID, "same buffer"),
    (lambda: layer(D=-3), INVALID, "D"),
    (lambda: layer(eps=-0.5, dt=F32), INVALID, "eps"),
    (lambda: rope(L=0), INVALID, "L"),
    (lambda: rope(rows=9, L=4), INVALID, "multiple of L"),
    (lambda: rope(dims=7), INVALID, "dims"),
    (lambda: rope(dims=0), INVALID, "dims"),
    (lambda: rope(dims=10, D=8), INVALID, "dims"),
    (lambda: rope(base=0.0), INVALID, "base"),
    (lambda: rope(base=-2.0), INVALID, "base"),
    (lambda: rope(base=math.inf), INVALID, "base"),
    (lambda: rope(scale=math.nan), INVALID, "scale"),
    (lambda: rope(offset=-1), INVALID, "offset"),
    (lambda: rope(eps=-1.0), INVALID, "eps"),
    (lambda: rope(x=None), INVALID, "x is NULL"),
    (lambda: rope_general(y_len=-1), INVALID, "y_len"),
    (lambda: rope_general(y_len=5, offset=2, L=4), INVALID, "cache length"),
    (lambda: rope_general(base=0.0), INVALID, "base"),
    (lambda: rope_general(base=0.0, freqs=FAKE, x=None), INVALID, "x is NULL"),
    (lambda: rope_general(dims=3), INVALID, "dims"),
    (lambda: vjp(w=FAKE), INVALID, "dw must be given"),
    (lambda: vjp(dw=FAKE), INVALID, "dw must be given"),
    (lambda: vjp(op="layer", w=FAKE), INVALID, "dw must be given"),
    (lambda: vjp(w=FAKE, dw=FAKE), INVALID, "workspace is NULL"),
    (lambda: vjp(w=FAKE, dw=FAKE, ws=FAKE, ws_bytes=16), INVALID, "workspace of 16 bytes"),
    (lambda: vjp(op="layer", db=FAKE, ws=FAKE, ws_bytes=16), INVALID, "workspace of 16"),
    (lambda: vjp_static(D=7), UNSUPPORTED, "vjp needs D"),
    (lambda: vjp_static(D=32768), UNSUPPORTED, "16384"),
    (lambda: vjp_static(dw=FAKE), INVALID, "dw must be given"),
    (lambda: vjp(g=None), INVALID, "g is NULL"),
    (lambda: allreduce(n=0), INVALID, "nparts"),
    (lambda: allreduce(parts=(FAKE,) * 9), INVALID, "nparts"),
    (lambda: allreduce(parts=None, n=2), INVALID, "parts is NULL"),
    (lambda: allreduce(parts=(FAKE, None)), INVALID, "parts[1] is NULL"),
    (lambda: allreduce(r=None), INVALID, "r is NULL"),
    (lambda: allreduce(h=None), INVALID, "h is NULL"),
    (lambda: allreduce(dt=F16), UNSUPPORTED, "F16"),
    (lambda: host_add(x=None), INVALID, "x_host is NULL"),
    (lambda: host_add(h=FAKE), INVALID, "same buffer"),
    (lambda: nv.library().nv_selftest_bounded_wait(0, None), INVALID, "ctas"),
    (lambda: nv.library().nv_selftest_bounded_wait(65, None), INVALID, "ctas"),
    (lambda: host_add(chunk=-1), INVALID, "chunk_rows"),
])
def test_invalid_arguments_are_rejected_on_the_host(call, status, words):
    assert call() == status
    assert words in last_error()


def test_zero_rows_is_a_no_op():
    assert rms(x=None, y=None, rows=0) == OK
    assert add(x=None, r=None, y=None, h=None, rows=0) == OK
    assert layer(x=None, y=None, rows=0) == OK
    assert rope(x=None, y=None, rows=0) == OK
    assert allreduce(parts=None, n=1, r=None, y=None, h=None, rows=0) == OK
    assert host_add(x=None, r=None, y=None, h=None, rows=0) == OK


def test_plain_rope_ignores_eps():
    # normalize == 0: eps is unused, so a negative eps is not an error (stops at x NULL)
    assert rope(normalize=0, eps=-1.0, x=None) == INVALID
    assert "x is NULL" in last_error()


@pytest.mark.parametrize("op, D, dtype, want", [
    ("add_rms_norm", 4096, "bf16", dict(path=1, vec_per_thread=4, threads_per_row=128,
                                        rows_per_cta=1, ctas_per_sm=0)),
    ("add_rms_norm", 5120, "bf16", dict(path=1, vec_per_thread=4, threads_per_row=160)),
    ("add_rms_norm", 16384, "f32", dict(path=1, vec_per_thread=8, threads_per_row=512)),
    ("add_rms_norm", 7, "bf16", dict(path=2)),
    ("add_rms_norm", 2 ** 17, "bf16", dict(path=2)),
    ("rms_norm", 512, "f32", dict(path=1, vec_per_thread=4, threads_per_row=32, rows_per_cta=4)),
    ("rms_norm", 128, "bf16", dict(path=1, vec_per_thread=4, threads_per_row=4, rows_per_cta=32)),
    ("rms_norm", 512, "bf16", dict(path=1, vec_per_thread=4, threads_per_row=16, rows_per_cta=8)),
    ("add_rms_norm", 128, "bf16", dict(path=1, vec_per_thread=1, threads_per_row=16, rows_per_cta=8)),
    ("add_rms_norm", 512, "bf16", dict(path=1, vec_per_thread=2, threads_per_row=32, rows_per_cta=4)),
    ("layer_norm", 32, "bf16", dict(path=1)),
    ("layer_norm", 64, "bf16", dict(path=5, vec_per_thread=4, threads_per_row=2, rows_per_cta=384,
                                    stages=1)),
    ("layer_norm", 128, "bf16", dict(path=5, vec_per_thread=4, threads_per_row=4, rows_per_cta=192,
                                     stages=1)),
    ("layer_norm", 256, "bf16", dict(path=5, vec_per_thread=4, threads_per_row=8, rows_per_cta=96,
                                     stages=1)),
    ("layer_norm", 512, "bf16", dict(path=5, vec_per_thread=4, threads_per_row=16, rows_per_cta=48,
                                     stages=1)),
    ("layer_norm", 768, "bf16", dict(path=5, vec_per_thread=6, threads_per_row=16, rows_per_cta=48,
                                     stages=1)),
    ("layer_norm", 1024, "bf16", dict(path=5, vec_per_thread=4, threads_per_row=32, rows_per_cta=24,
                                      stages=1)),
    ("layer_norm", 1536, "bf16", dict(path=5, vec_per_thread=6, threads_per_row=32, rows_per_cta=24,
                                      stages=1)),
    ("layer_norm", 2048, "bf16", dict(path=5, vec_per_thread=8, threads_per_row=32, rows_per_cta=24,
                                      stages=1)),
    ("layer_norm", 4096, "bf16", dict(path=5, vec_per_thread=8, threads_per_row=64, rows_per_cta=12,
                                      stages=1)),
    ("layer_norm", 8192, "bf16", dict(path=5, vec_per_thread=8, threads_per_row=128, rows_per_cta=6,
                                      stages=1)),
    ("layer_norm", 8192, "f32", dict(path=1, vec_per_thread=8, threads_per_row=256)),
    ("layer_norm", 128, "f32", dict(path=1, vec_per_thread=8, threads_per_row=4, rows_per_cta=32)),
    ("layer_norm", 512, "f32", dict(path=1, vec_per_thread=8, threads_per_row=16, rows_per_cta=8)),
    ("layer_norm", 32768, "bf16", dict(path=1)),
    ("norm_rope", 128, "bf16", dict(path=1, vec_per_thread=2, threads_per_row=8)),
    ("norm_rope", 1000, "bf16", dict(path=2)),
])
def test_plan_selection(op, D, dtype, want):
    import torch
    p = nv.nv_describe_plan(op, 8192, D, {"bf16": torch.bfloat16, "f32": torch.float32}[dtype])
    for k, v in want.items():
        assert p[k] == v, (op, D, dtype, p)


def test_vjp_workspace_size():
    lib = nv.library()
    assert lib.nv_norm_vjp_workspace_size(0, 8192, 4096) == 512 * 4096 * 4
    assert lib.nv_norm_vjp_workspace_size(2, 100, 1024) == 2 * 100 * 1024 * 4
    assert lib.nv_norm_vjp_workspace_size(1, 100, 1024) == 0
    assert lib.nv_norm_vjp_workspace_size(0, 0, 1024) == 0
    # narrow rows keep more partial sums (up to 2^21 / D of them)
    assert lib.nv_norm_vjp_workspace_size(0, 100000, 512) == 4096 * 512 * 4
    assert lib.nv_norm_vjp_workspace_size(2, 100000, 16384) == 2 * 512 * 16384 * 4


# ---- Llama 3 frequency scaling: a host-side helper, testable without a GPU ------------------

@pytest.mark.parametrize("args", [(128, 500000.0, 32.0, 1.0, 4.0, 8192),
                                  (64, 10000.0, 8.0, 2.0, 16.0, 4096),
                                  (256, 1000000.0, 16.0, 1.0, 8.0, 131072),
                                  (4, 16.0, 8.0, 1.0, 4.0, 50), (128, 500000.0, 1.0, 1.0, 4.0, 8192)])
def test_rope_llama3_freqs_matches_the_oracle(args):
    import numpy as np
    import oracle
    got = nv.rope_llama3_freqs(*args).numpy()
    want = oracle.llama3_freqs(args[0], args[1], args[2], args[3], args[4],
                               float(args[5])).astype(np.float32)
    ulps = np.abs(got.view(np.int32).astype(np.int64) - want.view(np.int32).astype(np.int64))
    assert ulps.max() <= 1, f"{int(ulps.max())} float ulps apart"


@pytest.mark.parametrize("kw, words", [
    (dict(dims=7), "dims"), (dict(dims=0), "dims"), (dict(base=0.0), "base"),
    (dict(factor=0.5), "factor"), (dict(low_freq_factor=4.0, high_freq_factor=4.0), "low_freq"),
    (dict(original_max_position=0), "original_max_position")])
def test_rope_llama3_freqs_rejects(kw, words):
    args = dict(dims=128, base=500000.0, factor=32.0, low_freq_factor=1.0, high_freq_factor=4.0,
                original_max_position=8192)
    args.update(kw)
    with pytest.raises(nv.NvError, match=words):
        nv.rope_llama3_freqs(**args)


# ---- YaRN frequency scaling: also a host-side helper ------------------------------------------

@pytest.mark.parametrize("args", [(128, 10000.0, 4.0, 4096, 1.0, 32.0),
                                  (128, 500000.0, 16.0, 8192, 1.0, 32.0),
                                  (64, 10000.0, 8.0, 2048, 2.0, 8.0),
                                  (8, 10000.0, 4.0, 4096, 1.0, 32.0),
                                  (128, 10000.0, 1.0, 4096, 1.0, 32.0)])
def test_rope_yarn_freqs_matches_the_oracle(args):
    import numpy as np
    import oracle
    got, m = nv.rope_yarn_freqs(*args)
    want, want_m = oracle.yarn_freqs(args[0], args[1], args[2], float(args[3]), args[4], args[5])
    got, want = got.numpy(), want.astype(np.float32)
    ulps = np.abs(got.view(np.int32).astype(np.int64) - want.view(np.int32).astype(np.int64))
    assert ulps.max() <= 1, f"{int(ulps.max())} float ulps apart"
    assert abs(m - want_m) <= 2.0 ** -23 * want_m


@pytest.mark.parametrize("kw, words", [
    (dict(dims=5), "dims"), (dict(base=-1.0), "base"), (dict(factor=0.9), "factor"),
    (dict(alpha=0.0), "alpha"), (dict(alpha=32.0, beta=32.0), "alpha"),
    (dict(original_max_position=-4), "original_max_position")])
def test_rope_yarn_freqs_rejects(kw, words):
    args = dict(dims=128, base=10000.0, factor=4.0, original_max_position=4096, alpha=1.0,
                beta=32.0)
    args.update(kw)
    with pytest.raises(nv.NvError, match=words):
        nv.rope_yarn_freqs(**args)


# ---- SuScaled (LongRoPE) frequency scaling: also a host-side helper ----------------------------

def _factors(n, lo, hi, seed):
    import numpy as np
    return np.random.default_rng(seed).uniform(lo, hi, n).astype(np.float32)


@pytest.mark.parametrize("dims, seq_len, max_pos, orig", [(128, 4096, 131072, 4096),
                                                          (128, 4097, 131072, 4096),
                                                          (96, 100000, 131072, 4096),
                                                          (64, 10, 2048, 2048),
                                                          (4, 0, 8192, 4096)])
def test_rope_suscaled_freqs_matches_the_oracle(dims, seq_len, max_pos, orig):
    import numpy as np
    import oracle
    sf, lf = _factors(dims // 2, 1.0, 1.2, 1), _factors(dims // 2, 1.0, 60.0, 2)
    got, m = nv.rope_suscaled_freqs(dims, sf, lf, seq_len, 10000.0, max_pos, orig)
    want, want_m = oracle.suscaled_freqs(dims, 10000.0, sf.astype(np.float64),
                                         lf.astype(np.float64), float(seq_len), float(max_pos),
                                         float(orig))
    got, want = got.numpy(), want.astype(np.float32)
    ulps = np.abs(got.view(np.int32).astype(np.int64) - want.view(np.int32).astype(np.int64))
    assert ulps.max() <= 1, f"{int(ulps.max())} float ulps apart"
    assert abs(m - want_m) <= 2.0 ** -23 * want_m


@pytest.mark.parametrize("kw, words", [
    (dict(dims=5), "dims"), (dict(base=-1.0), "base"), (dict(original_max_position=1), "original"),
    (dict(max_position=0), "max_position"), (dict(seq_len=-1), "seq_len"),
    (dict(long_factors=[1.0, 0.0]), "factor 1"), (dict(short_factors=[float("nan"), 1.0], seq_len=5),
                                                  "factor 0")])
def test_rope_suscaled_freqs_rejects(kw, words):
    args = dict(dims=4, short_factors=[1.0, 1.0], long_factors=[2.0, 2.0], seq_len=9000,
                base=10000.0, max_position=131072, original_max_position=4096)
    args.update(kw)
    with pytest.raises(nv.NvError, match=words):
        nv.rope_suscaled_freqs(**args)


@pytest.mark.skipif(__import__("torch").cuda.is_available(),
                    reason="checks the path taken when no CUDA device can be used")
@pytest.mark.parametrize("name, call", [
    ("rms_norm", lambda: rms()),
    ("add_rms_norm", lambda: add()),
    ("layer_norm", lambda: layer()),
    ("norm_rope", lambda: rope()),
    ("rope", lambda: rope_general()),
    ("rms_norm_vjp", lambda: vjp("rms")),
    ("layer_norm_vjp", lambda: vjp("layer")),
    ("allreduce_add_rms_norm", lambda: allreduce()),
    ("add_rms_norm_host", lambda: nv.library().nv_add_rms_norm_host(   # x, r, w=NULL, y, h
        *[ctypes.c_void_p(0x10000 * (i + 1)) for i in range(2)], None,  # on the host, then
        *[ctypes.c_void_p(0x10000 * (i + 3)) for i in range(6)], 4, 8,  # the four staging
        1e-5, BF16, 0, None)),                                            # device buffers
    ("selftest_bounded_wait", lambda: nv.library().nv_selftest_bounded_wait(1, None)),
])
def test_cuda_failures_are_reported_as_nv_err_cuda(name, call):
    """With no usable CUDA device, a well-formed call fails at its first CUDA runtime call:
    the status is NV_ERR_CUDA, the message names that call and the runtime's error, and no
    exception crosses the boundary (the process carries on)."""
    assert call() == nv.NV_ERR_CUDA, name
    msg = last_error()
    assert re.match(r"^\w[\w ]*: cudaError\w+ \(", msg), msg


def test_pointer_checks_switch_reports_the_former_setting():
    assert nv.nv_set_pointer_checks(False) is True     # on by default
    try:
        assert nv.nv_set_pointer_checks(False) is False
        # argument checks that need no driver query still apply with the queries off
        assert rms(D=0) == INVALID and "D" in last_error()
        assert add(h=FAKE) == INVALID and "same buffer" in last_error()
    finally:
        assert nv.nv_set_pointer_checks(True) is False
    assert nv.nv_set_pointer_checks(True) is True
