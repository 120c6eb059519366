"""nv_rms_norm_vjp_static: the gradient entry point for callers that cannot allocate.

Some callers are handed their buffers and may not allocate device memory themselves
(a plugin inside an inference engine that owns all memory, code under a fixed memory
budget, or a loop where cudaMalloc would synchronise the device).  For them the library
offers one entry point whose scratch memory is a fixed array inside the library instead
of a caller-provided workspace.  This file checks it through the C ABI against the
workspace entry point, on two calls in a row, and is collected last so that a run that
stops at the first failure has run every other test first.
"""
import ctypes

import pytest
import torch

import oracle
import rope_add_rms_b200 as nv
from rope_add_rms_b200 import synth
from checks import check_grad, to_host_bits

pytestmark = pytest.mark.gpu


def _static_vjp():
    fn = nv.library().nv_rms_norm_vjp_static
    vp, i64 = ctypes.c_void_p, ctypes.c_int64
    fn.argtypes = [vp, vp, vp, vp, vp, i64, i64, ctypes.c_float, ctypes.c_int32, vp]
    fn.restype = ctypes.c_int
    return fn


def _call(fn, x, w, g, dx, dw, eps, dt):
    rows, D = x.shape
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())  # noqa: E731
    st = fn(p(x), p(w), p(g), p(dx), p(dw), rows, D, eps, dt,
            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == nv.NV_OK, nv.library().nv_last_error().decode()


@pytest.mark.parametrize("dt", ["bf16", "f32"])
def test_static_scratch_vjp_matches_workspace_vjp_twice(dt):
    fn = _static_vjp()
    code = nv.NV_BF16 if dt == "bf16" else nv.NV_F32
    # two calls in a row on different shapes: the second must not see the first's partials
    for rows, D, seed in ((3000, 4096, 1), (777, 2048, 2), (3000, 4096, 1)):
        inp = synth.rms_inputs(rows, D, dt, seed=seed)
        g = synth.normal((rows, D), 0.0, 1.0, seed, 4, dt).cuda()
        x, w = inp["x"].cuda(), inp["w"].cuda()
        dx, dw = torch.empty_like(x), torch.empty_like(w)
        _call(fn, x, w, g, dx, dw, 1e-5, code)
        ref_dx, ref_dw = nv.rms_norm_vjp(x, w, g, eps=1e-5)        # workspace entry point
        torch.cuda.synchronize()
        assert torch.equal(dx, ref_dx), "dx must equal the workspace entry point's"
        o_dx, o_dw, mag_dx, mag_dw = oracle.rms_norm_vjp(synth.to_numpy(inp["x"]),
                                                         synth.to_numpy(inp["w"]),
                                                         to_host_bits(g), 1e-5)
        # both within the gradient bar of the oracle ...
        check_grad(dw, o_dw, mag_dw, "static dw")
        check_grad(ref_dw, o_dw, mag_dw, "workspace dw")
        # ... and of each other (the partial sums are grouped differently: each result
        # carries its own rounding, hence twice the magnitude allowance)
        ref_vals = ref_dw.double().cpu().numpy()
        check_grad(dw, ref_vals, 2 * mag_dw, "static vs workspace dw")


def test_static_scratch_vjp_widest_row_twice():
    """D = 16384: the scratch holds only 2^20 / D = 64 partial rows, so each CTA walks
    many rows; checked on two calls in a row against the workspace entry point."""
    fn = _static_vjp()
    rows, D = 4096, 16384
    inp = synth.rms_inputs(rows, D, "bf16", seed=3)
    g = synth.normal((rows, D), 0.0, 1.0, 3, 4, "bf16").cuda()
    x, w = inp["x"].cuda(), inp["w"].cuda()
    ref_dx, ref_dw = nv.rms_norm_vjp(x, w, g, eps=1e-6)
    o_dx, o_dw, mag_dx, mag_dw = oracle.rms_norm_vjp(synth.to_numpy(inp["x"]),
                                                     synth.to_numpy(inp["w"]),
                                                     to_host_bits(g), 1e-6)
    for _ in range(2):
        dx, dw = torch.full_like(x, float("nan")), torch.full_like(w, float("nan"))
        _call(fn, x, w, g, dx, dw, 1e-6, nv.NV_BF16)
        torch.cuda.synchronize()
        assert torch.equal(dx, ref_dx), "dx must equal the workspace entry point's"
        check_grad(dw, o_dw, mag_dw, "static dw, D = 16384")
        check_grad(dw, ref_dw.double().cpu().numpy(), 2 * mag_dw, "static vs workspace dw")


def test_static_scratch_vjp_zero_rows_gives_zero_dw():
    """rows = 0 with dw requested: dw is the sum over no rows, zero -- also right after a
    call that left partial sums in the scratch."""
    fn = _static_vjp()
    D = 4096
    inp = synth.rms_inputs(64, D, "bf16", seed=5)
    x, w = inp["x"].cuda(), inp["w"].cuda()
    g = synth.normal((64, D), 0.0, 1.0, 5, 4, "bf16").cuda()
    _call(fn, x, w, g, torch.empty_like(x), torch.empty_like(w), 1e-5, nv.NV_BF16)
    empty = torch.empty(0, D, dtype=torch.bfloat16, device="cuda")
    for _ in range(2):
        dw = torch.full_like(w, float("nan"))
        _call(fn, empty, w, empty, empty, dw, 1e-5, nv.NV_BF16)
        torch.cuda.synchronize()
        assert torch.count_nonzero(dw).item() == 0 and not torch.isnan(dw).any()


def test_static_scratch_vjp_rejects_wide_rows():
    fn = _static_vjp()
    x = torch.zeros(2, 32768, dtype=torch.bfloat16, device="cuda")
    w = torch.ones(32768, dtype=torch.bfloat16, device="cuda")
    st = fn(ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(w.data_ptr()),
            ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(x.data_ptr()),
            ctypes.c_void_p(w.data_ptr()), 2, 32768, 1e-5, nv.NV_BF16, None)
    assert st == nv.NV_ERR_UNSUPPORTED
    assert "16384" in nv.library().nv_last_error().decode()
