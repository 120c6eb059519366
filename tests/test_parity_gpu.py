"""GPU parity: every op and kernel variant of libnvnorm.so against the CPU oracle.

Inputs come from rope_add_rms_b200.synth (seeded, rounded to the I/O type on the host);
the same bytes go to the device and to the oracle.  Tolerances are those of
tests/checks.py: h bit-exact, bfloat16 y within one bfloat16 step of the oracle
rounded to bfloat16, float32 y within 1e-5 (1 + |ref|).
"""
import numpy as np
import pytest
import torch

import oracle
import rope_add_rms_b200 as nv
from rope_add_rms_b200 import synth
from checks import Guarded, check_exact, check_out, to_host_bits

pytestmark = pytest.mark.gpu

DT = {"bf16": torch.bfloat16, "f32": torch.float32}


def dev(t):
    return None if t is None else t.cuda()


def host(t):
    return None if t is None else synth.to_numpy(t)


def run_add(inp, eps, plan=None, guard=True):
    x, r, w = dev(inp["x"]), dev(inp["r"]), dev(inp["w"])
    if guard:
        gy, gh = Guarded(x.shape, x.dtype), Guarded(x.shape, x.dtype)
        y, h = gy.t, gh.t
    else:
        y, h = torch.empty_like(x), torch.empty_like(x)
    nv.nv_add_rms_norm(x, r, w, y, h, eps, plan=plan)
    torch.cuda.synchronize()
    if guard:
        assert gy.bands_intact() and gh.bands_intact(), "kernel wrote outside y or h"
    return y, h


# ---- add_rms_norm / rms_norm ---------------------------------------------------------------

ADD_SHAPES = [(147, 4096), (149, 5120), (33, 2048), (7, 16384), (1, 8192), (300, 1000),
              (64, 512), (3, 8), (256, 64), (5, 20000), (2, 32768)]


@pytest.mark.parametrize("dt", ["bf16", "f32"])
@pytest.mark.parametrize("rows,D", ADD_SHAPES)
def test_add_rms_norm(rows, D, dt):
    inp = synth.add_rms_inputs(rows, D, dt, seed=rows + D)
    eps = 1e-6
    y, h = run_add(inp, eps)
    ref, href = oracle.add_rms_norm(host(inp["x"]), host(inp["r"]), host(inp["w"]), eps)
    check_exact(h, href, "h")
    check_out(y, ref)


NARROW_PLANS = [None] + [dict(path=nv.PATH_ROWS, vec_per_thread=v, threads_per_row=g,
                               rows_per_cta=c)
                          for v, g, c in ((1, 8, 16), (2, 4, 64), (4, 2, 16), (4, 1, 32),
                                          (1, 16, 8), (2, 16, 2), (4, 4, 8))]


@pytest.mark.parametrize("dt", ["bf16", "f32"])
@pytest.mark.parametrize("D", [8, 16, 32, 64, 128, 256, 512])
def test_rms_rows_narrower_than_a_warp(D, dt):
    """rms_norm and add_rms_norm rows of fewer than 32 lanes, several rows to a warp, each
    reduced over its own lanes: automatic and forced shapes, a ragged row count (the last
    CTA partly empty), h bit-exact and guard bands around the outputs.  A shape whose CTA is
    not whole warps, or that does not cover the row, is refused."""
    rows = 1237
    inp = synth.add_rms_inputs(rows, D, dt, seed=D + 11)
    ref, href = oracle.add_rms_norm(host(inp["x"]), host(inp["r"]), host(inp["w"]), 1e-5)
    rref = oracle.rms_norm(host(inp["x"]), host(inp["w"]), 1e-5)
    x, w = dev(inp["x"]), dev(inp["w"])
    for p in NARROW_PLANS:
        plan = None if p is None else nv.Plan(**p)
        tag = f"D={D} {dt} {p}"
        try:
            y, h = run_add(inp, 1e-5, plan=plan)
        except nv.NvError as e:
            assert e.status == nv.NV_ERR_UNSUPPORTED, tag
            continue
        check_exact(h, href, "h " + tag)
        check_out(y, ref, tag)
        g = Guarded(x.shape, x.dtype)
        nv.nv_rms_norm(x, w, g.t, 1e-5, plan=plan)
        torch.cuda.synchronize()
        assert g.bands_intact(), tag
        check_out(g.t, rref, "rms " + tag)


@pytest.mark.parametrize("dt", ["bf16", "f32"])
@pytest.mark.parametrize("D", [8, 16, 32, 64, 128, 256])
def test_layer_rows_narrower_than_a_warp(D, dt):
    """layer_norm rows of fewer than 32 lanes in the register kernel, several rows to a warp:
    automatic and forced shapes, a ragged row count, rows whose mean dwarfs their spread
    (the centred second pass, voted warp-wide and kept only by the rows that asked for it)
    next to ordinary rows in the same warps, and guard bands."""
    rows = 1237
    x = synth.normal((rows, D), 0.5, 2.0, D, 0, dt)
    far = synth.normal((rows, D), 3000.0, 0.25, D, 1, dt)
    x[1::3] = far[1::3]   # every third row takes the centred pass
    w = synth.uniform((D,), 0.5, 1.5, D, 2, dt)
    b = synth.normal((D,), 0.0, 0.1, D, 3, dt)
    ref = oracle.layer_norm(host(x), host(w), host(b), 1e-5)
    xd, wd, bd = dev(x), dev(w), dev(b)
    for p in NARROW_PLANS:
        tag = f"D={D} {dt} {p}"
        g = Guarded(xd.shape, xd.dtype)
        try:
            nv.nv_layer_norm(xd, wd, bd, g.t, 1e-5, plan=None if p is None else nv.Plan(**p))
        except nv.NvError as e:
            assert e.status == nv.NV_ERR_UNSUPPORTED, tag
            continue
        torch.cuda.synchronize()
        assert g.bands_intact(), tag
        check_out(g.t, ref, tag)


@pytest.mark.parametrize("dt", ["bf16", "f32"])
@pytest.mark.parametrize("rows,D", [(17, 7), (3, 127), (2, 129), (9, 1), (5, 33), (4, 1001)])
def test_add_rms_norm_ragged_D_takes_generic_path(rows, D, dt):
    inp = synth.add_rms_inputs(rows, D, dt, seed=D)
    y, h = run_add(inp, 1e-5)
    ref, href = oracle.add_rms_norm(host(inp["x"]), host(inp["r"]), host(inp["w"]), 1e-5)
    check_exact(h, href, "h")
    check_out(y, ref)


# Forced variants for a [301, 4096] batch; threads_per_row is given for bfloat16
# (512 vectors per row) and doubled for float32 (1024 vectors per row).
VARIANTS = [dict(path=nv.PATH_GENERIC)] + [
    dict(path=nv.PATH_ROWS, vec_per_thread=v) for v in (1, 2, 4, 8)] + [
    dict(path=nv.PATH_ROWS, vec_per_thread=4, rows_per_cta=4, threads_per_row=128),
    dict(path=nv.PATH_ROWS, vec_per_thread=1, threads_per_row=512),
    dict(path=nv.PATH_ROWS, vec_per_thread=2, ctas_per_sm=1),
    dict(path=nv.PATH_ROWS, vec_per_thread=8, threads_per_row=64, rows_per_cta=4),
]


@pytest.mark.parametrize("dt", ["bf16", "f32"])
@pytest.mark.parametrize("plan", VARIANTS, ids=lambda p: "-".join(f"{k}{v}" for k, v in p.items()))
def test_add_rms_norm_every_variant(plan, dt):
    rows, D = 301, 4096
    plan = dict(plan)
    if dt == "f32" and "threads_per_row" in plan:
        plan["threads_per_row"] *= 2
        plan["rows_per_cta"] = max(1, plan.get("rows_per_cta", 1) // 2)
    inp = synth.add_rms_inputs(rows, D, dt, seed=11)
    y, h = run_add(inp, 1e-5, plan=nv.Plan(**plan))
    ref, href = oracle.add_rms_norm(host(inp["x"]), host(inp["r"]), host(inp["w"]), 1e-5)
    check_exact(h, href, "h")
    check_out(y, ref)


@pytest.mark.parametrize("dt", ["bf16", "f32"])
@pytest.mark.parametrize("rows,D,weight", [(64, 512, True), (129, 4096, False), (10, 7, True),
                                           (31, 16384, True)])
def test_rms_norm(rows, D, weight, dt):
    inp = synth.rms_inputs(rows, D, dt, seed=3, weight=weight)
    x, w = dev(inp["x"]), dev(inp["w"])
    g = Guarded(x.shape, x.dtype)
    nv.nv_rms_norm(x, w, g.t, 1e-6)
    torch.cuda.synchronize()
    assert g.bands_intact()
    check_out(g.t, oracle.rms_norm(host(inp["x"]), host(inp["w"]), 1e-6))


def test_rms_norm_small_config_fp32():
    """rms_norm fp32 x [64, 512] ~ N(0,1), w ~ U(0.5,1.5), eps 1e-6, seed 0 (full compare)."""
    inp = synth.rms_inputs(64, 512, "f32", seed=0)
    y = nv.rms_norm(dev(inp["x"]), dev(inp["w"]), eps=1e-6)
    torch.cuda.synchronize()
    check_out(y, oracle.rms_norm(host(inp["x"]), host(inp["w"]), 1e-6))


def test_add_rms_norm_equals_rms_norm_of_h():
    inp = synth.add_rms_inputs(97, 4096, "bf16", seed=5)
    y, h = run_add(inp, 1e-5)
    y2 = nv.rms_norm(h, dev(inp["w"]), eps=1e-5)
    torch.cuda.synchronize()
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16))


@pytest.mark.parametrize("alias", ["h=x", "h=r", "y=x", "y=r", "y=x,h=r"])
def test_add_rms_norm_in_place(alias):
    rows, D = 77, 4096
    inp = synth.add_rms_inputs(rows, D, "bf16", seed=6)
    ref, href = oracle.add_rms_norm(host(inp["x"]), host(inp["r"]), host(inp["w"]), 1e-5)
    x, r, w = dev(inp["x"]), dev(inp["r"]), dev(inp["w"])
    y, h = torch.empty_like(x), torch.empty_like(x)
    for a in alias.split(","):
        out, src = a.split("=")
        t = x if src == "x" else r
        if out == "y":
            y = t
        else:
            h = t
    nv.nv_add_rms_norm(x, r, w, y, h, 1e-5)
    torch.cuda.synchronize()
    check_exact(h, href, "h")
    check_out(y, ref)


def test_misaligned_pointers_take_generic_path():
    rows, D = 19, 4096
    inp = synth.add_rms_inputs(rows, D, "bf16", seed=8)
    n = rows * D
    big = torch.empty(4 * n + 16, dtype=torch.bfloat16, device="cuda")
    x, r, y, h = (big[1 + k * n: 1 + (k + 1) * n].view(rows, D) for k in range(4))  # 2-byte offset
    x.copy_(inp["x"])
    r.copy_(inp["r"])
    w = dev(inp["w"])
    nv.nv_add_rms_norm(x, r, w, y, h, 1e-5)
    torch.cuda.synchronize()
    ref, href = oracle.add_rms_norm(host(inp["x"]), host(inp["r"]), host(inp["w"]), 1e-5)
    check_exact(h, href, "h")
    check_out(y, ref)
    with pytest.raises(nv.NvError, match="UNSUPPORTED"):
        nv.nv_add_rms_norm(x, r, w, y, h, 1e-5, plan=nv.Plan(path=nv.PATH_ROWS))


def test_zero_and_special_rows():
    D = 4096
    x = torch.zeros(4, D, dtype=torch.bfloat16)
    x[1] = 3.0
    x[2, 5] = float("nan")
    x[3, 7] = float("inf")
    r = torch.zeros_like(x)
    w = torch.ones(D, dtype=torch.bfloat16)
    y, h = nv.add_rms_norm(x.cuda(), r.cuda(), w.cuda(), eps=1e-5)
    torch.cuda.synchronize()
    yh = y.float().cpu()
    assert (yh[0] == 0).all(), "a zero row normalises to zero when eps > 0"
    ref = oracle.add_rms_norm(host(x), host(r), host(w), 1e-5)[0]
    check_out(y[:2], ref[:2])
    assert torch.isnan(yh[2]).all() and torch.isnan(yh[3]).any(), "NaN/Inf stay in their row"


def test_zero_rows_launches_nothing():
    x = torch.empty(0, 4096, dtype=torch.bfloat16, device="cuda")
    y, h = nv.add_rms_norm(x, x.clone())
    assert y.shape == (0, 4096) and h.shape == (0, 4096)


def test_host_memory_undersized_and_overlapping_buffers_are_rejected():
    import ctypes
    x = torch.randn(8, 256, dtype=torch.bfloat16, device="cuda")
    w = torch.ones(256, dtype=torch.bfloat16, device="cuda")
    y = torch.empty_like(x)
    with pytest.raises(nv.NvError, match="not device memory"):
        nv.nv_rms_norm(x.cpu().pin_memory(), w, y, 1e-5)
    # 2^20 rows of 256 cannot fit the (at most a few MB) allocation holding x
    st = nv.library().nv_rms_norm(ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(w.data_ptr()),
                                  ctypes.c_void_p(y.data_ptr()), 1 << 20, 256, 1e-5, nv.NV_BF16,
                                  None)
    assert st == nv.NV_ERR_INVALID_ARG
    assert "past the end" in nv.library().nv_last_error().decode()
    with pytest.raises(nv.NvError, match="overlaps"):
        nv.nv_rms_norm(x, x[0], x, 1e-5)      # y == x is fine; w inside the output is not
    with pytest.raises(nv.NvError, match="same buffer"):
        nv.nv_add_rms_norm(x, x.clone(), w, y, y, 1e-5)
    big = torch.zeros(3 * 2048, dtype=torch.bfloat16, device="cuda")
    xs, ys = big[:2048].view(8, 256), big[128:128 + 2048].view(8, 256)
    with pytest.raises(nv.NvError, match="overlaps"):
        nv.nv_rms_norm(xs, w, ys, 1e-5)      # partial overlap of input and output


def test_pointer_checks_off_same_results_overlaps_still_rejected():
    """With the per-pointer driver queries off the ops give the same bits; a host buffer is
    caught only with them on; an output overlapping an input is rejected either way."""
    inp = synth.add_rms_inputs(300, 4096, "bf16", seed=21)
    x, r, w = dev(inp["x"]), dev(inp["r"]), dev(inp["w"])
    y0, h0 = nv.add_rms_norm(x, r, w, 1e-5)
    prev = nv.nv_set_pointer_checks(False)
    try:
        y1, h1 = nv.add_rms_norm(x, r, w, 1e-5)
        torch.cuda.synchronize()
        assert torch.equal(y0, y1) and torch.equal(h0, h1)
        big = torch.zeros(3 * 2048, dtype=torch.bfloat16, device="cuda")
        xs, ys = big[:2048].view(8, 256), big[128:128 + 2048].view(8, 256)
        with pytest.raises(nv.NvError, match="overlaps"):
            nv.nv_rms_norm(xs, w[:256], ys, 1e-5)
    finally:
        nv.nv_set_pointer_checks(prev)
    with pytest.raises(nv.NvError, match="not device memory"):
        nv.nv_rms_norm(x.cpu().pin_memory(), w, torch.empty_like(x), 1e-5)


# ---- staged (bulk-copy) path ----------------------------------------------------------------

STAGED = [dict(path=nv.PATH_STAGED),
          dict(path=nv.PATH_STAGED, rows_per_cta=2, ctas_per_sm=1),
          dict(path=nv.PATH_STAGED, rows_per_cta=4, ctas_per_sm=2, vec_per_thread=4),
          dict(path=nv.PATH_STAGED, rows_per_cta=3, ctas_per_sm=3, vec_per_thread=1),
          dict(path=nv.PATH_STAGED, rows_per_cta=5, ctas_per_sm=1, vec_per_thread=8)]


@pytest.mark.parametrize("dt", ["bf16", "f32"])
@pytest.mark.parametrize("plan", STAGED, ids=lambda p: "-".join(f"{k}{v}" for k, v in p.items()))
@pytest.mark.parametrize("rows,D", [(301, 4096), (1, 4096), (1000, 2048), (37, 5120), (5, 8192)])
def test_add_rms_norm_staged(rows, D, plan, dt):
    inp = synth.add_rms_inputs(rows, D, dt, seed=rows * 7 + D)
    try:
        y, h = run_add(inp, 1e-6, plan=nv.Plan(**plan))
    except nv.NvError as e:          # the shape does not fit this forced plan
        assert e.status == nv.NV_ERR_UNSUPPORTED
        pytest.skip(str(e))
    assert nv.nv_fault_count() == 0
    ref, href = oracle.add_rms_norm(host(inp["x"]), host(inp["r"]), host(inp["w"]), 1e-6)
    check_exact(h, href, "h")
    check_out(y, ref)


@pytest.mark.parametrize("dt", ["bf16", "f32"])
@pytest.mark.parametrize("weight", [True, False])
def test_rms_norm_staged(dt, weight):
    inp = synth.rms_inputs(513, 4096, dt, seed=1, weight=weight)
    x, w = dev(inp["x"]), dev(inp["w"])
    y = torch.empty_like(x)
    nv.nv_rms_norm(x, w, y, 1e-6, plan=nv.Plan(path=nv.PATH_STAGED))
    assert nv.nv_fault_count() == 0
    check_out(y, oracle.rms_norm(host(inp["x"]), host(inp["w"]), 1e-6))


def test_staged_in_place():
    inp = synth.add_rms_inputs(300, 4096, "bf16", seed=2)
    ref, href = oracle.add_rms_norm(host(inp["x"]), host(inp["r"]), host(inp["w"]), 1e-5)
    x, r, w = dev(inp["x"]), dev(inp["r"]), dev(inp["w"])
    nv.nv_add_rms_norm(x, r, w, x, r, 1e-5, plan=nv.Plan(path=nv.PATH_STAGED))   # y=x, h=r
    assert nv.nv_fault_count() == 0
    check_exact(r, href, "h")
    check_out(x, ref)


# ---- layer_norm --------------------------------------------------------------------------

@pytest.mark.parametrize("dt", ["bf16", "f32"])
@pytest.mark.parametrize("rows,D,wb", [(147, 8192, (1, 1)), (149, 5120, (1, 0)), (33, 4096, (0, 0)),
                                        (5, 16384, (1, 1)), (64, 512, (1, 1)), (9, 1001, (1, 1)),
                                        (3, 1, (1, 1)), (300, 256, (0, 1))])
def test_layer_norm(rows, D, wb, dt):
    inp = synth.layer_norm_inputs(rows, D, dt, seed=D + rows, weight=bool(wb[0]), bias=bool(wb[1]))
    x, w, b = dev(inp["x"]), dev(inp["w"]), dev(inp["b"])
    g = Guarded(x.shape, x.dtype)
    nv.nv_layer_norm(x, w, b, g.t, 1e-5)
    torch.cuda.synchronize()
    assert g.bands_intact()
    check_out(g.t, oracle.layer_norm(host(inp["x"]), host(inp["w"]), host(inp["b"]), 1e-5))


@pytest.mark.parametrize("dt", ["bf16", "f32"])
@pytest.mark.parametrize("plan", [dict(path=nv.PATH_GENERIC)] +
                         [dict(path=nv.PATH_ROWS, vec_per_thread=v) for v in (1, 2, 4, 8)] +
                         [dict(path=nv.PATH_ROWS, vec_per_thread=4, ctas_per_sm=2),
                          dict(path=nv.PATH_STAGED),
                          dict(path=nv.PATH_STAGED, vec_per_thread=2, rows_per_cta=3, ctas_per_sm=2),
                          dict(path=nv.PATH_STAGED, vec_per_thread=8, rows_per_cta=2, ctas_per_sm=3)],
                         ids=lambda p: "-".join(f"{k}{v}" for k, v in p.items()))
def test_layer_norm_every_variant(plan, dt):
    inp = synth.layer_norm_inputs(211, 4096, dt, seed=2)
    x = dev(inp["x"])
    y = torch.empty_like(x)
    try:
        nv.nv_layer_norm(x, dev(inp["w"]), dev(inp["b"]), y, 1e-5, plan=nv.Plan(**plan))
    except nv.NvError as e:
        assert e.status == nv.NV_ERR_UNSUPPORTED
        pytest.skip(str(e))
    torch.cuda.synchronize()
    assert nv.nv_fault_count() == 0
    check_out(y, oracle.layer_norm(host(inp["x"]), host(inp["w"]), host(inp["b"]), 1e-5))


@pytest.mark.parametrize("dt,mean,std", [("bf16", 0.5, 2.0), ("f32", 1e4, 1.0), ("bf16", 3000.0, 0.25)])
def test_layer_norm_staged_rows_and_means(dt, mean, std):
    for rows, D in ((1, 8192), (300, 8192), (1000, 1024)):
        x = synth.normal((rows, D), mean, std, 5, 0, dt)
        w = synth.uniform((D,), 0.5, 1.5, 5, 2, dt)
        b = synth.normal((D,), 0.0, 0.1, 5, 3, dt)
        y = torch.empty_like(x).cuda()
        nv.nv_layer_norm(x.cuda(), w.cuda(), b.cuda(), y, 1e-5, plan=nv.Plan(path=nv.PATH_STAGED))
        torch.cuda.synchronize()
        assert nv.nv_fault_count() == 0
        check_out(y, oracle.layer_norm(host(x), host(w), host(b), 1e-5))


@pytest.mark.parametrize("dt,mean,std", [("f32", 1e4, 1.0), ("f32", -3e5, 0.01), ("bf16", 3000.0, 40.0),
                                          ("bf16", 3000.0, 0.25), ("f32", 0.0, 1e-30)])
def test_layer_norm_mean_far_from_zero(dt, mean, std):
    """|mean| >> std takes the centred second pass of the statistics."""
    for D in (4096, 64):
        x = synth.normal((33, D), mean, std, 1, 0, dt)
        w = synth.uniform((D,), 0.5, 1.5, 1, 2, dt)
        b = synth.normal((D,), 0.0, 0.1, 1, 3, dt)
        y = nv.layer_norm(x.cuda(), w.cuda(), b.cuda(), eps=1e-5)
        torch.cuda.synchronize()
        check_out(y, oracle.layer_norm(host(x), host(w), host(b), 1e-5))


def test_layer_norm_in_place_and_large_mean():
    x = synth.normal((64, 4096), 300.0, 0.5, 0, 0, "bf16")   # |mean| >> std
    ref = oracle.layer_norm(host(x), None, None, 1e-5)
    xd = x.cuda()
    nv.nv_layer_norm(xd, None, None, xd, 1e-5)
    torch.cuda.synchronize()
    check_out(xd, ref)


SLOTS = [dict(path=nv.PATH_SLOTS), dict(path=nv.PATH_SLOTS, vec_per_thread=4),
         dict(path=nv.PATH_SLOTS, vec_per_thread=3), dict(path=nv.PATH_SLOTS, vec_per_thread=6),
         dict(path=nv.PATH_SLOTS, rows_per_cta=1), dict(path=nv.PATH_SLOTS, rows_per_cta=5),
         dict(path=nv.PATH_SLOTS, vec_per_thread=8, threads_per_row=64),
         dict(path=nv.PATH_SLOTS, stages=-1)]


@pytest.mark.parametrize("plan", SLOTS, ids=lambda p: "-".join(f"{k}{v}" for k, v in p.items()))
@pytest.mark.parametrize("rows,D,wb", [(147, 8192, (1, 1)), (149, 5120, (1, 0)), (33, 4096, (0, 0)),
                                        (5, 16384, (1, 1)), (64, 512, (1, 1)), (300, 256, (0, 1)),
                                        (1000, 2048, (1, 1)), (1, 8192, (1, 1)), (2, 8, (1, 1)),
                                        (77, 24576, (1, 1)), (500, 1024, (1, 1)),
                                        (129, 1536, (0, 1)), (311, 768, (1, 1)), (1001, 128, (1, 1)),
                                        (513, 384, (1, 1)), (65, 3072, (1, 1)),
                                        (999, 64, (1, 0)), (77, 32, (1, 1))])
def test_layer_norm_slots(rows, D, wb, plan):
    """The slots path (bfloat16): rows in registers, several per CTA sharing a float32 table
    of w and b, x consumed packed by bfloat16 -> double conversions and mixed-precision fma."""
    inp = synth.layer_norm_inputs(rows, D, "bf16", seed=D + 5 * rows, weight=bool(wb[0]),
                                  bias=bool(wb[1]))
    x, w, b = dev(inp["x"]), dev(inp["w"]), dev(inp["b"])
    g = Guarded(x.shape, x.dtype)
    try:
        nv.nv_layer_norm(x, w, b, g.t, 1e-5, plan=nv.Plan(**plan))
    except nv.NvError as e:
        assert e.status == nv.NV_ERR_UNSUPPORTED
        pytest.skip(str(e))
    torch.cuda.synchronize()
    assert g.bands_intact()
    check_out(g.t, oracle.layer_norm(host(inp["x"]), host(inp["w"]), host(inp["b"]), 1e-5))


@pytest.mark.parametrize("mean,std", [(3000.0, 40.0), (3000.0, 0.25), (0.5, 2.0), (-7.0e4, 3.0),
                                      (1.0, 1e-30)])
def test_layer_norm_slots_means_and_in_place(mean, std):
    """The slots path on rows whose mean is far from zero (centred second pass, two-step
    subtraction of the mean), near-constant rows, and in place (y == x)."""
    for rows, D in ((33, 4096), (300, 8192), (7, 64)):
        x = synth.normal((rows, D), mean, std, 6, 0, "bf16")
        w = synth.uniform((D,), 0.5, 1.5, 6, 2, "bf16")
        b = synth.normal((D,), 0.0, 0.1, 6, 3, "bf16")
        ref = oracle.layer_norm(host(x), host(w), host(b), 1e-5)
        xd = x.cuda()
        nv.nv_layer_norm(xd, w.cuda(), b.cuda(), xd, 1e-5, plan=nv.Plan(path=nv.PATH_SLOTS))
        torch.cuda.synchronize()
        check_out(xd, ref)


RING = [dict(path=nv.PATH_RING),
        dict(path=nv.PATH_RING, threads_per_row=32, rows_per_cta=4),
        dict(path=nv.PATH_RING, threads_per_row=64, rows_per_cta=3, stages=6),
        dict(path=nv.PATH_RING, threads_per_row=128, rows_per_cta=2, stages=4),
        dict(path=nv.PATH_RING, threads_per_row=96, rows_per_cta=1, stages=2, ctas_per_sm=2),
        dict(path=nv.PATH_RING, threads_per_row=32, rows_per_cta=5, stages=15),
        dict(path=nv.PATH_RING, threads_per_row=256, rows_per_cta=2)]


@pytest.mark.parametrize("dt", ["bf16", "f32"])
@pytest.mark.parametrize("plan", RING, ids=lambda p: "-".join(f"{k}{v}" for k, v in p.items()))
@pytest.mark.parametrize("rows,D,wb", [(147, 8192, (1, 1)), (149, 5120, (1, 0)), (33, 4096, (0, 0)),
                                        (5, 16384, (1, 1)), (64, 512, (1, 1)), (300, 256, (0, 1)),
                                        (1000, 2048, (1, 1)), (1, 8192, (1, 1)), (2, 8, (1, 1))])
def test_layer_norm_ring(rows, D, wb, plan, dt):
    """The ring path: row groups of a few warps fed by a ring of bulk-copied row buffers."""
    inp = synth.layer_norm_inputs(rows, D, dt, seed=D + 3 * rows, weight=bool(wb[0]),
                                  bias=bool(wb[1]))
    x, w, b = dev(inp["x"]), dev(inp["w"]), dev(inp["b"])
    g = Guarded(x.shape, x.dtype)
    try:
        nv.nv_layer_norm(x, w, b, g.t, 1e-5, plan=nv.Plan(**plan))
    except nv.NvError as e:
        assert e.status == nv.NV_ERR_UNSUPPORTED
        pytest.skip(str(e))
    torch.cuda.synchronize()
    assert nv.nv_fault_count() == 0
    assert g.bands_intact()
    check_out(g.t, oracle.layer_norm(host(inp["x"]), host(inp["w"]), host(inp["b"]), 1e-5))


@pytest.mark.parametrize("dt,mean,std", [("f32", 1e4, 1.0), ("f32", -3e5, 0.01), ("bf16", 3000.0, 40.0),
                                          ("bf16", 3000.0, 0.25), ("f32", 0.0, 1e-30),
                                          ("bf16", 0.5, 2.0)])
def test_layer_norm_ring_means_and_in_place(dt, mean, std):
    """The ring path on rows whose mean is far from zero (centred second pass, two-step
    subtraction of the mean) and in place (y == x)."""
    for rows, D in ((33, 4096), (300, 8192), (7, 64)):
        x = synth.normal((rows, D), mean, std, 4, 0, dt)
        w = synth.uniform((D,), 0.5, 1.5, 4, 2, dt)
        b = synth.normal((D,), 0.0, 0.1, 4, 3, dt)
        ref = oracle.layer_norm(host(x), host(w), host(b), 1e-5)
        xd = x.cuda()
        nv.nv_layer_norm(xd, w.cuda(), b.cuda(), xd, 1e-5, plan=nv.Plan(path=nv.PATH_RING))
        torch.cuda.synchronize()
        assert nv.nv_fault_count() == 0
        check_out(xd, ref)


# ---- norm_rope ---------------------------------------------------------------------------

ROPE_CASES = [
    # B, H, L, D, dims, traditional, offset, normalize, weight
    (2, 4, 64, 128, 128, 0, 0, 1, True),
    (2, 4, 64, 128, 128, 1, 4096, 1, True),
    (1, 3, 50, 128, 64, 0, 7, 1, True),
    (1, 3, 50, 128, 32, 1, 7, 1, True),
    (2, 2, 33, 64, 64, 0, 100000, 1, True),
    (1, 2, 40, 256, 256, 0, 5, 1, False),
    (1, 2, 40, 256, 128, 1, 5, 0, True),
    (3, 1, 17, 128, 128, 0, 0, 0, False),
    (1, 5, 9, 100, 50, 0, 3, 1, True),       # half = 25: generic path
    (1, 2, 12, 1000, 96, 1, 2, 1, True),     # D > 256: generic path
    (1, 1, 6, 6, 4, 0, 1, 1, True),
    (1, 600, 1, 128, 128, 0, 4095, 1, True),  # decode-like: one position, many rows
    (2, 3, 40, 96, 96, 0, 11, 1, True),      # two vectors per lane, lanes without a vector
    (2, 3, 40, 96, 96, 1, 11, 1, True),
    (1, 2, 30, 192, 192, 0, 5, 1, True),
]


@pytest.mark.parametrize("dt", ["bf16", "f32"])
@pytest.mark.parametrize("case", ROPE_CASES, ids=lambda c: "x".join(map(str, c)))
def test_norm_rope(case, dt):
    B, H, L, D, dims, trad, offset, normalize, weight = case
    inp = synth.norm_rope_inputs(B, H, L, D, dt, seed=L + D, weight=weight)
    x, w = dev(inp["x"]), dev(inp["w"])
    g = Guarded(x.shape, x.dtype)
    eps = 1e-6
    nv.nv_norm_rope(x, w, g.t, L, dims, trad, 10000.0, 1.0, offset, normalize, eps)
    torch.cuda.synchronize()
    assert g.bands_intact()
    ref = oracle.norm_rope(host(inp["x"]), host(inp["w"]), L, dims, trad, 10000.0, 1.0, offset,
                           normalize, eps)
    check_out(g.t, ref)


@pytest.mark.parametrize("trad", [0, 1])
def test_norm_rope_base_and_scale(trad):
    B, H, L, D = 1, 4, 32, 128
    inp = synth.norm_rope_inputs(B, H, L, D, "bf16", seed=9)
    x = dev(inp["x"])
    y = torch.empty_like(x)
    nv.nv_norm_rope(x, dev(inp["w"]), y, L, 128, trad, 500000.0, 0.125, 8192, 1, 1e-5)
    torch.cuda.synchronize()
    ref = oracle.norm_rope(host(inp["x"]), host(inp["w"]), L, 128, trad, 500000.0, 0.125, 8192, 1,
                           1e-5)
    check_out(y, ref)


@pytest.mark.parametrize("dt", ["bf16", "f32"])
@pytest.mark.parametrize("D", [128, 64, 256])
def test_norm_rope_every_variant(D, dt):
    """Generic path, one vector per lane, both halves per lane (halves, dims == D)."""
    inp = synth.norm_rope_inputs(2, 4, 64, D, dt, seed=1)
    x, w = dev(inp["x"]), dev(inp["w"])
    plans = [dict(path=nv.PATH_GENERIC), dict(path=nv.PATH_ROWS, vec_per_thread=1),
             dict(path=nv.PATH_ROWS, vec_per_thread=2), dict(path=nv.PATH_ROWS, rows_per_cta=3),
             dict(path=nv.PATH_ROWS, stages=6), dict(path=nv.PATH_ROWS, stages=4, rows_per_cta=40),
             dict(path=nv.PATH_ROWS, stages=-1), dict(path=nv.PATH_ROWS, stages=2)]
    for trad in (0, 1):
        ref = oracle.norm_rope(host(inp["x"]), host(inp["w"]), 64, D, trad, 10000.0, 1.0, 4096,
                               1, 1e-6)
        for p in plans:
            y = torch.empty_like(x)
            try:
                nv.nv_norm_rope(x, w, y, 64, D, trad, 10000.0, 1.0, 4096, 1, 1e-6,
                                plan=nv.Plan(**p))
            except nv.NvError as e:
                assert e.status == nv.NV_ERR_UNSUPPORTED
                continue
            torch.cuda.synchronize()
            check_out(y, ref, f"{p} trad={trad}")


@pytest.mark.parametrize("dt", ["bf16", "f32"])
@pytest.mark.parametrize("trad", [0, 1])
def test_norm_rope_near_cancellation(trad, dt):
    """Rows built so that many rotated outputs nearly cancel: every pair (p, q) of a row is
    a multiple of (cos phi, sin phi) of its own angle, so y_p = a_p cos - a_q sin is
    (nearly) zero before rounding: the error-free rotation must still meet the bar, on every
    kernel path."""
    B, H, L, D = 2, 8, 64, 128
    half = D // 2
    offset = 4096
    pos = offset + np.arange(L)[:, None]
    theta = 10000.0 ** (-2.0 * np.arange(half) / D)
    phi = pos * theta                                   # [L, half], double
    rng = np.random.default_rng(5)
    r = rng.uniform(0.5, 2.0, size=(B, H, L, half))
    # (x_p, x_q) = r (sin phi, cos phi) turns to (0, r): y_p cancels
    xp, xq = r * np.sin(phi), r * np.cos(phi)
    x = np.empty((B, H, L, D))
    if trad:
        x[..., 0::2], x[..., 1::2] = xp, xq
    else:
        x[..., :half], x[..., half:] = xp, xq
    tdt = torch.bfloat16 if dt == "bf16" else torch.float32
    xt = torch.from_numpy(x.reshape(-1, D)).to(tdt)
    w = torch.ones(D, dtype=tdt)
    ref = oracle.norm_rope(host(xt), host(w), L, D, trad, 10000.0, 1.0, offset, 1, 1e-6)
    for p in (None, dict(path=nv.PATH_ROWS, vec_per_thread=1), dict(path=nv.PATH_GENERIC),
              dict(path=nv.PATH_ROWS, stages=3), dict(path=nv.PATH_ROWS, stages=-1)):
        y = torch.empty_like(xt).cuda()
        nv.nv_norm_rope(xt.cuda(), w.cuda(), y, L, D, trad, 10000.0, 1.0, offset, 1, 1e-6,
                        plan=None if p is None else nv.Plan(**p))
        torch.cuda.synchronize()
        check_out(y, ref, f"near cancellation {p}")


@pytest.mark.parametrize("stages", [2, 3, 4, 6])
@pytest.mark.parametrize("case", [(3, 100, 9, 128, "bf16", 0), (3, 100, 9, 128, "bf16", 70),
                                  (2, 5, 30, 64, "bf16", 0), (2, 9, 20, 256, "bf16", 0),
                                  (3, 100, 9, 128, "f32", 0), (1, 600, 2, 128, "bf16", 96)],
                         ids=lambda c: "x".join(map(str, c)))
def test_norm_rope_async_rounds(case, stages):
    """Rows staged through the per-thread asynchronous-copy ring (stages = rounds in flight),
    ragged chunks (BH = 300 or 600 in chunks of 70 or 96) included, both pairings, in place
    too."""
    B, H, L, D, dt, bt = case
    inp = synth.norm_rope_inputs(B, H, L, D, dt, seed=L + D + stages)
    x, w = dev(inp["x"]), dev(inp["w"])
    for trad in (0, 1):
        ref = oracle.norm_rope(host(inp["x"]), host(inp["w"]), L, D, trad, 10000.0, 1.0, 2047, 1,
                               1e-6)
        plan = nv.Plan(path=nv.PATH_ROWS, stages=stages, rows_per_cta=bt)
        g = Guarded(x.shape, x.dtype)
        nv.nv_norm_rope(x, w, g.t, L, D, trad, 10000.0, 1.0, 2047, 1, 1e-6, plan=plan)
        torch.cuda.synchronize()
        assert g.bands_intact()
        check_out(g.t, ref, f"async rounds {case} stages={stages} trad={trad}")
        xi = x.clone()
        nv.nv_norm_rope(xi, w, xi, L, D, trad, 10000.0, 1.0, 2047, 1, 1e-6, plan=plan)
        torch.cuda.synchronize()
        check_out(xi, ref, f"async rounds in place {case} stages={stages} trad={trad}")


def test_norm_rope_async_rounds_rejects():
    x = torch.zeros(2 * 4 * 16, 128, dtype=torch.bfloat16, device="cuda")
    w = torch.ones(128, dtype=torch.bfloat16, device="cuda")
    for p, dims in ((dict(path=nv.PATH_ROWS, stages=7), 128),
                    (dict(path=nv.PATH_ROWS, stages=1), 128),
                    (dict(path=nv.PATH_ROWS, stages=-2), 128),
                    (dict(path=nv.PATH_ROWS, stages=4, vec_per_thread=1), 128),
                    (dict(path=nv.PATH_ROWS, stages=4), 24),
                    (dict(path=nv.PATH_ROWS, stages=4), 40),
                    (dict(path=nv.PATH_GENERIC, stages=4), 128)):
        with pytest.raises(nv.NvError) as e:
            nv.nv_norm_rope(x, w, x, 16, dims, 0, 10000.0, 1.0, 0, 1, 1e-6, plan=nv.Plan(**p))
        assert e.value.status == nv.NV_ERR_UNSUPPORTED, p


def _partial_pairs_ok(D, dims, trad, dt):
    """Whether the two-vectors-per-lane kernels take rotary dims < D: the rotated features
    fill an even number of whole 16-byte vectors (halves: dims / 2 of them on each side) and
    a row is 4, 8 or 16 lanes of two vectors."""
    vec = 8 if dt == "bf16" else 4
    whole = dims % (2 * vec) == 0 if trad else (dims // 2) % vec == 0
    return whole and (D // vec) // 2 in (4, 8, 16)


@pytest.mark.parametrize("dt", ["bf16", "f32"])
@pytest.mark.parametrize("D,dims_list", [(128, (16, 32, 48, 64, 96, 112, 120)),
                                         (64, (16, 32, 48, 8)), (256, (32, 64, 128, 192, 240))],
                         ids=lambda v: str(v) if isinstance(v, int) else "-".join(map(str, v)))
def test_norm_rope_partial_rotary_pairs(D, dims_list, dt):
    """Rotary dims < D through the two-vectors-per-lane kernels (register and ring forms):
    the rotated lanes hold partner vectors, the others the features past dims, which are
    only normalised and weighted.  Ragged chunks of rows, without weights, without
    normalisation, and in place too; a plan the shape cannot take is refused."""
    B, H, L = 2, 5, 21
    inp = synth.norm_rope_inputs(B, H, L, D, dt, seed=D + 17)
    x, w = dev(inp["x"]), dev(inp["w"])
    plans = [None, dict(path=nv.PATH_ROWS, stages=-1), dict(path=nv.PATH_ROWS, stages=2),
             dict(path=nv.PATH_ROWS, stages=4, rows_per_cta=7),
             dict(path=nv.PATH_ROWS, stages=-1, rows_per_cta=3),
             dict(path=nv.PATH_ROWS, vec_per_thread=1)]
    for dims in dims_list:
        for trad in (0, 1):
            ok = _partial_pairs_ok(D, dims, trad, dt)
            for normalize, wt in ((1, w), (0, w), (1, None)):
                wh = host(inp["w"]) if wt is not None else None
                ref = oracle.norm_rope(host(inp["x"]), wh, L, dims, trad, 10000.0, 1.0, 300,
                                       normalize, 1e-6)
                for p in plans:
                    tag = f"D={D} dims={dims} trad={trad} norm={normalize} w={wt is not None} {p}"
                    g = Guarded(x.shape, x.dtype)
                    # where the pairs kernels take the shape no plan is refused; where they
                    # do not, every ring plan is
                    ring = p is not None and p.get("stages", 0) >= 2
                    try:
                        nv.nv_norm_rope(x, wt, g.t, L, dims, trad, 10000.0, 1.0, 300, normalize,
                                        1e-6, plan=None if p is None else nv.Plan(**p))
                    except nv.NvError as e:
                        assert e.status == nv.NV_ERR_UNSUPPORTED, tag
                        assert not ok, tag
                        continue
                    assert ok or not ring, tag
                    torch.cuda.synchronize()
                    assert g.bands_intact(), tag
                    check_out(g.t, ref, tag)
            if ok:
                xi = x.clone()
                nv.nv_norm_rope(xi, w, xi, L, dims, trad, 10000.0, 1.0, 300, 1, 1e-6,
                                plan=nv.Plan(path=nv.PATH_ROWS, stages=3))
                torch.cuda.synchronize()
                ref = oracle.norm_rope(host(inp["x"]), host(inp["w"]), L, dims, trad, 10000.0,
                                       1.0, 300, 1, 1e-6)
                check_out(xi, ref, f"in place D={D} dims={dims} trad={trad}")


@pytest.mark.parametrize("dims", [32, 64, 96])
def test_norm_rope_partial_rotary_non_finite(dims):
    """A non-finite input stays in its row, and a lane past dims keeps exactly x w (times the
    row's 1/rms) whatever its partner vector holds: with normalize an Inf anywhere in a row
    makes its 1/rms zero, so the oracle's row is NaN at the Inf and its pair partner and
    zero elsewhere; without normalize an Inf past dims passes through as Inf and leaves every
    other element of its row alone.  Every kernel form, both ways of running the lanes past
    dims (dims 32: branched, 64 and 96: one instruction stream)."""
    B, H, L, D = 1, 4, 12, 128
    inp = synth.norm_rope_inputs(B, H, L, D, "bf16", seed=dims)
    xh = inp["x"].clone()
    rows = xh.shape[0]
    xh[3, D - 5] = float("inf")                # past dims, normalize and plain
    xh[7, dims + 1] = -float("inf")
    xh[20, 1] = float("inf")                   # rotated: normalize only
    w = dev(inp["w"])
    plans = [None, dict(path=nv.PATH_ROWS, stages=2), dict(path=nv.PATH_ROWS, stages=-1),
             dict(path=nv.PATH_ROWS, vec_per_thread=1), dict(path=nv.PATH_GENERIC)]
    for normalize in (1, 0):
        xn = xh.clone()
        if not normalize:
            xn[20, 1] = 0.0
        ref = oracle.norm_rope(host(xn), host(inp["w"]), L, dims, 0, 10000.0, 1.0, 5, normalize,
                               1e-6)
        x = dev(xn)
        for p in plans:
            y = torch.empty_like(x)
            nv.nv_norm_rope(x, w, y, L, dims, 0, 10000.0, 1.0, 5, normalize, 1e-6,
                            plan=None if p is None else nv.Plan(**p))
            torch.cuda.synchronize()
            check_out(y, ref, f"dims={dims} normalize={normalize} {p}")
        assert rows == B * H * L


def test_norm_rope_in_place():
    inp = synth.norm_rope_inputs(2, 4, 16, 128, "bf16", seed=4)
    ref = oracle.norm_rope(host(inp["x"]), host(inp["w"]), 16, 128, 1, 10000.0, 1.0, 4096, 1, 1e-6)
    x = dev(inp["x"])
    nv.nv_norm_rope(x, dev(inp["w"]), x, 16, 128, 1, 10000.0, 1.0, 4096, 1, 1e-6)
    torch.cuda.synchronize()
    check_out(x, ref)


# ---- all-reduce of partial sums + add_rms_norm --------------------------------------------

ALLREDUCE_CASES = [(257, 4096, 4, "bf16"), (100, 1024, 2, "f32"), (33, 8192, 8, "bf16"),
                   (17, 100, 3, "bf16"), (5, 16384, 2, "bf16"), (1, 512, 1, "f32"),
                   (64, 4096, 8, "f32"), (40, 12288, 3, "bf16")]


@pytest.mark.parametrize("rows,D,nparts,dt", ALLREDUCE_CASES, ids=lambda v: str(v))
def test_allreduce_add_rms_norm(rows, D, nparts, dt):
    inp = synth.allreduce_inputs(rows, D, nparts, dt, seed=rows + nparts)
    parts = [dev(p) for p in inp["parts"]]
    r, w = dev(inp["r"]), dev(inp["w"])
    gy, gh, gx = (Guarded(r.shape, r.dtype) for _ in range(3))
    nv.nv_allreduce_add_rms_norm(parts, r, w, gy.t, gh.t, 1e-5, x_out=gx.t)
    torch.cuda.synchronize()
    assert gy.bands_intact() and gh.bands_intact() and gx.bands_intact()
    y, h, x = oracle.allreduce_add_rms_norm([host(p) for p in inp["parts"]], host(inp["r"]),
                                            host(inp["w"]), 1e-5)
    check_exact(gx.t, x, "x")
    check_exact(gh.t, h, "h")
    check_out(gy.t, y, "y")


def test_peer_allreduce_one_rank_and_a_flag_that_never_comes():
    """The one-shot form on one GPU (a world of one rank, where nothing waits on another
    kernel): three steps through PeerAllReduce (publish, flag wait, slots alternating), each
    matching the oracle; then a call whose epoch no rank ever publishes -- its bounded waits
    run out (about a second), every CTA counts a fault and leaves its rows unwritten, and the
    next step runs normally on the same context."""
    import socket
    import torch.distributed as dist
    from rope_add_rms_b200 import tp
    sock = socket.socket()
    sock.bind(("127.0.0.1", 0))
    port = sock.getsockname()[1]
    sock.close()
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1)
    try:
        rows, D = 300, 4096
        par = tp.PeerAllReduce((rows, D), torch.bfloat16)
        nv.nv_fault_count(reset=True)

        def step(seed):
            inp = synth.allreduce_inputs(rows, D, 1, "bf16", seed=seed)
            par.partial().copy_(dev(inp["parts"][0]))
            y, h = par(dev(inp["r"]), dev(inp["w"]), 1e-5)
            torch.cuda.synchronize()
            y_ref, h_ref, _ = oracle.allreduce_add_rms_norm([host(inp["parts"][0])],
                                                            host(inp["r"]), host(inp["w"]), 1e-5)
            check_exact(h, h_ref, f"h, step {seed}")
            check_out(y, y_ref, f"y, step {seed}")

        for seed in range(3):
            step(seed)
        assert par.epoch == 3 and nv.nv_fault_count() == 0
        r = torch.zeros(4, D, dtype=torch.bfloat16, device="cuda")
        y = torch.full_like(r, 7.0)
        h = torch.full_like(r, 7.0)
        nv.nv_allreduce_add_rms_norm_peers([par.buf_ptrs[0]], r, None, y, h, 1e-5, par.flags,
                                           par.epoch + 5)
        torch.cuda.synchronize()
        assert nv.nv_fault_count(reset=True) == 4, "one fault per CTA (one CTA per row)"
        assert (y == 7).all() and (h == 7).all(), "rows of a CTA that gave up stay unwritten"
        step(3)
        assert nv.nv_fault_count() == 0
        par.close()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_peer_allreduce_emulated_ranks_on_one_gpu(world):
    """The one-shot form with `world` ranks emulated in one process on one GPU: each rank's
    buffer (two partial slots, then its flag array) is local memory, so every part pointer is
    an ordinary device address.  Per step, every rank publishes the step's epoch into every
    rank's flag array first, and only then does each rank's reduce run, so every flag it
    checks is already set and no kernel waits on another.  The slot of the other parity
    holds NaNs: a reduce that read it would show.  All ranks get the oracle's y and h
    bit-identically."""
    rows, D = 257, 4096
    esz = 2
    slot = rows * D * esz
    flags_off = (2 * slot + 255) // 256 * 256
    raws = [torch.zeros(flags_off + 8 * world, dtype=torch.uint8, device="cuda")
            for _ in range(world)]
    bufs = [r[:2 * slot].view(torch.bfloat16).view(2, rows, D) for r in raws]
    flags = [r[flags_off:].view(torch.int64) for r in raws]
    flag_ptrs = [f.data_ptr() for f in flags]
    nv.nv_fault_count(reset=True)
    for epoch in (1, 2, 3):
        inp = synth.allreduce_inputs(rows, D, world, "bf16", seed=40 + epoch)
        for k in range(world):
            bufs[k][epoch & 1].copy_(dev(inp["parts"][k]))
            bufs[k][(epoch + 1) & 1].fill_(float("nan"))
        for k in range(world):
            nv.nv_tp_publish(flag_ptrs, k, epoch)
        parts = [bufs[k][epoch & 1].data_ptr() for k in range(world)]
        r, w = dev(inp["r"]), dev(inp["w"])
        outs = []
        for k in range(world):
            y, h = torch.empty_like(r), torch.empty_like(r)
            nv.nv_allreduce_add_rms_norm_peers(parts, r, w, y, h, 1e-5, flags[k], epoch)
            outs.append((y, h))
        torch.cuda.synchronize()
        for k in range(world):
            assert (flags[k].cpu() == epoch).all(), f"rank {k}'s flags after epoch {epoch}"
        y_ref, h_ref, _ = oracle.allreduce_add_rms_norm([host(p) for p in inp["parts"]],
                                                        host(inp["r"]), host(inp["w"]), 1e-5)
        check_exact(outs[0][1], h_ref, f"h, epoch {epoch}")
        check_out(outs[0][0], y_ref, f"y, epoch {epoch}")
        for k in range(1, world):
            assert torch.equal(outs[k][0].view(torch.int16), outs[0][0].view(torch.int16))
            assert torch.equal(outs[k][1].view(torch.int16), outs[0][1].view(torch.int16))
    assert nv.nv_fault_count() == 0


def test_allreduce_in_place_ranks_agree_and_errors():
    rows, D, n = 300, 4096, 4
    inp = synth.allreduce_inputs(rows, D, n, "bf16", seed=77)
    y_ref, h_ref, x_ref = oracle.allreduce_add_rms_norm([host(p) for p in inp["parts"]],
                                                        host(inp["r"]), host(inp["w"]), 1e-5)
    w = dev(inp["w"])
    # every rank passes the parts in the same (rank) order, so every rank computes the
    # same bits -- emulated here by repeated calls on fresh copies
    outs = []
    for _ in range(2):
        parts = [dev(p) for p in inp["parts"]]
        r = dev(inp["r"])
        y = torch.empty_like(r)
        nv.nv_allreduce_add_rms_norm(parts, r, w, y, r, 1e-5, x_out=parts[0])  # h over r, x over part 0
        torch.cuda.synchronize()
        check_exact(r, h_ref, "h in place")
        check_exact(parts[0], x_ref, "x in place")
        check_out(y, y_ref, "y")
        outs.append(y)
    assert torch.equal(outs[0].view(torch.int16), outs[1].view(torch.int16))
    parts = [dev(p) for p in inp["parts"]]
    r = dev(inp["r"])
    with pytest.raises(nv.NvError, match="overlaps parts"):
        nv.nv_allreduce_add_rms_norm(parts, r, w, parts[1], torch.empty_like(r), 1e-5)
    with pytest.raises(nv.NvError, match="past the end"):
        short = torch.empty(10, D, dtype=r.dtype, device="cuda")   # its own small allocation
        nv.nv_allreduce_add_rms_norm([parts[0], short], r, w, torch.empty_like(r),
                                     torch.empty_like(r), 1e-5)


# ---- CUDA graphs ------------------------------------------------------------------------------

def test_cuda_graph_capture_and_replay():
    """A chain of the ops (with programmatic dependent launch) captured into one CUDA graph
    and replayed on new inputs gives the same bits as running the calls directly."""
    B, H, L, D = 2, 8, 64, 128
    rows = B * H * L
    inp = synth.add_rms_inputs(rows, D, "bf16", seed=23)
    x, r, w = dev(inp["x"]), dev(inp["r"]), dev(inp["w"])
    y, h, z, q = (torch.empty_like(x) for _ in range(4))
    parts = [dev(inp["x"]), dev(inp["r"])]
    a_y, a_h = torch.empty_like(x), torch.empty_like(x)

    def chain():
        nv.nv_add_rms_norm(x, r, w, y, h, 1e-5)
        nv.nv_layer_norm(y, w, None, z, 1e-5)
        nv.nv_norm_rope(z, w, q, L, D, 0, 10000.0, 1.0, 4096, 1, 1e-6)
        nv.nv_allreduce_add_rms_norm(parts, q, w, a_y, a_h, 1e-5)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        chain()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        chain()
    new = synth.add_rms_inputs(rows, D, "bf16", seed=24)
    x.copy_(dev(new["x"]))
    r.copy_(dev(new["r"]))
    graph.replay()
    torch.cuda.synchronize()
    got = [t.clone() for t in (y, h, z, q, a_y, a_h)]
    chain()
    torch.cuda.synchronize()
    for name, gt, et in zip("y h z q a_y a_h".split(), got, (y, h, z, q, a_y, a_h)):
        assert torch.equal(gt.view(torch.int16), et.view(torch.int16)), f"{name} differs"
    ref, href = oracle.add_rms_norm(host(new["x"]), host(new["r"]), host(inp["w"]), 1e-5)
    check_exact(got[1], href, "h from the graph")
    check_out(got[0], ref, "y from the graph")
    del graph


# ---- host-resident rows --------------------------------------------------------------------

@pytest.mark.parametrize("dt", ["bf16", "f32"])
@pytest.mark.parametrize("rows,D,chunk", [(3000, 4096, 0), (1000, 1024, 333), (7, 512, 1),
                                          (513, 2048, 1000), (64, 100, 10)])
def test_add_rms_norm_host(rows, D, chunk, dt):
    """Copies in, compute and copies out pipelined over row chunks: bit-identical to the
    device call, and the device staging buffers end up holding inputs and outputs."""
    inp = synth.add_rms_inputs(rows, D, dt, seed=rows + chunk)
    xh, rh = inp["x"].pin_memory(), inp["r"].pin_memory()
    w = dev(inp["w"])
    yh, hh = torch.empty_like(xh).pin_memory(), torch.empty_like(xh).pin_memory()
    xd, rd, yd, hd = (torch.empty(rows, D, dtype=xh.dtype, device="cuda") for _ in range(4))
    nv.nv_add_rms_norm_host(xh, rh, w, yh, hh, xd, rd, yd, hd, 1e-5, chunk_rows=chunk)
    torch.cuda.synchronize()
    y_ref, h_ref = torch.empty_like(xd), torch.empty_like(xd)
    nv.nv_add_rms_norm(dev(inp["x"]), dev(inp["r"]), w, y_ref, h_ref, 1e-5)
    torch.cuda.synchronize()
    bits = torch.int16 if dt == "bf16" else torch.int32
    assert torch.equal(yh.view(bits), y_ref.cpu().view(bits))
    assert torch.equal(hh.view(bits), h_ref.cpu().view(bits))
    assert torch.equal(yd.view(bits), y_ref.view(bits))
    ref, href = oracle.add_rms_norm(host(inp["x"]), host(inp["r"]), host(inp["w"]), 1e-5)
    check_exact(hh, href, "h")
    check_out(yh, ref, "y")


def test_add_rms_norm_host_in_place_and_errors():
    rows, D = 2048, 4096
    inp = synth.add_rms_inputs(rows, D, "bf16", seed=5)
    xh, rh = inp["x"].clone().pin_memory(), inp["r"].clone().pin_memory()
    w = dev(inp["w"])
    xd, rd = (torch.empty(rows, D, dtype=xh.dtype, device="cuda") for _ in range(2))
    nv.nv_add_rms_norm_host(xh, rh, w, xh, rh, xd, rd, xd, rd, 1e-5)   # y over x, h over r
    torch.cuda.synchronize()
    ref, href = oracle.add_rms_norm(host(inp["x"]), host(inp["r"]), host(inp["w"]), 1e-5)
    check_exact(rh, href, "h in place")
    check_out(xh, ref, "y in place")
    pageable = inp["x"].clone()
    with pytest.raises(nv.NvError, match="page-locked"):
        nv.nv_add_rms_norm_host(pageable, rh, w, xh, rh, xd, rd, xd, rd, 1e-5)
    other = torch.empty_like(xh).pin_memory()
    with pytest.raises(nv.NvError, match="overlaps"):
        nv.nv_add_rms_norm_host(xh, rh, w, other, xh, xd, rd, xd, rd, 1e-5)   # h over x
    with pytest.raises(nv.NvError, match="past the end"):
        small = torch.empty(100, D, dtype=xh.dtype, device="cuda")
        nv.nv_add_rms_norm_host(xh, rh, w, xh, rh, small, rd, small, rd, 1e-5)


# ---- programmatic dependent launch ---------------------------------------------------------

@pytest.mark.parametrize("launch", [nv.LAUNCH_DEFAULT, nv.LAUNCH_PLAIN])
@pytest.mark.parametrize("path", [nv.PATH_ROWS, nv.PATH_STAGED, nv.PATH_GENERIC])
def test_dependent_chain(path, launch):
    """Each call reads the previous call's outputs, launched back to back; every step
    must match the oracle applied to that step's own (device-produced) inputs."""
    rows, D, steps = 1024, 4096, 6
    inp = synth.add_rms_inputs(rows, D, "bf16", seed=21)
    x, r, w = dev(inp["x"]), dev(inp["r"]), dev(inp["w"])
    plan = nv.Plan(path=path, launch=launch)
    hist = [(x, r)]
    for _ in range(steps):
        y, h = torch.empty_like(x), torch.empty_like(x)
        nv.nv_add_rms_norm(x, r, w, y, h, 1e-5, plan=plan)
        x, r = y, h
        hist.append((x, r))
    torch.cuda.synchronize()
    assert nv.nv_fault_count() == 0
    for i in range(steps):
        (xi, ri), (yo, ho) = hist[i], hist[i + 1]
        ref, href = oracle.add_rms_norm(to_host_bits(xi), to_host_bits(ri), host(inp["w"]), 1e-5)
        check_exact(ho, href, f"h of step {i}")
        check_out(yo, ref, f"y of step {i}")


def test_dependent_chain_across_ops_in_place():
    """add_rms_norm -> layer_norm -> norm_rope -> rms_norm, each in place on the previous
    output, all launched back to back with programmatic dependent launch."""
    B, H, L, D = 2, 8, 64, 128
    rows = B * H * L
    inp = synth.add_rms_inputs(rows, D, "bf16", seed=22)
    x, r, w = dev(inp["x"]), dev(inp["r"]), dev(inp["w"])
    x0, r0 = to_host_bits(x), to_host_bits(r)
    y = torch.empty_like(x)
    nv.nv_add_rms_norm(x, r, w, y, r, 1e-5)               # h in place over r
    nv.nv_layer_norm(y, w, None, y, 1e-5)                  # in place
    nv.nv_norm_rope(y, w, y, L, D, 0, 10000.0, 1.0, 4096, 1, 1e-6)   # in place
    nv.nv_rms_norm(y, None, y, 1e-6)                       # in place
    torch.cuda.synchronize()
    # replay on the oracle, feeding each stage the bf16 values the GPU stage produced:
    # re-run the chain stage by stage on the device without overlap to get them
    a = dev(inp["x"]).clone()
    rr = dev(inp["r"]).clone()
    stages = []
    plain = nv.Plan(launch=nv.LAUNCH_PLAIN)
    s1 = torch.empty_like(a)
    nv.nv_add_rms_norm(a, rr, w, s1, rr, 1e-5, plan=plain); torch.cuda.synchronize()
    stages.append(s1.clone())
    nv.nv_layer_norm(s1, w, None, s1, 1e-5, plan=plain); torch.cuda.synchronize()
    stages.append(s1.clone())
    nv.nv_norm_rope(s1, w, s1, L, D, 0, 10000.0, 1.0, 4096, 1, 1e-6, plan=plain)
    torch.cuda.synchronize()
    stages.append(s1.clone())
    nv.nv_rms_norm(s1, None, s1, 1e-6, plan=plain); torch.cuda.synchronize()
    stages.append(s1.clone())
    assert torch.equal(y.view(torch.int16), stages[-1].view(torch.int16)), \
        "back-to-back launches changed the result"
    wh = host(inp["w"])
    ref1, _ = oracle.add_rms_norm(x0, r0, wh, 1e-5)
    check_out(stages[0], ref1, "add_rms_norm")
    check_out(stages[1], oracle.layer_norm(to_host_bits(stages[0]), wh, None, 1e-5), "layer_norm")
    check_out(stages[2], oracle.norm_rope(to_host_bits(stages[1]), wh, L, D, 0, 10000.0, 1.0, 4096,
                                          1, 1e-6), "norm_rope")
    check_out(stages[3], oracle.rms_norm(to_host_bits(stages[2]), None, 1e-6), "rms_norm")


# ---- general rope: cache form, explicit frequencies, inverse ----------------------------------

ROPE_PLANS = [None, dict(path=nv.PATH_GENERIC), dict(path=nv.PATH_ROWS, vec_per_thread=1),
              dict(path=nv.PATH_ROWS, vec_per_thread=2),
              dict(path=nv.PATH_ROWS, vec_per_thread=2, stages=4),
              dict(path=nv.PATH_ROWS, vec_per_thread=2, stages=-1)]


@pytest.mark.parametrize("dt", ["bf16", "f32"])
@pytest.mark.parametrize("trad", [0, 1])
@pytest.mark.parametrize("plan", ROPE_PLANS, ids=lambda p: "auto" if p is None else
                         "-".join(f"{k}{v}" for k, v in p.items()))
def test_norm_rope_into_cache(plan, trad, dt):
    """Row (b, h, l) lands in cache row (b, h, offset + l); every other row is untouched."""
    B, H, L, D, Lc, off = 2, 3, 16, 128, 50, 20
    inp = synth.norm_rope_inputs(B, H, L, D, dt, seed=31)
    x, w = dev(inp["x"]), dev(inp["w"])
    cache = torch.full((B * H * Lc, D), 7.25, dtype=x.dtype, device="cuda")
    try:
        nv.nv_rope(x, w, cache, L, D, trad, 10000.0, 1.0, off, 1, 1e-6, y_len=Lc,
                   plan=None if plan is None else nv.Plan(**plan))
    except nv.NvError as e:
        assert e.status == nv.NV_ERR_UNSUPPORTED
        pytest.skip(str(e))
    torch.cuda.synchronize()
    ref = np.full((B * H * Lc, D), 7.25)
    oracle.rope_ex(host(inp["x"]), host(inp["w"]), L, D, trad, 10000.0, 1.0, off, 1, 1e-6,
                   y=ref, y_len=Lc)
    inside = np.zeros(B * H * Lc, bool)
    for bh in range(B * H):
        inside[bh * Lc + off: bh * Lc + off + L] = True
    got = cache.float().cpu().numpy()
    assert (got[~inside] == 7.25).all(), "a cache row outside [offset, offset + L) changed"
    check_out(cache[torch.as_tensor(inside, device="cuda")], ref[inside])


@pytest.mark.parametrize("dt", ["bf16", "f32"])
@pytest.mark.parametrize("trad", [0, 1])
@pytest.mark.parametrize("plan", ROPE_PLANS, ids=lambda p: "auto" if p is None else
                         "-".join(f"{k}{v}" for k, v in p.items()))
def test_rope_freqs_and_inverse(plan, trad, dt):
    B, H, L, D = 2, 4, 32, 128
    inp = synth.norm_rope_inputs(B, H, L, D, dt, seed=32)
    x, w = dev(inp["x"]), dev(inp["w"])
    freqs = synth.uniform((D // 2,), 0.0, 0.5, 32, 5, "f32")
    p = None if plan is None else nv.Plan(**plan)
    for normalize in (0, 1):
        for forward in (True, False):
            for f in (None, freqs):
                y = torch.empty_like(x)
                try:
                    nv.nv_rope(x, w, y, L, D, trad, 500.0, 0.75, 4095, normalize, 1e-6,
                               freqs=None if f is None else f.cuda(), forward=forward, plan=p)
                except nv.NvError as e:
                    assert e.status == nv.NV_ERR_UNSUPPORTED
                    pytest.skip(str(e))
                torch.cuda.synchronize()
                ref = oracle.rope_ex(host(inp["x"]), host(inp["w"]), L, D, trad, 500.0, 0.75,
                                     4095, normalize, 1e-6, forward=forward,
                                     freqs=None if f is None else f.numpy().astype(np.float64))
                check_out(y, ref, f"normalize={normalize} forward={forward} freqs={f is not None}")


@pytest.mark.parametrize("trad", [0, 1])
@pytest.mark.parametrize("dt", ["bf16", "f32"])
def test_rope_llama3_scaled_frequencies(trad, dt):
    """NormRope with the Llama 3 scaled frequencies at positions past the original context."""
    B, H, L, D = 2, 4, 64, 128
    inp = synth.norm_rope_inputs(B, H, L, D, dt, seed=41)
    x, w = dev(inp["x"]), dev(inp["w"])
    freqs = nv.rope_llama3_freqs(D, 500000.0, 32.0, 1.0, 4.0, 8192)
    for offset in (0, 20000):
        y = torch.empty_like(x)
        nv.nv_rope(x, w, y, L, D, trad, 500000.0, 1.0, offset, 1, 1e-5, freqs=freqs.cuda())
        torch.cuda.synchronize()
        ref = oracle.rope_ex(host(inp["x"]), host(inp["w"]), L, D, trad, 500000.0, 1.0, offset, 1,
                             1e-5, freqs=freqs.numpy().astype(np.float64))
        check_out(y, ref, f"offset {offset}")


@pytest.mark.parametrize("trad", [0, 1])
def test_rope_yarn_scaled_frequencies(trad):
    """NormRope with YaRN frequencies (factor 8 over an original context of 4096) at
    positions past that context."""
    B, H, L, D = 2, 4, 64, 128
    inp = synth.norm_rope_inputs(B, H, L, D, "bf16", seed=47)
    x, w = dev(inp["x"]), dev(inp["w"])
    freqs, _ = nv.rope_yarn_freqs(D, 10000.0, 8.0, 4096, 1.0, 32.0)
    for offset in (0, 30000):
        y = torch.empty_like(x)
        nv.nv_rope(x, w, y, L, D, trad, 10000.0, 1.0, offset, 1, 1e-6, freqs=freqs.cuda())
        torch.cuda.synchronize()
        ref = oracle.rope_ex(host(inp["x"]), host(inp["w"]), L, D, trad, 10000.0, 1.0, offset, 1,
                             1e-6, freqs=freqs.numpy().astype(np.float64))
        check_out(y, ref, f"offset {offset}")


@pytest.mark.parametrize("dt", ["bf16", "f32"])
@pytest.mark.parametrize("trad", [0, 1])
def test_rope_suscaled_frequencies(trad, dt):
    """NormRope with SuScaled (LongRoPE) frequencies: the short factors within the original
    context of 4096, the long ones past it (positions up to ~100000)."""
    B, H, L, D = 2, 4, 64, 128
    inp = synth.norm_rope_inputs(B, H, L, D, dt, seed=53)
    x, w = dev(inp["x"]), dev(inp["w"])
    rng = np.random.default_rng(53)
    short, long_ = rng.uniform(1.0, 1.2, D // 2), rng.uniform(1.0, 60.0, D // 2)
    for offset in (0, 100000):
        freqs, m = nv.rope_suscaled_freqs(D, short, long_, offset + L, 10000.0, 131072, 4096)
        assert m > 1.0
        y = torch.empty_like(x)
        nv.nv_rope(x, w, y, L, D, trad, 10000.0, 1.0, offset, 1, 1e-6, freqs=freqs.cuda())
        torch.cuda.synchronize()
        ref = oracle.rope_ex(host(inp["x"]), host(inp["w"]), L, D, trad, 10000.0, 1.0, offset, 1,
                             1e-6, freqs=freqs.numpy().astype(np.float64))
        check_out(y, ref, f"offset {offset}")


def test_rope_round_trip_and_cache_rules():
    B, H, L, D = 1, 2, 8, 64
    x = synth.normal((B * H * L, D), 0.0, 1.0, 33, 0, "f32").cuda()
    y = nv.rope(x.view(B, H, L, D), offset=100).view(-1, D)
    back = nv.rope(y.view(B, H, L, D), offset=100, forward=False).view(-1, D)
    torch.cuda.synchronize()
    assert torch.allclose(back, x, rtol=1e-5, atol=1e-5)
    cache = torch.zeros(B * H * 20, D, device="cuda")
    with pytest.raises(nv.NvError, match="cache length"):
        nv.nv_rope(x, None, cache, L, D, 0, 10000.0, 1.0, 15, 0, 0.0, y_len=20)
    big = torch.zeros(B * H * L * D + B * H * 20 * D, device="cuda")
    xs = big[:B * H * L * D].view(-1, D)
    with pytest.raises(nv.NvError, match="overlaps"):
        nv.nv_rope(xs, None, big[B * H * L * D // 2:][:B * H * 20 * D].view(-1, D), L, D, 0,
                   10000.0, 1.0, 0, 0, 0.0, y_len=20)


# ---- gradients -----------------------------------------------------------------------------

from checks import check_grad  # noqa: E402

VJP_SHAPES = [(256, 4096), (1000, 2048), (33, 8192), (1, 512), (2000, 1024), (7, 16384)]


@pytest.mark.parametrize("dt", ["bf16", "f32"])
@pytest.mark.parametrize("weight", [True, False])
@pytest.mark.parametrize("rows,D", VJP_SHAPES)
def test_rms_norm_vjp(rows, D, weight, dt):
    inp = synth.rms_inputs(rows, D, dt, seed=rows + D, weight=weight)
    g = synth.normal((rows, D), 0.0, 1.0, rows + D, 4, dt)
    x, w, gd = dev(inp["x"]), dev(inp["w"]), dev(g)
    dx, dw = nv.rms_norm_vjp(x, w, gd, eps=1e-5)
    torch.cuda.synchronize()
    ref_dx, ref_dw, mag_dx, mag_dw = oracle.rms_norm_vjp(host(inp["x"]), host(inp["w"]), host(g),
                                                         1e-5)
    check_grad(dx, ref_dx, mag_dx, "dx")
    if weight:
        check_grad(dw, ref_dw, mag_dw, "dw")
    else:
        assert dw is None


@pytest.mark.parametrize("dt", ["bf16", "f32"])
@pytest.mark.parametrize("rows,D", [(1, 8), (7, 16), (1237, 64), (2049, 128), (333, 256), (517, 512),
                                    (64, 24), (4099, 128), (3, 200)])
def test_vjp_rows_of_at_most_64_vectors(rows, D, dt):
    """Rows of at most 64 vectors: row groups of G threads, several to a CTA, each walking its
    own rows and reducing over its own lanes, their column partial sums added in shared
    memory in group order.  Ragged row counts (groups of one warp running out of rows at
    different times), with and without w, both gradients, against the oracle; dw and db
    the same on a second call (the order of their sums is fixed)."""
    for weight in (True, False):
        inp = synth.layer_norm_inputs(rows, D, dt, seed=rows + 7 * D, weight=weight, bias=False)
        g = synth.normal((rows, D), 0.0, 1.0, rows + 7 * D, 4, dt)
        x, w, gd = dev(inp["x"]), dev(inp["w"]), dev(g)
        dx, dw = nv.rms_norm_vjp(x, w, gd, eps=1e-5)
        torch.cuda.synchronize()
        ref_dx, ref_dw, mag_dx, mag_dw = oracle.rms_norm_vjp(host(inp["x"]), host(inp["w"]),
                                                             host(g), 1e-5)
        check_grad(dx, ref_dx, mag_dx, f"rms dx D={D} w={weight}")
        if weight:
            check_grad(dw, ref_dw, mag_dw, f"rms dw D={D}")
            _, dw2 = nv.rms_norm_vjp(x, w, gd, eps=1e-5)
            torch.cuda.synchronize()
            assert torch.equal(dw, dw2), "rms dw not reproducible"
        ldx, ldw, ldb = nv.layer_norm_vjp(x, w, gd, eps=1e-5)
        torch.cuda.synchronize()
        ref = oracle.layer_norm_vjp(host(inp["x"]), host(inp["w"]), host(g), 1e-5)
        check_grad(ldx, ref[0], ref[3], f"layer dx D={D} w={weight}")
        if weight:
            check_grad(ldw, ref[1], ref[4], f"layer dw D={D}")
        check_grad(ldb, ref[2], ref[5], f"layer db D={D}")
        _, _, ldb2 = nv.layer_norm_vjp(x, w, gd, eps=1e-5)
        torch.cuda.synchronize()
        assert torch.equal(ldb, ldb2), "layer db not reproducible"


@pytest.mark.parametrize("dt", ["bf16", "f32"])
@pytest.mark.parametrize("weight", [True, False])
@pytest.mark.parametrize("rows,D", VJP_SHAPES)
def test_layer_norm_vjp(rows, D, weight, dt):
    inp = synth.layer_norm_inputs(rows, D, dt, seed=rows * 3 + D, weight=weight, bias=False)
    g = synth.normal((rows, D), 0.0, 1.0, rows * 3 + D, 4, dt)
    x, w, gd = dev(inp["x"]), dev(inp["w"]), dev(g)
    dx, dw, db = nv.layer_norm_vjp(x, w, gd, eps=1e-5)
    torch.cuda.synchronize()
    ref = oracle.layer_norm_vjp(host(inp["x"]), host(inp["w"]), host(g), 1e-5)
    check_grad(dx, ref[0], ref[3], "dx")
    if weight:
        check_grad(dw, ref[1], ref[4], "dw")
    check_grad(db, ref[2], ref[5], "db")


@pytest.mark.parametrize("dt", ["bf16", "f32"])
@pytest.mark.parametrize("rows,D,shift", [(37, 1001, 0), (300, 7, 0), (5, 40000, 0), (64, 4096, 1),
                                          (3, 1, 0), (1000, 333, 3), (9, 32768, 0)])
def test_vjp_generic_rows(rows, D, shift, dt):
    """Rows the register kernels cannot take -- D not a whole number of 16-byte vectors,
    rows wider than they are built for, pointers off the 16-byte grid (shift elements into
    a larger buffer) -- go to the generic kernel, and meet the same bar."""
    inp = synth.layer_norm_inputs(rows, D, dt, seed=rows + D, weight=True, bias=False)
    g = synth.normal((rows, D), 0.0, 1.0, rows + D, 4, dt)
    tdt = DT[dt]

    def placed(t):  # t as a view starting `shift` elements into a device buffer
        flat = torch.zeros(t.numel() + shift, dtype=tdt, device="cuda")
        flat[shift:] = t.reshape(-1).cuda()
        return flat[shift:].view(t.shape)

    x, w, gd = placed(inp["x"]), placed(inp["w"]), placed(g)
    for op in ("rms", "layer"):
        dx = placed(torch.zeros(rows, D, dtype=tdt))
        dw = placed(torch.zeros(D, dtype=tdt))
        db = placed(torch.zeros(D, dtype=tdt))
        if op == "rms":
            nv.nv_rms_norm_vjp(x, w, gd, dx, dw, 1e-5)
            torch.cuda.synchronize()
            ref = oracle.rms_norm_vjp(host(inp["x"]), host(inp["w"]), host(g), 1e-5)
            check_grad(dx, ref[0], ref[2], "rms dx")
            check_grad(dw, ref[1], ref[3], "rms dw")
        else:
            nv.nv_layer_norm_vjp(x, w, gd, dx, dw, db, 1e-5)
            torch.cuda.synchronize()
            ref = oracle.layer_norm_vjp(host(inp["x"]), host(inp["w"]), host(g), 1e-5)
            check_grad(dx, ref[0], ref[3], "layer dx")
            check_grad(dw, ref[1], ref[4], "layer dw")
            check_grad(db, ref[2], ref[5], "layer db")


@pytest.mark.parametrize("dt,mean,std", [("bf16", 300.0, 0.5), ("bf16", 3000.0, 40.0),
                                         ("f32", 300.0, 0.5), ("f32", -2.0e4, 3.0)])
def test_layer_norm_vjp_large_mean(dt, mean, std):
    # |mean| / std up to ~7000: the row mean has to be carried past float32 rounding of |mean|
    rows, D = 96, 4096
    x = synth.normal((rows, D), mean, std, 31, 0, dt)
    w = synth.normal((D,), 1.0, 0.1, 31, 2, dt)
    g = synth.normal((rows, D), 0.0, 1.0, 31, 4, dt)
    dx, dw, db = nv.layer_norm_vjp(dev(x), dev(w), dev(g), eps=1e-5)
    torch.cuda.synchronize()
    ref = oracle.layer_norm_vjp(host(x), host(w), host(g), 1e-5)
    check_grad(dx, ref[0], ref[3], "dx")
    check_grad(dw, ref[1], ref[4], "dw")
    check_grad(db, ref[2], ref[5], "db")


@pytest.mark.parametrize("dt,D", [("bf16", 1024), ("bf16", 8192), ("f32", 4096)])
def test_layer_norm_vjp_mixed_conditioning(dt, D):
    """Every CTA walks rows of several kinds in turn: means small against the spread, means
    that dwarf it (mean / std = 150) and means of the order of the spread (|mean| around
    std / 2 and above): any statistic that leans on E[x^2] - mean^2, or on a mean carried
    over from another row, fails on some of them."""
    rows = 1500
    x = synth.normal((rows, D), 0.5, 2.0, 47, 0, dt)
    x[1::3] += 300.0                 # mean / std = 150
    x[2::6] = x[2::6] * 0.5 + 0.25   # mean 0.5, std 1
    x[5::6] = x[5::6] * 0.25 + 0.5   # mean 0.625, std 0.5
    w = synth.normal((D,), 1.0, 0.1, 47, 2, dt)
    g = synth.normal((rows, D), 0.0, 1.0, 47, 4, dt)
    dx, dw, db = nv.layer_norm_vjp(dev(x), dev(w), dev(g), eps=1e-5)
    torch.cuda.synchronize()
    ref = oracle.layer_norm_vjp(host(x), host(w), host(g), 1e-5)
    check_grad(dx, ref[0], ref[3], "dx")
    check_grad(dw, ref[1], ref[4], "dw")
    check_grad(db, ref[2], ref[5], "db")


@pytest.mark.parametrize("dt,D", [("bf16", 1024), ("bf16", 4096), ("bf16", 16384), ("f32", 512),
                                  ("f32", 4096), ("f32", 8192)])
def test_layer_norm_vjp_rows_starting_far_from_their_mean(dt, D):
    """Rows whose leading elements sit far from the row mean (1000, 2.5 or 3.0 followed by
    N(0, 1) values), plain N(0, 1) rows and constant rows (variance 0), mixed within one
    CTA's rows: statistics that lean on a row's first elements, or on E[x^2] - mean^2,
    lose precision exactly here."""
    rows = 64
    x = synth.normal((rows, D), 0.0, 1.0, 43, 0, dt)
    for i, v in enumerate((1000.0, 2.5, 3.0)):
        x[i::5, :2] = v
    x[4::5] = 7.0
    w = synth.normal((D,), 1.0, 0.1, 43, 2, dt)
    g = synth.normal((rows, D), 0.0, 1.0, 43, 4, dt)
    dx, dw, db = nv.layer_norm_vjp(dev(x), dev(w), dev(g), eps=1e-5)
    torch.cuda.synchronize()
    ref = oracle.layer_norm_vjp(host(x), host(w), host(g), 1e-5)
    check_grad(dx, ref[0], ref[3], "dx")
    check_grad(dw, ref[1], ref[4], "dw")
    check_grad(db, ref[2], ref[5], "db")


@pytest.mark.parametrize("rows,D", [(20000, 512), (5000, 64), (3001, 1024)])
def test_vjp_many_narrow_rows(rows, D):
    # more rows than partial sums: every CTA walks many rows
    inp = synth.layer_norm_inputs(rows, D, "bf16", seed=rows, weight=True, bias=False)
    g = synth.normal((rows, D), 0.0, 1.0, rows, 4, "bf16")
    x, w, gd = dev(inp["x"]), dev(inp["w"]), dev(g)
    dx, dw, db = nv.layer_norm_vjp(x, w, gd, eps=1e-5)
    rdx, rdw = nv.rms_norm_vjp(x, w, gd, eps=1e-5)
    torch.cuda.synchronize()
    ref = oracle.layer_norm_vjp(host(inp["x"]), host(inp["w"]), host(g), 1e-5)
    check_grad(dx, ref[0], ref[3], "dx")
    check_grad(dw, ref[1], ref[4], "dw")
    check_grad(db, ref[2], ref[5], "db")
    rref = oracle.rms_norm_vjp(host(inp["x"]), host(inp["w"]), host(g), 1e-5)
    check_grad(rdx, rref[0], rref[2], "rms dx")
    check_grad(rdw, rref[1], rref[3], "rms dw")


def test_vjp_deterministic_in_place_and_empty():
    inp = synth.rms_inputs(3000, 4096, "bf16", seed=9)
    g = synth.normal((3000, 4096), 0.0, 1.0, 9, 4, "bf16").cuda()
    x, w = dev(inp["x"]), dev(inp["w"])
    a = nv.rms_norm_vjp(x, w, g)
    b = nv.rms_norm_vjp(x, w, g)
    torch.cuda.synchronize()
    assert torch.equal(a[0].view(torch.int16), b[0].view(torch.int16))
    assert torch.equal(a[1].view(torch.int16), b[1].view(torch.int16)), "dw must be deterministic"
    gg = g.clone()
    dw = torch.empty_like(w)
    nv.nv_rms_norm_vjp(x, w, gg, gg, dw, 1e-5)         # dx written over g
    torch.cuda.synchronize()
    assert torch.equal(gg.view(torch.int16), a[0].view(torch.int16))
    empty = torch.empty(0, 4096, dtype=torch.bfloat16, device="cuda")
    dw0 = torch.full_like(w, 3.0)
    nv.nv_rms_norm_vjp(empty, w, empty, empty, dw0, 1e-5)
    db0 = torch.full_like(w, 3.0)
    nv.nv_layer_norm_vjp(empty, None, empty, empty, None, db0, 1e-5)
    torch.cuda.synchronize()
    assert (dw0 == 0).all() and (db0 == 0).all(), "an empty batch has zero column gradients"


def test_bounded_wait_runs_out_is_counted_and_leaves_the_context_usable():
    """The failure path of the device-side bounded waits: waits on an mbarrier that nothing
    completes give up after about a second, each CTA counts one fault, the host reads the
    count, and the next kernels run normally."""
    import time
    nv.nv_fault_count(reset=True)
    t0 = time.monotonic()
    nv.nv_selftest_bounded_wait(3)
    assert nv.nv_fault_count(reset=True) == 3
    assert 0.5 < time.monotonic() - t0 < 60
    inp = synth.rms_inputs(64, 512, "f32", seed=5)
    x, w = dev(inp["x"]), dev(inp["w"])
    y = nv.rms_norm(x, w, eps=1e-6)
    torch.cuda.synchronize()
    check_out(y, oracle.rms_norm(host(inp["x"]), host(inp["w"]), 1e-6), "after the timed-out waits")
    assert nv.nv_fault_count() == 0
