"""GPU parity at the benchmark workloads' full sizes, in the launch configuration the
benchmark times (automatic plan, programmatic dependent launch).

Element-by-element against the CPU oracle for:
  - add_rms_norm bf16, x and r [8192, 4096] ~ N(0,1), w ~ U(0.5,1.5), eps 1e-5
  - layer_norm bf16, x [16384, 8192] ~ N(0.5, 2^2), w ~ U(0.5,1.5), b ~ N(0, 0.1^2), eps 1e-5
  - norm_rope bf16, x [8, 32, 2048, 128] ~ N(0,1), w ~ U(0.5,1.5), eps 1e-6, dims 128,
    base 10000, scale 1: halves at offset 0, and traditional at offset 4096
  - allreduce_add_rms_norm bf16, 8 parts [8192, 4096] ~ N(0, 1/8), r ~ N(0,1),
    w ~ U(0.5,1.5), eps 1e-5 (the TP8 workload of the benchmark)
  - the gradients: rms_norm_vjp bf16 [8192, 4096] and layer_norm_vjp bf16 [16384, 8192]
    on sampled rows (dx) and every column (dw, db) summed over all rows
and on sampled rows for the add_rms_norm sweep D x rows x {bf16, f32} (eps 1e-6) and for
tensors past 2^31 elements (add_rms_norm, layer_norm, norm_rope, rms_norm_vjp).
Large outputs are compared in row chunks to bound host memory.
"""
import numpy as np
import pytest
import torch

import oracle
import rope_add_rms_b200 as nv
from rope_add_rms_b200 import synth
from checks import check_bf16, check_exact, check_f32, check_grad, sample_rows, to_host_bits

pytestmark = pytest.mark.gpu

CHUNK = 2048


def host(t):
    return None if t is None else synth.to_numpy(t)


def compare_rows(y_dev, ref_fn, rows, what):
    """Compare the device output with ref_fn(r0, r1) row chunk by row chunk."""
    for r0 in range(0, rows, CHUNK):
        r1 = min(rows, r0 + CHUNK)
        got = to_host_bits(y_dev[r0:r1])
        ref = ref_fn(r0, r1)
        if got.dtype == np.uint16:
            check_bf16(got, ref, f"{what} rows {r0}:{r1}")
        else:
            check_f32(got, ref, f"{what} rows {r0}:{r1}")


def test_add_rms_norm_bf16_8192x4096():
    inp = synth.add_rms_inputs(8192, 4096, "bf16", seed=0)
    x, r, w = (inp[k].cuda() for k in ("x", "r", "w"))
    y, h = nv.add_rms_norm(x, r, w, eps=1e-5)
    torch.cuda.synchronize()
    xh, rh, wh = host(inp["x"]), host(inp["r"]), host(inp["w"])
    href_all = []

    def ref(r0, r1):
        yr, hr = oracle.add_rms_norm(xh[r0:r1], rh[r0:r1], wh, 1e-5)
        href_all.append(hr)
        return yr

    compare_rows(y, ref, 8192, "y")
    check_exact(h, np.concatenate(href_all), "h")


def test_layer_norm_bf16_16384x8192():
    inp = synth.layer_norm_inputs(16384, 8192, "bf16", seed=0)
    x, w, b = (inp[k].cuda() for k in ("x", "w", "b"))
    y = nv.layer_norm(x, w, b, eps=1e-5)
    torch.cuda.synchronize()
    xh, wh, bh = host(inp["x"]), host(inp["w"]), host(inp["b"])
    compare_rows(y, lambda r0, r1: oracle.layer_norm(xh[r0:r1], wh, bh, 1e-5), 16384, "y")


@pytest.mark.parametrize("trad,offset", [(0, 0), (1, 4096)])
def test_norm_rope_bf16_8x32x2048x128(trad, offset):
    B, H, L, D = 8, 32, 2048, 128
    inp = synth.norm_rope_inputs(B, H, L, D, "bf16", seed=0)
    x, w = inp["x"].cuda(), inp["w"].cuda()
    y = nv.norm_rope(x.view(B, H, L, D), w, dims=D, traditional=bool(trad), base=10000.0,
                     scale=1.0, offset=offset, eps=1e-6).view(-1, D)
    torch.cuda.synchronize()
    xh, wh = host(inp["x"]), host(inp["w"])
    # row chunks are whole multiples of L, so l = k mod L is preserved
    compare_rows(y, lambda r0, r1: oracle.norm_rope(xh[r0:r1], wh, L, D, trad, 10000.0, 1.0,
                                                    offset, 1, 1e-6), B * H * L, "y")


SWEEP = [(dt, D, rows) for dt in ("bf16", "f32") for D in (2048, 4096, 5120, 8192, 16384)
         for rows in (1, 16, 256, 4096, 65536)]


@pytest.mark.parametrize("dt,D,rows", SWEEP, ids=lambda v: str(v))
def test_add_rms_norm_sweep(dt, D, rows):
    seed = 0
    if rows * D <= 4096 * 4096:
        inp = synth.add_rms_inputs(rows, D, dt, seed)
        x, r, w = (inp[k].cuda() for k in ("x", "r", "w"))
    else:   # drawn on the device: hundreds of millions of values
        x = synth.normal_device((rows, D), 0.0, 1.0, seed, synth.X, dt)
        r = synth.normal_device((rows, D), 0.0, 1.0, seed, synth.R, dt)
        w = synth.uniform_device((D,), 0.5, 1.5, seed, synth.W, dt)
    y, h = nv.add_rms_norm(x, r, w, eps=1e-6)
    torch.cuda.synchronize()
    idx = torch.as_tensor(sample_rows(rows, 384, seed=D + rows), device="cuda")
    xs, rs, ws = to_host_bits(x[idx]), to_host_bits(r[idx]), to_host_bits(w)
    ref, href = oracle.add_rms_norm(xs, rs, ws, 1e-6)
    check_exact(h[idx], href, "h")
    got = to_host_bits(y[idx])
    (check_bf16 if dt == "bf16" else check_f32)(got, ref, "y")
    del x, r, y, h
    torch.cuda.empty_cache()


def test_allreduce_add_rms_norm_tp8_bf16_8192x4096():
    inp = synth.allreduce_inputs(8192, 4096, 8, "bf16", seed=0)
    parts = [p.cuda() for p in inp["parts"]]
    r, w = inp["r"].cuda(), inp["w"].cuda()
    y, h, x = nv.allreduce_add_rms_norm(parts, r, w, eps=1e-5)
    torch.cuda.synchronize()
    ph = [host(p) for p in inp["parts"]]
    rh, wh = host(inp["r"]), host(inp["w"])
    xs, hs = [], []

    def ref(r0, r1):
        yr, hr, xr = oracle.allreduce_add_rms_norm([p[r0:r1] for p in ph], rh[r0:r1], wh, 1e-5)
        xs.append(xr)
        hs.append(hr)
        return yr

    compare_rows(y, ref, 8192, "y")
    check_exact(h, np.concatenate(hs), "h")
    check_exact(x, np.concatenate(xs), "x")


@pytest.mark.parametrize("op,rows,D", [("rms", 8192, 4096), ("layer", 16384, 8192)])
def test_gradients_full_size(op, rows, D):
    """dx of every row chunk by chunk; dw (and db) of every column, the oracle's column sums
    accumulated over the chunks (the bar is relative to the magnitude sums, so the
    order of that accumulation does not matter)."""
    if op == "rms":
        inp = synth.rms_inputs(rows, D, "bf16", seed=0)
    else:
        inp = synth.layer_norm_inputs(rows, D, "bf16", seed=0, bias=False)
    g = synth.normal((rows, D), 0.0, 1.0, 0, synth.R, "bf16")
    x, w, gd = inp["x"].cuda(), inp["w"].cuda(), g.cuda()
    if op == "rms":
        dx, dw = nv.rms_norm_vjp(x, w, gd, eps=1e-5)
        db = None
    else:
        dx, dw, db = nv.layer_norm_vjp(x, w, gd, eps=1e-5)
    torch.cuda.synchronize()
    xh, wh, gh = host(inp["x"]), host(inp["w"]), host(g)
    sums = None
    for r0 in range(0, rows, CHUNK):
        r1 = min(rows, r0 + CHUNK)
        if op == "rms":
            rdx, rdw, mdx, mdw = oracle.rms_norm_vjp(xh[r0:r1], wh, gh[r0:r1], 1e-5)
            parts = [rdw, mdw]
        else:
            rdx, rdw, rdb, mdx, mdw, mdb = oracle.layer_norm_vjp(xh[r0:r1], wh, gh[r0:r1], 1e-5)
            parts = [rdw, rdb, mdw, mdb]
        check_grad(dx[r0:r1], rdx, mdx, f"dx rows {r0}:{r1}")
        parts = [np.asarray(p, np.float64) for p in parts]
        sums = parts if sums is None else [a + b for a, b in zip(sums, parts)]
    if op == "rms":
        check_grad(dw, sums[0], sums[1], "dw")
    else:
        check_grad(dw, sums[0], sums[2], "dw")
        check_grad(db, sums[1], sums[3], "db")


# ---- past 2^31 elements ---------------------------------------------------------------------
# Row offsets are 64-bit throughout the kernels; these runs place rows beyond element 2^31
# (byte 2^32 of a bf16 tensor) and compare sampled rows -- the rows straddling that boundary
# and the last row always among them -- with the oracle.  About 26 GB of device memory at
# the peak (four 4.3 GB tensors and the float32 draw of one).
def _rows_past(rows, D, seed, k=64):
    edge = (1 << 31) // D
    return np.unique(np.concatenate([sample_rows(rows, k, seed),
                                     np.arange(edge - 2, min(rows, edge + 3)), [rows - 1]]))


def test_add_rms_norm_and_layer_norm_past_2_31_elements():
    rows, D = (1 << 31) // 4096 + 5, 4096
    x = synth.normal_device((rows, D), 0.0, 1.0, 7, synth.X, "bf16")
    r = synth.normal_device((rows, D), 0.0, 1.0, 7, synth.R, "bf16")
    w = synth.uniform_device((D,), 0.5, 1.5, 7, synth.W, "bf16")
    b = synth.normal_device((D,), 0.0, 0.1, 7, synth.B, "bf16")
    y, h = nv.add_rms_norm(x, r, w, eps=1e-5)
    torch.cuda.synchronize()
    idx = torch.as_tensor(_rows_past(rows, D, 1), device="cuda")
    xs, rs, ws, bs = to_host_bits(x[idx]), to_host_bits(r[idx]), to_host_bits(w), to_host_bits(b)
    ref, href = oracle.add_rms_norm(xs, rs, ws, 1e-5)
    check_exact(h[idx], href, "h")
    check_bf16(to_host_bits(y[idx]), ref, "y")
    del r, y, h
    torch.cuda.empty_cache()
    yl = nv.layer_norm(x, w, b, eps=1e-5)
    torch.cuda.synchronize()
    check_bf16(to_host_bits(yl[idx]), oracle.layer_norm(xs, ws, bs, 1e-5), "layer_norm y")
    del x, yl
    torch.cuda.empty_cache()


def test_norm_rope_and_rms_norm_vjp_past_2_31_elements():
    H, L, D = 256, 65537, 128            # 16 777 472 rows of 128: 2^31 + 32 768 elements
    rows = H * L
    x = synth.normal_device((rows, D), 0.0, 1.0, 8, synth.X, "bf16")
    w = synth.uniform_device((D,), 0.5, 1.5, 8, synth.W, "bf16")
    y = nv.norm_rope(x.view(1, H, L, D), w, dims=D, traditional=False, base=10000.0,
                     scale=1.0, offset=0, eps=1e-6).view(rows, D)
    torch.cuda.synchronize()
    ks = _rows_past(rows, D, 2)
    idx = torch.as_tensor(ks, device="cuda")
    xs, ws, ys = to_host_bits(x[idx]), to_host_bits(w), to_host_bits(y[idx])
    for i, k in enumerate(ks):       # row k sits at position k mod L
        ref = oracle.norm_rope(xs[i:i + 1], ws, 1, D, 0, 10000.0, 1.0, int(k % L), 1, 1e-6)
        check_bf16(ys[i:i + 1], ref, f"norm_rope row {k}")
    del y
    torch.cuda.empty_cache()
    g = synth.normal_device((rows, D), 0.0, 1.0, 8, synth.R, "bf16")
    dx, dw = nv.rms_norm_vjp(x, w, g, eps=1e-5)
    torch.cuda.synchronize()
    rdx, _, mdx, _ = oracle.rms_norm_vjp(xs, ws, to_host_bits(g[idx]), 1e-5)
    check_grad(dx[idx], rdx, mdx, "rms_norm_vjp dx")
    assert torch.isfinite(dw.float()).all()
    del x, g, dx, dw
    torch.cuda.empty_cache()
