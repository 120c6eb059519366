"""Comparison helpers for the GPU-vs-oracle parity tests.

Tolerances (stated once, used everywhere):
  - h (the updated residual) must be bit-exact.
  - bfloat16 y: at most one bfloat16 step from the oracle's value rounded (once, to
    nearest even) to bfloat16 -- the ordinal distance between the two bit patterns
    is <= 1.  This is the "within 1 bf16 ulp" bar, taken in its strict form.
  - float32 y: |y - ref| <= 1e-5 * (1 + |ref|).
  - A NaN reference must give NaN; an infinite one the same infinity.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

F32_TOL = 1e-5


def to_host_bits(t: torch.Tensor) -> np.ndarray:
    """Device or host tensor -> numpy (bfloat16 as uint16 bits, float32 as float32)."""
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def bf16_ordinal(bits: np.ndarray) -> np.ndarray:
    """Monotone integer code of bfloat16 bit patterns (+0 and -0 both map to 0)."""
    b = bits.astype(np.int64)
    return np.where(b & 0x8000, -(b & 0x7FFF), b)


def check_bf16(y_bits: np.ndarray, ref: np.ndarray, what: str = "y"):
    """GPU bfloat16 output vs float64 oracle: within one bfloat16 step of RNE(ref)."""
    y_bits = np.asarray(y_bits, np.uint16).reshape(-1)
    ref = np.asarray(ref, np.float64).reshape(-1)
    want = oracle.round_bf16(ref)
    nan_ref = np.isnan(ref)
    ygot = (y_bits.astype(np.uint32) << 16).view(np.float32)
    nan_got = np.isnan(ygot)
    assert (nan_got == nan_ref).all(), f"{what}: NaN pattern differs " \
        f"({int(nan_ref.sum())} expected, {int(nan_got.sum())} got)"
    ok = ~nan_ref
    dist = np.abs(bf16_ordinal(y_bits[ok]) - bf16_ordinal(want[ok]))
    bad = dist > 1
    if bad.any():
        i = np.flatnonzero(ok)[np.argmax(dist)]
        raise AssertionError(
            f"{what}: {int(bad.sum())} of {ok.sum()} elements more than one bf16 step off; "
            f"worst at flat index {i}: got {float(ygot[i])!r}, oracle {float(ref[i])!r} "
            f"({int(dist.max())} steps)")
    return int(dist.max()) if dist.size else 0


def check_f32(y: np.ndarray, ref: np.ndarray, what: str = "y"):
    """GPU float32 output vs float64 oracle: |y - ref| <= 1e-5 (1 + |ref|)."""
    y = np.asarray(y, np.float32).reshape(-1).astype(np.float64)
    ref = np.asarray(ref, np.float64).reshape(-1)
    nan_ref = np.isnan(ref)
    assert (np.isnan(y) == nan_ref).all(), f"{what}: NaN pattern differs"
    ok = ~nan_ref
    err = np.abs(y[ok] - ref[ok])
    lim = F32_TOL * (1.0 + np.abs(ref[ok]))
    bad = err > lim
    if bad.any():
        i = np.argmax(err / lim)
        raise AssertionError(f"{what}: {int(bad.sum())} of {ok.sum()} elements off; worst "
                             f"got {y[ok][i]!r}, oracle {ref[ok][i]!r}")
    return float((err / (1.0 + np.abs(ref[ok]))).max()) if err.size else 0.0


def check_out(y_dev, ref, what="y"):
    host = to_host_bits(y_dev)
    if host.dtype == np.uint16:
        return check_bf16(host, ref, what)
    return check_f32(host, ref, what)


def check_exact(got_dev, want_host: np.ndarray, what="h"):
    got = to_host_bits(got_dev).reshape(-1)
    want = np.asarray(want_host).reshape(-1)
    same = got.view(np.uint32 if got.dtype == np.float32 else np.uint16) == \
        want.view(np.uint32 if want.dtype == np.float32 else np.uint16)
    assert same.all(), f"{what}: {int((~same).sum())} of {same.size} elements not bit-exact"


# ---- guard bands --------------------------------------------------------------------

CANARY_BYTES = 4096


class Guarded:
    """A device buffer with canary-filled bands on both sides of the tensor handed out."""

    def __init__(self, shape, dtype, device="cuda", fill=None):
        n = int(np.prod(shape))
        es = torch.empty((), dtype=dtype).element_size()
        pad = CANARY_BYTES // es
        self.raw = torch.empty(pad + n + pad, dtype=dtype, device=device)
        self._bytes = self.raw.view(torch.uint8)
        self._bytes.fill_(0xA5)
        self.pad = pad
        self.t = self.raw[pad:pad + n].view(shape)
        if fill is not None:
            self.t.copy_(fill)

    def bands_intact(self) -> bool:
        b = self._bytes
        head = b[:self.pad * self.t.element_size()]
        tail = b[(self.pad + self.t.numel()) * self.t.element_size():]
        return bool((head == 0xA5).all().item() and (tail == 0xA5).all().item())


def sample_rows(rows: int, k: int, seed: int = 0) -> np.ndarray:
    """k row indices spread over [0, rows): first, last and random ones in between."""
    if rows <= k:
        return np.arange(rows)
    rng = np.random.default_rng(seed)
    mid = rng.choice(np.arange(1, rows - 1), size=k - 2, replace=False)
    return np.unique(np.concatenate([[0, rows - 1], mid]))


# ---- gradients ------------------------------------------------------------------------
# The vjp outputs are formed in float32 from terms that can cancel; their bar, derived
# from that arithmetic: the bfloat16 (float32) bar above, or an absolute error of at
# most 2^-16 times the sum of the magnitudes of the terms (the oracle's mag_* output).

VJP_MAG = 2.0 ** -16


def check_grad(y_dev, ref, mag, what="grad"):
    host = to_host_bits(y_dev).reshape(-1)
    ref = np.asarray(ref, np.float64).reshape(-1)
    mag = np.asarray(mag, np.float64).reshape(-1)
    if host.dtype == np.uint16:
        got = (host.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        dist = np.abs(bf16_ordinal(host) - bf16_ordinal(oracle.round_bf16(ref)))
        ok = (dist <= 1) | (np.abs(got - ref) <= VJP_MAG * mag)
    else:
        got = host.astype(np.float64)
        ok = (np.abs(got - ref) <= F32_TOL * (1 + np.abs(ref))) | \
             (np.abs(got - ref) <= VJP_MAG * mag)
    if not ok.all():
        i = np.argmax(~ok)
        raise AssertionError(f"{what}: {int((~ok).sum())} of {ok.size} elements off; first at "
                             f"{i}: got {got[i]!r}, oracle {ref[i]!r}, magnitude {mag[i]!r}")
