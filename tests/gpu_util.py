"""Helpers of the GPU parity tests: upload seeded inputs, call the library,
compare with the oracle under |y - y_ref| <= 1e-5 * sum|x*w| + 1e-6."""

from __future__ import annotations

import numpy as np

import oracle


def torch():
    import torch as T
    return T


def dev(a):
    T = torch()
    return T.from_numpy(np.ascontiguousarray(a)).cuda()


def upload_w4(w: dict) -> dict:
    return {"qw": dev(w["qw"]), "scales": dev(w["scales"]), "zp": dev(w["zp"]), "K": w["K"], "N": w["N"]}


def guarded(M: int, N: int, ld: int | None = None, pad: int = 64):
    """A [M, ld] fp32 view inside a NaN-filled buffer with `pad` guard floats on
    both sides; returns (view, buffer)."""
    T = torch()
    ld = N if ld is None else ld
    buf = T.full((pad + M * ld + pad,), float("nan"), dtype=T.float32, device="cuda")
    # the view starts 64 floats (256 B) in: 16-byte aligned like a fresh tensor
    view = buf[pad:pad + M * ld].view(M, ld)[:, :N] if M > 0 else buf[pad:pad].view(0, N)
    return view, buf


def guards_intact(buf, M: int, N: int, ld: int, pad: int = 64) -> bool:
    T = torch()
    h = buf.cpu().numpy()
    ok = np.all(np.isnan(h[:pad])) and np.all(np.isnan(h[pad + M * ld:]))
    if ld > N and M > 0:
        body = h[pad:pad + M * ld].reshape(M, ld)
        ok = ok and np.all(np.isnan(body[:, N:]))
    return bool(ok)


def check(y_gpu, y_ref, a, what: str):
    y = y_gpu.detach().cpu().numpy().astype(np.float64) if hasattr(y_gpu, "cpu") else np.asarray(y_gpu)
    v = oracle.max_violation(y, y_ref, a)
    assert v <= 0, f"{what}: tolerance exceeded by {v:.3e} (max |err| {np.abs(y - y_ref).max():.3e})"
