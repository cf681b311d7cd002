"""B200 quantised-weight matmul library: Python binding of libw4b200.so.

Argument marshalling only: every step of the computation runs in the
library's CUDA kernels (sm_100a). PyTorch provides device memory and
streams. If the library is missing or the GPU is not a B200 the calls raise;
nothing falls back to another implementation.

Operations (see include/w4.h for layouts and error behaviour):
  w4_matmul(x, qw, scales, zp, K, N)        y = x . W, W 4-bit blocked
      (..., bias=, residual=, act=)         y = act(x . W + bias) + residual, fused
  w4_matmul_grouped([...])                  many independent ones, one launch
  w4_repack(qw, scales, zp, K, N)           the weight in the streaming layout (once, at load)
  w4r_matmul(x, wr, K, N) / _grouped        decode (M = 1) on repacked weights
  i8_head_logits(h, table, scales, K, V)    last-position logits, int8 head
  i8_head_repack(table, scales, K, V)       the head in the streaming layout (once, at load)
  i8r_head_logits(h, tr, K, V) / _argmax    M = 1 head on the repacked table
  w4i_matmul(x, wt, K, N)                   M = 1 on the tile layout: integer tensor-core MMAs
  i8t_head_repack(table, scales, K, V)      the head in the tensor cores' tile layout (once, at load)
  i8t_head_logits(h, tiles, K, V) / _argmax M <= 8 rows on the tensor-core head
  w4_quantize(w, block, scale_type)         the dq4 quantiser (GPU)
  i8_quantize_head(w)                       the embedding_int8 quantiser (GPU)
  pack_nibbles / unpack_nibbles             host-side UINT4 packing
"""

from __future__ import annotations

import ctypes as C
from typing import Sequence

import numpy as np

from . import _lib
from ._lib import ACTS, GROUP_MAX, PATHS, STATUS, W4Desc, W4LibraryMissing, W4RDesc  # noqa: F401


class W4Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        detail = ""
        try:
            detail = (_lib.load().w4_last_error() or b"").decode()
        except Exception:
            pass
        super().__init__(f"{where}: {STATUS.get(status, status)}: {detail}")


def _check(status: int, where: str) -> None:
    if status != 0:
        raise W4Error(status, where)


def lib():
    return _lib.load()


def abi_version() -> int:
    return lib().w4_abi_version()


# ---------------------------------------------------------------- torch helpers

def _torch():
    import torch
    return torch


def _ptr(t) -> int:
    return 0 if t is None else int(t.data_ptr())


def _stream_handle(stream) -> int:
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream)


_WS = {}  # device index -> zero-filled uint8 workspace tensor


def workspace(nbytes: int, device=None):
    """A zero-filled device workspace of at least nbytes (cached per device).

    The kernels leave it zero-filled, so it is zeroed only when allocated.
    Calls that may overlap on the GPU must not share one: pass your own.
    """
    torch = _torch()
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    idx = dev.index if dev.index is not None else torch.cuda.current_device()
    cur = _WS.get(idx)
    if nbytes == 0:
        return None
    if cur is None or cur.numel() < nbytes:
        cur = torch.zeros(max(nbytes, 1 << 20), dtype=torch.uint8, device=dev)
        _WS[idx] = cur
    return cur


def _ld(t, inner: int) -> int:
    """Row stride in elements; a single row has no stride of its own."""
    if t.dim() == 1 or t.shape[0] <= 1:
        return max(inner, 1)
    if t.stride(-1) != 1 and t.shape[-1] > 1:
        raise ValueError("innermost dimension must be contiguous")
    return int(t.stride(0))


# ---------------------------------------------------------------- body

def w4_matmul_workspace_size(M: int, K: int, N: int) -> int:
    return int(lib().w4_matmul_workspace_size(M, K, N))


def _epilogue(it: dict, N: int):
    """(bias ptr, residual ptr, ldr, act code) of an item's optional epilogue."""
    bias, res, act = it.get("bias"), it.get("residual"), it.get("act", "none")
    if act not in ACTS:
        raise ValueError(f"act must be one of {sorted(ACTS)}")
    return _ptr(bias), _ptr(res), (0 if res is None else _ld(res, N)), ACTS[act]


def w4_matmul(x, qw, scales, zp, K: int, N: int, y=None, path: str = "auto", ws=None, stream=None, bias=None,
              residual=None, act: str = "none"):
    """y[M, N] = x[M, K] . W[K, N] (fp32) with W given as packed nibbles,
    fp32 scales [K/32, N] and packed zero points; returns y.

    With bias ([N]), residual ([M, N], may be y itself) or act ("gelu_tanh",
    "gelu_erf") the kernel's final store computes act(x . W + bias) + residual."""
    torch = _torch()
    M = x.shape[0] if x.dim() == 2 else 1
    if y is None:
        y = torch.empty((M, N), dtype=torch.float32, device=x.device)
    need = w4_matmul_workspace_size(M, K, N)
    if ws is None:
        ws = workspace(need, x.device)
    if bias is not None or residual is not None or act != "none":
        b, r, ldr, a = _epilogue({"bias": bias, "residual": residual, "act": act}, N)
        d = W4Desc(_ptr(x), _ld(x, K), _ptr(qw), _ptr(scales), _ptr(zp), _ptr(y), _ld(y, N), M, K, N, b, r, ldr, a, 0)
        st = lib().w4_matmul_desc(C.byref(d), _ptr(ws), 0 if ws is None else ws.numel() * ws.element_size(),
                                  PATHS[path], _stream_handle(stream))
        _check(st, "w4_matmul")
        return y
    st = lib().w4_matmul_path(_ptr(x), _ld(x, K), _ptr(qw), _ptr(scales), _ptr(zp), _ptr(y), _ld(y, N), M, K, N,
                              _ptr(ws), 0 if ws is None else ws.numel() * ws.element_size(), PATHS[path],
                              _stream_handle(stream))
    _check(st, "w4_matmul")
    return y


def make_descs(items: Sequence[dict]):
    """ctypes descriptor array for w4_matmul_grouped; each item holds the
    tensors x, qw, scales, zp, y and the ints K, N (M from x), and optionally
    the fused epilogue "bias", "residual" and "act" (as in w4_matmul)."""
    arr = (W4Desc * len(items))()
    for i, it in enumerate(items):
        x, y = it["x"], it["y"]
        K, N = int(it["K"]), int(it["N"])
        M = x.shape[0] if x.dim() == 2 else 1
        b, r, ldr, a = _epilogue(it, N)
        arr[i] = W4Desc(_ptr(x), _ld(x, K), _ptr(it["qw"]), _ptr(it["scales"]), _ptr(it["zp"]), _ptr(y),
                        _ld(y, N), M, K, N, b, r, ldr, a, 0)
    return arr


def w4_matmul_grouped_workspace_size(descs) -> int:
    return int(lib().w4_matmul_grouped_workspace_size(descs, len(descs)))


def w4_matmul_grouped(items: Sequence[dict] | None = None, descs=None, ws=None, stream=None):
    """All matmuls of `items` (or a prepared descriptor array) in grouped launches."""
    if descs is None:
        descs = make_descs(items)
    need = w4_matmul_grouped_workspace_size(descs)
    if ws is None:
        ws = workspace(need)
    st = lib().w4_matmul_grouped(descs, len(descs), _ptr(ws), 0 if ws is None else ws.numel() * ws.element_size(),
                                 _stream_handle(stream))
    _check(st, "w4_matmul_grouped")


# ---------------------------------------------------------------- streaming layout (decode)

def w4_repacked_bytes(K: int, N: int) -> int:
    return int(lib().w4_repacked_bytes(K, N))


def w4_repack(qw, scales, zp, K: int, N: int, out=None, stream=None):
    """The weight (page format: packed nibbles, fp32 scales, packed zero
    points) in the streaming layout the decode GEMV reads: a uint8 device
    tensor of w4_repacked_bytes(K, N) bytes holding the same words, reordered."""
    torch = _torch()
    nbytes = w4_repacked_bytes(K, N)
    if nbytes == 0:
        raise ValueError(f"the streaming layout does not take K={K}, N={N} (K % 32 == 0, N % 8 == 0)")
    if out is None:
        out = torch.empty(nbytes, dtype=torch.uint8, device=qw.device)
    st = lib().w4_repack(_ptr(qw), _ptr(scales), _ptr(zp), K, N, _ptr(out), _stream_handle(stream))
    _check(st, "w4_repack")
    return out


def w4_repack_restore(wr, K: int, N: int, stream=None):
    """The page-format buffers (qw, scales, zp) of a repacked weight."""
    torch = _torch()
    nb = K // 32
    qw = torch.empty(K * N // 2, dtype=torch.uint8, device=wr.device)
    sc = torch.empty((nb, N), dtype=torch.float32, device=wr.device)
    zp = torch.empty(nb * N // 2, dtype=torch.uint8, device=wr.device)
    st = lib().w4_repack_restore(_ptr(wr), K, N, _ptr(qw), _ptr(sc), _ptr(zp), _stream_handle(stream))
    _check(st, "w4_repack_restore")
    return qw, sc, zp


def make_rdescs(items: Sequence[dict]):
    """ctypes w4r_desc array for w4r_matmul_grouped; each item holds the
    tensors x ([1, K] or [K]), wr (repacked), y and the ints K, N, and
    optionally "bias", "residual" and "act"."""
    arr = (W4RDesc * len(items))()
    for i, it in enumerate(items):
        x, y = it["x"], it["y"]
        K, N = int(it["K"]), int(it["N"])
        M = x.shape[0] if x.dim() == 2 else 1
        b, r, ldr, a = _epilogue(it, N)
        arr[i] = W4RDesc(_ptr(x), _ld(x, K), _ptr(it["wr"]), _ptr(y), _ld(y, N), M, K, N, b, r, ldr, a, 0)
    return arr


def w4r_matmul_grouped(items: Sequence[dict] | None = None, descs=None, stream=None):
    """All decode matmuls of `items` (or a prepared w4r_desc array)."""
    if descs is None:
        descs = make_rdescs(items)
    st = lib().w4r_matmul_grouped(descs, len(descs), _stream_handle(stream))
    _check(st, "w4r_matmul_grouped")


def w4r_matmul(x, wr, K: int, N: int, y=None, stream=None, bias=None, residual=None, act: str = "none"):
    """y[1, N] = act(x[1, K] . W + bias) + residual with W repacked (w4_repack)."""
    torch = _torch()
    if y is None:
        y = torch.empty((1, N), dtype=torch.float32, device=x.device)
    item = {"x": x, "wr": wr, "y": y, "K": K, "N": N, "bias": bias, "residual": residual, "act": act}
    w4r_matmul_grouped(descs=make_rdescs([item]), stream=stream)
    return y


# ---------------------------------------------------------------- tile layout (prefill)

_TWS: dict = {}


def tile_workspace(nbytes: int, device=None):
    """A device scratch of at least nbytes for w4t_matmul_grouped (cached per
    device; no zeroing needed). Calls that may overlap on the GPU must not
    share one: pass your own."""
    torch = _torch()
    if nbytes == 0:
        return None
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    idx = dev.index if dev.index is not None else torch.cuda.current_device()
    cur = _TWS.get(idx)
    if cur is None or cur.numel() < nbytes:
        cur = torch.empty(max(nbytes, 1 << 20), dtype=torch.uint8, device=dev)
        _TWS[idx] = cur
    return cur


def w4t_repacked_bytes(K: int, N: int) -> int:
    return int(lib().w4t_repacked_bytes(K, N))


def w4t_repack(qw, scales, zp, K: int, N: int, out=None, stream=None):
    """The weight (page format) in the tile layout the tensor-core tile GEMM
    reads: a uint8 device tensor of w4t_repacked_bytes(K, N) bytes."""
    torch = _torch()
    nbytes = w4t_repacked_bytes(K, N)
    if nbytes == 0:
        raise ValueError(f"the tile layout does not take K={K}, N={N} (K % 32 == 0, N % 8 == 0)")
    if out is None:
        out = torch.empty(nbytes, dtype=torch.uint8, device=qw.device)
    _check(lib().w4t_repack(_ptr(qw), _ptr(scales), _ptr(zp), K, N, _ptr(out), _stream_handle(stream)), "w4t_repack")
    return out


def w4t_repack_restore(wt, K: int, N: int, stream=None):
    """The page-format buffers (qw, scales, zp) of a weight in the tile layout."""
    torch = _torch()
    nb = K // 32
    qw = torch.empty(K * N // 2, dtype=torch.uint8, device=wt.device)
    sc = torch.empty((nb, N), dtype=torch.float32, device=wt.device)
    zp = torch.empty(nb * N // 2, dtype=torch.uint8, device=wt.device)
    _check(lib().w4t_repack_restore(_ptr(wt), K, N, _ptr(qw), _ptr(sc), _ptr(zp), _stream_handle(stream)),
           "w4t_repack_restore")
    return qw, sc, zp


def w4t_workspace_size(descs) -> int:
    return int(lib().w4t_workspace_size(descs, len(descs)))


def w4t_matmul_grouped(items: Sequence[dict] | None = None, descs=None, ws=None, stream=None):
    """Matmuls of any M on tile-layout weights ("wr" = w4t_repack output) on
    the tensor cores; items as for make_rdescs (x [M, K])."""
    if descs is None:
        descs = make_rdescs(items)
    need = w4t_workspace_size(descs)
    if ws is None:
        ws = tile_workspace(need)
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(lib().w4t_matmul_grouped(descs, len(descs), _ptr(ws), nbytes, _stream_handle(stream)),
           "w4t_matmul_grouped")


def w4t_matmul(x, wt, K: int, N: int, y=None, ws=None, stream=None, bias=None, residual=None, act: str = "none"):
    """y[M, N] = act(x[M, K] . W + bias) + residual with W in the tile layout
    (w4t_repack); returns y."""
    torch = _torch()
    if x.dim() == 1:
        x = x.view(1, -1)
    if y is None:
        y = torch.empty((x.shape[0], N), dtype=torch.float32, device=x.device)
    item = {"x": x, "wr": wt, "y": y, "K": K, "N": N, "bias": bias, "residual": residual, "act": act}
    w4t_matmul_grouped(descs=make_rdescs([item]), ws=ws, stream=stream)
    return y


def w4i_workspace_size(descs) -> int:
    return int(lib().w4i_workspace_size(descs, len(descs)))


def w4i_matmul_grouped(items: Sequence[dict] | None = None, descs=None, ws=None, stream=None):
    """Decode matmuls (M = 1) on tile-layout weights ("wr" = w4t_repack output)
    with integer tensor-core MMAs; items as for make_rdescs (x [1, K])."""
    if descs is None:
        descs = make_rdescs(items)
    need = w4i_workspace_size(descs)
    if ws is None:
        ws = tile_workspace(need)
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(lib().w4i_matmul_grouped(descs, len(descs), _ptr(ws), nbytes, _stream_handle(stream)),
           "w4i_matmul_grouped")


def w4i_matmul(x, wt, K: int, N: int, y=None, ws=None, stream=None, bias=None, residual=None, act: str = "none"):
    """y[1, N] = act(x[1, K] . W + bias) + residual with W in the tile layout
    (w4t_repack), on the integer tensor-core GEMV; returns y."""
    torch = _torch()
    if x.dim() == 1:
        x = x.view(1, -1)
    if y is None:
        y = torch.empty((x.shape[0], N), dtype=torch.float32, device=x.device)
    item = {"x": x, "wr": wt, "y": y, "K": K, "N": N, "bias": bias, "residual": residual, "act": act}
    w4i_matmul_grouped(descs=make_rdescs([item]), ws=ws, stream=stream)
    return y


# ---------------------------------------------------------------- head

def i8_head_workspace_size(M: int, K: int, V: int) -> int:
    return int(lib().i8_head_workspace_size(M, K, V))


def i8_head_logits(h, table, scales, K: int, V: int, ldt: int | None = None, logits=None, path: str = "auto",
                   ws=None, stream=None):
    """logits[M, V] = h[M, K] . (T[K, V] * s[V]) for the int8 tied head; h holds
    the last-position rows."""
    torch = _torch()
    M = h.shape[0] if h.dim() == 2 else 1
    ldt = V if ldt is None else ldt
    if logits is None:
        logits = torch.empty((M, V), dtype=torch.float32, device=h.device)
    if ws is None:
        ws = workspace(i8_head_workspace_size(M, K, V), h.device)
    st = lib().i8_head_logits_path(_ptr(h), _ld(h, K), _ptr(table), ldt, _ptr(scales), _ptr(logits),
                                   _ld(logits, V), M, K, V, _ptr(ws),
                                   0 if ws is None else ws.numel() * ws.element_size(), PATHS[path],
                                   _stream_handle(stream))
    _check(st, "i8_head_logits")
    return logits


def i8_head_argmax(h, table, scales, K: int, V: int, ldt: int | None = None, stream=None):
    """Greedy next tokens of the last-position rows h: (tokens int32 [M],
    best logits fp32 [M]), the argmax of the logits i8_head_logits gives
    (ties to the lowest token id)."""
    torch = _torch()
    M = h.shape[0] if h.dim() == 2 else 1
    ldt = V if ldt is None else ldt
    tokens = torch.empty(M, dtype=torch.int32, device=h.device)
    best = torch.empty(M, dtype=torch.float32, device=h.device)
    ws = workspace(int(lib().i8_head_argmax_workspace_size(M, K, V)), h.device)
    st = lib().i8_head_argmax(_ptr(h), _ld(h, K), _ptr(table), ldt, _ptr(scales), M, K, V, _ptr(tokens), _ptr(best),
                              _ptr(ws), 0 if ws is None else ws.numel() * ws.element_size(), _stream_handle(stream))
    _check(st, "i8_head_argmax")
    return tokens, best


def i8_head_repacked_bytes(K: int, V: int) -> int:
    return int(lib().i8_head_repacked_bytes(K, V))


def i8_head_repack(table, scales, K: int, V: int, ldt: int | None = None, stream=None):
    """The int8 head (page format) in the streaming layout the M = 1 head
    GEMV reads: a uint8 device tensor of i8_head_repacked_bytes(K, V) bytes."""
    torch = _torch()
    ldt = V if ldt is None else ldt
    n = i8_head_repacked_bytes(K, V)
    if n == 0:
        raise ValueError(f"the streaming head does not take K={K}, V={V}")
    out = torch.empty(n, dtype=torch.uint8, device=table.device)
    _check(lib().i8_head_repack(_ptr(table), ldt, _ptr(scales), K, V, _ptr(out), _stream_handle(stream)),
           "i8_head_repack")
    return out


def i8_head_repack_restore(tr, K: int, V: int, stream=None):
    """(table [K, V] int8, scales [V] fp32) of a repacked head."""
    torch = _torch()
    table = torch.empty((K, V), dtype=torch.int8, device=tr.device)
    sc = torch.empty(V, dtype=torch.float32, device=tr.device)
    _check(lib().i8_head_repack_restore(_ptr(tr), K, V, _ptr(table), V, _ptr(sc), _stream_handle(stream)),
           "i8_head_repack_restore")
    return table, sc


def i8r_head_logits(h, tr, K: int, V: int, logits=None, stream=None):
    """logits [1, V] of one last-position row h on a repacked head."""
    torch = _torch()
    if logits is None:
        logits = torch.empty((1, V), dtype=torch.float32, device=h.device)
    _check(lib().i8r_head_logits(_ptr(h), _ptr(tr), K, V, _ptr(logits), _stream_handle(stream)), "i8r_head_logits")
    return logits


def w4r_decode_step(items: Sequence[dict] | None, h, tr, K: int, V: int, logits=None, descs=None, stream=None):
    """One decode step in one launch: the matmuls of `items` (or a prepared
    w4r_desc array) and the head's logits [1, V] of h on the repacked head."""
    torch = _torch()
    if descs is None:
        descs = make_rdescs(items or [])
    if logits is None:
        logits = torch.empty((1, V), dtype=torch.float32, device=h.device)
    _check(lib().w4r_decode_step(descs, len(descs), _ptr(h), _ptr(tr), K, V, _ptr(logits), _stream_handle(stream)),
           "w4r_decode_step")
    return logits


def w4r_decode_step_argmax(items: Sequence[dict] | None, h, tr, K: int, V: int, descs=None, stream=None):
    """One decode step in one launch with greedy decoding: the matmuls of
    `items` and (token int32 [1], best logit fp32 [1]) of h on the head."""
    torch = _torch()
    if descs is None:
        descs = make_rdescs(items or [])
    tok = torch.empty(1, dtype=torch.int32, device=h.device)
    best = torch.empty(1, dtype=torch.float32, device=h.device)
    keys = torch.empty(1, dtype=torch.int64, device=h.device)
    _check(lib().w4r_decode_step_argmax(descs, len(descs), _ptr(h), _ptr(tr), K, V, _ptr(tok), _ptr(best), _ptr(keys),
                                        _stream_handle(stream)), "w4r_decode_step_argmax")
    return tok, best


def i8r_head_argmax(h, tr, K: int, V: int, stream=None):
    """(token int32 [1], best logit fp32 [1]) of one row h on a repacked head."""
    torch = _torch()
    tok = torch.empty(1, dtype=torch.int32, device=h.device)
    best = torch.empty(1, dtype=torch.float32, device=h.device)
    keys = torch.empty(1, dtype=torch.int64, device=h.device)
    _check(lib().i8r_head_argmax(_ptr(h), _ptr(tr), K, V, _ptr(tok), _ptr(best), _ptr(keys), _stream_handle(stream)),
           "i8r_head_argmax")
    return tok, best


def i8t_head_repacked_bytes(K: int, V: int) -> int:
    return int(lib().i8t_head_repacked_bytes(K, V))


def i8t_head_repack(table, scales, K: int, V: int, ldt: int | None = None, stream=None):
    """The int8 head (page format) in the tile layout the tensor-core head
    reads: a uint8 device tensor of i8t_head_repacked_bytes(K, V) bytes."""
    torch = _torch()
    ldt = V if ldt is None else ldt
    n = i8t_head_repacked_bytes(K, V)
    if n == 0:
        raise ValueError(f"the head tile layout does not take K={K}, V={V}")
    out = torch.empty(n, dtype=torch.uint8, device=table.device)
    _check(lib().i8t_head_repack(_ptr(table), ldt, _ptr(scales), K, V, _ptr(out), _stream_handle(stream)),
           "i8t_head_repack")
    return out


def i8t_head_repack_restore(tiles, K: int, V: int, stream=None):
    """(table [K, V] int8, scales [V] fp32) of a head in the tile layout."""
    torch = _torch()
    table = torch.empty((K, V), dtype=torch.int8, device=tiles.device)
    sc = torch.empty(V, dtype=torch.float32, device=tiles.device)
    _check(lib().i8t_head_repack_restore(_ptr(tiles), K, V, _ptr(table), V, _ptr(sc), _stream_handle(stream)),
           "i8t_head_repack_restore")
    return table, sc


def i8t_head_logits(h, tiles, K: int, V: int, logits=None, stream=None):
    """logits [M, V] of M <= 8 last-position rows h [M, K] on the tensor-core
    head (tile layout)."""
    torch = _torch()
    M = h.shape[0] if h.dim() == 2 else 1
    if logits is None:
        logits = torch.empty((M, V), dtype=torch.float32, device=h.device)
    _check(lib().i8t_head_logits(_ptr(h), _ld(h, K), _ptr(tiles), K, V, M, _ptr(logits), _ld(logits, V),
                                 _stream_handle(stream)), "i8t_head_logits")
    return logits


def i8t_head_argmax(h, tiles, K: int, V: int, stream=None):
    """(tokens int32 [M], best logits fp32 [M]) of M <= 8 rows h on the
    tensor-core head."""
    torch = _torch()
    M = h.shape[0] if h.dim() == 2 else 1
    tok = torch.empty(M, dtype=torch.int32, device=h.device)
    best = torch.empty(M, dtype=torch.float32, device=h.device)
    keys = torch.empty(max(M, 1), dtype=torch.int64, device=h.device)
    _check(lib().i8t_head_argmax(_ptr(h), _ld(h, K), _ptr(tiles), K, V, M, _ptr(tok), _ptr(best), _ptr(keys),
                                 _stream_handle(stream)), "i8t_head_argmax")
    return tok, best


def i8_embed_lookup(table, scales, tokens, K: int, V: int, ldt: int | None = None, out=None, stream=None):
    """out[i, k] = T[k, tokens[i]] * s[tokens[i]]: the token lookup on the tied
    int8 [K, V] table; tokens is a device int32 tensor."""
    torch = _torch()
    ldt = V if ldt is None else ldt
    n = int(tokens.numel())
    if tokens.dtype != torch.int32 or not tokens.is_contiguous():
        raise ValueError("tokens must be a contiguous int32 tensor")
    if out is None:
        out = torch.empty((n, K), dtype=torch.float32, device=table.device)
    st = lib().i8_embed_lookup(_ptr(table), ldt, _ptr(scales), _ptr(tokens), n, _ptr(out), _ld(out, K), K, V,
                               _stream_handle(stream))
    _check(st, "i8_embed_lookup")
    return out


# ---------------------------------------------------------------- quantisers

SCALE_TYPES = {"fp32": 0, "fp16": 1}


def w4_quantize(w, block: int = 32, scale_type: str = "fp32", stream=None):
    """The export's dq4 step on the GPU: fp32 w [K, N] -> (qw [K*N/2] uint8,
    scales [K/block, N] fp32 or fp16, zp [(K/block)*N/2] uint8)."""
    torch = _torch()
    if w.dim() != 2 or w.dtype != torch.float32:
        raise ValueError("w must be a 2-D fp32 tensor")
    if scale_type not in SCALE_TYPES:
        raise ValueError(f"scale_type must be one of {sorted(SCALE_TYPES)}")
    K, N = w.shape
    nb = K // block if block > 0 else 0
    qw = torch.empty(K * N // 2, dtype=torch.uint8, device=w.device)
    sc = torch.empty((nb, N), dtype=torch.float32 if scale_type == "fp32" else torch.float16, device=w.device)
    zp = torch.empty(nb * N // 2, dtype=torch.uint8, device=w.device)
    st = lib().w4_quantize(_ptr(w), _ld(w, N), K, N, block, SCALE_TYPES[scale_type], _ptr(qw), _ptr(sc), _ptr(zp),
                           _stream_handle(stream))
    _check(st, "w4_quantize")
    return qw, sc, zp


def i8_quantize_head(w, stream=None):
    """The export's embedding_int8 step on the GPU: fp32 w [K, V] ->
    (table [K, V] int8, scales [V] fp32)."""
    torch = _torch()
    if w.dim() != 2 or w.dtype != torch.float32:
        raise ValueError("w must be a 2-D fp32 tensor")
    K, V = w.shape
    table = torch.empty((K, V), dtype=torch.int8, device=w.device)
    sc = torch.empty(V, dtype=torch.float32, device=w.device)
    st = lib().i8_quantize_head(_ptr(w), _ld(w, V), K, V, _ptr(table), V, _ptr(sc), _stream_handle(stream))
    _check(st, "i8_quantize_head")
    return table, sc


# ---------------------------------------------------------------- host packing

def pack_nibbles(q) -> np.ndarray:
    q = np.ascontiguousarray(q, dtype=np.uint8).reshape(-1)
    out = np.zeros((q.size + 1) // 2, dtype=np.uint8)
    _check(lib().w4_pack_nibbles(q.ctypes.data, q.size, out.ctypes.data), "w4_pack_nibbles")
    return out


def unpack_nibbles(packed, n: int) -> np.ndarray:
    p = np.ascontiguousarray(packed, dtype=np.uint8).reshape(-1)
    if 2 * p.size < n:
        raise ValueError("buffer too small")
    out = np.zeros(n, dtype=np.uint8)
    _check(lib().w4_unpack_nibbles(p.ctypes.data, n, out.ctypes.data), "w4_unpack_nibbles")
    return out


# ---------------------------------------------------------------- diagnostics

def device_error(clear: bool = True):
    """(status, [status, kernel, block, detail]) of the current device's error word."""
    info = (C.c_int32 * 4)()
    st = lib().w4_device_error(info, 1 if clear else 0)
    return st, list(info)


def set_wait_timeout_ns(ns: int) -> None:
    _check(lib().w4_set_wait_timeout_ns(ns), "w4_set_wait_timeout_ns")


def debug_wait_timeout(ns: int, stream=None) -> None:
    _check(lib().w4_debug_wait_timeout(ns, _stream_handle(stream)), "w4_debug_wait_timeout")
