"""fp64 CPU oracle for Ulysses sequence-parallel self-attention.

TEST INFRASTRUCTURE: only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this package.  The
product path (``video_dit_sequence_b200``) never imports it and shares no code
with it.

What it computes, and the passages it follows:

* ``exchange_pack`` / ``exchange_unpack`` -- the same exchange seen from one
  rank when every rank is its own GPU: the send-buffer reorder in front of
  the all-to-all and the reverse reorder after the return all-to-all.
* ``pack`` / ``unpack`` -- the token<->head all-to-all of the fal.ai page
  "Generate video with WAN 2.2 across four GPUs", section "Splitting one
  generation across four GPUs" (each GPU attends over all tokens for its
  share of the heads, then the outputs go back to the token owners).  Index formulas in ``sp_oracle.c``.
* ``attention_rows_e4m3`` -- the same attention on 8-bit (E4M3) inputs with
  scale factors per block of tokens for Q and K and per channel for V, for
  the FP8 variant of the kernel.
* ``attention_rows_masked`` -- the same attention restricted by a block mask
  over cubes of consecutive tokens (the sparse stage of video sparse
  attention, which the FastVideo page names with 64-token tiles), for the
  block-sparse kernel.
* ``linear_rows`` -- the projection in front of attention (hidden state to
  q, k and v), a plain fp64 matrix product, for the projection kernel whose
  epilogue writes the attention layouts.
* ``attention_rows`` -- the unsharded softmax(q K^T scale) V of one head,
  two-pass exact softmax in fp64; the sequence-parallel result must equal it
  for every degree (LTX-2 "Multi-GPU Inference" README, Capabilities table:
  SP gives the single-GPU result).

Every function is pinned by ``tests/test_oracle_pins.py`` against closed
forms, invariants, a worked example, brute force and numpy's fp64 routines.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sp_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libsp_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compiles sp_oracle.c into libsp_oracle.so next to it."""
    if force or not os.path.exists(_LIB_PATH) or (
            os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-pthread",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _bind(path: str):
    lib = ctypes.CDLL(path)
    i64 = ctypes.c_int64
    vp = ctypes.c_void_p
    for name in ("sp_oracle_pack", "sp_oracle_unpack", "sp_oracle_exchange_pack",
                 "sp_oracle_exchange_unpack", "sp_oracle_shard", "sp_oracle_unshard"):
        f = getattr(lib, name)
        f.argtypes = [vp, vp, i64, i64, i64, i64, i64]
        f.restype = ctypes.c_int
    lib.sp_oracle_attention_rows.argtypes = [
        vp, vp, vp, i64, i64, i64, i64, ctypes.c_double, i64, vp, vp, vp,
        ctypes.c_int]
    lib.sp_oracle_attention_rows.restype = ctypes.c_int
    lib.sp_oracle_attention_rows_e4m3.argtypes = [
        vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, ctypes.c_double, i64, vp, vp, vp,
        ctypes.c_int]
    lib.sp_oracle_attention_rows_e4m3.restype = ctypes.c_int
    lib.sp_oracle_attention_rows_masked.argtypes = [
        vp, vp, vp, vp, i64, i64, i64, i64, i64, ctypes.c_double, i64, vp, vp, vp, ctypes.c_int]
    lib.sp_oracle_attention_rows_masked.restype = ctypes.c_int
    lib.sp_oracle_linear_rows.argtypes = [vp, vp, vp, i64, i64, i64, i64, vp, vp, ctypes.c_int]
    lib.sp_oracle_linear_rows.restype = ctypes.c_int
    lib.sp_oracle_e4m3_value.argtypes = [ctypes.c_uint8]
    lib.sp_oracle_e4m3_value.restype = ctypes.c_double
    return lib


def build_variant(src_text: str, out_path: str):
    """Compiles a modified copy of the oracle source (used by the tests that
    plant mistakes in the oracle to show the pins catch them) and binds it."""
    c_path = out_path + ".c"
    with open(c_path, "w") as f:
        f.write(src_text)
    subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-pthread",
                           "-o", out_path, c_path, "-lm"])
    return _bind(out_path)


def source_text() -> str:
    with open(_SRC) as f:
        return f.read()


def _load():
    global _lib
    if _lib is None:
        _lib = _bind(build())
    return _lib


def _dims(N: int, P: int) -> Tuple[int, int]:
    Nl = -(-N // P)
    return Nl, Nl * P


def pack(xs: np.ndarray, N: int, lib=None) -> np.ndarray:
    """Seq-sharded [P][B][Nl][H][D] -> head-sharded [P][B][Np][Hl][D]."""
    assert xs.dtype == np.uint16 and xs.ndim == 5
    P, B, Nl, H, D = xs.shape
    assert Nl == _dims(N, P)[0]
    if H % P:
        raise ValueError("the Ulysses degree must divide the head count")
    xs = np.ascontiguousarray(xs)
    out = np.empty((P, B, P * Nl, H // P, D), dtype=np.uint16)
    rc = (lib or _load()).sp_oracle_pack(xs.ctypes.data, out.ctypes.data, B, N, H, D, P)
    assert rc == 0
    return out


def unpack(oh: np.ndarray, N: int, H: int, lib=None) -> np.ndarray:
    """Head-sharded [P][B][Np][Hl][D] -> seq-sharded [P][B][Nl][H][D]."""
    assert oh.dtype == np.uint16 and oh.ndim == 5
    P, B, Np, Hl, D = oh.shape
    Nl, Np2 = _dims(N, P)
    assert Np == Np2 and Hl * P == H
    oh = np.ascontiguousarray(oh)
    out = np.empty((P, B, Nl, H, D), dtype=np.uint16)
    rc = (lib or _load()).sp_oracle_unpack(oh.ctypes.data, out.ctypes.data, B, N, H, D, P)
    assert rc == 0
    return out


def shard(x: np.ndarray, P: int, lib=None) -> np.ndarray:
    """Logical [B][N][H][D] -> P token shards [P][B][Nl][H][D], padding zero."""
    assert x.dtype == np.uint16 and x.ndim == 4
    B, N, H, D = x.shape
    Nl = _dims(N, P)[0]
    x = np.ascontiguousarray(x)
    out = np.empty((P, B, Nl, H, D), dtype=np.uint16)
    rc = (lib or _load()).sp_oracle_shard(x.ctypes.data, out.ctypes.data, B, N, H, D, P)
    assert rc == 0
    return out


def unshard(xs: np.ndarray, N: int, lib=None) -> np.ndarray:
    """P token shards [P][B][Nl][H][D] -> logical [B][N][H][D]."""
    assert xs.dtype == np.uint16 and xs.ndim == 5
    P, B, Nl, H, D = xs.shape
    assert Nl == _dims(N, P)[0]
    xs = np.ascontiguousarray(xs)
    out = np.empty((B, N, H, D), dtype=np.uint16)
    rc = (lib or _load()).sp_oracle_unshard(xs.ctypes.data, out.ctypes.data, B, N, H, D, P)
    assert rc == 0
    return out


def exchange_pack(xs_r: np.ndarray, N: int, P: int, lib=None) -> np.ndarray:
    """One rank's shard [B][Nl][H][D] -> its P send chunks [P][B][Nl][Hl][D]."""
    assert xs_r.dtype == np.uint16 and xs_r.ndim == 4
    B, Nl, H, D = xs_r.shape
    assert Nl == _dims(N, P)[0]
    if H % P:
        raise ValueError("the Ulysses degree must divide the head count")
    xs_r = np.ascontiguousarray(xs_r)
    out = np.empty((P, B, Nl, H // P, D), dtype=np.uint16)
    rc = (lib or _load()).sp_oracle_exchange_pack(xs_r.ctypes.data, out.ctypes.data, B, N, H, D, P)
    assert rc == 0
    return out


def exchange_unpack(recv: np.ndarray, N: int, H: int, lib=None) -> np.ndarray:
    """The P chunks returned to one rank [P][B][Nl][Hl][D] -> its shard [B][Nl][H][D]."""
    assert recv.dtype == np.uint16 and recv.ndim == 5
    P, B, Nl, Hl, D = recv.shape
    assert Nl == _dims(N, P)[0] and Hl * P == H
    recv = np.ascontiguousarray(recv)
    out = np.empty((B, Nl, H, D), dtype=np.uint16)
    rc = (lib or _load()).sp_oracle_exchange_unpack(recv.ctypes.data, out.ctypes.data, B, N, H, D, P)
    assert rc == 0
    return out


def attention_rows(q: np.ndarray, k: np.ndarray, v: np.ndarray,
                   rows: np.ndarray, scale: float = 0.0,
                   threads: Optional[int] = None, lib=None):
    """fp64 attention output and LSE for query rows (b, h, i).

    q, k, v: logical [B][N][H][D] bf16 bit patterns (uint16).
    rows: int64 array [R][3] of (b, h, i).
    Returns (O [R][D] float64, LSE [R] float64 natural log).
    """
    assert q.dtype == k.dtype == v.dtype == np.uint16
    assert q.shape == k.shape == v.shape and q.ndim == 4
    B, N, H, D = q.shape
    q, k, v = (np.ascontiguousarray(a) for a in (q, k, v))
    rows = np.ascontiguousarray(rows, dtype=np.int64).reshape(-1, 3)
    R = rows.shape[0]
    o = np.empty((R, D), dtype=np.float64)
    lse = np.empty(R, dtype=np.float64)
    if threads is None:
        threads = max(1, len(os.sched_getaffinity(0)))
    rc = (lib or _load()).sp_oracle_attention_rows(
        q.ctypes.data, k.ctypes.data, v.ctypes.data, B, N, H, D, float(scale),
        R, rows.ctypes.data, o.ctypes.data, lse.ctypes.data, int(threads))
    if rc != 0:
        raise RuntimeError(f"oracle attention failed ({rc})")
    return o, lse


def e4m3_value(byte: int, lib=None) -> float:
    """Exact value of one OCP E4M3 byte."""
    return float((lib or _load()).sp_oracle_e4m3_value(int(byte)))


def attention_rows_e4m3(q8, k8, v8, dq, dk, dv, rows, scale: float = 0.0,
                        threads: Optional[int] = None, block: int = 128, lib=None):
    """fp64 attention of e4m3 inputs (uint8 arrays, logical [B][N][H][D]).
    Element values are the exact e4m3 values times scale factors: Q and K
    element (b, t, h, c) take dq[b][h][t // block] and dk[b][h][t // block],
    V element (b, t, h, c) takes dv[b][h][c].  dq and dk broadcast to
    [B][H][ceil(N / block)] and dv to [B][H][D]; a [B][H] array gives one
    factor per (b, h).  Returns (O [R][D], LSE [R])."""
    for a in (q8, k8, v8):
        assert a.dtype == np.uint8 and a.shape == q8.shape and a.ndim == 4
    B, N, H, D = q8.shape
    nblk = -(-N // block)
    q8, k8, v8 = (np.ascontiguousarray(a) for a in (q8, k8, v8))

    def factors(d, last):
        d = np.asarray(d, dtype=np.float64)
        if d.ndim == 2:
            d = d[:, :, None]
        return np.ascontiguousarray(np.broadcast_to(d, (B, H, last)))

    dq, dk, dv = factors(dq, nblk), factors(dk, nblk), factors(dv, D)
    rows = np.ascontiguousarray(rows, dtype=np.int64).reshape(-1, 3)
    R = rows.shape[0]
    o = np.empty((R, D), dtype=np.float64)
    lse = np.empty(R, dtype=np.float64)
    if threads is None:
        threads = max(1, len(os.sched_getaffinity(0)))
    rc = (lib or _load()).sp_oracle_attention_rows_e4m3(
        q8.ctypes.data, k8.ctypes.data, v8.ctypes.data, dq.ctypes.data, dk.ctypes.data,
        dv.ctypes.data, int(block), B, N, H, D, float(scale), R, rows.ctypes.data,
        o.ctypes.data, lse.ctypes.data, int(threads))
    if rc != 0:
        raise RuntimeError(f"oracle attention failed ({rc})")
    return o, lse


def attention_rows_masked(q, k, v, mask, rows, scale: float = 0.0, cube: int = 64,
                          threads: Optional[int] = None, lib=None):
    """fp64 attention restricted by a block mask: query i of (b, h) attends
    key t only when mask[b][h][i // cube][t // cube] is non-zero (mask: bool
    or uint8 [B][H][ceil(N / cube)][ceil(N / cube)]).  A query that selects
    no key gets O = 0 and LSE = -inf.  Returns (O [R][D], LSE [R])."""
    for a in (q, k, v):
        assert a.dtype == np.uint16 and a.shape == q.shape and a.ndim == 4
    B, N, H, D = q.shape
    nc = -(-N // cube)
    mask = np.ascontiguousarray(np.asarray(mask).astype(np.uint8))
    assert mask.shape == (B, H, nc, nc), mask.shape
    q, k, v = (np.ascontiguousarray(a) for a in (q, k, v))
    rows = np.ascontiguousarray(rows, dtype=np.int64).reshape(-1, 3)
    R = rows.shape[0]
    o = np.empty((R, D), dtype=np.float64)
    lse = np.empty(R, dtype=np.float64)
    if threads is None:
        threads = max(1, len(os.sched_getaffinity(0)))
    rc = (lib or _load()).sp_oracle_attention_rows_masked(
        q.ctypes.data, k.ctypes.data, v.ctypes.data, mask.ctypes.data, int(cube), B, N, H, D,
        float(scale), R, rows.ctypes.data, o.ctypes.data, lse.ctypes.data, int(threads))
    if rc != 0:
        raise RuntimeError(f"oracle attention failed ({rc})")
    return o, lse


def linear_rows(x, w, bias, rows, threads: Optional[int] = None, lib=None):
    """fp64 linear layer on bf16 inputs for the requested rows:
    y[r][c] = sum_k x[rows[r]][k] * w[c][k] (+ bias[c]).  x: uint16 [M][K],
    w: uint16 [nout][K], bias: uint16 [nout] or None.  Returns [R][nout]."""
    assert x.dtype == np.uint16 and w.dtype == np.uint16 and x.ndim == 2 and w.ndim == 2
    M, K = x.shape
    nout, K2 = w.shape
    assert K2 == K
    x, w = np.ascontiguousarray(x), np.ascontiguousarray(w)
    if bias is not None:
        bias = np.ascontiguousarray(bias, dtype=np.uint16)
        assert bias.shape == (nout,)
    rows = np.ascontiguousarray(rows, dtype=np.int64).reshape(-1)
    y = np.empty((rows.size, nout), dtype=np.float64)
    if threads is None:
        threads = max(1, len(os.sched_getaffinity(0)))
    rc = (lib or _load()).sp_oracle_linear_rows(
        x.ctypes.data, w.ctypes.data, None if bias is None else bias.ctypes.data, M, K, nout,
        rows.size, rows.ctypes.data, y.ctypes.data, int(threads))
    if rc != 0:
        raise RuntimeError(f"oracle linear failed ({rc})")
    return y


def attention_full(q, k, v, scale: float = 0.0, threads: Optional[int] = None,
                   lib=None):
    """Every row of every (b, h); returns O [B][N][H][D] and LSE [B][H][N]."""
    B, N, H, D = q.shape
    b, h, i = np.meshgrid(np.arange(B), np.arange(H), np.arange(N), indexing="ij")
    rows = np.stack([b.ravel(), h.ravel(), i.ravel()], axis=1)
    o, lse = attention_rows(q, k, v, rows, scale, threads, lib)
    O = o.reshape(B, H, N, D).transpose(0, 2, 1, 3)
    return np.ascontiguousarray(O), lse.reshape(B, H, N)
