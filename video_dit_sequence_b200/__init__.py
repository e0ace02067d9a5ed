"""Ulysses sequence-parallel self-attention on one B200 (sm_100a).

Python binding of ``libsp.so`` (C ABI in ``include/sp.h``).  This module only
marshals arguments: every step of the path runs in the library's CUDA
kernels.  PyTorch supplies device memory and the current stream.  There is
no CPU or PyTorch fallback: without the built library, or without a CUDA
device, the calls raise.

The method (fal.ai, "Generate video with WAN 2.2 across four GPUs", section
"Splitting one generation across four GPUs"): P ranks each hold N/P tokens
of the sequence for all H heads; an all-to-all exchanges token shards for
head groups, each rank attends over all tokens for H/P heads, and the outputs
go back to the token owners.  With P virtual ranks on one GPU the exchange is
``pack`` / ``unpack``; ``attention_seqsharded`` fuses all three steps.

Layouts (bf16, contiguous):
  sequence-sharded  [P][B][Nl][H][D]    Nl = ceil(N/P)
  head-sharded      [P][B][Np][Hl][D]   Np = P*Nl, Hl = H/P
  lse (optional)    [B][H][Np] float32
"""
from __future__ import annotations

import ctypes
import dataclasses
import math
import os
from typing import Optional

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libsp.so")

SP_OK = 0
SP_ERR_NULL = 1
SP_ERR_SHAPE = 2
SP_ERR_HEADS_NOT_DIVISIBLE = 3
SP_ERR_ALIGN = 4
SP_ERR_UNSUPPORTED_D = 5
SP_ERR_CUDA = 6
SP_ERR_TIMEOUT = 7

EXPORTED = ("sp_padded_tokens", "sp_check_shape", "sp_pack", "sp_unpack",
            "sp_attention", "sp_attention_seqsharded", "sp_device_status",
            "sp_launch_count", "sp_status_str", "sp_selftest_wait_timeout",
            "sp_exchange_pack", "sp_exchange_unpack", "sp_attention_fp8_seqsharded",
            "sp_attention_ulysses_peer", "sp_ipc_export", "sp_ipc_open", "sp_ipc_close",
            "sp_attention_sparse_seqsharded", "sp_qkv_projection", "sp_out_projection",
            "sp_exchange_push", "sp_attention_ulysses_overlap", "sp_shard", "sp_unshard",
            "sp_copy_heads")


class sp_shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("N", ctypes.c_int32), ("H", ctypes.c_int32),
                ("D", ctypes.c_int32), ("P", ctypes.c_int32), ("scale", ctypes.c_float)]


class SpError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_str(status)} (status {status})")


_lib = None


def load(path: str = LIB_PATH):
    """Loads libsp.so (built by ``python -m video_dit_sequence_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(
            f"{path} is missing: build it with `python -m video_dit_sequence_b200.build`")
    lib = ctypes.CDLL(path)
    vp, sp_p = ctypes.c_void_p, ctypes.POINTER(sp_shape)
    lib.sp_padded_tokens.argtypes = [ctypes.c_int32, ctypes.c_int32]
    lib.sp_padded_tokens.restype = ctypes.c_int64
    lib.sp_check_shape.argtypes = [sp_p]
    lib.sp_check_shape.restype = ctypes.c_int
    for name in ("sp_pack", "sp_unpack", "sp_exchange_pack", "sp_exchange_unpack", "sp_shard",
                 "sp_unshard"):
        f = getattr(lib, name)
        f.argtypes = [vp, vp, sp_p, vp]
        f.restype = ctypes.c_int
    for name in ("sp_attention", "sp_attention_seqsharded"):
        f = getattr(lib, name)
        f.argtypes = [vp, vp, vp, vp, vp, sp_p, vp]
        f.restype = ctypes.c_int
    lib.sp_attention_fp8_seqsharded.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, sp_p, vp]
    lib.sp_attention_fp8_seqsharded.restype = ctypes.c_int
    lib.sp_qkv_projection.argtypes = [vp, vp, vp, vp, vp, vp, ctypes.c_int32, ctypes.c_int32,
                                      sp_p, vp]
    lib.sp_qkv_projection.restype = ctypes.c_int
    lib.sp_out_projection.argtypes = [vp, vp, vp, vp, ctypes.c_int32, ctypes.c_int32, sp_p, vp]
    lib.sp_out_projection.restype = ctypes.c_int
    lib.sp_attention_sparse_seqsharded.argtypes = [vp, vp, vp, vp, vp, vp, sp_p, vp]
    lib.sp_attention_sparse_seqsharded.restype = ctypes.c_int
    lib.sp_attention_ulysses_peer.argtypes = [
        ctypes.POINTER(vp), vp, vp, ctypes.POINTER(vp), vp, ctypes.c_int32, sp_p, vp]
    lib.sp_attention_ulysses_peer.restype = ctypes.c_int
    lib.sp_exchange_push.argtypes = [vp, vp, ctypes.POINTER(vp), ctypes.POINTER(vp),
                                     ctypes.POINTER(vp), ctypes.c_uint64, ctypes.c_int32, sp_p, vp]
    lib.sp_exchange_push.restype = ctypes.c_int
    lib.sp_attention_ulysses_overlap.argtypes = [
        ctypes.POINTER(vp), vp, vp, ctypes.POINTER(vp), vp, vp, ctypes.c_uint64, ctypes.c_uint64,
        ctypes.c_int32, sp_p, vp]
    lib.sp_attention_ulysses_overlap.restype = ctypes.c_int
    lib.sp_ipc_export.argtypes = [vp, vp, ctypes.POINTER(ctypes.c_int64)]
    lib.sp_ipc_export.restype = ctypes.c_int
    lib.sp_ipc_open.argtypes = [vp, ctypes.POINTER(vp)]
    lib.sp_ipc_open.restype = ctypes.c_int
    lib.sp_ipc_close.argtypes = [vp]
    lib.sp_ipc_close.restype = ctypes.c_int
    lib.sp_copy_heads.argtypes = [vp, ctypes.c_int32, ctypes.c_int32, vp, ctypes.c_int32,
                                  ctypes.c_int32, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32,
                                  vp]
    lib.sp_copy_heads.restype = ctypes.c_int
    lib.sp_device_status.argtypes = [vp]
    lib.sp_device_status.restype = ctypes.c_int
    lib.sp_selftest_wait_timeout.argtypes = [ctypes.c_uint64, vp]
    lib.sp_selftest_wait_timeout.restype = ctypes.c_int
    lib.sp_launch_count.argtypes = []
    lib.sp_launch_count.restype = ctypes.c_uint64
    lib.sp_status_str.argtypes = [ctypes.c_int]
    lib.sp_status_str.restype = ctypes.c_char_p
    _lib = lib
    return lib


def status_str(status: int) -> str:
    return load().sp_status_str(int(status)).decode()


FP8_BLOCK = 128  # tokens per Q/K scale block of the FP8 call (SP_FP8_BLOCK)


@dataclasses.dataclass(frozen=True)
class Shape:
    """Problem shape; scale <= 0 selects 1/sqrt(D)."""
    B: int
    N: int
    H: int
    D: int
    P: int
    scale: float = 0.0

    @property
    def Hl(self) -> int:
        return self.H // self.P

    @property
    def Nl(self) -> int:
        return -(-self.N // self.P)

    @property
    def Np(self) -> int:
        return self.Nl * self.P

    @property
    def seq_sharded(self):
        return (self.P, self.B, self.Nl, self.H, self.D)

    @property
    def head_sharded(self):
        return (self.P, self.B, self.Np, self.Hl, self.D)

    @property
    def rank_shard(self):
        """One rank's shard when every rank is its own GPU: [B][Nl][H][D]."""
        return (self.B, self.Nl, self.H, self.D)

    @property
    def send_chunks(self):
        """One rank's P exchange chunks: [P][B][Nl][Hl][D]."""
        return (self.P, self.B, self.Nl, self.Hl, self.D)

    def head_group(self) -> "Shape":
        """The problem one head group attends after the exchange: Hl heads
        over the whole sequence, still in P token shards."""
        return Shape(self.B, self.N, self.Hl, self.D, self.P, self.scale)

    @property
    def lse_shape(self):
        return (self.B, self.H, self.Np)

    @property
    def fp8_blocks(self) -> int:
        """Q/K scale blocks of the FP8 call: ceil(N / FP8_BLOCK)."""
        return -(-self.N // FP8_BLOCK)

    def c(self) -> sp_shape:
        return sp_shape(self.B, self.N, self.H, self.D, self.P, float(self.scale))


def padded_tokens(N: int, P: int) -> int:
    return int(load().sp_padded_tokens(N, P))


def check_shape(shape: Shape) -> int:
    """Returns the library's status code for a shape (0 = valid)."""
    s = shape.c()
    return int(load().sp_check_shape(ctypes.byref(s)))


def launch_count() -> int:
    return int(load().sp_launch_count())


# ---------------------------------------------------------------- tensors

def _torch():
    import torch
    return torch


def _ptr(t, shape, name, dtype=None):
    torch = _torch()
    if t is None:
        return None
    dtype = dtype or torch.bfloat16
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if tuple(t.shape) != tuple(shape) and t.numel() != math.prod(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream, device):
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream(device)
    elif stream.device != device:
        raise ValueError(f"stream is on {stream.device}, tensors on {device}")
    return ctypes.c_void_p(stream.cuda_stream)


def _resolve_device(stream, device):
    torch = _torch()
    if stream is not None:
        return stream.device
    d = torch.device(device) if device is not None else torch.device("cuda")
    return d if d.index is not None else torch.device("cuda", torch.cuda.current_device())


def _same_device(*tensors):
    """All operands must live on one CUDA device; the call runs with that
    device current (the library resolves its per-device state from it)."""
    torch = _torch()
    devs = {t.device for t in tensors if t is not None}
    if len(devs) != 1:
        raise ValueError(f"operands on several devices: {sorted(map(str, devs))}")
    dev = devs.pop()
    if dev.type != "cuda":
        raise TypeError("operands must be CUDA tensors")
    return torch.cuda.device(dev)


def _check(status: int, where: str):
    if status != SP_OK:
        raise SpError(status, where)


def shard(x, xs, shape: Shape, stream=None):
    """Logical [B][N][H][D] -> P token shards [P][B][Nl][H][D], padding slots
    zero (bit-exact)."""
    s = shape.c()
    with _same_device(x, xs):
        _check(load().sp_shard(_ptr(x, (shape.B, shape.N, shape.H, shape.D), "x"),
                               _ptr(xs, shape.seq_sharded, "xs"), ctypes.byref(s),
                               _stream(stream, x.device)), "sp_shard")


def unshard(xs, x, shape: Shape, stream=None):
    """P token shards [P][B][Nl][H][D] -> logical [B][N][H][D] (bit-exact)."""
    s = shape.c()
    with _same_device(xs, x):
        _check(load().sp_unshard(_ptr(xs, shape.seq_sharded, "xs"),
                                 _ptr(x, (shape.B, shape.N, shape.H, shape.D), "x"),
                                 ctypes.byref(s), _stream(stream, xs.device)), "sp_unshard")


def copy_heads(dst, dst_heads: int, dst_h0: int, src, src_heads: int, src_h0: int, rows: int,
               nh: int, D: int, stream=None):
    """dst[r][dst_h0 + h] = src[r][src_h0 + h] for rows r and heads h < nh
    (D bf16 elements per head): one strided copy between pinned host memory
    and the device, or within the device, enqueued on `stream`."""
    torch = _torch()
    ptrs, devs = [], set()
    for t, heads, name in ((dst, dst_heads, "dst"), (src, src_heads, "src")):
        if not isinstance(t, torch.Tensor) or t.dtype != torch.bfloat16:
            raise TypeError(f"{name} must be a bf16 tensor")
        if not t.is_contiguous() or t.numel() != rows * heads * D:
            raise ValueError(f"{name} must be contiguous with {rows} x {heads} x {D} elements")
        if t.is_cuda:
            devs.add(t.device)
        elif not t.is_pinned():
            raise ValueError(f"{name} is host memory that is not page-locked")
        ptrs.append(ctypes.c_void_p(t.data_ptr()))
    if len(devs) != 1:
        raise ValueError("copy_heads needs exactly one CUDA device among its tensors")
    dev = devs.pop()
    with torch.cuda.device(dev):
        _check(load().sp_copy_heads(ptrs[0], int(dst_heads), int(dst_h0), ptrs[1],
                                    int(src_heads), int(src_h0), int(rows), int(nh), int(D),
                                    _stream(stream, dev)), "sp_copy_heads")


def pack(xs, xh, shape: Shape, stream=None):
    """Sequence-sharded -> head-sharded (bit-exact permutation)."""
    s = shape.c()
    with _same_device(xs, xh):
        _check(load().sp_pack(_ptr(xs, shape.seq_sharded, "xs"), _ptr(xh, shape.head_sharded, "xh"),
                              ctypes.byref(s), _stream(stream, xs.device)), "sp_pack")


def unpack(oh, os_, shape: Shape, stream=None):
    """Head-sharded -> sequence-sharded (bit-exact permutation)."""
    s = shape.c()
    with _same_device(oh, os_):
        _check(load().sp_unpack(_ptr(oh, shape.head_sharded, "oh"), _ptr(os_, shape.seq_sharded, "os"),
                                ctypes.byref(s), _stream(stream, oh.device)), "sp_unpack")


def attention(qh, kh, vh, oh, shape: Shape, lse=None, stream=None):
    """Full-sequence attention per head group on head-sharded tensors."""
    torch = _torch()
    s = shape.c()
    hs = shape.head_sharded
    with _same_device(qh, kh, vh, oh, lse):
        _check(load().sp_attention(
            _ptr(qh, hs, "qh"), _ptr(kh, hs, "kh"), _ptr(vh, hs, "vh"), _ptr(oh, hs, "oh"),
            _ptr(lse, shape.lse_shape, "lse", torch.float32), ctypes.byref(s),
            _stream(stream, qh.device)), "sp_attention")


def attention_seqsharded(qs, ks, vs, os_, shape: Shape, lse=None, stream=None):
    """Fused pack + attention + unpack on sequence-sharded tensors."""
    torch = _torch()
    s = shape.c()
    ss = shape.seq_sharded
    with _same_device(qs, ks, vs, os_, lse):
        _check(load().sp_attention_seqsharded(
            _ptr(qs, ss, "qs"), _ptr(ks, ss, "ks"), _ptr(vs, ss, "vs"), _ptr(os_, ss, "os"),
            _ptr(lse, shape.lse_shape, "lse", torch.float32), ctypes.byref(s),
            _stream(stream, qs.device)), "sp_attention_seqsharded")


def attention_fp8_seqsharded(qs8, ks8, vs8, q_scale, k_scale, v_scale, os_, shape: Shape,
                             lse=None, stream=None):
    """FP8 (E4M3) variant of attention_seqsharded: qs8/ks8/vs8 are uint8
    [P][B][Nl][H][D] E4M3 bytes; q_scale and k_scale float32
    [B][H][shape.fp8_blocks] (one factor per block of FP8_BLOCK tokens),
    v_scale float32 [B][H][D] (one factor per channel); os_ bf16
    [P][B][Nl][H][D]."""
    torch = _torch()
    s = shape.c()
    ss = shape.seq_sharded
    blk = (shape.B, shape.H, shape.fp8_blocks)
    with _same_device(qs8, ks8, vs8, q_scale, k_scale, v_scale, os_, lse):
        _check(load().sp_attention_fp8_seqsharded(
            _ptr(qs8, ss, "qs8", torch.uint8), _ptr(ks8, ss, "ks8", torch.uint8),
            _ptr(vs8, ss, "vs8", torch.uint8),
            _ptr(q_scale, blk, "q_scale", torch.float32),
            _ptr(k_scale, blk, "k_scale", torch.float32),
            _ptr(v_scale, (shape.B, shape.H, shape.D), "v_scale", torch.float32),
            _ptr(os_, ss, "os"), _ptr(lse, shape.lse_shape, "lse", torch.float32),
            ctypes.byref(s), _stream(stream, qs8.device)), "sp_attention_fp8_seqsharded")


def exchange_pack(xs_r, send, shape: Shape, stream=None):
    """One rank's shard [B][Nl][H][D] -> its P send chunks [P][B][Nl][Hl][D]."""
    s = shape.c()
    with _same_device(xs_r, send):
        _check(load().sp_exchange_pack(_ptr(xs_r, shape.rank_shard, "xs_r"),
                                       _ptr(send, shape.send_chunks, "send"), ctypes.byref(s),
                                       _stream(stream, xs_r.device)), "sp_exchange_pack")


def exchange_unpack(recv, os_r, shape: Shape, stream=None):
    """The P chunks returned to one rank [P][B][Nl][Hl][D] -> its shard."""
    s = shape.c()
    with _same_device(recv, os_r):
        _check(load().sp_exchange_unpack(_ptr(recv, shape.send_chunks, "recv"),
                                         _ptr(os_r, shape.rank_shard, "os_r"), ctypes.byref(s),
                                         _stream(stream, recv.device)), "sp_exchange_unpack")


class UlyssesRank:
    """One rank of Ulysses attention when every rank is its own GPU (the
    form of fal.ai's "Splitting one generation across four GPUs").

    The step has three local phases around two all-to-alls:
      send_qkv(q, k, v)   shard [B][Nl][H][D] -> three [P][B][Nl][Hl][D]
                          chunk sets (sp_exchange_pack)
      -- all-to-all: chunk j of every rank to rank j, in rank order --
      attend(q, k, v)     this rank's head group over the whole sequence, on
                          the received rank-major shards (fused attention,
                          Hl heads, P token shards); the output is already
                          in chunk order for the way back
      -- all-to-all back --
      finish(back)        P returned chunks -> this rank's output shard
                          (sp_exchange_unpack)
    Keeping the phases apart lets the caller choose the exchange (NCCL over
    NVLink, or a copy between virtual ranks on one GPU).  The buffers a phase
    returns belong to this object and are reused by the next step: each
    step overwrites the previous step's results."""

    def __init__(self, shape: Shape):
        self.shape = shape
        self._bufs = {}

    def _buf(self, name, shape, like):
        torch = _torch()
        b = self._bufs.get(name)
        if b is None or b.device != like.device or b.dtype != like.dtype:
            b = self._bufs[name] = torch.empty(shape, dtype=like.dtype, device=like.device)
        return b

    def send_qkv(self, q, k, v, stream=None):
        out = []
        for name, x in (("send_q", q), ("send_k", k), ("send_v", v)):
            send = self._buf(name, self.shape.send_chunks, x)
            exchange_pack(x, send, self.shape, stream)
            out.append(send)
        return out

    def recv_buffers(self, like):
        """Three [P][B][Nl][Hl][D] buffers for the received Q, K, V chunks."""
        return [self._buf(n, self.shape.send_chunks, like) for n in ("recv_q", "recv_k", "recv_v")]

    def attend(self, q, k, v, lse=None, stream=None):
        o = self._buf("o", self.shape.send_chunks, q)
        attention_seqsharded(q, k, v, o, self.shape.head_group(), lse=lse, stream=stream)
        return o

    def finish(self, back, stream=None):
        out = self._buf("out", self.shape.rank_shard, back)
        exchange_unpack(back, out, self.shape, stream)
        return out

    def step(self, q, k, v, all_to_all):
        """The whole step with all_to_all(send, recv) filling recv: returns
        this rank's output shard (this object's buffer)."""
        recv = self.recv_buffers(q)
        for send, r in zip(self.send_qkv(q, k, v), recv):
            all_to_all(send, r)
        o = self.attend(*recv)
        back = self._buf("back", self.shape.send_chunks, o)
        all_to_all(o, back)
        return self.finish(back)


QKV_LAYOUTS = {"seq": 0, "head": 1, "send": 2}   # sp_qkv_layout


def qkv_projection(x, w, bias, q, k, v, shape: Shape, layout: str = "seq", stream=None):
    """The projection in front of attention (sp_qkv_projection), arguments in
    the C order: x the sequence-sharded hidden states [P][B][Nl][hidden] (one
    rank's [B][Nl][hidden] for layout "send"), w [3*H*D][hidden], bias
    [3*H*D] or None, all bf16; q, k, v receive the projection in `layout`:
    "seq" [P][B][Nl][H][D], "head" [P][B][Np][Hl][D] or "send"
    [P][B][Nl][Hl][D]."""
    torch = _torch()
    if layout not in QKV_LAYOUTS:
        raise ValueError(f"layout must be one of {sorted(QKV_LAYOUTS)}")
    hidden = int(w.shape[-1])
    rows = shape.rank_shard[:2] if layout == "send" else shape.seq_sharded[:3]
    out = {"seq": shape.seq_sharded, "head": shape.head_sharded, "send": shape.send_chunks}[layout]
    s = shape.c()
    with _same_device(x, w, bias, q, k, v):
        _check(load().sp_qkv_projection(
            _ptr(x, tuple(rows) + (hidden,), "x"), _ptr(w, (3 * shape.H * shape.D, hidden), "w"),
            _ptr(bias, (3 * shape.H * shape.D,), "bias"), _ptr(q, out, "q"), _ptr(k, out, "k"),
            _ptr(v, out, "v"), hidden, QKV_LAYOUTS[layout], ctypes.byref(s),
            _stream(stream, x.device)), "sp_qkv_projection")


O_LAYOUTS = {"seq": 0, "head": 1, "recv": 2}     # sp_o_layout


def out_projection(o, w, bias, y, shape: Shape, layout: str = "seq", stream=None):
    """The projection after attention (sp_out_projection), arguments in the C
    order: o the attention output in `layout` -- "seq" [P][B][Nl][H][D],
    "head" [P][B][Np][Hl][D] or "recv" one rank's P returned chunks
    [P][B][Nl][Hl][D] --, w [hidden][H*D], bias [hidden] or None, all bf16;
    y receives [P][B][Nl][hidden] (one rank's [B][Nl][hidden] for "recv")."""
    if layout not in O_LAYOUTS:
        raise ValueError(f"layout must be one of {sorted(O_LAYOUTS)}")
    hidden = int(w.shape[0])
    o_shape = {"seq": shape.seq_sharded, "head": shape.head_sharded,
               "recv": shape.send_chunks}[layout]
    rows = shape.rank_shard[:2] if layout == "recv" else shape.seq_sharded[:3]
    s = shape.c()
    with _same_device(o, w, bias, y):
        _check(load().sp_out_projection(
            _ptr(o, o_shape, "o"), _ptr(w, (hidden, shape.H * shape.D), "w"),
            _ptr(bias, (hidden,), "bias"), _ptr(y, tuple(rows) + (hidden,), "y"), hidden,
            O_LAYOUTS[layout], ctypes.byref(s), _stream(stream, o.device)), "sp_out_projection")


SPARSE_CUBE = 64         # SP_SPARSE_CUBE
SPARSE_MAX_CUBES = 8192  # SP_SPARSE_MAX_CUBES: ceil(N / SPARSE_CUBE) at most


def sparse_mask_words(mask):
    """A block mask as the sparse call takes it: mask is bool (or 0/1)
    [B][H][nc][nc] over cubes of SPARSE_CUBE tokens (mask[b][h][qc][kc]:
    query cube qc attends key cube kc); returns uint32 [B][H][nc][nwords]
    with bit kc % 32 of word kc // 32 set for a selected key cube."""
    import numpy as np
    m = np.asarray(mask).astype(bool)
    B, H, nc, nc2 = m.shape
    if nc != nc2:
        raise ValueError(f"mask must be square over cubes, got {m.shape}")
    nw = -(-nc // 32)
    padded = np.zeros((B, H, nc, nw * 32), dtype=bool)
    padded[..., :nc] = m
    bits = np.packbits(padded.reshape(B, H, nc, nw, 32), axis=-1, bitorder="little")
    return np.ascontiguousarray(bits.view(np.uint32).reshape(B, H, nc, nw))


def attention_sparse_seqsharded(qs, ks, vs, mask_words, os_, shape: Shape, lse=None,
                                stream=None):
    """Block-sparse fused attention: sequence-sharded bf16 qs/ks/vs/os_ as for
    attention_seqsharded, mask_words a CUDA int32/uint32 tensor
    [B][H][ncube][nwords] (sparse_mask_words); D = 128 and ncube = ceil(N / 64)
    <= SPARSE_MAX_CUBES."""
    torch = _torch()
    s = shape.c()
    ss = shape.seq_sharded
    nc = -(-shape.N // SPARSE_CUBE)
    mshape = (shape.B, shape.H, nc, -(-nc // 32))
    if not isinstance(mask_words, torch.Tensor) or mask_words.dtype not in (torch.int32,
                                                                            torch.uint32):
        raise TypeError("mask_words must be an int32 or uint32 CUDA tensor")
    with _same_device(qs, ks, vs, mask_words, os_, lse):
        _check(load().sp_attention_sparse_seqsharded(
            _ptr(qs, ss, "qs"), _ptr(ks, ss, "ks"), _ptr(vs, ss, "vs"),
            _ptr(mask_words, mshape, "mask_words", mask_words.dtype), _ptr(os_, ss, "os"),
            _ptr(lse, shape.lse_shape, "lse", torch.float32), ctypes.byref(s),
            _stream(stream, qs.device)), "sp_attention_sparse_seqsharded")


MAX_PEERS = 8            # SP_MAX_PEERS
IPC_HANDLE_BYTES = 64    # SP_IPC_HANDLE_BYTES


def attention_ulysses_peer(q_shards, k_group, v_group, o_shards, shape: Shape, rank: int,
                           lse=None, stream=None):
    """One rank's step of the multi-GPU form with the Q and O exchanges fused
    into the kernel (sp_attention_ulysses_peer).  q_shards / o_shards: P
    entries in rank order, each a CUDA tensor [B][Nl][H][D] bf16 or an int
    device address valid in this process (a peer buffer from ipc_open).
    k_group / v_group: this rank's received head group [P][B][Nl][Hl][D];
    lse: [B][Hl][Np] float32 or None."""
    torch = _torch()
    P = shape.P
    if len(q_shards) != P or len(o_shards) != P:
        raise ValueError(f"need {P} Q and {P} O shard addresses")
    local = [x for x in (*q_shards, *o_shards) if not isinstance(x, int)]

    def addr(x, name):
        return x if isinstance(x, int) else _ptr(x, shape.rank_shard, name).value

    qa = (ctypes.c_void_p * P)(*[addr(x, f"q_shards[{r}]") for r, x in enumerate(q_shards)])
    oa = (ctypes.c_void_p * P)(*[addr(x, f"o_shards[{r}]") for r, x in enumerate(o_shards)])
    s = shape.c()
    group = shape.send_chunks
    with _same_device(k_group, v_group, lse, *local):
        _check(load().sp_attention_ulysses_peer(
            qa, _ptr(k_group, group, "k_group"), _ptr(v_group, group, "v_group"), oa,
            _ptr(lse, (shape.B, shape.Hl, shape.Np), "lse", torch.float32), int(rank),
            ctypes.byref(s), _stream(stream, k_group.device)), "sp_attention_ulysses_peer")


def _require_ipc_exportable():
    """CUDA IPC exports allocations made by cudaMalloc.  With PyTorch's
    expandable_segments option, its caching allocator maps memory with
    cuMemCreate instead, and the export fails; say so before trying."""
    for var in ("PYTORCH_CUDA_ALLOC_CONF", "PYTORCH_ALLOC_CONF"):
        conf = os.environ.get(var, "").replace(" ", "").lower()
        if "expandable_segments:true" in conf:
            raise RuntimeError(
                f"{var} enables expandable_segments: CUDA IPC cannot export those "
                "allocations; unset it for the peer exchange")


def _addr_array(xs, shape_, name):
    """ctypes array of device addresses: CUDA tensors (checked against
    shape_) or ints (peer addresses valid in this process)."""
    def addr(x, i):
        if isinstance(x, int):
            return x
        if shape_ is None:
            if not isinstance(x, _torch().Tensor) or not x.is_cuda:
                raise TypeError(f"{name}[{i}] must be a CUDA tensor or an address")
            return x.data_ptr()
        return _ptr(x, shape_, f"{name}[{i}]").value
    return (ctypes.c_void_p * len(xs))(*[addr(x, i) for i, x in enumerate(xs)])


def exchange_push(k, v, k_groups, v_groups, counts, epoch: int, shape: Shape, rank: int,
                  stream=None):
    """One rank's K/V exchange over peer memory (sp_exchange_push): k, v this
    rank's shards [B][Nl][H][D]; k_groups / v_groups / counts: P entries in
    rank order, each a CUDA tensor or a peer address (ipc_open) -- every
    rank's received groups [P][B][Nl][Hl][D] bf16 and arrival counters
    int64 [P]; epoch: the step number (>= 1)."""
    torch = _torch()
    P = shape.P
    if not (len(k_groups) == len(v_groups) == len(counts) == P):
        raise ValueError(f"need {P} entries per address list")
    local = [x for x in (*k_groups, *v_groups, *counts) if not isinstance(x, int)]
    s = shape.c()
    with _same_device(k, v, *local):
        _check(load().sp_exchange_push(
            _ptr(k, shape.rank_shard, "k"), _ptr(v, shape.rank_shard, "v"),
            _addr_array(k_groups, shape.send_chunks, "k_groups"),
            _addr_array(v_groups, shape.send_chunks, "v_groups"),
            _addr_array(counts, None, "counts"), int(epoch), int(rank), ctypes.byref(s),
            _stream(stream, k.device)), "sp_exchange_push")


def attention_ulysses_overlap(q_shards, k_group, v_group, o_shards, counts, epoch: int,
                              shape: Shape, rank: int, lse=None, wait_ns: int = 0, stream=None):
    """The peer step while K/V chunks arrive (sp_attention_ulysses_overlap):
    as attention_ulysses_peer, and counts is this rank's arrival counters
    (int64 [P], CUDA tensor) for step `epoch`."""
    torch = _torch()
    P = shape.P
    if len(q_shards) != P or len(o_shards) != P:
        raise ValueError(f"need {P} Q and {P} O shard addresses")
    local = [x for x in (*q_shards, *o_shards) if not isinstance(x, int)]
    s = shape.c()
    group = shape.send_chunks
    with _same_device(k_group, v_group, counts, lse, *local):
        _check(load().sp_attention_ulysses_overlap(
            _addr_array(q_shards, shape.rank_shard, "q_shards"), _ptr(k_group, group, "k_group"),
            _ptr(v_group, group, "v_group"), _addr_array(o_shards, shape.rank_shard, "o_shards"),
            _ptr(lse, (shape.B, shape.Hl, shape.Np), "lse", torch.float32),
            _ptr(counts, (P,), "counts", torch.int64), int(epoch), int(wait_ns), int(rank),
            ctypes.byref(s), _stream(stream, k_group.device)), "sp_attention_ulysses_overlap")


def ipc_export(t):
    """(handle, offset): the CUDA IPC handle (bytes) of the allocation that
    holds CUDA tensor t, and t's byte offset from that allocation's base."""
    torch = _torch()
    h = (ctypes.c_uint8 * IPC_HANDLE_BYTES)()
    off = ctypes.c_int64()
    with torch.cuda.device(t.device):
        _check(load().sp_ipc_export(ctypes.c_void_p(t.data_ptr()), h, ctypes.byref(off)),
               "sp_ipc_export")
    return bytes(h), off.value


def ipc_open(handle: bytes) -> int:
    """Maps another process's exported allocation on the current device;
    returns its base address in this process (unmap with ipc_close)."""
    buf = (ctypes.c_uint8 * IPC_HANDLE_BYTES).from_buffer_copy(handle)
    base = ctypes.c_void_p()
    _check(load().sp_ipc_open(buf, ctypes.byref(base)), "sp_ipc_open")
    return int(base.value)


def ipc_close(base: int):
    _check(load().sp_ipc_close(ctypes.c_void_p(base)), "sp_ipc_close")


class CudaPeerBackend:
    """Memory and kernels of UlyssesPeerRank on a GPU: buffers from torch's
    allocator, peers' buffers mapped through CUDA IPC (each allocation once),
    the exchange reorder and the peer step of this library."""

    def __init__(self, device):
        torch = _torch()
        self.device = torch.device(device)
        self._opened = {}

    def empty(self, shape, dtype=None):
        torch = _torch()
        return torch.empty(shape, dtype=dtype or torch.bfloat16, device=self.device)

    def zeros(self, shape, dtype=None):
        """Zeroed and complete on the device before any peer can see it."""
        torch = _torch()
        t = torch.zeros(shape, dtype=dtype or torch.bfloat16, device=self.device)
        torch.cuda.synchronize(self.device)
        return t

    def export(self, t):
        _require_ipc_exportable()
        return ipc_export(t)

    def open(self, handle: bytes, offset: int):
        torch = _torch()
        if handle not in self._opened:
            with torch.cuda.device(self.device):
                self._opened[handle] = ipc_open(handle)
        return self._opened[handle] + offset

    @staticmethod
    def part(x, i: int, shape: Shape):
        """Sub-buffer i of an exported [2][B][Nl][H][D] buffer: a tensor index
        for this rank's own buffer, a byte offset for a mapped peer's."""
        if isinstance(x, int):
            return x + i * 2 * math.prod(shape.rank_shard)
        return x[i]

    def exchange_pack(self, x, send, shape: Shape):
        exchange_pack(x, send, shape)

    def peer_step(self, q_addrs, k_group, v_group, o_addrs, rank: int, shape: Shape):
        attention_ulysses_peer(q_addrs, k_group, v_group, o_addrs, shape, rank)

    def push(self, k, v, k_addrs, v_addrs, count_addrs, epoch: int, rank: int, shape: Shape):
        exchange_push(k, v, k_addrs, v_addrs, count_addrs, epoch, shape, rank)

    def overlap_step(self, q_addrs, k_group, v_group, o_addrs, counts, epoch: int, rank: int,
                     shape: Shape):
        attention_ulysses_overlap(q_addrs, k_group, v_group, o_addrs, counts, epoch, shape, rank)

    def close(self):
        torch = _torch()
        with torch.cuda.device(self.device):
            for base in self._opened.values():
                ipc_close(base)
        self._opened.clear()


class UlyssesPeerRank:
    """One rank of the multi-GPU form with the exchanges fused into the
    kernels.

    Construction allocates this rank's Q shard and output shard
    ([B][Nl][H][D] each, one buffer) and, with kv_exchange="push" (the
    default), its received K and V groups ([P][B][Nl][Hl][D] each, one
    buffer) and its arrival counters (int64 [P], zeroed); it exports them,
    gathers every rank's exports over the process group and maps the peers'
    buffers (each once), so that every rank holds all ranks' addresses in rank
    order.  step(k, v, q) then
      writes q into the Q shard (or the caller wrote it);
      push: stores k and v straight into every rank's received groups over
        peer memory (sp_exchange_push), and runs the attention step that
        waits for each chunk as it arrives (sp_attention_ulysses_overlap):
        Q tiles read from the ranks that hold them, O rows stored into the
        ranks that own them;
      nccl: reorders k and v into send chunks (sp_exchange_pack), exchanges
        them with an all-to-all, then runs the peer step
        (sp_attention_ulysses_peer);
      and ends with a one-element all-reduce.
    A rank's Q write precedes its push (or its all-to-all) in its stream, so
    a peer that has seen the chunk has seen the Q shard; the closing
    all-reduce follows every rank's kernel, so when it completes here every
    row of this rank's output shard has been written and no peer still reads
    a buffer the next step overwrites.  The returned output shard stays valid
    until the next step.  step(..., release_after=event) makes the closing
    all-reduce also wait (on the current stream) for that CUDA event: peers
    write this rank's output shard in the next step only after it, so a copy
    of the previous output that the event marks is safe (StepPipeline)."""

    def __init__(self, shape: Shape, group=None, backend=None, device=None,
                 kv_exchange: str = "push"):
        import torch.distributed as dist
        torch = _torch()
        if kv_exchange not in ("push", "nccl"):
            raise ValueError("kv_exchange must be 'push' or 'nccl'")
        self.shape, self.group, self.kv_exchange = shape, group, kv_exchange
        self.rank = dist.get_rank(group)
        if dist.get_world_size(group) != shape.P:
            raise ValueError(f"group of {dist.get_world_size(group)} ranks, shape has P = {shape.P}")
        if shape.P > MAX_PEERS:
            raise ValueError(f"P = {shape.P} > {MAX_PEERS}")
        if backend is None:
            backend = CudaPeerBackend(device if device is not None else torch.cuda.current_device())
        self.backend = be = backend
        self._qo = be.empty((2,) + tuple(shape.rank_shard))     # [Q shard, O shard]
        self.q_shard, self.o_shard = self._qo[0], self._qo[1]
        self._flag = be.empty((1,), torch.float32)
        self.epoch = 0
        push = kv_exchange == "push"
        if push:
            self._kv = be.empty((2,) + tuple(shape.send_chunks))  # [K group, V group]
            self.counts = be.zeros((shape.P,), torch.int64)
            mine = (be.export(self._qo), be.export(self._kv), be.export(self.counts))
        else:
            self._k_send, self._v_send, self._k_recv, self._v_recv = (
                be.empty(shape.send_chunks) for _ in range(4))
            mine = (be.export(self._qo),)
        table = [None] * shape.P
        dist.all_gather_object(table, mine, group=group)
        self.q_addrs, self.o_addrs = [], []
        self.k_addrs, self.v_addrs, self.count_addrs = [], [], []
        for r, exported in enumerate(table):
            own = r == self.rank
            qo = self._qo if own else be.open(*exported[0])
            self.q_addrs.append(be.part(qo, 0, shape))
            self.o_addrs.append(be.part(qo, 1, shape))
            if push:
                kv = self._kv if own else be.open(*exported[1])
                self.k_addrs.append(be.part(kv, 0, shape))
                self.v_addrs.append(be.part(kv, 1, shape))
                self.count_addrs.append(self.counts if own else be.open(*exported[2]))

    def step(self, k, v, q=None, release_after=None):
        import torch.distributed as dist
        be, s = self.backend, self.shape
        if q is not None:
            self.q_shard.copy_(q)
        self.epoch += 1
        if self.kv_exchange == "push":
            be.push(k, v, self.k_addrs, self.v_addrs, self.count_addrs, self.epoch, self.rank, s)
            be.overlap_step(self.q_addrs, self._kv[0], self._kv[1], self.o_addrs, self.counts,
                            self.epoch, self.rank, s)
        else:
            be.exchange_pack(k, self._k_send, s)
            be.exchange_pack(v, self._v_send, s)
            dist.all_to_all_single(self._k_recv, self._k_send, group=self.group)
            dist.all_to_all_single(self._v_recv, self._v_send, group=self.group)
            be.peer_step(self.q_addrs, self._k_recv, self._v_recv, self.o_addrs, self.rank, s)
        if release_after is not None:
            _torch().cuda.current_stream(self._flag.device).wait_event(release_after)
        self._flag.zero_()
        dist.all_reduce(self._flag, group=self.group)
        return self.o_shard

    def close(self):
        """Unmaps the peers' buffers; returns once every rank has done so, so
        that no rank frees a buffer another rank still maps."""
        import torch.distributed as dist
        self.backend.close()
        dist.barrier(group=self.group)


def nccl_all_to_all(group=None):
    """Exchange through torch.distributed: chunk j of this rank's [P][...]
    buffer goes to rank j; the result holds every rank's chunk in rank order.
    exchange(send, recv=None) fills recv (a new buffer when None) and
    returns it."""
    import torch.distributed as dist

    def exchange(send, recv=None):
        torch = _torch()
        if recv is None:
            recv = torch.empty_like(send)
        dist.all_to_all_single(recv, send, group=group)
        return recv
    return exchange


def ulysses_attention_distributed(q, k, v, shape: Shape, all_to_all=None, rank=None):
    """One rank's Ulysses attention step: q, k, v are this rank's shards
    [B][Nl][H][D] (rank = position in the group of shape.P ranks); returns
    the output shard.  all_to_all defaults to NCCL over the default group.
    Pass the same UlyssesRank as `rank` on every step to reuse its buffers
    (the returned shard is then overwritten by the next step)."""
    all_to_all = all_to_all or nccl_all_to_all()
    rank = rank or UlyssesRank(shape)
    return rank.step(q, k, v, all_to_all)


class StepPipeline:
    """Steps on host-resident inputs with the transfers hidden behind the
    compute, for any step function: one GPU's fused attention (HostPipeline)
    or one rank's step of the multi-GPU forms (UlyssesRank, UlyssesPeerRank).

    inputs: per buffer set, the device tensors a step reads (depth =
    len(inputs)).  step(k, tensors, previous_out_left) enqueues the step on
    the current stream (the pipeline's compute stream) for buffer set k and
    returns its device output: a buffer of its own that stays valid until the
    next step on the same set, or a fresh tensor; previous_out_left is the
    CUDA event that marks the previous step's output as copied back (None for
    the first), which a step whose output buffers other ranks write passes on
    (UlyssesPeerRank's release_after).  submit(host_inputs, host_output)
    copies the pinned host tensors into the next set on an H2D stream, runs
    the step once they have arrived, and copies its output into host_output
    on a D2H stream.  A set is reused only after its last output has left, so
    step i+1's inputs travel while step i computes and step i's output
    travels while step i+1 computes.  Nothing here synchronises the host;
    synchronize() waits for everything submitted.  Collectives inside the
    step run on the compute stream, in submission order on every rank.

    head_groups G > 1 runs every step as G problems of H/G heads, which
    attention allows because heads are independent: the host tensors hold
    rows of H heads of D elements ([..][H][D], bf16), each input of a set is
    [G][..][H/G][D] (one part per group), and group g's H/G heads are copied
    in (sp_copy_heads), stepped, and copied out while the next group's copy
    and step run.  Only one group's transfers then lie outside the compute of
    a run of steps.  The step is called with k = set * G + g on group g's
    parts, so it can keep state (a rank object, say) per set and group; its
    output is [..][H/G][D].  Every rank calls the groups in the same order."""

    def __init__(self, inputs, step, device=None, head_groups: int = 1):
        torch = _torch()
        self.inputs = [tuple(t) for t in inputs]
        self.step = step
        self.device = torch.device(device or self.inputs[0][0].device)
        self.h2d = torch.cuda.Stream(self.device)
        self.compute = torch.cuda.Stream(self.device)
        self.d2h = torch.cuda.Stream(self.device)
        self.head_groups = int(head_groups)
        if self.head_groups < 1:
            raise ValueError("head_groups must be at least 1")
        if self.head_groups > 1:
            for t in (x for st in self.inputs for x in st):
                if t.dim() < 3 or t.shape[0] != self.head_groups:
                    raise ValueError(f"grouped inputs are [{self.head_groups}][..][H/G][D], "
                                     f"got {tuple(t.shape)}")
        # per set and group: the event that marks its last output as copied back
        self.freed = [[None] * self.head_groups for _ in self.inputs]
        self.last_out_left = None
        self.count = 0

    def submit(self, host_inputs, host_output):
        torch = _torch()
        i = self.count % len(self.inputs)
        self.count += 1
        dev = self.inputs[i]
        if len(host_inputs) != len(dev):
            raise ValueError(f"{len(host_inputs)} host inputs for {len(dev)} device buffers")
        G = self.head_groups
        for g in range(G):
            if self.freed[i][g] is not None:
                self.h2d.wait_event(self.freed[i][g])
            parts = tuple(d[g] for d in dev) if G > 1 else dev
            with torch.cuda.stream(self.h2d):
                for d, h in zip(parts, host_inputs):
                    if G > 1:
                        hg, D = d.shape[-2], d.shape[-1]
                        copy_heads(d, hg, 0, h, G * hg, g * hg, d.numel() // (hg * D), hg, D,
                                   stream=self.h2d)
                    else:
                        d.copy_(h, non_blocking=True)
            arrived = torch.cuda.Event()
            arrived.record(self.h2d)
            self.compute.wait_event(arrived)
            with torch.cuda.stream(self.compute):
                out = self.step(i * G + g, parts, self.last_out_left)
            done = torch.cuda.Event()
            done.record(self.compute)
            self.d2h.wait_event(done)
            with torch.cuda.stream(self.d2h):
                if G > 1:
                    hg, D = out.shape[-2], out.shape[-1]
                    copy_heads(host_output, G * hg, g * hg, out, hg, 0, out.numel() // (hg * D),
                               hg, D, stream=self.d2h)
                else:
                    host_output.copy_(out, non_blocking=True)
            out.record_stream(self.d2h)   # a fresh output stays allocated until it has left
            left = torch.cuda.Event()
            left.record(self.d2h)
            self.freed[i][g] = self.last_out_left = left
        return self.last_out_left

    def synchronize(self):
        """Waits for everything submitted, then checks the device status word
        (raises SpError when a kernel gave up on a bounded wait)."""
        for st in (self.h2d, self.compute, self.d2h):
            st.synchronize()
        _check(device_status(self.compute), "StepPipeline")


def pipeline_head_groups(shape: Shape, sms: int = 148, max_groups: int = 8, gpus: int = 1) -> int:
    """Head groups per step for a StepPipeline: the largest G <= max_groups
    with P | H/G whose G calls of H/G heads run no more waves than one call
    over all H heads.  The attention kernel keeps one CTA on each of `sms` SMs
    and launches ceil(Np/256) * B CTAs per head; each of `gpus` GPUs attends
    1/gpus of a call's heads (1 for the one-GPU fused call, P for one rank's
    step of the multi-GPU form)."""
    per_head = -(-shape.Np // 256) * shape.B
    one = -(-(shape.H // gpus) * per_head // sms)
    best = 1
    for g in range(2, max_groups + 1):
        if shape.H % g == 0 and (shape.H // g) % shape.P == 0 and \
                g * -(-(shape.H // g // gpus) * per_head // sms) <= one:
            best = g
    return best


class HostPipeline(StepPipeline):
    """Fused attention on host-resident problems, with the transfers hidden
    behind the compute (a StepPipeline over sp_attention_seqsharded).

    submit(hq, hk, hv, ho) takes pinned host tensors in the sequence-sharded
    layout ([P][B][Nl][H][D] bf16) and enqueues, on three streams: the copy of
    the inputs into one of `depth` device buffer sets, the fused attention on
    that set, and the copy of the output back into `ho`.  A step runs as
    `head_groups` problems of H/G heads (P | H/G; default
    pipeline_head_groups), each group's output bit-identical to the same
    heads of one call over all H."""

    def __init__(self, shape: Shape, device=None, depth: int = 2, head_groups: int = 0):
        torch = _torch()
        self.shape = shape
        dev = torch.device(device or "cuda")
        if dev.index is None:
            dev = torch.device("cuda", torch.cuda.current_device())
        g = int(head_groups) or pipeline_head_groups(
            shape, torch.cuda.get_device_properties(dev).multi_processor_count)
        if g < 1 or shape.H % g or (shape.H // g) % shape.P:
            raise ValueError(f"{g} head groups: need G | H and P | H/G "
                             f"(H = {shape.H}, P = {shape.P})")
        gshape = Shape(shape.B, shape.N, shape.H // g, shape.D, shape.P, shape.scale)
        self.group_shape = gshape
        part = ((g,) if g > 1 else ()) + gshape.seq_sharded
        sets = [tuple(torch.empty(part, dtype=torch.bfloat16, device=dev) for _ in range(4))
                for _ in range(depth)]
        self._outs = [st[3] for st in sets]

        def fused(k, t, _left):
            o = self._outs[k // g]
            o = o[k % g] if g > 1 else o
            attention_seqsharded(t[0], t[1], t[2], o, gshape,
                                 stream=torch.cuda.current_stream(dev))
            return o
        super().__init__([st[:3] for st in sets], fused, dev, head_groups=g)

    def submit(self, hq, hk, hv, ho):
        return super().submit((hq, hk, hv), ho)


def device_status(stream=None, device=None) -> int:
    """Synchronises the stream and returns (and clears) the status word of
    the stream's device."""
    torch = _torch()
    dev = _resolve_device(stream, device)
    with torch.cuda.device(dev):
        return int(load().sp_device_status(_stream(stream, dev)))


def selftest_wait_timeout(limit_ns: int, stream=None, device=None):
    """Enqueues a kernel whose bounded wait must run out (see sp.h)."""
    torch = _torch()
    dev = _resolve_device(stream, device)
    with torch.cuda.device(dev):
        _check(load().sp_selftest_wait_timeout(int(limit_ns), _stream(stream, dev)),
               "sp_selftest_wait_timeout")


def ulysses_attention(q, k, v, P: int, scale: float = 0.0, fused: bool = True):
    """User-level call: q, k, v are [B, N, H, D] bf16 CUDA tensors (logical,
    unsharded, contiguous); returns O [B, N, H, D].  The tensors are laid out
    as P sequence shards (sp_shard, zero-padded to Np tokens), attended with
    P virtual ranks and read back (sp_unshard).  fused=False runs pack ->
    attention -> unpack instead of the fused kernel."""
    torch = _torch()
    B, N, H, D = q.shape
    shape = Shape(B, N, H, D, P, scale)
    ss = shape.seq_sharded

    def shards(x):
        xs = torch.empty(ss, dtype=x.dtype, device=x.device)
        shard(x, xs, shape)
        return xs

    qs, ks, vs = shards(q), shards(k), shards(v)
    os_ = torch.empty_like(qs)
    if fused:
        attention_seqsharded(qs, ks, vs, os_, shape)
    else:
        hs = shape.head_sharded
        qh, kh, vh, oh = (torch.empty(hs, dtype=q.dtype, device=q.device) for _ in range(4))
        pack(qs, qh, shape)
        pack(ks, kh, shape)
        pack(vs, vh, shape)
        attention(qh, kh, vh, oh, shape)
        unpack(oh, os_, shape)
    out = torch.empty_like(q)
    unshard(os_, out, shape)
    return out
