"""Seeded synthetic inputs for the Ulysses sequence-parallel attention path.

This package draws the Q/K/V tensors, the outlier key rows and the sampled
query rows that both the CUDA path and the fp64 oracle consume.  It holds
none of the method's arithmetic: no attention, no pack, no unpack.  It also
lays a logical ``[B][N][H][D]`` tensor out as the P per-rank shards that the
sequence-parallel ranks hold (``to_seq_shards``), which is the input format of
the path, and reads such shards back (``from_seq_shards``).

Workload shapes follow the video-DiT latent grids of the configurations the
path is measured on (``CONFIGS``): 480p and 720p frames at 81 frames as in the
fal.ai page "Generate video with WAN 2.2 across four GPUs" (resolution table
and the frame-count rule of its Input model), 40 attention heads with 10 per
rank at degree 4 ("Splitting one generation across four GPUs"), and a long
clip grid.  Values are i.i.d. N(0,1), rounded once to bf16.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
import subprocess
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB_PATH = os.path.join(_HERE, "libsynth.so")
_lib = None

TID_Q, TID_K, TID_V, TID_OUTLIER, TID_ROWS = 0, 1, 2, 3, 4


def build(force: bool = False) -> str:
    """Compiles synth.c into libsynth.so next to it (gcc, -O2, pthreads)."""
    if force or not os.path.exists(_LIB_PATH) or (
            os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-pthread",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        lib.synth_normal_bf16.argtypes = [
            ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint64, ctypes.c_int64,
            ctypes.c_double, ctypes.c_void_p, ctypes.c_int]
        lib.synth_normal_bf16.restype = None
        lib.synth_stream_out.argtypes = [ctypes.c_uint64] * 3
        lib.synth_stream_out.restype = ctypes.c_uint64
        lib.synth_normal_f64.argtypes = [ctypes.c_uint64] * 3
        lib.synth_normal_f64.restype = ctypes.c_double
        _lib = lib
    return _lib


def host_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)))


@dataclasses.dataclass(frozen=True)
class Shape:
    """One problem: batch B, true tokens N, heads H, head dim D, degree P."""
    B: int
    N: int
    H: int
    D: int
    P: int

    @property
    def Hl(self) -> int:
        return self.H // self.P

    @property
    def Nl(self) -> int:
        return -(-self.N // self.P)

    @property
    def Np(self) -> int:
        return self.Nl * self.P

    def flops(self) -> float:
        """Algorithmic attention FLOPs, 4*B*N^2*H*D (non-causal, true N)."""
        return 4.0 * self.B * self.N * self.N * self.H * self.D

    def shard_elems(self) -> int:
        return self.P * self.B * self.Nl * self.H * self.D


@dataclasses.dataclass(frozen=True)
class Config:
    name: str
    shape: Shape
    seed: int
    k_mul: float = 1.0            # K sample scaled before the bf16 rounding
    k_outlier_frac: float = 0.0   # fraction of K token rows scaled by 8
    grid: Tuple[int, int, int] = (0, 0, 0)


CONFIGS: Dict[str, Config] = {
    "tiny": Config("tiny", Shape(1, 1024, 4, 64, 2), seed=1, grid=(4, 16, 16)),
    "480p": Config("480p", Shape(1, 32760, 12, 128, 2), seed=2, k_mul=1.5,
                   grid=(21, 30, 52)),
    "720p": Config("720p", Shape(1, 75600, 40, 128, 4), seed=3,
                   grid=(21, 45, 80)),
    "1344x768": Config("1344x768", Shape(1, 124992, 40, 128, 8), seed=4,
                       k_outlier_frac=0.001, grid=(31, 48, 84)),
}
SWEEP_N = (4096, 32760, 75600, 75601)
SWEEP_P = (1, 2, 4, 8)
SWEEP_SEED = 5


def sweep_config(N: int, P: int) -> Config:
    return Config(f"sweep-N{N}-P{P}", Shape(1, N, 40, 128, P), seed=SWEEP_SEED)


def normal_bf16(seed: int, tid: int, e0: int, count: int, mul: float = 1.0,
                out: Optional[np.ndarray] = None,
                threads: Optional[int] = None) -> np.ndarray:
    """bf16 bit patterns (uint16) of elements e0..e0+count-1 of stream tid."""
    if out is None:
        out = np.empty(count, dtype=np.uint16)
    assert out.dtype == np.uint16 and out.flags.c_contiguous and out.size == count
    _load().synth_normal_bf16(seed, tid, e0, count, float(mul),
                              out.ctypes.data, threads or host_threads())
    return out


def stream_u64(seed: int, tid: int, idx: Sequence[int]) -> np.ndarray:
    lib = _load()
    return np.array([lib.synth_stream_out(seed, tid, int(i)) for i in idx],
                    dtype=np.uint64)


def _stream_u64_range(seed: int, tid: int, n: int) -> np.ndarray:
    """Outputs 0..n-1 of the SplitMix64 stream for (seed, tid), vectorised in
    numpy with the same constants as synth.c."""
    g = np.uint64(0x9E3779B97F4A7C15)

    def mix(z):
        z = (z ^ (z >> np.uint64(30))) * np.uint64(0xBF58476D1CE4E5B9)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(0x94D049BB133111EB)
        return z ^ (z >> np.uint64(31))

    with np.errstate(over="ignore"):
        key = mix(np.uint64(seed) * g + np.uint64((tid << 1) + 1))
        i = np.arange(1, n + 1, dtype=np.uint64)
        return mix(key + i * g)


def outlier_rows(cfg: Config) -> np.ndarray:
    """Token indices whose K rows are scaled by 8: round(frac*N) tokens,
    the ones with the smallest hash of the (seed, outlier) stream, i.e. a
    seeded sample without replacement.  Sorted ascending."""
    n = cfg.shape.N
    cnt = int(round(cfg.k_outlier_frac * n))
    if cnt == 0:
        return np.zeros(0, dtype=np.int64)
    h = _stream_u64_range(cfg.seed, TID_OUTLIER, n)
    order = np.lexsort((np.arange(n), h))
    return np.sort(order[:cnt]).astype(np.int64)


def logical_tensor(cfg: Config, tid: int, threads: Optional[int] = None) -> np.ndarray:
    """Logical [B][N][H][D] bf16 bits (uint16) of tensor tid (Q, K or V)."""
    s = cfg.shape
    count = s.B * s.N * s.H * s.D
    mul = cfg.k_mul if tid == TID_K else 1.0
    x = normal_bf16(cfg.seed, tid, 0, count, mul, threads=threads)
    x = x.reshape(s.B, s.N, s.H, s.D)
    if tid == TID_K and cfg.k_outlier_frac > 0:
        rows = outlier_rows(cfg)
        # x8 is exact in bf16 (exponent +3) for every finite normal value here.
        f = bf16_to_f32(x[:, rows])
        x[:, rows] = f32_to_bf16(f * np.float32(8.0))
    return x


def qkv_logical(cfg: Config, threads: Optional[int] = None):
    return tuple(logical_tensor(cfg, t, threads) for t in (TID_Q, TID_K, TID_V))


def to_seq_shards(x: np.ndarray, P: int) -> np.ndarray:
    """Logical [B][N][H][D] -> per-rank shards [P][B][Nl][H][D]; rank r holds
    tokens r*Nl .. r*Nl+Nl-1; token slots >= N are zero."""
    B, N, H, D = x.shape
    Nl = -(-N // P)
    Np = Nl * P
    if B == 1 and Np == N:
        return x.reshape(P, 1, Nl, H, D)
    padded = np.zeros((B, Np, H, D), dtype=x.dtype)
    padded[:, :N] = x
    return np.ascontiguousarray(
        padded.reshape(B, P, Nl, H, D).transpose(1, 0, 2, 3, 4))


def from_seq_shards(xs: np.ndarray, N: int) -> np.ndarray:
    """Inverse of to_seq_shards: [P][B][Nl][H][D] -> logical [B][N][H][D]."""
    P, B, Nl, H, D = xs.shape
    return np.ascontiguousarray(
        xs.transpose(1, 0, 2, 3, 4).reshape(B, P * Nl, H, D)[:, :N])


def sampled_rows(cfg: Config, per_head: int = 256,
                 extra_P: Sequence[int] = ()) -> np.ndarray:
    """Query rows checked on large problems: `per_head` distinct rows drawn
    by seed, always including 0, N-1 and every shard boundary r*Nl-1, r*Nl
    (r = 1..P-1) for the config's P and for each P in extra_P."""
    s = cfg.shape
    must = {0, s.N - 1}
    for P in (s.P, *extra_P):
        Nl = -(-s.N // P)
        for r in range(1, P):
            for t in (r * Nl - 1, r * Nl):
                if 0 <= t < s.N:
                    must.add(t)
    if per_head >= s.N:
        return np.arange(s.N, dtype=np.int64)
    h = _stream_u64_range(cfg.seed, TID_ROWS, s.N)
    order = np.lexsort((np.arange(s.N), h))
    rows: List[int] = sorted(must)
    chosen = set(rows)
    for t in order:
        if len(rows) >= per_head:
            break
        if int(t) not in chosen:
            rows.append(int(t))
            chosen.add(int(t))
    return np.array(sorted(rows), dtype=np.int64)


def bf16_to_f32(x: np.ndarray) -> np.ndarray:
    return (x.astype(np.uint32) << np.uint32(16)).view(np.float32)


def f32_to_bf16(f: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even narrowing of finite fp32 values to bf16 bits."""
    u = np.ascontiguousarray(f, dtype=np.float32).view(np.uint32)
    u = u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return (u >> np.uint32(16)).astype(np.uint16)


E4M3_MAX = 448.0


def to_e4m3(x: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even narrowing of fp32 values (|x| <= 448) to OCP
    E4M3 bytes (torch's float8_e4m3fn conversion)."""
    import torch
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(
        torch.float8_e4m3fn).view(torch.uint8).numpy()


SPARSE_CUBE = 64   # tokens per cube of a block-sparse mask


def cube_mask(cfg: Config, density: float = 0.2, group: int = 4, seed: int = 0):
    """A seeded block mask for the block-sparse call: over cubes of 64 tokens,
    each query cube selects key cubes independently with probability
    `density`, and each `group` consecutive query cubes share one selection
    (a spatially coherent pattern, as neighbouring video cubes tend to pick
    similar key cubes).  The pages give a sparsity (0.8) and the cube size but
    no selection rule; this pattern is a synthetic stand-in.  Returns bool
    [B][H][nc][nc]."""
    s = cfg.shape
    nc = -(-s.N // SPARSE_CUBE)
    rng = np.random.default_rng([cfg.seed, seed, 64])
    base = rng.random((s.B, s.H, -(-nc // group), nc)) < density
    return np.ascontiguousarray(np.repeat(base, group, axis=2)[:, :, :nc])


def attended_pairs(mask: np.ndarray, N: int) -> float:
    """(query, key) pairs a cube mask selects over N tokens, summed over
    batches and heads."""
    nc = mask.shape[-1]
    sizes = np.full(nc, SPARSE_CUBE, dtype=np.float64)
    sizes[-1] = N - SPARSE_CUBE * (nc - 1)
    return float(np.einsum("bhqk,q,k->", mask.astype(np.float64), sizes, sizes))


FP8_BLOCK = 128   # tokens per Q/K scale block of the 8-bit inputs


def fp8_qkv(cfg: Config, threads: Optional[int] = None, block: int = FP8_BLOCK):
    """8-bit inputs for the FP8 variant: the config's bf16 Q, K, V scaled so
    that each scale group's largest magnitude maps to 448, then rounded to
    E4M3.  Q and K have one factor per (batch, head, block of `block`
    tokens), V one per (batch, head, channel).  Returns q8, k8, v8 (logical
    [B][N][H][D] uint8) and the factors dq, dk [B][H][ceil(N / block)] and
    dv [B][H][D] (float32; element value = e4m3 value * factor)."""
    q, k, v = (bf16_to_f32(x) for x in qkv_logical(cfg, threads))
    B, N, H, D = q.shape
    nblk = -(-N // block)

    def factor(amax):
        return np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)

    def per_block(x):
        pad = np.zeros((B, nblk * block, H, D), dtype=np.float32)
        pad[:, :N] = np.abs(x)
        amax = pad.reshape(B, nblk, block, H, D).max(axis=(2, 4))    # [B][nblk][H]
        d = factor(amax.transpose(0, 2, 1))                           # [B][H][nblk]
        tok = np.arange(N) // block
        return to_e4m3(x / d.transpose(0, 2, 1)[:, tok, :, None]), np.ascontiguousarray(d)

    q8, dq = per_block(q)
    k8, dk = per_block(k)
    dv = factor(np.abs(v).max(axis=1))                                # [B][H][D]
    v8 = to_e4m3(v / dv[:, None, :, :])
    return q8, k8, v8, dq, dk, np.ascontiguousarray(dv)
