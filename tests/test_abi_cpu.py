"""The C-ABI library on a machine without a GPU: it loads, exports every
symbol include/sp.h declares, and its host-side checks reject bad arguments
before anything is enqueued (no compute call is made here)."""
import ctypes
import json
import os
import re

import pytest

import video_dit_sequence_b200 as sp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from video_dit_sequence_b200 import build
    build.build()
    return sp.load()


def declared_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(sp_[a-z0-9_]+)\s*\(", text))
    return names


def test_exports_every_declared_symbol(lib):
    names = declared_symbols()
    assert names >= {"sp_pack", "sp_unpack", "sp_attention", "sp_attention_seqsharded"}
    for n in names:
        assert hasattr(lib, n), n
    assert set(sp.EXPORTED) == names


def test_padded_tokens(lib):
    assert sp.padded_tokens(75600, 4) == 75600
    assert sp.padded_tokens(75601, 8) == 75608
    assert sp.padded_tokens(75601, 2) == 75602
    assert sp.padded_tokens(1024, 2) == 1024
    assert sp.padded_tokens(0, 2) == -1 and sp.padded_tokens(5, 0) == -1


def test_degree_rule_golden(lib):
    with open(os.path.join(ROOT, "tests", "golden", "degree_rule.json")) as f:
        g = json.load(f)
    for c in g["valid"]:
        assert sp.check_shape(sp.Shape(1, 4096, c["heads"], 128, c["degree"])) == sp.SP_OK
        assert sp.Shape(1, 4096, c["heads"], 128, c["degree"]).Hl == c["heads_per_rank"]
    for c in g["invalid"]:
        assert sp.check_shape(sp.Shape(1, 4096, c["heads"], 128, c["degree"])) == \
            sp.SP_ERR_HEADS_NOT_DIVISIBLE


def test_shape_errors(lib):
    ok = sp.Shape(1, 75600, 40, 128, 4)
    assert sp.check_shape(ok) == sp.SP_OK
    assert sp.check_shape(sp.Shape(1, 0, 40, 128, 4)) == sp.SP_ERR_SHAPE
    assert sp.check_shape(sp.Shape(0, 10, 40, 128, 4)) == sp.SP_ERR_SHAPE
    assert sp.check_shape(sp.Shape(1, 10, 40, 96, 4)) == sp.SP_ERR_UNSUPPORTED_D
    assert sp.check_shape(sp.Shape(1, 10, 40, 64, 3)) == sp.SP_ERR_HEADS_NOT_DIVISIBLE
    assert lib.sp_check_shape(None) == sp.SP_ERR_NULL
    # largest problem: a tensor's 16-byte vectors are indexed below 2^31
    assert sp.check_shape(sp.Shape(1, 2 ** 21 - 1, 64, 128, 1)) == sp.SP_OK
    assert sp.check_shape(sp.Shape(1, 2 ** 21, 64, 128, 1)) == sp.SP_ERR_SHAPE
    assert sp.check_shape(sp.Shape(1, 2 ** 21 - 7, 64, 128, 8)) == sp.SP_ERR_SHAPE  # padded
    assert sp.check_shape(sp.Shape(65536, 16, 8, 64, 1)) == sp.SP_ERR_SHAPE
    for code in range(8):
        assert isinstance(sp.status_str(code), str) and sp.status_str(code)


def _call(fn, *ptrs, shape):
    s = shape.c()
    return fn(*[ctypes.c_void_p(p) if p else None for p in ptrs], ctypes.byref(s), None)


def test_argument_errors_return_before_launch(lib):
    """Fake device addresses are only checked, never touched: every one of
    these calls must return its error without reaching the GPU."""
    shape = sp.Shape(1, 1024, 4, 64, 2)
    A, B_ = 0x10000, 0x20000
    assert _call(lib.sp_pack, 0, B_, shape=shape) == sp.SP_ERR_NULL
    assert _call(lib.sp_unpack, A, 0, shape=shape) == sp.SP_ERR_NULL
    assert _call(lib.sp_pack, A + 8, B_, shape=shape) == sp.SP_ERR_ALIGN
    assert _call(lib.sp_unpack, A, B_ + 2, shape=shape) == sp.SP_ERR_ALIGN
    bad = sp.Shape(1, 1024, 6, 64, 4)
    assert _call(lib.sp_pack, A, B_, shape=bad) == sp.SP_ERR_HEADS_NOT_DIVISIBLE
    s = shape.c()
    att = lambda fn, q, k, v, o, lse=None, shp=shape: fn(
        *[ctypes.c_void_p(x) if x else None for x in (q, k, v, o, lse)],
        ctypes.byref(shp.c()), None)
    for fn in (lib.sp_attention, lib.sp_attention_seqsharded):
        assert att(fn, A, A, 0, B_) == sp.SP_ERR_NULL
        assert att(fn, A, A, A + 4, B_) == sp.SP_ERR_ALIGN
        assert att(fn, A, A, A, B_, 0x30002) == sp.SP_ERR_ALIGN
        assert att(fn, A, A, A, B_, shp=sp.Shape(1, 1024, 4, 80, 2)) == sp.SP_ERR_UNSUPPORTED_D
    # heads are split only by the head-sharded call; the fused call shards
    # tokens alone and accepts any degree
    assert att(lib.sp_attention, A, A, A, B_, shp=sp.Shape(1, 1024, 4, 64, 3)) == \
        sp.SP_ERR_HEADS_NOT_DIVISIBLE
    assert lib.sp_check_shape(ctypes.byref(sp.Shape(1, 1024, 4, 64, 3).c())) == \
        sp.SP_ERR_HEADS_NOT_DIVISIBLE
    f8 = lambda q, k, v, dq, dk, dv, o, lse=None, shp=sp.Shape(1, 1024, 4, 128, 2): \
        lib.sp_attention_fp8_seqsharded(
            *[ctypes.c_void_p(x) if x else None for x in (q, k, v, dq, dk, dv, o, lse)],
            ctypes.byref(shp.c()), None)
    C = 0x40000
    assert f8(A, A, A, C, C, 0, B_) == sp.SP_ERR_NULL          # each factor array required
    assert f8(A, A, A, 0, C, C, B_) == sp.SP_ERR_NULL
    assert f8(A, A, A, C, 0, C, B_) == sp.SP_ERR_NULL
    assert f8(A, A, A, C, C + 2, C, B_) == sp.SP_ERR_ALIGN      # fp32 factors, 4-byte aligned
    assert f8(A, A, A + 8, C, C, C, B_) == sp.SP_ERR_ALIGN
    assert f8(A, A, A, C, C, C, B_, shp=sp.Shape(1, 1024, 4, 64, 2)) == sp.SP_ERR_UNSUPPORTED_D
    # the peer step: host arrays of P device addresses, D = 128, P <= 8
    def peer(qs, k, v, os_, rank, shp):
        arr = lambda xs: None if xs is None else (ctypes.c_void_p * len(xs))(*xs)
        return lib.sp_attention_ulysses_peer(arr(qs), ctypes.c_void_p(k) if k else None,
                                             ctypes.c_void_p(v) if v else None, arr(os_), None,
                                             rank, ctypes.byref(shp.c()), None)
    s4 = sp.Shape(1, 1000, 8, 128, 4)
    ok_q, ok_o = [A + 0x1000 * r for r in range(4)], [B_ + 0x1000 * r for r in range(4)]
    assert peer(None, A, A, ok_o, 0, s4) == sp.SP_ERR_NULL
    assert peer(ok_q, A, 0, ok_o, 0, s4) == sp.SP_ERR_NULL
    assert peer(ok_q[:3] + [0], A, A, ok_o, 0, s4) == sp.SP_ERR_NULL
    assert peer(ok_q, A, A, ok_o[:3] + [B_ + 8], 0, s4) == sp.SP_ERR_ALIGN
    assert peer(ok_q, A, A + 2, ok_o, 0, s4) == sp.SP_ERR_ALIGN
    assert peer(ok_q, A, A, ok_o, 4, s4) == sp.SP_ERR_SHAPE
    assert peer(ok_q, A, A, ok_o, -1, s4) == sp.SP_ERR_SHAPE
    assert peer(ok_q, A, A, ok_o, 0, sp.Shape(1, 1000, 8, 64, 4)) == sp.SP_ERR_UNSUPPORTED_D
    assert peer(ok_q, A, A, ok_o, 0, sp.Shape(1, 1000, 6, 128, 4)) == \
        sp.SP_ERR_HEADS_NOT_DIVISIBLE
    assert peer(ok_q * 4, A, A, ok_o * 4, 0, sp.Shape(1, 1000, 16, 128, 16)) == sp.SP_ERR_SHAPE
    sparse = lambda m, shp=sp.Shape(1, 1000, 4, 128, 2): lib.sp_attention_sparse_seqsharded(
        ctypes.c_void_p(A), ctypes.c_void_p(A), ctypes.c_void_p(A),
        ctypes.c_void_p(m) if m else None, ctypes.c_void_p(B_), None, ctypes.byref(shp.c()), None)
    assert sparse(0) == sp.SP_ERR_NULL
    assert sparse(C + 2) == sp.SP_ERR_ALIGN
    assert sparse(C, sp.Shape(1, 1000, 4, 64, 2)) == sp.SP_ERR_UNSUPPORTED_D
    big = sp.Shape(1, sp.SPARSE_CUBE * sp.SPARSE_MAX_CUBES + 1, 1, 128, 1)   # one cube too many
    assert sparse(C, big) == sp.SP_ERR_SHAPE
    proj = lambda x, w, b, q, k, v, hidden, layout, shp=sp.Shape(1, 1000, 4, 128, 2): \
        lib.sp_qkv_projection(*[ctypes.c_void_p(t) if t else None for t in (x, w, b, q, k, v)],
                              hidden, layout, ctypes.byref(shp.c()), None)
    assert proj(A, A, 0, B_, B_, 0, 512, 0) == sp.SP_ERR_NULL
    assert proj(A, A, 0, B_, B_, B_ + 8, 512, 0) == sp.SP_ERR_ALIGN
    assert proj(A, A, C + 1, B_, B_, B_, 512, 0) == sp.SP_ERR_ALIGN          # bf16 bias
    assert proj(A, A, 0, B_, B_, B_, 500, 0) == sp.SP_ERR_SHAPE              # hidden % 8
    assert proj(A, A, 0, B_, B_, B_, 512, 3) == sp.SP_ERR_SHAPE              # no such layout
    assert proj(A, A, 0, B_, B_, B_, 512, 1, sp.Shape(1, 1000, 6, 128, 4)) == \
        sp.SP_ERR_HEADS_NOT_DIVISIBLE
    assert proj(A, A, 0, B_, B_, B_, 512, 0, sp.Shape(1, 1000, 6, 96, 4)) == \
        sp.SP_ERR_UNSUPPORTED_D
    oproj = lambda o, w, b, y, hidden, layout, shp=sp.Shape(1, 1000, 4, 128, 2): \
        lib.sp_out_projection(*[ctypes.c_void_p(t) if t else None for t in (o, w, b, y)],
                              hidden, layout, ctypes.byref(shp.c()), None)
    assert oproj(0, A, 0, B_, 512, 0) == sp.SP_ERR_NULL
    assert oproj(A, 0, 0, B_, 512, 0) == sp.SP_ERR_NULL
    assert oproj(A, A, 0, 0, 512, 0) == sp.SP_ERR_NULL
    assert oproj(A + 8, A, 0, B_, 512, 0) == sp.SP_ERR_ALIGN
    assert oproj(A, A, C + 1, B_, 512, 0) == sp.SP_ERR_ALIGN                 # bf16 bias
    assert oproj(A, A, 0, B_, 500, 0) == sp.SP_ERR_SHAPE                     # hidden % 8
    assert oproj(A, A, 0, B_, 512, 3) == sp.SP_ERR_SHAPE                     # no such layout
    assert oproj(A, A, 0, B_, 512, -1) == sp.SP_ERR_SHAPE
    assert oproj(A, A, 0, B_, 512, 2, sp.Shape(1, 1000, 6, 128, 4)) == \
        sp.SP_ERR_HEADS_NOT_DIVISIBLE
    assert oproj(A, A, 0, B_, 512, 0, sp.Shape(1, 1000, 6, 96, 4)) == sp.SP_ERR_UNSUPPORTED_D
    # the overlapped form: push of K/V into every rank's groups, the step that
    # waits for them
    arr = lambda xs: None if xs is None else (ctypes.c_void_p * len(xs))(*xs)
    grp = [A + 0x1000 * r for r in range(4)]
    cnt = [C + 0x100 * r for r in range(4)]
    push = lambda k, v, kg, vg, cn, epoch, rank, shp=s4: lib.sp_exchange_push(
        ctypes.c_void_p(k) if k else None, ctypes.c_void_p(v) if v else None, arr(kg), arr(vg),
        arr(cn), epoch, rank, ctypes.byref(shp.c()), None)
    assert push(0, A, grp, grp, cnt, 1, 0) == sp.SP_ERR_NULL
    assert push(A, A, None, grp, cnt, 1, 0) == sp.SP_ERR_NULL
    assert push(A, A, grp, grp, None, 1, 0) == sp.SP_ERR_NULL
    assert push(A, A, grp[:3] + [0], grp, cnt, 1, 0) == sp.SP_ERR_NULL
    assert push(A + 8, A, grp, grp, cnt, 1, 0) == sp.SP_ERR_ALIGN
    assert push(A, A, grp, grp[:3] + [A + 8], cnt, 1, 0) == sp.SP_ERR_ALIGN
    assert push(A, A, grp, grp, cnt[:3] + [C + 4], 1, 0) == sp.SP_ERR_ALIGN   # 8-byte counters
    assert push(A, A, grp, grp, cnt, 0, 0) == sp.SP_ERR_SHAPE                  # epoch >= 1
    assert push(A, A, grp, grp, cnt, 1, 4) == sp.SP_ERR_SHAPE
    assert push(A, A, grp, grp, cnt, 1, 0, sp.Shape(1, 1000, 6, 128, 4)) == \
        sp.SP_ERR_HEADS_NOT_DIVISIBLE
    assert push(A * 1, A, grp * 4, grp * 4, cnt * 4, 1, 0, sp.Shape(1, 1000, 16, 128, 16)) == \
        sp.SP_ERR_SHAPE
    over = lambda qs, k, v, os_, cn, epoch, rank, shp=s4: lib.sp_attention_ulysses_overlap(
        arr(qs), ctypes.c_void_p(k) if k else None, ctypes.c_void_p(v) if v else None, arr(os_),
        None, ctypes.c_void_p(cn) if cn else None, epoch, 0, rank, ctypes.byref(shp.c()), None)
    assert over(ok_q, A, A, ok_o, 0, 1, 0) == sp.SP_ERR_NULL
    assert over(ok_q, A, A, ok_o, C + 4, 1, 0) == sp.SP_ERR_ALIGN
    assert over(ok_q, A, A, ok_o, C, 0, 0) == sp.SP_ERR_SHAPE
    assert over(ok_q, A, A, ok_o, C, 1, 4) == sp.SP_ERR_SHAPE
    assert over(ok_q, A, A + 2, ok_o, C, 1, 0) == sp.SP_ERR_ALIGN
    assert over(ok_q, A, A, ok_o, C, 1, 0, sp.Shape(1, 1000, 8, 64, 4)) == sp.SP_ERR_UNSUPPORTED_D
    h = (ctypes.c_uint8 * sp.IPC_HANDLE_BYTES)()
    off = ctypes.c_int64()
    base = ctypes.c_void_p()
    assert lib.sp_ipc_export(None, h, ctypes.byref(off)) == sp.SP_ERR_NULL
    assert lib.sp_ipc_export(ctypes.c_void_p(A), None, ctypes.byref(off)) == sp.SP_ERR_NULL
    assert lib.sp_ipc_open(None, ctypes.byref(base)) == sp.SP_ERR_NULL
    assert lib.sp_ipc_open(h, None) == sp.SP_ERR_NULL
    assert lib.sp_ipc_close(None) == sp.SP_ERR_NULL
    for fn in (lib.sp_shard, lib.sp_unshard):
        assert _call(fn, 0, B_, shape=shape) == sp.SP_ERR_NULL
        assert _call(fn, A + 8, B_, shape=shape) == sp.SP_ERR_ALIGN
        assert _call(fn, A, B_, shape=sp.Shape(1, 1024, 4, 80, 2)) == sp.SP_ERR_UNSUPPORTED_D
    for fn in (lib.sp_exchange_pack, lib.sp_exchange_unpack):
        assert _call(fn, 0, B_, shape=shape) == sp.SP_ERR_NULL
        assert _call(fn, A + 8, B_, shape=shape) == sp.SP_ERR_ALIGN
        assert _call(fn, A, B_, shape=bad) == sp.SP_ERR_HEADS_NOT_DIVISIBLE
    vp = ctypes.c_void_p
    cp = lambda d, dh, d0, s, sh, s0, rows, nh, D: lib.sp_copy_heads(
        vp(d) if d else None, dh, d0, vp(s) if s else None, sh, s0, rows, nh, D, None)
    assert cp(0, 8, 0, A, 40, 0, 10, 8, 128) == sp.SP_ERR_NULL
    assert cp(A, 8, 0, 0, 40, 0, 10, 8, 128) == sp.SP_ERR_NULL
    assert cp(A, 8, 1, B_, 40, 0, 10, 8, 128) == sp.SP_ERR_SHAPE     # past the dst row
    assert cp(A, 8, 0, B_, 40, 33, 10, 8, 128) == sp.SP_ERR_SHAPE    # past the src row
    assert cp(A, 8, -1, B_, 40, 0, 10, 8, 128) == sp.SP_ERR_SHAPE
    assert cp(A, 8, 0, B_, 40, 0, -1, 8, 128) == sp.SP_ERR_SHAPE
    assert cp(A, 8, 0, B_, 40, 0, 10, 0, 128) == sp.SP_ERR_SHAPE
    assert cp(A, 8, 0, B_, 40, 0, 10, 8, 0) == sp.SP_ERR_SHAPE
    assert cp(A, 1 << 23, 0, B_, 40, 0, 10, 8, 128) == sp.SP_ERR_SHAPE  # a 2 GiB row
    assert cp(A, 8, 0, B_, 40, 32, 0, 8, 128) == sp.SP_OK           # no rows: nothing enqueued
    assert lib.sp_launch_count() == 0


def test_pipeline_head_groups():
    """HostPipeline's head groups: P divides every group, and the groups'
    calls launch no more waves of 148 CTAs than one call over all heads."""
    g = sp.pipeline_head_groups
    assert g(sp.Shape(1, 75600, 40, 128, 4)) == 5      # 8 heads a group, 16 waves each
    assert g(sp.Shape(1, 32760, 12, 128, 2)) == 1      # 11 waves: any split adds one
    assert g(sp.Shape(1, 124992, 48, 128, 8)) == 3
    assert g(sp.Shape(1, 1000, 7, 64, 7)) == 1
    # one rank's step of the multi-GPU form attends H/P heads on its GPU
    assert g(sp.Shape(1, 75600, 40, 128, 8), gpus=8) == 5    # 1 head a rank, 2 waves each
    assert g(sp.Shape(1, 75600, 40, 128, 4), gpus=4) == 5
    for H, P, N, B in ((40, 4, 75600, 1), (24, 2, 4096, 2), (16, 1, 65536, 1), (64, 8, 99999, 1)):
        shp = sp.Shape(B, N, H, 128, P)
        G = g(shp)
        assert 1 <= G <= 8 and H % G == 0 and (H // G) % P == 0
        per_head = -(-shp.Np // 256) * B
        assert G * -(-(H // G) * per_head // 148) <= -(-H * per_head // 148)


def test_binding_refuses_cpu_tensors(lib):
    torch = pytest.importorskip("torch")
    shape = sp.Shape(1, 16, 2, 64, 2)
    x = torch.zeros(shape.seq_sharded, dtype=torch.bfloat16)
    with pytest.raises(TypeError):
        sp.pack(x, x, shape)


def test_binding_refuses_mixed_devices(lib):
    torch = pytest.importorskip("torch")
    shape = sp.Shape(1, 16, 2, 64, 2)
    a = torch.zeros(shape.seq_sharded, dtype=torch.bfloat16)
    b = torch.zeros(shape.head_sharded, dtype=torch.bfloat16, device="meta")
    with pytest.raises((ValueError, TypeError)):
        sp.pack(a, b, shape)


def test_header_is_plain_c_and_links(lib, tmp_path):
    """include/sp.h compiles as strict C99 and a C program links against
    libsp.so and calls its host-only entry points: the boundary needs no C++,
    Python or torch."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not available")
    src = tmp_path / "abi.c"
    src.write_text(r"""
#include <stdio.h>
#include "sp.h"
int main(void) {
  sp_shape ok = {1, 75601, 40, 128, 8, 0.0f};
  sp_shape bad = {1, 1000, 40, 128, 3, 0.0f};
  printf("%d %d ", SP_SPARSE_CUBE, SP_SPARSE_MAX_CUBES);
  printf("%lld %d %d %s\n", (long long)sp_padded_tokens(75601, 8), (int)sp_check_shape(&ok),
         (int)sp_check_shape(&bad), sp_status_str(SP_ERR_HEADS_NOT_DIVISIBLE));
  return 0;
}
""")
    exe = tmp_path / "abi"
    libdir = os.path.join(ROOT, "video_dit_sequence_b200")
    r = subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                        "-I", os.path.join(ROOT, "include"), "-o", str(exe), str(src),
                        "-L", libdir, "-lsp", f"-Wl,-rpath,{libdir}"],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, out.stderr
    cube, max_cubes, padded, st_ok, st_bad, text = out.stdout.split(" ", 5)
    assert (int(cube), int(max_cubes)) == (sp.SPARSE_CUBE, sp.SPARSE_MAX_CUBES)
    assert int(padded) == 75608 and int(st_ok) == sp.SP_OK
    assert int(st_bad) == sp.SP_ERR_HEADS_NOT_DIVISIBLE and text.strip()
