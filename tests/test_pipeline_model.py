"""StepPipeline's stream protocol, run on the CPU (no GPU).

StepPipeline (and HostPipeline on top of it) issues, per step and head group,
an H2D copy, the step and a D2H copy on three CUDA streams, ordered only by
events.  This test runs the real StepPipeline.submit with the streams, events
and sp_copy_heads replaced by recording fakes, then executes the recorded
stream programs in random interleavings that respect stream order and event
waits, tracking what every buffer holds.  It checks that
  * every step reads exactly its own inputs (none overwritten by a later
    step's H2D copy before the step ran);
  * every host output receives exactly its own step's result (no output
    buffer overwritten before its copy back);
for whole steps and for head groups, and that a pipeline whose H2D stream
ignores its waits is caught.
"""
import contextlib
import random

import pytest

torch = pytest.importorskip("torch")

import video_dit_sequence_b200 as sp


class FakeEvent:
    def __init__(self, *args, **kwargs):
        self.stream = None
        self.index = None

    def record(self, stream):
        self.stream = stream
        self.index = len(stream.ops)
        stream.ops.append(("mark", self))


class FakeStream:
    ignore_waits = False

    def __init__(self, device=None):
        self.ops = []

    def wait_event(self, ev):
        if not self.ignore_waits:
            self.ops.append(("wait", ev))


class Recorder:
    """Fakes for torch.cuda's streams and events and for sp.copy_heads."""

    def __init__(self):
        self.current = None

    @contextlib.contextmanager
    def stream(self, s):
        prev, self.current = self.current, s
        try:
            yield
        finally:
            self.current = prev

    def copy_heads(self, dst, dst_heads, dst_h0, src, src_heads, src_h0, rows, nh, D,
                   stream=None):
        # a region is (buffer, first head): the part a group's copy touches
        stream.ops.append(("copy", (dst.data_ptr(), dst_h0), (src.data_ptr(), src_h0)))


def execute(streams, mem, rng):
    """Runs the recorded programs; each step op checks and writes `mem`."""
    pos = {id(s): 0 for s in streams}
    done_marks = set()
    while True:
        ready = []
        for s in streams:
            i = pos[id(s)]
            if i == len(s.ops):
                continue
            op = s.ops[i]
            if op[0] == "wait" and op[1].index is not None and id(op[1]) not in done_marks:
                continue
            ready.append(s)
        if not ready:
            break
        s = rng.choice(ready)
        op = s.ops[pos[id(s)]]
        pos[id(s)] += 1
        if op[0] == "mark":
            done_marks.add(id(op[1]))
        elif op[0] == "copy":
            mem[op[1]] = mem.get(op[2])
        elif op[0] == "step":
            _, reads, want, write, tag = op
            for r, w in zip(reads, want):
                assert mem.get(r) == w, ("step read", tag, mem.get(r), w)
            mem[write] = tag
    assert all(pos[id(s)] == len(s.ops) for s in streams), "a stream never finished"


def run_pipeline(rng, depth, groups, steps, ignore_h2d_waits=False):
    rec = Recorder()
    rows, hg, D = 4, 2, 8
    H = groups * hg
    made = []

    def make_stream(device=None):
        s = FakeStream(device)
        made.append(s)
        return s

    inputs = [tuple(torch.empty((groups, rows, hg, D), dtype=torch.bfloat16) for _ in range(3))
              for _ in range(depth)]
    outs = {}                       # (set, group) -> device output buffer
    calls = []

    def step(k, tensors, left):
        g = k % groups
        o = outs.setdefault(k, torch.empty((rows, hg, D), dtype=torch.bfloat16))
        n = calls[-1]
        s = rec.current
        reads = [(t.data_ptr(), 0) for t in tensors]
        want = [("in", n, j, g) for j in range(3)]
        s.ops.append(("step", reads, want, (o.data_ptr(), 0), ("out", n, g)))
        return o

    mp = pytest.MonkeyPatch()
    try:
        mp.setattr(torch.cuda, "Stream", make_stream)
        mp.setattr(torch.cuda, "Event", FakeEvent)
        mp.setattr(torch.cuda, "stream", rec.stream)
        mp.setattr(torch.Tensor, "record_stream", lambda self, s: None)
        mp.setattr(sp, "copy_heads", rec.copy_heads)
        real_copy = torch.Tensor.copy_

        def copy_(self, src, non_blocking=False):
            # the whole-step path's copies, issued inside torch.cuda.stream(...)
            if rec.current is None:
                return real_copy(self, src, non_blocking)
            rec.current.ops.append(("copy", (self.data_ptr(), 0), (src.data_ptr(), 0)))
            return self
        mp.setattr(torch.Tensor, "copy_", copy_)
        pipe = sp.StepPipeline(inputs, step, device="cpu", head_groups=groups)
        if ignore_h2d_waits:
            pipe.h2d.ignore_waits = True
        host_in = [[torch.empty((rows, H, D), dtype=torch.bfloat16) for _ in range(3)]
                   for _ in range(steps)]
        host_out = [torch.empty((rows, H, D), dtype=torch.bfloat16) for _ in range(steps)]
        mem = {}
        for n in range(steps):
            for j in range(3):
                for g in range(groups):
                    mem[(host_in[n][j].data_ptr(), g * hg)] = ("in", n, j, g)
        for n in range(steps):
            calls.append(n)
            pipe.submit(host_in[n], host_out[n])
    finally:
        mp.undo()
    execute(made, mem, rng)
    for n in range(steps):
        for g in range(groups):
            got = mem.get((host_out[n].data_ptr(), g * hg))
            assert got == ("out", n, g), ("host output", n, g, got)


@pytest.mark.parametrize("depth,groups", [(2, 1), (3, 1), (2, 2), (2, 5), (3, 4), (1, 3)])
def test_step_pipeline_streams_keep_every_step_apart(depth, groups):
    rng = random.Random(depth * 10 + groups)
    for _ in range(60):
        run_pipeline(rng, depth, groups, steps=6)


@pytest.mark.parametrize("groups", [1, 2])
def test_step_pipeline_model_catches_a_missing_wait(groups):
    """With the H2D stream ignoring its waits, a later step's copy overwrites
    inputs a step has not read yet, in some interleaving."""
    rng = random.Random(5)
    caught = 0
    for _ in range(100):
        try:
            run_pipeline(rng, 2, groups, steps=6, ignore_h2d_waits=True)
        except AssertionError:
            caught += 1
    assert caught > 0
