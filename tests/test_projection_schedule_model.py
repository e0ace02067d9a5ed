"""CPU model of the projection kernel's tile protocol (no GPU).

projection_pair_kernel computes 256 x 512 tiles of y on CTA pairs.  A tile's
two 256-feature halves each accumulate in 256 of the 512 TMEM columns, so the
MMA thread cannot start a tile while the previous one drains.  It staggers
the halves instead:
  * over a tile's first D stages it issues half 0's MMAs and holds the
    stages until half 1 of the previous tile has left TMEM;
  * then both halves per stage;
  * over the last D stages it issues half 0 first and commits acc_full[0],
    so the epilogue drains half 0 while half 1's last MMAs run.
The ring has S = D + 1 slots; waits are on mbarrier parities.  This module
restates the protocol for the producer (ring loads), the MMA thread, the
epilogue and the asynchronous load completions, runs random interleavings,
and checks that:
  * nothing deadlocks, for 1 to 80 stages per tile;
  * every parity wait is unambiguous (the barrier is at most one phase short
    of, and never past, the phase waited for);
  * no MMA writes a half the epilogue is reading, and the epilogue reads a
    half only after its last MMA;
  * each MMA reads a ring slot that holds its stage.
The GPU tests check the kernel's results against the oracle.
"""
import random

S, D = 4, 3


def run(nk, ntiles, rng, wait_for_half1=True):
    full = [0] * S          # completions of full[s]
    empty = [0] * S         # completions of empty[s]
    acc_full = [0, 0]
    acc_empty = [0, 0]
    landing = []            # slots with a load in flight, in issue order
    owner = [None, None]    # ("mma", tile) / ("done", tile) / ("epi", tile)

    def parity_wait(counter, idx, target, first_free=False):
        # wait until counter[idx] >= target; a parity wait sees only the low
        # bit, so the count must be target - 1 or target when it looks
        while True:
            k = counter[idx]
            ok = k in (target - 1, target) or (first_free and target == 0 and k == 0)
            assert ok, ("ambiguous parity wait", k, target)
            if k >= target:
                return
            yield

    def producer():
        i = 0
        for _ in range(ntiles):
            for _ in range(nk):
                s = i % S
                yield from parity_wait(empty, s, i // S, first_free=True)
                landing.append(s)
                i += 1
                yield

    def mma():
        it = 0
        for n in range(ntiles):
            a = min(D, nk)
            c = max(a, nk - D)

            def land(kb):
                i = it + kb
                yield from parity_wait(full, i % S, i // S + 1)

            def acc_free(h):
                if h == 0 or wait_for_half1:
                    yield from parity_wait(acc_empty, h, n, first_free=True)
                else:
                    # a planted bug: half 1 taken without waiting for its drain
                    assert owner[h] is None or owner[h][0] != "epi", ("TMEM hazard", h, owner[h])
                owner[h] = ("mma", n)

            def issue(kb, h):
                assert owner[h] == ("mma", n), ("TMEM hazard", h, owner[h], n)
                i = it + kb
                assert full[i % S] == i // S + 1 and empty[i % S] == i // S, "slot not holding stage"

            def release(kb):
                empty[(it + kb) % S] += 1

            def done(h):
                acc_full[h] += 1
                owner[h] = ("done", n)

            yield from acc_free(0)
            for kb in range(a):
                yield from land(kb)
                issue(kb, 0)
                yield
            if a == nk:
                done(0)
            yield from acc_free(1)
            for kb in range(a):
                issue(kb, 1)
                release(kb)
                yield
            for kb in range(a, c):
                yield from land(kb)
                issue(kb, 0)
                issue(kb, 1)
                release(kb)
                yield
            if a < nk:
                for kb in range(c, nk):
                    yield from land(kb)
                    issue(kb, 0)
                    yield
                done(0)
                for kb in range(c, nk):
                    issue(kb, 1)
                    release(kb)
                    yield
            done(1)
            it += nk

    def epilogue():
        for n in range(ntiles):
            for h in range(2):
                yield from parity_wait(acc_full, h, n + 1)
                assert owner[h] == ("done", n), ("epilogue before the last MMA", owner[h], n)
                owner[h] = ("epi", n)
                for _ in range(rng.randint(0, 4)):
                    yield
                owner[h] = None
                acc_empty[h] += 1
                yield

    actors = {"producer": producer(), "mma": mma(), "epilogue": epilogue()}
    steps = 0
    while actors:
        steps += 1
        assert steps < 2_000_000, "deadlock"
        names = list(actors) + (["land"] if landing else [])
        who = rng.choice(names)
        if who == "land":
            full[landing.pop(0)] += 1
            continue
        try:
            next(actors[who])
        except StopIteration:
            del actors[who]
    assert acc_full == [ntiles, ntiles] and acc_empty == [ntiles, ntiles]
    assert sum(full) == sum(empty) == nk * ntiles


def test_projection_tile_protocol_random_interleavings():
    rng = random.Random(0)
    for nk in list(range(1, 10)) + [16, 80]:
        for ntiles in (1, 2, 3, 5):
            for _ in range(8):
                run(nk, ntiles, rng)


def test_projection_tile_protocol_model_catches_a_missing_wait():
    """With the wait for half 1's drain left out, some interleaving lets the
    MMA thread take half 1 while the epilogue still reads it, and the model
    reports it."""
    rng = random.Random(1)
    caught = 0
    for _ in range(200):
        try:
            run(6, 3, rng, wait_for_half1=False)
        except AssertionError as e:
            assert "TMEM hazard" in str(e) or "epilogue before" in str(e)
            caught += 1
    assert caught > 0
