"""CPU model of the block-sparse kernel's K/V ring protocol (no GPU).

The kernel (attention_sparse_kernel) builds, per CTA, one list of key cubes
per 128-row query tile -- the cubes both tiles visit first, then the tile's
own, each group in increasing order -- and walks each list two cubes per
step.  Its ring holds K and V slots in a fixed order that three roles follow:
two producer warps (one loads the K slots, one the V slots), the MMA thread
(which takes slots in that order and releases each after the last MMA that
reads it) and, through the MMA thread, the two softmax groups.  This module
restates that protocol in Python and checks, over random masks, the
properties the kernel relies on:
  * the producers' order and the MMA thread's takes agree, slot for slot;
  * each slot is released exactly once, after every MMA that reads it;
  * no take waits on a release that comes later in the MMA thread's order,
    and the three actors, interleaved at random, always run to completion;
  * each tile's S and PV MMAs cover exactly its list's pairs, in order;
  * with every cube selected the lists are 0, 1, 2, ... (the dense order).
The GPU parity tests check the kernel itself against the oracle.
"""
import random

import numpy as np

STAGES = 4


def build_lists(u0, u1, ncube):
    """Per tile: the cubes both tiles select, then the tile's own (each in
    increasing order), padded with ncube when their number is odd."""
    both = [c for c in range(ncube) if u0[c] and u1[c]]
    out = []
    for mine, other in ((u0, u1), (u1, u0)):
        lst = both + [c for c in range(ncube) if mine[c] and not other[c]]
        n = len(lst)
        out.append((lst + ([ncube] if n % 2 else []), n))
    return out


def pair_at(lst, i):
    return (lst[2 * i], lst[2 * i + 1])


def ring_order(lists):
    """The producers' slot order: K of both walks' first steps, then per step
    i the V of step i and the K of step i+1 for tile 0, then the same for
    tile 1; a slot is loaded once when both walks are at the same pair."""
    (l0, n0), (l1, n1) = lists
    seq = []
    a0, a1 = n0 > 0, n1 > 0
    c0 = pair_at(l0, 0) if a0 else None
    c1 = pair_at(l1, 0) if a1 else None
    if a0:
        seq.append(("K", c0))
    if a1 and not (a0 and c0 == c1):
        seq.append(("K", c1))
    i = 1
    while a0 or a1:
        na0, na1 = 2 * i < n0, 2 * i < n1
        x0 = pair_at(l0, i) if na0 else c0
        x1 = pair_at(l1, i) if na1 else c1
        sh_cur = a0 and a1 and c0 == c1
        sh_nxt = na0 and na1 and x0 == x1
        if a0:
            seq.append(("V", c0))
            if na0:
                seq.append(("K", x0))
        if a1 and not sh_cur:
            seq.append(("V", c1))
        if na1 and not sh_nxt:
            seq.append(("K", x1))
        c0, c1, a0, a1 = x0, x1, na0, na1
        i += 1
    return seq


def mma_program(lists):
    """The MMA thread's operations in issue order: ('take', n), ('rel', n),
    ('S', tile, n), ('PV', tile, n, first), ('O', tile)."""
    (l0, n0), (l1, n1) = lists
    prog = []
    it = [0]

    def take():
        n = it[0]
        it[0] += 1
        prog.append(("take", n))
        return n
    a0, a1 = n0 > 0, n1 > 0
    c0 = pair_at(l0, 0) if a0 else None
    c1 = pair_at(l1, 0) if a1 else None
    if not a0:
        prog.append(("O", 0))
    if not a1:
        prog.append(("O", 1))
    sh0 = a0 and a1 and c0 == c1
    k0 = None
    if a0:
        k0 = take()
        prog.append(("S", 0, k0))
        if not sh0:
            prog.append(("rel", k0))
    if a1:
        k1 = k0 if sh0 else take()
        prog.append(("S", 1, k1))
        prog.append(("rel", k1))
    jj = 0
    while a0 or a1:
        na0, na1 = 2 * (jj + 1) < n0, 2 * (jj + 1) < n1
        x0 = pair_at(l0, jj + 1) if na0 else c0
        x1 = pair_at(l1, jj + 1) if na1 else c1
        sh_cur = a0 and a1 and c0 == c1
        sh_nxt = na0 and na1 and x0 == x1
        sv0 = sk0 = None
        if a0:
            sv0 = take()
            if na0:
                sk0 = take()
            prog.append(("PV", 0, sv0, jj == 0))
            prog.append(("S", 0, sk0) if na0 else ("O", 0))
            if not sh_cur:
                prog.append(("rel", sv0))
            if na0 and not sh_nxt:
                prog.append(("rel", sk0))
        if a1:
            sv1, sk1 = sv0, sk0
            if not sh_cur:
                sv1 = take()
            if na1 and not sh_nxt:
                sk1 = take()
            prog.append(("PV", 1, sv1, jj == 0))
            prog.append(("S", 1, sk1) if na1 else ("O", 1))
            prog.append(("rel", sv1))
            if na1:
                prog.append(("rel", sk1))
        c0, c1, a0, a1 = x0, x1, na0, na1
        jj += 1
    return prog


def check_schedule(u0, u1, ncube, rng):
    lists = build_lists(u0, u1, ncube)
    for t, (lst, n) in enumerate(lists):
        assert sorted(lst[:n]) == [c for c in range(ncube) if (u0, u1)[t][c]]
    seq = ring_order(lists)
    prog = mma_program(lists)
    takes = [e[1] for e in prog if e[0] == "take"]
    assert takes == list(range(len(seq)))
    rel_at = {}
    for i, e in enumerate(prog):
        if e[0] == "rel":
            assert e[1] not in rel_at, "slot released twice"
            rel_at[e[1]] = i
    assert sorted(rel_at) == list(range(len(seq)))
    for i, e in enumerate(prog):
        if e[0] == "take" and e[1] >= STAGES:
            assert rel_at[e[1] - STAGES] < i, "take before the slot's previous release"
    for n in range(len(seq)):
        readers = [i for i, e in enumerate(prog) if e[0] in ("S", "PV") and e[2] == n]
        assert readers and rel_at[n] > max(readers)
    for t in range(2):
        lst, n = lists[t]
        walk = [pair_at(lst, i) for i in range((n + 1) // 2)]
        s_ops = [seq[e[2]] for e in prog if e[0] == "S" and e[1] == t]
        pv_ops = [e for e in prog if e[0] == "PV" and e[1] == t]
        assert [p for _, p in s_ops] == walk and all(k == "K" for k, _ in s_ops)
        assert [seq[e[2]][1] for e in pv_ops] == walk
        assert all(seq[e[2]][0] == "V" for e in pv_ops)
        assert [e[3] for e in pv_ops] == [i == 0 for i in range(len(walk))]
        assert sum(1 for e in prog if e[0] == "O" and e[1] == t) == 1
    # the two producer warps and the MMA thread as independent actors
    loaded = [False] * len(seq)
    released = [False] * len(seq)
    todo = {"K": [n for n in range(len(seq)) if seq[n][0] == "K"],
            "V": [n for n in range(len(seq)) if seq[n][0] == "V"]}
    pc = 0
    while True:
        moved = False
        for kind in rng.sample(["K", "V"], 2):
            if todo[kind]:
                n = todo[kind][0]
                if n < STAGES or released[n - STAGES]:
                    loaded[n] = True
                    todo[kind].pop(0)
                    moved = True
        if pc < len(prog):
            e = prog[pc]
            if e[0] != "take" or loaded[e[1]]:
                if e[0] == "rel":
                    released[e[1]] = True
                pc += 1
                moved = True
        if not moved:
            break
    assert not todo["K"] and not todo["V"] and pc == len(prog), "deadlock"
    return len(seq)


def test_sparse_ring_protocol_over_random_masks():
    rng = np.random.default_rng(0)
    prng = random.Random(0)
    for trial in range(3000):
        ncube = int(rng.integers(1, 40))
        d = rng.random()
        mode = trial % 5
        u0 = rng.random(ncube) < d
        if mode == 0:
            u1 = rng.random(ncube) < d          # independent
        elif mode == 1:
            u1 = u0.copy()                      # coherent
        elif mode == 2:
            u1 = u0 & (rng.random(ncube) < 0.8)
        elif mode == 3:
            u1 = np.zeros(ncube, bool)          # one tile selects nothing
        else:
            u0, u1 = np.zeros(ncube, bool), u0
        check_schedule(list(u0), list(u1), ncube, prng)


def test_full_selection_walks_dense_pairs_and_coherent_masks_share_every_load():
    full = [True] * 7
    lists = build_lists(full, full, 7)
    assert [pair_at(lists[0][0], i) for i in range(4)] == [(0, 1), (2, 3), (4, 5), (6, 7)]
    seq = ring_order(lists)
    assert len(seq) == 2 * 4                    # one K and one V slot per step
    rng = np.random.default_rng(1)
    u = list(rng.random(50) < 0.3)
    assert len(ring_order(build_lists(u, u, 50))) == 2 * ((sum(u) + 1) // 2)


def test_independent_masks_load_the_union_once():
    """Cubes both tiles select are loaded once; at density 0.2 over 1,182 cubes
    (the 720p grid) a CTA loads about the union of its two tiles' cubes."""
    rng = np.random.default_rng(2)
    nc = 1182
    slots = 0
    union = 0
    for _ in range(20):
        qc = rng.random((4, nc)) < 0.2
        u0, u1 = qc[0] | qc[1], qc[2] | qc[3]
        slots += len(ring_order(build_lists(list(u0), list(u1), nc)))
        union += int((u0 | u1).sum())
    # K and V per pair: about the union's cubes, plus at most a few half-empty pairs
    assert slots <= union + 4 * 20
