"""Checks that pin the fp64 oracle to facts other than its own code.

Each check takes an optional ``lib`` (a bound oracle library) so that the
mutant tests can run the same checks against copies of the oracle with a
planted mistake and show that some check fails.  Every check raises
AssertionError on failure.

Facts used:
* page facts: after the exchange, head group j holds the full sequence for
  heads j*Hl .. j*Hl+Hl-1 (fal.ai WAN 2.2 page, "Splitting one generation
  across four GPUs"); the degree must divide the head count ("Tuning cost and
  GPU count"); the outputs go back to the token owners afterwards.
* library routines: numpy's reshape/transpose for the permutation and
  numpy fp64 matmul/exp for softmax(q K^T scale) V on small problems;
  scipy's logsumexp for the LSE.
* closed forms and invariants of softmax attention: rows of the softmax sum
  to one; V = 1 gives O = 1; Q = 0 gives the mean of V; N = 1 gives V; a
  dominant key selects its value row; invariance under a key permutation and
  under a common shift of all keys; linearity in V; a two-token example.
"""
from __future__ import annotations

import math

import numpy as np
from scipy.special import logsumexp

import oracle
import synth

RNG_SEED = 1234


def _codes(shape, rng):
    """Distinct-ish 16-bit payloads; pack/unpack move words without reading
    them, so any bit pattern serves as a tag."""
    n = int(np.prod(shape))
    base = rng.permutation(65536)[: min(n, 65536)].astype(np.uint16)
    return np.resize(base, n).reshape(shape)


def _small_ints_bf16(shape, rng, lo=-3, hi=4):
    """Small integers, exact in bf16 and closed under the sums the checks use."""
    return synth.f32_to_bf16(rng.integers(lo, hi, size=shape).astype(np.float32))


def _bf16_normal(shape, rng, mul=1.0):
    return synth.f32_to_bf16((rng.standard_normal(shape) * mul).astype(np.float32))


def _f64(x):
    return synth.bf16_to_f32(x).astype(np.float64)


PACK_SHAPES = [(1, 16, 4, 8, 2), (2, 13, 6, 8, 3), (3, 10, 8, 16, 4),
               (1, 7, 4, 8, 4), (2, 9, 8, 8, 8), (1, 5, 2, 8, 1)]


def check_pack_heads_for_full_sequence(lib=None):
    """Group j's buffer holds the full sequence for heads j*Hl..(j+1)*Hl-1,
    tokens in order; padding slots stay zero."""
    rng = np.random.default_rng(RNG_SEED)
    for (B, N, H, D, P) in PACK_SHAPES:
        X = _codes((B, N, H, D), rng)
        X[X == 0] = 1  # keep zero for the padding check
        xh = oracle.pack(synth.to_seq_shards(X, P), N, lib=lib)
        Hl = H // P
        for j in range(P):
            assert np.array_equal(xh[j][:, :N], X[:, :, j * Hl:(j + 1) * Hl]), (B, N, H, D, P, j)
            assert not xh[j][:, N:].any()


def check_pack_matches_numpy_transpose(lib=None):
    """Library formulation: per-rank shards viewed as [P][B][Nl][P][Hl][D],
    moved to [P(group)][B][P(rank)][Nl][Hl][D] by numpy."""
    rng = np.random.default_rng(RNG_SEED + 1)
    for (B, N, H, D, P) in PACK_SHAPES:
        Nl = -(-N // P)
        xs = _codes((P, B, Nl, H, D), rng)
        ref = xs.reshape(P, B, Nl, P, H // P, D).transpose(3, 1, 0, 2, 4, 5)
        ref = ref.reshape(P, B, P * Nl, H // P, D)
        assert np.array_equal(oracle.pack(xs, N, lib=lib), ref)


def check_unpack_returns_shards(lib=None):
    """Outputs go back to the token owners: unpack(pack(x)) = x, and a
    head-sharded result built from a logical tensor unpacks to its shards."""
    rng = np.random.default_rng(RNG_SEED + 2)
    for (B, N, H, D, P) in PACK_SHAPES:
        Nl = -(-N // P)
        xs = _codes((P, B, Nl, H, D), rng)
        assert np.array_equal(oracle.unpack(oracle.pack(xs, N, lib=lib), N, H, lib=lib), xs)
        X = _codes((B, N, H, D), rng)
        Hl = H // P
        oh = np.zeros((P, B, P * Nl, Hl, D), dtype=np.uint16)
        for j in range(P):
            oh[j][:, :N] = X[:, :, j * Hl:(j + 1) * Hl]
        os_ = oracle.unpack(oh, N, H, lib=lib)
        assert np.array_equal(synth.from_seq_shards(os_, N), X)
        assert np.array_equal(os_, synth.to_seq_shards(X, P))


def check_pack_degree_one_is_copy(lib=None):
    rng = np.random.default_rng(RNG_SEED + 3)
    xs = _codes((1, 2, 11, 4, 8), rng)
    assert np.array_equal(oracle.pack(xs, 11, lib=lib), xs)
    assert np.array_equal(oracle.unpack(xs, 11, 4, lib=lib), xs)


def check_exchange_chunks_hold_head_groups(lib=None):
    """On rank r, send chunk j holds r's tokens for heads j*Hl..(j+1)*Hl-1;
    the return reorder puts every group's chunk back at its heads."""
    rng = np.random.default_rng(RNG_SEED + 4)
    for (B, N, H, D, P) in PACK_SHAPES:
        Nl, Hl = -(-N // P), H // P
        X = _codes((B, N, H, D), rng)
        X[X == 0] = 1  # keep zero for the padding check
        xs = synth.to_seq_shards(X, P)
        for r in range(P):
            send = oracle.exchange_pack(xs[r], N, P, lib=lib)
            lo, hi = r * Nl, max(r * Nl, min(N, (r + 1) * Nl))
            for j in range(P):
                assert np.array_equal(send[j][:, : hi - lo], X[:, lo:hi, j * Hl:(j + 1) * Hl])
                assert not send[j][:, hi - lo:].any()  # padding slots stay zero
            assert np.array_equal(oracle.exchange_unpack(send, N, H, lib=lib), xs[r])


def check_exchange_matches_numpy_and_single_gpu_pack(lib=None):
    """numpy formulation ([B*Nl][P][Hl*D] -> [P][B*Nl][Hl*D]); and the
    all-to-all of the P ranks' chunks (chunk j of rank r to rank j, in rank
    order) is exactly the one-GPU head-sharded pack for B = 1."""
    rng = np.random.default_rng(RNG_SEED + 5)
    for (B, N, H, D, P) in PACK_SHAPES:
        Nl, Hl = -(-N // P), H // P
        xs = _codes((P, B, Nl, H, D), rng)
        sends = [oracle.exchange_pack(xs[r], N, P, lib=lib) for r in range(P)]
        for r in range(P):
            ref = xs[r].reshape(B * Nl, P, Hl * D).transpose(1, 0, 2).reshape(P, B, Nl, Hl, D)
            assert np.array_equal(sends[r], ref)
        if B == 1:
            xh = oracle.pack(xs, N, lib=lib)
            for j in range(P):
                recv_j = np.concatenate([sends[r][j] for r in range(P)], axis=1)
                assert np.array_equal(recv_j, xh[j])


# ---------------------------------------------------------------- attention

def _np_attention(q, k, v, scale=None):
    """numpy fp64 softmax(q K^T scale) V per (b, h); returns O, LSE."""
    qf, kf, vf = _f64(q), _f64(k), _f64(v)
    B, N, H, D = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    O = np.empty((B, N, H, D))
    L = np.empty((B, H, N))
    for b in range(B):
        for h in range(H):
            s = (qf[b, :, h] @ kf[b, :, h].T) * scale
            L[b, h] = logsumexp(s, axis=1)
            p = np.exp(s - L[b, h][:, None])
            O[b, :, h] = p @ vf[b, :, h]
    return O, L


ATTN_SHAPES = [(1, 1, 1, 16), (2, 37, 3, 16), (1, 130, 2, 64), (1, 64, 2, 128)]


def check_attention_matches_numpy(lib=None):
    rng = np.random.default_rng(RNG_SEED + 10)
    for (B, N, H, D) in ATTN_SHAPES:
        q, k, v = (_bf16_normal((B, N, H, D), rng, m) for m in (1.0, 1.5, 1.0))
        O, L = oracle.attention_full(q, k, v, lib=lib, threads=2)
        On, Ln = _np_attention(q, k, v)
        assert np.max(np.abs(O - On)) < 1e-12, (B, N, H, D)
        assert np.max(np.abs(L - Ln)) < 1e-12, (B, N, H, D)


def check_softmax_rows_sum_to_one(lib=None):
    """sum_k exp(s_ik - LSE_i) = 1 with s computed by numpy."""
    rng = np.random.default_rng(RNG_SEED + 11)
    B, N, H, D = 1, 200, 2, 32
    q, k, v = (_bf16_normal((B, N, H, D), rng, 2.0) for _ in range(3))
    _, L = oracle.attention_full(q, k, v, lib=lib, threads=2)
    qf, kf = _f64(q), _f64(k)
    for h in range(H):
        s = (qf[0, :, h] @ kf[0, :, h].T) / math.sqrt(D)
        tot = np.exp(s - L[0, h][:, None]).sum(axis=1)
        assert np.max(np.abs(tot - 1.0)) < 1e-12


def check_closed_forms(lib=None):
    rng = np.random.default_rng(RNG_SEED + 12)
    B, N, H, D = 1, 50, 2, 16
    q, k = _bf16_normal((B, N, H, D), rng), _bf16_normal((B, N, H, D), rng)
    v = _bf16_normal((B, N, H, D), rng)
    # V = 1 -> O = 1 for every row.
    ones = synth.f32_to_bf16(np.ones((B, N, H, D), dtype=np.float32))
    O, _ = oracle.attention_full(q, k, ones, lib=lib, threads=2)
    assert np.max(np.abs(O - 1.0)) < 1e-13
    # Q = 0 -> uniform weights -> O = mean_k V and LSE = ln N.
    zeros = np.zeros((B, N, H, D), dtype=np.uint16)
    O, L = oracle.attention_full(zeros, k, v, lib=lib, threads=2)
    mean = _f64(v).mean(axis=1)  # [B][H][D]
    assert np.max(np.abs(O - mean[:, None])) < 1e-13
    assert np.max(np.abs(L - math.log(N))) < 1e-13
    # N = 1 -> O = V.
    O, L = oracle.attention_full(q[:, :1], k[:, :1], v[:, :1], lib=lib, threads=1)
    assert np.array_equal(O, _f64(v[:, :1]))


def check_dominant_key(lib=None):
    """A key aligned with q and scaled far above the rest takes all weight."""
    rng = np.random.default_rng(RNG_SEED + 13)
    B, N, H, D = 1, 40, 1, 16
    q = _small_ints_bf16((B, N, H, D), rng, 1, 3)          # entries 1..2
    k = _small_ints_bf16((B, N, H, D), rng, -1, 2)          # entries -1..1
    v = _bf16_normal((B, N, H, D), rng)
    star = 17
    k[0, star, 0] = synth.f32_to_bf16(np.full(D, 64.0, dtype=np.float32))
    O, _ = oracle.attention_full(q, k, v, lib=lib, threads=2)
    # logit gap >= (64*16 - 2*16)/4 = 248 -> other weights < N*e^-248.
    assert np.max(np.abs(O[0, :, 0] - _f64(v[0, star, 0])[None])) < 1e-12


def check_invariances(lib=None):
    rng = np.random.default_rng(RNG_SEED + 14)
    B, N, H, D = 2, 33, 2, 16
    q = _small_ints_bf16((B, N, H, D), rng)
    k = _small_ints_bf16((B, N, H, D), rng)
    v1 = _small_ints_bf16((B, N, H, D), rng)
    v2 = _small_ints_bf16((B, N, H, D), rng)
    scale = 0.125
    O, L = oracle.attention_full(q, k, v1, scale, lib=lib, threads=2)
    # Permuting the key/value tokens together changes nothing.
    perm = rng.permutation(N)
    Op, _ = oracle.attention_full(q, k[:, perm], v1[:, perm], scale, lib=lib, threads=2)
    assert np.max(np.abs(Op - O)) < 1e-12
    # Permuting the queries permutes the rows.
    Oq, _ = oracle.attention_full(q[:, perm], k, v1, scale, lib=lib, threads=2)
    assert np.max(np.abs(Oq - O[:, perm])) < 1e-12
    # A common shift u of all keys adds scale*q.u to every score of a row:
    # O unchanged, LSE shifted by exactly that amount.
    u = rng.integers(-2, 3, size=D).astype(np.float32)
    ks = synth.f32_to_bf16(synth.bf16_to_f32(k) + u)
    Os, Ls = oracle.attention_full(q, ks, v1, scale, lib=lib, threads=2)
    assert np.max(np.abs(Os - O)) < 1e-12
    shift = scale * np.einsum("bnhd,d->bhn", _f64(q), u.astype(np.float64))
    assert np.max(np.abs(Ls - (L + shift))) < 1e-11
    # Linear in V.
    v12 = synth.f32_to_bf16(synth.bf16_to_f32(v1) + synth.bf16_to_f32(v2))
    O2, _ = oracle.attention_full(q, k, v2, scale, lib=lib, threads=2)
    O12, _ = oracle.attention_full(q, k, v12, scale, lib=lib, threads=2)
    assert np.max(np.abs(O12 - (O + O2))) < 1e-12
    # Scores scale with K: (2K, scale/2) gives the same result.
    k2 = synth.f32_to_bf16(synth.bf16_to_f32(k) * 2)
    Ok, Lk = oracle.attention_full(q, k2, v1, scale / 2, lib=lib, threads=2)
    assert np.max(np.abs(Ok - O)) < 1e-12 and np.max(np.abs(Lk - L)) < 1e-12
    # scale <= 0 means 1/sqrt(D).
    Od, _ = oracle.attention_full(q, k, v1, 0.0, lib=lib, threads=2)
    Oe, _ = oracle.attention_full(q, k, v1, 1.0 / math.sqrt(D), lib=lib, threads=2)
    assert np.array_equal(Od, Oe)


def check_two_token_example(lib=None):
    """Worked by hand: D = 4, scale = 1/2, one head.  q = (2,0,0,0),
    k0 = (1,0,0,0), k1 = (0,0,0,0): scores (1, 0), weights e/(e+1) and
    1/(e+1); v0 = (1,2,3,4), v1 = (-1,0,0,8)."""
    f = lambda a: synth.f32_to_bf16(np.array(a, dtype=np.float32))
    q = f([[[[2, 0, 0, 0]], [[0, 0, 0, 0]]]])
    k = f([[[[1, 0, 0, 0]], [[0, 0, 0, 0]]]])
    v = f([[[[1, 2, 3, 4]], [[-1, 0, 0, 8]]]])
    O, L = oracle.attention_full(q, k, v, lib=lib, threads=1)
    e = math.e
    w0, w1 = e / (e + 1), 1 / (e + 1)
    want0 = [w0 * 1 + w1 * -1, w0 * 2, w0 * 3, w0 * 4 + w1 * 8]
    assert np.max(np.abs(O[0, 0, 0] - want0)) < 1e-15
    assert abs(L[0, 0, 0] - math.log(e + 1)) < 1e-15
    # query 1 is all zeros: uniform over the two keys.
    assert np.max(np.abs(O[0, 1, 0] - [0, 1, 1.5, 6])) < 1e-15
    assert abs(L[0, 0, 1] - math.log(2)) < 1e-15


def check_rows_api(lib=None):
    """attention_rows on a subset equals the same rows of attention_full."""
    rng = np.random.default_rng(RNG_SEED + 15)
    B, N, H, D = 2, 70, 3, 16
    q, k, v = (_bf16_normal((B, N, H, D), rng) for _ in range(3))
    O, L = oracle.attention_full(q, k, v, lib=lib, threads=3)
    rows = np.array([[1, 2, 69], [0, 0, 0], [1, 0, 35]], dtype=np.int64)
    o, l = oracle.attention_rows(q, k, v, rows, lib=lib, threads=2)
    for r, (b, h, i) in enumerate(rows):
        assert np.array_equal(o[r], O[b, i, h]) and l[r] == L[b, h, i]


def check_e4m3_decode_matches_torch(lib=None):
    """All 256 E4M3 bytes decode as torch's float8_e4m3fn does."""
    import torch
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([oracle.e4m3_value(int(c), lib=lib) for c in codes])
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(got[ok], ref[ok])


def _e4m3_from_float(x):
    import torch
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(
        torch.float8_e4m3fn).view(torch.uint8).numpy()


def check_fp8_attention_reduces_to_bf16(lib=None):
    """Small integers are exact in both formats: with unit scales the e4m3
    path equals the (pinned) bf16 path; scale factors act as their closed
    forms (dv scales O, dq*dk scales the logits)."""
    rng = np.random.default_rng(RNG_SEED + 16)
    B, N, H, D = 2, 33, 2, 16
    fq, fk, fv = (rng.integers(-3, 4, size=(B, N, H, D)).astype(np.float32) for _ in range(3))
    q8, k8, v8 = (_e4m3_from_float(x) for x in (fq, fk, fv))
    qb, kb, vb = (synth.f32_to_bf16(x) for x in (fq, fk, fv))
    rows = np.array([(b, h, i) for b in range(B) for h in range(H) for i in range(N)], np.int64)
    scale = 0.125
    o8, l8 = oracle.attention_rows_e4m3(q8, k8, v8, 1.0, 1.0, 1.0, rows, scale, 2, lib=lib)
    ob, lb = oracle.attention_rows(qb, kb, vb, rows, scale, 2, lib=lib)
    assert np.max(np.abs(o8 - ob)) < 1e-13 and np.max(np.abs(l8 - lb)) < 1e-13
    dq = rng.uniform(0.5, 2.0, size=(B, H))
    dk = rng.uniform(0.5, 2.0, size=(B, H))
    dv = rng.uniform(0.5, 2.0, size=(B, H))
    o8s, _ = oracle.attention_rows_e4m3(q8, k8, v8, dq, dk, dv, rows, scale, 2, lib=lib)
    for r, (b, h, i) in enumerate(rows):
        # logits scale by dq*dk: the same as the unit-scale problem at scale*dq*dk
        want, _ = oracle.attention_rows_e4m3(q8, k8, v8, 1.0, 1.0, 1.0, rows[r:r + 1],
                                             scale * dq[b, h] * dk[b, h], 1, lib=lib)
        assert np.max(np.abs(o8s[r] - dv[b, h] * want[0])) < 1e-12


def check_fp8_block_factors_match_dequantized_bf16(lib=None):
    """Q and K factors per block of tokens and V factors per channel, all
    powers of two, times small integers give values exact in bf16: the e4m3
    attention must equal the (pinned) bf16 attention of the dequantized
    tensors.  Block size 8 over N = 33 leaves a ragged last block."""
    rng = np.random.default_rng(RNG_SEED + 17)
    B, N, H, D, blk = 2, 33, 3, 16, 8
    nblk = -(-N // blk)
    fq, fk, fv = (rng.integers(-3, 4, size=(B, N, H, D)).astype(np.float32) for _ in range(3))
    q8, k8, v8 = (_e4m3_from_float(x) for x in (fq, fk, fv))
    dq = 2.0 ** rng.integers(-2, 3, size=(B, H, nblk))
    dk = 2.0 ** rng.integers(-2, 3, size=(B, H, nblk))
    dv = 2.0 ** rng.integers(-2, 3, size=(B, H, D))
    tok_blk = np.arange(N) // blk
    deq_q = fq * dq.transpose(0, 2, 1)[:, tok_blk, :, None]
    deq_k = fk * dk.transpose(0, 2, 1)[:, tok_blk, :, None]
    deq_v = fv * dv[:, None, :, :]
    qb, kb, vb = (synth.f32_to_bf16(x.astype(np.float32)) for x in (deq_q, deq_k, deq_v))
    for x, xb in ((deq_q, qb), (deq_k, kb), (deq_v, vb)):
        assert np.array_equal(synth.bf16_to_f32(xb), x.astype(np.float32))  # exact in bf16
    rows = np.array([(b, h, i) for b in range(B) for h in range(H) for i in range(N)], np.int64)
    scale = 0.05
    o8, l8 = oracle.attention_rows_e4m3(q8, k8, v8, dq, dk, dv, rows, scale, 2, block=blk,
                                        lib=lib)
    ob, lb = oracle.attention_rows(qb, kb, vb, rows, scale, 2, lib=lib)
    assert np.max(np.abs(o8 - ob)) < 1e-12 * max(1.0, np.max(np.abs(ob)))
    assert np.max(np.abs(l8 - lb)) < 1e-12 * max(1.0, np.max(np.abs(lb)))


def _all_rows(B, N, H):
    return np.array([(b, h, i) for b in range(B) for h in range(H) for i in range(N)],
                    dtype=np.int64)


def check_masked_attention(lib=None):
    """Block-masked attention (the sparse stage of video sparse attention)
    against what the mask means, on a ragged last cube (N = 45, cubes of 8):
    * every cube selected -> the dense oracle, exactly;
    * one key cube per query cube -> dense attention over that cube's keys
      alone (the dense oracle on the sliced K and V);
    * a random selection -> numpy's fp64 softmax with the unselected scores
      set to -inf (scipy logsumexp for the LSE);
    * a query cube that selects nothing -> O = 0 and LSE = -inf."""
    rng = np.random.default_rng(RNG_SEED + 18)
    B, N, H, D, cube = 2, 45, 2, 16, 8
    nc = -(-N // cube)
    q, k, v = (_bf16_normal((B, N, H, D), rng, m) for m in (1.0, 1.5, 1.0))
    rows = _all_rows(B, N, H)
    full = np.ones((B, H, nc, nc), np.uint8)
    Om, Lm = oracle.attention_rows_masked(q, k, v, full, rows, cube=cube, threads=2, lib=lib)
    Od, Ld = oracle.attention_rows(q, k, v, rows, threads=2, lib=lib)
    assert np.array_equal(Om, Od) and np.array_equal(Lm, Ld)

    pick = rng.integers(0, nc, size=(B, H, nc))
    one = np.zeros((B, H, nc, nc), np.uint8)
    for b in range(B):
        for h in range(H):
            one[b, h, np.arange(nc), pick[b, h]] = 1
    O1, L1 = oracle.attention_rows_masked(q, k, v, one, rows, cube=cube, threads=2, lib=lib)
    for r, (b, h, i) in enumerate(rows):
        c = pick[b, h, i // cube]
        ks = slice(c * cube, min(N, (c + 1) * cube))
        kc = np.ascontiguousarray(k[b:b + 1, ks, h:h + 1])
        vc = np.ascontiguousarray(v[b:b + 1, ks, h:h + 1])
        qc = np.zeros_like(kc)
        qc[0, 0, 0] = q[b, i, h]                     # the query as row 0 of a dense problem
        want, wl = oracle.attention_rows(qc, kc, vc, np.zeros((1, 3), np.int64),
                                         scale=1.0 / math.sqrt(D), threads=1, lib=lib)
        assert np.max(np.abs(O1[r] - want[0])) < 1e-13 and abs(L1[r] - wl[0]) < 1e-13

    sel = (rng.random((B, H, nc, nc)) < 0.3).astype(np.uint8)
    sel[0, 1, 2] = 0                                 # query cube 2 of (0, 1) selects nothing
    sel[1, 0, :, nc - 1] = 1                         # the ragged last cube is selected
    Os, Ls = oracle.attention_rows_masked(q, k, v, sel, rows, cube=cube, threads=2, lib=lib)
    qf, kf, vf = _f64(q), _f64(k), _f64(v)
    tok = np.arange(N) // cube
    for r, (b, h, i) in enumerate(rows):
        keep = sel[b, h, i // cube][tok].astype(bool)
        if not keep.any():
            assert np.all(Os[r] == 0) and Ls[r] == -np.inf
            continue
        sc = np.where(keep, kf[b, :, h] @ qf[b, i, h] / math.sqrt(D), -np.inf)
        lse = logsumexp(sc)
        assert abs(Ls[r] - lse) < 1e-12
        assert np.max(np.abs(Os[r] - np.exp(sc - lse) @ vf[b, :, h])) < 1e-12
    assert np.any(~sel[0, 1, 2].astype(bool))


def check_linear_projection(lib=None):
    """The projection oracle: a worked 2 x 2 example by hand, the identity
    weight returning x exactly, and numpy's fp64 x @ w.T + b on random
    shapes (row subsets in any order, with and without a bias)."""
    x = synth.f32_to_bf16(np.array([[1, 2], [3, 4]], np.float32))
    w = synth.f32_to_bf16(np.array([[1, 0], [1, 1], [0, -2]], np.float32))
    b = synth.f32_to_bf16(np.array([0.5, -1, 0.25], np.float32))
    y = oracle.linear_rows(x, w, b, [1, 0], threads=1, lib=lib)
    assert np.array_equal(y, np.array([[3.5, 6.0, -7.75], [1.5, 2.0, -3.75]]))
    rng = np.random.default_rng(RNG_SEED + 19)
    xi = _bf16_normal((9, 16), rng)
    eye = synth.f32_to_bf16(np.eye(16, dtype=np.float32))
    assert np.array_equal(oracle.linear_rows(xi, eye, None, np.arange(9), threads=2, lib=lib),
                          _f64(xi))
    for (M, K, nout) in [(7, 33, 12), (20, 64, 48)]:
        xr, wr = _bf16_normal((M, K), rng), _bf16_normal((nout, K), rng, 0.1)
        br = _bf16_normal((nout,), rng)
        rows = rng.permutation(M)[: M // 2]
        for bias in (None, br):
            got = oracle.linear_rows(xr, wr, bias, rows, threads=2, lib=lib)
            want = _f64(xr)[rows] @ _f64(wr).T + (0.0 if bias is None else _f64(bias))
            assert np.max(np.abs(got - want)) < 1e-12 * max(1.0, np.max(np.abs(want)))


def check_shard_splits_the_sequence(lib=None):
    """Rank r holds tokens r*Nl .. r*Nl+Nl-1 of the logical tensor (the page's
    division of the token sequence, written as numpy slicing); the slots past
    the last token are zero."""
    rng = np.random.default_rng(RNG_SEED + 40)
    for (B, N, H, D, P) in PACK_SHAPES + [(2, 3, 2, 8, 8)]:
        X = _codes((B, N, H, D), rng)
        X[X == 0] = 1
        xs = oracle.shard(X, P, lib=lib)
        Nl = -(-N // P)
        assert xs.shape == (P, B, Nl, H, D)
        for r in range(P):
            lo, hi = min(r * Nl, N), min(r * Nl + Nl, N)
            assert np.array_equal(xs[r][:, :hi - lo], X[:, lo:hi]), (B, N, H, D, P, r)
            assert not xs[r][:, hi - lo:].any()


def check_shard_matches_numpy_and_inverts(lib=None):
    """Library formulation: zero-pad the sequence to P*Nl and move
    [B][P][Nl] to [P][B][Nl] with numpy; unshard inverts shard and, on shards
    with junk in the padding slots, equals numpy's inverse reshape."""
    rng = np.random.default_rng(RNG_SEED + 41)
    for (B, N, H, D, P) in PACK_SHAPES + [(2, 3, 2, 8, 8)]:
        X = _codes((B, N, H, D), rng)
        Nl = -(-N // P)
        pad = np.zeros((B, P * Nl, H, D), dtype=np.uint16)
        pad[:, :N] = X
        ref = pad.reshape(B, P, Nl, H, D).transpose(1, 0, 2, 3, 4)
        assert np.array_equal(oracle.shard(X, P, lib=lib), ref)
        assert np.array_equal(oracle.unshard(oracle.shard(X, P, lib=lib), N, lib=lib), X)
        xs = _codes((P, B, Nl, H, D), rng)
        want = xs.transpose(1, 0, 2, 3, 4).reshape(B, P * Nl, H, D)[:, :N]
        assert np.array_equal(oracle.unshard(xs, N, lib=lib), want)


PACK_CHECKS = [check_pack_heads_for_full_sequence, check_pack_matches_numpy_transpose,
               check_unpack_returns_shards, check_pack_degree_one_is_copy,
               check_exchange_chunks_hold_head_groups,
               check_exchange_matches_numpy_and_single_gpu_pack,
               check_shard_splits_the_sequence, check_shard_matches_numpy_and_inverts]
ATTENTION_CHECKS = [check_attention_matches_numpy, check_softmax_rows_sum_to_one,
                    check_closed_forms, check_dominant_key, check_invariances,
                    check_two_token_example, check_rows_api,
                    check_e4m3_decode_matches_torch, check_fp8_attention_reduces_to_bf16,
                    check_fp8_block_factors_match_dequantized_bf16, check_masked_attention,
                    check_linear_projection]
ALL_CHECKS = PACK_CHECKS + ATTENTION_CHECKS
