"""The seeded input generator (CPU only)."""
import numpy as np

import synth


def test_splitmix64_known_answers():
    # SplitMix64 from state 0: the first three outputs published with the
    # generator's reference implementation.
    g = np.uint64(0x9E3779B97F4A7C15)
    with np.errstate(over="ignore"):
        z = g * np.arange(1, 4, dtype=np.uint64)
        z = (z ^ (z >> np.uint64(30))) * np.uint64(0xBF58476D1CE4E5B9)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(0x94D049BB133111EB)
        z = z ^ (z >> np.uint64(31))
    assert [int(x) for x in z] == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4,
                                   0x06C45D188009454F]


def test_c_and_numpy_streams_agree():
    idx = [0, 1, 2, 1000, 123456]
    c = synth.stream_u64(7, 3, idx)
    n = synth._stream_u64_range(7, 3, 123457)[idx]
    assert np.array_equal(c, n)


def test_normals_look_standard_and_are_deterministic():
    a = synth.normal_bf16(11, 0, 0, 1 << 20)
    b = synth.normal_bf16(11, 0, 0, 1 << 20, threads=3)
    assert np.array_equal(a, b)
    f = synth.bf16_to_f32(a).astype(np.float64)
    assert abs(f.mean()) < 5e-3 and abs(f.std() - 1) < 5e-3
    # offsets address the same stream
    c = synth.normal_bf16(11, 0, 500, 100)
    assert np.array_equal(c, a[500:600])
    # another tensor id gives other numbers
    d = synth.normal_bf16(11, 1, 0, 1 << 10)
    assert not np.array_equal(d, a[: 1 << 10])


def test_bf16_rounding_is_nearest_even():
    f = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 1.0 + 2 ** -9], np.float32)
    got = synth.bf16_to_f32(synth.f32_to_bf16(f))
    assert list(got) == [1.0, 1.0, 1.0 + 2 ** -6, -2.5, 1.0]


def test_logical_values_do_not_depend_on_degree():
    cfg = synth.CONFIGS["tiny"]
    q = synth.logical_tensor(cfg, synth.TID_Q)
    for P in (1, 2, 4):
        xs = synth.to_seq_shards(q, P)
        assert np.array_equal(synth.from_seq_shards(xs, cfg.shape.N), q)


def test_shards_zero_pad_ragged_tail():
    x = synth.normal_bf16(3, 0, 0, 2 * 11 * 4 * 8).reshape(2, 11, 4, 8)
    xs = synth.to_seq_shards(x, 4)
    assert xs.shape == (4, 2, 3, 4, 8)
    assert not xs[3][:, 2:].any()          # tokens 11 of 12 slots: slot 11 pad
    assert np.array_equal(xs[1][1, 0], x[1, 3])


def test_k_modifications():
    c480 = synth.CONFIGS["480p"]
    small = synth.Config("k15", synth.Shape(1, 64, 2, 8, 2), seed=c480.seed, k_mul=1.5)
    k = synth.bf16_to_f32(synth.logical_tensor(small, synth.TID_K))
    ref = synth.bf16_to_f32(synth.normal_bf16(c480.seed, synth.TID_K, 0, k.size, 1.5))
    assert np.array_equal(k.ravel(), ref)
    out_cfg = synth.Config("o", synth.Shape(1, 5000, 2, 8, 2), seed=4, k_outlier_frac=0.001)
    rows = synth.outlier_rows(out_cfg)
    assert len(rows) == 5 and len(set(rows.tolist())) == 5
    k = synth.bf16_to_f32(synth.logical_tensor(out_cfg, synth.TID_K))
    base = synth.bf16_to_f32(synth.normal_bf16(4, synth.TID_K, 0, k.size)).reshape(k.shape)
    assert np.array_equal(k[:, rows], base[:, rows] * 8)
    mask = np.ones(5000, bool)
    mask[rows] = False
    assert np.array_equal(k[:, mask], base[:, mask])
    big = synth.CONFIGS["1344x768"]
    assert len(synth.outlier_rows(big)) == 125


def test_sampled_rows_cover_boundaries():
    cfg = synth.CONFIGS["720p"]
    rows = synth.sampled_rows(cfg, 256, extra_P=(1, 2, 8))
    s = cfg.shape
    assert len(rows) == 256 and len(set(rows.tolist())) == 256
    for t in (0, s.N - 1, 18900 - 1, 18900, 37800, 56700, 9450, 9450 - 1):
        assert t in rows


def test_fp8_quantisation_groups():
    """Q/K factors per (batch, head, 128-token block), V factors per (batch,
    head, channel): each group's largest magnitude becomes 448 exactly, and
    every dequantized value is within E4M3's rounding of the bf16 value."""
    import torch
    cfg = synth.Config("f8", synth.Shape(2, 300, 3, 16, 1), seed=11)
    q, k, v = (synth.bf16_to_f32(x) for x in synth.qkv_logical(cfg))
    q8, k8, v8, dq, dk, dv = synth.fp8_qkv(cfg)
    assert dq.shape == dk.shape == (2, 3, 3) and dv.shape == (2, 3, 16)

    def val(x8):
        return torch.from_numpy(x8).view(torch.float8_e4m3fn).float().numpy()

    tok = np.arange(300) // 128
    for x, x8, d in ((q, q8, dq), (k, k8, dk)):
        deq = val(x8) * d.transpose(0, 2, 1)[:, tok, :, None]
        groups = np.abs(val(x8)).max(axis=3)                      # [B][N][H]
        for blk in range(3):
            sel = tok == blk
            assert np.all(groups[:, sel].max(axis=1) == 448.0)
        bound = 2.0 ** -4 * np.abs(x) + 2.0 ** -10 * d.transpose(0, 2, 1)[:, tok, :, None]
        assert np.all(np.abs(deq - x) <= bound)
    deq_v = val(v8) * dv[:, None]
    assert np.all(np.abs(val(v8)).max(axis=1) == 448.0)
    assert np.all(np.abs(deq_v - v) <= 2.0 ** -4 * np.abs(v) + 2.0 ** -10 * dv[:, None])


def test_cube_mask_and_attended_pairs():
    cfg = synth.Config("m", synth.Shape(2, 1000, 3, 128, 1), seed=5)
    m = synth.cube_mask(cfg, density=0.2, group=4)
    nc = 16                                            # ceil(1000 / 64)
    assert m.shape == (2, 3, nc, nc) and m.dtype == bool
    assert np.array_equal(m[:, :, 0], m[:, :, 3]) and np.array_equal(m[:, :, 12], m[:, :, 15])
    assert 0.1 < m.mean() < 0.3
    assert np.array_equal(m, synth.cube_mask(cfg, density=0.2, group=4))
    # brute force over tokens on a small case
    small = synth.Config("s", synth.Shape(1, 150, 1, 16, 1), seed=6)
    ms = synth.cube_mask(small, density=0.5, group=1)
    tok = np.arange(150) // 64
    brute = ms[0, 0][tok][:, tok].sum()
    assert synth.attended_pairs(ms, 150) == brute
