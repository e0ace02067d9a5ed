"""Pins of the fp64 oracle (CPU only).  See tests/oracle_pins.py."""
import json
import os

import numpy as np
import pytest

import oracle
import synth
from oracle_pins import ALL_CHECKS

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.mark.parametrize("check", ALL_CHECKS, ids=lambda c: c.__name__)
def test_oracle_pin(check):
    check()


def test_oracle_degree_rule_golden():
    """The pages' head/degree examples: valid degrees split the heads evenly,
    others are rejected."""
    with open(os.path.join(GOLDEN, "degree_rule.json")) as f:
        g = json.load(f)
    for case in g["valid"]:
        H, P = case["heads"], case["degree"]
        xs = np.zeros((P, 1, 2, H, 8), dtype=np.uint16)
        xh = oracle.pack(xs, 2 * P)
        assert xh.shape[3] == case["heads_per_rank"]
    for case in g["invalid"]:
        H, P = case["heads"], case["degree"]
        with pytest.raises(ValueError):
            oracle.pack(np.zeros((P, 1, 2, H, 8), dtype=np.uint16), 2 * P)


def test_oracle_pack_on_tiny_config_round_trip():
    cfg = synth.CONFIGS["tiny"]
    s = cfg.shape
    q = synth.logical_tensor(cfg, synth.TID_Q)
    xs = synth.to_seq_shards(q, s.P)
    xh = oracle.pack(xs, s.N)
    assert xh.shape == (s.P, s.B, s.Np, s.Hl, s.D)
    assert np.array_equal(oracle.unpack(xh, s.N, s.H), xs)
