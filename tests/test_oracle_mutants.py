"""Plants plausible mistakes in copies of the oracle source and checks that
the pins catch every one (CPU only; the oracle itself is never modified)."""
import pytest

import oracle
from oracle_pins import ALL_CHECKS

# (name, exact text in sp_oracle.c, replacement)
MUTANTS = [
    ("pack-swaps-rank-and-group",
     "int64_t src = (((r * B + b) * Nl + n) * H + (j * Hl + hh)) * D + c;\n"
     "                            int64_t dst",
     "int64_t src = (((j * B + b) * Nl + n) * H + (r * Hl + hh)) * D + c;\n"
     "                            int64_t dst"),
    ("unpack-interleaves-tokens",
     "int64_t src = (((j * B + b) * Np + (r * Nl + n)) * Hl + hh) * D + c;",
     "int64_t src = (((j * B + b) * Np + (n * P + r)) * Hl + hh) * D + c;"),
    ("pack-wrong-local-head",
     "(j * Hl + hh)) * D + c;\n                            int64_t dst",
     "(j * Hl + (Hl - 1 - hh))) * D + c;\n                            int64_t dst"),
    ("exchange-pack-wrong-head",
     "xs_r[((b * Nl + n) * H + (j * Hl + hh)) * D + c];",
     "xs_r[((b * Nl + n) * H + (hh * P + j)) * D + c];"),
    ("exchange-unpack-wrong-chunk",
     "recv[(((j * B + b) * Nl + n) * Hl + hh) * D + c];",
     "recv[((((P - 1 - j) * B + b) * Nl + n) * Hl + hh) * D + c];"),
    ("scale-dropped", "s[kk] = J->scale * dot;", "s[kk] = dot;"),
    ("lse-sign", "m + log(l)", "m - log(l)"),
    ("no-normalisation", "o[c] /= l;", "o[c] /= 1.0;"),
    ("exp-sign", "exp(s[kk] - m)", "exp(m - s[kk])"),
    ("sum-of-squares", "l += w;", "l += w * w;"),
    ("v-uses-query-token", "J->v + ((b * N + kk) * H + h) * D",
     "J->v + ((b * N + i) * H + h) * D"),
    ("k-wrong-head", "J->k + ((b * N + kk) * H + h) * D",
     "J->k + ((b * N + kk) * H + (H - 1 - h)) * D"),
    ("q-head-zero", "J->q + ((b * N + i) * H + h) * D",
     "J->q + ((b * N + i) * H + 0) * D"),
    ("dot-drops-last-channel", "for (int64_t c = 0; c < D; ++c) dot +=",
     "for (int64_t c = 0; c + 1 < D; ++c) dot +="),
    ("second-pass-drops-last-key",
     "for (int64_t kk = 0; kk < N; ++kk) {\n        double w",
     "for (int64_t kk = 0; kk + 1 < N; ++kk) {\n        double w"),
    ("k-transposed-with-q", "dot += bf16_to_f64(qi[c]) * bf16_to_f64(kr[c]);",
     "dot += bf16_to_f64(qi[c]) * bf16_to_f64(qi[c]);"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_kill_mutant(name, old, new, tmp_path):
    src = oracle.source_text()
    assert src.count(old) == 1, f"mutation site for {name} not unique"
    lib = oracle.build_variant(src.replace(old, new), str(tmp_path / f"m_{name}.so"))
    failed = []
    for check in ALL_CHECKS:
        try:
            check(lib=lib)
        except (AssertionError, ValueError, RuntimeError, FloatingPointError):
            failed.append(check.__name__)
    assert failed, f"no pin caught mutant {name}"
