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
    ("shard-interleaves-tokens", "int64_t t = r * Nl + n;", "int64_t t = n * P + r;"),
    ("shard-pads-with-last-token",
     "xs[dst] = t < N ? x[((b * N + t) * H + h) * D + c] : 0;",
     "xs[dst] = x[((b * N + (t < N ? t : N - 1)) * H + h) * D + c];"),
    ("unshard-wrong-rank", "int64_t r = t / Nl, n = t % Nl;", "int64_t r = t % P, n = t / P;"),
    ("scale-dropped", "s[kk] = J->scale * dot;", "s[kk] = dot;"),
    ("lse-sign", "m + log(l)", "m - log(l)"),
    ("no-normalisation", "o[c] /= l;", "o[c] /= 1.0;"),
    ("exp-sign", "exp(s[kk] - m)", "exp(m - s[kk])"),
    ("sum-of-squares", "l += w;", "l += w * w;"),
    ("v-uses-query-token", "int64_t vr = ((b * N + kk) * H + h) * D;",
     "int64_t vr = ((b * N + i) * H + h) * D;"),
    ("k-wrong-head", "int64_t kr = ((b * N + kk) * H + h) * D;",
     "int64_t kr = ((b * N + kk) * H + (H - 1 - h)) * D;"),
    ("q-head-zero", "int64_t qi = ((b * N + i) * H + h) * D;",
     "int64_t qi = ((b * N + i) * H + 0) * D;"),
    ("dot-drops-last-channel", "for (int64_t c = 0; c < D; ++c)\n            dot +=",
     "for (int64_t c = 0; c + 1 < D; ++c)\n            dot +="),
    ("second-pass-drops-last-key",
     "for (int64_t kk = 0; kk < N; ++kk) {\n        if (s[kk] == -INFINITY) continue;\n        double w",
     "for (int64_t kk = 0; kk + 1 < N; ++kk) {\n        if (s[kk] == -INFINITY) continue;\n        double w"),
    ("k-transposed-with-q",
     "elem(J->k, J->k8, sk, kr + c);",
     "elem(J->q, J->q8, sq, qi + c);"),
    ("e4m3-exponent-bias", "else v = ldexp(1.0 + (double)m / 8.0, e - 7);",
     "else v = ldexp(1.0 + (double)m / 8.0, e - 8);"),
    ("e4m3-subnormal-scale", "if (e == 0) v = ldexp((double)m / 8.0, -6);",
     "if (e == 0) v = ldexp((double)m / 8.0, -7);"),
    ("descale-dropped", "return e4m3_to_f64(x8[e]) * scale;",
     "return e4m3_to_f64(x8[e]);"),
    ("q-factor-first-head-only", "J->dq[bh * J->nblk + i / J->blk]",
     "J->dq[i / J->blk]"),
    ("q-factor-next-block", "J->dq[bh * J->nblk + i / J->blk]",
     "J->dq[bh * J->nblk + (i + 1) / J->blk - ((i + 1) / J->blk == J->nblk)]"),
    ("k-factor-of-query-block", "J->dk[bh * J->nblk + kk / J->blk]",
     "J->dk[bh * J->nblk + i / J->blk]"),
    ("v-factor-of-channel-0", "J->dv[bh * D + c]", "J->dv[bh * D]"),
    ("v-takes-q-factor", "J->v8 ? J->dv[bh * D + c] : 1.0", "J->v8 ? sq : 1.0"),
    ("mask-query-cube-off-by-one", "(bh * J->ncube + i / J->cube) * J->ncube",
     "(bh * J->ncube + (i + 1) / J->cube - ((i + 1) / J->cube == J->ncube)) * J->ncube"),
    ("mask-key-cube-of-query", "if (sel && !sel[kk / J->cube]) {",
     "if (sel && !sel[i / J->cube]) {"),
    ("mask-head-ignored", "J->mask + (bh * J->ncube + i / J->cube) * J->ncube",
     "J->mask + (b * H * J->ncube + i / J->cube) * J->ncube"),
    ("linear-bias-dropped", "yr[c] = acc + (J->bias ? bf16_to_f64(J->bias[c]) : 0.0);",
     "yr[c] = acc;"),
    ("linear-weight-row-of-next-feature", "const uint16_t *wc = J->w + c * J->K;",
     "const uint16_t *wc = J->w + ((c + 1) % J->nout) * J->K;"),
    ("linear-drops-last-input", "for (int64_t k = 0; k < J->K; ++k) acc +=",
     "for (int64_t k = 0; k + 1 < J->K; ++k) acc +="),
    ("linear-row-ignored", "const uint16_t *xr = J->x + J->rows[r] * J->K;",
     "const uint16_t *xr = J->x + r * J->K;"),
    ("mask-empty-row-not-zero", "        if (J->out_lse) J->out_lse[r] = -INFINITY;\n        return;",
     "        if (J->out_lse) J->out_lse[r] = -INFINITY;\n        o[0] = 1.0;\n        return;"),
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
