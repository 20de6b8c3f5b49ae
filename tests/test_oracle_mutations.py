"""Plant plausible mistakes in a copy of the oracle; the pins must catch each.

The mistake is planted in the oracle's C source (a temporary copy), on the CPU,
and the whole pin set runs against the mutant.  A mutant that passes every pin
would mean the pins leave that part of the oracle unchecked.
"""
import os

import pytest

import oracle_pins
from oracle import Oracle
from oracle import build as oracle_build

MUTATIONS = [
    ("gate and up swapped", "a[i] = silu(g) * u;", "a[i] = silu(u) * g;"),
    ("silu sign", "return g / (1.0 + exp(-g));", "return g / (1.0 + exp(g));"),
    ("router bias dropped", "acc += bias[e];", "acc += 0.0 * bias[e];"),
    ("ties to the higher id", "return ea < eb;", "return ea > eb;"),
    ("no renormalisation", "weights[t * top_k + j] = p[order[j]] / s;",
     "weights[t * top_k + j] = p[order[j]];"),
    ("softmax without the max", "p[e] = exp(l[e] - m);", "p[e] = exp(l[e]);"),
    ("down projection transposed", "acc += bf16_value(w_down[r * I + i]) * a[i];",
     "acc += bf16_value(w_down[i * H + r]) * a[i];"),
    ("remainder on the last ranks", "int64_t share = base + (r < extra ? 1 : 0);",
     "int64_t share = base + (r >= ranks - extra ? 1 : 0);"),
    ("bands summed in reverse rank order", "for (int32_t r = 0; r < nbands; ++r) {",
     "for (int32_t r = nbands - 1; r >= 0; --r) {"),
    ("picks not sorted by id", "while (pos > 0 && ids_t[slot_order[pos - 1]] > ids_t[j]) {",
     "while (0) {"),
    ("shared expert dropped", "yt[h] = yt[h] + f[h];", "yt[h] = yt[h];"),
    ("routing weight dropped", "double c = w_t[j] * f[h];", "double c = f[h];"),
    ("sigmoid sign", "sc[e] = 1.0 / (1.0 + exp(-l));", "sc[e] = 1.0 / (1.0 + exp(l));"),
    ("sigmoid bias ignored in the selection", "key[e] = bias != NULL ? sc[e] + bias[e] : sc[e];",
     "key[e] = sc[e];"),
    ("sigmoid weights from the biased keys",
     "weights[t * top_k + j] = normalize ? scale * (sc[order[j]] / sum) : scale * sc[order[j]];",
     "weights[t * top_k + j] = normalize ? scale * (key[order[j]] / sum) : scale * key[order[j]];"),
    ("sigmoid normalisation ignored",
     "weights[t * top_k + j] = normalize ? scale * (sc[order[j]] / sum) : scale * sc[order[j]];",
     "weights[t * top_k + j] = scale * sc[order[j]];"),
    ("sigmoid scale ignored",
     "weights[t * top_k + j] = normalize ? scale * (sc[order[j]] / sum) : scale * sc[order[j]];",
     "weights[t * top_k + j] = normalize ? (sc[order[j]] / sum) : sc[order[j]];"),
    ("gate row index off by a transpose", "g += bf16_value(w_gate[i * H + h]) * xt[h];",
     "g += bf16_value(w_gate[(i * H + h) % (I * H)]) * xt[(h + 1) % H];"),
]


@pytest.mark.parametrize("what,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_pins_catch_planted_mistake(tmp_path, what, old, new):
    with open(oracle_build.SOURCE) as f:
        text = f.read()
    assert text.count(old) == 1, f"mutation site not found once: {old!r}"
    lib = oracle_build.build_variant(text.replace(old, new), os.path.join(tmp_path, "mutant.so"))
    mutant = Oracle(lib)
    caught = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(mutant)
        except Exception as exc:  # noqa: BLE001 - any failure counts as caught
            caught.append((pin.__name__, type(exc).__name__))
    assert caught, f"no pin caught the planted mistake: {what}"
