"""Plant plausible mistakes in a copy of the oracle's C source and check that
the pin suite catches every one.  The mistakes are planted in the oracle, on
the CPU, in a temporary directory; the committed oracle is never modified."""
import os

import pytest

import oracle
from tests import oracle_pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "attn_oracle.c")

# (name, [(original text, mistaken text), ...])
MUTANTS = [
    ("causal mask off by one", [("(int64_t)i + 1 + Nk - N < allowed_end)\n                allowed_end = (int)((int64_t)i + 1 + Nk - N);",
                                 "(int64_t)i + Nk - N < allowed_end)\n                allowed_end = (int)((int64_t)i + Nk - N);")]),
    ("scale dropped", [("s[j] = sigma * acc;", "s[j] = acc;")]),
    ("scale applied twice", [("s[j] = sigma * acc;", "s[j] = sigma * sigma * acc;")]),
    ("max missing from lse", [("lse[t] = m + log(l);", "lse[t] = log(l);")]),
    ("key padding ignored", [("L = k_len[b];", "L = N;")]),
    ("batch index of key length", [("const int b = (int)(bh / H);", "const int b = (int)(bh % H);")]),
    ("output sums K instead of V", [("const uint16_t *vj = vb + (int64_t)j * d;",
                                     "const uint16_t *vj = kb + (int64_t)j * d;")]),
    ("softmax not normalised", [("const double p = s[j] / l;", "const double p = s[j];")]),
    # query row i taken from K and key j from Q (j wrapped into the query range so the
    # mistaken reads stay inside the buffers): the transposed score matrix when N_q = N_k
    ("transposed scores", [("const uint16_t *qi = q + r * d;", "const uint16_t *qi = k + (bh_kv * Nk + i) * d;"),
                           ("const uint16_t *kj = kb + (int64_t)j * d;",
                            "const uint16_t *kj = q + (bh * N + j % N) * d;")]),
    ("no max subtraction", [("s[j] = exp(s[j] - m);", "s[j] = exp(s[j]);"),
                            ("lse[t] = m + log(l);", "lse[t] = log(l);")]),
    ("sign of dot product", [("acc += qrow[c] *", "acc -= qrow[c] *")]),
    ("output overwritten, not accumulated", [("oi[c] += p *", "oi[c] = p *")]),
    ("last allowed key dropped", [("for (int j = 0; j < allowed_end; ++j) {\n                const double p",
                                   "for (int j = 0; j < allowed_end - 1; ++j) {\n                const double p")]),
    ("empty row gives zero lse", [("lse[t] = -INFINITY;", "lse[t] = 0.0;")]),
    ("grouped head taken modulo", [("h / (H / H_kv);", "h % H_kv;")]),
    ("causal diagonal not shifted", [("allowed_end = (int)((int64_t)i + 1 + Nk - N);", "allowed_end = i + 1;")]),
]


@pytest.mark.parametrize("name,edits", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(tmp_path, name, edits):
    src = open(SRC).read()
    for old, new in edits:
        assert src.count(old) >= 1, f"mutation target missing: {old!r}"
        src = src.replace(old, new)
    p = tmp_path / "mutant.c"
    p.write_text(src)
    lib = oracle.load_library(oracle.build(force=True, src=str(p), out=str(tmp_path / "libmutant.so")))
    caught = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(lib)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin caught the planted mistake '{name}'"
