"""The fp64 backward oracle against its pins, and plausible mistakes planted in
a temporary copy of its C source that the pins must catch (CPU only)."""
import os

import pytest

import oracle
from tests import oracle_bwd_pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "attn_bwd_oracle.c")


@pytest.fixture(scope="module")
def lib():
    return oracle.load_bwd_library(oracle.build_bwd())


@pytest.mark.parametrize("pin", oracle_bwd_pins.ALL_BWD_PINS, ids=lambda f: f.__name__)
def test_bwd_oracle_pin(lib, pin):
    pin(lib)


MUTANTS = [
    ("D term dropped", [("dp[j] = p[j] * (acc - Di);", "dp[j] = p[j] * acc;")]),
    ("scale dropped from dQ and dK", [("const double ds = sigma * dp[j];", "const double ds = dp[j];")]),
    ("dV from dS instead of P", [("dvj[c] += p[j] * doi[c];", "dvj[c] += dp[j] * doi[c];")]),
    ("dK from dO instead of Q", [("dkj[c] += ds * qi[c];", "dkj[c] += ds * doi[c];")]),
    ("D from Q instead of O", [("Di += doi[c] * oi[c];", "Di += doi[c] * qi[c];")]),
    ("dQ from V instead of K", [("dqi[c] += ds * bf16_to_double(kj[c]);",
                                 "dqi[c] += ds * bf16_to_double(vb[(int64_t)j * d + c]);")]),
    ("softmax not normalised", [("for (int j = 0; j < end; ++j) p[j] /= l;", "")]),
    ("causal mask off by one", [("(int64_t)i + 1 + Nk - N < end) end = (int)((int64_t)i + 1 + Nk - N);",
                                 "(int64_t)i + Nk - N < end) end = (int)((int64_t)i + Nk - N);")]),
    ("only the first head of a group", [("for (int h = hk * group; h < (hk + 1) * group; ++h)",
                                         "for (int h = hk * group; h < hk * group + 1; ++h)")]),
    ("key padding ignored", [("L = k_len[b];", "L = Nk;")]),
]


@pytest.mark.parametrize("name,edits", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_bwd_pins_catch_mutant(tmp_path, name, edits):
    src = open(SRC).read()
    for old, new in edits:
        assert src.count(old) >= 1, f"mutation target missing: {old!r}"
        src = src.replace(old, new)
    p = tmp_path / "mutant.c"
    p.write_text(src)
    lib = oracle.load_bwd_library(oracle.build_bwd(force=True, src=str(p), out=str(tmp_path / "libmutant.so")))
    caught = []
    for pin in oracle_bwd_pins.ALL_BWD_PINS:
        try:
            pin(lib)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin caught the planted mistake '{name}'"
