"""The oracle and the input recipe respect the constants the pages fix
(tests/golden/pages_constants.txt, each line cited)."""
import os

import numpy as np

from cell_updates_b200 import synth
from oracle import c_oracle as co
from oracle import np_oracle as no

HERE = os.path.dirname(os.path.abspath(__file__))


def _constants():
    out = {}
    with open(os.path.join(HERE, "golden", "pages_constants.txt")) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                k, v = (t.strip() for t in line.split("=", 1))
                out[k] = v
    return out


def test_group_size_and_widths():
    c = _constants()
    g = int(c["group_size"])
    widths = [int(v) for v in c["widths"].split(",")]
    assert no.GROUP == g
    w = np.linspace(-1, 1, 2 * g, dtype=np.float32).reshape(1, 2 * g)
    for b in range(0, 10):
        _, _, _, st = co.quantize(w, np.array([b, b], np.uint8))
        assert (st == 0) == (b in widths), b
    assert int(c["release_bits"]) in widths


def test_vbq_recipe_matches_allocation_statistics():
    c = _constants()
    bits = synth.vbq_bits(1 << 18, seed=2)
    assert abs((bits == 1).mean() - float(c["frac_groups_1bit"])) < 0.005
    # the drawn recipe's mean width is within 0.05 bits of the page's 1.82
    assert abs(bits.mean() - float(c["mean_bits"])) < 0.05


def test_verify_scale_is_reachable_in_chunks():
    c = _constants()
    n = float(c["verified_weights"])
    # the chunked verify API addresses weights with 64-bit indices
    assert n < 2 ** 63 and n % 64 == 0
