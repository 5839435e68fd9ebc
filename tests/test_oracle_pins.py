"""CPU: the fp64 oracle against facts fixed outside itself (closed forms, library
routines, invariants and the pages' worked examples)."""
import json
import os

import pytest

import oracle
import workloads
from oracle_pins import ALL_PINS, GOLDEN


@pytest.fixture(scope="module")
def o():
    return oracle.default()


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda f: f.__name__)
def test_pin(o, pin):
    pin(o)


def test_kv_byte_accounting_matches_worked_examples():
    """The byte-accounting helper reproduces the KV-cache sizes worked on the page
    about KV caches (exercises 1 and 2, and the LLaMA-65B example)."""
    g = json.load(open(os.path.join(GOLDEN, "kv_cache_bytes.json")))
    for c in g["cases"]:
        per_tok = workloads.kv_cache_bytes_per_token(c["layers"], c["kv_heads"], c["head_dim"],
                                                     c["elem_bytes"])
        assert per_tok == c["bytes_per_token"], c["what"]
        assert per_tok * c["tokens"] == c["total_bytes"], c["what"]
    # The GQA exercise is exactly one quarter of the MHA one.
    assert g["cases"][1]["total_bytes"] * 4 == g["cases"][0]["total_bytes"]


def test_bf16_widening_exact(o):
    assert o.bf16_to_double(0x3F80) == 1.0
    assert o.bf16_to_double(0xC000) == -2.0
    assert o.bf16_to_double(0x3F81) == 1.0 + 2.0 ** -7
    assert o.bf16_to_double(0x0001) == 2.0 ** -133
