"""The oracle's pins must reject plausible mistakes in the oracle itself.

Each mutant is pa_oracle.c compiled with one PAO_MUTANT_* define (a dropped or wrong term, a
wrong index, an off-by-one mask); it runs on the CPU only. The test passes when at least one
pin from tests/oracle_pins.py fails on it.
"""
import os

import pytest

import oracle
import oracle_pins
from oracle import build as obuild

MUTANTS = [
    "PAO_MUTANT_CAUSAL_STRICT",   # key t == p masked
    "PAO_MUTANT_WINDOW_WIDE",     # window keeps one key too many
    "PAO_MUTANT_IDENTITY_TABLE",  # block table ignored (pages assumed contiguous)
    "PAO_MUTANT_GQA_MODULO",      # query head h reads KV head h % Hkv
    "PAO_MUTANT_LEFT_ALIGNED",    # query j at position j instead of L - n + j
    "PAO_MUTANT_DROP_ROPE",       # MLA positional score term dropped
    "PAO_MUTANT_LSE_NO_MAX",      # lse loses the max shift
    "PAO_MUTANT_UNNORMALISED",    # output not divided by the softmax sum
    "PAO_MUTANT_SCALE_DROPPED",   # scores not scaled
    "PAO_MUTANT_BWD_NO_D",        # backward without the rowsum(dO * O) term
    "PAO_MUTANT_SPARSE_FLOOR",    # partial last block dropped (floor block count)
    "PAO_MUTANT_SPARSE_PROXY_LAST",  # proxy from the last query head of the group
    "PAO_MUTANT_SPARSE_TIES_HIGH",   # equal scores rank the higher block index first
    "PAO_MUTANT_SPARSE_MIN",      # lowest-scoring blocks selected
    "PAO_MUTANT_SPARSE_UNMASKED", # proxy ignores the causal/window mask
]


@pytest.mark.parametrize("mutant", MUTANTS)
def test_pins_reject_mutant(mutant, tmp_path):
    path = obuild.build(str(tmp_path / f"lib_{mutant}.so"), extra_defines=[mutant])
    bad = oracle.Oracle(path)
    failed = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(bad)
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, f"no pin caught {mutant}"
