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


# The MLA backward is composed in the oracle's Python front end (the GQA backward on the key
# [latent | rope], value latent); its plausible mistakes are planted there, on the CPU.
def _mla_bwd_drop_value_term(orc):
    """The latent's gradient keeps only its key part (the value part P dO is dropped)."""
    import torch

    def bad(q_latent, q_rope, latent_cache, rope_cache, d_out, seq_lens, query_offsets, block_tables, page_size,
            scale, causal=True, window=0, nthreads=None):
        r = q_latent.shape[2]
        dq, dk, _ = orc.attention_backward(torch.cat([q_latent, q_rope], 2), torch.cat([latent_cache, rope_cache], 3),
                                           latent_cache, d_out, seq_lens, query_offsets, block_tables, page_size,
                                           scale, causal, window, nthreads)
        return dq[..., :r], dq[..., r:], dk[..., :r], dk[..., r:]
    return bad


def _mla_bwd_swapped_rope(orc):
    """The rope gradient is taken from the latent columns (a wrong column split)."""
    real = orc.mla_backward

    def bad(*a, **k):
        dql, dqr, dlat, drope = real(*a, **k)
        pr = drope.shape[-1]
        return dql, dql[..., :pr].clone(), dlat, dlat[..., :pr].clone()
    return bad


@pytest.mark.parametrize("plant", [_mla_bwd_drop_value_term, _mla_bwd_swapped_rope])
def test_pins_reject_mla_backward_mistakes(plant):
    orc = oracle.get()
    bad = oracle.Oracle(orc.path) if hasattr(orc, "path") else orc
    original = bad.mla_backward
    bad.mla_backward = plant(bad)
    try:
        with pytest.raises(AssertionError):
            oracle_pins.pin_mla_backward_finite_differences(bad)
    finally:
        bad.mla_backward = original
