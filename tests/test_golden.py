"""Stored oracle outputs for the alice-llm GQA fixture (tests/golden/make_golden.py)."""
import os

import torch

import oracle_pins

GOLD = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "alice_fixture_gqa.txt")


def load_alice_golden():
    out = torch.empty(3, 4, 8, dtype=torch.float64)
    lse = torch.empty(3, 4, dtype=torch.float64)
    with open(GOLD) as f:
        for line in f:
            if line.startswith("#"):
                continue
            parts = line.split()
            i, h = int(parts[0]), int(parts[1])
            lse[i, h] = float(parts[2])
            out[i, h] = torch.tensor([float(x) for x in parts[3:]], dtype=torch.float64)
    return out, lse


def test_oracle_matches_stored_alice_fixture(orc):
    q, k, v, sl, qo, bt, ps, scale = oracle_pins.alice_fixture()
    out, lse = orc.attention(q, k, v, sl, qo, bt, ps, scale, causal=False, window=0)
    gout, glse = load_alice_golden()
    assert torch.allclose(out, gout, rtol=1e-14, atol=1e-15)
    assert torch.allclose(lse, glse, rtol=1e-14, atol=1e-15)
