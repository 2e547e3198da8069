"""Write tests/golden/*.txt from the fp64 oracle (this script calls only oracle/).

alice_fixture_gqa.txt: the deterministic GQA fixture of alice-llm's llama3_bridge tests
(`fixture_gqa`: tq=3, hq=4, hkv=2, head_dim=8, seq_len=12, q = sin(0.05 i), k = cos(0.07 i),
v = sin(0.03 i) over the flat index; non-causal; scale 1/sqrt(8)), laid out in pages of 4 with
an identity block table. The page prints the fixture's inputs, not its outputs, so the stored
outputs are the oracle's; the oracle itself is pinned to torch's fp64 SDPA on this fixture.
Format: one line per (query, head): `q h lse out[0..7]`, floats as Python repr.
"""
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))
sys.path.insert(0, os.path.dirname(HERE))

import oracle  # noqa: E402
import oracle_pins  # noqa: E402


def main():
    q, k, v, sl, qo, bt, ps, scale = oracle_pins.alice_fixture()
    out, lse = oracle.get().attention(q, k, v, sl, qo, bt, ps, scale, causal=False, window=0)
    lines = ["# alice-llm fixture_gqa through the fp64 oracle: q h lse out[0..7]"]
    for i in range(out.shape[0]):
        for h in range(out.shape[1]):
            vals = " ".join(repr(float(x)) for x in out[i, h])
            lines.append(f"{i} {h} {float(lse[i, h])!r} {vals}")
    with open(os.path.join(HERE, "alice_fixture_gqa.txt"), "w") as f:
        f.write("\n".join(lines) + "\n")


if __name__ == "__main__":
    main()
