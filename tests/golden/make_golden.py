"""Write tests/golden/tiny_oracle_anchor.json from the oracle alone.

The anchor freezes a few oracle outputs of the tiny workload (T=64, d=256,
ffn=512, seed 0) so that any later change to the oracle's arithmetic shows up
as a failing test.  Run:  python tests/golden/make_golden.py
"""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import moe_synth  # noqa: E402
import oracle  # noqa: E402


def main():
    inp = moe_synth.make_inputs("tiny", device="cpu")
    tokens = [0, 1, 31, 63]
    out, idx, gate = oracle.forward(inp.layers[0], inp.x, tokens=tokens)
    doc = {
        "_about": "oracle output anchor for the tiny workload (written by make_golden.py, oracle only)",
        "workload": "tiny: T=64, d=256, ffn=512, E=8, k=2, seed 0",
        "input_checksum": {"wl_sum": int(inp.layers[0]["wl"].to(torch.int64).sum())},
        "tokens": tokens,
        "idx": idx.tolist(),
        "gate": gate.tolist(),
        "out_head": out[:, :16].tolist(),
    }
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_oracle_anchor.json")
    with open(path, "w") as f:
        json.dump(doc, f, indent=1)
    print("wrote", path)


if __name__ == "__main__":
    main()
