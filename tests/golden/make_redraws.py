"""Write the redraw tables for the synthetic layer configurations.

Each configuration's hidden rows are drawn from the seeded generator; a row
whose router logits (computed by the oracle, from the rounded inputs) have a
gap smaller than 1e-3 anywhere among the top k+1 is redrawn with the next
attempt index until every row passes.  The table {(step, row): attempt} is
stored as JSON so the benchmark uses the very same inputs without running the
oracle.  Calls only the oracle and the generator.

    python tests/golden/make_redraws.py [config ...]
"""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import synth  # noqa: E402


def screen(name: str, T: int, steps: int, seed: int = 0):
    cfg = synth.CONFIGS[name]
    layer = synth.Layer(cfg, seed)
    Wr = layer.router_f32()
    b = layer.bias()

    def ok(x):
        return oracle.margin_ok(oracle.router_logits(x, Wr, b), cfg.k, synth.MARGIN)

    return synth.screen_hidden(layer, T, steps, ok)


def write(name: str, T: int, steps: int, seed: int = 0) -> str:
    table = screen(name, T, steps, seed)
    path = synth.redraw_path(name, T)
    with open(path, "w") as f:
        json.dump({"config": name, "T": T, "steps": steps, "seed": seed, "margin": synth.MARGIN,
                   "redraws": sorted([s, r, a] for (s, r), a in table.items())}, f)
    return path


JOBS = {
    "tiny": [(16, 1)],
    "35b_decode": [(64, 1)],
    "35b_prefill": [(8192, 1)],
    "284b_trace": [(32, 256)],
    "753b_nvfp4": [(16384, 1)],
}

if __name__ == "__main__":
    names = sys.argv[1:] or list(JOBS)
    for n in names:
        for T, steps in JOBS[n]:
            print(write(n, T, steps))
