"""Write the oracle regression fixtures in this folder.

Calls only the oracle (oracle/) and the seeded input generator (workloads/).
The page ("Latent-Condensed Transformer for Efficient Long Context Modeling")
prints no worked numeric example, so no fixture here holds a value taken from
the page; these files freeze the oracle's own output on tiny seeded cases so
that an unintended change to its arithmetic shows up as a diff.

Run from the repository root:  python tests/golden/make_golden.py
"""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

from oracle import oracle as orc  # noqa: E402
import workloads  # noqa: E402

CASES = [
    workloads.small("golden_f32", B=1, H=2, L=29, g=4, w=5, d_c=8, d_r=4, dtype="f32", seed=3),
    workloads.small("golden_bf16", B=1, H=2, L=37, g=8, w=3, d_c=16, d_r=8, dtype="bf16", seed=4),
]


def main() -> None:
    for wl in CASES:
        x = workloads.generate(wl, threads=1)
        res = orc.lca(x.q_c, x.q_r, x.c_kv, x.k_r, g=wl.g, w=wl.w)
        dense = orc.mla(x.q_c, x.q_r, x.c_kv, x.k_r)
        doc = {
            "source": "oracle/lca_oracle.c via tests/golden/make_golden.py (regression, not page values)",
            "workload": {k: getattr(wl, k) for k in ("B", "H", "d_c", "d_r", "L", "g", "w", "dtype", "seed",
                                                      "q_scale", "kv_scale")},
            "lca_out": [[float.hex(float(v)) for v in row] for row in res.out[0]],
            "lca_anchor": res.anchor[0].tolist(),
            "mla_out": [[float.hex(float(v)) for v in row] for row in dense[0]],
        }
        with open(os.path.join(HERE, f"{wl.name}.json"), "w") as f:
            json.dump(doc, f, indent=1)
            f.write("\n")


if __name__ == "__main__":
    main()
