"""Writes ``pr1_ref_seed0.txt``: oracle outputs for the small fp32 reference workload.

The workload is B1 H2 T256 dk = dv = 32, C32, float32 q/k/v ~ N(0, 1) drawn on the CPU
from seed 0, ELU+1 feature map, normalised, no decay.  This script calls only the
oracle (and the seeded input generator); no value in the file comes from the CUDA path.

Run from the repository root:  python tests/golden/make_golden.py
"""

from __future__ import annotations

import sys
from pathlib import Path

import numpy as np

HERE = Path(__file__).resolve().parent
ROOT = HERE.parent.parent
if str(ROOT) not in sys.path:
    sys.path.insert(0, str(ROOT))

FILE = HERE / "pr1_ref_seed0.txt"
SAMPLE_T = (0, 1, 2, 31, 32, 33, 100, 127, 128, 200, 254, 255)


def compute_golden(oracle=None) -> dict[str, np.ndarray]:
    from chunked_causal_linear_b200.workloads import WORKLOADS, make_inputs
    if oracle is None:
        from oracle.oracle import default_oracle
        oracle = default_oracle()
    w = WORKLOADS["pr1_ref"]
    q, k, v = make_inputs(w, seed=0, device="cpu")
    out, S, Z = oracle.forward(q.numpy(), k.numpy(), v.numpy(), feature_map=w.feature_map,
                               gamma=w.gammas(), normalize=w.normalize)
    return {"out_sampled": out[:, :, list(SAMPLE_T), :], "S_final": S, "Z_final": Z}


def write_golden(values: dict[str, np.ndarray]) -> None:
    lines = [
        "# Oracle outputs for the small fp32 reference workload (B1 H2 T256 d32 C32, fp32",
        "# N(0,1) from a CPU generator seeded with 0, elu+1, normalised, no decay).",
        "# Written by tests/golden/make_golden.py, which calls only the fp64 oracle.",
        f"# out_sampled holds out[:, :, t, :] for t in {list(SAMPLE_T)}.",
        "# format: name shape, then one value per line (repr of a double).",
    ]
    for name, arr in values.items():
        lines.append(f"@ {name} {' '.join(str(s) for s in arr.shape)}")
        lines.extend(repr(float(x)) for x in arr.reshape(-1))
    FILE.write_text("\n".join(lines) + "\n")


def load_golden() -> dict[str, np.ndarray]:
    values: dict[str, np.ndarray] = {}
    name, shape, buf = None, None, []
    for line in FILE.read_text().splitlines():
        if line.startswith("#") or not line.strip():
            continue
        if line.startswith("@"):
            if name is not None:
                values[name] = np.array(buf, dtype=np.float64).reshape(shape)
            parts = line.split()
            name, shape, buf = parts[1], tuple(int(s) for s in parts[2:]), []
        else:
            buf.append(float(line))
    if name is not None:
        values[name] = np.array(buf, dtype=np.float64).reshape(shape)
    return values


if __name__ == "__main__":
    write_golden(compute_golden())
    print(f"wrote {FILE}")
