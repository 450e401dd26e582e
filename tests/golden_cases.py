"""Parser for tests/golden/worked_blocks.txt (hand-worked RaZeR rows)."""
import os

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "worked_blocks.txt")


def load_cases(path: str = GOLDEN):
    cases = []
    cur = None
    for line in open(path):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        key, _, rest = line.partition(" ")
        if key == "case":
            cur = {"name": rest}
            cases.append(cur)
        elif key in ("fmt", "dtype"):
            cur[key] = rest
        elif key in ("codes", "scales"):
            cur[key] = np.array([int(t, 16) for t in rest.split()], np.uint8)
        elif key in ("x", "dequant"):
            cur[key] = [float(t) for t in rest.split()]
        elif key in ("ts", "ones"):
            cur[key] = float(rest)
        else:
            raise ValueError(f"unknown key {key}")
    return cases


def case_tensor(case) -> torch.Tensor:
    """The row as a [1, 32] fp16/bf16 CPU tensor (library conversion)."""
    dt = {"f16": torch.float16, "bf16": torch.bfloat16}[case["dtype"]]
    return torch.tensor(case["x"], dtype=torch.float64).to(torch.float32).to(dt).view(1, -1)
