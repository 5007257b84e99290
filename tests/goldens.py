"""Reader of the hand-worked golden groups in tests/golden/quant_worked_groups.txt.

Shared by the oracle's pins and by the GPU test that runs the same groups
through libcf; it holds no codec arithmetic, only the fixture format.
"""
import os

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "quant_worked_groups.txt")


def read_golden():
    cases, cur = {}, None
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        if line.startswith("["):
            cur = cases.setdefault(line[1:-1], {})
            continue
        k, v = [s.strip() for s in line.split("=", 1)]
        cur[k] = v
    return cases


def num(v):
    """A fixture number: decimal, or a C99 hex float such as 0x1p-120."""
    v = v.strip()
    return float.fromhex(v) if v.lstrip("+-").lower().startswith("0x") else float(v)


def floats(s):
    return np.array([num(v) for v in s.split(",")], np.float32)


def bf16(values):
    """Raw bf16 bit patterns of values that must be exact in bf16."""
    t = torch.tensor(values, dtype=torch.float32)
    b = t.to(torch.bfloat16)
    assert torch.equal(b.float(), t), "fixture values must be exact in bf16"
    return b.view(torch.int16).numpy().view(np.uint16).copy()


CASES = read_golden()
