"""Shared helpers of the GPU parity tests: device transfer, full-path runners and report lines."""
from __future__ import annotations

import json
import os

import numpy as np
import torch


def lib():
    """The CUDA binding, built in-tree first if needed (the GPU machine has nvcc)."""
    from long_context_sparse_mean_b200 import build
    build.build()
    from long_context_sparse_mean_b200 import binding
    return binding


def dev(x, dtype):
    return torch.from_numpy(np.ascontiguousarray(x)).to(dtype).cuda()


def kdtype(wl):
    return torch.bfloat16 if wl.dtype == "bf16" else torch.float32


def host(t):
    return t.detach().cpu().numpy()


def report(name, **kv):
    """Print one summary line (tie-band swaps, recalls, IoU) and append it to gpu_parity.jsonl."""
    line = json.dumps({"case": name, **kv})
    print(line)
    out = os.environ.get("MISA_PARITY_LOG")
    if out:
        with open(out, "a") as f:
            f.write(line + "\n")
