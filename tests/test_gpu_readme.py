"""The README's Python example runs as written (on the GPU) and leaves consistent results."""
import os

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _example():
    lines = open(os.path.join(ROOT, "README.md")).read().splitlines()
    start = lines.index("## Python use") + 1
    block = []
    for line in lines[start:]:
        if line.startswith("## "):
            break
        if line.startswith("    ") or (block and not line.strip()):
            block.append(line[4:])
        elif block and line.strip():
            break
    return "\n".join(block)


def test_readme_example_runs(cuda_device):
    code = _example()
    assert "km.km_fit" in code and "km.km_update_next" in code
    env = {}
    exec(compile(code, "README.md", "exec"), env)
    torch.cuda.synchronize()
    km = env["km"]
    assert km.km_device_error() == 0
    C, counts, ids = env["C"], env["counts"], env["ids"]
    assert torch.isfinite(C).all()
    # the last update's counts are the histogram of the labels it was given
    hist = torch.stack([torch.bincount(ids[b].long(), minlength=1024) for b in range(ids.shape[0])])
    assert torch.equal(hist.to(torch.int32), counts)
