"""The Python example in README.md runs as written (on the GPU)."""
import os
import re

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.gpu
def test_readme_example_runs():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    with open(os.path.join(ROOT, "README.md")) as f:
        code = re.search(r"```python\n(.*?)```", f.read(), re.S).group(1)
    scope = {}
    exec(compile(code, "README.md", "exec"), scope)
    torch.cuda.synchronize()
    master, ag = scope["master"], scope["ag"]
    assert torch.isfinite(master).all()
    # the fused call wrote the bf16 copy of the updated master
    assert torch.equal(ag, master.to(torch.bfloat16))
