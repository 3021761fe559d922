"""The README's decode-step example runs as written."""
import os
import re

import pytest

pytestmark = pytest.mark.gpu


def test_readme_decode_example_runs(pkv):
    path = os.path.join(os.path.dirname(os.path.dirname(__file__)),
                        "README.md")
    blocks = re.findall(r"```python\n(.*?)```", open(path).read(), re.S)
    scope = {}
    exec(compile(blocks[0], "README.md", "exec"), scope)
    import torch
    out = scope["out"]
    torch.cuda.synchronize()
    assert out.shape == (2, 64, 128) and torch.isfinite(out.float()).all()
    # one token per sequence: the output is that token's V, head by head
    v = scope["v_new"].float().repeat_interleave(8, dim=1)
    assert (out.float() - v).abs().max().item() <= 1e-2
