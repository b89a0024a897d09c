"""The README's usage example runs as written on the GPU (the documented
calls and shapes stay true)."""
import os
import re

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_readme_example_runs():
    pytest.importorskip("w4a4_post_quantization_b200")
    text = open(os.path.join(ROOT, "README.md")).read()
    blocks = re.findall(r"```python\n(.*?)```", text, flags=re.S)
    assert blocks, "README has a python example"
    scope = {}
    exec(compile(blocks[0], "README.md", "exec"), scope)
    y, q, s = scope["y"], scope["q"], scope["s"]
    assert tuple(y.shape) == (4096, 3072) and tuple(q.shape) == (4096, 1536)
    assert tuple(s.shape) == (4096, 96)
