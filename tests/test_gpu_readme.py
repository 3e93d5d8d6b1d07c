"""The README's single-GPU Python example runs as printed."""
import os
import re

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_readme_single_gpu_example_runs():
    text = open(os.path.join(ROOT, "README.md")).read()
    block = re.findall(r"```python\n(.*?)```", text, re.S)[0]
    exec(compile(block, "README.md", "exec"), {})
