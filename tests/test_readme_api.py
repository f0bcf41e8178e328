"""The README's Python example calls only functions and constants the binding
defines (CPU: names only, nothing is run)."""
import os
import re

from fp8_block_scaled_11_b200 import ops

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_readme_example_names_exist():
    text = open(os.path.join(ROOT, "README.md")).read()
    code = "\n".join(re.findall(r"```python\n(.*?)```", text, re.S))
    names = set(re.findall(r"\bops\.(\w+)", code))
    assert names, "no ops.* names found in the README example"
    missing = sorted(n for n in names if not hasattr(ops, n))
    assert not missing, missing
