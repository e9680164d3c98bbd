"""The README's Python examples stay valid against the binding: every block parses, and every
call to the binding's functions binds to their current signatures."""
import ast
import inspect
import os
import re

from exact_io_aware_93_b200 import api

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _blocks():
    with open(os.path.join(ROOT, "README.md")) as f:
        return re.findall(r"```python\n(.*?)```", f.read(), re.S)


def test_readme_has_examples():
    assert len(_blocks()) >= 3


def test_readme_blocks_parse_and_bind():
    for block in _blocks():
        tree = ast.parse(block)
        for node in ast.walk(tree):
            if not (isinstance(node, ast.Call) and isinstance(node.func, ast.Attribute)):
                continue
            if not (isinstance(node.func.value, ast.Name) and node.func.value.id == "api"):
                continue
            fn = getattr(api, node.func.attr)   # the function exists
            args = [object()] * len(node.args)
            kwargs = {k.arg: object() for k in node.keywords if k.arg is not None}
            inspect.signature(fn).bind(*args, **kwargs)
