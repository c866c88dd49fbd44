"""Static check of the repository's Python files: every global name a function
reads is bound at module level (an assignment, def, class or import) or is a
builtin. Parts of bench.py only run on a GPU, so a missing import there would
otherwise surface only on the GPU machine."""

import builtins
import dis
import os
import types

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FILES = ["bench.py", "__graft_entry__.py"] + [
    os.path.join(d, f)
    for d in ("rotation_preconditioned_quantization_b200", "oracle", "tests")
    for f in sorted(os.listdir(os.path.join(ROOT, d)))
    if f.endswith(".py")
]

_BINDING_OPS = ("STORE_NAME", "STORE_GLOBAL", "IMPORT_NAME", "DELETE_NAME")


def _undefined_globals(path):
    src = open(os.path.join(ROOT, path)).read()
    code = compile(src, path, "exec")
    bound = {ins.argval.split(".")[0] for ins in dis.get_instructions(code) if ins.opname in _BINDING_OPS}
    # names bound by `global x; x = ...` inside functions count too
    stack, found = [code], []
    while stack:
        co = stack.pop()
        for ins in dis.get_instructions(co):
            if ins.opname == "STORE_GLOBAL":
                bound.add(ins.argval)
        stack.extend(c for c in co.co_consts if isinstance(c, types.CodeType))
    stack = [(code, "<module>")]
    while stack:
        co, where = stack.pop()
        for ins in dis.get_instructions(co):
            if ins.opname == "LOAD_GLOBAL" and ins.argval not in bound and not hasattr(builtins, ins.argval):
                found.append(f"{where}: {ins.argval}")
        stack.extend((c, f"{where}.{c.co_name}") for c in co.co_consts if isinstance(c, types.CodeType))
    return sorted(set(found))


@pytest.mark.parametrize("path", FILES)
def test_no_undefined_globals(path):
    assert _undefined_globals(path) == []
