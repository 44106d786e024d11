"""Static checks of the Python sources whose GPU paths the CPU suite cannot run.

bench.py's timed arms, the GPU tests and __graft_entry__.smoke() only execute
on a device; a misspelt name there would first show as a failed run on the
GPU.  These checks catch the usual slips on the CPU: a name used but never
bound (symbol tables), an attribute of the package, the workloads module or
the oracle that does not exist, and a call into them with a keyword or
positional argument their signatures do not take.
"""
import ast
import builtins
import glob
import inspect
import os
import symtable

import pytest

import oracle
import selective_state_space_momentum_b200 as mm
from selective_state_space_momentum_b200 import workloads as wl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SOURCES = sorted([os.path.join(ROOT, "bench.py"), os.path.join(ROOT, "__graft_entry__.py")] +
                 glob.glob(os.path.join(ROOT, "selective_state_space_momentum_b200", "*.py")) +
                 glob.glob(os.path.join(ROOT, "oracle", "*.py")) +
                 glob.glob(os.path.join(ROOT, "tests", "*.py")))
CALLERS = [p for p in SOURCES if os.path.basename(p) in ("bench.py", "__graft_entry__.py")
           or os.sep + "tests" + os.sep in p]
MODULES = {"mm": mm, "wl": wl, "oracle": oracle}
IMPLICIT = {"__file__", "__name__", "__doc__", "__spec__", "__builtins__"}


def _unbound_names(path):
    src = open(path).read()
    top = symtable.symtable(src, path, "exec")
    bound = {s.get_name() for s in top.get_symbols()
             if s.is_assigned() or s.is_imported() or s.is_namespace()}
    found = []

    def walk(tab):
        for sym in tab.get_symbols():
            name = sym.get_name()
            global_ref = sym.is_global() or (tab.get_type() == "module" and not (
                sym.is_assigned() or sym.is_imported() or sym.is_namespace()))
            if global_ref and sym.is_referenced() and name not in bound and name not in IMPLICIT \
                    and not hasattr(builtins, name):
                found.append(f"{tab.get_name()}:{tab.get_lineno()} {name}")
        for child in tab.get_children():
            walk(child)
    walk(top)
    return found


@pytest.mark.parametrize("path", SOURCES, ids=lambda p: os.path.relpath(p, ROOT))
def test_every_name_is_bound(path):
    assert _unbound_names(path) == []


@pytest.mark.parametrize("path", CALLERS, ids=lambda p: os.path.relpath(p, ROOT))
def test_module_attributes_and_calls_match(path):
    problems = []
    tree = ast.parse(open(path).read())
    for node in ast.walk(tree):
        if isinstance(node, ast.Attribute) and isinstance(node.value, ast.Name) and node.value.id in MODULES:
            if not hasattr(MODULES[node.value.id], node.attr):
                problems.append(f"{node.lineno}: {node.value.id}.{node.attr} does not exist")
        if not (isinstance(node, ast.Call) and isinstance(node.func, ast.Attribute)
                and isinstance(node.func.value, ast.Name) and node.func.value.id in MODULES):
            continue
        fn = getattr(MODULES[node.func.value.id], node.func.attr, None)
        if not callable(fn):
            continue
        try:
            params = inspect.signature(fn).parameters
        except (TypeError, ValueError):
            continue
        kinds = {p.kind for p in params.values()}
        if inspect.Parameter.VAR_KEYWORD not in kinds:
            for kw in node.keywords:
                if kw.arg is not None and kw.arg not in params:
                    problems.append(f"{node.lineno}: {node.func.attr}() takes no argument {kw.arg!r}")
        if inspect.Parameter.VAR_POSITIONAL not in kinds and not any(isinstance(a, ast.Starred) for a in node.args):
            room = sum(1 for p in params.values()
                       if p.kind in (inspect.Parameter.POSITIONAL_ONLY, inspect.Parameter.POSITIONAL_OR_KEYWORD))
            if len(node.args) > room:
                problems.append(f"{node.lineno}: {node.func.attr}() takes {room} positional arguments, "
                                f"given {len(node.args)}")
    assert problems == []
