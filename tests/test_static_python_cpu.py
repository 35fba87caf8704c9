"""Undefined names and attributes in the Python that only a GPU runs.

bench.py's CUDA arm, the binding's device classes, __graft_entry__.smoke()
and the GPU tests cannot execute on a machine without a GPU, so a misspelt
or removed name in them would first show on the GPU machine. This walks every
function and method of those files and checks that each name it reads is a
parameter, assigned or imported in the function (or an enclosing one), a
module-level name, or a builtin; that every attribute read from one of
this repository's modules (the binding, synth, the oracle, the parity
rules) names something that module defines; and that every attribute read
from an object a function makes with one of the binding's classes is one
that class defines.
"""
import ast
import builtins
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FILES = ["bench.py", "__graft_entry__.py", os.path.join("strided_verify_propose_b200", "binding.py"),
         os.path.join("strided_verify_propose_b200", "build.py"), os.path.join("tests", "_parity.py")] + \
    sorted(os.path.join("tests", f) for f in os.listdir(os.path.join(ROOT, "tests"))
           if f.startswith(("test_gpu_", "test_zz_")) and f.endswith(".py"))


def _bound(node):
    """Names a function binds anywhere in its body (nested scopes included)."""
    names = set()
    for n in ast.walk(node):
        if isinstance(n, ast.Name) and isinstance(n.ctx, (ast.Store, ast.Del)):
            names.add(n.id)
        elif isinstance(n, (ast.Import, ast.ImportFrom)):
            names.update((a.asname or a.name).split(".")[0] for a in n.names)
        elif isinstance(n, (ast.FunctionDef, ast.AsyncFunctionDef, ast.Lambda)):
            if not isinstance(n, ast.Lambda):
                names.add(n.name)
            a = n.args
            names.update(x.arg for x in a.posonlyargs + a.args + a.kwonlyargs)
            names.update(x.arg for x in (a.vararg, a.kwarg) if x is not None)
        elif isinstance(n, ast.ClassDef):
            names.add(n.name)
        elif isinstance(n, ast.ExceptHandler) and n.name:
            names.add(n.name)
        elif isinstance(n, (ast.Global, ast.Nonlocal)):
            names.update(n.names)
    return names


def _module_names(tree):
    names = set(dir(builtins)) | {"__file__", "__name__"}
    for node in tree.body:
        if isinstance(node, (ast.FunctionDef, ast.AsyncFunctionDef, ast.ClassDef)):
            names.add(node.name)
        elif isinstance(node, (ast.Import, ast.ImportFrom)):
            names.update((a.asname or a.name).split(".")[0] for a in node.names)
        else:
            for n in ast.walk(node):
                if isinstance(n, ast.Name) and isinstance(n.ctx, ast.Store):
                    names.add(n.id)
                elif isinstance(n, (ast.Import, ast.ImportFrom)):
                    names.update((a.asname or a.name).split(".")[0] for a in n.names)
    return names


@pytest.mark.parametrize("rel", FILES)
def test_no_undefined_names(rel):
    tree = ast.parse(open(os.path.join(ROOT, rel)).read(), rel)
    module = _module_names(tree)
    functions = [n for n in tree.body if isinstance(n, (ast.FunctionDef, ast.AsyncFunctionDef))]
    for cls in (n for n in tree.body if isinstance(n, ast.ClassDef)):
        functions += [n for n in cls.body if isinstance(n, (ast.FunctionDef, ast.AsyncFunctionDef))]
    assert functions
    missing = []
    for fn in functions:
        bound = _bound(fn)
        for n in ast.walk(fn):
            if isinstance(n, ast.Name) and isinstance(n.ctx, ast.Load) and n.id not in bound | module:
                missing.append(f"{rel}:{n.lineno} {fn.name}: {n.id}")
    assert not missing, missing


OWN_MODULES = ("strided_verify_propose_b200.binding", "synth", "oracle.isd", "oracle.model",
               "oracle.pages", "tests._parity", "bench")


def _aliases(tree):
    """local name -> module, for every import of one of this repository's
    modules anywhere in the file."""
    out = {}
    for n in ast.walk(tree):
        if isinstance(n, ast.ImportFrom) and n.module:
            for a in n.names:
                full = f"{n.module}.{a.name}"
                if full in OWN_MODULES:
                    out[a.asname or a.name] = full
        elif isinstance(n, ast.Import):
            for a in n.names:
                if a.name in OWN_MODULES:
                    out[a.asname or a.name.split(".")[0]] = a.name
    return out


@pytest.mark.parametrize("rel", FILES)
def test_module_attributes_exist(rel):
    """Every `alias.name` read from one of this repository's modules names
    something that module defines."""
    import importlib
    import sys
    sys.path.insert(0, ROOT)
    tree = ast.parse(open(os.path.join(ROOT, rel)).read(), rel)
    aliases = _aliases(tree)
    missing = []
    for n in ast.walk(tree):
        if (isinstance(n, ast.Attribute) and isinstance(n.value, ast.Name) and n.value.id in aliases
                and isinstance(n.ctx, ast.Load)):
            mod = importlib.import_module(aliases[n.value.id])
            if not hasattr(mod, n.attr):
                missing.append(f"{rel}:{n.lineno} {n.value.id}.{n.attr}")
    assert not missing, missing


def _class_members(rel, classes):
    """Per class of the file: its methods, class-level names and every
    attribute its methods store on self."""
    tree = ast.parse(open(os.path.join(ROOT, rel)).read(), rel)
    out = {}
    for cls in (n for n in tree.body if isinstance(n, ast.ClassDef) and n.name in classes):
        names = set()
        for item in cls.body:
            if isinstance(item, (ast.FunctionDef, ast.AsyncFunctionDef)):
                names.add(item.name)
            elif isinstance(item, ast.Assign):
                names.update(t.id for t in item.targets if isinstance(t, ast.Name))
        for n in ast.walk(cls):
            if (isinstance(n, ast.Attribute) and isinstance(n.ctx, ast.Store)
                    and isinstance(n.value, ast.Name) and n.value.id == "self"):
                names.add(n.attr)
        out[cls.name] = names
    return out


BINDING_CLASSES = ("Model", "KVCache", "StepState", "StepGraph")


@pytest.mark.parametrize("rel", FILES)
def test_binding_object_attributes_exist(rel):
    """Where a function holds an object made by one of the binding's classes
    (`st = B.StepState(...)`), every attribute it reads from it is one that
    class defines."""
    members = _class_members(os.path.join("strided_verify_propose_b200", "binding.py"), BINDING_CLASSES)
    assert set(members) == set(BINDING_CLASSES)
    tree = ast.parse(open(os.path.join(ROOT, rel)).read(), rel)
    aliases = {k for k, v in _aliases(tree).items() if v == "strided_verify_propose_b200.binding"}
    in_binding = rel.endswith("binding.py")
    missing = []
    for fn in (n for n in ast.walk(tree) if isinstance(n, (ast.FunctionDef, ast.AsyncFunctionDef))):
        held = {}
        for n in ast.walk(fn):
            if (isinstance(n, ast.Assign) and len(n.targets) == 1 and isinstance(n.targets[0], ast.Name)
                    and isinstance(n.value, ast.Call)):
                f = n.value.func
                cls = None
                if isinstance(f, ast.Attribute) and isinstance(f.value, ast.Name) and f.value.id in aliases:
                    cls = f.attr
                elif in_binding and isinstance(f, ast.Name):
                    cls = f.id
                if cls in BINDING_CLASSES:
                    held[n.targets[0].id] = cls
        for n in ast.walk(fn):
            if (isinstance(n, ast.Attribute) and isinstance(n.value, ast.Name) and n.value.id in held
                    and n.attr not in members[held[n.value.id]]):
                missing.append(f"{rel}:{n.lineno} {n.value.id}.{n.attr} ({held[n.value.id]})")
    assert not missing, missing
