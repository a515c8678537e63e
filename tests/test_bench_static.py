"""bench.py's GPU arm only runs on a GPU machine, so a name left undefined by an
edit there would surface only at the end of a run.  This CPU test walks the
module's syntax tree and checks that every name a function reads is bound
somewhere in that function (its nested functions and lambdas included), at
module level, or is a builtin."""
import ast
import builtins
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bound_names(node: ast.AST) -> set[str]:
    names: set[str] = set()
    for n in ast.walk(node):
        if isinstance(n, ast.Name) and isinstance(n.ctx, (ast.Store, ast.Del)):
            names.add(n.id)
        elif isinstance(n, (ast.FunctionDef, ast.AsyncFunctionDef, ast.ClassDef)):
            names.add(n.name)
        elif isinstance(n, ast.arg):
            names.add(n.arg)
        elif isinstance(n, (ast.Import, ast.ImportFrom)):
            for a in n.names:
                names.add((a.asname or a.name).split(".")[0])
        elif isinstance(n, ast.ExceptHandler) and n.name:
            names.add(n.name)
        elif isinstance(n, (ast.Global, ast.Nonlocal)):
            names.update(n.names)
    return names


def test_bench_functions_read_only_bound_names():
    with open(os.path.join(ROOT, "bench.py")) as f:
        tree = ast.parse(f.read())
    module_names = {n.name for n in tree.body if isinstance(n, (ast.FunctionDef, ast.ClassDef))}
    for n in tree.body:
        if isinstance(n, (ast.Assign, ast.AnnAssign, ast.Import, ast.ImportFrom)):
            module_names |= _bound_names(n)
    known = module_names | set(dir(builtins))
    missing = []
    for fn in tree.body:
        if not isinstance(fn, ast.FunctionDef):
            continue
        bound = _bound_names(fn) | known
        for n in ast.walk(fn):
            if isinstance(n, ast.Name) and isinstance(n.ctx, ast.Load) and n.id not in bound:
                missing.append(f"{fn.name}: {n.id} (line {n.lineno})")
    assert not missing, missing
