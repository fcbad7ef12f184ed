"""__graft_entry__.smoke() runs only on a GPU; this CPU test catches the class
of bug that would otherwise surface there first: a name it loads that nothing
defines (a helper renamed in one place, a missing import)."""
import ast
import builtins
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _undefined_names(path: str) -> set[str]:
    tree = ast.parse(open(path).read())
    defined = {"__file__", "__name__"}
    for n in ast.walk(tree):
        if isinstance(n, ast.Name) and isinstance(n.ctx, (ast.Store, ast.Del)):
            defined.add(n.id)
        elif isinstance(n, (ast.FunctionDef, ast.AsyncFunctionDef, ast.ClassDef)):
            defined.add(n.name)
            if not isinstance(n, ast.ClassDef):
                for a in n.args.args + n.args.kwonlyargs:
                    defined.add(a.arg)
                if n.args.vararg:
                    defined.add(n.args.vararg.arg)
                if n.args.kwarg:
                    defined.add(n.args.kwarg.arg)
        elif isinstance(n, (ast.Import, ast.ImportFrom)):
            for a in n.names:
                defined.add((a.asname or a.name).split(".")[0])
        elif isinstance(n, ast.ExceptHandler) and n.name:
            defined.add(n.name)
        elif isinstance(n, ast.comprehension):
            for t in ast.walk(n.target):
                if isinstance(t, ast.Name):
                    defined.add(t.id)
    loads = {n.id for n in ast.walk(tree) if isinstance(n, ast.Name) and isinstance(n.ctx, ast.Load)}
    return {x for x in loads if x not in defined and not hasattr(builtins, x)}


def test_graft_entry_defines_every_name_it_uses():
    assert _undefined_names(os.path.join(ROOT, "__graft_entry__.py")) == set()


def test_bench_defines_every_name_it_uses():
    assert _undefined_names(os.path.join(ROOT, "bench.py")) == set()
