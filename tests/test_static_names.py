"""Every name a function of the package, the bench or the oracle loads resolves.

The bindings run only on a GPU machine, so a misspelt or dropped local there would
surface only there; a scope-aware pass over the symbol tables finds it here."""
import builtins
import os
import symtable

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FILES = ["bench.py", "__graft_entry__.py", "oracle/__init__.py"] + [
    os.path.join("combine_warp_top_router_b200", f)
    for f in sorted(os.listdir(os.path.join(ROOT, "combine_warp_top_router_b200")))
    if f.endswith(".py")]


def _unresolved(table, module_names, out):
    for s in table.get_symbols():
        n = s.get_name()
        if (s.is_referenced() and s.is_global() and not s.is_assigned()
                and n not in module_names and not hasattr(builtins, n) and n != "__file__"):
            out.append(f"{table.get_name()}: {n}")
    for c in table.get_children():
        _unresolved(c, module_names, out)


@pytest.mark.parametrize("rel", FILES)
def test_no_unresolved_names(rel):
    path = os.path.join(ROOT, rel)
    top = symtable.symtable(open(path).read(), path, "exec")
    names = {s.get_name() for s in top.get_symbols() if s.is_assigned() or s.is_imported()}
    out = []
    for c in top.get_children():
        _unresolved(c, names, out)
    assert not out, out
