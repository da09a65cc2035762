"""bench.py's code paths that need a GPU cannot run here; at least every global
name its functions read must exist (catches a renamed or removed variable)."""
import builtins
import os
import symtable

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _global_reads(table, out):
    for child in table.get_children():
        for sym in child.get_symbols():
            if sym.is_referenced() and sym.is_global() and not sym.is_local():
                out.add((child.get_name(), sym.get_name()))
        _global_reads(child, out)


def test_bench_reads_only_defined_globals():
    path = os.path.join(ROOT, "bench.py")
    with open(path) as f:
        src = f.read()
    mod = symtable.symtable(src, path, "exec")
    defined = {s.get_name() for s in mod.get_symbols() if s.is_assigned() or s.is_imported()}
    defined |= set(dir(builtins))
    reads = set()
    _global_reads(mod, reads)
    missing = sorted((fn, name) for fn, name in reads if name not in defined)
    assert not missing, missing
