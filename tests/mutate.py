"""Load a copy of an oracle Python module with planted mistakes (helper for
the mutant tests; not a test module)."""
import importlib.util
import sys


def load_mutant(src_text: str, tmp_path, tag: str):
    path = tmp_path / f"mutant_{tag}.py"
    path.write_text(src_text)
    name = f"oracle._mutant_{tag}"
    spec = importlib.util.spec_from_file_location(name, path)
    mod = importlib.util.module_from_spec(spec)
    sys.modules[name] = mod
    try:
        spec.loader.exec_module(mod)
    finally:
        sys.modules.pop(name, None)
    return mod


def apply(src: str, edits, name: str) -> str:
    for old, new in edits:
        assert src.count(old) == 1, f"mutation anchor for {name} not unique: {old!r}"
        src = src.replace(old, new)
    return src


def first_failure(mod, checks):
    for check in checks:
        try:
            check(mod)
        except Exception as exc:  # a failed assertion or an error both count as caught
            return check.__name__, exc
    return None
