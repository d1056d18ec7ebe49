"""The product path never routes through the oracle and computes nothing outside the
library's kernels.  Read from the sources with `ast` (no GPU needed):

* no module of the package (`target_attention_b200/`) or of the input generators
  (`workloads/`) imports `oracle`;
* in `bench.py` the oracle is imported only by `oracle_sample`, and only the CPU baseline
  and the reference arm (`cpu_baseline`, `run_reference`) call it;
* the training composition (`target_attention_b200/training.py`) touches torch only for
  device memory, dtypes, streams and graphs: every arithmetic step is a library call."""
import ast
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _py_files(sub):
    for dirpath, _, files in os.walk(os.path.join(ROOT, sub)):
        if "_build" in dirpath or "__pycache__" in dirpath:
            continue
        for f in files:
            if f.endswith(".py"):
                yield os.path.join(dirpath, f)


def _imported_modules(tree):
    for n in ast.walk(tree):
        if isinstance(n, ast.Import):
            for a in n.names:
                yield a.name, n
        elif isinstance(n, ast.ImportFrom) and n.module:
            yield n.module, n


def test_package_and_workloads_never_import_the_oracle():
    offenders = []
    for sub in ("target_attention_b200", "workloads"):
        for path in _py_files(sub):
            tree = ast.parse(open(path).read(), path)
            for mod, node in _imported_modules(tree):
                if mod == "oracle" or mod.startswith("oracle."):
                    offenders.append(f"{os.path.relpath(path, ROOT)}:{node.lineno}")
    assert not offenders, offenders


def test_bench_reaches_the_oracle_only_from_its_cpu_legs():
    tree = ast.parse(open(os.path.join(ROOT, "bench.py")).read())
    importers, callers = set(), set()
    for fn in ast.walk(tree):
        if not isinstance(fn, ast.FunctionDef):
            continue
        for n in ast.walk(fn):
            if isinstance(n, (ast.Import, ast.ImportFrom)):
                mods = [a.name for a in n.names] if isinstance(n, ast.Import) else [n.module or ""]
                if any(m == "oracle" or m.startswith("oracle.") for m in mods):
                    importers.add(fn.name)
            if isinstance(n, ast.Call) and getattr(n.func, "id", None) == "oracle_sample":
                callers.add(fn.name)
    top = [a.name for n in tree.body if isinstance(n, ast.Import) for a in n.names] + \
          [n.module or "" for n in tree.body if isinstance(n, ast.ImportFrom)]
    assert not any(m == "oracle" or m.startswith("oracle.") for m in top), top
    assert importers == {"oracle_sample"}, importers
    assert callers == {"cpu_baseline", "run_reference"}, callers


def test_training_composition_uses_torch_only_for_memory_and_streams():
    allowed = {"empty", "zeros", "from_numpy", "bfloat16", "float32", "int32", "int16", "uint8", "cuda",
               "Stream", "CUDAGraph", "stream", "graph", "current_stream"}
    path = os.path.join(ROOT, "target_attention_b200", "training.py")
    tree = ast.parse(open(path).read(), path)
    used = set()
    for n in ast.walk(tree):
        if isinstance(n, ast.Attribute):
            base = n.value
            if isinstance(base, ast.Name) and base.id == "torch":
                used.add(n.attr)
            elif isinstance(base, ast.Attribute) and isinstance(base.value, ast.Name) and base.value.id == "torch" \
                    and base.attr == "cuda":
                used.add(n.attr)
    assert used <= allowed, sorted(used - allowed)
    # and no tensor arithmetic (or casts) on the buffers of the layer and step classes;
    # `device_weights` only uploads the host arrays (a copy to the device)
    banned = {"add_", "mul_", "sum", "matmul", "mm", "bmm", "copy_", "clone", "cat", "stack", "exp", "sqrt", "mean",
              "softmax", "to", "float", "half", "bfloat16", "zero_", "fill_"}
    for cls in (n for n in tree.body if isinstance(n, ast.ClassDef)):
        calls = {c.func.attr for c in ast.walk(cls) if isinstance(c, ast.Call) and isinstance(c.func, ast.Attribute)}
        assert not (calls & banned), (cls.name, sorted(calls & banned))
