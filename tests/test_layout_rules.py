"""Static checks of the separation the parity claims rest on: the product
package never imports the FP64 oracle, the oracle never imports the product
package, the two share no source file, the seeded input recipe (synth.py)
imports neither, and bench.py's oracle arm runs without loading the product
library."""

import ast
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _py_files(sub):
    for dirpath, _, names in os.walk(os.path.join(ROOT, sub)):
        for n in names:
            if n.endswith(".py"):
                yield os.path.join(dirpath, n)


def _imported_modules(path):
    tree = ast.parse(open(path, encoding="utf-8").read(), filename=path)
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            for a in node.names:
                yield a.name
        elif isinstance(node, ast.ImportFrom) and node.module and node.level == 0:
            yield node.module


def test_product_package_never_imports_the_oracle():
    for path in _py_files("lora_gemm_b200"):
        for mod in _imported_modules(path):
            assert not mod.split(".")[0] == "oracle", f"{path} imports {mod}"


def test_oracle_never_imports_the_product_package():
    for path in _py_files("oracle"):
        for mod in _imported_modules(path):
            assert not mod.startswith("lora_gemm_b200"), f"{path} imports {mod}"


def test_product_sources_do_not_mention_the_oracle_package():
    csrc = os.path.join(ROOT, "lora_gemm_b200", "csrc")
    for name in os.listdir(csrc):
        if name.endswith((".cu", ".cuh", ".h", ".inc")):
            text = open(os.path.join(csrc, name), encoding="utf-8").read()
            assert "oracle/" not in text and "import oracle" not in text, name


def test_binding_fails_loudly_without_the_library(tmp_path):
    """A copy of the package without liblora_gemm.so raises ImportError on
    import: there is no CPU fallback to fall back to."""
    import shutil
    import subprocess
    import sys

    pkg = tmp_path / "lora_gemm_b200"
    pkg.mkdir()
    for name in ("__init__.py", "dist.py"):
        shutil.copy(os.path.join(ROOT, "lora_gemm_b200", name), pkg / name)
    code = ("import sys\nsys.path.insert(0, sys.argv[1])\n"
            "try:\n    import lora_gemm_b200\nexcept ImportError as e:\n    print('ImportError', e)\n"
            "else:\n    print('imported')\n")
    out = subprocess.run([sys.executable, "-c", code, str(tmp_path)], capture_output=True, text=True, timeout=300)
    assert out.stdout.startswith("ImportError"), out.stdout + out.stderr


def test_input_recipe_imports_neither_side():
    for mod in _imported_modules(os.path.join(ROOT, "synth.py")):
        top = mod.split(".")[0]
        assert top not in ("oracle", "lora_gemm_b200"), f"synth.py imports {mod}"


def _function_imports(path, names):
    """Modules imported inside the named top-level functions / classes of a file."""
    tree = ast.parse(open(path, encoding="utf-8").read(), filename=path)
    out = {}
    for node in tree.body:
        if isinstance(node, (ast.FunctionDef, ast.ClassDef)) and node.name in names:
            mods = []
            for sub in ast.walk(node):
                if isinstance(sub, ast.Import):
                    mods += [a.name for a in sub.names]
                elif isinstance(sub, ast.ImportFrom) and sub.module:
                    mods.append(sub.module)
            out[node.name] = mods
    return out


def test_bench_oracle_arm_never_imports_the_product_package():
    names = ("OracleStep", "_oracle_tokens_for", "cpu_baseline", "run_reference", "blas_threads")
    found = _function_imports(os.path.join(ROOT, "bench.py"), names)
    assert set(found) == set(names)
    for fn, mods in found.items():
        assert not any(m.startswith("lora_gemm_b200") for m in mods), f"bench.{fn} imports {mods}"
    # bench.py's module-level imports must not load the product either.
    tree = ast.parse(open(os.path.join(ROOT, "bench.py"), encoding="utf-8").read())
    for node in tree.body:
        if isinstance(node, ast.Import):
            assert not any(a.name.startswith("lora_gemm_b200") for a in node.names)
        elif isinstance(node, ast.ImportFrom):
            assert not (node.module or "").startswith("lora_gemm_b200")


def test_bench_reference_arm_runs_without_the_product_library():
    """The oracle arm, run end to end on a tiny sample, leaves lora_gemm_b200
    (and so liblora_gemm.so) unloaded."""
    import subprocess
    import sys

    code = (
        "import sys, types\n"
        f"sys.path.insert(0, {ROOT!r})\n"
        "import bench\n"
        "args = types.SimpleNamespace(workload='tiny', steps=1, warmup=3, reference_seconds=2.0)\n"
        "line = bench.run_reference(args, 0, 1)\n"
        "assert line['impl'] == 'reference' and line['value'] > 0, line\n"
        "loaded = [m for m in sys.modules if m.startswith('lora_gemm_b200')]\n"
        "import ctypes, os\n"
        "maps = open('/proc/self/maps').read() if os.path.exists('/proc/self/maps') else ''\n"
        "print('LOADED', loaded, 'liblora_gemm' in maps)\n"
    )
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    assert "LOADED [] False" in out.stdout, out.stdout
