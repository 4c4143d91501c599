"""Static checks of the separation the parity claims rest on: the product
package never imports the FP64 oracle, the oracle never imports the product
package, and the two share no source file."""

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
    for name in ("__init__.py", "synth.py", "dist.py"):
        shutil.copy(os.path.join(ROOT, "lora_gemm_b200", name), pkg / name)
    code = ("import sys\nsys.path.insert(0, sys.argv[1])\n"
            "try:\n    import lora_gemm_b200\nexcept ImportError as e:\n    print('ImportError', e)\n"
            "else:\n    print('imported')\n")
    out = subprocess.run([sys.executable, "-c", code, str(tmp_path)], capture_output=True, text=True, timeout=300)
    assert out.stdout.startswith("ImportError"), out.stdout + out.stderr
