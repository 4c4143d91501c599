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
