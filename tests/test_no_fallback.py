"""The product path has no fallback: without the compiled library the binding
raises, and nothing in the package reaches the CPU oracle."""
import ast
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "encoder_decision_model_b200")


def test_missing_library_fails_loudly(tmp_path):
    code = ("import encoder_decision_model_b200._lib as jl\n"
            "try:\n"
            "    jl.lib()\n"
            "except FileNotFoundError as e:\n"
            "    print('raised', e)\n"
            "else:\n"
            "    print('loaded')\n")
    env = dict(os.environ, JD_LIB=str(tmp_path / "absent.so"))
    out = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True, text=True,
                         timeout=120)
    assert out.returncode == 0, out.stderr
    assert out.stdout.startswith("raised"), out.stdout


def test_package_never_imports_the_oracle():
    for dirpath, _, files in os.walk(PKG):
        for f in files:
            if not f.endswith(".py"):
                continue
            tree = ast.parse(open(os.path.join(dirpath, f)).read())
            for node in ast.walk(tree):
                names = []
                if isinstance(node, ast.Import):
                    names = [a.name for a in node.names]
                elif isinstance(node, ast.ImportFrom):
                    names = [node.module or ""]
                for n in names:
                    assert n.split(".")[0] not in ("oracle", "tests"), (f, n)
