"""The product path has no fallback: without libgqe.so the binding raises on
its first call instead of computing anything itself, and no file of the
package or the public header reaches the CPU oracle (which is test
infrastructure only)."""
import os
import re
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "routed_head_gqa_b200")

_CHILD = r"""
import sys
sys.path.insert(0, {root!r})
import routed_head_gqa_b200 as g
g.LIB_PATH = {missing!r}
g._lib_handle = None
try:
    g.gqe_chunk_count(100)
except ImportError as e:
    print("RAISED:", e)
else:
    print("NO ERROR")
"""


def test_missing_library_raises(tmp_path):
    missing = str(tmp_path / "absent" / "libgqe.so")
    proc = subprocess.run([sys.executable, "-c", _CHILD.format(root=ROOT, missing=missing)],
                          capture_output=True, text=True, timeout=300)
    assert proc.returncode == 0, proc.stderr[-2000:]
    assert "RAISED:" in proc.stdout and missing in proc.stdout, proc.stdout


def _product_files():
    for base in (PKG, os.path.join(ROOT, "include")):
        for dirpath, dirnames, filenames in os.walk(base):
            dirnames[:] = [d for d in dirnames if d not in ("_build", "__pycache__")]
            for f in filenames:
                if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp", ".c")):
                    yield os.path.join(dirpath, f)


def test_product_does_not_reach_the_oracle():
    pattern = re.compile(r"^\s*(import\s+oracle|from\s+oracle\b)|gqe_oracle|liboracle|oracle_[a-z_]+\s*\(", re.M)
    hits = []
    for path in _product_files():
        text = open(path, encoding="utf-8", errors="replace").read()
        for m in pattern.finditer(text):
            line = text.count("\n", 0, m.start()) + 1
            hits.append(f"{os.path.relpath(path, ROOT)}:{line}: {m.group(0).strip()}")
    assert not hits, "product files reach the oracle:\n" + "\n".join(hits)
