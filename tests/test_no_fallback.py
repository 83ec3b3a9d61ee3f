"""The product path has no fallback: without libdma.so every entry point
raises before doing any work, and the package never imports the oracle.
CPU only (the library path is pointed at a file that does not exist, in a
child process, so the loaded library of this test session is untouched)."""
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "trainable_dynamic_mask_b200")

_CHILD = r"""
import sys
sys.path.insert(0, %(root)r)
import trainable_dynamic_mask_b200 as dma
from trainable_dynamic_mask_b200 import _lib
assert not any(m == "oracle" or m.startswith("oracle.") for m in sys.modules), "package imported the oracle"
_lib.LIB_PATH = %(missing)r
_lib._lib = None
p = dma.make_params(1, 2, 1, 256, 64, 64)
calls = {
    "workspace_size": lambda: dma.workspace_size(p),
    "gate": lambda: dma.gate(p, None, None, None, None),
    "topk_mask": lambda: dma.topk_mask(p, None, None, None),
    "topk_append": lambda: dma.topk_append(p, None, None),
    "gate_append": lambda: dma.gate_append(p, None, None, None, None),
    "attn_fwd": lambda: dma.attn_fwd(p, None, None, None, None, None, None, None, None),
    "attn_bwd": lambda: dma.attn_bwd(p, *([None] * 13)),
    "gate_bwd": lambda: dma.gate_bwd(p, *([None] * 10)),
    "gate_bwd_noalloc": lambda: dma.gate_bwd_noalloc(p, *([None] * 9)),
}
for name, fn in calls.items():
    try:
        fn()
    except RuntimeError as e:
        assert "no fallback" in str(e) and "build" in str(e), (name, str(e))
    else:
        raise AssertionError(name + " ran without libdma.so")
print("ok")
"""


def test_entry_points_raise_without_the_library():
    missing = os.path.join(ROOT, "no_such_dir", "libdma.so")
    assert not os.path.exists(missing)
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    r = subprocess.run([sys.executable, "-c", _CHILD % {"root": ROOT, "missing": missing}], env=env,
                       capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), r.stdout + r.stderr


def test_package_sources_do_not_reference_the_oracle():
    for dirpath, _, files in os.walk(PKG):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".c", ".cpp")):
                text = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in text and "from oracle" not in text, f
                assert "dma_oracle" not in text, f
