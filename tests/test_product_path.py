"""The product path has no fallback: without the CUDA library every entry point of the binding
raises, and no module of the package imports the oracle (which only the tests, the smoke run
and the benchmark's CPU baseline use)."""
import ast
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "communication_compressed_optimizer_momentum_b200")

MISSING = r'''
import sys
sys.path.insert(0, %r)
from communication_compressed_optimizer_momentum_b200 import _abi
_abi.LIB_PATH = "/nonexistent/libonebit_adam.so"
import communication_compressed_optimizer_momentum_b200 as ob
from communication_compressed_optimizer_momentum_b200 import dp
calls = {
    "init": lambda: ob.onebit_adam_init(1000, 2, 256),
    "dp_init": lambda: ob.onebit_dp_init(1000, 2, 256, 0.9, 0.999, 1e-8, 2, 0),
    "chunk_range": lambda: ob.onebit_dp_chunk_range(4, 2, 0),
    "OneBitAdam": lambda: ob.OneBitAdam(1000, 2, 256, device="cpu"),
    "OneBitAdamRank": lambda: dp.OneBitAdamRank(1000, 2, 256, 2, 0, device="cpu"),
    "zo_init": lambda: ob.onebit01_init(1000, 2, 256, 0.9, 0.999, 1e-8, 2, 1),
    "zo_dp_init": lambda: ob.onebit01_dp_init(1000, 2, 256, 0.9, 0.999, 1e-8, 2, 1, 2, 0),
    "ZeroOneAdam": lambda: ob.ZeroOneAdam(1000, 2, 256, 2, 1, device="cpu"),
    "ZeroOneAdamRank": lambda: dp.ZeroOneAdamRank(1000, 2, 256, 2, 0, 2, 1, device="cpu"),
    "server_layout": lambda: ob.onebit_server_layout(1000, 2, 256),
}
for name, fn in calls.items():
    try:
        fn()
    except RuntimeError as e:
        assert "not built" in str(e), (name, str(e))
        continue
    raise SystemExit("%%s did not raise" %% name)
print("all raised")
''' % ROOT


def test_every_entry_point_raises_without_the_library():
    r = subprocess.run([sys.executable, "-c", MISSING], capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "all raised" in r.stdout


def test_package_never_imports_the_oracle():
    for name in sorted(os.listdir(PKG)):
        if not name.endswith(".py"):
            continue
        tree = ast.parse(open(os.path.join(PKG, name)).read())
        for node in ast.walk(tree):
            if isinstance(node, ast.Import):
                mods = [a.name for a in node.names]
            elif isinstance(node, ast.ImportFrom):
                mods = [node.module or ""]
            else:
                continue
            assert not any(m == "oracle" or m.startswith("oracle.") for m in mods), name
