"""The problem ea_router_static_scratch must refuse, and the refusal checked in a child
process that sees no GPU (shared by the CPU and GPU tests of that entry point)."""
import os
import subprocess
import sys

_ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# The refused problem: 64 samples x D = 32768 (the pooled states alone fill the 8 MiB array,
# and the projection partial sums come on top).
REFUSED = dict(B=64, S=1, D=32768, H_kv=8, d=128)


def refusal_without_a_gpu() -> int:
    """Status of ea_router_static_scratch on the refused problem in a child process that sees
    no GPU.  The size check runs on the host before any CUDA call; if it ever stopped
    refusing, the call would fail on the missing device (EA_ERR_CUDA), never launch."""
    code = (
        "import ctypes, sys\n"
        "sys.path.insert(0, %r)\n"
        "from sparse_gqa_attention_b200 import abi\n"
        "lib = abi._lib()\n"
        "fake = ctypes.c_void_p(0x10000)\n"
        "w = abi.RouterWeights(*([fake] * 9))\n"
        "prm = abi.RouterParams(100)\n"
        "print(lib.ea_router_static_scratch(fake, abi.EA_DT_BF16, %d, %d, %d, %d, %d, ctypes.byref(w),"
        " ctypes.byref(prm), fake, None, None))\n"
    ) % (_ROOT, REFUSED["B"], REFUSED["S"], REFUSED["D"], REFUSED["H_kv"], REFUSED["d"])
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    res = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=300)
    assert res.returncode == 0, res.stderr
    return int(res.stdout.strip().splitlines()[-1])
