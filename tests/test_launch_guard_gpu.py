"""The register guard of the tensor-core kernels is kept per instantiation.

The forward and backward kernels move registers between warpgroups with
setmaxnreg, which is only safe when each thread is launched with exactly the
registers the split assumes.  Every instantiation (forward / backward, D 64 /
128, causal or not) must compile to that count, and the library must check
each instantiation itself before its first launch rather than let one result
stand for all kernels of the same function type.
"""
import os
import subprocess
import sys

import pytest

import exact_tiled_attention_46_b200 as fa

from parity import need_gpu

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    need_gpu()


@pytest.mark.parametrize("bwd", [0, 1])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("causal", [0, 1])
def test_every_instantiation_compiles_to_the_split_register_count(bwd, D, causal):
    regs, expected, _ = fa.launch_guard(bwd, D, causal)
    assert regs == expected, f"{'bwd' if bwd else 'fwd'}<{D},{causal}>: {regs} registers, split assumes {expected}"


@pytest.mark.parametrize("causal", [0, 1])
def test_fp8_forward_compiles_to_the_split_register_count(causal):
    regs, expected, _ = fa.launch_guard(0, -128, causal)
    assert regs == expected, f"fwd_fp8<{causal}>: {regs} registers, split assumes {expected}"


CHILD = r"""
import torch, exact_tiled_attention_46_b200 as fa
def states():
    return {(b, D, c): fa.launch_guard(b, D, c, query_regs=False)[2] for b in (0, 1) for D in (64, 128) for c in (0, 1)}
assert all(s == 0 for s in states().values())
q = torch.randn(1, 200, 2, 128, device="cuda").to(torch.bfloat16)
fa.fwd(q, q, q, causal=True)
torch.cuda.synchronize()
s = states()
assert s[(0, 128, 1)] == 1 and sum(s.values()) == 1, s
q = torch.randn(1, 200, 2, 64, device="cuda").to(torch.bfloat16)
o, lse = fa.fwd(q, q, q, causal=True)
fa.bwd(q, q, q, o, q, lse, causal=True)
torch.cuda.synchronize()
s = states()
assert s[(0, 64, 1)] == 1 and s[(1, 64, 1)] == 1 and sum(s.values()) == 3, s
print("per-instantiation guard ok")
"""


def test_guard_checks_each_instantiation_before_its_first_launch():
    """In a fresh process, launching one instantiation marks that one checked
    and leaves every other instantiation unchecked."""
    env = dict(os.environ, PYTHONPATH=ROOT + os.pathsep + os.environ.get("PYTHONPATH", ""))
    r = subprocess.run([sys.executable, "-c", CHILD], cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "per-instantiation guard ok" in r.stdout
