"""GPU parity of the kernel configurations that the library selects from the
environment at its first call (so each needs a process of its own):

  * PA_PREFILL_BN=128  — prefill and shared-prefix pass in blocks of 128 keys,
                         one CTA per SM (the default is 64 keys, two CTAs);
  * PA_PREFILL_MMA=sync — the warp-level mma.sync prefill and prefix pass.

Each runs the prefill and shared-prefix parity suites against the oracle in
a child pytest process with the variable set.
"""
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
_VARS = ("PA_PREFILL_BN", "PA_PREFILL_MMA")


@pytest.mark.parametrize("var,value", [("PA_PREFILL_BN", "128"), ("PA_PREFILL_MMA", "sync")])
def test_configuration_matches_oracle(var, value):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    if any(os.environ.get(v) for v in _VARS):
        pytest.skip("already running under a configuration variable")
    env = {k: v for k, v in os.environ.items() if k not in _VARS}
    env[var] = value
    suites = [os.path.join(HERE, "test_prefill_gpu.py"), os.path.join(HERE, "test_prefix_gpu.py")]
    r = subprocess.run([sys.executable, "-m", "pytest", *suites, "-q", "-x", "-m", "gpu", "-p", "no:cacheprovider"],
                       env=env, cwd=os.path.dirname(HERE), capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, f"{var}={value}:\n{r.stdout[-3000:]}\n{r.stderr[-2000:]}"
    assert " passed" in r.stdout
