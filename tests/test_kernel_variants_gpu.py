"""GPU parity of the kernel configurations that the library selects from the
environment at its first call (so each needs a process of its own):

  * PA_PREFILL_BN=128  — prefill and shared-prefix pass in blocks of 128 keys,
                         one CTA per SM (the default is 64 keys, two CTAs);
  * PA_PREFILL_MMA=sync — the warp-level mma.sync prefill and prefix pass;
  * PA_PREFIX_SPLITS=1 / 16 — the fewest and the most key ranges of the
                         shared-prefix pass (the decode folds one or sixteen
                         range partials per member);
  * PA_DECODE_MATH=simt — the decode's per-page math in fp32 on the CUDA
                         cores instead of mma.sync (head_dim * Hq/Hkv <= 256;
                         the suites skip the shapes it is not built for).

Each runs the parity suites it affects against the oracle in a child pytest
process with the variable set.
"""
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
_VARS = ("PA_PREFILL_BN", "PA_PREFILL_MMA", "PA_PREFIX_SPLITS", "PA_DECODE_MATH")


@pytest.mark.parametrize("var,value,suites", [
    ("PA_PREFILL_BN", "128", ("test_prefill_gpu.py", "test_prefix_gpu.py")),
    ("PA_PREFILL_MMA", "sync", ("test_prefill_gpu.py", "test_prefix_gpu.py")),
    ("PA_PREFIX_SPLITS", "1", ("test_prefix_gpu.py",)),
    ("PA_PREFIX_SPLITS", "16", ("test_prefix_gpu.py",)),
    ("PA_DECODE_MATH", "simt", ("test_parity_gpu.py", "test_prefix_gpu.py")),
])
def test_configuration_matches_oracle(var, value, suites):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    if any(os.environ.get(v) for v in _VARS):
        pytest.skip("already running under a configuration variable")
    env = {k: v for k, v in os.environ.items() if k not in _VARS}
    env[var] = value
    paths = [os.path.join(HERE, x) for x in suites]
    r = subprocess.run([sys.executable, "-m", "pytest", *paths, "-q", "-x", "-m", "gpu", "-p", "no:cacheprovider"],
                       env=env, cwd=os.path.dirname(HERE), capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, f"{var}={value}:\n{r.stdout[-3000:]}\n{r.stderr[-2000:]}"
    assert " passed" in r.stdout
