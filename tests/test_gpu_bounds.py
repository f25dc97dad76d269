"""The bounds-check build (SURVEY's stand-in for a memory sanitizer, which the
test machines do not offer): the small parity cases run on a library whose
kernels compare every checked index with its extent, record the site and skip
the access instead of going out of range.  They must match the oracle and
record nothing; the build's self-test probe must record its site."""
import json
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


def test_small_cases_on_the_bounds_check_build():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lib = os.path.join(os.path.dirname(HERE), "lfsr_seeded_moe_b200", "_build", "boundscheck", "libnslm.so")
    assert os.path.exists(lib), "build it with python -m lfsr_seeded_moe_b200.build --bounds-check"
    env = dict(os.environ, NSLM_LIB_VARIANT="boundscheck")
    env.pop("NSLM_STREAM_SOURCE", None)
    r = subprocess.run([sys.executable, os.path.join(HERE, "bounds_cases.py")], env=env, capture_output=True,
                       text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    res = json.loads(r.stdout.strip().splitlines()[-1])
    assert res["status_start"] == 0
    for k, v in res.items():
        # fp32 decode paths to 1e-5; the tensor-core path (bf16 weights and h)
        # and the stack (its layer chaining rounds to bf16) to the stated 2e-3
        if k.startswith(("gemv_", "ffn_", "stack_")):
            assert v <= (2e-3 if k.startswith(("ffn_T12", "stack_")) else 1e-5), (k, v)
    assert res["decompress_exact"] is True
    assert res["status_after_cases"] == 0          # no checked index left its buffer
    assert res["status_after_probe"] == 1          # the probe's copy was refused at site 1
    assert res["status_cleared"] == 0


def test_bounds_exports_refuse_in_the_normal_build():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from lfsr_seeded_moe_b200 import nslm
    if nslm.LIB_PATH.endswith(os.path.join("boundscheck", "libnslm.so")):
        pytest.skip("running on the bounds-check build")
    assert nslm.raw().nslm_debug_bounds_status() == nslm.NSLM_ERR_UNSUPPORTED
