"""The table-form ablation of the one-token stack (phase A's dot products from
per-position tables of x, "NanoSeedLM" decode FFN): slower than the direct
form on B200, so not the default, but built, run and held to the same bar.
Its cases run in a subprocess on _build/tableform/libnslm.so."""
import json
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
TOL = 2e-3    # the stated bar
TIGHT = 1e-5  # the fp32 decode path's own accuracy (layer 0 and the single-layer FFN)


def test_table_form_stacks_match_the_oracle():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lib = os.path.join(os.path.dirname(HERE), "lfsr_seeded_moe_b200", "_build", "tableform", "libnslm.so")
    assert os.path.exists(lib), "build it with python -m lfsr_seeded_moe_b200.build --table-form"
    env = dict(os.environ, NSLM_LIB_VARIANT="tableform")
    env.pop("NSLM_STREAM_SOURCE", None)
    r = subprocess.run([sys.executable, os.path.join(HERE, "tableform_cases.py")], env=env, capture_output=True,
                       text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    res = json.loads(r.stdout.strip().splitlines()[-1])
    assert len(res) == 4
    for name, v in res.items():
        assert all(s == 0 for s in v["status"]), (name, v)
        assert v["layers"][0] <= TIGHT, (name, v)
        assert all(e <= TOL for e in v["layers"][1:]), (name, v)
        assert v["ffn"] <= TIGHT, (name, v)
