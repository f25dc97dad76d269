"""The trace build of the one-token decode kernel (global-timer stamps at the
phase boundaries, read by `bench.py --profile anatomy`): run in a subprocess
on _build/trace/libnslm.so, its stamps must be ordered as the phases run and
its output must equal the default build's."""
import json
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)

CASE = r"""
import json, sys
sys.path.insert(0, sys.argv[1])
import numpy as np, torch
from lfsr_seeded_moe_b200 import nslm, synth
dev = torch.device("cuda")
L, E, H, I, K = 5, 8, 1024, 256, 4
layers = [synth.moe_layer(l, E, H, I, 4, device=dev, config=953) for l in range(L)]
arr = nslm.moe_layers([(m.gate, m.up, m.down) for m in layers])
lg = torch.stack([synth.router_logits((953, l), 1, E) for l in range(L)]).to(dev).contiguous()
x = synth.activations((953,), 1, H).to(dev).contiguous()
y = torch.empty(1, H, device=dev)
wsb = nslm.nslm_workspace_bytes(nslm.NSLM_OP_MOE_STACK, 1, E, H, I, K, L)
ws = torch.zeros(wsb, dtype=torch.uint8, device=dev)
nslm.nslm_moe_stack_decode(arr, L, E, K, lg, x, 1, y, ws, wsb)
torch.cuda.synchronize()
res = {"lib": nslm.LIB_PATH, "status": nslm.nslm_device_status(ws), "y": y.cpu().numpy().ravel().tolist()}
if nslm.LIB_PATH.endswith("trace/libnslm.so"):
    t = nslm.nslm_debug_stack_trace().astype(np.int64)
    G = torch.cuda.get_device_properties(dev).multi_processor_count
    order = [0, 1, 2, 3, 5, 6, 4]
    ok = True
    for l in range(L):
        for c in range(min(G, 256)):
            seq = [int(t[k, c, l]) for k in (order if l < L - 1 else order[:-1])]
            ok &= all(a <= b for a, b in zip(seq, seq[1:])) and seq[0] > 0
            if l + 1 < L and l < L - 1:
                ok &= int(t[4, c, l]) <= int(t[0, c, l + 1])
    res["ordered"] = bool(ok)
print(json.dumps(res))
"""


def _run(variant):
    env = dict(os.environ)
    env.pop("NSLM_STREAM_SOURCE", None)
    if variant:
        env["NSLM_LIB_VARIANT"] = variant
    else:
        env.pop("NSLM_LIB_VARIANT", None)
    r = subprocess.run([sys.executable, "-c", CASE, ROOT], env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    return json.loads(r.stdout.strip().splitlines()[-1])


def test_trace_build_stamps_in_order_and_same_output():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lib = os.path.join(ROOT, "lfsr_seeded_moe_b200", "_build", "trace", "libnslm.so")
    assert os.path.exists(lib), "build it with python -m lfsr_seeded_moe_b200.build --trace"
    tr, main = _run("trace"), _run(None)
    assert tr["lib"].endswith(os.path.join("trace", "libnslm.so"))
    assert tr["status"] == 0 and main["status"] == 0
    assert tr["ordered"] is True
    assert tr["y"] == main["y"]  # the stamps change no arithmetic
