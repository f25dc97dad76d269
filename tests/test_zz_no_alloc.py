"""The allocation-free decode FFN entry point (nslm_moe_seed_ffn_static).

It exists for callers that may not allocate device memory -- code inside a
host application whose allocator owns the GPU, latency-critical loops, or
callers that are only handed input and output pointers.  It must give the
same result as nslm_moe_seed_ffn with a caller-provided workspace, and keep
giving it when called again (its scratch array keeps the previous call's
contents); it must match the oracle on its own; and a call after the first
must not take any device memory.  This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import guard

from oracle import oracle as O
from lfsr_seeded_moe_b200 import synth

pytestmark = pytest.mark.gpu

TIGHT = 1e-5


@pytest.fixture(scope="module")
def nslm():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from lfsr_seeded_moe_b200 import nslm as n
    return n


def _rel(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-30))


@pytest.mark.parametrize("E,hidden,inter,P,T,k", [
    (100, 2048, 1408, 4, 1, 8),   # the one-token decode layer
    (16, 256, 128, 3, 5, 4),
    (16, 512, 256, 4, 8, 8),      # T = 8, the largest batch of the decode path
])
def test_static_scratch_matches_workspace_entry_point_and_oracle_twice(nslm, E, hidden, inter, P, T, k):
    dev = torch.device("cuda")
    L = synth.moe_layer(0, E, hidden, inter, P, device=dev, config=950)
    xb = synth.activations((950, T), T, hidden)
    x = xb.to(dev)
    logits = synth.router_logits((950, T), T, E)
    ids = guard.buffer((T, k), torch.int32)
    w = guard.buffer((T, k), torch.float32)
    nslm.nslm_moe_route_topk(logits.to(dev), T, E, k, ids, w)

    ref = guard.buffer((T, hidden), torch.float32, fill=float("nan"))
    wsb = nslm.nslm_workspace_bytes(nslm.NSLM_OP_MOE_FFN, T, E, hidden, inter, k)
    ws = guard.buffer(wsb, torch.uint8)
    nslm.nslm_moe_seed_ffn(L.gate, L.up, L.down, E, x, ids, w, T, k, ref, ws, wsb)

    outs = [guard.buffer((T, hidden), torch.float32, fill=float("nan")) for _ in range(2)]
    nslm.nslm_moe_seed_ffn_static(L.gate, L.up, L.down, E, x, ids, w, T, k, outs[0])
    torch.cuda.synchronize()
    free_before = torch.cuda.mem_get_info()[0]
    nslm.nslm_moe_seed_ffn_static(L.gate, L.up, L.down, E, x, ids, w, T, k, outs[1])
    torch.cuda.synchronize()
    free_after = torch.cuda.mem_get_info()[0]
    assert free_after >= free_before, "a repeated call took device memory"
    assert nslm.nslm_device_status(None) == nslm.NSLM_OK

    r = ref.cpu().numpy()
    assert np.all(np.isfinite(r))
    g, u, d = (getattr(L, n).numpy() for n in ("gate", "up", "down"))
    want = O.moe_ffn(g, u, d, E, hidden, inter, synth.bf16_bits(xb).numpy().view(np.uint16),
                     ids.cpu().numpy(), w.cpu().numpy().astype(np.float64), mode=0)
    for y in outs:
        yy = y.cpu().numpy()
        assert np.all(np.isfinite(yy))
        assert _rel(yy, r) <= TIGHT
        assert O.normwise_rel_err(yy, want) <= TIGHT, O.elementwise_rel_err(yy, want)


def test_static_scratch_rejects_a_problem_larger_than_its_array(nslm):
    # T=8, k=8, inter=hidden=4096: the h buffer alone is 1 MiB, so the call
    # must refuse before launching anything (dummy, aligned pointers).
    E, hidden, inter = 2, 4096, 4096
    g = nslm.nslm_seed_matrix(0x10000, 0x20000, 0x30000, 0x40000, E * inter, hidden, 4)
    d = nslm.nslm_seed_matrix(0x10000, 0x20000, 0x30000, 0x40000, E * hidden, inter, 4)
    rc = nslm.raw().nslm_moe_seed_ffn_static(ctypes.byref(g), ctypes.byref(g), ctypes.byref(d), E,
                                             0x50000, 0x60000, 0x70000, 8, 8, 0x80000, 0)
    assert rc == nslm.NSLM_ERR_WORKSPACE
    assert nslm.nslm_last_launch_count() == 0
