"""Small parity cases run on the bounds-check build of the library.

Started by tests/test_gpu_bounds.py in a subprocess with
NSLM_LIB_VARIANT=boundscheck (the binding then loads
_build/boundscheck/libnslm.so, whose kernels compare every checked index with
its extent and record the site instead of making an out-of-range access).
Prints one JSON line: each case's normwise error against the oracle, the
bounds status after all cases (0: no index left its buffer) and the status
after the self-test probe (site 1).
"""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from lfsr_seeded_moe_b200 import nslm, synth  # noqa: E402
from oracle import oracle as O  # noqa: E402


def main():
    assert nslm.LIB_PATH.endswith(os.path.join("boundscheck", "libnslm.so")), nslm.LIB_PATH
    dev = torch.device("cuda")
    res = {"status_start": nslm.nslm_debug_bounds_status()}

    def x_of(tag, M, K):
        xb = synth.activations(tag, M, K)
        return xb.to(dev), synth.bf16_bits(xb).numpy().view(np.uint16)

    # seed GEMV: whole and ragged chunks, one and three vectors, P = 3, 4, 5-bit P = 3
    for P, N, K, M in [(4, 256, 1024, 1), (3, 77, 520, 3), (4, 130, 4160, 1), (35, 64, 1024, 2)]:
        m = synth.seed_matrix(N, K, P, (990, N, K, P))
        x, xh = x_of((990, N), M, K)
        y = torch.full((M, N), float("nan"), device=dev)
        nslm.nslm_seed_gemv(m.to(dev), x, M, y)
        torch.cuda.synchronize()
        res[f"gemv_P{P}_{N}x{K}_M{M}"] = O.normwise_rel_err(y.cpu().numpy(), O.seed_matvec(m.numpy(), xh))

    # debug decompression (fp32 and bf16) on ragged rows
    m = synth.seed_matrix(37, 104, 3, (991,))
    w = torch.empty(37, 104, device=dev)
    nslm.nslm_debug_decompress(m.to(dev), w)
    wb = torch.empty(37, 104, dtype=torch.int16, device=dev)
    nslm.nslm_debug_decompress_bf16(m.to(dev), wb)
    torch.cuda.synchronize()
    res["decompress_exact"] = bool(np.array_equal(w.cpu().numpy(), O.decompress(m.numpy(), np.float32)) and
                                   np.array_equal(wb.cpu().numpy().view(np.uint16), O.decompress_bf16(m.numpy())))

    # routed FFN: decode (T = 1, 3) and tensor-core (T = 12) paths
    for E, hidden, inter, P, T, k in [(16, 256, 128, 4, 1, 4), (12, 272, 120, 3, 3, 8), (16, 256, 128, 3, 12, 4)]:
        L = synth.moe_layer(0, E, hidden, inter, P, config=992)
        x, xh = x_of((992, T), T, hidden)
        logits = synth.router_logits((992, T), T, E)
        ids, wts = O.route_topk(logits.numpy(), k)
        y = torch.full((T, hidden), float("nan"), device=dev)
        wsb = nslm.nslm_workspace_bytes(nslm.NSLM_OP_MOE_FFN, T, E, hidden, inter, k)
        ws = torch.zeros(wsb, dtype=torch.uint8, device=dev)
        w32 = wts.astype(np.float32)
        nslm.nslm_moe_seed_ffn(L.gate.to(dev), L.up.to(dev), L.down.to(dev), E, x, torch.from_numpy(ids).to(dev),
                               torch.from_numpy(w32).to(dev), T, k, y, ws, wsb)
        torch.cuda.synchronize()
        g, u, d = (getattr(L, n).numpy() for n in ("gate", "up", "down"))
        ref = O.moe_ffn(g, u, d, E, hidden, inter, xh, ids, w32.astype(np.float64), mode=1 if T > 8 else 0)
        res[f"ffn_T{T}_P{P}"] = O.normwise_rel_err(y.cpu().numpy(), ref)

    # a three-layer stack in one persistent launch (one token)
    Lyr, E, hidden, inter, P, k, T = 3, 8, 256, 128, 4, 2, 1
    layers = [synth.moe_layer(l, E, hidden, inter, P, config=993) for l in range(Lyr)]
    logits = torch.stack([synth.router_logits((993, l), T, E) for l in range(Lyr)])
    x, xh = x_of((993,), T, hidden)
    y = torch.full((T, hidden), float("nan"), device=dev)
    wsb = nslm.nslm_workspace_bytes(nslm.NSLM_OP_MOE_STACK, T, E, hidden, inter, k, Lyr)
    ws = torch.zeros(wsb, dtype=torch.uint8, device=dev)
    dl = [(m.gate.to(dev), m.up.to(dev), m.down.to(dev)) for m in layers]
    nslm.nslm_moe_stack_decode(dl, Lyr, E, k, logits.to(dev).contiguous(), x, T, y, ws, wsb)
    torch.cuda.synchronize()
    hl = [tuple(getattr(m, n).numpy() for n in ("gate", "up", "down")) for m in layers]
    ref, _ = O.layer_stack(hl, logits.numpy(), xh, hidden, inter, E, k, mode=0)
    res["stack_3_layers"] = O.normwise_rel_err(y.cpu().numpy(), ref)

    res["status_after_cases"] = nslm.nslm_debug_bounds_status()
    probe = synth.seed_matrix(2, 64, 4, (994,))
    nslm.nslm_debug_bounds_probe(probe.to(dev))
    res["status_after_probe"] = nslm.nslm_debug_bounds_status()
    res["status_cleared"] = nslm.nslm_debug_bounds_status()
    print(json.dumps(res))


if __name__ == "__main__":
    main()
