"""One-token stacks run on the table-form build of the library.

Started by tests/test_gpu_tableform.py in a subprocess with
NSLM_LIB_VARIANT=tableform (the binding then loads
_build/tableform/libnslm.so, whose one-token stack takes phase A's dot
products from per-position tables of x wherever the hidden size is a multiple
of 1024).  Prints one JSON line: for each shape, every layer's normwise error
against the oracle on the GPU's own input, the single-layer FFN's error and
the device status words.
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

SHAPES = [(8, 1024, 256, 3, 4), (6, 2048, 192, 4, 3), (5, 3072, 128, 4, 2), (100, 2048, 1408, 4, 8)]


def main():
    assert nslm.LIB_PATH.endswith(os.path.join("tableform", "libnslm.so")), nslm.LIB_PATH
    dev = torch.device("cuda")
    res = {}
    for E, hidden, inter, P, k in SHAPES:
        name = f"E{E}_{hidden}x{inter}_P{P}_k{k}"
        Lyr, T = (2 if E == 100 else 3), 1
        layers = [synth.moe_layer(l, E, hidden, inter, P, config=951) for l in range(Lyr)]
        logits = torch.stack([synth.router_logits((951, l, hidden), T, E) for l in range(Lyr)])
        xb = synth.activations((951, hidden), T, hidden)
        x, xh = xb.to(dev).contiguous(), synth.bf16_bits(xb).numpy().view(np.uint16)
        dl = [tuple(getattr(m, n).to(dev) for n in ("gate", "up", "down")) for m in layers]
        ys, status = [], []
        for n in range(1, Lyr + 1):
            y = torch.full((T, hidden), float("nan"), device=dev)
            wsb = nslm.nslm_workspace_bytes(nslm.NSLM_OP_MOE_STACK, T, E, hidden, inter, k, n)
            ws = torch.zeros(wsb, dtype=torch.uint8, device=dev)
            nslm.nslm_moe_stack_decode(dl[:n], n, E, k, logits[:n].to(dev).contiguous(), x, T, y, ws, wsb)
            status.append(nslm.nslm_device_status(ws))
            ys.append(y.cpu().numpy().astype(np.float64))
        errs = []
        for l in range(Lyr):
            g, u, d = (getattr(layers[l], n).numpy() for n in ("gate", "up", "down"))
            xl = xh if l == 0 else O.rms_chain(ys[l - 1])
            ids, w = O.route_topk(logits[l].numpy(), k)
            errs.append(O.normwise_rel_err(ys[l], O.moe_ffn(g, u, d, E, hidden, inter, xl, ids, w, mode=0)))
        res[name] = {"layers": errs, "status": status}
        # the single-layer FFN (one persistent launch of one layer)
        L0 = layers[0]
        ids, w = O.route_topk(logits[0].numpy(), k)
        y = torch.full((T, hidden), float("nan"), device=dev)
        wsb = nslm.nslm_workspace_bytes(nslm.NSLM_OP_MOE_FFN, T, E, hidden, inter, k)
        ws = torch.zeros(wsb, dtype=torch.uint8, device=dev)
        nslm.nslm_moe_seed_ffn(*dl[0], E, x, torch.from_numpy(ids).to(dev), torch.from_numpy(w.astype(np.float32)).to(dev),
                               T, k, y, ws, wsb)
        torch.cuda.synchronize()
        g, u, d = (getattr(L0, n).numpy() for n in ("gate", "up", "down"))
        ref = O.moe_ffn(g, u, d, E, hidden, inter, xh, ids, w.astype(np.float32).astype(np.float64), mode=0)
        res[name]["ffn"] = O.normwise_rel_err(y.cpu().numpy(), ref)
    print(json.dumps(res))


if __name__ == "__main__":
    main()
