"""GPU parity of the tensor-core batched path (tcgen05) against the oracle.

The batched path rounds each regenerated weight to bf16 (nearest even) and
the hidden activation h to bf16; the oracle mirrors exactly that arithmetic in
fp64 (seed_matvec_bf16w, moe_ffn mode 1).  Products of bf16 values are exact
in fp32, so the GEMM matches to fp32 accumulation error; the FFN also sees
occasional one-ulp differences of bf16(h) between fp32 and fp64 SiLU*up.
"""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from lfsr_seeded_moe_b200 import synth

pytestmark = pytest.mark.gpu

TOL = 2e-3


@pytest.fixture(scope="module")
def nslm():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from lfsr_seeded_moe_b200 import nslm as n
    return n


def _status(ws):
    return int(ws[:4].view(torch.int32).item())


@pytest.mark.parametrize("P", [3, 4])
@pytest.mark.parametrize("rows,K,counts", [
    (256, 512, [0, 5, 40, 300]),      # an empty expert; one expert over 256 rows (two N tiles)
    (200, 192, [17, 1, 64]),          # ragged row tile (200 = 128 + 72), K of three slices
    (128, 2048, [256, 3]),
])
def test_grouped_gemm_matches_bf16_oracle(nslm, P, rows, K, counts):
    E = len(counts)
    R = sum(counts)
    W = synth.seed_matrix(rows, K, P, (960, rows, K, P), E)
    xb = synth.activations((960, R), R, K)
    offs = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    y = torch.full((R, rows), float("nan"), device="cuda")
    wsb = nslm.nslm_workspace_bytes(nslm.NSLM_OP_GROUPED_GEMM, R, E, K, rows, 1)
    ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
    nslm.nslm_seed_grouped_gemm(W.to("cuda"), E, xb.cuda(), torch.from_numpy(offs).cuda(), R, y, ws, wsb)
    torch.cuda.synchronize()
    assert _status(ws) == 0
    got = y.cpu().numpy()
    xf = xb.double().numpy()
    for e in range(E):
        a, b = offs[e], offs[e + 1]
        if a == b:
            continue
        ref = O.seed_matvec_bf16w(W.expert(e).numpy(), xf[a:b])
        err = O.normwise_rel_err(got[a:b], ref)
        assert err <= 1e-5, (e, err)


def _batched_case(nslm, E, hidden, inter, P, T, k, tag, zipf=None, sample=None):
    dev = torch.device("cuda")
    L = synth.moe_layer(0, E, hidden, inter, P, config=tag)
    xb = synth.activations((tag, T), T, hidden)
    logits = synth.router_logits((tag, T), T, E, zipf)
    ids, w = O.route_topk(logits.numpy(), k)
    y = torch.full((T, hidden), float("nan"), device=dev)
    wsb = nslm.nslm_workspace_bytes(nslm.NSLM_OP_MOE_FFN, T, E, hidden, inter, k)
    ws = torch.zeros(wsb, dtype=torch.uint8, device=dev)
    w32 = w.astype(np.float32)
    nslm.nslm_moe_seed_ffn(L.gate.to(dev), L.up.to(dev), L.down.to(dev), E, xb.to(dev),
                           torch.from_numpy(ids).to(dev), torch.from_numpy(w32).to(dev), T, k, y, ws, wsb)
    torch.cuda.synchronize()
    assert _status(ws) == 0
    toks = np.arange(T) if sample is None else np.asarray(sample)
    g, u, d = (getattr(L, n).numpy() for n in ("gate", "up", "down"))
    xh = synth.bf16_bits(xb).numpy().view(np.uint16)
    ref = O.moe_ffn(g, u, d, E, hidden, inter, xh[toks], ids[toks], w32[toks].astype(np.float64), mode=1)
    return y.cpu().numpy()[toks], ref


@pytest.mark.parametrize("P", [3, 4])
@pytest.mark.parametrize("T", [9, 64])
def test_batched_ffn_small(nslm, P, T):
    got, ref = _batched_case(nslm, 16, 256, 128, P, T, 4, 961)
    assert np.all(np.isfinite(got))
    assert O.normwise_rel_err(got, ref) <= TOL


def test_batched_ffn_zipf_skew(nslm):
    # skewed routing: popular experts receive many rows (several N tiles)
    got, ref = _batched_case(nslm, 24, 320, 192, 3, 300, 8, 962, zipf=1.1)
    assert O.normwise_rel_err(got, ref) <= TOL


def _every_row_within(got, ref):
    # every token row on its own scale, so an error confined to one tile of
    # one expert cannot hide behind the other rows' magnitudes
    assert np.all(np.isfinite(got))
    errs = [O.normwise_rel_err(got[t], ref[t]) for t in range(got.shape[0])]
    worst = int(np.argmax(errs))
    assert errs[worst] <= TOL, (worst, errs[worst], O.elementwise_rel_err(got[worst], ref[worst]))
    assert O.normwise_rel_err(got, ref) <= TOL


def test_batched_ffn_layer_64_tokens(nslm):
    # batched MoE layer: 64 tokens, 100 experts, hidden 2048, intermediate 1408, P=3, top-8;
    # every token row against the oracle
    got, ref = _batched_case(nslm, 100, 2048, 1408, 3, 64, 8, 963)
    _every_row_within(got, ref)


@pytest.mark.parametrize("zipf", [None, 1.1])
def test_batched_ffn_layer_512_tokens(nslm, zipf):
    # the benchmarked batched layers (uniform and Zipf s=1.1 routing), every
    # token row against the oracle: hot experts take several N tiles, and the
    # last ragged M tile and late tiles' epilogues are all compared
    got, ref = _batched_case(nslm, 100, 2048, 1408, 3, 512, 8, 964, zipf=zipf)
    _every_row_within(got, ref)
