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

import guard

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


@pytest.mark.parametrize("P", [3, 4, 35])
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
    y = guard.buffer((R, rows), torch.float32, fill=float("nan"))
    wsb = nslm.nslm_workspace_bytes(nslm.NSLM_OP_GROUPED_GEMM, R, E, K, rows, 1)
    ws = guard.buffer(wsb, torch.uint8, fill=0)
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
    y = guard.buffer((T, hidden), torch.float32, fill=float("nan"))
    wsb = nslm.nslm_workspace_bytes(nslm.NSLM_OP_MOE_FFN, T, E, hidden, inter, k)
    ws = guard.buffer(wsb, torch.uint8, fill=0)
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


@pytest.mark.parametrize("P", [3, 4, 35])
@pytest.mark.parametrize("T", [9, 64])
def test_batched_ffn_small(nslm, P, T):
    got, ref = _batched_case(nslm, 16, 256, 128, P, T, 4, 961)
    assert np.all(np.isfinite(got))
    assert O.normwise_rel_err(got, ref) <= TOL


def test_batched_ffn_zipf_skew(nslm):
    # skewed routing: popular experts receive many rows (several N tiles)
    got, ref = _batched_case(nslm, 24, 320, 192, 3, 300, 8, 962, zipf=1.1)
    assert O.normwise_rel_err(got, ref) <= TOL


def _split_case(nslm, E, hidden, inter, P, T, k, tag, zipf=None):
    """One tensor-core FFN call, checked stage by stage.

    The kernel rounds the hidden activation h = SiLU(g) * u to bf16 from its
    fp32 accumulators, the oracle from fp64.  Where h lies within that fp32
    error of a bf16 midpoint the two round differently, and with these fields
    (a few large-code blocks dominate a row) one such flip moves a row of y by
    up to ~3e-3.  So the checks are: (1) the kernel's h equals the oracle's
    bf16(h) except for rare entries one rounding step away; (2) each token row
    of y equals the oracle's down projection of the kernel's own h (the kernel
    takes the rounding decision, as the tests do wherever floating point
    decides a discrete value); (3) the whole output is within the stated bar of
    the oracle's end-to-end result."""
    dev = torch.device("cuda")
    L = synth.moe_layer(0, E, hidden, inter, P, config=tag)
    xb = synth.activations((tag, T), T, hidden)
    logits = synth.router_logits((tag, T), T, E, zipf)
    ids, w = O.route_topk(logits.numpy(), k)
    y = guard.buffer((T, hidden), torch.float32, fill=float("nan"))
    wsb = nslm.nslm_workspace_bytes(nslm.NSLM_OP_MOE_FFN, T, E, hidden, inter, k)
    ws = guard.buffer(wsb, torch.uint8, fill=0)
    w32 = w.astype(np.float32)
    nslm.nslm_moe_seed_ffn(L.gate.to(dev), L.up.to(dev), L.down.to(dev), E, xb.to(dev),
                           torch.from_numpy(ids).to(dev), torch.from_numpy(w32).to(dev), T, k, y, ws, wsb)
    hg = guard.buffer((T * k, inter), torch.int16, fill=-1)
    nslm.nslm_debug_batched_hidden(ws, wsb, T, E, hidden, inter, k, hg)
    torch.cuda.synchronize()
    assert _status(ws) == 0
    y = y.cpu().numpy().astype(np.float64)
    hg = O.bf16_to_f64(hg.cpu().numpy().view(np.uint16))
    x64 = O.bf16_to_f64(synth.bf16_bits(xb).numpy().view(np.uint16))
    h64 = np.zeros((T * k, inter))
    hbound = np.zeros((T * k, inter))
    y_e2e = np.zeros((T, hidden))
    y_own_h = np.zeros((T, hidden))
    flat = ids.reshape(-1)
    for e in np.unique(flat):
        pairs = np.nonzero(flat == e)[0]
        toks = pairs // k  # a token routes to an expert at most once
        G, U, D = (O.bf16_to_f64(O.decompress_bf16(getattr(L, n).expert(int(e)).numpy()))
                   for n in ("gate", "up", "down"))
        g = O.dense_matvec(G, x64[toks])
        u = O.dense_matvec(U, x64[toks])
        # a bound on the kernel's error in h before rounding: a sum of K
        # exact products accumulated in fp32, in any order and even with
        # truncating additions, is within K * 2^-23 of the sum of |terms|;
        # propagated through SiLU(g) * u (|SiLU'| <= 1.1), plus 2^-20 |h| for
        # the fast exp and divide
        dg = hidden * 2.0 ** -23 * O.dense_matvec(np.abs(G), np.abs(x64[toks]))
        du = hidden * 2.0 ** -23 * O.dense_matvec(np.abs(U), np.abs(x64[toks]))
        with np.errstate(over="ignore"):
            sg = O.silu(g)
            hh = sg * u
        hbound[pairs] = 1.1 * np.abs(u) * dg + np.abs(sg) * du + 2.0 ** -20 * np.abs(hh)
        h64[pairs] = hh
        wp = w32[pairs // k, pairs % k].astype(np.float64)[:, None]
        y_e2e[toks] += wp * O.dense_matvec(D, O.bf16_to_f64(O.f64_to_bf16(hh)))
        y_own_h[toks] += wp * O.dense_matvec(D, hg[pairs])
    return y, hg, h64, hbound, y_own_h, y_e2e


def _check_split(y, hg, h64, hbound, y_own_h, y_e2e):
    assert np.all(np.isfinite(y)) and np.all(np.isfinite(hg))
    # (1) h: where the kernel's bf16 h differs from the oracle's bf16(h), the
    # kernel's value must lie within its fp32 error bound of the oracle's fp64
    # h, plus its own rounding to bf16 (half a step, at most 2^-8 relative):
    # a rounding flip, or a few steps where g or u cancel, never more
    hb = O.bf16_to_f64(O.f64_to_bf16(h64))
    diff = hb != hg
    bad = diff & (np.abs(hg - h64) > hbound + 2.0 ** -8 * np.abs(hg))
    if np.any(bad):
        idx = np.argwhere(bad)[:6]
        info = [(int(a), int(b), h64[a, b], hb[a, b], hg[a, b], hbound[a, b]) for a, b in idx]
        raise AssertionError(f"{int(np.sum(bad))} h entries outside the fp32 error bound "
                             f"(pair, col, h64, bf16(h64), kernel, bound): {info}")
    assert np.mean(diff) <= 0.1, float(np.mean(diff))
    # (2) every token row against the down projection of the kernel's own h
    errs = [O.normwise_rel_err(y[t], y_own_h[t]) for t in range(y.shape[0])]
    worst = int(np.argmax(errs))
    assert errs[worst] <= 1e-4, (worst, errs[worst], O.elementwise_rel_err(y[worst], y_own_h[worst]))
    # (3) the whole output against the oracle end to end
    assert O.normwise_rel_err(y, y_e2e) <= TOL


def test_batched_ffn_layer_64_tokens(nslm):
    # batched MoE layer: 64 tokens, 100 experts, hidden 2048, intermediate 1408, P=3, top-8
    _check_split(*_split_case(nslm, 100, 2048, 1408, 3, 64, 8, 963))


@pytest.mark.parametrize("zipf", [None, 1.1])
def test_batched_ffn_layer_512_tokens(nslm, zipf):
    # the benchmarked batched layers (uniform and Zipf s=1.1 routing), every
    # token row: hot experts take several N tiles, and the last ragged M tile
    # and late tiles' epilogues are all compared
    _check_split(*_split_case(nslm, 100, 2048, 1408, 3, 512, 8, 964, zipf=zipf))


def test_batched_hidden_export_rejects_decode_sizes(nslm):
    import ctypes
    rc = nslm.raw().nslm_debug_batched_hidden(ctypes.c_void_p(0x10000), 1 << 20, 8, 4, 256, 128, 2,
                                              ctypes.c_void_p(0x20000), None)
    assert rc == nslm.NSLM_ERR_SHAPE
