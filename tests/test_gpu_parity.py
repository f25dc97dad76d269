"""GPU parity: the CUDA library (through its C ABI) against the CPU oracle.

Regenerated weights must be bit-exact; products must be within 2e-3 of the
fp64 oracle in the normwise relative error max|y - ref| / max|ref|.
"""
import numpy as np
import pytest
import torch

import guard

from oracle import oracle as O
from lfsr_seeded_moe_b200 import synth

pytestmark = pytest.mark.gpu

TOL = 2e-3          # the stated bar (fp32 accumulate vs fp64 oracle)
TIGHT = 1e-5        # what the fp32 decode path actually reaches; a regression guard


@pytest.fixture(scope="module")
def nslm():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from lfsr_seeded_moe_b200 import nslm as n
    return n


def _out(*shape):
    """Output buffer pre-filled with NaN, so an entry the kernel never wrote fails."""
    return guard.buffer(shape, torch.float32, fill=float("nan"))


def _dev(m):
    return m.to("cuda")


def _x(tag, M, K):
    xb = synth.activations(tag, M, K)
    return xb.cuda().contiguous(), synth.bf16_bits(xb).numpy().view(np.uint16)


def _all_seed_matrix(P, bias_lo=-100, bias_hi=100):
    """512 x 1024 matrix whose 65,536 blocks hold every seed value 0..65535 once."""
    N, K = 512, 1024
    m = synth.seed_matrix(N, K, P, (900, P))
    m.seeds = torch.arange(65536, dtype=torch.int32).to(torch.int16).reshape(N, K // 8).contiguous()
    m.exp_bias = torch.linspace(bias_lo, bias_hi, N).round().to(torch.int32)
    return m


@pytest.mark.parametrize("P", [3, 4, 35])
def test_decompress_fp32_bit_exact_all_seeds(nslm, P):
    m = _all_seed_matrix(P)
    md = _dev(m)
    w = _out(m.N, m.K)
    nslm.nslm_debug_decompress(md, w)
    torch.cuda.synchronize()
    ref = O.decompress(m.numpy(), np.float32)
    got = w.cpu().numpy()
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))


@pytest.mark.parametrize("P", [3, 4, 35])
def test_decompress_bf16_bit_exact_all_seeds(nslm, P):
    # the tensor-core tile producer's routine, over every seed and biases
    # -100..100 (every weight a normal bf16 number)
    m = _all_seed_matrix(P)
    md = _dev(m)
    w = guard.buffer((m.N, m.K), torch.int16, fill=-1)
    nslm.nslm_debug_decompress_bf16(md, w)
    torch.cuda.synchronize()
    ref = O.decompress_bf16(m.numpy())
    assert np.array_equal(w.cpu().numpy().view(np.uint16), ref)


@pytest.mark.parametrize("P,N,K", [(3, 37, 8 * 13), (4, 29, 16 * 7), (3, 5, 8), (4, 3, 16)])
def test_decompress_ragged_rows_bit_exact(nslm, P, N, K):
    # rows whose block count is not a multiple of 8 (the decode kernels' ragged
    # chunk loads) or is odd (the bf16 producer's last block pairs with an
    # empty one); every entry is written, none past the end
    m = synth.seed_matrix(N, K, P, (905, N, K, P))
    m.exp_bias = torch.linspace(-100, 100, N).round().to(torch.int32)
    md = _dev(m)
    pad = 64
    w = guard.buffer((N * K + pad,), torch.float32, fill=float("nan"))
    nslm.nslm_debug_decompress(md, w)
    wb = guard.buffer((N * K + pad,), torch.int16, fill=-1)
    nslm.nslm_debug_decompress_bf16(md, wb)
    torch.cuda.synchronize()
    got = w.cpu().numpy()
    ref = O.decompress(m.numpy(), np.float32).reshape(-1)
    assert np.array_equal(got[:N * K].view(np.uint32), ref.view(np.uint32))
    assert np.all(np.isnan(got[N * K:]))
    gb = wb.cpu().numpy().view(np.uint16)
    assert np.array_equal(gb[:N * K], O.decompress_bf16(m.numpy()).reshape(-1))
    assert np.all(gb[N * K:] == 0xFFFF)


GEMV_SHAPES = [(512, 1024), (2048, 4096), (4096, 2048), (1408, 2048), (2048, 1408)]


@pytest.mark.parametrize("P", [3, 4, 35])
@pytest.mark.parametrize("N,K", GEMV_SHAPES)
def test_gemv_matches_oracle(nslm, P, N, K):
    m = synth.seed_matrix(N, K, P, (901, N, K, P))
    x, xh = _x((901, K), 1, K)
    y = _out(1, N)
    nslm.nslm_seed_gemv(_dev(m), x, 1, y)
    torch.cuda.synchronize()
    ref = O.seed_matvec(m.numpy(), xh)
    err = O.normwise_rel_err(y.cpu().numpy(), ref)
    assert err <= TOL and err <= TIGHT, err


@pytest.mark.parametrize("P", [4, 35])
def test_gemv_long_rows_matches_oracle(nslm, P):
    # 16,384-weight rows: two CTAs' shared memory no longer fit on one SM, so
    # the one-vector kernel runs one CTA per SM (eight rounds of tasks each)
    N, K = 2048, 16384
    m = synth.seed_matrix(N, K, P, (905, N, K, P))
    x, xh = _x((905, K), 1, K)
    y = _out(1, N)
    nslm.nslm_seed_gemv(_dev(m), x, 1, y)
    torch.cuda.synchronize()
    ref = O.seed_matvec(m.numpy(), xh)
    err = O.normwise_rel_err(y.cpu().numpy(), ref)
    assert err <= TOL and err <= TIGHT, (err, O.elementwise_rel_err(y.cpu().numpy(), ref))


@pytest.mark.parametrize("P", [3, 4, 35])
def test_gemv_fields_ready_chain_matches_oracle(nslm, P):
    # back-to-back GEMVs with NSLM_GEMV_FIELDS_READY (each one's weight copies
    # start before its predecessor ends); the activations of the second are
    # written by the kernel just before it, which the flag must still wait for
    N, K = 2048, 4096
    ms = [synth.seed_matrix(N, K, P, (904, c, P)) for c in range(3)]
    x, xh = _x((904, P), 1, K)
    ys = [_out(1, N) for _ in ms]
    x2 = torch.empty_like(x)
    for i, m in enumerate(ms):
        if i == 1:
            x2.copy_(x)                       # a kernel that writes the next GEMV's input
        nslm.nslm_seed_gemv_flags(_dev(m), x2 if i >= 1 else x, 1, ys[i], nslm.NSLM_GEMV_FIELDS_READY)
    torch.cuda.synchronize()
    for m, y in zip(ms, ys):
        ref = O.seed_matvec(m.numpy(), xh)
        assert O.normwise_rel_err(y.cpu().numpy(), ref) <= TIGHT


@pytest.mark.parametrize("M", [2, 3, 8])
@pytest.mark.parametrize("P", [3, 4, 35])
def test_gemv_multi_token(nslm, M, P):
    N, K = 704, 2048
    m = synth.seed_matrix(N, K, P, (902, M, P))
    x, xh = _x((902, M), M, K)
    y = _out(M, N)
    nslm.nslm_seed_gemv(_dev(m), x, M, y)
    torch.cuda.synchronize()
    ref = O.seed_matvec(m.numpy(), xh)
    err = O.normwise_rel_err(y.cpu().numpy(), ref)
    assert err <= TIGHT, err


@pytest.mark.parametrize("P,N,K", [(3, 999, 1000), (4, 1001, 1008), (3, 1, 8), (4, 3, 16),
                                   (4, 130, 4096 + 64 + 16), (3, 77, 520)])
def test_gemv_ragged_shapes(nslm, P, N, K):
    m = synth.seed_matrix(N, K, P, (903, N, K, P))
    x, xh = _x((903, K), 2, K)
    y = _out(2, N)
    nslm.nslm_seed_gemv(_dev(m), x, 2, y)
    torch.cuda.synchronize()
    ref = O.seed_matvec(m.numpy(), xh)
    assert O.normwise_rel_err(y.cpu().numpy(), ref) <= TIGHT


def test_gemv_extreme_fields(nslm):
    # seed 0 (all-zero register), all codes 15, coefficients -8 and 7, bias -100 and +90
    N, K, P = 64, 512, 4
    m = synth.seed_matrix(N, K, P, (904,))
    m.seeds[::3] = 0
    m.coefs[1::2] = torch.tensor(0x8888, dtype=torch.int32).to(torch.int16)
    m.coefs[::2] = 0x7777
    m.codes[:] = torch.tensor(0xFF, dtype=torch.uint8)
    m.exp_bias = torch.tensor([90 if i % 2 else -100 for i in range(N)], dtype=torch.int32)
    x, xh = _x((904,), 1, K)
    y = _out(1, N)
    nslm.nslm_seed_gemv(_dev(m), x, 1, y)
    torch.cuda.synchronize()
    ref = O.seed_matvec(m.numpy(), xh)
    for rows in (slice(0, None, 2), slice(1, None, 2)):  # two magnitudes: compare each
        assert O.normwise_rel_err(y.cpu().numpy()[:, rows], ref[:, rows]) <= TIGHT


def test_route_topk_matches_oracle(nslm):
    T, E, k = 64, 100, 8
    logits = synth.router_logits((905,), T, E)
    logits[3, :] = 0.5                          # all tied
    logits[4, 7] = logits[4, 90] = 5.0          # tie at the top
    ids = guard.buffer((T, k), torch.int32)
    w = _out(T, k)
    nslm.nslm_moe_route_topk(logits.cuda(), T, E, k, ids, w)
    torch.cuda.synchronize()
    rid, rw = O.route_topk(logits.numpy(), k)
    assert np.array_equal(ids.cpu().numpy(), rid)
    assert np.max(np.abs(w.cpu().numpy() - rw)) <= 1e-6


def _ffn_case(nslm, E, hidden, inter, P, T, k, tag, zipf=None):
    L = synth.moe_layer(0, E, hidden, inter, P, config=tag)
    x, xh = _x((tag, T), T, hidden)
    logits = synth.router_logits((tag,), T, E, zipf)
    rid, rw = O.route_topk(logits.numpy(), k)
    ids = torch.from_numpy(rid).cuda()
    w = torch.from_numpy(rw.astype(np.float32)).cuda()
    y = _out(T, hidden)
    wsb = nslm.nslm_workspace_bytes(nslm.NSLM_OP_MOE_FFN, T, E, hidden, inter, k)
    ws = guard.buffer(wsb, torch.uint8)
    nslm.nslm_moe_seed_ffn(_dev(L.gate), _dev(L.up), _dev(L.down), E, x, ids, w, T, k, y, ws, wsb)
    torch.cuda.synchronize()
    g, u, d = (getattr(L, n).numpy() for n in ("gate", "up", "down"))
    ref = O.moe_ffn(g, u, d, E, hidden, inter, xh, rid, rw.astype(np.float32).astype(np.float64), mode=0)
    return y.cpu().numpy(), ref


def _ffn_with_ids(nslm, L, E, hidden, inter, x, rid, w32, k):
    T = rid.shape[0]
    y = _out(T, hidden)
    wsb = nslm.nslm_workspace_bytes(nslm.NSLM_OP_MOE_FFN, T, E, hidden, inter, k)
    ws = guard.buffer(wsb, torch.uint8)
    nslm.nslm_moe_seed_ffn(_dev(L.gate), _dev(L.up), _dev(L.down), E, x, torch.from_numpy(rid).cuda(),
                           torch.from_numpy(w32).cuda(), T, k, y, ws, wsb)
    torch.cuda.synchronize()
    return y.cpu().numpy()


@pytest.mark.parametrize("E,hidden,inter,P,k", [
    (16, 256, 128, 3, 4),      # whole 64-weight chunks
    (12, 272, 120, 3, 8),      # ragged rows in both projections
    (8, 4160, 208, 4, 2),      # 65 chunks per gate row (two rounds per lane), ragged down rows
    (4, 64, 64, 4, 1),         # one chunk per row, one expert per token
    (6, 4096, 128, 4, 2),      # two full rounds of bulk-copied gate/up chunks per lane
    (5, 2560, 192, 3, 3),      # bulk copies: a full round, then 8 chunks
    (4, 2304, 128, 4, 2),      # bulk copies: a full round, then 4 chunks (16 bytes of codes)
])
def test_ffn_one_token_shapes(nslm, E, hidden, inter, P, k):
    tag = 920 + hidden
    y, ref = _ffn_case(nslm, E, hidden, inter, P, 1, k, tag)
    assert O.normwise_rel_err(y, ref) <= TIGHT


def test_ffn_one_token_duplicate_and_dropped_ids(nslm):
    # a token that lists one expert twice gets both contributions; pairs whose
    # expert id is outside [0, E) contribute nothing
    E, hidden, inter, P, k = 10, 512, 256, 4, 6
    L = synth.moe_layer(0, E, hidden, inter, P, config=930)
    x, xh = _x((930, 1), 1, hidden)
    rid = np.array([[3, 3, 7, -1, 12, 0]], dtype=np.int32)
    w32 = np.array([[0.3, 0.2, 0.25, 0.1, 0.05, 0.1]], dtype=np.float32)
    y = _ffn_with_ids(nslm, L, E, hidden, inter, x, rid, w32, k)
    keep = (rid >= 0) & (rid < E)
    oid = np.where(keep, rid, 0).astype(np.int32)
    ow = np.where(keep, w32.astype(np.float64), 0.0)
    g, u, d = (getattr(L, n).numpy() for n in ("gate", "up", "down"))
    ref = O.moe_ffn(g, u, d, E, hidden, inter, xh, oid, ow, mode=0)
    assert O.normwise_rel_err(y, ref) <= TIGHT


def test_ffn_one_token_all_ids_dropped_gives_zero(nslm):
    E, hidden, inter, P, k = 6, 256, 128, 3, 2
    L = synth.moe_layer(0, E, hidden, inter, P, config=931)
    x, _ = _x((931, 1), 1, hidden)
    y = _ffn_with_ids(nslm, L, E, hidden, inter, x, np.array([[-1, 6]], dtype=np.int32),
                      np.array([[0.5, 0.5]], dtype=np.float32), k)
    assert np.array_equal(y, np.zeros_like(y))


def test_ffn_decode_one_token_full_layer(nslm):
    # one MoE layer decode: 100 experts, hidden 2048, intermediate 1408, P=4, top-8
    y, ref = _ffn_case(nslm, 100, 2048, 1408, 4, 1, 8, 906)
    assert O.normwise_rel_err(y, ref) <= TIGHT, O.elementwise_rel_err(y, ref)


@pytest.mark.parametrize("T", [2, 5, 8])
@pytest.mark.parametrize("P", [3, 4])
def test_ffn_decode_batch(nslm, T, P):
    y, ref = _ffn_case(nslm, 16, 256, 128, P, T, 4, 907 + T)
    assert O.normwise_rel_err(y, ref) <= TIGHT


def test_ffn_decode_batch8_full_layer(nslm):
    # 8 tokens on the 100-expert 2048/1408 P=4 layer: about 49 distinct
    # experts, and the 64 routed h vectors are staged for the down projection
    # in several groups
    y, ref = _ffn_case(nslm, 100, 2048, 1408, 4, 8, 8, 940)
    assert O.normwise_rel_err(y, ref) <= TIGHT, O.elementwise_rel_err(y, ref)


@pytest.mark.parametrize("P", [3, 4])
def test_ffn_decode_batch_shared_experts_split_slots(nslm, P):
    # all 8 tokens pick the same experts, so an expert carries up to 9 pairs
    # and the plan splits it into slots of at most 4; one token lists an
    # expert twice, and two pairs name experts outside [0, E)
    E, hidden, inter, k, T = 12, 512, 256, 8, 8
    L = synth.moe_layer(0, E, hidden, inter, P, config=941)
    x, xh = _x((941, T), T, hidden)
    rid = np.tile(np.array([5, 1, 9, 0, 11, 3, 7, 2], dtype=np.int32), (T, 1))
    rid[2, 3] = 5
    rid[6, 0] = -1
    rid[7, 7] = E
    w32 = np.random.default_rng(941).uniform(0.05, 0.3, size=(T, k)).astype(np.float32)
    y = _ffn_with_ids(nslm, L, E, hidden, inter, x, rid, w32, k)
    keep = (rid >= 0) & (rid < E)
    g, u, d = (getattr(L, n).numpy() for n in ("gate", "up", "down"))
    ref = O.moe_ffn(g, u, d, E, hidden, inter, xh, np.where(keep, rid, 0).astype(np.int32),
                    np.where(keep, w32.astype(np.float64), 0.0), mode=0)
    assert O.normwise_rel_err(y, ref) <= TIGHT


def test_ffn_decode_batch_all_ids_dropped_gives_zero(nslm):
    E, hidden, inter, P, k, T = 6, 256, 128, 4, 2, 3
    L = synth.moe_layer(0, E, hidden, inter, P, config=942)
    x, _ = _x((942, T), T, hidden)
    y = _ffn_with_ids(nslm, L, E, hidden, inter, x, np.full((T, k), -1, dtype=np.int32),
                      np.full((T, k), 0.5, dtype=np.float32), k)
    assert np.array_equal(y, np.zeros_like(y))


@pytest.mark.parametrize("P", [3, 4])
def test_ffn_decode_batch_with_an_empty_token(nslm, P):
    # token 2 of 4 has every id out of range: its row is exactly zero and the
    # other tokens still match the oracle (persistent batched kernel)
    E, hidden, inter, k, T = 20, 512, 256, 4, 4
    L = synth.moe_layer(0, E, hidden, inter, P, config=944)
    x, xh = _x((944, T), T, hidden)
    rng = np.random.default_rng(944)
    rid = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    rid[2] = [-1, E, E + 3, -5]
    w32 = rng.uniform(0.05, 0.3, size=(T, k)).astype(np.float32)
    y = _ffn_with_ids(nslm, L, E, hidden, inter, x, rid, w32, k)
    assert np.array_equal(y[2], np.zeros(hidden, np.float32))
    keep = (rid >= 0) & (rid < E)
    g, u, d = (getattr(L, n).numpy() for n in ("gate", "up", "down"))
    ref = O.moe_ffn(g, u, d, E, hidden, inter, xh, np.where(keep, rid, 0).astype(np.int32),
                    np.where(keep, w32.astype(np.float64), 0.0), mode=0)
    assert O.normwise_rel_err(y, ref) <= TIGHT


@pytest.mark.parametrize("T", [1, 3, 12])
def test_ffn_hybrid_p3_p4_experts(nslm, T):
    # experts 0..4 packed with P=3, 5..11 with P=4; one routed pair dropped
    E3, E4, hidden, inter, k = 5, 7, 512, 256, 4
    E = E3 + E4
    L3 = synth.moe_layer(0, E3, hidden, inter, 3, config=945)
    L4 = synth.moe_layer(0, E4, hidden, inter, 4, config=946)
    x, xh = _x((945, T), T, hidden)
    rng = np.random.default_rng(945 + T)
    rid = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    rid[0, 1] = E + 2
    w32 = rng.uniform(0.05, 0.3, (T, k)).astype(np.float32)
    y = _out(T, hidden)
    wsb = nslm.nslm_workspace_bytes(nslm.NSLM_OP_MOE_FFN_HYBRID, T, E, hidden, inter, k)
    ws = guard.buffer(wsb, torch.uint8)
    d3 = tuple(_dev(getattr(L3, n)) for n in ("gate", "up", "down"))
    d4 = tuple(_dev(getattr(L4, n)) for n in ("gate", "up", "down"))
    nslm.nslm_moe_seed_ffn_hybrid(d3, E3, d4, E4, x, torch.from_numpy(rid).cuda(), torch.from_numpy(w32).cuda(),
                                  T, k, y, ws, wsb)
    torch.cuda.synchronize()
    mode = 0 if T <= 8 else 1  # T > 8: the tensor-core path (bf16 weights and h)
    ref = 0.0
    for L, lo, hi in ((L3, 0, E3), (L4, E3, E)):
        keep = (rid >= lo) & (rid < hi)
        g, u, d = (getattr(L, n).numpy() for n in ("gate", "up", "down"))
        ref = ref + O.moe_ffn(g, u, d, hi - lo, hidden, inter, xh, np.where(keep, rid - lo, 0).astype(np.int32),
                              np.where(keep, w32.astype(np.float64), 0.0), mode=mode)
    assert O.normwise_rel_err(y.cpu().numpy(), ref) <= (TIGHT if T <= 8 else TOL)


@pytest.mark.parametrize("T", [1, 3])
def test_ffn_decode_p3c5_layer(nslm, T):
    # the 5-bit P=3 format through the decode FFN (the persistent kernels:
    # T = 1 one-token, T = 3 batched)
    y, ref = _ffn_case(nslm, 10, 512, 256, 35, T, 4, 947 + T)
    assert O.normwise_rel_err(y, ref) <= TIGHT


def test_ffn_decode_p3c5_full_layer(nslm):
    # the benchmarked layer shape (100 experts, 2048/1408, top-8) in the 5-bit format, one token
    y, ref = _ffn_case(nslm, 100, 2048, 1408, 35, 1, 8, 949)
    assert O.normwise_rel_err(y, ref) <= TIGHT, O.elementwise_rel_err(y, ref)


@pytest.mark.parametrize("T", [1, 2])
def test_stack_decode_p3c5(nslm, T):
    Lyr, E, hidden, inter, P, k = 4, 8, 256, 128, 35, 2
    layers = [synth.moe_layer(l, E, hidden, inter, P, config=948) for l in range(Lyr)]
    logits = torch.stack([synth.router_logits((948, l), T, E) for l in range(Lyr)])
    x, xh = _x((948, T), T, hidden)
    dl = [(_dev(m.gate), _dev(m.up), _dev(m.down)) for m in layers]
    ys = [_stack_prefix(nslm, dl, logits, x, T, E, hidden, inter, k, n) for n in range(1, Lyr + 1)]
    for l in range(Lyr):  # each layer on the GPU's own input (a long stack is chaotic)
        g, u, d = (getattr(layers[l], n).numpy() for n in ("gate", "up", "down"))
        xl = xh if l == 0 else O.rms_chain(ys[l - 1])
        ids, w = O.route_topk(logits[l].numpy(), k)
        ref = O.moe_ffn(g, u, d, E, hidden, inter, xl, ids, w, mode=0)
        assert O.normwise_rel_err(ys[l], ref) <= TOL, l


def test_ffn_decode_ragged_and_zipf(nslm):
    y, ref = _ffn_case(nslm, 12, 272, 120, 3, 3, 8, 908, zipf=1.1)
    assert O.normwise_rel_err(y, ref) <= TIGHT


@pytest.mark.parametrize("T", [1, 3])
def test_stack_decode_matches_oracle(nslm, T):
    Lyr, E, hidden, inter, P, k = 4, 8, 256, 128, 4, 2
    layers = [synth.moe_layer(l, E, hidden, inter, P, config=909) for l in range(Lyr)]
    logits = torch.stack([synth.router_logits((909, l), T, E) for l in range(Lyr)])
    x, xh = _x((909, T), T, hidden)
    dl = [(_dev(m.gate), _dev(m.up), _dev(m.down)) for m in layers]
    y = _out(T, hidden)
    wsb = nslm.nslm_workspace_bytes(nslm.NSLM_OP_MOE_STACK, T, E, hidden, inter, k, Lyr)
    ws = guard.buffer(wsb, torch.uint8)
    nslm.nslm_moe_stack_decode(dl, Lyr, E, k, logits.cuda().contiguous(), x, T, y, ws, wsb)
    torch.cuda.synchronize()
    hl = [tuple(getattr(m, n).numpy() for n in ("gate", "up", "down")) for m in layers]
    ref, _ = O.layer_stack(hl, logits.numpy(), xh, hidden, inter, E, k, mode=0)
    assert O.normwise_rel_err(y.cpu().numpy(), ref) <= TOL


def _stack_prefix(nslm, dl, logits, x, T, E, hidden, inter, k, n):
    """Output of the first n layers of a stack (status word checked)."""
    y = _out(T, hidden)
    wsb = nslm.nslm_workspace_bytes(nslm.NSLM_OP_MOE_STACK, T, E, hidden, inter, k, n)
    ws = guard.buffer(wsb, torch.uint8, fill=0)
    nslm.nslm_moe_stack_decode(dl[:n], n, E, k, logits[:n].cuda().contiguous(), x, T, y, ws, wsb)
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == 0
    return y.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("T", [1, 8])
def test_stack_decode_full_layers_pinned(nslm, T):
    # the benchmarked stack configuration (100 experts, 2048/1408, P=4, top-8),
    # one token and 8 tokens, through two layers of one persistent launch;
    # each layer checked against the oracle on the GPU's own input
    Lyr, E, hidden, inter, P, k = 2, 100, 2048, 1408, 4, 8
    layers = [synth.moe_layer(l, E, hidden, inter, P, config=943) for l in range(Lyr)]
    logits = torch.stack([synth.router_logits((943, l, T), T, E) for l in range(Lyr)])
    x, xh = _x((943, T), T, hidden)
    dl = [(_dev(m.gate), _dev(m.up), _dev(m.down)) for m in layers]
    ys = [_stack_prefix(nslm, dl, logits, x, T, E, hidden, inter, k, n) for n in (1, 2)]
    for l in range(Lyr):
        g, u, d = (getattr(layers[l], n).numpy() for n in ("gate", "up", "down"))
        xl = xh if l == 0 else O.rms_chain(ys[l - 1])
        ids, w = O.route_topk(logits[l].numpy(), k)
        ref = O.moe_ffn(g, u, d, E, hidden, inter, xl, ids, w, mode=0)
        # layer 0 to the fp32 decode path's own accuracy; later layers to the
        # stated bar, since the GPU's fp32 normalisation of y and the oracle's
        # fp64 one may round a few inputs to neighbouring bf16 values
        assert O.normwise_rel_err(ys[l], ref) <= (TIGHT if l == 0 else TOL), (l, O.elementwise_rel_err(ys[l], ref))
    assert np.array_equal(ys[1], _stack_prefix(nslm, dl, logits, x, T, E, hidden, inter, k, 2))


@pytest.mark.parametrize("T", [1, 2])
def test_stack_decode_past_one_launch_per_layer(nslm, T):
    # 70 layers run as two persistent launches (64 + 6).  A long
    # stack is chaotic (one bf16 ulp of a layer input changes everything
    # downstream), so each checked layer is fed the GPU's own input: the
    # prefix of l layers gives y_{l-1}, and layer l's output from the prefix
    # of l+1 layers must match the oracle applied to bf16(y_{l-1} / rms).
    Lyr, E, hidden, inter, P, k = 70, 4, 64, 64, 4, 2
    layers = [synth.moe_layer(l, E, hidden, inter, P, config=950) for l in range(Lyr)]
    logits = torch.stack([synth.router_logits((950, l, T), T, E) for l in range(Lyr)])
    x, _ = _x((950, T), T, hidden)
    dl = [(_dev(m.gate), _dev(m.up), _dev(m.down)) for m in layers]

    def prefix(n):
        return _stack_prefix(nslm, dl, logits, x, T, E, hidden, inter, k, n)

    for l in (63, 64, 69):  # the last layer of launch 1, the first and last of launch 2
        y_prev, y_l = prefix(l), prefix(l + 1)
        g, u, d = (getattr(layers[l], n).numpy() for n in ("gate", "up", "down"))
        xl = O.rms_chain(y_prev)
        ids, w = O.route_topk(logits[l].numpy(), k)
        ref = O.moe_ffn(g, u, d, E, hidden, inter, xl, ids, w, mode=0)
        assert O.normwise_rel_err(y_l, ref) <= TOL, l
    y70 = prefix(Lyr)
    assert np.array_equal(y70, prefix(Lyr))  # deterministic run to run
