"""Pins for the CPU oracle: each check ties the oracle to something other than
itself -- a hand-derived fixture, a closed form, brute force, an invariant of
the mathematics, or a library routine."""
import os

import numpy as np
import pytest
import torch

from oracle import oracle as O
from lfsr_seeded_moe_b200 import synth

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _read_rows(name):
    rows = []
    with open(os.path.join(GOLD, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line)
    return rows


class _M:
    """A packed matrix as plain NumPy arrays."""

    def __init__(self, seeds, coefs, codes, eb, P):
        self.seeds, self.coefs, self.codes, self.exp_bias, self.P = seeds, coefs, codes, eb, P


# ------------------------------------------------------------------ LFSR

def test_period_is_maximal_and_visits_every_state():
    # maximal length: from any non-zero seed the register returns after exactly
    # 65,535 steps, visiting every non-zero state once (the pages search all
    # 65,535 seeds, so the register must be maximal)
    s = O.states(1, 65536)
    assert s[65535] == 1
    body = s[:65535].astype(np.int64)
    assert np.all(body != 0)
    assert len(np.unique(body)) == 65535
    for seed in (2, 0x1234, 0xFFFF, 0x8000):
        assert O.lfsr_period(seed) == 65535


def test_zero_seed_is_fixed():
    assert np.all(O.states(0, 40) == 0)
    assert O.lfsr_period(0) == 0


def test_states_match_hand_derivation():
    rows = [r.split() for r in _read_rows("lfsr_seed1.txt")]
    want = np.array([int(h, 16) for _, h in rows], np.uint16)
    assert np.array_equal(O.states(1, len(want)), want)


def test_states_are_windows_of_the_output_bit_stream():
    # s_t = (W >> t) & 0xFFFF where bit 16+k of W is the recurrence
    # W_k ^ W_{k+2} ^ W_{k+3} ^ W_{k+5} on the bit stream (not register stepping)
    rng = np.random.default_rng(7)
    for seed in list(rng.integers(1, 65536, 200)) + [1, 0xFFFF]:
        bits = [(int(seed) >> i) & 1 for i in range(16)]
        for k in range(40):
            bits.append(bits[k] ^ bits[k + 2] ^ bits[k + 3] ^ bits[k + 5])
        W = sum(b << i for i, b in enumerate(bits))
        st = O.states(int(seed), 41)
        for t in range(41):
            assert int(st[t]) == (W >> t) & 0xFFFF


# ----------------------------------------------------------------- basis

def test_basis_fill_order_and_offset_match_hand_blocks():
    for line in _read_rows("blocks_seed1.txt"):
        cs, ws = line.split("|")
        c = [int(v) for v in cs.split()]
        want = np.array([float(v) for v in ws.split()])
        got = O.regen_block(1, c, code=15, bias=0)
        assert np.array_equal(got, want), (c, got, want)


def test_basis_values_are_centred_states():
    U = O.basis(0x1234, 4)
    st = O.states(0x1234, 33).astype(np.float64)
    for r in range(8):
        for j in range(4):
            assert U[r, j] == (st[1 + 8 * j + r] - 32768.0) / 32768.0
    assert np.all(U >= -1.0) and np.all(U < 1.0)


def test_p3_basis_is_first_three_columns_of_p4():
    for seed in (1, 77, 0xBEEF, 65535):
        assert np.array_equal(O.basis(seed, 3), O.basis(seed, 4)[:, :3])


def test_regen_is_linear_and_scaled_by_powers_of_two():
    rng = np.random.default_rng(3)
    for _ in range(50):
        seed = int(rng.integers(1, 65536))
        a = rng.integers(-4, 4, 4)
        b = rng.integers(-4, 4, 4)
        wa = O.regen_block(seed, a, 3, -2)
        wb = O.regen_block(seed, b, 3, -2)
        assert np.array_equal(O.regen_block(seed, a + b, 3, -2), wa + wb)
        assert np.array_equal(O.regen_block(seed, a, 4, -2), 2.0 * wa)
        assert np.array_equal(O.regen_block(seed, a, 0, 1), wa)


def test_zero_seed_closed_form():
    # every state is 0 -> every basis entry is -1 -> w_r = -2^(code+bias) sum(c)
    for c, code, bias in [((1, 2, 3, 4), 5, -5), ((-8, 7, 0, 1), 15, -12), ((3, -2, 1), 0, 4)]:
        w = O.regen_block(0, c, code, bias)
        assert np.all(w == -(2.0 ** (code + bias)) * sum(c))


# --------------------------------------------------------------- packing

def test_packed_field_positions():
    for line in _read_rows("pack_examples.txt"):
        head, cc, wv = line.split("|")
        P, coefs, codes, parity, bias = head.split()
        P, coefs, codes, parity, bias = int(P), int(coefs, 16), int(codes, 16), int(parity), int(bias)
        want_w = float(wv)
        nb = 2  # two blocks so both code nibbles exist
        seeds = np.zeros((1, nb), np.uint16)
        cf = np.zeros((1, nb), np.uint16)
        cf[0, parity] = coefs
        cd = np.array([[codes]], np.uint8) if P == 4 else None
        m = _M(seeds, cf, cd, np.array([bias], np.int32), P)
        w = O.decompress(m, np.float64)
        assert np.all(w[0, 8 * parity: 8 * parity + 8] == want_w), (line, w)


def test_bits_per_weight_match_the_published_pack_sizes():
    # "120.8 B routed expert weights ... 68.0 GB, at 4.5 bits each" (P4) and
    # 60.4 GB expert bytes for P3 (Qwen3.8-Flash-Next-NanoSeedLM-P4 card, "The family")
    n_weights = 120.8e9
    p4 = O.packed_bytes(8, 16 * 1024, 4) - 4 * 8   # streams only
    p3 = O.packed_bytes(8, 16 * 1024, 3) - 4 * 8
    bpw4 = p4 * 8 / (8 * 16 * 1024)
    bpw3 = p3 * 8 / (8 * 16 * 1024)
    assert bpw4 == 4.5 and bpw3 == 4.0
    assert round(n_weights * bpw4 / 8 / 1e9, 1) == 68.0
    assert round(n_weights * bpw3 / 8 / 1e9, 1) == 60.4


def test_decompress_is_exact_in_fp32():
    for P in (3, 4):
        m = synth.seed_matrix(64, 256, P, (101, P)).numpy()
        for bias in (-100, -12, 0, 100):
            m.exp_bias = np.full(64, bias, np.int32)
            w32 = O.decompress(m, np.float32)
            w64 = O.decompress(m, np.float64)
            assert np.array_equal(w32.astype(np.float64), w64)


# --------------------------------------------------------------- matvec

@pytest.mark.parametrize("P", [3, 4])
def test_seed_matvec_equals_dense_fp64_product(P):
    N, K, M = 96, 512, 3
    m = synth.seed_matrix(N, K, P, (102, P)).numpy()
    x = synth.bf16_bits(synth.activations((102, P), M, K)).numpy().view(np.uint16)
    y = O.seed_matvec(m, x)
    w = O.decompress(m, np.float64)
    y_dense = O.dense_matvec(w, O.bf16_to_f64(x))
    assert np.max(np.abs(y - y_dense)) <= 1e-12 * np.max(np.abs(y_dense))


def test_bf16_rounding_matches_torch_rne():
    rng = np.random.default_rng(11)
    v = rng.standard_normal(20000).astype(np.float32)
    # exact ties: low 16 bits 0x8000
    ties = (rng.integers(0, 2**31, 2000, dtype=np.int64).astype(np.uint32) & 0x7FFF0000) | 0x8000
    ties = (ties & 0x7F7FFFFF).view(np.float32)
    v = np.concatenate([v, ties, -ties, np.float32([1.0, -2.5, 3e38, 1e-30])])
    got = O.f64_to_bf16(v.astype(np.float64))
    want = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, want)
    assert np.array_equal(O.bf16_to_f64(want), torch.from_numpy(want.view(np.int16)).view(torch.bfloat16).double().numpy())


def test_bf16_weights_matvec_matches_rounded_dense_product():
    m = synth.seed_matrix(40, 256, 3, (104,)).numpy()
    x = np.random.default_rng(1).standard_normal((2, 256))
    w = O.decompress(m, np.float32)
    wb = torch.from_numpy(w).to(torch.bfloat16).double().numpy()
    y = O.seed_matvec_bf16w(m, x)
    y_ref = x @ wb.T
    assert np.max(np.abs(y - y_ref)) <= 1e-12 * np.max(np.abs(y_ref))


# -------------------------------------------------------------- routing

def test_route_topk_matches_sort_and_softmax():
    rng = np.random.default_rng(5)
    logits = rng.standard_normal((50, 100)).astype(np.float32)
    logits[3, :] = 0.25                      # all tied -> ids 0..7
    logits[4, 10] = logits[4, 20] = 9.0      # a tie at the top -> 10 before 20
    ids, w = O.route_topk(logits, 8)
    for t in range(50):
        order = np.lexsort((np.arange(100), -logits[t].astype(np.float64)))[:8]
        assert np.array_equal(ids[t], order)
        sel = logits[t, order].astype(np.float64)
        sm = np.exp(sel - sel.max())
        assert np.allclose(w[t], sm / sm.sum(), rtol=1e-14, atol=0)
    assert np.array_equal(ids[3], np.arange(8))
    assert np.allclose(w[3], 1 / 8)
    assert ids[4, 0] == 10 and ids[4, 1] == 20


# ---------------------------------------------------------------- FFN

@pytest.mark.parametrize("mode", [0, 1])
def test_moe_ffn_equals_dense_composition(mode):
    E, hidden, inter, P, T, k = 6, 64, 48, 4, 3, 2
    L = synth.moe_layer(0, E, hidden, inter, P, config=103)
    g, u, d = (getattr(L, n).numpy() for n in ("gate", "up", "down"))
    x = synth.bf16_bits(synth.activations((103,), T, hidden)).numpy().view(np.uint16)
    logits = synth.router_logits((103,), T, E).numpy()
    ids, w = O.route_topk(logits, k)
    y = O.moe_ffn(g, u, d, E, hidden, inter, x, ids, w, mode=mode)

    def dense(m):
        wt = O.decompress(m, np.float64)
        if mode == 1:
            wt = torch.from_numpy(wt.astype(np.float32)).to(torch.bfloat16).double().numpy()
        return wt

    Wg, Wu, Wd = dense(g), dense(u), dense(d)
    xf = O.bf16_to_f64(x)
    y_ref = np.zeros((T, hidden))
    for t in range(T):
        for q in range(k):
            e = ids[t, q]
            gg = Wg[e * inter:(e + 1) * inter] @ xf[t]
            uu = Wu[e * inter:(e + 1) * inter] @ xf[t]
            h = gg / (1 + np.exp(-gg)) * uu
            if mode == 1:
                h = torch.from_numpy(h.astype(np.float32)).to(torch.bfloat16).double().numpy() \
                    if np.all(np.abs(h) < 3e38) else h
            y_ref[t] += w[t, q] * (Wd[e * hidden:(e + 1) * hidden] @ h)
    tol = 1e-12 if mode == 0 else 1e-2 / 256  # mode 1: h rounded from fp32 vs fp64 may tie-flip
    assert O.normwise_rel_err(y, y_ref) <= tol


def test_silu_closed_forms():
    assert O.silu(0.0) == 0.0
    assert abs(O.silu(40.0) - 40.0) < 1e-12
    assert abs(O.silu(-40.0)) < 1e-15
    assert abs(O.silu(1.0) - 1.0 / (1.0 + np.exp(-1.0))) < 1e-16


def test_layer_stack_chaining_normalises():
    E, hidden, inter, P, L, k = 4, 32, 16, 4, 3, 2
    layers = []
    for li in range(L):
        m = synth.moe_layer(li, E, hidden, inter, P, config=105)
        layers.append(tuple(getattr(m, n).numpy() for n in ("gate", "up", "down")))
    logits = np.stack([synth.router_logits((105, li), 1, E).numpy() for li in range(L)])
    x0 = synth.bf16_bits(synth.activations((105,), 1, hidden)).numpy().view(np.uint16)
    y, xs = O.layer_stack(layers, logits, x0, hidden, inter, E, k)
    assert len(xs) == L and np.array_equal(xs[0], x0)
    for li in range(1, L):
        xf = O.bf16_to_f64(xs[li])
        assert abs(np.sqrt(np.mean(xf * xf)) - 1.0) < 1e-2


# Closed forms for the layer chaining x' = bf16(y / sqrt(mean(y^2) + 1e-6)),
# worked by hand.  bf16 keeps 8 significant bits, so a value v in [2^e, 2^(e+1))
# is a multiple of 2^(e-7) after rounding.
#   * y = (3, 4, 0, 0): mean(y^2) = 25/4, r = 2.5 (the 1e-6 moves r by 2e-7):
#     1.2 lies between 1.1953125 and 1.203125 (step 2^-7) and is nearer the
#     upper; 1.6 lies between 1.59375 and 1.6015625, nearer the upper.  A sum
#     in place of the mean would give r = 5 and (0.6, 0.8).
#   * y = 1e-4 everywhere: mean(y^2) = 1e-8, r = sqrt(1.01e-6), so every
#     entry is 1e-4 / sqrt(1.01e-6) = 1 / sqrt(101) = 0.0995037...; in
#     [2^-4, 2^-3) the step is 2^-11, and 0.0995037 * 2048 = 203.78, so RNE
#     gives 204 / 2048 = 0.099609375 where truncation gives 203 / 2048.  Without
#     the epsilon every entry would be 1.0; with 1e-5 it would be 0.0316...
_RMS_CASES = [
    (np.array([3.0, 4.0, 0.0, 0.0]), np.array([1.203125, 1.6015625, 0.0, 0.0])),
    (np.array([-3.0, 0.0, 4.0, 0.0]), np.array([-1.203125, 0.0, 1.6015625, 0.0])),
    (np.full(8, 1e-4), np.full(8, 204.0 / 2048.0)),
]


@pytest.mark.parametrize("case", range(len(_RMS_CASES)))
def test_rms_chain_closed_forms(case):
    y, want = _RMS_CASES[case]
    got = O.bf16_to_f64(O.rms_chain(y[None, :]))[0]
    assert np.array_equal(got, want)


def test_rms_chain_normalises_each_token_on_its_own():
    # three tokens whose scales differ by 10^6: per-token normalisation maps
    # each to the same closed form (3, 4, 0, 0) -> (1.203125, 1.6015625, 0, 0);
    # one norm over the whole batch would shrink the small tokens to ~0
    y = np.array([[3.0, 4.0, 0.0, 0.0], [3e3, 4e3, 0.0, 0.0], [-6.0, -8.0, 0.0, 0.0]])
    got = O.bf16_to_f64(O.rms_chain(y))
    assert np.array_equal(got[0], [1.203125, 1.6015625, 0.0, 0.0])
    assert np.array_equal(got[1], [1.203125, 1.6015625, 0.0, 0.0])
    assert np.array_equal(got[2], [-1.203125, -1.6015625, 0.0, 0.0])


def test_layer_stack_feeds_each_layer_its_predecessors_normalised_output():
    # layer l+1's input must be the normalised OUTPUT of layer l (not its input):
    # run the layers one at a time with moe_ffn (pinned on its own above), then
    # check the chained input is proportional to that output, at unit RMS, to
    # bf16 precision
    E, hidden, inter, P, L, k, T = 6, 64, 32, 4, 3, 2, 3
    layers = []
    for li in range(L):
        m = synth.moe_layer(li, E, hidden, inter, P, config=106)
        layers.append(tuple(getattr(m, n).numpy() for n in ("gate", "up", "down")))
    logits = np.stack([synth.router_logits((106, li), T, E).numpy() for li in range(L)])
    x0 = synth.bf16_bits(synth.activations((106,), T, hidden)).numpy().view(np.uint16)
    _, xs = O.layer_stack(layers, logits, x0, hidden, inter, E, k)
    for li in range(L - 1):
        g, u, d = layers[li]
        ids, w = O.route_topk(logits[li], k)
        y = O.moe_ffn(g, u, d, E, hidden, inter, xs[li], ids, w, mode=0)
        nxt = O.bf16_to_f64(xs[li + 1])
        for t in range(T):
            rms = np.sqrt(np.mean(y[t] ** 2))
            # each entry within half a bf16 step (2^-8 relative) of y / rms
            assert np.all(np.abs(nxt[t] - y[t] / rms) <= (2.0 ** -8 + 1e-4) * np.abs(y[t] / rms))
            assert abs(np.sqrt(np.mean(nxt[t] ** 2)) - 1.0) < 4e-3


# --------------------------------------------------------------- search

@pytest.mark.parametrize("P", [3, 4])
def test_search_recovers_a_planted_block_with_zero_error(P):
    rng = np.random.default_rng(20 + P)
    for _ in range(2):
        seed = int(rng.integers(1, 65536))
        c = rng.integers(-8, 8, P)
        c[int(rng.integers(0, P))] |= 1          # an odd entry makes the code identifiable
        code = int(rng.integers(0, 16))
        bias = -12
        w = O.regen_block(seed, c, code, bias)
        s, cc, cd, err = O.search_block(w, P, bias)
        assert (s, cd, err) == (seed, code, 0.0)
        assert np.array_equal(cc, c)


def test_search_without_the_planted_seed_has_positive_error():
    w = O.regen_block(40000, [3, -5, 1, 7], 9, -12)
    s, c, code, err = O.search_block(w, 4, -12, 1, 39999)
    assert err > 0 and s != 40000


def test_search_matches_brute_force_on_a_tiny_range():
    # brute force over 32 seeds x 16 codes x all 16^3 coefficient vectors (P=3)
    rng = np.random.default_rng(9)
    w = rng.standard_normal(8) * 0.01
    bias = -12
    s, c, code, err = O.search_block(w, 3, bias, 100, 131)
    grid = np.stack(np.meshgrid(*[np.arange(-8, 8)] * 3, indexing="ij"), -1).reshape(-1, 3)
    best = np.inf
    for seed in range(100, 132):
        U = O.basis(seed, 3)
        V = grid @ U.T                                   # [4096][8]
        for cd in range(16):
            e = np.sum((w[None, :] - 2.0 ** (cd + bias) * V) ** 2, axis=1)
            best = min(best, e.min())
    # the search rounds least-squares coefficients, so it can only be >= the true optimum;
    # on random blocks rounding the LS solution is close to optimal
    assert err >= best - 1e-18
    assert err <= 4.0 * best


# ---- activation-weighted search ([QWEN] "How it works": the error of each
# weight weighted by the mean square of its input activation)

def _weighted_search_numpy(w, d, P, bias, lo, hi):
    """The weighted search restated with numpy's least squares: for every seed
    and code, c = clamp(rint(argmin_c |D^1/2 (w - 2^e U c)|)), err weighted;
    smallest error, then larger code, then lower seed."""
    sq = np.sqrt(d)
    best = (np.inf, 0, 0, 0, None)
    for seed in range(lo, hi + 1):
        U = O.basis(seed, P)
        proj = np.linalg.lstsq(sq[:, None] * U, sq * w, rcond=None)[0]
        for code in range(15, -1, -1):
            sc = 2.0 ** (code + bias)
            c = np.clip(np.rint(proj / sc), -8, 7).astype(np.int64)
            err = float(np.sum(d * (w - sc * (U @ c)) ** 2))
            key = (err, -code, seed)
            if key < best[:3]:
                best = (err, -code, seed, code, c)
    return best[2], best[4], best[3], best[0]


@pytest.mark.parametrize("P", [3, 4])
def test_weighted_search_matches_a_numpy_least_squares_restatement(P):
    rng = np.random.default_rng(70 + P)
    bias = -12
    for _ in range(3):
        w = rng.standard_normal(8) * 2.0 ** (bias + 14)
        d = rng.uniform(0.05, 4.0, 8)
        s, c, code, err = O.search_block(w, P, bias, 500, 531, d8=d)
        rs, rc, rcode, rerr = _weighted_search_numpy(w, d, P, bias, 500, 531)
        assert (s, code) == (rs, rcode)
        assert np.array_equal(c, rc)
        assert abs(err - rerr) <= 1e-12 * rerr


def test_weighted_search_with_unit_importances_is_the_plain_search():
    rng = np.random.default_rng(80)
    w = rng.standard_normal(8) * 2.0 ** 3
    s, c, code, err = O.search_block(w, 4, -12, 1, 2000, d8=np.ones(8))
    s0, c0, code0, err0 = O.search_block(w, 4, -12, 1, 2000)
    assert (s, code, err) == (s0, code0, err0) and np.array_equal(c, c0)


@pytest.mark.parametrize("P", [3, 4])
def test_weighted_search_scales_with_the_importances(P):
    # importances times a power of two: same choice, error times that power
    # exactly (d enters the fit and the error consistently)
    rng = np.random.default_rng(90 + P)
    w = rng.standard_normal(8) * 2.0 ** 2
    d = rng.uniform(0.1, 3.0, 8)
    s, c, code, err = O.search_block(w, P, -12, 1, 3000, d8=d)
    s2, c2, code2, err2 = O.search_block(w, P, -12, 1, 3000, d8=d * 8.0)
    assert (s, code) == (s2, code2) and np.array_equal(c, c2)
    assert err2 == 8.0 * err


@pytest.mark.parametrize("P", [3, 4])
def test_weighted_search_recovers_a_planted_block(P):
    rng = np.random.default_rng(100 + P)
    seed = int(rng.integers(1, 65536))
    c = rng.integers(-8, 8, P)
    c[0] |= 1
    code = int(rng.integers(0, 16))
    w = O.regen_block(seed, c, code, -12)
    s, cc, cd, err = O.search_block(w, P, -12, d8=rng.uniform(0.01, 10.0, 8))
    assert (s, cd, err) == (seed, code, 0.0)
    assert np.array_equal(cc, c)


def test_weighting_changes_the_choice():
    # a block with a large weight at one position: the weighted search fits
    # that position better than the plain one does
    rng = np.random.default_rng(110)
    w = rng.standard_normal(8) * 2.0 ** 2
    d = np.full(8, 1e-3)
    d[5] = 1.0
    s, c, code, _ = O.search_block(w, 4, -12, 1, 4000)
    sw, cw, codew, _ = O.search_block(w, 4, -12, 1, 4000, d8=d)
    fit = lambda s_, c_, code_: abs(w[5] - O.regen_block(s_, c_, code_, -12)[5])
    assert (s, code) != (sw, codew)
    assert fit(sw, cw, codew) < fit(s, c, code)


# ---- the nibbles layout (seeds, nibbles, exp_bias)

def test_nibbles_layout_matches_hand_encoded_rows():
    n = 0
    for line in _read_rows("nibbles_examples.txt"):
        P, blocks, hexs = [t.strip() for t in line.split("|")]
        P = int(P)
        cs, cds = [], []
        for blk in blocks.split():
            cc, cd = blk.split(":")
            cs.append([int(v) for v in cc.split(",")])
            cds.append(int(cd))
        nib = O.nibbles_from_blocks([cs], [cds], P)
        assert [int(v, 16) for v in hexs.split()] == nib[0].tolist()
        c, code = O.blocks_from_nibbles(nib, 1, 8 * len(cs), P)
        assert c[0].tolist() == cs and code[0].tolist() == cds
        n += 1
    assert n == 4


@pytest.mark.parametrize("P", [3, 4])
def test_nibbles_round_trip_and_p3_identity(P):
    m = synth.seed_matrix(5, 64, P, (700, P))
    c, code = O.blocks_from_streams(m)
    nib = O.nibbles_from_blocks(c, code, P)
    assert nib.shape == (5, (P + 1) * 8 // 2)
    c2, code2 = O.blocks_from_nibbles(nib, 5, 64, P)
    assert np.array_equal(c, c2) and np.array_equal(code, code2)
    if P == 3:  # 4 nibbles per block in the same order as the coefs word
        assert np.array_equal(nib, m.coefs.numpy().view(np.uint16).astype("<u2").view(np.uint8).reshape(5, -1))


# ---- P = 3 with 5-bit coefficients (P = 35)

def test_p3c5_layout_matches_hand_encoded_blocks():
    n = 0
    for line in _read_rows("p3c5_examples.txt"):
        q, row, b, bias, fields, weight = [t.strip() for t in line.split("|")]
        b, bias = int(b), int(bias)
        m = synth.seed_matrix(1, 64, 35, (720,))
        m.seeds.zero_()
        m.coefs.zero_()
        m.coefs[0, b] = int(np.array(int(q, 16), np.uint16).view(np.int16))
        m.codes[0] = torch.tensor([int(v, 16) for v in row.split()], dtype=torch.uint8)
        m.exp_bias.fill_(bias)
        w = O.decompress(m, np.float64)[0].reshape(8, 8)
        assert np.all(w[b] == float(weight)), (line, w[b])
        c0, c1, c2, code = (int(v) for v in fields.split())
        assert float(weight) == -2.0 ** (code + bias) * (c0 + c1 + c2)
        others = [i for i in range(8) if i != b]
        assert np.all(w[others] == 0.0)  # zero coefficients, whatever their codes
        n += 1
    assert n == 3


def test_p3c5_matvec_equals_dense_product_and_reaches_5bit_values():
    m = synth.seed_matrix(16, 128, 35, (721,))
    x = synth.activations((721,), 2, 128)
    xb = synth.bf16_bits(x).numpy().view(np.uint16)
    w = O.decompress(m, np.float64)
    assert O.normwise_rel_err(O.seed_matvec(m, xb), O.dense_matvec(w, O.bf16_to_f64(xb))) <= 1e-14
    # coefficients beyond the int4 range occur: |sum_j c_j U| reaches 3 * 16
    assert np.max(np.abs(w)) * 2.0 ** 12 > 24.0

