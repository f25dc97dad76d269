"""GPU seed search (the encoder) against the oracle's brute-force search.

The search must return the oracle's answer bit for bit: the same seed, code
and coefficients, and the same fp64 error, for every block
("NanoSeedLM: LLM inference using pseudo-random numbers", "'GPU search ==
CPU search'").
"""
import numpy as np
import pytest
import torch

import guard

from oracle import oracle as O
from lfsr_seeded_moe_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nslm():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from lfsr_seeded_moe_b200 import nslm as n
    return n


class _Out:
    """Device buffers of a packed matrix for the search to fill."""

    def __init__(self, N, K, P, bias):
        nb = K // 8
        self.N, self.K, self.P = N, K, P
        self.seeds = guard.buffer((N, nb), torch.int16, fill=-1)
        self.coefs = guard.buffer((N, nb), torch.int16, fill=-1)
        self.codes = guard.buffer((N, nb // 2), torch.uint8, fill=0xEE) if P == 4 else None
        self.exp_bias = torch.as_tensor(np.asarray(bias, np.int32)).cuda()

    def fields(self):
        """(seed, c[P], code) per block, unpacked on the host."""
        s = self.seeds.cpu().numpy().view(np.uint16).astype(np.int64)
        q = self.coefs.cpu().numpy().view(np.uint16).astype(np.int64)
        c = np.stack([(((q >> (4 * j)) & 0xF) ^ 8) - 8 for j in range(self.P)], axis=-1)
        if self.P == 4:
            cb = self.codes.cpu().numpy().astype(np.int64)
            code = np.stack([cb & 0xF, cb >> 4], axis=-1).reshape(self.N, -1)
        else:
            code = (q >> 12) & 0xF
        return s, c, code


def _run(nslm, w, P, bias, lo, hi, imp=None):
    N, K = w.shape
    out = _Out(N, K, P, bias)
    err = guard.buffer((N, K // 8), torch.float64, fill=float("nan"))
    dimp = None if imp is None else torch.as_tensor(imp, dtype=torch.float32).cuda()
    nslm.nslm_seed_search(torch.as_tensor(w, dtype=torch.float32).cuda(), out, lo, hi, err, imp=dimp)
    torch.cuda.synchronize()
    s, c, code = out.fields()
    return s, c, code, err.cpu().numpy()


def _compare_with_oracle(w, P, bias, lo, hi, s, c, code, err, imp=None):
    N, K = w.shape
    for i in range(N):
        for b in range(K // 8):
            d8 = None if imp is None else np.asarray(imp[8 * b:8 * b + 8], np.float32).astype(np.float64)
            rs, rc, rcode, rerr = O.search_block(w[i, 8 * b:8 * b + 8].astype(np.float64), P, int(bias[i]), lo, hi,
                                                 d8=d8)
            assert (s[i, b], code[i, b]) == (rs, rcode), (i, b, s[i, b], code[i, b], rs, rcode)
            assert np.array_equal(c[i, b], rc), (i, b)
            assert err[i, b] == rerr, (i, b, err[i, b], rerr)  # bit-identical fp64


@pytest.mark.parametrize("P", [3, 4])
def test_search_recovers_planted_blocks_over_all_seeds(nslm, P):
    # planted (seed, c, code) with an odd coefficient (the code is then
    # identifiable), encoded back from the exact weights over all 65,535 seeds
    rng = np.random.default_rng(40 + P)
    N, K = 2, 32
    bias = [-12, 5]
    w = np.zeros((N, K), np.float32)
    planted = []
    for i in range(N):
        for b in range(K // 8):
            seed = int(rng.integers(1, 65536))
            c = rng.integers(-8, 8, size=P).astype(np.int32)
            c[0] = 2 * int(rng.integers(-4, 4)) + 1
            code = int(rng.integers(0, 16))
            w[i, 8 * b:8 * b + 8] = O.regen_block(seed, c, code, bias[i])
            planted.append((i, b, seed, c, code))
    s, c, code, err = _run(nslm, w, P, bias, 1, 65535)
    for i, b, seed, cc, cd in planted:
        assert (s[i, b], code[i, b]) == (seed, cd)
        assert np.array_equal(c[i, b], cc)
        assert err[i, b] == 0.0


@pytest.mark.parametrize("P,bias", [(3, [-12, -100]), (4, [-12, 90])])
def test_search_matches_oracle_on_gaussian_weights(nslm, P, bias):
    # weights that no seed reproduces exactly: the winner is an approximation,
    # and every step of the fp64 arithmetic decides it
    rng = np.random.default_rng(50 + P)
    N, K = 2, 32
    w = np.zeros((N, K), np.float32)
    for i in range(N):
        w[i] = (rng.standard_normal(K) * 2.0 ** (bias[i] + 14)).astype(np.float32)
    lo, hi = 1000, 2999
    s, c, code, err = _run(nslm, w, P, bias, lo, hi)
    _compare_with_oracle(w, P, bias, lo, hi, s, c, code, err)


@pytest.mark.parametrize("P,bias", [(3, [-12, -40]), (4, [-12, 60])])
def test_weighted_search_matches_oracle(nslm, P, bias):
    # per-column importances (mean square activations): the weighted fit and
    # error, bit for bit
    rng = np.random.default_rng(150 + P)
    N, K = 2, 32
    w = np.zeros((N, K), np.float32)
    for i in range(N):
        w[i] = (rng.standard_normal(K) * 2.0 ** (bias[i] + 14)).astype(np.float32)
    imp = rng.uniform(0.01, 5.0, K).astype(np.float32)
    imp[3] = 0.0  # a column that does not count
    lo, hi = 2000, 3999
    s, c, code, err = _run(nslm, w, P, bias, lo, hi, imp)
    _compare_with_oracle(w, P, bias, lo, hi, s, c, code, err, imp)


@pytest.mark.parametrize("P", [3, 4])
def test_weighted_search_recovers_planted_blocks(nslm, P):
    rng = np.random.default_rng(160 + P)
    N, K = 1, 32
    w = np.zeros((N, K), np.float32)
    planted = []
    for b in range(K // 8):
        seed = int(rng.integers(1, 65536))
        c = rng.integers(-8, 8, size=P).astype(np.int32)
        c[0] = 2 * int(rng.integers(-4, 4)) + 1
        code = int(rng.integers(0, 16))
        w[0, 8 * b:8 * b + 8] = O.regen_block(seed, c, code, -12)
        planted.append((b, seed, c, code))
    s, c, code, err = _run(nslm, w, P, [-12], 1, 65535, rng.uniform(0.1, 8.0, K))
    for b, seed, cc, cd in planted:
        assert (s[0, b], code[0, b]) == (seed, cd)
        assert np.array_equal(c[0, b], cc)
        assert err[0, b] == 0.0


def test_search_full_range_matches_oracle(nslm):
    rng = np.random.default_rng(60)
    w = (rng.standard_normal((1, 16)) * 2.0 ** 2).astype(np.float32)
    s, c, code, err = _run(nslm, w, 4, [-12], 1, 65535)
    _compare_with_oracle(w, 4, [-12], 1, 65535, s, c, code, err)


def test_search_ties_go_to_the_largest_code_then_the_lowest_seed(nslm):
    # all-zero weights: every candidate has c = 0 and error 0
    w = np.zeros((1, 16), np.float32)
    s, c, code, err = _run(nslm, w, 4, [-12], 777, 1234)
    assert list(s[0]) == [777, 777] and list(code[0]) == [15, 15]
    assert np.all(c == 0) and np.all(err == 0.0)
    _compare_with_oracle(w, 4, [-12], 777, 1234, s, c, code, err)


def test_search_argument_checks(nslm):
    w = torch.zeros(1, 16, device="cuda")
    out = _Out(1, 16, 4, [-12])
    for lo, hi in [(0, 10), (10, 65536), (20, 10)]:
        with pytest.raises(nslm.NslmError):
            nslm.nslm_seed_search(w, out, lo, hi)
