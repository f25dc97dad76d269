"""The nibbles layout of seed packs: device conversion against the oracle's
definition ("Qwen3.8-Flash-Next-NanoSeedLM-P4", "Files"), byte for byte."""
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


@pytest.mark.parametrize("P,N,K", [(4, 7, 48), (4, 64, 1024), (3, 5, 40), (3, 33, 512)])
def test_unpack_and_pack_match_the_oracle_layout(nslm, P, N, K):
    m = synth.seed_matrix(N, K, P, (710, P, N, K))
    c, code = O.blocks_from_streams(m)
    nib = O.nibbles_from_blocks(c, code, P)
    # unpack into buffers pre-filled with junk
    out = synth.seed_matrix(N, K, P, (711, P, N, K)).to("cuda")
    out.seeds = m.seeds.cuda()
    out.exp_bias = m.exp_bias.cuda()
    out.coefs.fill_(0x5A5A)
    if P == 4:
        out.codes.fill_(0xA5)
    nslm.nslm_unpack_nibbles(torch.from_numpy(nib).cuda(), out)
    torch.cuda.synchronize()
    assert torch.equal(out.coefs.cpu(), m.coefs)
    if P == 4:
        assert torch.equal(out.codes.cpu(), m.codes)
    # and back
    nb = guard.buffer(nib.shape, torch.uint8, fill=0xEE)
    md = m.to("cuda")
    nslm.nslm_pack_nibbles(md, nb)
    torch.cuda.synchronize()
    assert np.array_equal(nb.cpu().numpy(), nib)


def test_unpacked_pack_gives_the_same_products(nslm):
    # a pack that arrives in the nibbles layout runs the same GEMV once unpacked
    N, K, P = 256, 2048, 4
    m = synth.seed_matrix(N, K, P, (712,))
    c, code = O.blocks_from_streams(m)
    nib = torch.from_numpy(O.nibbles_from_blocks(c, code, P)).cuda()
    out = synth.seed_matrix(N, K, P, (713,)).to("cuda")
    out.seeds, out.exp_bias = m.seeds.cuda(), m.exp_bias.cuda()
    nslm.nslm_unpack_nibbles(nib, out)
    x = synth.activations((712,), 1, K).cuda()
    y0 = guard.buffer((1, N), torch.float32, fill=float("nan"))
    y1 = guard.buffer((1, N), torch.float32, fill=float("nan"))
    md = m.to("cuda")
    nslm.nslm_seed_gemv(nslm.matrix(md), x, 1, y0)
    nslm.nslm_seed_gemv(nslm.matrix(out), x, 1, y1)
    torch.cuda.synchronize()
    assert torch.equal(y0, y1)
