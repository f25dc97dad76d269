"""Failure detection: the bounded device waits give up after their limit and
report it (status and abort words), the kernel returns, and the context
stays usable.  Nothing here faults, traps or hangs a GPU: each wait is for an
event that never comes, with a limit of about 10 ms."""
import time

import numpy as np
import pytest
import torch

import guard

from oracle import oracle as O
from lfsr_seeded_moe_b200 import synth

pytestmark = pytest.mark.gpu

LIMIT = 20_000_000  # SM clocks, ~10 ms


@pytest.fixture(scope="module")
def nslm():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from lfsr_seeded_moe_b200 import nslm as n
    return n


def _gemv_still_works(nslm):
    m = synth.seed_matrix(64, 256, 4, (980,))
    x = synth.activations((980,), 1, 256)
    y = guard.buffer((1, 64), torch.float32, fill=float("nan"))
    md = m.to("cuda")
    nslm.nslm_seed_gemv(md, x.cuda(), 1, y)
    torch.cuda.synchronize()
    ref = O.seed_matvec(m.numpy(), synth.bf16_bits(x).numpy().view(np.uint16))
    assert O.normwise_rel_err(y.cpu().numpy(), ref) <= 1e-5


def test_grid_barrier_wait_gives_up_and_reports(nslm):
    out = torch.tensor([0, 0, 0, 0, 7], dtype=torch.int32, device="cuda")  # no arrival will come
    t0 = time.time()
    nslm.nslm_debug_wait_probe(0, out, LIMIT)
    torch.cuda.synchronize()
    assert time.time() - t0 < 5.0
    assert out.cpu().tolist() == [1, 0, 1, 0, 0]  # status 1, abort raised, the wait returned false
    # out[0..3] are laid out as the head of a decode workspace: the status
    # reader maps the give-up to NSLM_ERR_TIMEOUT
    assert nslm.nslm_device_status(out) == nslm.NSLM_ERR_TIMEOUT
    _gemv_still_works(nslm)


def test_grid_barrier_wait_passes_once_arrived(nslm):
    out = torch.tensor([0, 1, 0, 0, 7], dtype=torch.int32, device="cuda")
    nslm.nslm_debug_wait_probe(0, out, LIMIT)
    torch.cuda.synchronize()
    assert out.cpu().tolist() == [0, 1, 0, 0, 1]
    assert nslm.nslm_device_status(out) == nslm.NSLM_OK


def test_grid_barrier_wait_stops_at_the_abort_flag(nslm):
    # another CTA gave up first: the wait ends early and leaves the status alone
    out = torch.tensor([0, 0, 1, 0, 7], dtype=torch.int32, device="cuda")
    t0 = time.time()
    nslm.nslm_debug_wait_probe(0, out, 2_000_000_000)  # ~1 s limit; the flag ends the wait at once
    torch.cuda.synchronize()
    assert time.time() - t0 < 0.5
    assert out.cpu().tolist() == [0, 0, 1, 0, 0]  # a timeout would have set the status word


def test_mbarrier_wait_gives_up_and_passes(nslm):
    out = torch.full((5,), 7, dtype=torch.int32, device="cuda")
    nslm.nslm_debug_wait_probe(1, out, LIMIT)  # nothing completes the phase
    torch.cuda.synchronize()
    assert int(out[0].item()) == 0
    nslm.nslm_debug_wait_probe(2, out, LIMIT)  # one arrival completed it first
    torch.cuda.synchronize()
    assert int(out[0].item()) == 1
    _gemv_still_works(nslm)


def _tag_words(tag, value_bits, abort=0):
    # status, arrivals, abort, spare, passed, seen, then one 64-bit word
    # (value bits, tag) at out[6..7]
    return torch.tensor([0, 0, abort, 0, 7, 7, value_bits, tag], dtype=torch.int32, device="cuda")


def test_tagged_word_wait_gives_up_and_reports(nslm):
    out = _tag_words(0, 12345)  # the tag the wait expects (1) never arrives
    t0 = time.time()
    nslm.nslm_debug_wait_probe(3, out, LIMIT)
    torch.cuda.synchronize()
    assert time.time() - t0 < 5.0
    got = out.cpu().tolist()
    assert got[:5] == [1, 0, 1, 0, 0]  # status 1, abort raised, the wait returned false
    assert nslm.nslm_device_status(out) == nslm.NSLM_ERR_TIMEOUT
    _gemv_still_works(nslm)


def test_tagged_word_wait_passes_and_sees_the_value(nslm):
    bits = int(np.float32(-2.5).view(np.int32))
    out = _tag_words(1, bits)
    nslm.nslm_debug_wait_probe(3, out, LIMIT)
    torch.cuda.synchronize()
    got = out.cpu().tolist()
    assert got[:6] == [0, 0, 0, 0, 1, bits]
    assert nslm.nslm_device_status(out) == nslm.NSLM_OK


def test_tagged_word_wait_stops_at_the_abort_flag(nslm):
    out = _tag_words(0, 0, abort=1)
    t0 = time.time()
    nslm.nslm_debug_wait_probe(3, out, 2_000_000_000)
    torch.cuda.synchronize()
    assert time.time() - t0 < 0.5
    assert out.cpu().tolist()[:5] == [0, 0, 1, 0, 0]
