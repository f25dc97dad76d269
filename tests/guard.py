"""Canary-padded device buffers for the GPU tests.

There is no compute-sanitizer on the test machines, so the tests check
writes past a buffer's ends themselves: every output, hidden-activation and
workspace buffer handed to the library is carved from a larger allocation with
GUARD bytes on each side filled with a sentinel (0xA5), and after each test
the conftest fixture checks that every sentinel byte is intact.  GUARD is a
multiple of 256, so payloads keep the library's 16-byte alignment.
"""
import torch

GUARD = 1024
SENTINEL = 0xA5
_live = []


def buffer(shape, dtype, fill=None, device="cuda"):
    """A device tensor of `shape`/`dtype` between two sentinel-filled guard
    regions; `fill` (if not None) pre-fills the payload (NaN for outputs, so an
    entry the kernel never writes fails its comparison)."""
    shape = tuple(int(s) for s in (shape if isinstance(shape, (tuple, list)) else (shape,)))
    n = 1
    for s in shape:
        n *= s
    nbytes = n * torch.empty((), dtype=dtype).element_size()
    pad = (-nbytes) % 256
    raw = torch.full((GUARD + nbytes + pad + GUARD,), SENTINEL, dtype=torch.uint8, device=device)
    payload = raw[GUARD:GUARD + nbytes].view(dtype).view(shape)
    if fill is not None:
        payload.fill_(fill)
    _live.append((raw, nbytes + pad))
    return payload


def check_all():
    """Every guard region registered since the last call is intact (then forget them)."""
    if not _live:
        return
    torch.cuda.synchronize()
    bad = []
    for raw, body in _live:
        head = raw[:GUARD]
        tail = raw[GUARD + body:]
        if not bool(torch.all(head == SENTINEL)) or not bool(torch.all(tail == SENTINEL)):
            bad.append((raw.numel() - 2 * GUARD, int(torch.sum(head != SENTINEL)), int(torch.sum(tail != SENTINEL))))
    _live.clear()
    assert not bad, f"writes past a buffer's ends (payload bytes, bytes changed before, after): {bad}"


def forget():
    _live.clear()
