"""Routed experts in pinned host memory behind the VRAM expert cache: the
device LRU against a plain LRU restated here, and the layer through the cache
against the oracle ("NanoSeedLM" README, "Highlights": experts in host memory,
a VRAM cache of the recently used ones)."""
import numpy as np
import pytest
import torch

import guard

from oracle import oracle as O
from lfsr_seeded_moe_b200 import synth

pytestmark = pytest.mark.gpu

TIGHT = 1e-5


@pytest.fixture(scope="module")
def nslm():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from lfsr_seeded_moe_b200 import nslm as n
    return n


class _LRU:
    """The cache policy: pairs in order; a hit refreshes its slot; a miss takes
    an empty slot (lowest first), else the least recently used slot not used in
    this step (ties to the lowest slot)."""

    def __init__(self, S):
        self.key = [None] * S
        self.tick = [0] * S
        self.clock = 0
        self.hits = self.misses = 0

    def step(self, layer, E, ids):
        self.clock += 1
        out, jobs = [], []
        for e in ids:
            if e < 0 or e >= E:
                out.append(-1)
                continue
            k = (layer, e)
            if k in self.key:
                s = self.key.index(k)
                self.hits += 1
            else:
                cand = [(0 if self.key[s] is None else self.tick[s], s) for s in range(len(self.key))
                        if self.tick[s] != self.clock or self.key[s] is None]
                s = min(cand)[1]
                self.key[s] = k
                jobs.append((e, s))
                self.misses += 1
            self.tick[s] = self.clock
            out.append(s)
        return out, jobs


def _pinned(m):
    return synth.SeedMatrix(m.seeds.pin_memory(), m.coefs.pin_memory(),
                            None if m.codes is None else m.codes.pin_memory(), m.exp_bias.pin_memory(),
                            m.rows, m.K, m.P, m.n_experts)


def _empty_cache(S, rows, K, P):
    nb = K // 8
    return synth.SeedMatrix(guard.buffer((S * rows, nb), torch.int16, fill=0),
                            guard.buffer((S * rows, nb), torch.int16, fill=0),
                            guard.buffer((S * rows, nb // 2), torch.uint8, fill=0) if P == 4 else None,
                            guard.buffer((S * rows,), torch.int32, fill=0), rows, K, P, S)


@pytest.mark.parametrize("T,P", [(1, 4), (2, 3)])
def test_expert_cache_lru_and_layers(nslm, T, P):
    L, E, hidden, inter, k, S = 3, 10, 256, 128, 4, 9
    layers = [synth.moe_layer(l, E, hidden, inter, P, config=960 + P) for l in range(L)]
    host = [tuple(_pinned(getattr(m, n)) for n in ("gate", "up", "down")) for m in layers]
    cache = (_empty_cache(S, inter, hidden, P), _empty_cache(S, inter, hidden, P), _empty_cache(S, hidden, inter, P))
    state = guard.buffer(nslm.nslm_expert_cache_state_bytes(S), torch.uint8, fill=0)
    ref = _LRU(S)
    rng = np.random.default_rng(961)
    wsb = nslm.nslm_workspace_bytes(nslm.NSLM_OP_MOE_FFN, T, S, hidden, inter, k)
    ws = guard.buffer(wsb, torch.uint8)
    for step in range(5):
        for l in range(L):
            ids = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
            if step == 3 and l == 1:
                ids[0, 2] = -1  # a dropped pair
            w = rng.uniform(0.05, 0.4, (T, k)).astype(np.float32)
            dids = torch.from_numpy(ids).cuda()
            slots = guard.buffer((T, k), torch.int32, fill=-7)
            nslm.nslm_expert_cache_fetch(host[l], E, l, cache, S, state, dids, T, k, slots)
            want, _ = ref.step(l, E, ids.reshape(-1).tolist())
            assert slots.cpu().numpy().reshape(-1).tolist() == want, (step, l)
            xb = synth.activations((962, step, l), T, hidden)
            xd, wd = xb.cuda(), torch.from_numpy(w).cuda()
            y = guard.buffer((T, hidden), torch.float32, fill=float("nan"))
            nslm.nslm_moe_seed_ffn(cache[0], cache[1], cache[2], S, xd, slots, wd, T, k, y, ws, wsb)
            torch.cuda.synchronize()
            g, u, d = (getattr(layers[l], n).numpy() for n in ("gate", "up", "down"))
            keep = (ids >= 0) & (ids < E)
            yref = O.moe_ffn(g, u, d, E, hidden, inter, synth.bf16_bits(xb).numpy().view(np.uint16),
                             np.where(keep, ids, 0).astype(np.int32), np.where(keep, w.astype(np.float64), 0.0))
            assert O.normwise_rel_err(y.cpu().numpy(), yref) <= TIGHT, (step, l)
    st = state[:16].view(torch.int32).cpu().tolist()
    assert st[0] == 5 * L and (st[2], st[3]) == (ref.hits, ref.misses)
    assert ref.misses > S  # the steps forced evictions
