"""The adapter slot policy on the host (page "LoRA hot load and adapter routing",
adapter lifecycle: least recently used adapter out when the slots are full), and
the load call's argument checks.  No GPU: nothing here launches a kernel or copy."""
import ctypes
import random

import pytest

import lora_adapter_application_b200 as lora
from lora_adapter_application_b200 import LoraError


class Model:
    """The policy written out plainly: a hit keeps its slot; a miss takes the lowest
    free slot, else the unpinned slot acquired longest ago."""

    def __init__(self, n):
        self.key = [-1] * n
        self.last = [0] * n
        self.pins = [0] * n
        self.t = 0

    def acquire(self, k):
        self.t += 1
        if k in self.key:
            i = self.key.index(k)
            self.last[i] = self.t
            self.pins[i] += 1
            return i, True
        free = [i for i, v in enumerate(self.key) if v < 0]
        if free:
            i = free[0]
        else:
            cand = [i for i in range(len(self.key)) if self.pins[i] == 0]
            if not cand:
                return None
            i = min(cand, key=lambda j: self.last[j])
        self.key[i], self.last[i], self.pins[i] = k, self.t, 1
        return i, False

    def release(self, i):
        self.pins[i] -= 1


@pytest.fixture(scope="module")
def lib():
    from lora_adapter_application_b200 import build
    build.build()
    return lora.load()


@pytest.mark.parametrize("seed", range(6))
def test_lru_matches_the_plain_policy(lib, seed):
    g = random.Random(seed)
    n = g.choice([1, 2, 4, 8])
    cache, model = lora.SlotCache(n), Model(n)
    held = []
    for _ in range(400):
        if held and g.random() < 0.45:
            i = held.pop(g.randrange(len(held)))
            cache.release(i)
            model.release(i)
            continue
        k = g.randrange(3 * n)
        want = model.acquire(k)
        if want is None:
            with pytest.raises(LoraError, match="CAPACITY"):
                cache.acquire(k)
            continue
        assert cache.acquire(k) == want
        held.append(want[0])
        for s in range(n):
            assert cache.key(s) == model.key[s]


def test_pins_and_eviction(lib):
    c = lora.SlotCache(2)
    assert c.acquire(7) == (0, False)
    assert c.acquire(9) == (1, False)
    with pytest.raises(LoraError, match="CAPACITY"):   # both slots pinned
        c.acquire(11)
    with pytest.raises(LoraError, match="CAPACITY"):   # pinned: cannot evict
        c.evict(7)
    c.release(0)
    with pytest.raises(LoraError, match="SHAPE"):      # no pin left to release
        c.release(0)
    assert c.acquire(11) == (0, False)                 # 7 was the only unpinned one
    c.release(0)
    c.release(1)
    c.evict(9)
    assert c.key(1) == -1
    assert c.acquire(9) == (1, False)                  # a free slot again
    assert c.acquire(11) == (0, True)
    with pytest.raises(LoraError):
        lora.SlotCache(0)


def test_load_host_checks(lib):
    fake = ctypes.c_void_p(0x1000)
    sl = (lora.lora_slice * 1)()
    sl[0].A, sl[0].B, sl[0].d_out, sl[0].col_off = 0x1000, 0x1000, 64, 0
    src = (ctypes.c_void_p * 1)(0x1000)

    def call(n=0, r=8, r_max=16, N=4, dtype=0, slices=sl, S=1):
        return lib.lora_load_adapter(slices, S, 128, r_max, N, n, r, src, src, 16.0, fake, fake,
                                     dtype, None)
    assert call(r=0) == -4 and call(r=17) == -4            # LORA_ERR_RANK
    assert call(n=4) == -3 and call(n=-1) == -3 and call(S=0) == -3   # LORA_ERR_SHAPE
    assert call(dtype=3) == -2                             # LORA_ERR_DTYPE
    assert lib.lora_load_adapter(None, 1, 128, 16, 4, 0, 8, src, src, 1.0, fake, fake, 0, None) == -1
