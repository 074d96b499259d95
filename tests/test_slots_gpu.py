"""Adapters loaded into slots and evicted, batch after batch, then applied:
every batch's rows match the oracle on the adapters the slots hold
(page "LoRA hot load and adapter routing", adapter lifecycle; page
"Multi-LoRA Serving", section 3.2, max_loras resident adapters)."""
import numpy as np
import pytest
import torch

import lora_adapter_application_b200 as lora
import oracle
from gpu_helpers import assert_within

pytestmark = pytest.mark.gpu


def test_load_evict_cycles_then_apply(cuda_lib):
    g = torch.Generator().manual_seed(3)
    d_in, d_out, r_max, n_slots, T = 256, [192, 64], 32, 4, 160
    pool = []   # adapters on the host: (rank, alpha, [A_s [r, d_in]], [B_s [d_out_s, r]])
    for k in range(10):
        r = [8, 16, 32, 5, 24][k % 5]
        A = [(torch.randn(r, d_in, generator=g) / d_in ** 0.5).to(torch.bfloat16) for _ in d_out]
        B = [(torch.randn(d, r, generator=g) / d_in ** 0.5).to(torch.bfloat16) for d in d_out]
        pool.append((r, float(4 + 4 * (k % 4)), A, B))
    # the stacks start as NaN: a load must overwrite every slot element, padding included
    A = [torch.full((n_slots, r_max, d_in), float("nan"), dtype=torch.bfloat16, device="cuda")
         for _ in d_out]
    B = [torch.full((n_slots, d, r_max), float("nan"), dtype=torch.bfloat16, device="cuda")
         for d in d_out]
    ranks = torch.ones(n_slots, dtype=torch.int32, device="cuda")
    alphas = torch.zeros(n_slots, dtype=torch.float32, device="cuda")
    cache = lora.SlotCache(n_slots)
    meta = lora.Meta(T, n_slots, 64, 0, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    loads = 0
    for batch in range(8):
        keys = torch.randperm(10, generator=g)[: 1 + batch % 4].tolist()
        slot_of = {}
        for j, k in enumerate(keys):
            slot, resident = cache.acquire(k)
            slot_of[k] = slot
            if not resident:
                r, alpha, sa, sb = pool[k]
                if j % 2:   # from pinned host memory
                    src_a, src_b = [t.pin_memory() for t in sa], [t.pin_memory() for t in sb]
                else:       # from device memory
                    src_a, src_b = [t.cuda() for t in sa], [t.cuda() for t in sb]
                lora.lora_load_adapter(A, B, slot, src_a, src_b, alpha, ranks, alphas)
                loads += 1
        # a batch over the resident adapters (and some rows without one)
        which = torch.randint(0, len(keys), (T,), generator=g)
        ids = torch.tensor([slot_of[keys[int(i)]] for i in which], dtype=torch.int32)
        ids[torch.rand(T, generator=g) < 0.1] = -1
        x = torch.randn(T, d_in, generator=g).to(torch.bfloat16)
        y0 = torch.randn(T, sum(d_out), generator=g).to(torch.bfloat16)
        lora.lora_build_segments(ids.cuda(), meta, status)
        y = y0.cuda()
        lora.lora_add_linear(y, x.cuda(), A, B, [0, d_out[0]], ranks, alphas, meta, status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        # reference: the logical adapters, zero-padded, per slot
        A_ref = [torch.zeros(n_slots, r_max, d_in, dtype=torch.bfloat16) for _ in d_out]
        B_ref = [torch.zeros(n_slots, d, r_max, dtype=torch.bfloat16) for d in d_out]
        rk = torch.ones(n_slots, dtype=torch.int32)
        for k, s in slot_of.items():
            r, alpha, sa, sb = pool[k]
            rk[s] = r
            for i in range(len(d_out)):
                A_ref[i][s, :r] = sa[i]
                B_ref[i][s, :, :r] = sb[i]
        ref = y0.double().numpy().copy()
        for k, s in slot_of.items():
            rows = np.nonzero((ids == s).numpy())[0].astype(np.int32)
            if len(rows):
                ref[rows] = oracle.lora_apply(x, A_ref, B_ref, [0, d_out[0]], rk, pool[k][1], ids,
                                              y0, rows=rows)
        assert_within(y.cpu().double().numpy(), ref, torch.bfloat16, f"batch {batch}")
        for s in slot_of.values():
            cache.release(s)
    assert loads > n_slots   # slots were reused: some loads evicted an earlier adapter
    assert torch.equal(ranks.cpu(), torch.tensor([pool[cache.key(s)][0] for s in range(n_slots)],
                                                 dtype=torch.int32))
