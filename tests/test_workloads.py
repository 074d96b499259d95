"""The seeded input generators produce the batches the benchmark configurations
describe: sizes, id distributions, rank mixes, request structure.  The batch
structure is drawn before any layer tensor, so it is the same at small layer
widths, which keep these checks fast."""
import numpy as np
import pytest
import torch
from scipy import stats

import workloads


def _zipf_fit_pvalue(ids, N, s):
    """Chi-square goodness of fit of the valid ids to P(n) ~ (n + 1)^-s, with the
    tail pooled so that every expected count is at least 5."""
    ids = ids[ids >= 0]
    p = np.arange(1, N + 1, dtype=np.float64) ** -s
    p /= p.sum()
    obs = np.bincount(ids, minlength=N).astype(np.float64)
    exp = p * len(ids)
    cut = int(np.argmax(exp < 5)) if (exp < 5).any() else N
    cut = max(cut, 2)
    o = np.concatenate([obs[:cut], [obs[cut:].sum()]]) if cut < N else obs
    e = np.concatenate([exp[:cut], [exp[cut:].sum()]]) if cut < N else exp
    return stats.chisquare(o, e).pvalue


@pytest.mark.parametrize("name,kw", [
    ("tiny", {}), ("decode_qproj", {"d": 64}), ("prefill", {"d": 32, "n_req": 8}),
    ("multislice_8b", {"T": 64, "hidden": 64, "kv": 16, "inter": 128}),
    ("mixed_70b", {"T": 1024, "n_req": 4, "hidden": 64, "inter": 128}),
])
def test_generators_are_seeded(name, kw):
    a, b, c = (workloads.make(name, seed=s, **kw) for s in (1, 1, 2))
    assert torch.equal(a.ids, b.ids) and torch.equal(a.ranks, b.ranks)
    for la, lb in zip(a.layers, b.layers):
        assert torch.equal(la.x, lb.x) and torch.equal(la.y0, lb.y0)
        assert all(torch.equal(p, q) for p, q in zip(la.A + la.B, lb.A + lb.B))
    assert not torch.equal(a.layers[0].x, c.layers[0].x)


def test_decode_qproj_recipe():
    w = workloads.decode_qproj(seed=0, d=64)
    ids = w.ids.numpy()
    assert (w.T, w.N, w.r_max, w.alpha) == (256, 32, 16, 32.0)
    assert (w.ranks == 16).all()
    assert ids.min() >= -1 and ids.max() < 32
    assert 0.04 <= (ids == -1).mean() <= 0.18           # 10 % without an adapter
    assert _zipf_fit_pvalue(ids, 32, 1.1) > 1e-3
    assert _zipf_fit_pvalue(ids, 32, 0.0) < 1e-3       # and clearly not uniform


def test_prefill_recipe():
    w = workloads.prefill(seed=0, d=32)
    lens = np.array(w.info["lengths"])
    req = np.array(w.info["req_ids"])
    assert len(lens) == 64 and lens.min() >= 128 and lens.max() <= 2048
    assert w.T == int(lens.sum()) == 77431
    assert (req == -1).sum() == 1                       # one base-only request
    per_adapter = np.bincount(req[req >= 0], minlength=8)
    assert per_adapter.sum() == 63 and per_adapter.max() - per_adapter.min() <= 1   # round-robin
    np.testing.assert_array_equal(w.ids.numpy(), np.repeat(req, lens))
    assert (w.N, w.r_max) == (8, 16)


def test_multislice_8b_recipe():
    w = workloads.multislice_8b(seed=0, hidden=64, kv=16, inter=128)
    assert (w.T, w.N, w.r_max) == (1024, 100, 64)
    assert set(w.ranks.tolist()) <= {8, 16, 32, 64} and len(set(w.ranks.tolist())) == 4
    assert [len(l.d_out) for l in w.layers] == [3, 1, 2, 1]
    assert [l.d_out for l in w.layers] == [[64, 16, 16], [64], [128, 128], [64]]
    assert [l.d_in for l in w.layers] == [64, 64, 64, 128]
    assert (w.ids.numpy() >= 0).all()
    assert _zipf_fit_pvalue(w.ids.numpy(), 100, 1.1) > 1e-3
    for l in w.layers:
        assert l.col_off == list(np.cumsum([0] + l.d_out[:-1]))
        for a, b in zip(l.A, l.B):   # ranks beyond r_n are zero padding
            for n, r in enumerate(w.ranks.tolist()):
                assert not a[n, r:].any() and not b[n, :, r:].any()


def test_mixed_70b_recipe():
    w = workloads.mixed_70b(seed=0, hidden=64, inter=128)
    lens = np.array(w.info["lengths"])
    assert w.T == 8192 and len(lens) == 32
    assert lens.min() >= 64 and lens.max() <= 512
    assert w.info["prefill_tokens"] == int(lens.sum()) == 7892
    assert w.info["decode_rows"] == 8192 - 7892 == 300
    # the prompts come first, each one id throughout
    starts = np.concatenate([[0], np.cumsum(lens)])
    ids = w.ids.numpy()
    for a, b in zip(starts[:-1], starts[1:]):
        assert (ids[a:b] == ids[a]).all()
    units = np.concatenate([ids[starts[:-1]], ids[starts[-1]:]])
    assert 0.08 <= (units == -1).mean() <= 0.22         # 15 % of requests without an adapter
    assert [(l.d_in, l.d_out) for l in w.layers] == [(64, [128]), (128, [64])]
    assert (w.N, w.r_max) == (16, 16) and (w.ranks == 16).all()


def test_tiny_recipe():
    w = workloads.tiny(seed=0)
    assert (w.T, w.N, w.r_max, w.dtype) == (64, 4, 8, torch.float32)
    assert set(w.ids.tolist()) <= {-1, 0, 1, 2, 3}


def test_value_scales():
    """x and y0 ~ N(0, 1); adapter entries ~ N(0, 1/d_in) on live ranks."""
    w = workloads.decode_qproj(seed=0, d=1024)
    l = w.layers[0]
    assert abs(l.x.float().std().item() - 1.0) < 0.05
    assert abs(l.y0.float().std().item() - 1.0) < 0.05
    for t in l.A + l.B:
        assert abs(t.float().std().item() * 1024 ** 0.5 - 1.0) < 0.05
