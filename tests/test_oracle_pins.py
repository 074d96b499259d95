"""Pins of the fp64 oracle against what the pages and the mathematics fix.

None of these re-types the oracle's loops: each compares it with a different
statement of the same fact (a materialised low-rank product, a dense matmul of
a library, a bit-exact symmetry, a printed or hand-worked value).
"""
import json
import os

import numpy as np
import pytest
from hypothesis import given, settings
from hypothesis import strategies as st
import torch

import oracle
import workloads

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


def _f64(t):
    return t.to(torch.float64)


def _merged_reference(w, layer, rows=None):
    """y0 + (alpha/r_n) * (B_n A_n) x  with Delta W = B A materialised in fp64
    (the merged form of page 'LoRA service', section 1, used here only as an
    independent statement of the same sum)."""
    T = w.T
    rows = list(range(T)) if rows is None else list(rows)
    out = _f64(layer.y0[rows]).clone()
    for q, i in enumerate(rows):
        n = int(w.ids[i])
        if n < 0 or n >= w.N:
            continue
        r = int(w.ranks[n])
        s = w.alpha / r
        for sl in range(len(layer.A)):
            A = _f64(layer.A[sl][n, :r, :])           # [r, d_in]
            B = _f64(layer.B[sl][n, :, :r])           # [d_out, r]
            dW = B @ A                                 # [d_out, d_in]
            off, d = layer.col_off[sl], layer.d_out[sl]
            out[q, off:off + d] += s * (dW @ _f64(layer.x[i]))
    return out.numpy()


def _apply(w, layer, rows=None, ids=None):
    return oracle.lora_apply(layer.x, layer.A, layer.B, layer.col_off, w.ranks, w.alpha,
                             w.ids if ids is None else ids, layer.y0, rows=rows)


# ---------------------------------------------------------------- formulas

def test_param_count_matches_page_example():
    g = _gold("formulas.json")["param_count"]
    got = oracle.lora_param_count(g["d"], g["k"], g["r"])
    assert got == g["adapter_params"]
    assert g["d"] * g["k"] == g["full_params"]
    assert g["full_params"] // got == g["ratio"] and g["full_params"] % got == 0
    assert round(got / 1000) == 131                       # printed "131K"
    assert round(g["full_params"] / 1e5) / 10 == 16.8     # printed "16.8M"
    # page 1's ~122x is 16M / 131K with 4096^2 rounded down to 16M
    assert int(16e6 / got) == g["page1_printed_ratio"]


def test_adapter_memory_formula_matches_page_example():
    g = _gold("formulas.json")["adapter_bytes"]
    got = oracle.adapter_bytes(g["num_layers"], g["r"], g["hidden"], g["dtype_bytes"])
    assert got == g["formula_bytes"]
    # the page's printed product is the same product without the leading 2
    assert got == 2 * g["page_printed_product_bytes"]
    # "100 adapters ~ 2 GB" follows the printed 20 MB figure
    assert abs(100 * g["page_printed_product_bytes"] / 1e9 - 2.1) < 0.1


def test_rank_cost_is_linear_in_rank():
    g = _gold("formulas.json")["rank_cost"]
    lo = oracle.adapter_bytes(32, g["r_small"], 4096, 2)
    hi = oracle.adapter_bytes(32, g["r_large"], 4096, 2)
    assert hi == g["ratio"] * lo
    assert oracle.lora_param_count(4096, 4096, g["r_large"]) == \
        g["ratio"] * oracle.lora_param_count(4096, 4096, g["r_small"])


# ---------------------------------------------------------------- delta values

@pytest.mark.parametrize("seed,T,N,d_in,d_out,r_max", [
    (1, 3, 2, 4, 5, 2), (2, 7, 3, 9, 6, 3), (3, 16, 4, 33, [12, 7], 5)])
def test_equals_materialised_low_rank_product(seed, T, N, d_in, d_out, r_max):
    """B(Ax) = (BA)x (page 'Multi-LoRA Serving', section 3.1: Delta W x is computed
    as B(Ax) and never materialised): brute force on tiny shapes."""
    w = workloads.random_case(seed, T, N, d_in, d_out, r_max, none_frac=0.25,
                              dtype=torch.float32)
    lay = w.layers[0]
    got = _apply(w, lay)
    ref = _merged_reference(w, lay)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_tiny_workload_equals_materialised_product():
    w = workloads.tiny()
    lay = w.layers[0]
    np.testing.assert_allclose(_apply(w, lay), _merged_reference(w, lay), rtol=1e-12, atol=1e-12)


def test_bf16_inputs_widen_exactly():
    w = workloads.random_case(4, 9, 3, 24, 16, 4, dtype=torch.bfloat16)
    lay = w.layers[0]
    np.testing.assert_allclose(_apply(w, lay), _merged_reference(w, lay), rtol=1e-12, atol=1e-12)


def test_none_rows_keep_base_output_bit_exact():
    """id -1 means the base model only (page 'LoRA hot load ...', None = base model;
    page 'Multi-LoRA Serving', section 4: a None request gets the bare base)."""
    w = workloads.random_case(5, 40, 4, 32, 24, 4, none_frac=0.5, dtype=torch.bfloat16)
    lay = w.layers[0]
    got = _apply(w, lay)
    none = (w.ids == -1).numpy()
    assert none.any() and (~none).any()
    np.testing.assert_array_equal(got[none], _f64(lay.y0).numpy()[none])
    # rows with an adapter really change (the "output equals base" symptom)
    assert (np.abs(got[~none] - _f64(lay.y0).numpy()[~none]).max(axis=1) > 0).all()


def test_invalid_ids_are_treated_as_no_adapter():
    w = workloads.random_case(6, 12, 3, 16, 8, 2, none_frac=0.0, dtype=torch.float32)
    lay = w.layers[0]
    ids = w.ids.clone()
    ids[3], ids[7] = 3, -5
    got = _apply(w, lay, ids=ids)
    y0 = _f64(lay.y0).numpy()
    np.testing.assert_array_equal(got[[3, 7]], y0[[3, 7]])


def test_row_permutation_equivariance_bit_exact():
    """Each row is computed on its own (per-row formula, page 'Multi-LoRA Serving',
    section 2), so permuting rows and ids permutes the output bit for bit."""
    w = workloads.random_case(7, 50, 5, 40, 24, 6, dtype=torch.bfloat16)
    lay = w.layers[0]
    base = _apply(w, lay)
    g = torch.Generator().manual_seed(11)
    p = torch.randperm(w.T, generator=g)
    w2 = workloads.Workload(w.name, w.dtype, w.T, w.N, w.r_max, w.alpha, w.ids[p].clone(),
                            w.ranks, [workloads.Layer(lay.name, lay.d_in, lay.d_out, lay.col_off,
                                                      lay.x[p].contiguous(), lay.A, lay.B,
                                                      lay.y0[p].contiguous())])
    got = _apply(w2, w2.layers[0])
    np.testing.assert_array_equal(got, base[p.numpy()])


def test_single_adapter_equals_dense_low_rank_matmul():
    """All rows on one adapter = one dense low-rank product (page 'LoRA service',
    section 2: one adapter performs like plain batched matmuls):
    Y = Y0 + s (X A^T) B^T, computed by torch's fp64 matmul."""
    w = workloads.random_case(8, 37, 3, 64, 48, 8, ranks=[8, 8, 8], none_frac=0.0,
                              dtype=torch.bfloat16)
    lay = w.layers[0]
    k = 1
    ids = torch.full((w.T,), k, dtype=torch.int32)
    got = _apply(w, lay, ids=ids)
    X, A, B = _f64(lay.x), _f64(lay.A[0][k]), _f64(lay.B[0][k])
    ref = _f64(lay.y0) + (w.alpha / 8) * (X @ A.T) @ B.T
    np.testing.assert_allclose(got, ref.numpy(), rtol=1e-12, atol=1e-12)


def test_rank_padding_is_invisible_bit_exact():
    """Adapters stored in r_max slots (page 'Multi-LoRA Serving', 3.2: max-lora-rank
    sizes the slots) give the same result as unpadded storage; the scale uses the
    adapter's own rank, not the slot size."""
    w = workloads.random_case(9, 30, 4, 48, 40, 8, ranks=[2, 8, 5, 3], none_frac=0.1,
                              dtype=torch.float32)
    lay = w.layers[0]
    base = _apply(w, lay)
    pad = 64
    A = torch.zeros(w.N, pad, lay.d_in)
    B = torch.zeros(w.N, lay.d_out[0], pad)
    A[:, :8, :] = lay.A[0]
    B[:, :, :8] = lay.B[0]
    got = oracle.lora_apply(lay.x, [A], [B], lay.col_off, w.ranks, w.alpha, w.ids, lay.y0)
    np.testing.assert_array_equal(got, base)


def test_padding_contents_are_never_read():
    w = workloads.random_case(10, 20, 3, 32, 16, 8, ranks=[4, 8, 2], dtype=torch.float32)
    lay = w.layers[0]
    base = _apply(w, lay)
    A, B = lay.A[0].clone(), lay.B[0].clone()
    for n, r in enumerate(w.ranks.tolist()):
        A[n, r:, :] = 1e30
        B[n, :, r:] = -1e30
    got = oracle.lora_apply(lay.x, [A], [B], lay.col_off, w.ranks, w.alpha, w.ids, lay.y0)
    np.testing.assert_array_equal(got, base)


def test_multi_slice_equals_separate_slices():
    """A fused QKV-style layer (several output slices sharing x) equals applying
    each slice on its own and placing it at its column offset."""
    w = workloads.random_case(12, 25, 4, 32, [16, 8, 8], 4, dtype=torch.bfloat16)
    lay = w.layers[0]
    got = _apply(w, lay)
    for s in range(3):
        off, d = lay.col_off[s], lay.d_out[s]
        y0s = lay.y0[:, off:off + d].contiguous()
        one = oracle.lora_apply(lay.x, [lay.A[s]], [lay.B[s]], [0], w.ranks, w.alpha, w.ids, y0s)
        np.testing.assert_array_equal(got[:, off:off + d], one)


def test_routing_each_row_gets_its_own_adapter():
    """Rows of different adapters in one batch each match their own adapter's
    single-adapter result (page 'LoRA hot load ...', debugging: outputs that all
    look like one adapter mean broken routing)."""
    w = workloads.random_case(13, 24, 4, 32, 16, 4, ranks=[4, 4, 4, 4], none_frac=0.0,
                              dtype=torch.float32)
    lay = w.layers[0]
    got = _apply(w, lay)
    for i in range(w.T):
        n = int(w.ids[i])
        X = _f64(lay.x[i:i + 1])
        ref = _f64(lay.y0[i:i + 1]) + (w.alpha / 4) * (X @ _f64(lay.A[0][n]).T) @ _f64(lay.B[0][n]).T
        np.testing.assert_allclose(got[i:i + 1], ref.numpy(), rtol=1e-12, atol=1e-12)
        for m in range(w.N):
            if m != n:
                wrong = _f64(lay.y0[i:i + 1]) + (w.alpha / 4) * (X @ _f64(lay.A[0][m]).T) @ \
                    _f64(lay.B[0][m]).T
                assert np.abs(got[i:i + 1] - wrong.numpy()).max() > 1e-3


def test_row_subset_matches_full():
    w = workloads.random_case(14, 33, 4, 24, 16, 4, dtype=torch.bfloat16)
    lay = w.layers[0]
    full = _apply(w, lay)
    rows = [32, 0, 17, 5]
    np.testing.assert_array_equal(_apply(w, lay, rows=rows), full[rows])


# ---------------------------------------------------------------- grouping

def test_segments_hand_worked_example():
    g = _gold("segments_example.json")
    got = oracle.build_segments(g["ids"], g["N"], g["rows_per_tile"], g["min_run"], g["long_tile"])
    assert got["status"] == g["status"]
    np.testing.assert_array_equal(got["perm"], g["perm"])
    np.testing.assert_array_equal(got["seg_start"], g["seg_start"])
    np.testing.assert_array_equal(got["seg_adapter"], g["seg_adapter"])
    np.testing.assert_array_equal(got["contig_tiles"], np.array(g["contig_tiles"]).reshape(-1, 4))
    np.testing.assert_array_equal(got["grow"], g["grow"])
    np.testing.assert_array_equal(got["gather_tiles"], np.array(g["gather_tiles"]).reshape(-1, 4))


def _check_segments_against_library_sort(ids, N, R, min_run, LT):
    ids = np.asarray(ids, np.int32)
    T = ids.shape[0]
    got = oracle.build_segments(ids, N, R, min_run, LT)
    valid = (ids >= 0) & (ids < N)
    key = np.where(valid, ids, N)
    # numpy's stable argsort and Python's sorted() are two independent statements
    np.testing.assert_array_equal(got["perm"], np.argsort(key, kind="stable"))
    assert list(got["perm"]) == sorted(range(T), key=lambda i: (key[i], i))
    counts = np.bincount(ids[valid], minlength=N)
    np.testing.assert_array_equal(got["seg_start"], np.concatenate([[0], np.cumsum(counts)]))
    np.testing.assert_array_equal(got["seg_adapter"], np.nonzero(counts)[0])
    assert got["status"] == (0 if ((ids >= -1) & (ids < N)).all() else 1)

    # tiles cover every valid row exactly once, each tile on one adapter
    covered = np.zeros(T, np.int32)
    for n, row0, cnt, _ in got["contig_tiles"]:
        assert 0 < cnt <= LT
        rows = np.arange(row0, row0 + cnt)
        assert (ids[rows] == n).all()
        covered[rows] += 1
        # the run containing the tile is long
        lo = row0
        while lo > 0 and ids[lo - 1] == n:
            lo -= 1
        hi = row0 + cnt
        while hi < T and ids[hi] == n:
            hi += 1
        assert min_run > 0 and hi - lo >= min_run
    grow = got["grow"]
    prev = None
    for n, q0, cnt, _ in got["gather_tiles"]:
        assert 0 < cnt <= R
        rows = grow[q0:q0 + cnt]
        assert (ids[rows] == n).all()
        covered[rows] += 1
        if prev is not None:
            assert (prev[0], prev[1]) < (n, q0)
        prev = (n, q0)
    assert list(grow) == sorted(grow, key=lambda i: (ids[i], i))
    np.testing.assert_array_equal(covered, valid.astype(np.int32))
    # gathered rows are exactly the rows outside long runs (run lengths by brute force)
    run_lo, run_len = np.zeros(T, np.int64), np.zeros(T, np.int64)
    i = 0
    while i < T:
        j = i
        while j < T and ids[j] == ids[i]:
            j += 1
        run_lo[i:j], run_len[i:j] = i, j - i
        i = j
    long_row = valid & (run_len >= min_run) if min_run > 0 else np.zeros(T, bool)
    assert sorted(grow) == sorted(np.nonzero(valid & ~long_row)[0])
    # contiguous tiles: each long run cut every LT rows from its first row
    for n, row0, cnt, _ in got["contig_tiles"]:
        assert (row0 - run_lo[row0]) % LT == 0
        assert cnt == min(LT, run_lo[row0] + run_len[row0] - row0)
    if min_run == 0:
        assert len(got["contig_tiles"]) == 0
        np.testing.assert_array_equal(grow, got["perm"][:valid.sum()])
    # tile counts: every segment cut into full tiles plus one partial
    short_counts = np.bincount(ids[grow], minlength=N) if len(grow) else np.zeros(N, int)
    assert len(got["gather_tiles"]) == int(sum((c + R - 1) // R for c in short_counts))
    return got


@pytest.mark.parametrize("seed", range(6))
def test_segments_against_library_sort_random(seed):
    rng = np.random.default_rng(seed)
    T = int(rng.integers(1, 400))
    N = int(rng.integers(1, 12))
    ids = rng.integers(-1, N, size=T)
    if seed % 2:   # runs like prefill requests
        lens = rng.integers(1, 90, size=12)
        ids = np.repeat(rng.integers(-1, N, size=12), lens)
    _check_segments_against_library_sort(ids, N, int(rng.integers(1, 17)),
                                         int(rng.choice([0, 8, 32])), int(rng.choice([16, 128])))


@settings(max_examples=60, deadline=None)
@given(st.integers(1, 9).flatmap(lambda N: st.tuples(
           st.just(N),
           st.lists(st.tuples(st.integers(-1, N - 1), st.integers(1, 40)), min_size=0, max_size=12),
           st.integers(1, 16), st.sampled_from([0, 1, 5, 24]), st.sampled_from([4, 16, 128]))))
def test_segments_properties_hypothesis(case):
    """Random batches as runs of (id, length): the grouping's definition checked
    by brute force (stable order, offsets, every row once, long runs tiled)."""
    N, runs, R, min_run, LT = case
    ids = np.array([i for (i, L) in runs for _ in range(L)], np.int32)
    _check_segments_against_library_sort(ids, N, R, min_run, LT)


@pytest.mark.parametrize("ids,N", [
    ([], 3), ([-1, -1, -1], 2), ([1] * 50, 2), ([0], 1), ([-1] * 5 + [0] + [-1] * 5, 1),
    ([3, -1, -1, 3], 4)])
def test_segments_edge_cases(ids, N):
    _check_segments_against_library_sort(ids, N, 4, 8, 16)


def test_segments_workload_shapes():
    w = workloads.prefill(n_req=10, len_lo=20, len_hi=200, d=16)
    got = _check_segments_against_library_sort(w.ids.numpy(), w.N, 16, 64, 128)
    # every long prompt is tiled contiguously, so prompts >= 64 tokens leave no gathered rows
    lens = np.array(w.info["lengths"])
    rq = np.array(w.info["req_ids"])
    assert got["n_short"] <= int(lens[(lens < 64) & (rq >= 0)].sum())
    assert got["n_contig"] >= int(((lens >= 64) & (rq >= 0)).sum() > 0)


def test_shrink_equals_library_matmul():
    """v = A_n x_i (page 'Multi-LoRA Serving', section 3.4: add_shrink computes the
    rank-r v = A x) against torch's fp64 matmul, per adapter."""
    w = workloads.random_case(15, 29, 3, 40, [8, 8], 6, ranks=[6, 2, 4], none_frac=0.2,
                              dtype=torch.bfloat16)
    lay = w.layers[0]
    v = oracle.lora_shrink(lay.x, lay.A, w.ranks, w.ids)
    for i in range(w.T):
        n = int(w.ids[i])
        for s in range(2):
            if n < 0:
                assert (v[i, s] == 0).all()
                continue
            r = int(w.ranks[n])
            ref = (_f64(lay.A[s][n, :r]) @ _f64(lay.x[i])).numpy()
            np.testing.assert_allclose(v[i, s, :r], ref, rtol=1e-12, atol=1e-12)
            assert (v[i, s, r:] == 0).all()
