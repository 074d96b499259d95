"""Pins of the oracle's merged weight W + sign * (alpha/r) * B A (page "LoRA
service: multi-adapter dynamic loading", section 1, W' = W + B A; the scale
alpha/r of page "Multi-LoRA Serving", section 3.1), against things other than
itself: a library fp64 matmul, the per-row delta applied to the columns of an
identity matrix, merge then unmerge, and padding that is never read."""
import numpy as np
import pytest
import torch

import oracle


def _case(seed, d_out, d_in, r_max, r, dtype=torch.bfloat16, ld_extra=0):
    g = torch.Generator().manual_seed(seed)
    W = torch.randn(d_out, d_in + ld_extra, generator=g).to(dtype)
    A = (torch.randn(r_max, d_in, generator=g) / d_in ** 0.5).to(dtype)
    B = (torch.randn(d_out, r_max, generator=g) / d_in ** 0.5).to(dtype)
    A[r:] = 0
    B[:, r:] = 0
    return W, A, B


@pytest.mark.parametrize("d_out,d_in,r_max,r,ld_extra", [(48, 40, 16, 16, 0), (33, 72, 32, 5, 8),
                                                        (7, 9, 8, 1, 3)])
@pytest.mark.parametrize("sign", [1, -1])
def test_merge_equals_library_matmul(d_out, d_in, r_max, r, ld_extra, sign):
    W, A, B = _case(1, d_out, d_in, r_max, r, ld_extra=ld_extra)
    got = oracle.lora_merge(W, A, B, r, 24.0, sign)
    Wd, Ad, Bd = W.double()[:, :d_in], A.double(), B.double()
    want = Wd + sign * (24.0 / r) * (Bd[:, :r] @ Ad[:r, :])
    np.testing.assert_allclose(got, want.numpy(), rtol=1e-12, atol=1e-12)


def test_merge_equals_the_per_row_delta_on_identity_columns():
    """Column i of the merged weight is W[:, i] plus the delta of the input e_i:
    lora_apply on x = I (d_in rows), y0 = W^T, gives (W + s B A)^T."""
    d_out, d_in, r_max, r = 24, 40, 16, 11
    W, A, B = _case(2, d_out, d_in, r_max, r)
    merged = oracle.lora_merge(W, A, B, r, 16.0)
    x = torch.eye(d_in, dtype=torch.bfloat16)
    y0 = W.t().contiguous()
    ids = np.zeros(d_in, dtype=np.int32)
    per_row = oracle.lora_apply(x, [A[None]], [B[None]], [0], [r], 16.0, ids, y0)
    np.testing.assert_allclose(merged, per_row.T, rtol=1e-12, atol=1e-12)


def test_merge_then_unmerge_is_the_identity():
    W, A, B = _case(3, 40, 56, 32, 32, dtype=torch.float32)
    m = oracle.lora_merge(W, A, B, 32, 8.0, 1)
    back = oracle.lora_merge(torch.from_numpy(m).float(), A, B, 32, 8.0, -1)
    # the fp32 round trip of m is the only rounding
    np.testing.assert_allclose(back, W.double().numpy(), atol=1e-5)


def test_merge_never_reads_padding():
    W, A, B = _case(4, 20, 24, 16, 6)
    clean = oracle.lora_merge(W, A, B, 6, 4.0)
    A[6:] = float("nan")
    B[:, 6:] = float("nan")
    np.testing.assert_array_equal(oracle.lora_merge(W, A, B, 6, 4.0), clean)


def test_merge_rejects_bad_arguments():
    W, A, B = _case(5, 8, 8, 8, 4)
    for r, sign in [(0, 1), (9, 1), (4, 0)]:
        with pytest.raises(ValueError):
            oracle.lora_merge(W, A, B, r, 1.0, sign)
