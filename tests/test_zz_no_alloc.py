"""lora_build_segments_static: batch grouping that allocates nothing.

Callers that cannot allocate device memory when they group a batch (a memory
pool that owns the whole device, a hook or callback that must not call
cudaMalloc) use this entry point: its scratch is a fixed array inside the
library.  Its results must equal those of lora_build_segments, which takes
caller-provided scratch, call after call (the array keeps the previous call's
contents).  This file runs last so that a failure here never hides the rest.
"""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def _ids(rng, T, N):
    lens = rng.integers(1, 400, size=T // 100)
    ids = np.repeat(rng.integers(-1, N, size=lens.shape[0]), lens)[:T]
    tail = rng.integers(-1, N, size=max(0, T - ids.shape[0]))
    return np.concatenate([ids, tail]).astype(np.int32)


def _call_static(lib, ids_d, meta, status):
    return lib.lora_build_segments_static(ctypes.c_void_p(ids_d.data_ptr()), ctypes.byref(meta.c),
                                          ctypes.c_void_p(status.data_ptr()),
                                          ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_static_scratch_matches_caller_scratch_twice(cuda_lib):
    lora = cuda_lib
    lib = lora.load()
    rng = np.random.default_rng(2024)
    T, N = 20000, 100                     # beyond one block (> 8192 rows): the grouping needs scratch
    assert 0 < lora.lora_segments_scratch_bytes(T, N) <= (1 << 20)
    for call in range(2):
        ids_d = torch.as_tensor(_ids(rng, T, N)).cuda()
        ref = lora.Meta(T, N, 16, 64)
        st_ref = torch.zeros(1, dtype=torch.int32, device="cuda")
        lora.lora_build_segments(ids_d, ref, st_ref)
        got = lora.Meta(T, N, 16, 64)
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        assert _call_static(lib, ids_d, got, st) == 0
        torch.cuda.synchronize()
        a, b = ref.host(), got.host()
        for k in a:
            np.testing.assert_array_equal(np.asarray(a[k]), np.asarray(b[k]), err_msg=f"call {call}: {k}")
        assert int(st.item()) == int(st_ref.item()) == 0


def test_static_scratch_small_batch_and_limit(cuda_lib):
    lora = cuda_lib
    lib = lora.load()
    # one block, no scratch needed
    ids_d = torch.as_tensor(np.random.default_rng(5).integers(-1, 8, size=300).astype(np.int32)).cuda()
    ref, got = lora.Meta(300, 8, 16, 64), lora.Meta(300, 8, 16, 64)
    st = torch.zeros(2, dtype=torch.int32, device="cuda")
    lora.lora_build_segments(ids_d, ref, st[:1])
    assert _call_static(lib, ids_d, got, st[1:]) == 0
    torch.cuda.synchronize()
    for k, v in ref.host().items():
        np.testing.assert_array_equal(np.asarray(v), np.asarray(got.host()[k]))
    # beyond the fixed array: a clear error, nothing launched
    T, N = 131072, 4096
    assert lora.lora_segments_scratch_bytes(T, N) > (1 << 20)
    big = lora.Meta(T, N, 16, 0)
    ids_big = torch.zeros(T, dtype=torch.int32, device="cuda")
    assert _call_static(lib, ids_big, big, st[:1]) == -6          # LORA_ERR_WORKSPACE
    assert lib.lora_status_string(-6) == b"LORA_ERR_WORKSPACE"
