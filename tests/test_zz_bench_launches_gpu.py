"""The kernel count per step that bench.py reports is the count the device sees:
one step of each shape, profiled with CUPTI, launches exactly that many kernels,
all of them this library's."""
import pytest

import bench
import workloads
from gpu_helpers import kernels_of

pytestmark = pytest.mark.gpu

SHAPES = {
    "decode_qproj": lambda: workloads.decode_qproj(seed=3),
    "multislice_8b": lambda: workloads.multislice_8b(seed=3, T=64),
    "prefill_one_block": lambda: workloads.prefill(seed=3, n_req=6, d=512),
    "mixed_70b_small": lambda: workloads.mixed_70b(seed=3, T=2048, n_req=4, hidden=512,
                                                   inter=1024),
    "mixed_70b_wide": lambda: workloads.mixed_70b(seed=3, T=2048, n_req=4, hidden=8192,
                                                  inter=8192),
    "mixed_70b_one_wide": lambda: workloads.mixed_70b(seed=3, T=2048, n_req=4, hidden=1024,
                                                      inter=8192),
    "multi_block_grouping": lambda: workloads.random_case(3, 3000, 1100, 256, [128], 16,
                                                          ranks=[16] * 1100),
}
OURS = ("seg_", "bgmv_kernel", "bgmv_tc_kernel", "sgmv_tc_kernel", "simt_", "lora_")


@pytest.mark.parametrize("shape", list(SHAPES))
def test_step_launch_count(cuda_lib, shape):
    w = SHAPES[shape]()
    ds = bench.DeviceSet(w, "cuda", *bench.segment_params(w))
    bench.step(ds)                              # first call: lazy host-side setup
    _, kernels, launches = kernels_of(lambda: bench.step(ds))
    assert int(ds.status.item()) == 0
    assert len(kernels) == launches == bench.launches_per_step(w), (kernels, launches)
    foreign = [k for k in kernels if not any(t in k for t in OURS)]
    assert not foreign, foreign
