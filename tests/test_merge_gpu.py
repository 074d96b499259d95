"""Merge / unmerge of one adapter into a base weight on the GPU against the fp64
oracle (page "LoRA service: multi-adapter dynamic loading", section 1):
W += sign * (alpha_n / r_n) * B_n A_n, W rounded once.  bf16 takes the tcgen05
kernel, fp32 the plain one.  Tolerance: |gpu - oracle| <= 1e-2 * max(1, |oracle|)
for bf16, 1e-4 for fp32."""
import pytest
import torch

import lora_adapter_application_b200 as lora
import oracle
from gpu_helpers import assert_within

pytestmark = pytest.mark.gpu


def _stacks(seed, N, d_out, d_in, r_max, ranks, dtype, pad=0.0):
    g = torch.Generator().manual_seed(seed)
    A = (torch.randn(N, r_max, d_in, generator=g) / d_in ** 0.5).to(dtype)
    B = (torch.randn(N, d_out, r_max, generator=g) / d_in ** 0.5).to(dtype)
    for n, r in enumerate(ranks):
        A[n, r:] = pad
        B[n, :, r:] = pad
    return A, B


@pytest.mark.parametrize("d_out,d_in,ld_extra,ranks,n", [
    (4096, 4096, 0, [64, 16, 8, 17], 0),     # Llama-3-8B q_proj shape, rank 64
    (4096, 4096, 0, [64, 16, 8, 17], 3),     # rank 17: K padded to 32, ranks 17..31 zeroed
    (1000, 520, 8, [8, 33], 1),              # ragged tiles, W rows wider than d_in
    (14336, 4096, 0, [16], 0),               # gate/up slice shape
])
@pytest.mark.parametrize("sign", [1, -1])
def test_merge_bf16_tensor_core(cuda_lib, d_out, d_in, ld_extra, ranks, n, sign):
    N = len(ranks)
    A, B = _stacks(7, N, d_out, d_in, 64, ranks, torch.bfloat16, pad=float("nan"))
    g = torch.Generator().manual_seed(8)
    W = torch.randn(d_out, d_in + ld_extra, generator=g).to(torch.bfloat16)
    alphas = torch.tensor([16.0, 32.0, 8.0, 24.0][:N], dtype=torch.float32)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    Wd = W.cuda()
    lora.lora_merge_adapter(Wd, A.cuda(), B.cuda(), n, torch.tensor(ranks, dtype=torch.int32).cuda(),
                            alphas.cuda(), status, sign=sign)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    A0, B0 = A[n].clone(), B[n].clone()
    A0[ranks[n]:] = 0
    B0[:, ranks[n]:] = 0
    ref = oracle.lora_merge(W, A0, B0, ranks[n], float(alphas[n]), sign)
    got = Wd.cpu()
    assert_within(got[:, :d_in].double().numpy(), ref, torch.bfloat16, "merge")
    if ld_extra:
        assert torch.equal(got[:, d_in:], W[:, d_in:])   # columns past d_in untouched


def test_merge_fp32_and_unmerge(cuda_lib):
    ranks = [12, 32]
    A, B = _stacks(9, 2, 300, 200, 32, ranks, torch.float32)
    W = torch.randn(300, 200, generator=torch.Generator().manual_seed(10))
    rk, al = torch.tensor(ranks, dtype=torch.int32).cuda(), torch.tensor([8.0, 4.0]).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    Wd = W.cuda()
    lora.lora_merge_adapter(Wd, A.cuda(), B.cuda(), 0, rk, al, status, sign=1)
    torch.cuda.synchronize()
    assert_within(Wd.cpu().double().numpy(), oracle.lora_merge(W, A[0], B[0], 12, 8.0, 1),
                  torch.float32, "fp32 merge")
    lora.lora_merge_adapter(Wd, A.cuda(), B.cuda(), 0, rk, al, status, sign=-1)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert_within(Wd.cpu().double().numpy(), W.double().numpy(), torch.float32, "unmerge")


def test_merge_bad_rank_leaves_w(cuda_lib):
    A, B = _stacks(11, 2, 256, 256, 16, [16, 16], torch.bfloat16)
    W = torch.randn(256, 256).to(torch.bfloat16)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    Wd = W.cuda()
    lora.lora_merge_adapter(Wd, A.cuda(), B.cuda(), 1, torch.tensor([16, 17], dtype=torch.int32).cuda(),
                            torch.ones(2).cuda(), status)
    torch.cuda.synchronize()
    assert int(status.item()) & lora.DEV_BAD_RANK
    assert torch.equal(Wd.cpu(), W)
