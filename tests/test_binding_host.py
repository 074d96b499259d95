"""The Python binding's operand checks, on the host: every shape, dtype or layout
disagreement that the library (which sees only pointers) would turn into an
out-of-bounds access is refused before anything reaches the device."""
import pytest
import torch

import lora_adapter_application_b200 as lora
from lora_adapter_application_b200 import LoraError

T, N, D_IN, R = 8, 3, 64, 16
D_OUT = [32, 16]


def _ops(dtype=torch.bfloat16):
    A = [torch.zeros(N, R, D_IN, dtype=dtype) for _ in D_OUT]
    B = [torch.zeros(N, d, R, dtype=dtype) for d in D_OUT]
    x = torch.zeros(T, D_IN, dtype=dtype)
    y = torch.zeros(T, sum(D_OUT), dtype=dtype)
    ranks = torch.full((N,), R, dtype=torch.int32)
    alphas = torch.ones(N, dtype=torch.float32)
    meta = lora.Meta(T, N, 16, 0, device="cpu")
    return dict(y=y, x=x, A=A, B=B, col_off=[0, 32], ranks=ranks, alphas=alphas, meta=meta,
                status=torch.zeros(1, dtype=torch.int32))


def _call(**over):
    o = _ops()
    o.update(over)
    return lora.lora_add_linear(o["y"], o["x"], o["A"], o["B"], o["col_off"], o["ranks"],
                                o["alphas"], o["meta"], o["status"])


def test_well_formed_operands_reach_the_device_check():
    with pytest.raises(LoraError, match="CUDA tensor"):
        _call()


@pytest.mark.parametrize("case,match", [
    (lambda o: {"A": [o["A"][0], torch.zeros(N, 8, D_IN, dtype=torch.bfloat16)]}, "every A slice"),
    (lambda o: {"B": [o["B"][0], torch.zeros(N, 16, 8, dtype=torch.bfloat16)]}, "every B slice"),
    (lambda o: {"A": [a[:2].contiguous() for a in o["A"]],
                "B": [b[:2].contiguous() for b in o["B"]]}, "slots"),
    (lambda o: {"x": o["x"][:T - 1]}, "at least T rows"),
    (lambda o: {"x": o["x"][:, :D_IN - 8]}, "d_in columns"),
    (lambda o: {"y": o["y"][:T - 1]}, "at least T rows"),
    (lambda o: {"col_off": [0, 40]}, "run past y"),
    (lambda o: {"col_off": [0]}, "one column offset"),
    (lambda o: {"ranks": o["ranks"].long()}, "ranks"),
    (lambda o: {"alphas": o["alphas"][:N - 1]}, "alphas"),
    (lambda o: {"x": o["x"].float()}, "one dtype"),
    (lambda o: {"B": o["B"][:1]}, "one A and one B"),
    (lambda o: {"A": [a.transpose(1, 2) for a in o["A"]]}, "contiguous 3-D"),
])
def test_mismatched_operands_are_refused(case, match):
    o = _ops()
    with pytest.raises(LoraError, match=match):
        _call(**case(o))


def test_expand_and_shrink_check_v():
    o = _ops()
    v_small = torch.zeros(2, T, R - 1)
    with pytest.raises(LoraError, match="v must be"):
        lora.lora_sgmv_expand(o["y"], v_small, o["B"], o["col_off"], o["ranks"], o["alphas"],
                              o["meta"], o["status"])
    with pytest.raises(LoraError, match="v must be"):
        lora.lora_sgmv_shrink(torch.zeros(2, T, R, dtype=torch.float64), o["x"], o["A"],
                              o["ranks"], o["meta"], o["status"])
    with pytest.raises(LoraError, match="CUDA tensor"):
        lora.lora_sgmv_shrink(torch.zeros(2, T, R), o["x"], o["A"], o["ranks"], o["meta"],
                              o["status"])
