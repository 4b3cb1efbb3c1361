"""The Python binding rejects host tensors and wrong dtypes before any pointer
reaches the library: a clear exception, never a call with a host address.
Runs without a GPU (the library is loaded, no kernel is launched)."""
import pytest
import torch

import expert_combine_b200 as eb

T, H, E, K = 4, 64, 16, 4
BF16, F32, I32, U8 = torch.bfloat16, torch.float32, torch.int32, torch.uint8


def _host_calls():
    """Each public call with host tensors of the right dtypes."""
    return {
        "moe_route": lambda: eb.moe_route(torch.zeros(T, E), torch.zeros(E), torch.ones(T, dtype=U8), K),
        "norm_quant_nvfp4": lambda: eb.norm_quant_nvfp4(torch.zeros(T, H, dtype=BF16), T, torch.zeros(H, dtype=BF16),
                                                        0.0, 1e-6, torch.ones(1)),
        "moe_route_norm_quant": lambda: eb.moe_route_norm_quant(torch.zeros(T, E), torch.zeros(E),
                                                                torch.ones(T, dtype=U8), K,
                                                                torch.zeros(T, H, dtype=BF16),
                                                                torch.zeros(H, dtype=BF16), 0.0, 1e-6, torch.ones(1)),
        "expert_combine": lambda: eb.expert_combine(torch.zeros(8, H, dtype=BF16), 8, torch.zeros(T, K, dtype=I32),
                                                    torch.zeros(T, K), torch.zeros(H, dtype=BF16), 0.0, 1e-6),
        "expert_combine_join": lambda: eb.expert_combine_join(
            torch.zeros(8, H, dtype=BF16), 8, torch.zeros(T, K, dtype=I32), torch.zeros(T, K),
            torch.zeros(H, dtype=BF16), 0.0, 1e-6, torch.zeros(T, H), torch.zeros(H, dtype=BF16), 1.0, 1.0, 1e-6),
        "residual_join": lambda: eb.residual_join(torch.zeros(T, H), torch.zeros(T, H, dtype=BF16),
                                                  torch.zeros(H, dtype=BF16), 1.0, 1.0, 1e-6),
        "moe_dispatch": lambda: eb.moe_dispatch(torch.zeros(T, K, dtype=I32), E),
        "moe_dispatch_noalloc": lambda: eb.moe_dispatch_noalloc(torch.zeros(T, K, dtype=I32), E),
        "router_weight_prepare": lambda: eb.router_weight_prepare(torch.zeros(E, H)),
        "router_logits": lambda: eb.router_logits(torch.zeros(T, H, dtype=BF16), torch.zeros(3, E, H, dtype=BF16)),
    }


@pytest.mark.parametrize("name", sorted(_host_calls()))
def test_host_tensors_are_rejected(name):
    with pytest.raises(ValueError, match="CUDA tensor"):
        _host_calls()[name]()


@pytest.mark.parametrize("call", [
    lambda: eb.moe_route(torch.zeros(T, E, dtype=torch.float64), torch.zeros(E), torch.ones(T, dtype=U8), K),
    lambda: eb.norm_quant_nvfp4(torch.zeros(T, H, dtype=F32), T, torch.zeros(H, dtype=BF16), 0.0, 1e-6,
                                torch.ones(1)),
    lambda: eb.expert_combine(torch.zeros(8, H, dtype=torch.float16), 8, torch.zeros(T, K, dtype=I32),
                              torch.zeros(T, K), torch.zeros(H, dtype=BF16), 0.0, 1e-6),
    lambda: eb.moe_dispatch(torch.zeros(T, K, dtype=torch.int64), E),
    lambda: eb.router_logits(torch.zeros(T, H, dtype=F32), torch.zeros(3, E, H, dtype=BF16)),
], ids=["route-logits-f64", "norm-quant-x-f32", "combine-rows-f16", "dispatch-ids-i64", "router-logits-x-f32"])
def test_wrong_dtypes_are_rejected(call):
    with pytest.raises(TypeError, match="expected"):
        call()
