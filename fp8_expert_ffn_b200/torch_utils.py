"""PyTorch plumbing for the library: device copies of a layer's weights,
workspace allocation and bf16 bit-pattern conversions. No layer arithmetic."""
from __future__ import annotations

import numpy as np
import torch

from . import LayerWeights, MoeLayer, moe_workspace_size


def to_device(a: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


def bf16_tensor(bits: np.ndarray, device="cuda") -> torch.Tensor:
    """uint16 bf16 bit patterns -> torch.bfloat16 tensor on `device`."""
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def upload_layer(host, device="cuda", routed_scaling=None, share_experts: MoeLayer = None) -> MoeLayer:
    """host: an object with shape (H, E, K, F, ld_f) and the numpy weight arrays
    router_w, w_gate, s_gate, w_up, s_up, w_down, s_down; optional router
    settings routed_scaling, n_group, topk_group, norm_topk and router_bias
    (numpy [E]) are read from it when present. With share_experts, the expert
    tensors of that layer are reused and only the router is copied."""
    sh = host.shape
    if share_experts is not None:
        src = share_experts.weights
        w = LayerWeights(w_gate=src.w_gate, w_up=src.w_up, w_down=src.w_down, s_gate=src.s_gate,
                         s_up=src.s_up, s_down=src.s_down, router_w=to_device(host.router_w, device))
    else:
        w = LayerWeights(
            w_gate=to_device(host.w_gate, device), w_up=to_device(host.w_up, device),
            w_down=to_device(host.w_down, device), s_gate=to_device(host.s_gate, device),
            s_up=to_device(host.s_up, device), s_down=to_device(host.s_down, device),
            router_w=to_device(host.router_w, device))
    if routed_scaling is None:
        routed_scaling = getattr(host, "routed_scaling", 1.0)
    bias = getattr(host, "router_bias", None)
    bias_dev = None if bias is None else to_device(np.asarray(bias, np.float32), device)
    return MoeLayer(sh.H, sh.E, sh.K, sh.F, w, ld_h=host.w_gate.shape[2], ld_f=host.w_down.shape[2],
                    routed_scaling=routed_scaling, n_shared=getattr(sh, "S", 1),
                    n_group=getattr(host, "n_group", 1), topk_group=getattr(host, "topk_group", 1),
                    norm_topk=getattr(host, "norm_topk", True), router_bias=bias_dev)


def workspace(layer: MoeLayer, T: int, device="cuda") -> torch.Tensor:
    n = moe_workspace_size(layer, T)
    if n == 0:
        raise ValueError("moe_workspace_size returned 0")
    return torch.empty(n, dtype=torch.uint8, device=device)
