"""gpt_attn_bwd_static_ws: the backward entry point for callers that cannot
allocate device memory (code under a framework allocator that owns the whole
device, in a plugin host that only lends out its own tensors, or in a loop
where allocation is forbidden).  Its delta scratch is a fixed array inside the
library instead of a caller buffer.  Checked here against gpt_attn_bwd, through the C ABI, on two
calls in a row (the second call finds the first call's scratch contents).

This file sorts last so that a run stopping at its first failure has already
run every other test."""
import numpy as np
import pytest
import torch

from causal_self_attention_mha_b200 import abi, inputs

pytestmark = pytest.mark.gpu

GRAD_TOL = 2e-2


def rel_l2(a, b):
    a, b = a.double().cpu().numpy(), b.double().cpu().numpy()
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-3 * np.sqrt(b.size)))


@pytest.mark.parametrize("name", ["gpt2_small", "doc_packed"])
def test_static_workspace_backward_matches(name, cuda_device):
    w = inputs.WORKLOADS[name]
    q, k, v, do, doc = (t.to(cuda_device) if t is not None else None for t in inputs.make_workload(w))
    o, lse = abi.attention_forward(q, k, v, w.scale, doc)
    ref = abi.attention_backward(q, k, v, o, lse, do, w.scale, doc)
    for call in range(2):
        got = [torch.full_like(q, float("nan")) for _ in range(3)]
        torch.cuda.synchronize()
        allocs0 = torch.cuda.memory_stats().get("allocation.all.allocated", 0)
        free0 = torch.cuda.mem_get_info()[0]
        abi.gpt_attn_bwd_static_ws(q, k, v, o, do, lse, *got, w.scale, doc)
        torch.cuda.synchronize()
        if call == 1:
            # the first library call on a device may load the library's device code (and with it
            # the scratch array); from then on a call allocates nothing, through torch or not
            assert torch.cuda.memory_stats().get("allocation.all.allocated", 0) == allocs0
            assert torch.cuda.mem_get_info()[0] == free0
        for g, r in zip(got, ref):
            assert torch.isfinite(g).all()
            assert rel_l2(g, r) <= GRAD_TOL
            assert torch.equal(g, r)  # same kernels, same inputs: bit-identical
    assert abi.gpt_attn_device_status(clear=True) == 0


def test_static_workspace_rejects_oversize(cuda_device):
    B, H, T, d = 1, 1, (1 << 20) + 1, 32
    q = torch.zeros(B, H, T, d, dtype=torch.bfloat16, device=cuda_device)
    lse = torch.zeros(B, H, T, device=cuda_device)
    with pytest.raises(abi.AttnError) as e:
        abi.gpt_attn_bwd_static_ws(q, q, q, q, q, lse, q, q, q, 0.1)
    assert e.value.status == abi.GPT_ATTN_ERR_TOO_LARGE
