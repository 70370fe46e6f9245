"""bench.py's timed region on the GPU: the per-kernel durations come from CUDA events inside
it (sampled steps only, never the first), and they add up to the step time."""
import os
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from causal_self_attention_mha_b200 import abi, inputs  # noqa: E402


@pytest.mark.gpu
def test_timed_steps_per_kernel_durations_add_up_to_the_step():
    dev = torch.device("cuda:0")
    B, H, T, d = 2, 4, 1024, 64
    q, k, v, do = (t.to(dev) for t in inputs.make_qkvdo(B, H, T, d, 3))
    scale = inputs.fp32_scale(d)
    o = torch.empty_like(q)
    lse = torch.empty(B, H, T, device=dev, dtype=torch.float32)
    delta = torch.empty_like(lse)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    stream = torch.cuda.Stream(dev)
    launches = []

    def step(ev=None):
        calls = (lambda: abi.gpt_attn_fwd(q, k, v, o, lse, scale, None, stream),
                 lambda: abi.gpt_attn_bwd_dq_delta(q, k, v, o, do, lse, delta, dq, scale, None, stream),
                 lambda: abi.gpt_attn_bwd_dkdv(q, k, v, do, lse, delta, dk, dv, scale, None, stream))
        for j, c in enumerate(calls):
            if ev is not None:
                ev[j].record(stream)
            c()
        if ev is not None:
            ev[len(calls)].record(stream)
        launches.append(ev is not None)

    with torch.cuda.stream(stream):
        for _ in range(3):
            step()
        torch.cuda.synchronize(dev)
        launches.clear()
        steps = 40
        elapsed, per = bench.timed_steps(step, stream, steps, 3, dev)
    assert len(launches) == steps and not launches[0]
    assert sum(launches) == len(bench.sampled_indices(steps))
    assert all(x > 0 for x in per)
    ratio, _ = bench.kernel_sum_check(per, elapsed / steps)
    assert 0.9 < ratio < 1.1
    # too short to sample: the durations come from a profile phase after the region
    launches.clear()
    with torch.cuda.stream(stream):
        elapsed2, per2 = bench.timed_steps(step, stream, 2, 3, dev)
    assert launches[:2] == [False, False] and len(launches) == 2 + bench.PROFILE_STEPS
    assert all(x > 0 for x in per2)
    assert abi.gpt_attn_device_status(clear=True) == 0
