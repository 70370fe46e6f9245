"""The debug-checks build (libcausalattn_debug.so, compiled with CA_DEBUG_CHECKS): its kernels
check every TMA coordinate and every global index they compute on the device, and record a
failed check in the device status word instead of making the access.  A child process runs a
spread of shapes through it (ragged lengths, d = 32 / 64 / 128, document masks, a sliding
window, the FP8 forward, KV-cache decode, the RoPE + QK-norm prologue); no check may fail, no
wait may time out, and every output must be bit-identical to the release library's."""
import os
import subprocess
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from causal_self_attention_mha_b200 import abi, build, inputs  # noqa: E402

CASES_SRC = r'''
import torch
from causal_self_attention_mha_b200 import abi, inputs


def run_cases():
    dev = torch.device("cuda:0")
    out = {}
    for (B, H, T, d, doc, window, seed) in [(2, 3, 300, 128, False, None, 1),
                                            (1, 2, 257, 64, True, None, 2),
                                            (1, 4, 129, 32, False, None, 3),
                                            (2, 2, 1000, 128, True, None, 4),
                                            (2, 2, 700, 128, False, 200, 5),
                                            (1, 2, 1, 128, False, None, 6)]:
        q, k, v, do = (t.to(dev) for t in inputs.make_qkvdo(B, H, T, d, seed))
        ds = inputs.random_doc_start(B, T, seed, 16, 200).to(dev) if doc else None
        o, lse = abi.attention_forward(q, k, v, doc_offsets=ds, window=window)
        dq, dk, dv = abi.attention_backward(q, k, v, o, lse, do, doc_offsets=ds, window=window)
        out[f"attn{seed}"] = [o, lse, dq, dk, dv]
    q8, k8, v8 = (t.to(dev) for t in inputs.make_qkv_e4m3(1, 2, 300, 128, 7))
    s = inputs.FP8_DESCALE
    out["fp8"] = list(abi.attention_forward_fp8(q8, k8, v8, s, s, s))
    qd, kc, vc = (t.to(dev) for t in inputs.make_decode(2, 4, 3, 500, 128, 8))
    out["decode"] = list(abi.attention_decode(qd, kc, vc))
    xq, xk, _, _ = (t.to(dev) for t in inputs.make_prologue(2, 3, 300, 128, 9))
    out["prologue"] = list(abi.rope_qknorm(xq, xk))
    torch.cuda.synchronize()
    return out
'''


def _cases():
    ns = {}
    exec(compile(CASES_SRC, "debug_cases", "exec"), ns)
    return ns["run_cases"]


@pytest.mark.gpu
def test_debug_build_finds_no_bad_access_and_matches_release(tmp_path):
    lib = build.build(debug=True)
    script = tmp_path / "child.py"
    dump = tmp_path / "out.pt"
    script.write_text(
        f"import sys, torch\nsys.path.insert(0, {ROOT!r})\n" + CASES_SRC +
        "from causal_self_attention_mha_b200 import abi\n"
        "abi.gpt_attn_device_status(clear=True)\n"
        "out = run_cases()\n"
        "status = abi.gpt_attn_device_status(clear=True)\n"
        f"torch.save({{'out': {{k: [t.cpu() for t in v] for k, v in out.items()}}, "
        f"'status': status}}, {str(dump)!r})\n")
    env = dict(os.environ, CAUSALATTN_LIBRARY=lib)
    r = subprocess.run([sys.executable, str(script)], env=env, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    res = torch.load(str(dump))
    assert res["status"] == 0, f"device status word {res['status']:#x}"
    abi.gpt_attn_device_status(clear=True)
    ref = _cases()()
    assert abi.gpt_attn_device_status(clear=True) == 0
    assert set(ref) == set(res["out"])
    for name, tensors in ref.items():
        for i, (a, b) in enumerate(zip(tensors, res["out"][name])):
            assert torch.equal(a.cpu(), b), (name, i)
