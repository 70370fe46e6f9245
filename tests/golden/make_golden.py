"""Writes the oracle regression fixtures in this folder.

The pages print no worked numeric example of the attention step, so nothing here is a value
from the pages: every fixture is the oracle's output on a tiny seeded bf16 input, written by
this script, which calls only `oracle/` and the seeded input generators.  The fixtures pin the
oracle against accidental change (a later edit of its arithmetic must reproduce them or name,
in its commit message, the passage that justifies the new values); its correctness is pinned
separately by closed forms, invariants, finite differences and independent library routines.

Run from the repository root:  python tests/golden/make_golden.py
"""
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from causal_self_attention_mha_b200 import inputs  # noqa: E402

# name -> (citation, builder); each builder returns (inputs dict, outputs dict) of arrays
CASES = {}


def case(name, citation):
    def wrap(fn):
        CASES[name] = (citation, fn)
        return fn
    return wrap


@case("causal_T5_d4", "Stanford CS336 walkthrough (lmnt.cn), section 5.1 model.py "
      "CausalSelfAttention.forward; backward by the chain rule (section 5.2 loss.backward)")
def _causal():
    q, k, v, do = inputs.make_qkvdo(1, 1, 5, 4, 101)
    o, lse = oracle.attention_forward(q, k, v, 0.5)
    dq, dk, dv = oracle.attention_backward(q, k, v, do, 0.5)
    return dict(q=q, k=k, v=v, do=do), dict(o=o, lse=lse, dq=dq, dk=dk, dv=dv)


@case("documents_T6_d4", "How to build an LLM by hand (agmtopy.github.io), section 5.5: "
      "BOS-aligned packing, documents starting at positions 0 and 3")
def _docs():
    q, k, v, do = inputs.make_qkvdo(1, 1, 6, 4, 102)
    doc = inputs.doc_start_from_lengths([[3, 3]], 6)
    o, lse = oracle.attention_forward(q, k, v, 0.5, doc)
    dq, dk, dv = oracle.attention_backward(q, k, v, do, 0.5, doc)
    return dict(q=q, k=k, v=v, do=do, doc=doc), dict(o=o, lse=lse, dq=dq, dk=dk, dv=dv)


@case("window2_T6_d4", "How to build an LLM by hand (agmtopy.github.io), section 9: "
      "sliding-window attention, window of 2 keys")
def _window():
    q, k, v, do = inputs.make_qkvdo(1, 1, 6, 4, 103)
    o, lse = oracle.attention_forward(q, k, v, 0.5, window=2)
    dq, dk, dv = oracle.attention_backward(q, k, v, do, 0.5, window=2)
    return dict(q=q, k=k, v=v, do=do), dict(o=o, lse=lse, dq=dq, dk=dk, dv=dv)


@case("decode_Tq2_L5_d4", "How to build an LLM by hand (agmtopy.github.io), section 2: "
      "KV-cache decode, two new tokens over a cache of five positions")
def _decode():
    q, kc, vc = inputs.make_decode(1, 1, 2, 5, 4, 104)
    o, lse = oracle.decode_forward(q, kc, vc, 0.5)
    return dict(q=q, k_cache=kc, v_cache=vc), dict(o=o, lse=lse)


@case("prologue_T4_d8", "How to build an LLM by hand (agmtopy.github.io), section 9: "
      "RoPE then QK Norm (x1.2), base 10000, eps 1e-6")
def _prologue():
    x, _, dz, _ = inputs.make_prologue(1, 1, 4, 8, 105)
    return dict(x=x, dz=dz), dict(z=oracle.qk_prologue_forward(x),
                                  dx=oracle.qk_prologue_backward(x, dz))


def to_array(t):
    if hasattr(t, "detach"):
        import torch
        return t.detach().to(torch.float64).numpy()
    return np.asarray(t, dtype=np.float64)


def write(name, citation, ins, outs):
    with open(os.path.join(HERE, f"{name}.txt"), "w") as f:
        f.write(f"# {name}\n# source: {citation}\n")
        f.write("# written by tests/golden/make_golden.py from the oracle (regression fixture)\n")
        for kind, arrs in (("in", ins), ("out", outs)):
            for key, a in arrs.items():
                a = to_array(a)
                f.write(f"{kind} {key} {' '.join(str(s) for s in a.shape)}\n")
                f.write(" ".join(repr(float(x)) for x in a.ravel()) + "\n")


def read(path):
    """-> (inputs dict, outputs dict) of float64 arrays."""
    ins, outs = {}, {}
    with open(path) as f:
        lines = [l.rstrip("\n") for l in f if not l.startswith("#")]
    for head, body in zip(lines[0::2], lines[1::2]):
        kind, key, *shape = head.split()
        a = np.array([float(x) for x in body.split()], dtype=np.float64).reshape(
            [int(s) for s in shape])
        (ins if kind == "in" else outs)[key] = a
    return ins, outs


if __name__ == "__main__":
    for name, (citation, fn) in CASES.items():
        write(name, citation, *fn())
        print("wrote", name)
