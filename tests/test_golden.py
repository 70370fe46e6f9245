"""Oracle regression fixtures (tests/golden/): the oracle, run on each fixture's stored
inputs, reproduces the stored outputs, and the seeded generators still produce the stored
inputs.  The fixtures were written by tests/golden/make_golden.py from the oracle itself, so
they guard against unintended change; correctness is pinned in test_oracle_pins.py."""
import glob
import importlib.util
import os

import numpy as np
import pytest

import oracle

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
_spec = importlib.util.spec_from_file_location("make_golden", os.path.join(HERE, "make_golden.py"))
make_golden = importlib.util.module_from_spec(_spec)
_spec.loader.exec_module(make_golden)

FILES = sorted(glob.glob(os.path.join(HERE, "*.txt")))


def test_every_case_has_a_fixture():
    assert {os.path.basename(f)[:-4] for f in FILES} == set(make_golden.CASES)


@pytest.mark.parametrize("path", FILES, ids=[os.path.basename(f)[:-4] for f in FILES])
def test_oracle_reproduces_fixture(path):
    name = os.path.basename(path)[:-4]
    ins, outs = make_golden.read(path)
    # the generators still give the stored inputs
    gen_ins, _ = make_golden.CASES[name][1]()
    for key, a in ins.items():
        np.testing.assert_array_equal(make_golden.to_array(gen_ins[key]), a)
    # the oracle on the stored inputs gives the stored outputs
    if name.startswith("decode"):
        o, lse = oracle.decode_forward(ins["q"], ins["k_cache"], ins["v_cache"], 0.5)
        got = dict(o=o, lse=lse)
    elif name.startswith("prologue"):
        got = dict(z=oracle.qk_prologue_forward(ins["x"]),
                   dx=oracle.qk_prologue_backward(ins["x"], ins["dz"]))
    else:
        doc = ins["doc"].astype(np.int32) if "doc" in ins else None
        window = 2 if name.startswith("window2") else None
        o, lse = oracle.attention_forward(ins["q"], ins["k"], ins["v"], 0.5, doc, window=window)
        dq, dk, dv = oracle.attention_backward(ins["q"], ins["k"], ins["v"], ins["do"], 0.5, doc,
                                               window=window)
        got = dict(o=o, lse=lse, dq=dq, dk=dk, dv=dv)
    assert set(got) == set(outs)
    for key in outs:
        np.testing.assert_allclose(got[key], outs[key], rtol=0, atol=1e-12, err_msg=key)
