"""The seeded input recipe: deterministic, bf16, and the document layout follows its rule."""
import torch

from causal_self_attention_mha_b200 import inputs


def test_qkvdo_deterministic_and_bf16():
    a = inputs.make_qkvdo(1, 2, 5, 8, 3)
    b = inputs.make_qkvdo(1, 2, 5, 8, 3)
    for x, y in zip(a, b):
        assert x.dtype == torch.bfloat16 and x.shape == (1, 2, 5, 8)
        assert torch.equal(x, y)
    assert not torch.equal(a[0], a[1])


def test_doc_lengths_rule():
    for B, T, seed in ((4, 2048, 4), (3, 1000, 11), (2, 50, 1)):
        rows = inputs.doc_lengths(B, T, seed)
        assert len(rows) == B
        for lens in rows:
            assert sum(lens) == T
            assert all(inputs.DOC_MIN_LEN <= n <= inputs.DOC_MAX_LEN for n in lens[:-1])
            assert 1 <= lens[-1] <= inputs.DOC_MAX_LEN


def test_doc_start_format():
    ds = inputs.doc_start_from_lengths([[3, 2], [5]], 5)
    assert ds.tolist() == [[0, 0, 0, 3, 3], [0, 0, 0, 0, 0]]


def test_packed_workload_pair_count():
    """Visible pairs of the packed workload = H * sum over documents of L(L+1)/2."""
    w = inputs.WORKLOADS["doc_packed"]
    rows = inputs.doc_lengths(w.B, w.T, w.seed)
    expect = w.H * sum(n * (n + 1) // 2 for lens in rows for n in lens)
    ds = inputs.doc_start_from_lengths(rows, w.T)
    assert inputs.visible_pairs(w.B, w.H, w.T, ds) == expect
    assert inputs.visible_pairs(1, 1, 64) == 64 * 65 // 2
