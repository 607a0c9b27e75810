"""Synthetic-input recipe checks (no GPU): shapes, seeds, mask structure and
the sparsity each workload is meant to have."""

import numpy as np
import pytest
import torch

from sparse_attention_diffusion_rt_b200 import inputs

EXPECTED_SPARSITY = {            # 1 - kept / nkb
    "tiny": 0.75, "pixart": 1 - 2 / 32, "hunyuan": 1 - 3 / 34, "cogvideox": 1 - 4 / 139,
    "longvideo-25": 1 - 225 / 900, "longvideo-12.5": 1 - 113 / 900,
    "longvideo-6.25": 1 - 56 / 900, "longvideo-3.1": 1 - 28 / 900,
}


@pytest.mark.parametrize("name", list(inputs.WORKLOADS))
def test_mask_structure(name):
    w = inputs.WORKLOADS[name]
    m = inputs.block_mask(w)
    assert m.shape == (1, w.nqb, w.nkb) and m.dtype == np.uint8
    counts = m[0].sum(1)
    assert np.all(counts == w.kept)
    assert np.all(np.diag(m[0]) == 1)                       # a block always sees itself
    cent, has_text = inputs.block_centroids(w)
    assert np.all(m[0][:, has_text] == 1)                   # text key blocks always kept
    np.testing.assert_allclose(1 - m.mean(), EXPECTED_SPARSITY[name], atol=1e-12)


def test_mask_locality_pixart_band():
    m = inputs.block_mask(inputs.WORKLOADS["pixart"])[0]
    for qb in range(1, 32):
        assert set(np.nonzero(m[qb])[0]) == {qb - 1, qb}
    assert set(np.nonzero(m[0])[0]) == {0, 1}


def test_mask_text_first_cogvideox():
    w = inputs.WORKLOADS["cogvideox"]
    cent, has_text = inputs.block_centroids(w)
    assert list(np.nonzero(has_text)[0]) == [0, 1]          # 226 text tokens span blocks 0 and 1
    assert np.isnan(cent[0, 0]) and not np.isnan(cent[1, 0])
    assert w.nqb == 139 and w.L - 138 * 128 == 112          # ragged tail block


def test_seeded_inputs_reproducible_and_drift():
    w = inputs.Workload("t", 1, 2, 100, 16, 64, kept=1, n_sparse_steps=2, seed=7)
    a = inputs.qkv_steps(w, 3)
    b = inputs.qkv_steps(w, 3)
    for sa, sb in zip(a, b):
        for x, y in zip(sa, sb):
            assert x.dtype == torch.bfloat16 and x.shape == (1, 2, 100, 16)
            assert torch.equal(x, y)
    dq = (a[1][0].float() - a[0][0].float())
    assert 0.03 < dq.std().item() < 0.07                   # 0.05 N(0,1) drift, bf16-rounded
    assert abs(a[0][0].float().std().item() - 1.0) < 0.1


def test_head_range_draws_the_whole_problems_values():
    """A rank that owns heads h0..h1-1 draws exactly the whole problem's values
    there, at every step, without drawing the other heads."""
    w = inputs.Workload("t", 2, 5, 130, 16, 64, kept=1, n_sparse_steps=2, seed=3)
    whole = inputs.qkv_steps(w, 3)
    for h0, h1 in ((0, 2), (2, 5), (4, 5)):
        part = inputs.qkv_steps(w, 3, heads=(h0, h1))
        for sw, sp in zip(whole, part):
            for x, y in zip(sw, sp):
                assert y.shape == (2, h1 - h0, 130, 16)
                assert torch.equal(x[:, h0:h1], y)
    # distinct slabs are distinct draws
    q = whole[0][0].float()
    assert not torch.equal(q[0, 0], q[0, 1]) and not torch.equal(q[0, 0], q[1, 0])
    assert not torch.equal(whole[0][0], whole[0][1])
    import pytest
    with pytest.raises(ValueError):
        inputs.initial_qkv(w, heads=(3, 6))
