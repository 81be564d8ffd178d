"""The padded row layout of the layers above the gate (CPU only).

The pruned forward can run on a fixed, padded row count so that one captured CUDA
graph serves calls with different kept totals ("TokenGate: Adapting LLMs for Fast and
Memory-Efficient Prefill with Learned Token Pruning" (paper digest), sections
方法关键点 and 工作参考价值).  The layout puts the padding rows at the end of the last
request.  These tests check the host rule, and check on the oracle that trailing
padding rows change no kept row: a kept row's keys never include a padding row,
because attention is causal within a request.
"""
import numpy as np
import pytest
import torch

import oracle as O
import synthetic_inputs as S


@pytest.fixture(scope="module")
def tg():
    import learned_token_pruning_scoring_b200 as m
    return m


def test_padded_layout_rules(tg):
    assert tg.padded_layout([0, 5, 9]).tolist() == [0, 5, 9]
    assert tg.padded_layout([0, 5, 9], 9).tolist() == [0, 5, 9]
    assert tg.padded_layout([0, 5, 9], 16).tolist() == [0, 5, 16]
    assert tg.padded_layout([0, 700], 1024).tolist() == [0, 1024]
    assert tg.padded_layout([0, 0], 256).tolist() == [0, 256]
    with pytest.raises(ValueError):
        tg.padded_layout([0, 5, 9], 8)
    with pytest.raises(ValueError):
        tg.padded_layout([0], 8)
    assert [tg.k_bucket(k) for k in (0, 1, 255, 256, 257, 1638, 13107)] == \
        [256, 256, 256, 256, 512, 1792, 13312]
    assert tg.k_bucket(1638, 128) == 1664
    with pytest.raises(ValueError):
        tg.k_bucket(10, 0)


def _kept_inputs(wl, seed):
    """Kept rows, positions and bias of a seeded selection (any valid one will do)."""
    rng = np.random.default_rng(seed)
    h = O.as_f64(S.hidden_rows(wl))
    cu = wl.cu_seqlens()
    idx, pos, ck = [], [], [0]
    for b, k in enumerate(wl.budgets):
        lo, hi = int(cu[b]), int(cu[b + 1])
        keep = np.sort(rng.choice(hi - lo, size=k, replace=False))
        idx += (keep + lo).tolist()
        pos += keep.tolist()
        ck.append(ck[-1] + k)
    bias = rng.standard_normal(len(idx))
    return h[np.array(idx)], np.array(pos), bias, np.array(ck)


@pytest.mark.parametrize("lengths,budgets,k_pad", [([600], [150], 256),
                                                   ([500, 400], [120, 90], 384)])
def test_trailing_padding_changes_no_kept_row(lengths, budgets, k_pad):
    """One gated layer of the oracle on the kept rows, and on the same rows followed by
    padding rows (row 0 of the input at position 0 with zero bias, as the pipeline
    fills them) appended to the last request: the kept rows' outputs and KV-cache rows
    agree to the last bits of float64."""
    wl = S.custom(lengths, [8] * len(lengths), budgets, n_layers=1, name="pad")
    L = S.layer_weights(wl, 0)
    x, pos, bias, ck = _kept_inputs(wl, 7)
    K = int(ck[-1])
    args = (L["Wqkv"], L["Wo"], L["gamma"], L["beta"])
    shape = (wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.rope_theta)
    x1, k1, v1, _ = O.gated_layer(x, *args, ck, pos, bias, *shape)

    n_pad = k_pad - K
    h0 = O.as_f64(S.hidden_rows(wl))[0]
    xp = np.concatenate([x, np.repeat(h0[None], n_pad, 0)])
    posp = np.concatenate([pos, np.zeros(n_pad, dtype=pos.dtype)])
    biasp = np.concatenate([bias, np.zeros(n_pad)])
    ckp = ck.copy()
    ckp[-1] = k_pad
    xp1, kp1, vp1, _ = O.gated_layer(xp, *args, ckp, posp, biasp, *shape)
    assert xp1.shape[0] == k_pad
    for got, want in ((xp1[:K], x1), (kp1[:K], k1), (vp1[:K], v1)):
        np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)
    # the rule the pipeline uses for the layout
    import learned_token_pruning_scoring_b200 as tg
    assert tg.padded_layout(torch.from_numpy(ck.astype(np.int32)), k_pad).tolist() == \
        ckp.tolist()
