"""Pins of the CPU oracle against things other than itself (no GPU needed).

Each test checks an oracle function against a hand-derived closed form, brute force
on tiny inputs, a library routine for a special case, or an invariant the
mathematics fixes.  The cases are chosen so that a dropped term, a wrong sign,
a wrong index or a transposed operand in the oracle fails at least one of them.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ------------------------------------------------------------------ closed form

def test_closed_form_normalisation_and_selection():
    g = _golden("closed_form_4tok.json")
    inp, exp = g["inputs"], g["expected"]
    s = np.array(inp["s"])
    pr = np.array(inp["prunable"])
    cu = np.array([0, 4])
    z, bias = O.sequence_rmsnorm(s, cu, pr, inp["eps_seq"])
    c = exp["c"]
    np.testing.assert_allclose(z, s * c, rtol=0, atol=1e-15)
    np.testing.assert_allclose(bias, np.array([1.0, -1.0, 1.4, 0.0]) * c, atol=1e-15)
    cu_kept = O.kept_counts(pr, cu, [inp["budget"]])
    assert list(cu_kept) == [0, 3]
    idx, pos, kb = O.select_topk(z.astype(np.float32), pr, cu, cu_kept)
    assert list(pos) == exp["kept_pos"] and list(idx) == exp["kept_pos"]
    np.testing.assert_allclose(kb, np.array(exp["kept_bias_over_c"]) * c, rtol=1e-7)


def test_closed_form_temperature():
    g = _golden("closed_form_4tok.json")
    tau = O.temperature([0, 1, 2], g["expected"]["kept_pos"], g["inputs"]["beta"])
    np.testing.assert_allclose(tau, g["expected"]["tau"], rtol=0, atol=1e-15)


def _closed_form_attention(gamma, beta):
    g = _golden("closed_form_4tok.json")
    inp, exp = g["inputs"], g["expected"]
    c = exp["c"]
    Q = np.array(inp["q_by_rank"], dtype=np.float64)[:, None, :]
    K = np.array(inp["k_by_rank"], dtype=np.float64)[:, None, :]
    V = np.array(inp["v_by_rank"], dtype=np.float64)[:, None, :]
    bias = np.array(exp["kept_bias_over_c"]) * c
    out, lse = O.gated_attention(Q, K, V, [0, 3], exp["kept_pos"], bias, [gamma], beta)
    return out[:, 0, :3], lse, exp


def test_closed_form_attention_weights():
    out, _, exp = _closed_form_attention(1.0, 1.0)
    np.testing.assert_allclose(out, np.array(exp["weights"]), rtol=0, atol=1e-14)


def test_closed_form_plain_causal():
    out, _, exp = _closed_form_attention(0.0, 1.0)
    # gamma = 0 removes the bias but tau still scales rank 2 by ln3/ln4
    assert not np.allclose(out[2], exp["weights_rank2_gamma0_beta1"], atol=1e-6)
    # with every position equal to its rank, tau = beta = 1: plain causal softmax
    g = _golden("closed_form_4tok.json")
    inp = g["inputs"]
    Q = np.array(inp["q_by_rank"], dtype=np.float64)[:, None, :]
    K = np.array(inp["k_by_rank"], dtype=np.float64)[:, None, :]
    V = np.array(inp["v_by_rank"], dtype=np.float64)[:, None, :]
    o2, _ = O.gated_attention(Q, K, V, [0, 3], [0, 1, 2], np.zeros(3), [0.0], 1.0)
    np.testing.assert_allclose(o2[2, 0, :3], exp["weights_rank2_gamma0_beta1"], atol=1e-14)


# ------------------------------------------------------------------ selection brute force

def _brute_topk(z32, prunable, kd):
    """Enumerate every kd-subset of prunable tokens; exactly one beats every dropped token."""
    cand = [i for i in range(len(z32)) if prunable[i]]

    def better(i, j):  # token i strictly ahead of token j
        zi, zj = float(z32[i]), float(z32[j])
        if math.isnan(zi) or math.isnan(zj):
            if math.isnan(zi) and math.isnan(zj):
                return i < j
            return math.isnan(zj)
        if zi != zj:
            return zi > zj
        return i < j

    winners = []
    for sub in itertools.combinations(cand, kd):
        rest = [j for j in cand if j not in sub]
        if all(better(i, j) for i in sub for j in rest):
            winners.append(sub)
    assert len(winners) == 1
    kept = sorted(set(winners[0]) | {i for i in range(len(z32)) if not prunable[i]})
    return kept


@pytest.mark.parametrize("seed", range(40))
def test_selection_brute_force(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(1, 11))
    z = rng.normal(size=n).astype(np.float32)
    if seed % 3 == 0:  # heavy ties
        z = np.round(z * 2.0).astype(np.float32) / np.float32(2.0)
    if seed % 5 == 0 and n > 2:
        z[0] = np.float32(-0.0)
        z[1] = np.float32(0.0)
    if seed % 7 == 0 and n > 3:
        z[2] = np.float32(np.nan)
        z[3] = np.float32(-np.inf)
    pr = (rng.random(n) < 0.7).astype(np.uint8)
    d = int(pr.sum())
    q = n - d
    budget = int(rng.integers(0, n + 2))
    cu_kept = O.kept_counts(pr, [0, n], [budget])
    kd = int(cu_kept[1]) - q
    assert kd == min(d, max(0, budget - q))
    idx, pos, kb = O.select_topk(z, pr, [0, n], cu_kept)
    assert list(pos) == _brute_topk(z, pr, kd)
    for i, p in enumerate(pos):
        want = z[p] if pr[p] else np.float32(0.0)
        assert (np.isnan(want) and np.isnan(kb[i])) or kb[i] == want


def test_selection_packed_requests_and_offsets():
    z = np.array([0.5, 0.1, 0.9, -1.0, 3.0, 2.0, 2.0, 1.0, 0.0], dtype=np.float32)
    pr = np.array([1, 1, 1, 0, 1, 1, 1, 1, 0], dtype=np.uint8)
    cu = [0, 4, 9]
    cu_kept = O.kept_counts(pr, cu, [2, 3])
    assert list(cu_kept) == [0, 2, 5]
    idx, pos, kb = O.select_topk(z, pr, cu, cu_kept)
    # request 0: question token 3 plus best doc token 2
    # request 1: question token 8 plus tokens 0 (3.0) and 1 (2.0, lower index of the tie)
    assert list(idx) == [2, 3, 4, 5, 8]
    assert list(pos) == [2, 3, 0, 1, 4]
    np.testing.assert_array_equal(kb, np.array([0.9, 0.0, 3.0, 2.0, 0.0], dtype=np.float32))


def test_kept_counts_rules():
    pr = np.array([1] * 6 + [0] * 2, dtype=np.uint8)
    cu = [0, 8]
    assert list(O.kept_counts(pr, cu, [0])) == [0, 2]      # budget below question size
    assert list(O.kept_counts(pr, cu, [5])) == [0, 5]
    assert list(O.kept_counts(pr, cu, [100])) == [0, 8]    # budget above request size


def test_selection_scale_invariance():
    rng = np.random.default_rng(3)
    s = rng.normal(size=200)
    pr = (rng.random(200) < 0.8).astype(np.uint8)
    cu = [0, 200]
    ck = O.kept_counts(pr, cu, [60])
    z1, _ = O.sequence_rmsnorm(s, cu, pr, 0.0)
    z2, _ = O.sequence_rmsnorm(s * 7.5, cu, pr, 0.0)
    np.testing.assert_allclose(z1, z2, rtol=1e-13)
    a = O.select_topk(z1.astype(np.float32), pr, cu, ck)[0]
    b = O.select_topk(z2.astype(np.float32), pr, cu, ck)[0]
    assert np.array_equal(a, b)
    # every question token kept, kept positions strictly increasing
    idx, pos, _ = O.select_topk(z1.astype(np.float32), pr, cu, ck)
    assert set(np.nonzero(pr == 0)[0]) <= set(idx.tolist())
    assert np.all(np.diff(pos) > 0) and len(idx) == ck[1]


def test_sequence_rmsnorm_per_request():
    s = np.array([3.0, 4.0, 1.0, 1.0, 1.0])
    z, _ = O.sequence_rmsnorm(s, [0, 2, 5], np.ones(5), 0.0)
    np.testing.assert_allclose(z, [3 / math.sqrt(12.5), 4 / math.sqrt(12.5), 1, 1, 1])


# ------------------------------------------------------------------ scorer

def test_gate_score_against_library_special_case():
    """W1 selecting input channels turns the scorer into sum_f w2_f SiLU(RMSNorm(h)[perm_f])."""
    H, Fw, T = 12, 5, 7
    g = torch.Generator().manual_seed(11)
    h = torch.randn((T, H), generator=g, dtype=torch.float64) * 3.0
    norm_w = torch.rand((H,), generator=g, dtype=torch.float64) + 0.5
    perm = [7, 0, 11, 3, 3]
    W1 = torch.zeros((Fw, H), dtype=torch.float64)
    for f, j in enumerate(perm):
        W1[f, j] = 1.0
    w2 = torch.tensor([0.5, -1.25, 2.0, 0.75, -0.3], dtype=torch.float64)
    want = F.silu(F.rms_norm(h, (H,), weight=norm_w, eps=1e-6))[:, perm] @ w2
    got = O.gate_score(h, norm_w, W1, w2, 1e-6)
    np.testing.assert_allclose(got, want.numpy(), rtol=1e-13, atol=1e-13)


def test_gate_score_row_scale_invariance_and_general_mlp():
    rng = np.random.default_rng(5)
    H, Fw = 16, 6
    h = rng.normal(size=(9, H))
    W1 = rng.normal(size=(Fw, H))
    w2 = rng.normal(size=Fw)
    s1 = O.gate_score(h, None, W1, w2, 0.0)
    s2 = O.gate_score(h * 13.0, None, W1, w2, 0.0)
    np.testing.assert_allclose(s1, s2, rtol=1e-12)
    # general weights against torch's Linear + SiLU + RMSNorm stack
    ht = torch.tensor(h)
    want = F.linear(F.silu(F.linear(F.rms_norm(ht, (H,), eps=1e-6), torch.tensor(W1))),
                    torch.tensor(w2)[None, :])[:, 0]
    np.testing.assert_allclose(O.gate_score(h, None, W1, w2, 1e-6), want.numpy(), rtol=1e-12)


# ------------------------------------------------------------------ RoPE

def test_rope_matches_complex_rotation():
    rng = np.random.default_rng(9)
    d, theta = 16, 1.0e6
    x = rng.normal(size=(5, 3, d))
    pos = np.array([0, 1, 17, 4095, 131071])
    got = O.rope(x, pos, theta)
    half = d // 2
    zc = x[..., :half] + 1j * x[..., half:]
    freq = theta ** (-np.arange(half) * 2.0 / d)
    rot = zc * np.exp(1j * pos[:, None, None] * freq[None, None, :])
    want = np.concatenate([rot.real, rot.imag], axis=-1)
    np.testing.assert_allclose(got, want, atol=1e-12)
    np.testing.assert_allclose(got[0], x[0], atol=0)       # position 0 is the identity


def test_rope_relative_position():
    rng = np.random.default_rng(10)
    d = 32
    q = rng.normal(size=(1, 1, d))
    k = rng.normal(size=(1, 1, d))
    a = np.sum(O.rope(q, [100], 1e4) * O.rope(k, [60], 1e4))
    b = np.sum(O.rope(q, [1040], 1e4) * O.rope(k, [1000], 1e4))
    c = np.sum(O.rope(q, [60], 1e4) * O.rope(k, [100], 1e4))
    assert abs(a - b) < 1e-10 and abs(a - c) > 1e-3


# ------------------------------------------------------------------ attention

def _attn_loops(Q, K, V, cu, pos, bias, gamma, beta):
    """Explicit per-(request, head, query, key) loops; tiny sizes only."""
    Kt, Hq, d = Q.shape
    grp = Hq // K.shape[1]
    out = np.zeros_like(Q)
    for b in range(len(cu) - 1):
        for h in range(Hq):
            for r in range(cu[b + 1] - cu[b]):
                p = pos[cu[b] + r]
                tau = beta if p == 0 else beta * math.log(r + 1) / math.log(p + 1)
                ls = []
                for c in range(r + 1):
                    dot = sum(Q[cu[b] + r, h, i] * K[cu[b] + c, h // grp, i] for i in range(d))
                    ls.append(tau * dot / math.sqrt(d) + gamma[h] * bias[cu[b] + c])
                m = max(ls)
                w = [math.exp(x - m) for x in ls]
                tot = sum(w)
                for c in range(r + 1):
                    out[cu[b] + r, h] += w[c] / tot * V[cu[b] + c, h // grp]
    return out


def _rand_attn_case(seed, lens, Hq=4, Hkv=2, d=8):
    rng = np.random.default_rng(seed)
    cu = np.concatenate([[0], np.cumsum(lens)])
    Kt = int(cu[-1])
    Q = rng.normal(size=(Kt, Hq, d))
    K = rng.normal(size=(Kt, Hkv, d))
    V = rng.normal(size=(Kt, Hkv, d))
    pos = np.concatenate([np.sort(rng.choice(4 * n + 3, size=n, replace=False)) for n in lens])
    bias = rng.normal(size=Kt) * (rng.random(Kt) < 0.8)
    gamma = rng.uniform(0.5, 2.0, size=Hq)
    return Q, K, V, cu, pos, bias, gamma


@pytest.mark.parametrize("seed", range(4))
def test_attention_brute_force_loops(seed):
    Q, K, V, cu, pos, bias, gamma = _rand_attn_case(seed, [5, 1, 7])
    beta = 0.8 + 0.1 * seed
    got, _ = O.gated_attention(Q, K, V, cu, pos, bias, gamma, beta, block=3)
    want = _attn_loops(Q, K, V, cu, pos, bias, gamma, beta)
    np.testing.assert_allclose(got, want, atol=1e-12)


def test_attention_reduces_to_library_causal_gqa():
    """K = N, gamma = 0, positions = ranks (tau = 1): plain causal GQA attention."""
    Q, K, V, cu, _, bias, gamma = _rand_attn_case(21, [33], Hq=8, Hkv=2, d=16)
    pos = np.arange(33)
    got, lse = O.gated_attention(Q, K, V, cu, pos, bias, np.zeros(8), 1.0)
    q = torch.tensor(Q).permute(1, 0, 2)[None]
    k = torch.tensor(K).permute(1, 0, 2).repeat_interleave(4, dim=0)[None]
    v = torch.tensor(V).permute(1, 0, 2).repeat_interleave(4, dim=0)[None]
    want = F.scaled_dot_product_attention(q, k, v, is_causal=True)[0].permute(1, 0, 2)
    np.testing.assert_allclose(got, want.numpy(), atol=1e-12)
    # LSE against logsumexp of the causal logits
    s = torch.einsum("hqd,hkd->hqk", q[0], k[0]) / 4.0
    s = s.masked_fill(torch.triu(torch.ones(33, 33, dtype=torch.bool), 1), float("-inf"))
    np.testing.assert_allclose(lse, torch.logsumexp(s, -1).numpy(), atol=1e-12)


def test_attention_invariants():
    Q, K, V, cu, pos, bias, gamma = _rand_attn_case(4, [40, 9])
    ones = np.ones_like(V)
    o1, _ = O.gated_attention(Q, K, ones, cu, pos, bias, gamma, 1.0)
    np.testing.assert_allclose(o1, 1.0, atol=1e-13)                   # rows sum to 1
    o, _ = O.gated_attention(Q, K, V, cu, pos, bias, gamma, 1.0)
    for b in range(2):
        for h in range(4):
            np.testing.assert_allclose(o[cu[b], h], V[cu[b], h // 2], atol=1e-14)  # rank 0
    # a bias constant over a request (all keys prunable) cancels in the softmax
    const = np.full_like(bias, 0.7)
    oa, _ = O.gated_attention(Q, K, V, cu, pos, const, gamma, 1.0)
    ob, _ = O.gated_attention(Q, K, V, cu, pos, const, np.zeros(4), 1.0)
    np.testing.assert_allclose(oa, ob, atol=1e-13)
    # but a non-constant bias with gamma > 0 does matter, and in the sign's direction
    hi = np.zeros_like(bias)
    hi[cu[0] + 3] = 5.0
    oc, _ = O.gated_attention(Q, K, ones * np.arange(1, 1 + V.shape[0])[:, None, None],
                              cu, pos, hi, gamma, 1.0)
    od, _ = O.gated_attention(Q, K, ones * np.arange(1, 1 + V.shape[0])[:, None, None],
                              cu, pos, -hi, gamma, 1.0)
    r = cu[0] + 10
    assert abs(oc[r, 0, 0] - 4.0) < abs(od[r, 0, 0] - 4.0)


def test_attention_kv_head_mapping():
    """q head h must read kv head h // (Hq/Hkv): zero all but one kv head's values."""
    Q, K, V, cu, pos, bias, gamma = _rand_attn_case(8, [12], Hq=4, Hkv=2)
    V2 = np.zeros_like(V)
    V2[:, 1] = 1.0
    o, _ = O.gated_attention(Q, K, V2, cu, pos, bias, gamma, 1.0)
    np.testing.assert_allclose(o[:, :2], 0.0, atol=0)
    np.testing.assert_allclose(o[:, 2:], 1.0, atol=1e-13)


def test_attention_sampled_rows_match_full():
    Q, K, V, cu, pos, bias, gamma = _rand_attn_case(13, [30, 25])
    full, lf = O.gated_attention(Q, K, V, cu, pos, bias, gamma, 1.1)
    rows = [0, 7, 29, 30, 54]
    part, lp = O.gated_attention(Q, K, V, cu, pos, bias, gamma, 1.1, rows=rows, block=2)
    np.testing.assert_allclose(part[rows], full[rows], atol=1e-13)
    np.testing.assert_allclose(lp[:, rows], lf[:, rows], atol=1e-13)
    assert np.isnan(part[1]).all()


# ------------------------------------------------------------------ layer / pipeline

def test_layer_zero_output_projection_keeps_residual():
    rng = np.random.default_rng(2)
    Hq, Hkv, d, H = 2, 1, 8, 16
    x = rng.normal(size=(6, H))
    Wqkv = rng.normal(size=((Hq + 2 * Hkv) * d, H)) * 0.3
    Wo = np.zeros((H, Hq * d))
    pos = np.array([0, 3, 4, 8, 9, 11])
    x2, k, v, parts = O.gated_layer(x, Wqkv, Wo, [1.0, 1.5], 1.0, [0, 6], pos,
                                    np.zeros(6), Hq, Hkv, d, 1e4)
    np.testing.assert_allclose(x2, x, atol=0)
    a = x / np.sqrt(np.mean(x * x, 1, keepdims=True) + 1e-6)
    kk = (a @ Wqkv.T)[:, Hq * d:(Hq + Hkv) * d].reshape(6, Hkv, d)
    np.testing.assert_allclose(k, O.rope(kk, pos, 1e4), atol=1e-12)
    vv = (a @ Wqkv.T)[:, (Hq + Hkv) * d:].reshape(6, Hkv, d)
    np.testing.assert_allclose(v, vv, atol=1e-12)


def test_layer_output_projection_against_torch():
    """x + Wo . O with H != Hq d and a non-zero Wo: with gamma = 0, beta = 1 and positions
    equal to ranks the layer is a plain pre-norm causal GQA layer, written here with
    torch's rms_norm, linear and scaled_dot_product_attention (heads concatenated in head
    order before Wo, the usual layout).  A transposed or wrongly reshaped O, or Wo used
    transposed, fails this."""
    import torch
    import torch.nn.functional as F
    rng = np.random.default_rng(7)
    Hq, Hkv, d, H, T = 2, 1, 12, 16, 9
    x = rng.normal(size=(T, H))
    Wqkv = rng.normal(size=((Hq + 2 * Hkv) * d, H)) * 0.3
    Wo = rng.normal(size=(H, Hq * d)) * 0.3
    pos = np.arange(T)
    x2, _, _, _ = O.gated_layer(x, Wqkv, Wo, np.zeros(Hq), 1.0, [0, T], pos, np.zeros(T),
                                Hq, Hkv, d, 1e4)
    xt = torch.from_numpy(x)
    qkv = F.linear(F.rms_norm(xt, (H,), eps=1e-6), torch.from_numpy(Wqkv))
    q = torch.from_numpy(O.rope(qkv[:, :Hq * d].reshape(T, Hq, d).numpy(), pos, 1e4))
    k = torch.from_numpy(O.rope(qkv[:, Hq * d:(Hq + Hkv) * d].reshape(T, Hkv, d).numpy(),
                                pos, 1e4))
    v = qkv[:, (Hq + Hkv) * d:].reshape(T, Hkv, d)
    heads = lambda t, rep: t.permute(1, 0, 2).repeat_interleave(rep, 0)[None]
    o = F.scaled_dot_product_attention(heads(q, 1), heads(k, Hq // Hkv), heads(v, Hq // Hkv),
                                       is_causal=True)[0]
    want = xt + F.linear(o.permute(1, 0, 2).reshape(T, Hq * d), torch.from_numpy(Wo))
    np.testing.assert_allclose(x2, want.numpy(), atol=1e-10)


def test_prefill_tiny_pipeline_consistency():
    import synthetic_inputs as S
    wl = S.custom([40, 24], [4, 6], [10, 12], n_layers=1, hidden=32, scorer_width=8,
                  n_q_heads=4, n_kv_heads=2, head_dim=8)
    h = S.hidden_rows(wl)
    gate = S.gate_weights(wl)
    layer = S.layer_weights(wl, 0)
    pr = S.prunable_mask(wl)
    out = O.prefill(h, pr, wl.cu_seqlens(), wl.budgets, gate, [layer], 4, 2, 8)
    assert list(out["cu_kept"]) == [0, 10, 22]
    assert len(out["kept_idx"]) == 22
    # question tokens (last Q_b of each request) are all kept
    for b, (lo, n, q) in enumerate(zip(wl.cu_seqlens()[:-1], wl.lengths, wl.questions)):
        kept_b = set(out["kept_idx"][out["cu_kept"][b]:out["cu_kept"][b + 1]].tolist())
        assert set(range(lo + n - q, lo + n)) <= kept_b
    assert out["x"].shape == (22, 32)


# ------------------------------------------------------------------ layers below the gate

def test_request_positions_restart_per_request():
    np.testing.assert_array_equal(O.request_positions([0, 3, 3, 5]), [0, 1, 2, 0, 1])
    assert O.request_positions([0]).size == 0


def test_causal_attention_against_library_per_request():
    """Ordinary causal GQA attention of each request against torch's SDPA (float64)."""
    Q, K, V, cu, _, _, _ = _rand_attn_case(31, [17, 1, 9], Hq=8, Hkv=2, d=16)
    got = O.causal_attention(Q, K, V, cu, block=5)
    for b in range(3):
        lo, hi = cu[b], cu[b + 1]
        q = torch.tensor(Q[lo:hi]).permute(1, 0, 2)[None]
        k = torch.tensor(K[lo:hi]).permute(1, 0, 2).repeat_interleave(4, dim=0)[None]
        v = torch.tensor(V[lo:hi]).permute(1, 0, 2).repeat_interleave(4, dim=0)[None]
        want = F.scaled_dot_product_attention(q, k, v, is_causal=True)[0].permute(1, 0, 2)
        np.testing.assert_allclose(got[lo:hi], want.numpy(), atol=1e-12)


def test_causal_attention_brute_force_and_gated_special_case():
    """Explicit loops with gamma = 0, tau = 1 (positions = ranks), and the gated
    oracle with every token kept, gamma = 0 and beta = 1: all three agree."""
    Q, K, V, cu, _, bias, _ = _rand_attn_case(5, [6, 4])
    pos = O.request_positions(cu)
    want = _attn_loops(Q, K, V, cu, pos, bias, np.zeros(4), 1.0)
    got = O.causal_attention(Q, K, V, cu, block=4)
    np.testing.assert_allclose(got, want, atol=1e-12)
    gated, _ = O.gated_attention(Q, K, V, cu, pos, bias, np.zeros(4), 1.0)
    np.testing.assert_allclose(got, gated, atol=1e-12)


def _lower_case(seed, lens, Hq=4, Hkv=2, d=8, H=32):
    rng = np.random.default_rng(seed)
    cu = np.concatenate([[0], np.cumsum(lens)])
    x = rng.normal(size=(int(cu[-1]), H))
    Wqkv = rng.normal(size=((Hq + 2 * Hkv) * d, H)) * 0.2
    Wo = rng.normal(size=(H, Hq * d)) * 0.2
    return x, Wqkv, Wo, cu


def test_full_context_layer_requests_are_independent():
    """Packing requests side by side must not change any of them: positions restart
    at 0 and attention stays inside the request (a packed-index position or a
    cross-request key would break this)."""
    x, Wqkv, Wo, cu = _lower_case(3, [11, 7])
    xo, k, v = O.full_context_layer(x, Wqkv, Wo, cu, 4, 2, 8, 1e4)
    for b in range(2):
        lo, hi = cu[b], cu[b + 1]
        xb, kb, vb = O.full_context_layer(x[lo:hi], Wqkv, Wo, [0, hi - lo], 4, 2, 8, 1e4)
        np.testing.assert_allclose(xo[lo:hi], xb, atol=1e-12)
        np.testing.assert_allclose(k[lo:hi], kb, atol=1e-12)
        np.testing.assert_allclose(v[lo:hi], vb, atol=1e-12)


def test_full_context_layer_is_the_gated_layer_with_nothing_pruned():
    x, Wqkv, Wo, cu = _lower_case(4, [9, 5])
    pos = O.request_positions(cu)
    xo, k, v = O.full_context_layer(x, Wqkv, Wo, cu, 4, 2, 8, 1e4)
    xg, kg, vg, _ = O.gated_layer(x, Wqkv, Wo, np.zeros(4), 1.0, cu, pos,
                                  np.ones(len(pos)), 4, 2, 8, 1e4)
    np.testing.assert_allclose(xo, xg, atol=1e-12)
    np.testing.assert_allclose(k, kg, atol=1e-12)
    np.testing.assert_allclose(v, vg, atol=1e-12)
    # zero output projection: the residual passes unchanged, K carries RoPE at the
    # in-request positions
    x0, k0, _ = O.full_context_layer(x, Wqkv, np.zeros_like(Wo), cu, 4, 2, 8, 1e4)
    np.testing.assert_allclose(x0, x, atol=0)
    a = x / np.sqrt(np.mean(x * x, 1, keepdims=True) + 1e-6)
    kk = (a @ Wqkv.T)[:, 32:48].reshape(-1, 2, 8)
    np.testing.assert_allclose(k0, O.rope(kk, pos, 1e4), atol=1e-12)


def test_prefill_with_lower_layers_composes_and_trims():
    """The gate reads the lower layers' output; trimmed lower caches are exactly the
    kept rows of the full-length ones."""
    import synthetic_inputs as S
    wl = S.custom([40, 24], [4, 6], [10, 12], n_layers=1, hidden=32, scorer_width=8,
                  n_q_heads=4, n_kv_heads=2, head_dim=8)
    h = S.hidden_rows(wl)
    gate = S.gate_weights(wl)
    upper = [S.layer_weights(wl, 0)]
    lower = S.lower_layer_weights(wl, 2)
    pr = S.prunable_mask(wl)
    cu = wl.cu_seqlens()
    out = O.prefill(h, pr, cu, wl.budgets, gate, upper, 4, 2, 8, lower_layers=lower)
    hg = O.as_f64(h)
    for L in lower:
        hg, _, _ = O.full_context_layer(hg, L["Wqkv"], L["Wo"], cu, 4, 2, 8)
    np.testing.assert_allclose(out["h_gate"], hg, atol=1e-12)
    direct = O.prefill(hg, pr, cu, wl.budgets, gate, upper, 4, 2, 8)
    np.testing.assert_array_equal(out["kept_idx"], direct["kept_idx"])
    np.testing.assert_allclose(out["x"], direct["x"], atol=1e-12)
    assert len(out["lower_caches"]) == 2
    for (kf, vf), (kt, vt) in zip(out["lower_caches_full"], out["lower_caches"]):
        assert kf.shape[0] == wl.total_tokens and kt.shape[0] == len(out["kept_idx"])
        np.testing.assert_array_equal(kt, kf[out["kept_idx"]])
        np.testing.assert_array_equal(vt, vf[out["kept_idx"]])


# ------------------------------------------------------------------ full layer body

def test_rmsnorm_heads_against_library():
    rng = np.random.default_rng(40)
    x = rng.normal(size=(5, 3, 16)) * 2.0
    w = rng.uniform(0.8, 1.2, size=16)
    want = F.rms_norm(torch.tensor(x), (16,), torch.tensor(w), eps=1e-6).numpy()
    np.testing.assert_allclose(O.rmsnorm_heads(x, w), want, atol=1e-12)


def test_swiglu_mlp_against_library():
    rng = np.random.default_rng(41)
    H, Fw = 24, 40
    x = rng.normal(size=(7, H))
    nw = rng.uniform(0.8, 1.2, size=H)
    Wg, Wu, Wd = (rng.normal(size=s) * 0.3 for s in ((Fw, H), (Fw, H), (H, Fw)))
    xt = torch.tensor(x)
    b = F.rms_norm(xt, (H,), torch.tensor(nw), eps=1e-6)
    want = xt + F.linear(F.silu(F.linear(b, torch.tensor(Wg))) * F.linear(b, torch.tensor(Wu)),
                         torch.tensor(Wd))
    np.testing.assert_allclose(O.swiglu_mlp(x, nw, Wg, Wu, Wd), want.numpy(), atol=1e-12)
    np.testing.assert_allclose(O.swiglu_mlp(x, nw, Wg, Wu, np.zeros_like(Wd)), x, atol=0)


def _body_case(seed, Hq=4, Hkv=2, d=8, H=32, Fw=48, n=11):
    rng = np.random.default_rng(seed)
    x = rng.normal(size=(n, H))
    Wqkv = rng.normal(size=((Hq + 2 * Hkv) * d, H)) * 0.2
    Wo = rng.normal(size=(H, Hq * d)) * 0.2
    parts = {"attn_norm": rng.uniform(0.8, 1.2, H), "q_norm": rng.uniform(0.8, 1.2, d),
             "k_norm": rng.uniform(0.8, 1.2, d),
             "mlp": {"norm_w": rng.uniform(0.8, 1.2, H),
                     "W_gate": rng.normal(size=(Fw, H)) * 0.2,
                     "W_up": rng.normal(size=(Fw, H)) * 0.2,
                     "W_down": rng.normal(size=(H, Fw)) * 0.2}}
    pos = np.sort(rng.choice(4 * n, size=n, replace=False))
    bias = rng.normal(size=n)
    gamma = rng.uniform(0.5, 2.0, Hq)
    return x, Wqkv, Wo, parts, pos, bias, gamma


def test_full_layer_cache_is_qk_normed_before_rope():
    """K cache = RoPE(RMSNorm_head(W_k RMSNorm(x; attn_norm); k_norm)), built here from
    torch's rms_norm and linear (RoPE itself is pinned above)."""
    x, Wqkv, Wo, parts, pos, bias, gamma = _body_case(42)
    _, k, v, _ = O.gated_layer(x, Wqkv, Wo, gamma, 1.0, [0, 11], pos, bias, 4, 2, 8, 1e4,
                               **parts)
    a = F.rms_norm(torch.tensor(x), (32,), torch.tensor(parts["attn_norm"]), eps=1e-6)
    kk = F.linear(a, torch.tensor(Wqkv[32:48])).view(11, 2, 8)
    kn = F.rms_norm(kk, (8,), torch.tensor(parts["k_norm"]), eps=1e-6).numpy()
    np.testing.assert_allclose(k, O.rope(kn, pos, 1e4), atol=1e-12)
    vv = F.linear(a, torch.tensor(Wqkv[48:])).view(11, 2, 8).numpy()
    np.testing.assert_allclose(v, vv, atol=1e-12)


def test_qk_norm_removes_the_scale_of_q_and_k():
    """With QK-norm, scaling W_q and W_k by 3 changes nothing (eps aside); without it the
    logits scale by 9 and the output moves."""
    x, Wqkv, Wo, parts, pos, bias, gamma = _body_case(43)
    W2 = Wqkv.copy()
    W2[:48] *= 3.0
    a1, *_ = O.gated_layer(x, Wqkv, Wo, gamma, 1.0, [0, 11], pos, bias, 4, 2, 8, 1e4, **parts)
    a2, *_ = O.gated_layer(x, W2, Wo, gamma, 1.0, [0, 11], pos, bias, 4, 2, 8, 1e4, **parts)
    np.testing.assert_allclose(a1, a2, atol=1e-5)
    no_qk = {k: v for k, v in parts.items() if k not in ("q_norm", "k_norm")}
    b1, *_ = O.gated_layer(x, Wqkv, Wo, gamma, 1.0, [0, 11], pos, bias, 4, 2, 8, 1e4, **no_qk)
    b2, *_ = O.gated_layer(x, W2, Wo, gamma, 1.0, [0, 11], pos, bias, 4, 2, 8, 1e4, **no_qk)
    assert np.abs(b1 - b2).max() > 1e-2


def test_full_layer_mlp_follows_attention():
    x, Wqkv, Wo, parts, pos, bias, gamma = _body_case(44)
    m = parts["mlp"]
    xo, _, _, pp = O.gated_layer(x, Wqkv, Wo, gamma, 1.0, [0, 11], pos, bias, 4, 2, 8, 1e4,
                                 **parts)
    no_mlp = {k: v for k, v in parts.items() if k != "mlp"}
    xa, _, _, _ = O.gated_layer(x, Wqkv, Wo, gamma, 1.0, [0, 11], pos, bias, 4, 2, 8, 1e4,
                                **no_mlp)
    np.testing.assert_allclose(pp["x_attn"], xa, atol=1e-13)
    np.testing.assert_allclose(xo, O.swiglu_mlp(xa, m["norm_w"], m["W_gate"], m["W_up"],
                                                m["W_down"]), atol=1e-13)
    # the same body below the gate: full context layer = gated layer with nothing pruned
    cu = [0, 6, 11]
    rp = O.request_positions(cu)
    f, kf, _ = O.full_context_layer(x, Wqkv, Wo, cu, 4, 2, 8, 1e4, **parts)
    g, kg, _, _ = O.gated_layer(x, Wqkv, Wo, np.zeros(4), 1.0, cu, rp, bias, 4, 2, 8, 1e4,
                                **parts)
    np.testing.assert_allclose(f, g, atol=1e-12)
    np.testing.assert_allclose(kf, kg, atol=1e-12)


# ------------------------------------------------------------------ attention gradients

def _torch_gated_attention(Q, K, V, cu, pos, bias, gamma, beta):
    """The gated attention written directly in torch (float64), for autograd."""
    Kt, Hq, d = Q.shape
    grp = Hq // K.shape[1]
    outs = []
    for b in range(len(cu) - 1):
        lo, hi = int(cu[b]), int(cu[b + 1])
        n = hi - lo
        r = torch.arange(n, dtype=torch.float64)
        p = torch.tensor(np.asarray(pos[lo:hi]), dtype=torch.float64)
        ratio = torch.where(p > 0, torch.log(r + 1) / torch.log(p.clamp(min=1) + 1),
                            torch.ones_like(r))
        tau = beta * ratio
        mask = torch.triu(torch.ones(n, n, dtype=torch.bool), 1)
        heads = []
        for h in range(Hq):
            s = Q[lo:hi, h] @ K[lo:hi, h // grp].T / math.sqrt(d)
            logit = tau[:, None] * s + gamma[h] * bias[None, lo:hi]
            w = torch.softmax(logit.masked_fill(mask, float("-inf")), dim=1)
            heads.append(w @ V[lo:hi, h // grp])
        outs.append(torch.stack(heads, 1))
    return torch.cat(outs, 0)


@pytest.mark.parametrize("seed", range(3))
def test_bias_grad_against_autograd(seed):
    """d_bias, d_gamma, d_beta against torch.autograd through the forward written in torch."""
    Q, K, V, cu, pos, bias, gamma = _rand_attn_case(60 + seed, [9, 1, 14])
    beta = 0.7 + 0.2 * seed
    dO = np.random.default_rng(70 + seed).normal(size=Q.shape)
    tb = torch.tensor(bias, requires_grad=True)
    tg_ = torch.tensor(gamma, requires_grad=True)
    tbeta = torch.tensor(beta, dtype=torch.float64, requires_grad=True)
    out = _torch_gated_attention(torch.tensor(Q), torch.tensor(K), torch.tensor(V), cu, pos,
                                 tb, tg_, tbeta)
    (out * torch.tensor(dO)).sum().backward()
    db, dg, dbeta = O.gated_attention_bias_grad(Q, K, V, dO, cu, pos, bias, gamma, beta)
    np.testing.assert_allclose(db, tb.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(dg, tg_.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(dbeta, tbeta.grad.item(), atol=1e-11)


def test_bias_grad_finite_differences_and_invariants():
    Q, K, V, cu, pos, bias, gamma = _rand_attn_case(80, [7, 5])
    dO = np.random.default_rng(81).normal(size=Q.shape)
    db, dg, dbeta = O.gated_attention_bias_grad(Q, K, V, dO, cu, pos, bias, gamma, 0.9)

    def loss(bias_=bias, gamma_=gamma, beta_=0.9):
        o, _ = O.gated_attention(Q, K, V, cu, pos, bias_, gamma_, beta_)
        return float(np.sum(o * dO))
    eps = 1e-6
    for c in (0, 3, 8, 11):
        e = np.zeros_like(bias)
        e[c] = eps
        fd = (loss(bias_=bias + e) - loss(bias_=bias - e)) / (2 * eps)
        assert abs(fd - db[c]) < 1e-7
    fd = (loss(beta_=0.9 + eps) - loss(beta_=0.9 - eps)) / (2 * eps)
    assert abs(fd - dbeta) < 1e-7
    e = np.zeros_like(gamma)
    e[2] = eps
    assert abs((loss(gamma_=gamma + e) - loss(gamma_=gamma - e)) / (2 * eps) - dg[2]) < 1e-7
    # softmax shift invariance: a bias constant over a request has zero total gradient
    for b in range(2):
        assert abs(db[cu[b]:cu[b + 1]].sum()) < 1e-10
    # gamma = 0 leaves the bias gradient zero; the first row of a request (one key) has none
    db0, _, _ = O.gated_attention_bias_grad(Q, K, V, dO, cu, pos, bias, np.zeros(4), 0.9)
    np.testing.assert_allclose(db0, 0.0, atol=0)


def test_gate_score_backward_against_autograd():
    """Scorer parameter gradients from dL/d(kept_bias), against torch.autograd through
    RMSNorm -> MLP -> sequence RMSNorm -> kept bias written directly in torch."""
    rng = np.random.default_rng(90)
    lens = [13, 1, 9]
    cu = np.concatenate([[0], np.cumsum(lens)])
    T, H, Fw = int(cu[-1]), 16, 6
    h = rng.normal(size=(T, H))
    W1 = rng.normal(size=(Fw, H)) * 0.5
    w2 = rng.normal(size=Fw)
    nw = rng.uniform(0.8, 1.2, size=H)
    pr = (rng.random(T) < 0.7).astype(np.uint8)
    kept = np.sort(rng.choice(T, size=12, replace=False))
    g = rng.normal(size=len(kept))
    th, tW1 = torch.tensor(h), torch.tensor(W1, requires_grad=True)
    tw2, tnw = torch.tensor(w2, requires_grad=True), torch.tensor(nw, requires_grad=True)
    x = F.rms_norm(th, (H,), tnw, eps=1e-6)
    s = F.silu(x @ tW1.T) @ tw2
    z = torch.cat([s[cu[b]:cu[b + 1]] / torch.sqrt(torch.mean(s[cu[b]:cu[b + 1]] ** 2) + 1e-6)
                   for b in range(3)])
    bias = z * torch.tensor(pr, dtype=torch.float64)
    (bias[torch.tensor(kept)] * torch.tensor(g)).sum().backward()
    out = O.gate_score_backward(h, nw, W1, w2, cu, pr, kept, g)
    np.testing.assert_allclose(out["dW1"], tW1.grad.numpy(), atol=1e-10)
    np.testing.assert_allclose(out["dw2"], tw2.grad.numpy(), atol=1e-10)
    np.testing.assert_allclose(out["dnorm_w"], tnw.grad.numpy(), atol=1e-10)
    # question tokens and pruned tokens receive no dz
    dz = out["dz"]
    assert np.all(dz[pr == 0] == 0)
    assert np.all(dz[np.setdiff1d(np.arange(T), kept)] == 0)
    # the sequence norm makes z scale-free: ds is orthogonal to s within each request
    s_np = O.gate_score(h, nw, W1, w2)
    for b in range(3):
        lo, hi = cu[b], cu[b + 1]
        assert abs(np.dot(out["ds"][lo:hi], s_np[lo:hi])) < 1e-6 * (1 + np.abs(s_np[lo:hi]).sum())


def test_gate_score_backward_finite_differences_and_scale_invariance():
    """Central differences of the oracle's own forward (scores -> sequence RMSNorm ->
    kept bias) for entries of W1, w2 and the norm weight; and, as z does not change when
    w2 is scaled (eps aside), the w2 gradient is orthogonal to w2."""
    rng = np.random.default_rng(92)
    lens = [11, 6]
    cu = np.concatenate([[0], np.cumsum(lens)])
    T, H, Fw = int(cu[-1]), 12, 5
    h = rng.normal(size=(T, H))
    W1 = rng.normal(size=(Fw, H)) * 0.6
    w2 = rng.normal(size=Fw)
    nw = rng.uniform(0.8, 1.2, size=H)
    pr = np.ones(T, dtype=np.uint8)
    pr[[4, 10, 16]] = 0
    kept = np.array([0, 2, 4, 7, 9, 10, 12, 13, 16])
    g = rng.normal(size=len(kept))

    def loss(W1_=W1, w2_=w2, nw_=nw):
        s = O.gate_score(h, nw_, W1_, w2_)
        _, bias = O.sequence_rmsnorm(s, cu, pr)
        return float(np.dot(bias[kept], g))
    out = O.gate_score_backward(h, nw, W1, w2, cu, pr, kept, g)
    eps = 1e-6
    for f, i in ((0, 0), (2, 7), (4, 11)):
        e = np.zeros_like(W1)
        e[f, i] = eps
        fd = (loss(W1_=W1 + e) - loss(W1_=W1 - e)) / (2 * eps)
        assert abs(fd - out["dW1"][f, i]) < 1e-7 * (1 + abs(fd))
    for f in (1, 3):
        e = np.zeros_like(w2)
        e[f] = eps
        fd = (loss(w2_=w2 + e) - loss(w2_=w2 - e)) / (2 * eps)
        assert abs(fd - out["dw2"][f]) < 1e-7 * (1 + abs(fd))
    for i in (0, 5):
        e = np.zeros_like(nw)
        e[i] = eps
        fd = (loss(nw_=nw + e) - loss(nw_=nw - e)) / (2 * eps)
        assert abs(fd - out["dnorm_w"][i]) < 1e-7 * (1 + abs(fd))
    # z(c w2) = z(w2) up to eps_seq: d/dc L(c w2) at c = 1 is w2 . dw2 ~ 0
    assert abs(np.dot(w2, out["dw2"])) < 1e-4 * np.abs(w2).dot(np.abs(out["dw2"]))
