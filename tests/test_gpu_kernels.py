"""Per-kernel parity of the CUDA path against the CPU oracle (needs a B200).

Every call goes through the C ABI (the ctypes binding).  Integer and index work is
compared bit for bit; floating point within the stated tolerances:
  * attention output: max-abs <= 2e-2 and mean-abs <= 1e-3 (bf16 inputs, fp32 accumulation);
  * gate z: max-abs <= 1e-2, mean-abs <= 1e-3 with the unit RMSNorm weight of the
    workloads.  A non-unit weight is folded into W1 rounded to bf16, a relative operand
    rounding of up to 2^-9 per product (the same order as a bf16 RMSNorm output); the
    z error then averages about 2^-9 |z| ~ 1.5e-3, so that case uses mean-abs <= 2.5e-3;
  * bf16 outputs of projections / RoPE: the bf16 rounding of the result plus fp32
    accumulation error, i.e. |err| <= 2^-7 |ref| + atol (atol stated per test).
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
import synthetic_inputs as S

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

ATT_MAX, ATT_MEAN = 2e-2, 1e-3
Z_MAX, Z_MEAN = 1e-2, 1e-3


@pytest.fixture(scope="module")
def tg():
    import learned_token_pruning_scoring_b200 as m
    assert m.tg_device_supported(torch.cuda.current_device())
    return m


def _dev(t):
    return t.to("cuda")


def _f64(t):
    return O.as_f64(t)


def _status():
    return torch.zeros(1, dtype=torch.int32, device="cuda")


# ------------------------------------------------------------------ RoPE table / gather

def test_rope_table(tg):
    tab = tg.tg_rope_table(4099, 128, 1.0e6).cpu().double().numpy()
    ang = O.rope_angles(np.arange(4099), 128, 1.0e6)
    assert np.abs(tab[..., 0] - np.cos(ang)).max() < 1e-7
    assert np.abs(tab[..., 1] - np.sin(ang)).max() < 1e-7


def test_rope_table_large_positions(tg):
    tab = tg.tg_rope_table(131072, 128, 1.0e6).cpu().double().numpy()
    rows = np.array([0, 1, 65535, 100003, 131071])
    ang = O.rope_angles(rows, 128, 1.0e6)
    assert np.abs(tab[rows, :, 0] - np.cos(ang)).max() < 1e-7
    assert np.abs(tab[rows, :, 1] - np.sin(ang)).max() < 1e-7


@pytest.mark.parametrize("n_src,n_rows,width", [(1000, 333, 2048), (50, 50, 8), (7, 3, 264)])
def test_gather_bit_exact(tg, n_src, n_rows, width):
    src = _dev(S.uniform_rows(n_src, width, seed=n_rows))
    idx = torch.randint(0, n_src, (n_rows,), generator=torch.Generator().manual_seed(1),
                        dtype=torch.int32)
    out = tg.tg_gather_rope(src, row_idx=_dev(idx))
    assert torch.equal(out.cpu(), src.cpu()[idx.long()])


@pytest.mark.parametrize("n_src,n_rows,width,ssq", [
    (1000, 1, 2048, True), (1000, 3, 2048, False), (1000, 5, 2048, True),
    (20000, 1638, 2048, True), (131072, 13107, 2048, True),   # kept rows of the 16k / 128k steps
    (5000, 4000, 8192, False),                                  # three stages: refills at lag 2
    (300, 299, 64, False), (300, 77, 192, False), (300, 257, 4096, True)])
@pytest.mark.parametrize("tma", [True, False])
def test_gather_tma_and_copy_kernels(tg, n_src, n_rows, width, ssq, tma):
    """The gather mode's two kernels (TMA row gather, warp-per-row copy) move the same
    bytes, tail groups of fewer than four rows and ring refills included, and write the
    same row sums of squares."""
    src = _dev(S.uniform_rows(n_src, width, seed=n_rows + width))
    idx = torch.randint(0, n_src, (n_rows,), generator=torch.Generator().manual_seed(n_rows),
                        dtype=torch.int32)
    prev = tg.tg_get_gather_tma()
    try:
        tg.tg_set_gather_tma(tma)
        st = _status()
        q = torch.full((n_rows, width // 128), float("nan"), device="cuda") if ssq else None
        out = tg.tg_gather_rope(src, row_idx=_dev(idx), row_ssq=q, status=st)
        assert tg.tg_status_read(st) == 0
    finally:
        tg.tg_set_gather_tma(prev)
    want = src.cpu()[idx.long()]
    assert torch.equal(out.cpu(), want)
    if ssq:
        ref = (want.double() ** 2).view(n_rows, width // 128, 128).sum(-1)
        assert torch.allclose(q.cpu().double(), ref, rtol=1e-5, atol=1e-5)


@pytest.mark.parametrize("tma", [True, False])
def test_gather_out_of_range_rows_are_skipped(tg, tma):
    """Indices outside the source set TG_STATUS_BOUNDS and leave their destination rows
    as they were; the other rows of the same group of four are still copied."""
    n_src, width = 100, 2048
    src = _dev(S.uniform_rows(n_src, width, seed=4))
    idx = torch.tensor([3, -1, 7, 9, 100, 11, 12, 13, 50], dtype=torch.int32)
    dst = torch.full((len(idx), width), 7.0, dtype=torch.bfloat16, device="cuda")
    prev = tg.tg_get_gather_tma()
    try:
        tg.tg_set_gather_tma(tma)
        st = _status()
        tg.tg_gather_rope(src, dst, row_idx=_dev(idx), status=st)
        assert tg.tg_status_read(st) & tg.STATUS_BOUNDS
    finally:
        tg.tg_set_gather_tma(prev)
    got = dst.cpu()
    for r, i in enumerate(idx.tolist()):
        if 0 <= i < n_src:
            assert torch.equal(got[r], src.cpu()[i]), r
        else:
            assert torch.all(got[r] == 7.0), r


def test_gather_strided_views(tg):
    big = _dev(S.uniform_rows(300, 4096, seed=3))
    src = big[:, 1024:3072]
    dst_big = torch.zeros((100, 2560), dtype=torch.bfloat16, device="cuda")
    dst = dst_big[:, 256:2304]
    idx = torch.arange(299, 0, -3, dtype=torch.int32)[:100]
    tg.tg_gather_rope(src, dst, row_idx=_dev(idx))
    assert torch.equal(dst.cpu(), src.cpu()[idx.long()])
    assert torch.count_nonzero(dst_big[:, :256]) == 0 and torch.count_nonzero(dst_big[:, 2304:]) == 0


def test_rope_in_place_against_oracle(tg):
    Hq, Hkv, d = 16, 8, 128
    n = 257
    qkv = S.uniform_rows(n, (Hq + 2 * Hkv) * d, seed=5)
    pos = torch.sort(torch.randperm(131072, generator=torch.Generator().manual_seed(2))[:n])[0]
    pos = pos.to(torch.int32)
    cs = tg.tg_rope_table(131072, d, 1.0e6)
    x = _dev(qkv.clone())
    tg.tg_gather_rope(x, x, rope_pos=_dev(pos), rope_cols=(0, (Hq + Hkv) * d), head_dim=d,
                      cos_sin=cs)
    got = _f64(x.cpu())
    src = _f64(qkv)
    want = np.concatenate([
        O.rope(src[:, :(Hq + Hkv) * d].reshape(n, Hq + Hkv, d), pos, 1.0e6).reshape(n, -1),
        src[:, (Hq + Hkv) * d:]], axis=1)
    err = np.abs(got - want)
    assert np.all(err <= 2.0 ** -7 * np.abs(want) + 1e-5), err.max()
    # V columns are untouched bit for bit
    assert torch.equal(x.cpu()[:, (Hq + Hkv) * d:], qkv[:, (Hq + Hkv) * d:])


def test_kv_compact_bit_exact(tg):
    qkv = _dev(S.uniform_rows(200, 4096, seed=9))
    k, v = qkv[:, 2048:3072], qkv[:, 3072:]
    ck = torch.zeros((260, 1024), dtype=torch.bfloat16, device="cuda")
    cv = torch.zeros_like(ck)
    tg.tg_kv_compact(k, v, ck, cv, slot_offset=60)
    assert torch.equal(ck[60:].cpu(), k.cpu()) and torch.equal(cv[60:].cpu(), v.cpu())
    assert torch.count_nonzero(ck[:60]) == 0
    idx = _dev(torch.tensor([5, 0, 199, 17], dtype=torch.int32))
    tg.tg_kv_compact(k, v, ck, cv, row_idx=idx, slot_offset=0)
    assert torch.equal(ck[:4].cpu(), k.cpu()[idx.long().cpu()])
    assert torch.equal(cv[:4].cpu(), v.cpu()[idx.long().cpu()])


# ------------------------------------------------------------------ selection

def _topk_case(tg, z32, prunable, lengths, budgets):
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    nq = [int((prunable[cu[b]:cu[b + 1]] == 0).sum()) for b in range(len(lengths))]
    ck = tg.tg_plan_kept(cu, nq, budgets)
    assert np.array_equal(ck.numpy(), O.kept_counts(prunable, cu, budgets))
    st = _status()
    idx, pos, kb = tg.tg_topk_compact(_dev(torch.from_numpy(z32)),
                                      _dev(torch.from_numpy(prunable)),
                                      _dev(torch.from_numpy(cu)), cu, _dev(ck), ck, status=st)
    assert tg.tg_status_read(st) == 0
    w_idx, w_pos, w_kb = O.select_topk(z32, prunable, cu, ck.numpy())
    assert np.array_equal(idx.cpu().numpy(), w_idx)
    assert np.array_equal(pos.cpu().numpy(), w_pos)
    assert np.array_equal(kb.cpu().numpy().view(np.uint32), w_kb.view(np.uint32))


@pytest.mark.parametrize("seed", range(6))
def test_topk_random_ragged(tg, seed):
    rng = np.random.default_rng(seed)
    lengths = [1, 31, 33, 1000, 4097, 0, 257][: 3 + seed % 5]
    T = sum(lengths)
    z = rng.normal(size=T).astype(np.float32)
    if seed % 2:
        z = (np.round(z * 3) / 3).astype(np.float32)  # many ties
    pr = (rng.random(T) < 0.85).astype(np.uint8)
    budgets = [int(rng.integers(0, n + 3)) for n in lengths]
    _topk_case(tg, z, pr, lengths, budgets)


def test_topk_special_values(tg):
    z = np.array([np.nan, -0.0, 0.0, np.inf, -np.inf, 1.0, 1.0, np.nan, -0.0, 5.0, -1e30, 1e-45],
                 dtype=np.float32)
    pr = np.array([1, 1, 1, 1, 1, 1, 1, 1, 1, 0, 1, 1], dtype=np.uint8)
    for budget in range(0, 13):
        _topk_case(tg, z, pr, [12], [budget])


def test_topk_all_equal_and_extremes(tg):
    z = np.full(5000, 0.25, dtype=np.float32)
    pr = np.ones(5000, dtype=np.uint8)
    pr[-10:] = 0
    for budget in (0, 10, 11, 2500, 4999, 5000, 9000):
        _topk_case(tg, z, pr, [5000], [budget])


def test_topk_planted_cluster_full_size(tg):
    wl = S.n128k()
    s = S.drawn_scores(wl)
    pr = S.prunable_mask(wl).numpy()
    z, _ = O.sequence_rmsnorm(s, wl.cu_seqlens(), pr)
    _topk_case(tg, z.astype(np.float32), pr, list(wl.lengths), list(wl.budgets))


def test_topk_ragged8_full_size(tg):
    wl = S.ragged8()
    T = wl.total_tokens
    rng = np.random.default_rng(8)
    z = rng.normal(size=T).astype(np.float32)
    _topk_case(tg, z, S.prunable_mask(wl).numpy(), list(wl.lengths), list(wl.budgets))


def test_topk_long_request_uncached_path(tg):
    n = 300_000  # slices exceed the per-CTA shared-memory key cache
    rng = np.random.default_rng(4)
    z = rng.normal(size=n).astype(np.float32)
    pr = np.ones(n, dtype=np.uint8)
    pr[-100:] = 0
    _topk_case(tg, z, pr, [n], [30_000])


def test_topk_budget_inconsistency_sets_status(tg):
    z = torch.randn(100, device="cuda")
    pr = torch.ones(100, dtype=torch.uint8, device="cuda")
    pr[-20:] = 0
    cu = np.array([0, 100], dtype=np.int32)
    ck = np.array([0, 10], dtype=np.int32)  # fewer than the 20 question tokens
    st = _status()
    idx = torch.full((10,), -7, dtype=torch.int32, device="cuda")
    tg.tg_topk_compact(z, pr, _dev(torch.from_numpy(cu)), cu, _dev(torch.from_numpy(ck)), ck,
                       kept_idx=idx, status=st)
    assert tg.tg_status_read(st) & tg.STATUS_BUDGET
    assert torch.all(idx == -7)  # nothing written


# ------------------------------------------------------------------ gate score

def _gate_case(tg, lengths, questions, seed, norm_w_random=False, rows=None):
    wl = S.custom(lengths, questions, [0] * len(lengths), seeds=[seed + i for i in range(len(lengths))])
    h = S.hidden_rows(wl)
    gw = S.gate_weights(wl)
    if norm_w_random:
        gw["norm_w"] = (0.5 + torch.rand(wl.hidden, generator=torch.Generator().manual_seed(7)))
        gw["norm_w"] = gw["norm_w"].to(torch.float32)
    pr = S.prunable_mask(wl)
    cu = np.array(wl.cu_seqlens(), dtype=np.int32)
    st = _status()
    s, z, bias = tg.tg_gate_score(_dev(h), _dev(gw["W1"]), _dev(gw["w2"]),
                                  _dev(torch.from_numpy(cu)), cu, _dev(pr),
                                  norm_w=_dev(gw["norm_w"]), status=st)
    assert tg.tg_status_read(st) == 0
    w_s = O.gate_score(h, gw["norm_w"], gw["W1"], gw["w2"])
    w_z, w_b = O.sequence_rmsnorm(w_s, cu, pr)
    g_s, g_z, g_b = s.cpu().double().numpy(), z.cpu().double().numpy(), bias.cpu().double().numpy()
    scale = np.sqrt(np.mean(w_s ** 2))
    assert np.abs(g_s - w_s).max() <= 1e-2 * scale
    z_mean_tol = 2.5e-3 if norm_w_random else Z_MEAN
    assert np.abs(g_z - w_z).max() <= Z_MAX and np.abs(g_z - w_z).mean() <= z_mean_tol
    assert np.abs(g_b - w_b).max() <= Z_MAX
    assert np.all(g_b[pr.numpy() == 0] == 0)
    return g_z, w_z


def test_gate_score_n1k(tg):
    _gate_case(tg, [1024], [64], seed=0)


def test_gate_score_ragged_requests_and_norm_weight(tg):
    # lengths not multiples of the 128-row tile or the 32-row partial chunks
    _gate_case(tg, [100, 37, 900, 1, 31, 33], [5, 0, 64, 1, 3, 33], seed=3, norm_w_random=True)


def test_gate_score_n16k_full(tg):
    _gate_case(tg, [16384], [64], seed=0)


@pytest.mark.parametrize("lengths", [[1], [200], [256], [257], [5000, 3000], [16384],
                                     [700, 37, 900, 1], [40000]])
def test_scorer_pair_matches_one_cta_kernel(tg, lengths):
    """The CTA-pair scorer and the one-CTA scorer form the same products and reduce them
    in the same order: s, z and bias agree bit for bit (tails of a 256-row pair tile,
    requests shorter than a tile, several tiles per cluster at 40k)."""
    wl = S.custom(lengths, [min(64, n) for n in lengths], [0] * len(lengths))
    h = _dev(S.hidden_rows(wl))
    gw = {k: _dev(v) for k, v in S.gate_weights(wl).items()}
    nw = _dev(0.8 + 0.4 * torch.rand(wl.hidden, generator=torch.Generator().manual_seed(5)))
    pr = _dev(S.prunable_mask(wl))
    cu = np.array(wl.cu_seqlens(), dtype=np.int32)
    cud = _dev(torch.from_numpy(cu))
    prev = tg.tg_get_scorer_pair()
    outs = []
    try:
        for pair in (True, False):
            tg.tg_set_scorer_pair(pair)
            st = _status()
            outs.append(tg.tg_gate_score(h, gw["W1"], gw["w2"], cud, cu, pr, norm_w=nw, status=st))
            assert tg.tg_status_read(st) == 0
    finally:
        tg.tg_set_scorer_pair(prev)
    for name, a, b in zip(("s", "z", "bias"), *outs):
        assert torch.equal(a, b), (name, (a - b).abs().max().item())


def test_gate_score_deterministic(tg):
    wl = S.custom([5000, 3000], [64, 16], [0, 0])
    h = _dev(S.hidden_rows(wl))
    gw = {k: _dev(v) for k, v in S.gate_weights(wl).items()}
    pr = _dev(S.prunable_mask(wl))
    cu = np.array(wl.cu_seqlens(), dtype=np.int32)
    outs = [tg.tg_gate_score(h, gw["W1"], gw["w2"], _dev(torch.from_numpy(cu)), cu, pr,
                             norm_w=gw["norm_w"]) for _ in range(2)]
    for a, b in zip(*outs):
        assert torch.equal(a, b)


# ------------------------------------------------------------------ projections

# shapes with N % 256 == 0 and no folded norm run on CTA pairs (256 x 256 tiles)
@pytest.mark.parametrize("M,N,K,rms,res", [(1, 128, 64, False, False), (100, 256, 2048, True, False),
                                           (1638, 4096, 2048, True, False),
                                           (1638, 2048, 2048, False, True),
                                           (300, 384, 192, True, True),
                                           (1, 256, 64, False, False),
                                           (257, 512, 1024, False, True),
                                           (1638, 4096, 2048, False, False)])
def test_linear_against_oracle(tg, M, N, K, rms, res):
    a = S.uniform_rows(M, K, seed=M + 1)
    w = S.uniform_rows(N, K, seed=N + 2, scale=0.02)
    r = S.uniform_rows(M, N, seed=3) if res else None
    st = _status()  # a bounded wait that expired would show here, not as wrong values
    c = tg.tg_linear(_dev(a), _dev(w), rmsnorm=rms, residual=_dev(r) if res else None,
                     status=st)
    assert tg.tg_status_read(st) == 0
    A = O.rmsnorm_rows(a) if rms else _f64(a)
    want = A @ _f64(w).T + (_f64(r) if res else 0.0)
    got = _f64(c.cpu())
    err = np.abs(got - want)
    bad = np.argwhere(err > 2.0 ** -7 * np.abs(want) + 2e-3)
    assert bad.size == 0, (err.max(), len(bad), bad[:8].tolist())  # which rows / columns


def test_one_cta_gemm_repeats_bit_for_bit(tg):
    """The one-CTA GEMM with the RMSNorm accumulated from its A stages (the scorer's path
    and tg_linear's path for shapes the pair kernel does not take) is deterministic: 200
    repeats of tg_linear(rmsnorm) at 1638 x 4096 x 2048 and of the 16k scorer must each
    equal the first call bit for bit.  A race between the stage reads and the ring's
    refills would show as a rare differing element."""
    M, N, K = 1638, 4096, 2048
    a = _dev(S.uniform_rows(M, K, seed=M + 1))
    w = _dev(S.uniform_rows(N, K, seed=N + 2, scale=0.02))
    st = _status()
    first = tg.tg_linear(a, w, rmsnorm=True, status=st)
    out = torch.empty_like(first)
    bad = []
    for i in range(200):
        tg.tg_linear(a, w, out, rmsnorm=True, status=st)
        if not torch.equal(out, first):
            bad.append((i, int((out != first).sum())))
    wl = S.custom([16384], [64], [0])
    h = _dev(S.hidden_rows(wl))
    gw = {k: _dev(v) for k, v in S.gate_weights(wl).items()}
    pr = _dev(S.prunable_mask(wl))
    cu = np.array(wl.cu_seqlens(), dtype=np.int32)
    cud = _dev(torch.from_numpy(cu))
    s0 = tg.tg_gate_score(h, gw["W1"], gw["w2"], cud, cu, pr, status=st)[0].clone()
    for i in range(200):
        s = tg.tg_gate_score(h, gw["W1"], gw["w2"], cud, cu, pr, status=st)[0]
        if not torch.equal(s, s0):
            bad.append(("scorer", i, int((s != s0).sum())))
    assert tg.tg_status_read(st) == 0
    assert not bad, bad


@pytest.mark.parametrize("N", [384, 2048])
def test_linear_row_sums_of_squares(tg, N):
    M, K = 333, 512
    a = _dev(S.uniform_rows(M, K, seed=6))
    w = _dev(S.uniform_rows(N, K, seed=7, scale=0.05))
    r = _dev(S.uniform_rows(M, N, seed=8))
    ssq = torch.full((M, N // 128), float("nan"), device="cuda")
    st = _status()
    c = tg.tg_linear(a, w, residual=r, row_ssq=ssq, status=st)
    assert tg.tg_status_read(st) == 0
    want = (c.double() ** 2).view(M, N // 128, 128).sum(-1)
    assert torch.allclose(ssq.double(), want, rtol=1e-5, atol=1e-5)


def _gemm_flags(ws):
    """The ready flags of a stream-K workspace: they follow the partial sums (256 KB per
    cluster) and must be zero again after every call."""
    part = ws.numel() // 262144 * 262144
    return ws[part:]


@pytest.mark.parametrize("M,N", [(1638, 2048), (1638, 4096), (300, 2048), (7000, 2048)])
def test_linear_stream_k_against_oracle(tg, M, N):
    """Residual + row sums of squares on the CTA-pair kernel with the stream-K tail: the
    output projection's shape at 16k (56 tiles on 74 clusters: every tile split), a QKV
    width, a small M, and a shape whose tail is too short to split; results within the
    GEMM tolerance of the oracle and bit-reproducible."""
    K = 2048
    a = _dev(S.uniform_rows(M, K, seed=M + 11))
    w = _dev(S.uniform_rows(N, K, seed=N + 12, scale=0.02))
    r = _dev(S.uniform_rows(M, N, seed=13))
    ws = torch.zeros(tg.tg_gemm_workspace_size(), dtype=torch.uint8, device="cuda")
    outs = []
    for _ in range(2):
        ssq = torch.full((M, N // 128), float("nan"), device="cuda")
        st = _status()
        c = tg.tg_linear(a, w, residual=r, row_ssq=ssq, status=st, workspace=ws)
        assert tg.tg_status_read(st) == 0
        outs.append((c, ssq))
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])
    assert torch.count_nonzero(_gemm_flags(ws)) == 0
    c, ssq = outs[0]
    want = _f64(a.cpu()) @ _f64(w.cpu()).T + _f64(r.cpu())
    err = np.abs(_f64(c.cpu()) - want)
    bad = np.argwhere(err > 2.0 ** -7 * np.abs(want) + 2e-3)
    assert bad.size == 0, (err.max(), len(bad), bad[:8].tolist())
    want_ssq = (c.double() ** 2).view(M, N // 128, 128).sum(-1)
    assert torch.allclose(ssq.double(), want_ssq, rtol=1e-5, atol=1e-5)


def test_linear_residual_in_place(tg):
    x = _dev(S.uniform_rows(257, 256, seed=1))
    x0 = x.clone()
    o = _dev(S.uniform_rows(257, 512, seed=2))
    w = _dev(S.uniform_rows(256, 512, seed=3, scale=0.02))
    tg.tg_linear(o, w, x, residual=x)
    want = _f64(x0.cpu()) + _f64(o.cpu()) @ _f64(w.cpu()).T
    err = np.abs(_f64(x.cpu()) - want)
    assert np.all(err <= 2.0 ** -7 * np.abs(want) + 2e-3)


# ------------------------------------------------------------------ attention

def _attn_inputs(lengths, Hq, Hkv, seed, pos_spread=4, dense=False):
    d = 128
    g = torch.Generator().manual_seed(seed)
    Kt = int(sum(lengths))
    q = (torch.randn((Kt, Hq * d), generator=g)).to(torch.bfloat16)
    k = (torch.randn((Kt, Hkv * d), generator=g)).to(torch.bfloat16)
    v = (torch.randn((Kt, Hkv * d), generator=g)).to(torch.bfloat16)
    pos, bias = [], []
    for n in lengths:
        if dense:
            pos.append(torch.arange(n, dtype=torch.int32))
        else:
            pos.append(torch.sort(torch.randperm(max(1, pos_spread * n + 5), generator=g)[:n])[0]
                       .to(torch.int32))
        b = torch.randn((n,), generator=g) * (torch.rand((n,), generator=g) < 0.9)
        bias.append(b.to(torch.float32))
    pos = torch.cat(pos) if pos else torch.zeros(0, dtype=torch.int32)
    bias = torch.cat(bias) if bias else torch.zeros(0)
    gamma = (0.5 + 1.5 * torch.rand((Hq,), generator=g)).to(torch.float32)
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    return q, k, v, pos, bias, gamma, cu


def _run_attention(tg, q, k, v, pos, bias, gamma, beta, cu, Hq, Hkv, lse=True, split=True):
    Kt = q.shape[0]
    lse_t = torch.full((Hq, Kt), float("nan"), device="cuda") if lse else None
    st = _status()
    ws = None if split else torch.empty(0, dtype=torch.uint8, device="cuda")
    o = tg.tg_gated_attention(_dev(q), _dev(k), _dev(v), _dev(torch.from_numpy(cu)), cu, Hq, Hkv,
                              _dev(pos), _dev(bias), _dev(gamma), beta, lse=lse_t, workspace=ws,
                              status=st)
    assert tg.tg_status_read(st) == 0
    return o.cpu(), (lse_t.cpu() if lse else None)


def _check_attention(o_gpu, lse_gpu, q, k, v, pos, bias, gamma, beta, cu, Hq, Hkv, rows=None):
    d = 128
    Kt = q.shape[0]
    Q = _f64(q).reshape(Kt, Hq, d)
    K = _f64(k).reshape(Kt, Hkv, d)
    V = _f64(v).reshape(Kt, Hkv, d)
    want, wlse = O.gated_attention(Q, K, V, cu, pos, bias, gamma, beta, rows=rows)
    got = _f64(o_gpu).reshape(Kt, Hq, d)
    sel = slice(None) if rows is None else np.asarray(rows)
    err = np.abs(got[sel] - want[sel])
    assert err.max() <= ATT_MAX, err.max()
    assert err.mean() <= ATT_MEAN, err.mean()
    if lse_gpu is not None:
        lerr = np.abs(_f64(lse_gpu)[:, sel] - wlse[:, sel])
        assert lerr.max() <= 1e-3, lerr.max()


@pytest.mark.parametrize("lengths", [[1], [5], [127], [128], [129], [300], [256, 1, 129, 77]])
def test_attention_small_shapes(tg, lengths):
    q, k, v, pos, bias, gamma, cu = _attn_inputs(lengths, 16, 8, seed=sum(lengths))
    o, lse = _run_attention(tg, q, k, v, pos, bias, gamma, 1.0, cu, 16, 8)
    _check_attention(o, lse, q, k, v, pos, bias, gamma, 1.0, cu, 16, 8)


def test_attention_group4_and_beta(tg):
    q, k, v, pos, bias, gamma, cu = _attn_inputs([700, 190], 8, 2, seed=11)
    o, lse = _run_attention(tg, q, k, v, pos, bias, gamma, 0.7, cu, 8, 2)
    _check_attention(o, lse, q, k, v, pos, bias, gamma, 0.7, cu, 8, 2)


@pytest.mark.parametrize("split", [True, False])
def test_attention_n16k_kept_1638(tg, split):
    cu_h = np.array([0, 1638], dtype=np.int32)
    assert tg.tg_gated_attention_workspace_size(cu_h, 16, 8) > 0  # this layout splits
    q, k, v, pos, bias, gamma, cu = _attn_inputs([1638], 16, 8, seed=1638, pos_spread=10)
    o, lse = _run_attention(tg, q, k, v, pos, bias, gamma, 1.0, cu, 16, 8, split=split)
    _check_attention(o, lse, q, k, v, pos, bias, gamma, 1.0, cu, 16, 8)


def test_attention_split_varlen_requests(tg):
    lengths = [2000, 60, 3, 1100]
    q, k, v, pos, bias, gamma, cu = _attn_inputs(lengths, 16, 8, seed=77, pos_spread=6)
    assert tg.tg_gated_attention_workspace_size(cu, 16, 8) > 0
    o, lse = _run_attention(tg, q, k, v, pos, bias, gamma, 0.9, cu, 16, 8)
    _check_attention(o, lse, q, k, v, pos, bias, gamma, 0.9, cu, 16, 8)
    o2, lse2 = _run_attention(tg, q, k, v, pos, bias, gamma, 0.9, cu, 16, 8, split=False)
    assert (o.double() - o2.double()).abs().max() <= 2 ** -7
    assert (lse - lse2).abs().max() <= 1e-4


def test_attention_split_many_parts(tg):
    # One head group (2 q heads, 1 kv head): the plan cuts the request's 16 query tiles
    # into several key-range parts each, which the last-arriving part merges in part
    # order.  The chunk is read back from the workspace size (items x per-item bytes).
    n, Hq, Hkv = 2000, 2, 1
    q, k, v, pos, bias, gamma, cu = _attn_inputs([n], Hq, Hkv, seed=n, pos_spread=5)
    per_item = Hq * (128 * 128 + 2 * 128) * 4 + 8 * (Hq // 2)
    items = tg.tg_gated_attention_workspace_size(cu, Hq, Hkv) // per_item
    tiles = -(-n // 128)
    chunks = [c for c in range(1, tiles + 1)
              if sum(-(-(qt + 1) // c) for qt in range(tiles)) == items]
    assert chunks and -(-tiles // chunks[-1]) > 2, (items, chunks)
    o, lse = _run_attention(tg, q, k, v, pos, bias, gamma, 1.0, cu, Hq, Hkv)
    _check_attention(o, lse, q, k, v, pos, bias, gamma, 1.0, cu, Hq, Hkv)
    o2, lse2 = _run_attention(tg, q, k, v, pos, bias, gamma, 1.0, cu, Hq, Hkv, split=False)
    assert (o.double() - o2.double()).abs().max() <= 2 ** -7
    assert (lse - lse2).abs().max() <= 1e-4


def test_attention_n128k_kept_13107_sampled_rows(tg):
    q, k, v, pos, bias, gamma, cu = _attn_inputs([13107], 16, 8, seed=13107, pos_spread=10)
    o, lse = _run_attention(tg, q, k, v, pos, bias, gamma, 1.0, cu, 16, 8)
    rng = np.random.default_rng(0)
    rows = np.unique(np.concatenate([[0, 1, 127, 128, 13106], rng.integers(0, 13107, 120)]))
    _check_attention(o, lse, q, k, v, pos, bias, gamma, 1.0, cu, 16, 8, rows=rows)


def test_attention_dense_matches_sdpa(tg):
    """K = N, gamma = 0, positions = ranks: plain causal GQA attention (library SDPA)."""
    n = 1000
    q, k, v, pos, bias, gamma, cu = _attn_inputs([n], 16, 8, seed=5, dense=True)
    o, _ = _run_attention(tg, q, k, v, pos, bias, torch.zeros(16), 1.0, cu, 16, 8, lse=False)
    qt = q.view(n, 16, 128).permute(1, 0, 2)[None].cuda().float()
    kt = k.view(n, 8, 128).permute(1, 0, 2).repeat_interleave(2, 0)[None].cuda().float()
    vt = v.view(n, 8, 128).permute(1, 0, 2).repeat_interleave(2, 0)[None].cuda().float()
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True)
    ref = ref[0].permute(1, 0, 2).reshape(n, -1).cpu().double()
    err = (o.double() - ref).abs()
    assert err.max() <= ATT_MAX and err.mean() <= ATT_MEAN


def test_attention_beta_zero(tg):
    """beta = 0: tau is 0 on every row, so the logits are the gate term gamma_h z_c alone
    (q.k drops out).  The kernel clamps its per-row temperature at 2^-66, which makes the
    gain operand of the bias step about 1e20 gamma; the result must still match."""
    q, k, v, pos, bias, gamma, cu = _attn_inputs([300, 1, 129], 16, 8, seed=21)
    o, lse = _run_attention(tg, q, k, v, pos, bias, gamma, 0.0, cu, 16, 8)
    _check_attention(o, lse, q, k, v, pos, bias, gamma, 0.0, cu, 16, 8)


@pytest.mark.parametrize("lengths", [[1638], [2000, 60, 3, 1100], [13107]])
def test_attention_split_and_unsplit_repeat(tg, lengths):
    """Without a workspace every query tile runs whole in one CTA; with one, long tiles are
    split and merged.  Each way a second call repeats the result bit for bit (the split
    workspace is left zeroed by the first), and the split result matches the oracle."""
    q, k, v, pos, bias, gamma, cu = _attn_inputs(lengths, 16, 8, seed=sum(lengths), pos_spread=6)
    args = (_dev(q), _dev(k), _dev(v), _dev(torch.from_numpy(cu)), cu, 16, 8, _dev(pos),
            _dev(bias), _dev(gamma), 0.9)
    full = torch.zeros(max(16, tg.tg_gated_attention_workspace_size(cu, 16, 8)),
                       dtype=torch.uint8, device="cuda")
    empty = torch.zeros(0, dtype=torch.uint8, device="cuda")
    outs = []
    for ws in (empty, empty, full, full):
        st = _status()
        outs.append(tg.tg_gated_attention(*args, workspace=ws, status=st).cpu())
        assert tg.tg_status_read(st) == 0
    assert torch.equal(outs[0], outs[1])
    assert torch.equal(outs[2], outs[3])
    rows = np.unique(np.concatenate([[0, cu[-1] - 1], np.random.default_rng(3).integers(0, cu[-1], 60)]))
    _check_attention(outs[2], None, q, k, v, pos, bias, gamma, 0.9, cu, 16, 8, rows=rows)


def test_attention_rows_sum_to_one(tg):
    q, k, v, pos, bias, gamma, cu = _attn_inputs([517, 300], 16, 8, seed=2)
    ones = torch.ones_like(v)
    o, _ = _run_attention(tg, q, k, ones, pos, bias, gamma, 1.0, cu, 16, 8, lse=False)
    assert (o.double() - 1.0).abs().max() <= 2 ** -8


def test_attention_deterministic(tg):
    q, k, v, pos, bias, gamma, cu = _attn_inputs([900], 16, 8, seed=3)
    a, la = _run_attention(tg, q, k, v, pos, bias, gamma, 1.0, cu, 16, 8)
    b, lb = _run_attention(tg, q, k, v, pos, bias, gamma, 1.0, cu, 16, 8)
    assert torch.equal(a, b) and torch.equal(la, lb)


def test_attention_dirty_workspace_times_out_and_reports(tg):
    """Failure detection without a fault: a split workspace that was not zero-filled.
    One tile's arrival counter starts at 1, so that tile's first part counts itself last
    and waits for a ready flag that never comes (its other part sees the counter out of
    range and publishes nothing).  The bounded wait runs out (about 2 s); the call
    reports TIMEOUT | WORKSPACE and returns, and the next call on a clean workspace is
    correct."""
    import time
    q, k, v, pos, bias, gamma, cu = _attn_inputs([1638], 16, 8, seed=4, pos_spread=10)
    need = tg.tg_gated_attention_workspace_size(cu, 16, 8)
    groups = 8
    per_item = 16 * 66560 + 8 * groups   # partials for 16 q heads, counter + flag per group
    assert need > 0 and need % per_item == 0
    n_items = need // per_item
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    ws[n_items * 16 * 66560:].view(torch.int32)[0] = 1  # item 0 (a split tile), group 0
    st = _status()
    t0 = time.time()
    tg.tg_gated_attention(_dev(q), _dev(k), _dev(v), _dev(torch.from_numpy(cu)), cu, 16, 8,
                          _dev(pos), _dev(bias), _dev(gamma), 1.0, workspace=ws, status=st)
    got = tg.tg_status_read(st)
    assert got & tg.STATUS_TIMEOUT and got & tg.STATUS_WORKSPACE, hex(got)
    assert time.time() - t0 < 30
    o, lse = _run_attention(tg, q, k, v, pos, bias, gamma, 1.0, cu, 16, 8)
    _check_attention(o, lse, q, k, v, pos, bias, gamma, 1.0, cu, 16, 8)


# ------------------------------------------------------------------ fused QKV + RoPE + cache

@pytest.mark.parametrize("M", [1, 257, 1638])
def test_qkv_rope_cache_against_oracle(tg, M):
    Hq, Hkv, d, H = 16, 8, 128, 2048
    x = S.uniform_rows(M, H, seed=M)
    w = S.uniform_rows((Hq + 2 * Hkv) * d, H, seed=M + 1, scale=0.02)
    pos = torch.sort(torch.randperm(16384, generator=torch.Generator().manual_seed(M))[:M])[0]
    pos = pos.to(torch.int32)
    cs = tg.tg_rope_table(16384, d, 1.0e6)
    slot = 5
    ck = torch.zeros((M + slot, Hkv * d), dtype=torch.bfloat16, device="cuda")
    cv = torch.zeros_like(ck)
    st = _status()
    q = tg.tg_qkv_rope_cache(_dev(x), _dev(w), _dev(pos), cs, ck, cv, Hq, Hkv, slot_offset=slot,
                             status=st)
    assert tg.tg_status_read(st) == 0
    a = O.rmsnorm_rows(x)
    qkv = a @ _f64(w).T
    want_q = O.rope(qkv[:, :Hq * d].reshape(M, Hq, d), pos, 1.0e6).reshape(M, -1)
    want_k = O.rope(qkv[:, Hq * d:(Hq + Hkv) * d].reshape(M, Hkv, d), pos, 1.0e6).reshape(M, -1)
    want_v = qkv[:, (Hq + Hkv) * d:]
    for got, want in ((q, want_q), (ck[slot:], want_k), (cv[slot:], want_v)):
        err = np.abs(_f64(got.cpu()) - want)
        assert np.all(err <= 2.0 ** -7 * np.abs(want) + 2e-3), err.max()
    assert torch.count_nonzero(ck[:slot]) == 0 and torch.count_nonzero(cv[:slot]) == 0


@pytest.mark.parametrize("split", [False, True])
@pytest.mark.parametrize("M", [1, 300, 1638, 4000])
def test_qkv_rope_cache_with_row_sums_against_oracle(tg, M, split):
    """Precomputed row sums of squares select the CTA-pair kernel; with a GEMM workspace its
    last round of tiles is shared along K (stream-K; M = 1638: 112 tiles on 74 clusters,
    one whole round and 16-17 k-blocks of the rest per cluster)."""
    Hq, Hkv, d, H = 16, 8, 128, 2048
    x = S.uniform_rows(M, H, seed=M + 40)
    w = S.uniform_rows((Hq + 2 * Hkv) * d, H, seed=M + 41, scale=0.02)
    pos = torch.arange(0, 5 * M, 5, dtype=torch.int32)
    cs = tg.tg_rope_table(5 * M + 1, d, 1.0e6)
    ssq = torch.from_numpy((_f64(x) ** 2).reshape(M, H // 128, 128).sum(-1)).float()
    ck = torch.zeros((M, Hkv * d), dtype=torch.bfloat16, device="cuda")
    cv = torch.zeros_like(ck)
    ws = (torch.zeros(tg.tg_gemm_workspace_size(), dtype=torch.uint8, device="cuda") if split
          else None)
    st = _status()
    q = tg.tg_qkv_rope_cache(_dev(x), _dev(w), _dev(pos), cs, ck, cv, Hq, Hkv, row_ssq=_dev(ssq),
                             status=st, workspace=ws)
    assert tg.tg_status_read(st) == 0
    if split:  # the flags are left at zero, and a second call gives the same bits
        assert torch.count_nonzero(_gemm_flags(ws)) == 0
        q2 = tg.tg_qkv_rope_cache(_dev(x), _dev(w), _dev(pos), cs, ck.clone(), cv.clone(), Hq,
                                  Hkv, row_ssq=_dev(ssq), workspace=ws)
        assert torch.equal(q, q2)
    a = O.rmsnorm_rows(x)
    qkv = a @ _f64(w).T
    want_q = O.rope(qkv[:, :Hq * d].reshape(M, Hq, d), pos, 1.0e6).reshape(M, -1)
    want_k = O.rope(qkv[:, Hq * d:(Hq + Hkv) * d].reshape(M, Hkv, d), pos, 1.0e6).reshape(M, -1)
    want_v = qkv[:, (Hq + Hkv) * d:]
    for got, want in ((q, want_q), (ck, want_k), (cv, want_v)):
        err = np.abs(_f64(got.cpu()) - want)
        assert np.all(err <= 2.0 ** -7 * np.abs(want) + 2e-3), err.max()


def test_gather_row_sums_of_squares(tg):
    src = _dev(S.uniform_rows(500, 2048, seed=12))
    idx = _dev(torch.randint(0, 500, (321,), generator=torch.Generator().manual_seed(3),
                             dtype=torch.int32))
    ssq = torch.full((321, 16), float("nan"), device="cuda")
    out = tg.tg_gather_rope(src, row_idx=idx, row_ssq=ssq)
    want = (out.double() ** 2).view(321, 16, 128).sum(-1)
    assert torch.allclose(ssq.double(), want, rtol=1e-5, atol=1e-5)


def test_qkv_rope_cache_matches_unfused_path(tg):
    """The fused call equals projection -> RoPE -> KV copy up to one bf16 rounding."""
    M, Hq, Hkv, d, H = 300, 16, 8, 128, 2048
    x = _dev(S.uniform_rows(M, H, seed=4))
    w = _dev(S.uniform_rows((Hq + 2 * Hkv) * d, H, seed=5, scale=0.02))
    pos = _dev(torch.arange(0, 3 * M, 3, dtype=torch.int32))
    cs = tg.tg_rope_table(4096, d, 1.0e6)
    ck = torch.empty((M, Hkv * d), dtype=torch.bfloat16, device="cuda")
    cv = torch.empty_like(ck)
    q = tg.tg_qkv_rope_cache(x, w, pos, cs, ck, cv, Hq, Hkv)
    qkv = tg.tg_linear(x, w, rmsnorm=True)
    tg.tg_gather_rope(qkv, qkv, rope_pos=pos, rope_cols=(0, (Hq + Hkv) * d), head_dim=d,
                      cos_sin=cs)
    ref = qkv.double()
    # The unfused path rounds to bf16 before rotating: per element its error is bounded
    # by 2^-8 of the rotation pair's magnitude (which the rotation preserves) plus one
    # final rounding of each path.
    for got, want in ((q, ref[:, :Hq * d]), (ck, ref[:, Hq * d:(Hq + Hkv) * d]),
                      (cv, ref[:, (Hq + Hkv) * d:])):
        w = want.view(M, -1, 2, d // 2)
        pair = torch.sqrt(w[:, :, 0] ** 2 + w[:, :, 1] ** 2).repeat(1, 1, 2).view(M, -1)
        err = (got.double() - want).abs()
        assert (err <= 2.0 ** -7 * pair + 2.0 ** -8 * want.abs() + 1e-3).all(), err.max()


def test_qkv_rope_cache_position_out_of_table_sets_status(tg):
    M, Hq, Hkv, d, H = 4, 2, 2, 128, 64
    x = _dev(S.uniform_rows(M, H, seed=1))
    w = _dev(S.uniform_rows((Hq + 2 * Hkv) * d, H, seed=2, scale=0.1))
    pos = _dev(torch.tensor([0, 1, 99, 2], dtype=torch.int32))
    cs = tg.tg_rope_table(8, d, 1.0e6)
    ck = torch.empty((M, Hkv * d), dtype=torch.bfloat16, device="cuda")
    cv = torch.empty_like(ck)
    st = _status()
    tg.tg_qkv_rope_cache(x, w, pos, cs, ck, cv, Hq, Hkv, status=st)
    assert tg.tg_status_read(st) & tg.STATUS_BOUNDS


@pytest.mark.parametrize("M", [300, 1638, 4000])
def test_out_proj_qkv_chain_equals_the_two_calls(tg, M):
    """One layer boundary in one launch gives, bit for bit, what the two separate calls
    give (same tiles, same epilogues; only the scheduling differs).  M = 4000 has more
    output-projection tiles than clusters, so QKV tiles also wait for tiles that other
    clusters start later.  The counters come back zero."""
    Hq, Hkv, d, H = 16, 8, 128, 2048
    o = _dev(S.uniform_rows(M, Hq * d, seed=M + 1))
    x0 = _dev(S.uniform_rows(M, H, seed=M + 2, scale=3.0))
    wo = _dev(S.uniform_rows(H, Hq * d, seed=M + 3, scale=0.02))
    wqkv = _dev(S.uniform_rows((Hq + 2 * Hkv) * d, H, seed=M + 4, scale=0.02))
    pos = _dev(torch.arange(0, 7 * M, 7, dtype=torch.int32))
    cs = tg.tg_rope_table(7 * M + 1, d, 1.0e6)

    def fresh():
        return (x0.clone(), torch.full((M, H // 128), float("nan"), device="cuda"),
                torch.empty((M, Hq * d), dtype=torch.bfloat16, device="cuda"),
                torch.empty((M, Hkv * d), dtype=torch.bfloat16, device="cuda"),
                torch.empty((M, Hkv * d), dtype=torch.bfloat16, device="cuda"))

    x1, ssq1, q1, k1, v1 = fresh()
    tg.tg_linear(o, wo, x1, residual=x1, row_ssq=ssq1)
    tg.tg_qkv_rope_cache(x1, wqkv, pos, cs, k1, v1, Hq, Hkv, q_out=q1, row_ssq=ssq1)
    x2, ssq2, q2, k2, v2 = fresh()
    ws = torch.zeros(tg.tg_out_proj_qkv_workspace_size(M), dtype=torch.uint8, device="cuda")
    st = _status()
    for _ in range(2):  # the second call reuses the workspace the first left zeroed
        x2.copy_(x0)
        tg.tg_out_proj_qkv_next(o, wo, x2, ssq2, wqkv, pos, cs, k2, v2, Hq, Hkv, q2, ws, status=st)
    assert tg.tg_status_read(st) == 0
    assert torch.equal(x1, x2) and torch.equal(ssq1, ssq2)
    assert torch.equal(q1, q2) and torch.equal(k1, k2) and torch.equal(v1, v2)
    assert int(ws.count_nonzero()) == 0


# ------------------------------------------------------------------ full layer body parts

def test_weight_packing_bit_exact(tg):
    """tg_fold_norm_weight / tg_pack_gate_up against the same products rounded by torch."""
    F_, H = 256, 2048
    wg = S.uniform_rows(F_, H, seed=70, scale=0.02)
    wu = S.uniform_rows(F_, H, seed=71, scale=0.02)
    nw = (0.8 + 0.4 * torch.rand(H, generator=torch.Generator().manual_seed(72))).float()
    folded = tg.tg_fold_norm_weight(_dev(wg), _dev(nw)).cpu()
    assert torch.equal(folded, (wg.float() * nw).to(torch.bfloat16))
    packed = tg.tg_pack_gate_up(_dev(wg), _dev(wu), _dev(nw)).cpu()
    want = torch.empty((2 * F_, H), dtype=torch.bfloat16)
    for j in range(F_ // 64):
        want[128 * j:128 * j + 64] = (wg[64 * j:64 * j + 64].float() * nw).to(torch.bfloat16)
        want[128 * j + 64:128 * j + 128] = (wu[64 * j:64 * j + 64].float() * nw).to(torch.bfloat16)
    assert torch.equal(packed, want)
    plain = tg.tg_pack_gate_up(_dev(wg), _dev(wu)).cpu()
    assert torch.equal(plain[64:128], wu[:64]) and torch.equal(plain[128:192], wg[64:128])


def _ssq_rows(x, H):
    return torch.from_numpy((_f64(x) ** 2).reshape(x.shape[0], H // 128, 128).sum(-1)).float()


@pytest.mark.parametrize("M", [1, 300, 1638])
def test_qkv_qknorm_rope_cache_against_oracle(tg, M):
    """QK-norm and RoPE in the epilogue, on a Wqkv with a weighted attention norm folded
    in.  The oracle gets the same folded bf16 weight the kernel reads (the fold itself is
    bit-exact against torch in test_weight_packing_bit_exact; its rounding, ~1e-3 of a
    normalised head, belongs to the end-to-end tolerance study, not to this kernel)."""
    Hq, Hkv, d, H = 16, 8, 128, 2048
    x = S.uniform_rows(M, H, seed=M + 80)
    w = S.uniform_rows((Hq + 2 * Hkv) * d, H, seed=M + 81, scale=0.02)
    g = torch.Generator().manual_seed(M + 82)
    attn_norm = (0.8 + 0.4 * torch.rand(H, generator=g)).float()
    qn = (0.8 + 0.4 * torch.rand(d, generator=g)).float()
    kn = (0.8 + 0.4 * torch.rand(d, generator=g)).float()
    pos = torch.arange(0, 3 * M, 3, dtype=torch.int32)
    cs = tg.tg_rope_table(3 * M + 1, d, 1.0e6)
    ck = torch.zeros((M, Hkv * d), dtype=torch.bfloat16, device="cuda")
    cv = torch.zeros_like(ck)
    L = tg.prepare_layer({"Wqkv": _dev(w), "Wo": _dev(w[:H, :H]), "attn_norm": _dev(attn_norm),
                          "q_norm": _dev(qn), "k_norm": _dev(kn)})
    st = _status()
    q = tg.tg_qkv_rope_cache(_dev(x), L.Wqkv, _dev(pos), cs, ck, cv, Hq, Hkv,
                             row_ssq=_dev(_ssq_rows(x, H)), q_norm_w=L.q_norm, k_norm_w=L.k_norm,
                             status=st)
    assert tg.tg_status_read(st) == 0
    w_folded = (w.float() * attn_norm).to(torch.bfloat16)
    _, _, _, parts = O.gated_layer(x, w_folded, w[:H, :H], np.zeros(Hq), 1.0, [0, M], pos,
                                   np.zeros(M), Hq, Hkv, d, 1.0e6, q_norm=qn, k_norm=kn)
    for got, want in ((q, parts["q"]), (ck, parts["k"]), (cv, parts["v"])):
        want = want.reshape(M, -1)
        err = np.abs(_f64(got.cpu()) - want)
        assert np.all(err <= 2.0 ** -7 * np.abs(want) + 2e-3), err.max()


@pytest.mark.parametrize("M", [1, 300, 1638, 4000])
def test_swiglu_against_oracle(tg, M):
    H, F_ = 2048, 6144
    x = S.uniform_rows(M, H, seed=M + 90)
    g = torch.Generator().manual_seed(M + 91)
    nw = (0.8 + 0.4 * torch.rand(H, generator=g)).float()
    wg = (torch.randn((F_, H), generator=g) * 0.02).to(torch.bfloat16)
    wu = (torch.randn((F_, H), generator=g) * 0.02).to(torch.bfloat16)
    w_gu = tg.tg_pack_gate_up(_dev(wg), _dev(wu), _dev(nw))
    st = _status()
    h = tg.tg_swiglu(_dev(x), w_gu, _dev(_ssq_rows(x, H)), status=st)
    assert tg.tg_status_read(st) == 0
    # the oracle reads the folded bf16 weights the kernel reads (see the QK-norm test)
    b = O.rmsnorm_rows(x)
    want = (O.silu(b @ _f64((wg.float() * nw).to(torch.bfloat16)).T)
            * (b @ _f64((wu.float() * nw).to(torch.bfloat16)).T))
    err = np.abs(_f64(h.cpu()) - want)
    assert np.all(err <= 2.0 ** -7 * np.abs(want) + 2e-3), err.max()
    assert err.mean() <= 1e-3


# ------------------------------------------------------------------ attention backward
#
# The backward forms delta_r = dO_r . O_r from the forward's bf16 output O, the one
# rounding on its path that the float64 oracle does not make.  An oracle-only study
# (delta from bf16(O) against exact O, lengths [300], [1, 129, 700], [1638], 16 q / 8 kv
# heads, N(0, 1) inputs) moves d_bias by at most 0.0026 max|d_bias| (rms 0.0015 of its
# rms), d_gamma by 0.0045 max|d_gamma| and d_beta by 0.001 of its size.  Bounds: 3-4x.

def _bias_grad_case(tg, lengths, seed, beta=1.0, gamma_zero=False, with_beta=True):
    Hq, Hkv, d = 16, 8, 128
    q, k, v, pos, bias, gamma, cu = _attn_inputs(lengths, Hq, Hkv, seed)
    if gamma_zero:
        gamma = torch.zeros_like(gamma)
    d_o = (torch.randn(q.shape, generator=torch.Generator().manual_seed(seed + 1))
           ).to(torch.bfloat16)
    o, lse = _run_attention(tg, q, k, v, pos, bias, gamma, beta, cu, Hq, Hkv)
    st = _status()
    dg = torch.full((Hq,), float("nan"), device="cuda")
    dbeta = torch.full((1,), float("nan"), device="cuda") if with_beta else None
    db = tg.tg_gated_attention_bias_grad(_dev(q), _dev(k), _dev(v), _dev(o), _dev(d_o), _dev(lse),
                                         _dev(torch.from_numpy(cu)), cu, Hq, Hkv, _dev(pos),
                                         _dev(bias), _dev(gamma), beta, d_gamma=dg, d_beta=dbeta,
                                         status=st)
    assert tg.tg_status_read(st) == 0
    return (q, k, v, d_o, pos, bias, gamma, cu), db.cpu(), dg.cpu(), (
        dbeta.cpu() if with_beta else None)


def _check_bias_grad(inputs, db, dg, dbeta, beta):
    q, k, v, d_o, pos, bias, gamma, cu = inputs
    Kt = q.shape[0]
    want_b, want_g, want_beta = O.gated_attention_bias_grad(
        _f64(q).reshape(Kt, 16, 128), _f64(k).reshape(Kt, 8, 128), _f64(v).reshape(Kt, 8, 128),
        _f64(d_o).reshape(Kt, 16, 128), cu, pos, bias, gamma, beta)
    err = np.abs(_f64(db) - want_b)
    scale = np.abs(want_b).max()
    # absolute floor 1e-3: fp32 accumulation where the exact gradient vanishes (a
    # one-key row has P = 1 and dl = dP - delta = 0); the gradients here are O(10-100)
    assert err.max() <= 0.01 * scale + 1e-3, (err.max(), scale)
    assert err.mean() <= 0.004 * np.sqrt(np.mean(want_b ** 2)) + 1e-3, err.mean()
    eg = np.abs(_f64(dg) - want_g)
    assert eg.max() <= 0.015 * np.abs(want_g).max() + 1e-3, (eg.max(), np.abs(want_g).max())
    if dbeta is not None:
        assert abs(float(dbeta[0]) - want_beta) <= 0.01 * max(abs(want_beta),
                                                                np.abs(want_g).max()) + 1e-3, \
            (float(dbeta[0]), want_beta)


@pytest.mark.parametrize("lengths", [[1], [300], [1, 129, 700, 0, 257]])
def test_bias_grad_against_oracle(tg, lengths):
    inputs, db, dg, dbeta = _bias_grad_case(tg, lengths, seed=len(lengths) * 7 + lengths[0])
    _check_bias_grad(inputs, db, dg, dbeta, 1.0)


def test_bias_grad_kept_1638_and_beta(tg):
    """One request at the 16k workload's kept count, a non-unit temperature scale."""
    inputs, db, dg, dbeta = _bias_grad_case(tg, [1638], seed=5, beta=0.8)
    _check_bias_grad(inputs, db, dg, dbeta, 0.8)


def test_bias_grad_deterministic_and_gamma_zero(tg):
    _, db1, dg1, dbeta1 = _bias_grad_case(tg, [700, 333], seed=9)
    _, db2, dg2, dbeta2 = _bias_grad_case(tg, [700, 333], seed=9)
    assert torch.equal(db1, db2) and torch.equal(dg1, dg2) and torch.equal(dbeta1, dbeta2)
    _, db0, _, _ = _bias_grad_case(tg, [700, 333], seed=9, gamma_zero=True, with_beta=False)
    assert torch.count_nonzero(db0) == 0


# ------------------------------------------------------------------ scorer backward

def _scorer_bwd_case(tg, lengths, questions, budgets, seed=91, with_norm=True):
    """The scorer's parameter gradients from a drawn dL/d(kept_bias) on the oracle's own
    kept set (both are inputs of the backward), GPU against the float64 oracle."""
    wl = S.custom(lengths, questions, budgets, seeds=[seed + i for i in range(len(lengths))])
    h, gw, pr = S.hidden_rows(wl), S.gate_weights(wl), S.prunable_mask(wl)
    g = torch.Generator().manual_seed(seed)
    nw = (0.8 + 0.4 * torch.rand(wl.hidden, generator=g, dtype=torch.float64)).float()
    cu = np.array(wl.cu_seqlens(), dtype=np.int32)
    s_ref = O.gate_score(h, nw, gw["W1"], gw["w2"])
    z_ref, _ = O.sequence_rmsnorm(s_ref, cu, pr)
    ck = np.asarray(O.kept_counts(pr, cu, wl.budgets), dtype=np.int32)
    kept, _, _ = O.select_topk(z_ref.astype(np.float32), pr, cu, ck)
    kept = np.asarray(kept, dtype=np.int32)
    dkb = torch.randn(len(kept), generator=g, dtype=torch.float64).float()
    ref = O.gate_score_backward(h, nw if with_norm else None, gw["W1"], gw["w2"], cu, pr,
                                kept, dkb)
    st = _status()
    hd, w1, w2 = _dev(h), _dev(gw["W1"]), _dev(gw["w2"])
    cud, prd = _dev(torch.from_numpy(cu)), _dev(pr)
    nwd = _dev(nw) if with_norm else None
    s_gpu, _, _ = tg.tg_gate_score(hd, w1, w2, cud, cu, prd, norm_w=nwd, status=st)
    args = (hd, w1, w2, s_gpu, cud, cu, prd, _dev(torch.from_numpy(ck)), ck,
            _dev(torch.from_numpy(kept)), _dev(dkb))
    out = tg.tg_gate_score_backward(*args, norm_w=nwd, status=st)
    again = tg.tg_gate_score_backward(*args, norm_w=nwd, status=st)
    assert tg.tg_status_read(st) == 0
    return ref, out, again


@pytest.mark.parametrize("lengths,questions,budgets",
                         [([700, 1500, 333], [16, 64, 5], [100, 800, 300]),
                          ([1, 37, 900], [1, 0, 64], [1, 10, 80]),  # one-token request
                          ([1, 37, 900], [1, 0, 64], [1, 0, 64]),   # no prunable row kept
                          ([16384], [64], [1638])])
def test_gate_score_backward_against_oracle(tg, lengths, questions, budgets):
    """Bounds from tests/tolerance_study.py (scorer_bwd): the CUDA path's roundings (W1
    folded with the norm weight in bf16, r du rounded to bf16) alone move dW1, dnorm_w
    and dw2 by at most 2.4e-3 of their largest magnitude, mean 5e-4."""
    ref, out, again = _scorer_bwd_case(tg, lengths, questions, budgets)
    for name, got in zip(("ds", "dW1", "dw2", "dnorm_w"), out):
        want = ref[name]
        err = np.abs(got.cpu().double().numpy() - want)
        scale = np.abs(want).max() + 1e-12
        assert err.max() <= 1e-2 * scale and err.mean() <= 2e-3 * scale, \
            (name, err.max(), err.mean(), scale)
    for a, b in zip(out, again):  # fixed reduction orders: bit-reproducible
        assert torch.equal(a, b)


def test_gate_score_backward_without_norm_weight(tg):
    ref, out, _ = _scorer_bwd_case(tg, [300, 129], [5, 3], [60, 40], with_norm=False)
    assert out[3] is None
    for name, got in zip(("ds", "dW1", "dw2"), out[:3]):
        want = ref[name]
        err = np.abs(got.cpu().double().numpy() - want)
        assert err.max() <= 1e-2 * np.abs(want).max(), (name, err.max())


def test_rope_rows_copies_the_position_rows(tg):
    """tg_rope_rows is a transposed gather of tg_rope_table rows: bit-exact, and a
    position outside the table raises TG_STATUS_BOUNDS and takes row 0."""
    d, n = 128, 1000
    g = torch.Generator().manual_seed(5)
    pos = torch.sort(torch.randperm(8000, generator=g)[:n])[0].to(torch.int32)
    cs = tg.tg_rope_table(8000, d, 1.0e6)
    st = _status()
    rot = tg.tg_rope_rows(_dev(pos), cs, status=st)
    assert tg.tg_status_read(st) == 0
    want = cs.view(8000, d // 4, 4)[pos.long().cuda()].permute(1, 0, 2)
    assert torch.equal(rot, want)
    bad = pos.clone()
    bad[7] = 8000
    st = _status()
    rot = tg.tg_rope_rows(_dev(bad), cs, status=st)
    assert tg.tg_status_read(st) & 4  # TG_STATUS_BOUNDS
    assert torch.equal(rot[:, 7], cs.view(8000, d // 4, 4)[0])


@pytest.mark.parametrize("M", [1, 300, 1638])
def test_qkv_per_row_table_matches_positions(tg, M):
    """pos = NULL with the per-row table gives the same bits as (pos, table) on the
    CTA-pair kernel (row sums given), the one-CTA kernel (none), QK-norm, and the fused
    output projection + next QKV."""
    Hq, Hkv, d, H = 16, 8, 128, 2048
    x = _dev(S.uniform_rows(M, H, seed=M + 90))
    w = _dev(S.uniform_rows((Hq + 2 * Hkv) * d, H, seed=M + 91, scale=0.02))
    g = torch.Generator().manual_seed(M + 92)
    pos = _dev(torch.sort(torch.randperm(10 * M + 1, generator=g)[:M])[0].to(torch.int32))
    cs = tg.tg_rope_table(10 * M + 1, d, 1.0e6)
    rot = tg.tg_rope_rows(pos, cs)
    ssq = _dev(_ssq_rows(x.cpu(), H))
    qn = _dev((0.8 + 0.4 * torch.rand(d, generator=g)).float())
    kn = _dev((0.8 + 0.4 * torch.rand(d, generator=g)).float())

    def run(p, table, **kw):
        ck = torch.zeros((M, Hkv * d), dtype=torch.bfloat16, device="cuda")
        cv = torch.zeros_like(ck)
        st = _status()
        q = tg.tg_qkv_rope_cache(x, w, p, table, ck, cv, Hq, Hkv, status=st, **kw)
        assert tg.tg_status_read(st) == 0
        return q, ck, cv

    for kw in ({"row_ssq": ssq}, {}, {"row_ssq": ssq, "q_norm_w": qn, "k_norm_w": kn}):
        for a, b in zip(run(pos, cs, **kw), run(None, rot, **kw)):
            assert torch.equal(a, b)
    o = _dev(S.uniform_rows(M, Hq * d, seed=M + 93))
    wo = _dev(S.uniform_rows(H, Hq * d, seed=M + 94, scale=0.02))
    outs = []
    for p, table in ((pos, cs), (None, rot)):
        xx, ss = x.clone(), torch.empty((M, H // 128), device="cuda")
        ck = torch.zeros((M, Hkv * d), dtype=torch.bfloat16, device="cuda")
        cv = torch.zeros_like(ck)
        q = torch.empty((M, Hq * d), dtype=torch.bfloat16, device="cuda")
        ws = torch.zeros(max(16, tg.tg_out_proj_qkv_workspace_size(M)), dtype=torch.uint8,
                         device="cuda")
        tg.tg_out_proj_qkv_next(o, wo, xx, ss, w, p, table, ck, cv, Hq, Hkv, q, ws)
        outs.append((xx, q, ck, cv))
    for a, b in zip(*outs):
        assert torch.equal(a, b)
