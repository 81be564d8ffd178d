"""The C ABI library loads on the host and exports every symbol the header declares;
host-only logic (argument checks that return before any launch, kept-count planning)
is exercised without a GPU."""
import ctypes as C
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "tokengate.h")


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(tg_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from learned_token_pruning_scoring_b200 import _lib
    return _lib.load()


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert len(names) >= 14
    for n in names:
        assert hasattr(lib, n), n


def test_binding_covers_header(lib):
    from learned_token_pruning_scoring_b200 import _lib
    assert set(_declared()) == set(_lib.SIGNATURES)


def test_error_strings(lib):
    for code in range(0, -8, -1):
        s = lib.tg_error_string(code)
        assert s and s != b"unknown error"


def test_plan_kept_rules(lib):
    import learned_token_pruning_scoring_b200 as tg
    import oracle as O
    rng = np.random.default_rng(0)
    for _ in range(50):
        B = int(rng.integers(1, 6))
        lengths = rng.integers(0, 40, B)
        cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
        pr = (rng.random(int(cu[-1])) < 0.7).astype(np.uint8)
        nq = [int((pr[cu[b]:cu[b + 1]] == 0).sum()) for b in range(B)]
        budgets = rng.integers(-3, 50, B)
        got = tg.tg_plan_kept(cu, nq, budgets).numpy()
        assert np.array_equal(got, O.kept_counts(pr, cu, budgets))


def test_plan_kept_rejects_bad_layout(lib):
    import learned_token_pruning_scoring_b200 as tg
    with pytest.raises(tg.TokenGateError):
        tg.tg_plan_kept([0, 5, 3], [0, 0], [1, 1])        # decreasing cu_seqlens
    with pytest.raises(tg.TokenGateError):
        tg.tg_plan_kept([0, 5], [6], [1])                 # more questions than tokens


def test_host_side_argument_errors(lib):
    """Shape and argument errors return before any device work."""
    p = C.c_void_p(0x10000)  # never dereferenced: the calls fail their checks first
    cu = (C.c_int32 * 2)(0, 8)
    # attention: head_dim other than 128 is not implemented
    assert lib.tg_gated_attention(p, 2048, p, 1024, p, 1024, p, cu, 1, 16, 8, 64, p, p, p,
                                  1.0, p, 2048, None, None, 0, None, None) == -6
    # attention: odd GQA group
    assert lib.tg_gated_attention(p, 2048, p, 1024, p, 1024, p, cu, 1, 3, 3, 128, p, p, p,
                                  1.0, p, 2048, None, None, 0, None, None) == -6
    # attention: the temperature scale beta must be finite and non-negative
    for beta in (-0.5, float("nan"), float("inf")):
        assert lib.tg_gated_attention(p, 2048, p, 1024, p, 1024, p, cu, 1, 16, 8, 128, p, p, p,
                                      beta, p, 2048, None, None, 0, None, None) == -1
    # projections: N not a multiple of 128, K not a multiple of 64
    assert lib.tg_linear(p, 64, p, 64, p, 100, 4, 100, 64, 0, 0.0, None, 0, None, 0, None, 0,
                         None, None) == -6
    assert lib.tg_linear(p, 96, p, 96, p, 128, 4, 128, 96, 0, 0.0, None, 0, None, 0, None, 0,
                         None, None) == -6
    # scorer: width other than 256
    assert lib.tg_gate_score(p, 2048, 8, 2048, None, p, 128, p, 1e-6, p, cu, 1, 1e-6, p, p,
                             p, p, p, 1 << 20, None, None) == -6
    # selection: K_b > N_b
    ck = (C.c_int32 * 2)(0, 9)
    assert lib.tg_topk_compact(p, p, p, cu, p, ck, 1, p, p, p, None, None) == -1
    # gather: misaligned pointer
    assert lib.tg_gather_rope(C.c_void_p(0x10002), 64, 4, None, 4, 64, None, 0, 0, 128, None,
                              0, p, 64, None, 0, None, None) == -2
    # KV cache: slots beyond the cache
    assert lib.tg_kv_compact(p, 64, p, 64, 10, None, 10, 64, p, p, 64, 12, 5, None, None) == -1
    # workspace too small
    assert lib.tg_gate_score(p, 2048, 8, 2048, None, p, 256, p, 1e-6, p, cu, 1, 1e-6, p, p,
                             p, p, p, 16, None, None) == -4


def test_launch_overlap_switch(lib):
    """The overlap switch is host state only (no device needed)."""
    prev = lib.tg_get_launch_overlap()
    assert prev in (0, 1)
    assert lib.tg_set_launch_overlap(0) == 0 and lib.tg_get_launch_overlap() == 0
    assert lib.tg_set_launch_overlap(7) == 0 and lib.tg_get_launch_overlap() == 1
    lib.tg_set_launch_overlap(prev)


def test_prefetch_argument_checks(lib):
    """tg_prefetch_l2 rejects bad pointers on the host; zero bytes is a no-op."""
    assert lib.tg_prefetch_l2(None, 0, None) == 0
    assert lib.tg_prefetch_l2(C.c_void_p(0x10000), 0, None) == 0
    assert lib.tg_prefetch_l2(None, 4096, None) == -1
    assert lib.tg_prefetch_l2(C.c_void_p(0x10004), 4096, None) == -2


def test_out_proj_qkv_argument_checks(lib):
    """The layer-boundary launch needs 256-multiple widths and its counter workspace."""
    p = C.c_void_p(0x10000)

    def call(hidden, ws, ws_bytes):
        return lib.tg_out_proj_qkv_next(p, 2048, p, 2048, p, hidden, p, 16, 8, hidden, 2048, p,
                                        hidden, 16, 8, 128, 1e-6, p, p, 100, p, 2048, p, p,
                                        1024, 0, ws, ws_bytes, None, None)
    assert call(1920, p, 64) == -6
    assert call(2048, None, 0) == -4
    assert call(2048, p, 4) == -4
    assert lib.tg_out_proj_qkv_workspace_size(0) == 0
    assert lib.tg_out_proj_qkv_workspace_size(257) == 16


def test_full_body_argument_checks(lib):
    """QK-norm needs both weights and the row sums of squares; the SwiGLU GEMM needs
    128-multiple widths and the row sums of squares; the weight packers check shapes."""
    p = C.c_void_p(0x10000)

    def qkn(qw, kw, ssq):
        return lib.tg_qkv_qknorm_rope_cache(p, 2048, p, 2048, 16, 2048, 16, 8, 128, 1e-6, qw,
                                            kw, p, p, 100, p, 2048, p, p, 1024, 0, ssq, 16,
                                            None, 0, None, None)
    assert qkn(None, p, p) == -1
    assert qkn(p, None, p) == -1
    assert qkn(p, p, None) == -1

    def swi(hidden, ffn, ssq, ld_ssq=16):
        return lib.tg_swiglu(p, hidden, p, hidden, 16, hidden, ffn, 1e-6, ssq, ld_ssq, p, ffn,
                             None, None)
    assert swi(2048, 6000, p) == -6   # ffn not a multiple of 128
    assert swi(2000, 6144, p) == -6   # hidden not a multiple of 128
    assert swi(2048, 6144, None) == -1
    assert swi(2048, 6144, p, ld_ssq=8) == -1
    assert lib.tg_swiglu(p, 2048, p, 2048, 0, 2048, 6144, 1e-6, p, 16, p, 6144, None,
                         None) == 0  # nothing to do
    assert lib.tg_pack_gate_up(p, 2048, p, 2048, 100, 2048, None, p, 2048, None) == -6
    assert lib.tg_pack_gate_up(p, 2048, None, 2048, 128, 2048, None, p, 2048, None) == -1
    assert lib.tg_fold_norm_weight(p, 2048, 16, 2048, None, p, 2048, None) == -1
    assert lib.tg_fold_norm_weight(p, 2048, 0, 2048, p, p, 2048, None) == 0


def test_bias_grad_argument_checks(lib):
    p = C.c_void_p(0x10000)
    ck = (C.c_int32 * 2)(0, 300)

    def call(beta=1.0, ws=p, ws_bytes=1 << 30, d_bias=p, head_dim=128, hq=16):
        return lib.tg_gated_attention_bias_grad(p, 2048, p, 1024, p, 1024, p, 2048, p, 2048, p, p,
                                                ck, 1, hq, 8, head_dim, p, p, p, beta, d_bias,
                                                None, None, ws, ws_bytes, None, None)
    assert call(head_dim=64) == -6
    assert call(hq=24) == -6          # odd group of q heads per kv head
    assert call(hq=12) == -1          # not a multiple of the kv heads
    assert call(beta=-1.0) == -1
    assert call(d_bias=None) == -1
    assert lib.tg_gated_attention_bias_grad_workspace_size(ck, 1, 16, 8, 64) == 0


def test_scorer_backward_argument_checks(lib):
    p = C.c_void_p(0x10000)
    cu = (C.c_int32 * 3)(0, 300, 500)
    ck = (C.c_int32 * 3)(0, 30, 50)

    def call(hidden=2048, width=256, cu_h=cu, ck_h=ck, batch=2, T=500, dW1=p, dw2=p,
             eps=1e-6):
        return lib.tg_gate_score_backward(p, hidden, T, hidden, None, p, width, p, eps, p, p,
                                          cu_h, batch, 1e-6, p, p, ck_h, p, p, p, dW1, None,
                                          dw2, p, 1 << 30, None, None)
    assert call(width=128) == -6
    assert call(hidden=2112) == -6                          # not a multiple of 128
    assert call(T=499) == -1                                # cu_seqlens[batch] != T
    assert call(ck_h=(C.c_int32 * 3)(0, 301, 320)) == -1    # K_0 > N_0
    assert call(ck_h=(C.c_int32 * 3)(0, 30, 20)) == -1      # decreasing
    assert call(cu_h=None) == -1
    assert call(eps=-1.0) == -1
    assert call(dW1=None) == -1 and call(dw2=None) == -1
    assert call(batch=0, T=5) == -1
    assert lib.tg_gate_score_backward_workspace_size(500, 2048, 128, 2) == 0
    small = lib.tg_gate_score_backward_workspace_size(500, 2048, 256, 2)
    big = lib.tg_gate_score_backward_workspace_size(50000, 2048, 256, 2)
    # du' alone is 512 bytes per token
    assert small > 500 * 512 and big - small >= (50000 - 500) * 512


def test_attention_split_plan(lib):
    # The split plan is host logic: tg_gated_attention_workspace_size is the number of
    # work items times the per-item bytes (partials of every q head, counter and flag
    # per head group), 0 when no query tile is split.
    def items(lengths, hq, hkv):
        cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
        ws = lib.tg_gated_attention_workspace_size(cu.ctypes.data_as(C.c_void_p), len(lengths),
                                                   hq, hkv, 128)
        return ws // (hq * (128 * 128 + 2 * 128) * 4 + 8 * (hq // 2))

    def chunk_of(lengths, n_items):
        tiles = [-(-n // 128) for n in lengths]
        return [c for c in range(1, max(tiles) + 1)
                if sum(-(-(qt + 1) // c) for t in tiles for qt in range(t)) == n_items]

    # 16 q / 8 kv heads, one 1638-row request: the six heaviest query tiles in two parts
    n = items([1638], 16, 8)
    assert n == 19 and chunk_of([1638], n) == [7]
    # long single requests and the eight-request ragged batch balance without splitting
    assert items([13107], 16, 8) == 0
    assert items([8192], 16, 8) == 0
    assert items([1638, 819, 410, 1229, 205, 1024, 614, 1433], 16, 8) == 0
    # one head group: most tiles split, the longest into six parts
    n = items([2000], 2, 1)
    assert chunk_of([2000], n) == [3]


def test_rope_rows_argument_checks(lib):
    p = C.c_void_p(0x10000)
    # per-row table: row stride below the row count; head_dim not a multiple of 4
    assert lib.tg_rope_rows(p, 10, p, 100, 128, p, 9, None, None) == -1
    assert lib.tg_rope_rows(p, 10, p, 100, 126, p, 10, None, None) == -6
    assert lib.tg_rope_rows(p, 10, C.c_void_p(0x10004), 100, 128, p, 10, None, None) == -2
    assert lib.tg_rope_rows(p, 0, p, 100, 128, p, 0, None, None) == 0
    # QKV with pos = NULL reads a per-row table whose row stride (max_pos) must cover M
    assert lib.tg_qkv_rope_cache(p, 2048, p, 2048, 300, 2048, 16, 8, 128, 1e-6, None, p, 299,
                                 p, 2048, p, p, 1024, 0, p, 16, None, 0, None, None) == -1
