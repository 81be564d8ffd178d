"""tg_gate_score_noalloc: gate scoring for callers that may not allocate device memory.

A serving engine that plans all device memory ahead, or a plug-in limited to the
buffers its host framework hands it, cannot give tg_gate_score a workspace it had to
allocate.  The no-allocation entry point takes its scratch from a fixed array inside
the library instead.  These tests call it through the C ABI and check that it gives
the same results as the workspace entry point on two calls in a row with different
shapes, so the second call runs on scratch that still holds the first call's contents.
Both entry points launch the same kernels with the same reduction order, so the
results must agree bit for bit.  Collected last on purpose.
"""
import numpy as np
import pytest
import torch

import synthetic_inputs as S

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def _inputs(lengths, questions, seed, random_norm_weight):
    wl = S.custom(lengths, questions, [0] * len(lengths),
                  seeds=[seed + i for i in range(len(lengths))])
    h = S.hidden_rows(wl).cuda()
    gw = S.gate_weights(wl)
    if random_norm_weight:
        gw["norm_w"] = (0.5 + torch.rand(wl.hidden, generator=torch.Generator().manual_seed(seed)))
    gw = {k: v.to(torch.float32 if k != "W1" else torch.bfloat16).cuda() for k, v in gw.items()}
    pr = S.prunable_mask(wl).cuda()
    cu = np.array(wl.cu_seqlens(), dtype=np.int32)
    return h, gw, pr, cu


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    import learned_token_pruning_scoring_b200 as tg
    cases = [([3000, 1200, 77], [64, 16, 5], 0, True),   # larger first call
             ([1000], [64], 5, False)]                    # then a smaller one on reused scratch
    for lengths, questions, seed, rnw in cases:
        h, gw, pr, cu = _inputs(lengths, questions, seed, rnw)
        cu_d = torch.from_numpy(cu).cuda()
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        ref = tg.tg_gate_score(h, gw["W1"], gw["w2"], cu_d, cu, pr, norm_w=gw["norm_w"], status=st)
        got = tg.tg_gate_score_noalloc(h, gw["W1"], gw["w2"], cu_d, cu, pr, norm_w=gw["norm_w"],
                                       status=st)
        torch.cuda.synchronize()
        assert tg.tg_status_read(st) == 0
        for name, a, b in zip(("s", "z", "bias"), got, ref):
            assert torch.equal(a, b), name
        assert torch.all(got[2][pr == 0] == 0)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    import ctypes as C

    import learned_token_pruning_scoring_b200 as tg
    lib = tg.lib
    p = C.c_void_p(0x10000)  # never dereferenced: the size check fails first
    cu = (C.c_int32 * 2)(0, (1 << 20) + 1)
    rc = lib.tg_gate_score_noalloc(p, 2048, (1 << 20) + 1, 2048, None, p, 256, p, 1e-6, p, cu,
                                   1, 1e-6, p, p, p, p, None, None)
    assert rc == -7 and b"scratch" in lib.tg_error_string(rc)
    rc = lib.tg_gate_score_noalloc(p, 8192, 8, 8192, None, p, 256, p, 1e-6, p, cu, 1, 1e-6, p, p,
                                   p, p, None, None)
    assert rc == -7
    # a scorer width the kernels do not take is a shape error, as for tg_gate_score
    rc = lib.tg_gate_score_noalloc(p, 2048, 8, 2048, None, p, 512, p, 1e-6, p, cu, 1, 1e-6, p, p,
                                   p, p, None, None)
    assert rc == -6 and rc == lib.tg_gate_score(p, 2048, 8, 2048, None, p, 512, p, 1e-6, p, cu, 1,
                                                1e-6, p, p, p, p, p, 1 << 20, None, None)
