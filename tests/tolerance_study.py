"""Tolerance derivation for the multi-layer end-to-end check (CPU only, not collected).

Runs the oracle's gated layers twice from the same seeded inputs: once in float64,
once with bf16 rounding at the points where the CUDA path rounds (q, k, v after the
projection and after RoPE, the attention output O, the residual stream x).  The gap
between the two is the error a correct bf16 implementation is expected to show; the
end-to-end test's bounds are set above it.  Usage: python tests/tolerance_study.py
"""
import os
import sys

import numpy as np
import torch

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import oracle as O  # noqa: E402
import synthetic_inputs as S  # noqa: E402


def bf16(x):
    return (torch.from_numpy(np.ascontiguousarray(x)).to(torch.float32)
            .to(torch.bfloat16).to(torch.float64).numpy())


def layer_rounded(x, L, cu_kept, pos, bias, wl):
    hq, hkv, d = wl.n_q_heads, wl.n_kv_heads, wl.head_dim
    Kt = x.shape[0]
    qkv = bf16(O.rmsnorm_rows(x) @ O.as_f64(L["Wqkv"]).T)
    q = bf16(O.rope(qkv[:, :hq * d].reshape(Kt, hq, d), pos, wl.rope_theta))
    k = bf16(O.rope(qkv[:, hq * d:(hq + hkv) * d].reshape(Kt, hkv, d), pos, wl.rope_theta))
    v = qkv[:, (hq + hkv) * d:].reshape(Kt, hkv, d)
    o, _ = O.gated_attention(q, k, v, cu_kept, pos, bias, L["gamma"], L["beta"])
    return bf16(x + bf16(o.reshape(Kt, -1)) @ O.as_f64(L["Wo"]).T)


def study(wl, report=(1, 2, 4, 8, 16, 28)):
    h, pr, gate = S.hidden_rows(wl), S.prunable_mask(wl), S.gate_weights(wl)
    ref = O.prefill(h, pr, wl.cu_seqlens(), wl.budgets, gate, [], wl.n_q_heads,
                    wl.n_kv_heads, wl.head_dim, wl.rope_theta)
    ck, pos, kb = ref["cu_kept"], ref["kept_pos"], ref["kept_bias"]
    x64 = O.gather_rows(h, ref["kept_idx"])
    xr = x64.copy()
    for i in range(wl.n_layers):
        L = S.layer_weights(wl, i)
        x64, *_ = O.gated_layer(x64, L["Wqkv"], L["Wo"], L["gamma"], L["beta"], ck, pos, kb,
                                wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.rope_theta)
        xr = layer_rounded(xr, L, ck, pos, kb, wl)
        if i + 1 in report or i + 1 == wl.n_layers:
            e = np.abs(xr - x64)
            print(f"{wl.name} layer {i + 1}: max {e.max():.4f} mean {e.mean():.5f} "
                  f"|x|max {np.abs(x64).max():.2f}", flush=True)


def study_lower(wl, n_lower):
    """Layers below the gate, float64 against bf16-rounded, and what that does to the
    gate's scores s and z read from their output."""
    h, pr, gate = S.hidden_rows(wl), S.prunable_mask(wl), S.gate_weights(wl)
    cu = wl.cu_seqlens()
    pos = O.request_positions(cu)
    zero_bias = np.zeros(wl.total_tokens)
    x64 = O.as_f64(h)
    xr = x64.copy()
    for L in S.lower_layer_weights(wl, n_lower):
        x64, _, _ = O.full_context_layer(x64, L["Wqkv"], L["Wo"], cu, wl.n_q_heads,
                                         wl.n_kv_heads, wl.head_dim, wl.rope_theta)
        Lg = dict(L, gamma=np.zeros(wl.n_q_heads), beta=1.0)
        xr = layer_rounded(xr, Lg, cu, pos, zero_bias, wl)
    e = np.abs(xr - x64)
    s64 = O.gate_score(x64, gate["norm_w"], gate["W1"], gate["w2"])
    sr = O.gate_score(xr, gate["norm_w"], gate["W1"], gate["w2"])
    z64, _ = O.sequence_rmsnorm(s64, cu, pr)
    zr, _ = O.sequence_rmsnorm(sr, cu, pr)
    print(f"{wl.name} {n_lower} lower layers: x max {e.max():.4f} mean {e.mean():.5f}; "
          f"s max {np.abs(sr - s64).max():.5f} mean {np.abs(sr - s64).mean():.6f}; "
          f"z max {np.abs(zr - z64).max():.5f} mean {np.abs(zr - z64).mean():.6f}", flush=True)


def layer_rounded_full(x, L, body, cu_kept, pos, bias, wl):
    """A full layer body with bf16 rounding where the CUDA path rounds: the folded norm
    weights (Wqkv * attn_norm, W_gate/W_up * mlp norm), q/k after QK-norm and RoPE, v,
    O, the residual after attention, the SwiGLU output and the residual after the MLP."""
    hq, hkv, d = wl.n_q_heads, wl.n_kv_heads, wl.head_dim
    Kt = x.shape[0]
    m = body["mlp"]
    wqkv = bf16(O.as_f64(L["Wqkv"]) * O.as_f64(body["attn_norm"])[None, :])
    qkv = O.rmsnorm_rows(x) @ wqkv.T
    q = O.rmsnorm_heads(qkv[:, :hq * d].reshape(Kt, hq, d), body["q_norm"])
    k = O.rmsnorm_heads(qkv[:, hq * d:(hq + hkv) * d].reshape(Kt, hkv, d), body["k_norm"])
    q = bf16(O.rope(q, pos, wl.rope_theta))
    k = bf16(O.rope(k, pos, wl.rope_theta))
    v = bf16(qkv[:, (hq + hkv) * d:].reshape(Kt, hkv, d))
    o, _ = O.gated_attention(q, k, v, cu_kept, pos, bias, L["gamma"], L["beta"])
    x = bf16(x + bf16(o.reshape(Kt, -1)) @ O.as_f64(L["Wo"]).T)
    nw = O.as_f64(m["norm_w"])[None, :]
    b = O.rmsnorm_rows(x)
    hmid = bf16(O.silu(b @ bf16(O.as_f64(m["W_gate"]) * nw).T)
                * (b @ bf16(O.as_f64(m["W_up"]) * nw).T))
    return bf16(x + hmid @ O.as_f64(m["W_down"]).T)


def study_full(wl, n_layers):
    """Full layer bodies above the gate (QK-norm, weighted norms, SwiGLU MLP)."""
    h, pr, gate = S.hidden_rows(wl), S.prunable_mask(wl), S.gate_weights(wl)
    ref = O.prefill(h, pr, wl.cu_seqlens(), wl.budgets, gate, [], wl.n_q_heads,
                    wl.n_kv_heads, wl.head_dim, wl.rope_theta)
    ck, pos, kb = ref["cu_kept"], ref["kept_pos"], ref["kept_bias"]
    x64 = O.gather_rows(h, ref["kept_idx"])
    xr = x64.copy()
    for i in range(n_layers):
        L = S.layer_weights(wl, i)
        body = S.layer_body_parts(wl, i)
        x64, *_ = O.gated_layer(x64, L["Wqkv"], L["Wo"], L["gamma"], L["beta"], ck, pos, kb,
                                wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.rope_theta,
                                **body)
        xr = layer_rounded_full(xr, L, body, ck, pos, kb, wl)
        e = np.abs(xr - x64)
        print(f"{wl.name} full layer {i + 1}: max {e.max():.4f} mean {e.mean():.5f} "
              f"|x|max {np.abs(x64).max():.2f}", flush=True)


def study_scorer_backward(wl, seed=91):
    """Scorer parameter gradients, float64 against the CUDA path's rounding: W1 folded
    with the norm weight and rounded to bf16 for the recomputed u, and the row-scaled
    du rounded to bf16 before it meets h in the weight-gradient GEMM."""
    h, pr, gate = S.hidden_rows(wl), S.prunable_mask(wl), S.gate_weights(wl)
    g = torch.Generator().manual_seed(seed)
    nw = (0.8 + 0.4 * torch.rand(wl.hidden, generator=g, dtype=torch.float64)).numpy()
    cu = wl.cu_seqlens()
    W1, w2 = O.as_f64(gate["W1"]), O.as_f64(gate["w2"])
    s = O.gate_score(h, nw, W1, w2)
    z, _ = O.sequence_rmsnorm(s, cu, pr)
    ck = O.kept_counts(pr, cu, wl.budgets)
    kept, _, _ = O.select_topk(z.astype(np.float32), pr, cu, ck)
    dkb = torch.randn(len(kept), generator=g, dtype=torch.float64).numpy()
    ref = O.gate_score_backward(h, nw, W1, w2, cu, pr, kept, dkb)
    hh = O.as_f64(h)
    r = 1.0 / np.sqrt(np.mean(hh * hh, axis=1) + 1e-6)
    u = (hh @ bf16(W1 * nw[None, :]).T) * r[:, None]
    sig = 1.0 / (1.0 + np.exp(-u))
    du = bf16(r[:, None] * ref["ds"][:, None] * w2[None, :] * sig * (1.0 + u * (1.0 - sig)))
    M = hh.T @ du                                   # [H, F]
    got = {"dW1": (M * nw[:, None]).T, "dnorm_w": np.sum(W1.T * M, axis=1),
           "dw2": (u * sig).T @ ref["ds"]}
    for k, v in got.items():
        e = np.abs(v - ref[k])
        scale = np.abs(ref[k]).max()
        print(f"{wl.name} {k}: max {e.max():.3e} mean {e.mean():.3e} |ref|max {scale:.3e} "
              f"max/|ref|max {e.max() / scale:.3e}", flush=True)


if __name__ == "__main__":
    if len(sys.argv) > 1 and sys.argv[1] == "full":
        study_full(S.custom([700, 1500, 333], [16, 64, 5], [100, 800, 300], n_layers=2,
                            name="ragged3"), 2)
        sys.exit(0)
    if len(sys.argv) > 1 and sys.argv[1] == "scorer_bwd":
        study_scorer_backward(S.custom([700, 1500, 333], [16, 64, 5], [100, 800, 300],
                                       name="ragged3"))
        study_scorer_backward(S.n16k())
        sys.exit(0)
    if len(sys.argv) > 1 and sys.argv[1] == "lower":
        study_lower(S.custom([700, 1500, 333], [16, 64, 5], [100, 800, 300], n_layers=1,
                             name="ragged3"), 2)
        sys.exit(0)
    study(S.custom([700, 1500, 333], [16, 64, 5], [100, 800, 300], n_layers=2, name="ragged3"))
    study(S.n16k())
