"""Plain float64 CPU oracle of the TokenGate hot path (test infrastructure only).

Sources, cited below by tag (page title, then the section or figure used):
  [fluxbbs]    "TokenGate 长上下文预填充提速 11.3 倍，斯坦福伯克利开源门控剪枝"
  [digest]     "TokenGate: Adapting LLMs for Fast and Memory-Efficient Prefill with
                Learned Token Pruning" (paper digest)
  [farwalk]    "斯坦福与 UC Berkeley 提出 TokenGate：token 门控注意力让长上下文预填充最高快 11.3 倍"
  [aiwillknow] "TokenGate：让模型学会跳读，而不只压缩 KV 缓存"

What the pages fix, and what this oracle reads into the gaps (each reading is also
listed with its reason in the design notes of the repository):
  * gate at layer L: RMSNorm of the post-attention residual, a small scoring MLP
    giving one scalar per token ([fluxbbs] 门控到底插在模型的哪个位置; [digest]
    方法关键点; [farwalk] How does TokenGate learned token pruning work?).
    Reading: MLP 2048 -> 256 -> 1, SiLU, no biases; RMSNorm eps 1e-6.
  * scores RMSNorm-normalised along the sequence ([fluxbbs] same section).
    Reading: the RMS runs over all tokens of the request, no gain, eps 1e-6.
  * top-K over prunable (document) tokens only; question tokens are always kept
    ([farwalk] same section; [digest] 方法关键点).  Reading: order "larger score
    first, equal scores -> lower index first", NaN below every number, -0 == +0;
    the budget counts every kept token, question included.
  * kept tokens keep their original positions ([aiwillknow] 图1(a)(b)).
  * token-gated attention: the kept token's score enters the upper layers' logits as
    a per-key bias with a learnable per-head gain, plus an SSMax-style temperature
    that rescales by the log-ratio of kept rank to original position ([fluxbbs]
    端到端训练的关键在 token 门控注意力; [farwalk] What is token-gated attention?;
    [aiwillknow] 图1(c)).  The formula adopted by this library:
        logit[r, c] = tau_r * (q_r . k_c) / sqrt(d) + gamma_h * z_c     (c <= r)
        tau_r       = beta * ln(r + 1) / ln(p_r + 1),   tau_r = beta when p_r = 0
    with r the query's 0-based rank in the kept list, p_r its original position and
    z_c = 0 for non-prunable keys.
  * upper layers keep KV only for kept tokens ([farwalk] How does TokenGate learned
    token pruning work?; [digest] 方法关键点).
  * a full transformer layer body (optional, both below and above the gate): the
    Qwen3-shaped layer the pages evaluate on adds a weighted pre-attention RMSNorm,
    per-head RMSNorm of q and k before RoPE (QK-norm) and a SwiGLU MLP behind its own
    weighted RMSNorm; the pages say pruned tokens skip the upper MLPs too ([fluxbbs]
    门控到底插在模型的哪个位置).  Reading: eps 1e-6 everywhere, QK-norm weight shared by
    the heads, MLP x + W_down (SiLU(W_gate b) * W_up b) with b the normalised x.
  * layers below the gate see every token with ordinary causal attention; their KV
    may optionally be trimmed to the kept tokens as well ([digest] 方法关键点;
    [aiwillknow] 图1(a)(b)).  Reading: trimming keeps exactly the gate's kept rows.
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "as_f64", "rmsnorm_rows", "gate_score", "sequence_rmsnorm", "kept_counts",
    "select_topk", "gather_rows", "rope", "rope_angles", "temperature",
    "gated_attention", "kv_compact", "gated_layer", "prefill", "silu",
    "request_positions", "causal_attention", "full_context_layer",
    "rmsnorm_heads", "swiglu_mlp", "gated_attention_bias_grad", "gate_score_backward",
]


def as_f64(x) -> np.ndarray:
    """Any torch tensor / array (bf16 included) as a float64 NumPy array, exactly."""
    if hasattr(x, "detach"):
        import torch  # local: the oracle itself needs only NumPy
        x = x.detach().to("cpu")
        if x.dtype in (torch.bfloat16, torch.float16):
            x = x.to(torch.float32)
        x = x.numpy()
    return np.asarray(x, dtype=np.float64)


def _as_int(x) -> np.ndarray:
    if hasattr(x, "detach"):
        x = x.detach().to("cpu").numpy()
    return np.asarray(x, dtype=np.int64)


def silu(u: np.ndarray) -> np.ndarray:
    """u * sigmoid(u), written so that large |u| neither overflows nor loses the sign."""
    out = np.empty_like(u)
    pos = u >= 0
    out[pos] = u[pos] / (1.0 + np.exp(-u[pos]))
    e = np.exp(u[~pos])
    out[~pos] = u[~pos] * e / (1.0 + e)
    return out


# ------------------------------------------------------------------ gate scoring

def rmsnorm_rows(x, weight=None, eps: float = 1e-6) -> np.ndarray:
    """x_t * w / sqrt(mean(x_t^2) + eps), row by row."""
    x = as_f64(x)
    inv = 1.0 / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    y = x * inv
    if weight is not None:
        y = y * as_f64(weight)
    return y


def gate_score(h, norm_w, W1, w2, eps: float = 1e-6) -> np.ndarray:
    """Per-token gate score s_t = w2 . SiLU(W1 RMSNorm(h_t)).

    [fluxbbs] 门控到底插在模型的哪个位置: a small MLP reads each token's normalised
    residual and gives one scalar; [digest] 方法关键点 and [farwalk] How does TokenGate
    learned token pruning work?: the residual is the post-attention residual at L.
    W1 is stored [F, H] (output rows), w2 is [F].
    """
    x = rmsnorm_rows(h, norm_w, eps)
    u = x @ as_f64(W1).T
    return silu(u) @ as_f64(w2)


def sequence_rmsnorm(s, cu_seqlens, prunable, eps: float = 1e-6):
    """z_t = s_t / sqrt(mean_{t' in request} s_t'^2 + eps); bias_t = z_t on prunable tokens, else 0.

    [fluxbbs] 门控到底插在模型的哪个位置: the scores are RMSNorm-normalised along the
    sequence.  The mean runs over every token of the request.
    """
    s = as_f64(s)
    cu = _as_int(cu_seqlens)
    pr = _as_int(prunable).astype(bool)
    z = np.empty_like(s)
    for b in range(len(cu) - 1):
        lo, hi = cu[b], cu[b + 1]
        seg = s[lo:hi]
        rms = math.sqrt(float(np.mean(seg * seg)) + eps) if hi > lo else 1.0
        z[lo:hi] = seg / rms
    bias = np.where(pr, z, 0.0)
    return z, bias


# ------------------------------------------------------------------ selection

def kept_counts(prunable, cu_seqlens, budgets) -> np.ndarray:
    """cu_kept from per-request budgets: K_b = Q_b + min(D_b, max(0, budget_b - Q_b)).

    [farwalk] How do you deploy TokenGate?: the user gives a budget of kept prefill
    tokens; [farwalk] How does TokenGate learned token pruning work?: the question
    is never pruned.  The budget is read as counting every kept token.
    """
    cu = _as_int(cu_seqlens)
    pr = _as_int(prunable).astype(bool)
    out = [0]
    for b in range(len(cu) - 1):
        seg = pr[cu[b]:cu[b + 1]]
        d = int(seg.sum())
        q = int(seg.size - d)
        kd = min(d, max(0, int(budgets[b]) - q))
        out.append(out[-1] + q + kd)
    return np.asarray(out, dtype=np.int64)


def _selection_order(values: np.ndarray, index: np.ndarray) -> np.ndarray:
    """Indices of `values` sorted by: numbers before NaN, larger first, lower index first."""
    isnan = np.isnan(values)
    neg = np.where(isnan, 0.0, -(values.astype(np.float64) + 0.0))  # + 0.0 maps -0 to +0
    return np.lexsort((index, neg, isnan))


def select_topk(z, prunable, cu_seqlens, cu_kept):
    """Prunable-only top-K with the question kept, listed in original order.

    For each request: among prunable tokens keep the Kd_b = K_b - Q_b best under the
    order of `_selection_order`, add every non-prunable token, and list the kept
    tokens by ascending position.  Decisions are taken on the float32 values given.
    Returns (kept_idx [packed row id], kept_pos [position in request],
    kept_bias [z on prunable rows, 0 on question rows]) with float32 bias.
    [fluxbbs] 门控到底插在模型的哪个位置 (top-K, question never pruned);
    [aiwillknow] 图1(a)(b) (original positions kept).
    """
    z32 = np.asarray(as_f64(z), dtype=np.float32) if not (
        isinstance(z, np.ndarray) and z.dtype == np.float32) else z
    cu = _as_int(cu_seqlens)
    ck = _as_int(cu_kept)
    pr = _as_int(prunable).astype(bool)
    idx_out, pos_out, bias_out = [], [], []
    for b in range(len(cu) - 1):
        lo, hi = cu[b], cu[b + 1]
        seg_z = z32[lo:hi]
        seg_p = pr[lo:hi]
        cand = np.nonzero(seg_p)[0]
        keep_q = np.nonzero(~seg_p)[0]
        kd = int(ck[b + 1] - ck[b]) - keep_q.size
        if kd < 0 or kd > cand.size:
            raise ValueError(f"request {b}: kept count {ck[b + 1] - ck[b]} inconsistent with mask")
        order = _selection_order(seg_z[cand], cand)
        chosen = cand[order[:kd]]
        kept = np.sort(np.concatenate([chosen, keep_q]))
        idx_out.append(lo + kept)
        pos_out.append(kept)
        bias_out.append(np.where(seg_p[kept], seg_z[kept], np.float32(0.0)).astype(np.float32))
    cat = (lambda xs, dt: np.concatenate(xs).astype(dt) if xs else np.zeros(0, dt))
    return cat(idx_out, np.int64), cat(pos_out, np.int64), cat(bias_out, np.float32)


def gather_rows(h, idx) -> np.ndarray:
    """Rows of h at the kept indices: pruned rows stop at the gate
    ([fluxbbs] 门控到底插在模型的哪个位置)."""
    return as_f64(h)[_as_int(idx)]


# ------------------------------------------------------------------ RoPE, temperature

def rope_angles(pos, head_dim: int, theta: float) -> np.ndarray:
    """angle[r, i] = p_r * theta^(-2 i / head_dim), i < head_dim / 2, in float64."""
    pos = _as_int(pos).astype(np.float64)
    i = np.arange(head_dim // 2, dtype=np.float64)
    inv_freq = theta ** (-2.0 * i / head_dim)
    return pos[:, None] * inv_freq[None, :]


def rope(x, pos, theta: float = 1.0e6) -> np.ndarray:
    """Rotate-half rotary embedding of x [rows, heads, d] at positions pos [rows].

    Pairs (i, i + d/2) rotate by angle p * theta^(-2i/d).  The kept rows use their
    original positions ([aiwillknow] 图1(a)(b))."""
    x = as_f64(x)
    d = x.shape[-1]
    half = d // 2
    ang = rope_angles(pos, d, theta)[:, None, :]
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def temperature(rank, pos, beta: float) -> np.ndarray:
    """tau = beta * ln(r + 1) / ln(p + 1); tau = beta where p = 0 (the limit r = p).

    [fluxbbs] 端到端训练的关键在 token 门控注意力: a learnable temperature scaled by the
    log-ratio of kept count to original position, after SSMax."""
    r = _as_int(rank).astype(np.float64)
    p = _as_int(pos).astype(np.float64)
    out = np.full(r.shape, float(beta))
    nz = p > 0
    out[nz] = beta * np.log(r[nz] + 1.0) / np.log(p[nz] + 1.0)
    return out


# ------------------------------------------------------------------ attention

def gated_attention(Q, K, V, cu_kept, kept_pos, kept_bias, gamma, beta,
                    rows=None, block: int = 1024):
    """Causal GQA attention over the kept rows with key bias and temperature.

    Q [Kt, Hq, d], K/V [Kt, Hkv, d]; q head h reads kv head h // (Hq/Hkv).  Within
    each request (rows cu_kept[b]..cu_kept[b+1]) query rank r attends to key ranks
    c <= r with logits tau_r * q.k / sqrt(d) + gamma_h * bias_c, softmax over c.
    Returns O [Kt, Hq, d] and the natural-log LSE [Hq, Kt] (float64).  With `rows`
    (packed query row ids) only those rows are computed, others stay NaN.
    [fluxbbs] 端到端训练的关键在 token 门控注意力; [farwalk] What is token-gated
    attention?; [aiwillknow] 图1(c).
    """
    Q, K, V = as_f64(Q), as_f64(K), as_f64(V)
    ck = _as_int(cu_kept)
    pos = _as_int(kept_pos)
    bias = as_f64(kept_bias)
    gamma = as_f64(gamma)
    Kt, Hq, d = Q.shape
    Hkv = K.shape[1]
    grp = Hq // Hkv
    O = np.full(Q.shape, np.nan)
    lse = np.full((Hq, Kt), np.nan)
    want = None if rows is None else np.zeros(Kt, dtype=bool)
    if want is not None:
        want[_as_int(rows)] = True
    for b in range(len(ck) - 1):
        lo, hi = ck[b], ck[b + 1]
        n = hi - lo
        if n == 0:
            continue
        rank = np.arange(n)
        tau = temperature(rank, pos[lo:hi], beta)
        qsel = np.arange(n) if want is None else np.nonzero(want[lo:hi])[0]
        for start in range(0, qsel.size, block):
            qi = qsel[start:start + block]
            if qi.size == 0:
                continue
            kmax = int(qi.max()) + 1
            causal = np.arange(kmax)[None, :] <= qi[:, None]
            for h in range(Hq):
                g = h // grp
                S = Q[lo + qi, h, :] @ K[lo:lo + kmax, g, :].T
                logit = tau[qi, None] * S / math.sqrt(d) + gamma[h] * bias[None, lo:lo + kmax]
                logit = np.where(causal, logit, -np.inf)
                m = logit.max(axis=1, keepdims=True)
                e = np.exp(logit - m)
                den = e.sum(axis=1, keepdims=True)
                O[lo + qi, h, :] = (e / den) @ V[lo:lo + kmax, g, :]
                lse[h, lo + qi] = (m + np.log(den))[:, 0]
    return O, lse


def gated_attention_bias_grad(Q, K, V, dO, cu_kept, kept_pos, kept_bias, gamma, beta):
    """Gradients of a loss L through token-gated attention, given dL/dO, with respect to
    the key bias, the per-head gains and the temperature scale: what training the gate
    end to end needs ([fluxbbs] 端到端训练的关键在 token 门控注意力: the gate is trained
    through the attention it biases; [digest] 方法关键点).

    With l[r, c] = tau_r s[r, c] + gamma_h b_c, s = q.k / sqrt(d), P = softmax_c(l),
    O_r = sum_c P[r, c] v_c, the softmax Jacobian gives
        dl[r, c] = P[r, c] (dO_r.v_c - dO_r.O_r),
    and l is linear in b_c (slope gamma_h), gamma_h (slope b_c) and beta (slope
    (tau_r / beta) s[r, c], with tau_r / beta = ln(r + 1) / ln(p_r + 1), 1 at p_r = 0).
    Returns (d_bias [Kt], d_gamma [Hq], d_beta) in float64.
    """
    Q, K, V, dO = as_f64(Q), as_f64(K), as_f64(V), as_f64(dO)
    ck = _as_int(cu_kept)
    pos = _as_int(kept_pos)
    bias = as_f64(kept_bias)
    gamma = as_f64(gamma)
    Kt, Hq, d = Q.shape
    grp = Hq // K.shape[1]
    d_bias = np.zeros(Kt)
    d_gamma = np.zeros(Hq)
    d_beta = 0.0
    for b in range(len(ck) - 1):
        lo, hi = ck[b], ck[b + 1]
        n = hi - lo
        if n == 0:
            continue
        rank = np.arange(n)
        rho = temperature(rank, pos[lo:hi], 1.0)  # tau / beta
        causal = np.arange(n)[None, :] <= np.arange(n)[:, None]
        for h in range(Hq):
            g = h // grp
            s = Q[lo:hi, h, :] @ K[lo:hi, g, :].T / math.sqrt(d)
            logit = np.where(causal, beta * rho[:, None] * s + gamma[h] * bias[None, lo:hi],
                             -np.inf)
            P = np.exp(logit - logit.max(axis=1, keepdims=True))
            P /= P.sum(axis=1, keepdims=True)
            O = P @ V[lo:hi, g, :]
            dP = dO[lo:hi, h, :] @ V[lo:hi, g, :].T
            delta = np.sum(dO[lo:hi, h, :] * O, axis=1)
            dl = np.where(causal, P * (dP - delta[:, None]), 0.0)
            d_bias[lo:hi] += gamma[h] * dl.sum(axis=0)
            d_gamma[h] += np.sum(dl * bias[None, lo:hi])
            d_beta += np.sum(dl * rho[:, None] * s)
    return d_bias, d_gamma, d_beta


def gate_score_backward(h, norm_w, W1, w2, cu_seqlens, prunable, kept_idx, d_kept_bias,
                        eps_norm: float = 1e-6, eps_seq: float = 1e-6):
    """Gradients of the gate's parameters from dL/d(kept_bias), the other half of training
    the gate end to end ([fluxbbs] 端到端训练的关键在 token 门控注意力).

    kept_bias[r] = z[kept_idx[r]] on prunable rows (0 on question rows); the top-K choice
    itself is piecewise constant and passes no gradient.  With z = s / rms_b over the
    request, s_t = sum_f w2_f SiLU(u_tf), u_t = W1 (n_t * norm_w), n_t = h_t / rms(h_t):
        ds_t = (dz_t - z_t mean_b(dz z)) / rms_b
        dw2_f = sum_t ds_t SiLU(u_tf);  du_tf = ds_t w2_f SiLU'(u_tf)
        dW1 = sum_t du_t (n_t * norm_w)^T;  d norm_w_k = sum_t n_tk sum_f du_tf W1_fk
    with SiLU'(u) = sig(u) (1 + u (1 - sig(u))).  Returns a dict of dz, ds, dw2, dW1,
    dnorm_w (float64)."""
    h = as_f64(h)
    W1 = as_f64(W1)
    w2 = as_f64(w2)
    w = np.ones(h.shape[1]) if norm_w is None else as_f64(norm_w)
    cu = _as_int(cu_seqlens)
    pr = _as_int(prunable)
    n = h / np.sqrt(np.mean(h * h, axis=1, keepdims=True) + eps_norm)
    xh = n * w[None, :]
    u = xh @ W1.T
    sig = 1.0 / (1.0 + np.exp(-u))
    s = (u * sig) @ w2
    dz = np.zeros(h.shape[0])
    idx = _as_int(kept_idx)
    dz[idx] = as_f64(d_kept_bias) * (pr[idx] != 0)
    ds = np.zeros_like(dz)
    for b in range(len(cu) - 1):
        lo, hi = cu[b], cu[b + 1]
        if hi == lo:
            continue
        rms = math.sqrt(float(np.mean(s[lo:hi] ** 2)) + eps_seq)
        z = s[lo:hi] / rms
        ds[lo:hi] = (dz[lo:hi] - z * np.mean(dz[lo:hi] * z)) / rms
    dsilu = sig * (1.0 + u * (1.0 - sig))
    dw2 = (u * sig).T @ ds
    du = ds[:, None] * w2[None, :] * dsilu
    dW1 = du.T @ xh
    dnorm_w = np.sum(n * (du @ W1), axis=0)
    return {"dz": dz, "ds": ds, "dw2": dw2, "dW1": dW1, "dnorm_w": dnorm_w}


def kv_compact(K, V, row_idx=None):
    """Compacted KV cache rows: K and V of the kept rows only ([farwalk] How does
    TokenGate learned token pruning work?: no KV entries for pruned tokens)."""
    K, V = as_f64(K), as_f64(V)
    if row_idx is None:
        return K.copy(), V.copy()
    i = _as_int(row_idx)
    return K[i], V[i]


# ------------------------------------------------------------------ layer body parts

def rmsnorm_heads(x, weight, eps: float = 1e-6) -> np.ndarray:
    """RMSNorm of each head's d values (the last axis) times a weight [d] shared by
    the heads: the QK-norm of a Qwen3-shaped layer, applied to q and k before RoPE."""
    x = as_f64(x)
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps) * as_f64(weight)


def swiglu_mlp(x, norm_w, W_gate, W_up, W_down, eps: float = 1e-6) -> np.ndarray:
    """Residual SwiGLU MLP: x + W_down (SiLU(W_gate b) * (W_up b)), b = RMSNorm(x) * norm_w.
    W_gate and W_up are [F, H], W_down is [H, F].  Pruned tokens never reach it above
    the gate ([fluxbbs] 门控到底插在模型的哪个位置)."""
    x = as_f64(x)
    b = rmsnorm_rows(x, norm_w, eps)
    g = b @ as_f64(W_gate).T
    u = b @ as_f64(W_up).T
    return x + (silu(g) * u) @ as_f64(W_down).T


def _attention_inputs(x, Wqkv, pos, n_q_heads, n_kv_heads, head_dim, theta, eps,
                      attn_norm=None, q_norm=None, k_norm=None):
    """a = RMSNorm(x) (times attn_norm), [q, k, v] = a Wqkv^T, optional QK-norm, then
    RoPE of q and k at `pos`."""
    a = rmsnorm_rows(x, attn_norm, eps)
    qkv = a @ as_f64(Wqkv).T
    nq, nk = n_q_heads * head_dim, n_kv_heads * head_dim
    rows = x.shape[0]
    q = qkv[:, :nq].reshape(rows, n_q_heads, head_dim)
    k = qkv[:, nq:nq + nk].reshape(rows, n_kv_heads, head_dim)
    v = qkv[:, nq + nk:].reshape(rows, n_kv_heads, head_dim)
    if q_norm is not None:
        q = rmsnorm_heads(q, q_norm, eps)
    if k_norm is not None:
        k = rmsnorm_heads(k, k_norm, eps)
    return a, qkv, rope(q, pos, theta), rope(k, pos, theta), v


# ------------------------------------------------------------------ one gated layer

def gated_layer(x, Wqkv, Wo, gamma, beta, cu_kept, kept_pos, kept_bias,
                n_q_heads: int, n_kv_heads: int, head_dim: int,
                theta: float = 1.0e6, eps: float = 1e-6,
                attn_norm=None, q_norm=None, k_norm=None, mlp=None):
    """One upper layer on the kept rows: x + Wo . Attn(RoPE(Wq a), RoPE(Wk a), Wv a), a = RMSNorm(x).

    Wqkv [(Hq + 2 Hkv) d, H] holds Wq, Wk, Wv row blocks; Wo is [H, Hq d].  RoPE uses
    the original positions.  Optional full-layer parts: `attn_norm` [H] weights the
    pre-attention RMSNorm, `q_norm` / `k_norm` [d] turn on QK-norm, `mlp` (a dict with
    norm_w, W_gate, W_up, W_down) appends the SwiGLU MLP.  Returns (x_out, K_cache,
    V_cache, parts) with the intermediates in `parts` for teacher-forced checks.
    """
    x = as_f64(x)
    a, qkv, q, k, v = _attention_inputs(x, Wqkv, kept_pos, n_q_heads, n_kv_heads, head_dim,
                                        theta, eps, attn_norm, q_norm, k_norm)
    Kt = x.shape[0]
    o, lse = gated_attention(q, k, v, cu_kept, kept_pos, kept_bias, gamma, beta)
    x_out = x + o.reshape(Kt, n_q_heads * head_dim) @ as_f64(Wo).T
    parts = {"a": a, "qkv": qkv, "q": q, "k": k, "v": v, "o": o, "lse": lse,
             "x_attn": x_out}
    if mlp is not None:
        x_out = swiglu_mlp(x_out, mlp["norm_w"], mlp["W_gate"], mlp["W_up"], mlp["W_down"], eps)
    return x_out, k, v, parts


# ------------------------------------------------------------------ layers below the gate

def request_positions(cu_seqlens) -> np.ndarray:
    """Position of every packed token within its own request: 0 .. N_b - 1 per request."""
    cu = _as_int(cu_seqlens)
    return np.concatenate([np.arange(cu[b + 1] - cu[b]) for b in range(len(cu) - 1)]
                          + [np.zeros(0, dtype=np.int64)])


def causal_attention(Q, K, V, cu_seqlens, block: int = 1024):
    """Ordinary causal GQA softmax attention inside each request.

    o_i = sum_{j <= i} softmax_j(q_i . k_j / sqrt(d)) v_j, q head h reading kv head
    h // (Hq / Hkv).  This is what every layer below the gate computes: all tokens
    are still present there and no gate term exists yet ([fluxbbs] 门控到底插在模型的
    哪个位置).  Written from the definition, independently of `gated_attention`.
    Returns O [T, Hq, d] (float64).
    """
    Q, K, V = as_f64(Q), as_f64(K), as_f64(V)
    cu = _as_int(cu_seqlens)
    T, Hq, d = Q.shape
    grp = Hq // K.shape[1]
    O = np.zeros(Q.shape)
    for b in range(len(cu) - 1):
        lo, hi = cu[b], cu[b + 1]
        for i0 in range(lo, hi, block):
            i1 = min(hi, i0 + block)
            # query i (absolute) may read keys lo .. i
            allowed = np.arange(lo, i1)[None, :] <= np.arange(i0, i1)[:, None]
            for h in range(Hq):
                g = h // grp
                logit = (Q[i0:i1, h, :] @ K[lo:i1, g, :].T) / math.sqrt(d)
                logit[~allowed] = -np.inf
                w = np.exp(logit - logit.max(axis=1, keepdims=True))
                w /= w.sum(axis=1, keepdims=True)
                O[i0:i1, h, :] = w @ V[lo:i1, g, :]
    return O


def full_context_layer(x, Wqkv, Wo, cu_seqlens, n_q_heads: int, n_kv_heads: int,
                       head_dim: int, theta: float = 1.0e6, eps: float = 1e-6,
                       attn_norm=None, q_norm=None, k_norm=None, mlp=None):
    """One layer below the gate on all tokens: x + Wo . Attn(RoPE(Wq a), RoPE(Wk a), Wv a)
    with a = RMSNorm(x), RoPE at each token's position in its request and ordinary
    causal attention; the optional full-layer parts as in `gated_layer`.  Returns
    (x_out, K_cache, V_cache): the full-length post-RoPE K and V, [T, Hkv, d]."""
    x = as_f64(x)
    T = x.shape[0]
    pos = request_positions(cu_seqlens)
    _, _, q, k, v = _attention_inputs(x, Wqkv, pos, n_q_heads, n_kv_heads, head_dim, theta,
                                      eps, attn_norm, q_norm, k_norm)
    o = causal_attention(q, k, v, cu_seqlens)
    x = x + o.reshape(T, n_q_heads * head_dim) @ as_f64(Wo).T
    if mlp is not None:
        x = swiglu_mlp(x, mlp["norm_w"], mlp["W_gate"], mlp["W_up"], mlp["W_down"], eps)
    return x, k, v


def _body_parts(L) -> dict:
    """The optional full-layer parts present in a layer's weight dict."""
    return {k: L[k] for k in ("attn_norm", "q_norm", "k_norm", "mlp") if L.get(k) is not None}


def prefill(h, prunable, cu_seqlens, budgets, gate, layers, n_q_heads, n_kv_heads,
            head_dim, theta=1.0e6, norm_eps=1e-6, seq_eps=1e-6, scores=None,
            lower_layers=()):
    """Lower layers + gate + selection + gathered upper layers, end to end.

    `gate` holds norm_w, W1, w2; `layers` (above the gate) and `lower_layers` (below
    it) are lists of dicts with Wqkv and Wo (plus gamma, beta above the gate, and
    optionally attn_norm, q_norm, k_norm and mlp for a full layer body).  The
    lower layers run on every token; the gate reads their output, the residual at
    the gate layer.  Their K/V caches come back both full-length and trimmed to the
    kept rows.  With `scores` given, selection consumes those raw scores instead of
    the scorer's (the planted-cluster workload).
    """
    lower_full = []
    for L in lower_layers:
        h, k, v = full_context_layer(h, L["Wqkv"], L["Wo"], cu_seqlens, n_q_heads,
                                     n_kv_heads, head_dim, theta, norm_eps,
                                     **_body_parts(L))
        lower_full.append((k, v))
    s = gate_score(h, gate["norm_w"], gate["W1"], gate["w2"], norm_eps) if scores is None \
        else as_f64(scores)
    z, bias = sequence_rmsnorm(s, cu_seqlens, prunable, seq_eps)
    cu_kept = kept_counts(prunable, cu_seqlens, budgets)
    kept_idx, kept_pos, kept_bias = select_topk(z.astype(np.float32), prunable,
                                                cu_seqlens, cu_kept)
    x = gather_rows(h, kept_idx)
    caches = []
    for L in layers:
        x, k, v, _ = gated_layer(x, L["Wqkv"], L["Wo"], L["gamma"], L["beta"], cu_kept,
                                 kept_pos, kept_bias, n_q_heads, n_kv_heads, head_dim,
                                 theta, norm_eps, **_body_parts(L))
        caches.append((k, v))
    return {"s": s, "z": z, "bias": bias, "cu_kept": cu_kept, "kept_idx": kept_idx,
            "kept_pos": kept_pos, "kept_bias": kept_bias, "x": x, "caches": caches,
            "h_gate": as_f64(h), "lower_caches_full": lower_full,
            "lower_caches": [kv_compact(k, v, kept_idx) for k, v in lower_full]}
