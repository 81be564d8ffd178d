"""TokenGate gate layer and token-gated attention on B200 (sm_100a).

Thin Python binding of ``libtokengate.so`` (declared in ``include/tokengate.h``).
Every function named ``tg_*`` here marshals torch tensors into the C call of the same
name; all arithmetic of the path runs in the library's CUDA kernels.  PyTorch only
provides device memory and the stream.  If the shared library is missing, importing
this package raises: there is no fallback implementation.

``GatedPrefill`` strings the calls together for one prefill step: gate scores and
their sequence normalisation, prunable-only top-K with order-preserving compaction,
the row gather, then per upper layer the RMSNorm-folded QKV projection, RoPE at the
original positions, the compacted KV-cache write, token-gated attention and the
output projection with its residual add.
"""
from __future__ import annotations

import ctypes as C
from dataclasses import dataclass

import torch

from . import _lib

__all__ = [
    "TokenGateError", "lib", "tg_version", "tg_device_supported", "tg_plan_kept",
    "tg_rope_table", "tg_rope_rows", "tg_gate_score_workspace_size", "tg_gate_score", "tg_topk_compact",
    "tg_gate_score_noalloc", "tg_seq_rmsnorm", "tg_gather_rope", "tg_kv_compact", "tg_gated_attention", "tg_linear",
    "tg_status_clear", "tg_status_read", "tg_set_launch_overlap", "tg_get_launch_overlap",
    "tg_set_gather_tma", "tg_get_gather_tma", "tg_set_scorer_pair", "tg_get_scorer_pair",
    "tg_gemm_workspace_size",
    "tg_prefetch_l2", "tg_out_proj_qkv_next", "tg_out_proj_qkv_workspace_size",
    "tg_swiglu", "tg_fold_norm_weight", "tg_pack_gate_up", "prepare_layer",
    "tg_gated_attention_bias_grad", "tg_gated_attention_bias_grad_workspace_size",
    "tg_gate_score_backward", "tg_gate_score_backward_workspace_size",
    "GatedPrefill", "FullContextLayers", "padded_layout", "k_bucket", "LayerWeights", "STATUS_TIMEOUT", "STATUS_BUDGET",
    "STATUS_BOUNDS", "STATUS_WORKSPACE",
]

lib = _lib.load()

STATUS_TIMEOUT = 0x1
STATUS_BUDGET = 0x2
STATUS_BOUNDS = 0x4
STATUS_WORKSPACE = 0x8

# Kernel launches issued through this binding (a benchmark reads it to report how many
# of the library's kernels ran in its timed region).
launch_count = 0


def _count(n: int = 1) -> None:
    global launch_count
    launch_count += n


class TokenGateError(RuntimeError):
    def __init__(self, msg, code):
        super().__init__(msg)
        self.code = code


def _check(rc: int, name: str) -> None:
    if rc != 0:
        msg = lib.tg_error_string(rc).decode()
        if rc == -5:
            msg += f" (cudaError {lib.tg_last_cuda_error()})"
        raise TokenGateError(f"{name}: {msg}", rc)


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return C.c_void_p(stream.cuda_stream)


def _host_i32(x) -> torch.Tensor:
    t = torch.as_tensor(x, dtype=torch.int32, device="cpu").contiguous()
    return t


def _mat(t: torch.Tensor, name: str):
    if t.dim() != 2 or t.stride(1) != 1:
        raise ValueError(f"{name}: expected a 2-D row-major view, got shape {tuple(t.shape)} "
                         f"stride {t.stride()}")
    return t.stride(0)


def tg_version() -> int:
    return lib.tg_version()


def tg_device_supported(device: int = 0) -> bool:
    return bool(lib.tg_device_supported(device))


def tg_status_clear(status: torch.Tensor, stream=None) -> None:
    _check(lib.tg_status_clear(_ptr(status), _stream(stream)), "tg_status_clear")


def tg_set_launch_overlap(enable: bool) -> None:
    """Launch every kernel with programmatic stream serialisation (default off)."""
    _check(lib.tg_set_launch_overlap(1 if enable else 0), "tg_set_launch_overlap")


def tg_get_launch_overlap() -> bool:
    return bool(lib.tg_get_launch_overlap())


def tg_set_gather_tma(enable: bool) -> None:
    """Gather mode of tg_gather_rope: the TMA row gather (True) or the warp-per-row
    copy (False, default)."""
    _check(lib.tg_set_gather_tma(1 if enable else 0), "tg_set_gather_tma")


def tg_get_gather_tma() -> bool:
    return bool(lib.tg_get_gather_tma())


def tg_set_scorer_pair(enable: bool) -> None:
    """Scorer GEMM of tg_gate_score: CTA pairs (True, default) or one CTA per tile."""
    _check(lib.tg_set_scorer_pair(1 if enable else 0), "tg_set_scorer_pair")


def tg_get_scorer_pair() -> bool:
    return bool(lib.tg_get_scorer_pair())


def tg_prefetch_l2(t: torch.Tensor, stream=None) -> None:
    """Bring a contiguous device tensor into L2 ahead of its use (a hint)."""
    if not t.is_contiguous():
        raise ValueError("tg_prefetch_l2 needs a contiguous tensor")
    _check(lib.tg_prefetch_l2(_ptr(t), t.numel() * t.element_size(), _stream(stream)),
           "tg_prefetch_l2")
    _count()


def tg_status_read(status: torch.Tensor, stream=None) -> int:
    out = C.c_uint32(0)
    _check(lib.tg_status_read(_ptr(status), C.byref(out), _stream(stream)), "tg_status_read")
    return int(out.value)


def tg_plan_kept(cu_seqlens_host, n_question_host, budgets_host) -> torch.Tensor:
    """Host-only: cu_kept from budgets (see include/tokengate.h)."""
    cu = _host_i32(cu_seqlens_host)
    nq = _host_i32(n_question_host)
    bud = _host_i32(budgets_host)
    batch = cu.numel() - 1
    out = torch.zeros(batch + 1, dtype=torch.int32)
    _check(lib.tg_plan_kept(_ptr(cu), _ptr(nq), _ptr(bud), batch, _ptr(out)), "tg_plan_kept")
    return out


def padded_layout(cu_kept_host, k_pad=None) -> torch.Tensor:
    """Row layout of the layers above the gate (host int32 [B + 1]).

    Without `k_pad` it is the kept layout itself.  With `k_pad` >= K (the kept total)
    the last request takes k_pad - K extra trailing rows, so the layers always run on
    k_pad rows and one CUDA graph of them serves every later call with the same layout
    (for a single request: every kept total up to k_pad).  The pruned forward is
    captured as a CUDA graph over a fixed padded size in "TokenGate: Adapting LLMs for
    Fast and Memory-Efficient Prefill with Learned Token Pruning" (paper digest),
    sections 方法关键点 and 工作参考价值.

    Each kept row keeps its index, and as attention is causal within a request and the
    padding rows follow every kept row of theirs, no kept row's keys include a padding
    row.  Kept rows therefore get the unpadded results, up to the fp32 summation order
    of the attention when the longer layout splits the key range differently."""
    ckh = _host_i32(cu_kept_host).clone()
    if k_pad is None:
        return ckh
    K = int(ckh[-1])
    k_pad = int(k_pad)
    if ckh.numel() < 2:
        raise ValueError("padded_layout: the layout needs at least one request")
    if k_pad < K:
        raise ValueError(f"padded_layout: k_pad={k_pad} is below the kept total {K}")
    ckh[-1] = k_pad
    return ckh


def k_bucket(K: int, granule: int = 256) -> int:
    """The padded row count of a kept total: K rounded up to a multiple of `granule`
    (at least one granule), so calls whose kept totals round to the same bucket share
    one captured graph of the layers above the gate."""
    if granule <= 0:
        raise ValueError("k_bucket: granule must be positive")
    return max(granule, -(-int(K) // granule) * granule)


def tg_rope_table(max_pos: int, head_dim: int, theta: float, out=None, device=None,
                  stream=None) -> torch.Tensor:
    if out is None:
        out = torch.empty((max_pos, head_dim // 2, 2), dtype=torch.float32,
                          device=device or "cuda")
    _check(lib.tg_rope_table(_ptr(out), max_pos, head_dim, float(theta), _stream(stream)),
           "tg_rope_table")
    _count()
    return out


def tg_rope_rows(pos, cos_sin, out=None, status=None, stream=None) -> torch.Tensor:
    """Per-row rotary table [head_dim/4, ld_rot, 4] of the rows' positions (cos_sin from
    tg_rope_table); pass it as cos_sin with pos=None to the QKV entry points."""
    n = pos.numel()
    head_dim = cos_sin.shape[1] * cos_sin.shape[2] if cos_sin.dim() == 3 else cos_sin.shape[1]
    if out is None:
        out = torch.empty((head_dim // 4, max(n, 1), 4), dtype=torch.float32, device=pos.device)
    _check(lib.tg_rope_rows(_ptr(pos), n, _ptr(cos_sin), cos_sin.shape[0], head_dim, _ptr(out),
                            out.shape[1], _ptr(status), _stream(stream)), "tg_rope_rows")
    _count()
    return out


def _rope_rows_arg(pos, cos_sin):
    """max_pos argument of the QKV entry points: table rows, or the per-row table's stride."""
    return cos_sin.shape[0] if pos is not None else cos_sin.shape[1]


def tg_gate_score_workspace_size(total_tokens: int, hidden: int, width: int, batch: int) -> int:
    return int(lib.tg_gate_score_workspace_size(total_tokens, hidden, width, batch))


def tg_gate_score(h, W1, w2, cu_seqlens, cu_seqlens_host, prunable, norm_w=None,
                  eps_norm=1e-6, eps_seq=1e-6, s_out=None, z_out=None, bias_out=None,
                  workspace=None, status=None, stream=None):
    ld_h = _mat(h, "h")
    T, hidden = h.shape
    width = W1.shape[0]
    cuh = _host_i32(cu_seqlens_host)
    batch = cuh.numel() - 1
    dev = h.device
    s_out = torch.empty(T, dtype=torch.float32, device=dev) if s_out is None else s_out
    z_out = torch.empty(T, dtype=torch.float32, device=dev) if z_out is None else z_out
    bias_out = torch.empty(T, dtype=torch.float32, device=dev) if bias_out is None else bias_out
    need = tg_gate_score_workspace_size(T, hidden, width, batch)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    rc = lib.tg_gate_score(_ptr(h), ld_h, T, hidden, _ptr(norm_w), _ptr(W1), width, _ptr(w2),
                           float(eps_norm), _ptr(cu_seqlens), _ptr(cuh), batch, float(eps_seq),
                           _ptr(prunable), _ptr(s_out), _ptr(z_out), _ptr(bias_out),
                           _ptr(workspace), workspace.numel(), _ptr(status), _stream(stream))
    _check(rc, "tg_gate_score")
    _count(3 if norm_w is not None else 2)
    return s_out, z_out, bias_out


def tg_gate_score_noalloc(h, W1, w2, cu_seqlens, cu_seqlens_host, prunable, norm_w=None,
                          eps_norm=1e-6, eps_seq=1e-6, s_out=None, z_out=None, bias_out=None,
                          status=None, stream=None):
    """tg_gate_score without a workspace: for callers that may not allocate device
    memory.  Scratch is a fixed array inside the library (limits and the one-time
    per-device set-up are described in include/tokengate.h); calls that can overlap on
    the GPU share that array and race, so serialise them.  This wrapper allocates the
    outputs only when they are not passed in."""
    ld_h = _mat(h, "h")
    T, hidden = h.shape
    width = W1.shape[0]
    cuh = _host_i32(cu_seqlens_host)
    batch = cuh.numel() - 1
    dev = h.device
    s_out = torch.empty(T, dtype=torch.float32, device=dev) if s_out is None else s_out
    z_out = torch.empty(T, dtype=torch.float32, device=dev) if z_out is None else z_out
    bias_out = torch.empty(T, dtype=torch.float32, device=dev) if bias_out is None else bias_out
    rc = lib.tg_gate_score_noalloc(_ptr(h), ld_h, T, hidden, _ptr(norm_w), _ptr(W1), width,
                                   _ptr(w2), float(eps_norm), _ptr(cu_seqlens), _ptr(cuh), batch,
                                   float(eps_seq), _ptr(prunable), _ptr(s_out), _ptr(z_out),
                                   _ptr(bias_out), _ptr(status), _stream(stream))
    _check(rc, "tg_gate_score_noalloc")
    _count(3 if norm_w is not None else 2)
    return s_out, z_out, bias_out


def tg_seq_rmsnorm(s, cu_seqlens, cu_seqlens_host, prunable, eps_seq=1e-6, z_out=None,
                   bias_out=None, stream=None):
    cuh = _host_i32(cu_seqlens_host)
    z_out = torch.empty_like(s) if z_out is None else z_out
    bias_out = torch.empty_like(s) if bias_out is None else bias_out
    rc = lib.tg_seq_rmsnorm(_ptr(s), _ptr(cu_seqlens), _ptr(cuh), cuh.numel() - 1, _ptr(prunable),
                            float(eps_seq), _ptr(z_out), _ptr(bias_out), _stream(stream))
    _check(rc, "tg_seq_rmsnorm")
    _count()
    return z_out, bias_out


def tg_topk_compact(z, prunable, cu_seqlens, cu_seqlens_host, cu_kept, cu_kept_host,
                    kept_idx=None, kept_pos=None, kept_bias=None, status=None, stream=None):
    cuh = _host_i32(cu_seqlens_host)
    ckh = _host_i32(cu_kept_host)
    batch = cuh.numel() - 1
    K = int(ckh[-1])
    dev = z.device
    kept_idx = torch.empty(K, dtype=torch.int32, device=dev) if kept_idx is None else kept_idx
    kept_pos = torch.empty(K, dtype=torch.int32, device=dev) if kept_pos is None else kept_pos
    kept_bias = torch.empty(K, dtype=torch.float32, device=dev) if kept_bias is None else kept_bias
    rc = lib.tg_topk_compact(_ptr(z), _ptr(prunable), _ptr(cu_seqlens), _ptr(cuh),
                             _ptr(cu_kept), _ptr(ckh), batch, _ptr(kept_idx), _ptr(kept_pos),
                             _ptr(kept_bias), _ptr(status), _stream(stream))
    _check(rc, "tg_topk_compact")
    _count()
    return kept_idx, kept_pos, kept_bias


def tg_gather_rope(src, dst=None, row_idx=None, n_rows=None, rope_pos=None,
                   rope_cols=(0, 0), head_dim=128, cos_sin=None, row_ssq=None, status=None,
                   stream=None):
    ld_src = _mat(src, "src")
    width = src.shape[1]
    if n_rows is None:
        n_rows = row_idx.numel() if row_idx is not None else src.shape[0]
    if dst is None:
        dst = torch.empty((n_rows, width), dtype=src.dtype, device=src.device)
    ld_dst = _mat(dst, "dst")
    max_pos = cos_sin.shape[0] if cos_sin is not None else 0
    ld_ssq = _mat(row_ssq, "row_ssq") if row_ssq is not None else 0
    rc = lib.tg_gather_rope(_ptr(src), ld_src, src.shape[0], _ptr(row_idx), n_rows, width,
                            _ptr(rope_pos), int(rope_cols[0]), int(rope_cols[1]), head_dim,
                            _ptr(cos_sin), max_pos, _ptr(dst), ld_dst, _ptr(row_ssq), ld_ssq,
                            _ptr(status), _stream(stream))
    _check(rc, "tg_gather_rope")
    _count()
    return dst


def tg_kv_compact(k, v, cache_k, cache_v, row_idx=None, n_rows=None, slot_offset=0,
                  status=None, stream=None):
    ld_k, ld_v = _mat(k, "k"), _mat(v, "v")
    ld_c = _mat(cache_k, "cache_k")
    if _mat(cache_v, "cache_v") != ld_c:
        raise ValueError("cache_k and cache_v must share a row stride")
    width = k.shape[1]
    if n_rows is None:
        n_rows = row_idx.numel() if row_idx is not None else k.shape[0]
    if v.shape[0] != k.shape[0] or cache_v.shape[0] != cache_k.shape[0]:
        raise ValueError("k/v and cache_k/cache_v must have matching row counts")
    rc = lib.tg_kv_compact(_ptr(k), ld_k, _ptr(v), ld_v, k.shape[0], _ptr(row_idx), n_rows,
                           width, _ptr(cache_k), _ptr(cache_v), ld_c, cache_k.shape[0],
                           int(slot_offset), _ptr(status), _stream(stream))
    _check(rc, "tg_kv_compact")
    _count()


def tg_gated_attention_workspace_size(cu_kept_host, n_q_heads, n_kv_heads, head_dim=128) -> int:
    ckh = _host_i32(cu_kept_host)
    return int(lib.tg_gated_attention_workspace_size(_ptr(ckh), ckh.numel() - 1, n_q_heads,
                                                     n_kv_heads, head_dim))


def tg_gated_attention(q, k, v, cu_kept, cu_kept_host, n_q_heads, n_kv_heads, kept_pos,
                       kept_bias, gamma, beta, o=None, lse=None, head_dim=128, workspace=None,
                       status=None, stream=None):
    """Token-gated attention.  `workspace=None` allocates the split-KV workspace the
    layout asks for (pass a zero-filled uint8 tensor to reuse one: calls leave it zeroed;
    an empty one disables splitting)."""
    ld_q, ld_k, ld_v = _mat(q, "q"), _mat(k, "k"), _mat(v, "v")
    ckh = _host_i32(cu_kept_host)
    batch = ckh.numel() - 1
    if o is None:
        o = torch.empty((q.shape[0], n_q_heads * head_dim), dtype=q.dtype, device=q.device)
    ld_o = _mat(o, "o")
    if workspace is None:
        need = tg_gated_attention_workspace_size(ckh, n_q_heads, n_kv_heads, head_dim)
        workspace = torch.zeros(need, dtype=torch.uint8, device=q.device)
    ws_ptr = _ptr(workspace) if workspace.numel() else None
    rc = lib.tg_gated_attention(_ptr(q), ld_q, _ptr(k), ld_k, _ptr(v), ld_v, _ptr(cu_kept),
                                _ptr(ckh), batch, n_q_heads, n_kv_heads, head_dim,
                                _ptr(kept_pos), _ptr(kept_bias), _ptr(gamma), float(beta),
                                _ptr(o), ld_o, _ptr(lse), ws_ptr, workspace.numel(),
                                _ptr(status), _stream(stream))
    _check(rc, "tg_gated_attention")
    _count()
    return o


def tg_gated_attention_bias_grad_workspace_size(cu_kept_host, n_q_heads, n_kv_heads,
                                                head_dim=128) -> int:
    ckh = _host_i32(cu_kept_host)
    return int(lib.tg_gated_attention_bias_grad_workspace_size(_ptr(ckh), ckh.numel() - 1,
                                                               n_q_heads, n_kv_heads, head_dim))


def tg_gated_attention_bias_grad(q, k, v, o, d_o, lse, cu_kept, cu_kept_host, n_q_heads,
                                 n_kv_heads, kept_pos, kept_bias, gamma, beta, d_bias=None,
                                 d_gamma=None, d_beta=None, head_dim=128, workspace=None,
                                 status=None, stream=None):
    """Gradients of token-gated attention w.r.t. the key bias (returned), and into
    d_gamma [Hq] / d_beta [1] when given, from the forward's o and lse and dO."""
    ckh = _host_i32(cu_kept_host)
    batch = ckh.numel() - 1
    if d_bias is None:
        d_bias = torch.empty(q.shape[0], dtype=torch.float32, device=q.device)
    if workspace is None:
        need = tg_gated_attention_bias_grad_workspace_size(ckh, n_q_heads, n_kv_heads, head_dim)
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    rc = lib.tg_gated_attention_bias_grad(
        _ptr(q), _mat(q, "q"), _ptr(k), _mat(k, "k"), _ptr(v), _mat(v, "v"), _ptr(o),
        _mat(o, "o"), _ptr(d_o), _mat(d_o, "d_o"), _ptr(lse), _ptr(cu_kept), _ptr(ckh), batch,
        n_q_heads, n_kv_heads, head_dim, _ptr(kept_pos), _ptr(kept_bias), _ptr(gamma),
        float(beta), _ptr(d_bias), _ptr(d_gamma), _ptr(d_beta), _ptr(workspace),
        workspace.numel(), _ptr(status), _stream(stream))
    _check(rc, "tg_gated_attention_bias_grad")
    _count(4 if int(ckh[-1]) > 0 else 1)
    return d_bias



def tg_gate_score_backward_workspace_size(total_tokens, hidden, width, batch):
    return int(lib.tg_gate_score_backward_workspace_size(int(total_tokens), int(hidden),
                                                         int(width), int(batch)))


def tg_gate_score_backward(h, W1, w2, s, cu_seqlens, cu_seqlens_host, prunable, cu_kept,
                           cu_kept_host, kept_idx, d_kept_bias, norm_w=None, eps_norm=1e-6,
                           eps_seq=1e-6, ds_out=None, dW1=None, dnorm_w=None, dw2=None,
                           workspace=None, status=None, stream=None):
    """Scorer parameter gradients from dL/d(kept_bias): returns (ds, dW1, dw2, dnorm_w);
    dnorm_w is computed when norm_w is given or dnorm_w is passed in.  `s` is the s_out
    of tg_gate_score on the same inputs."""
    ld_h = _mat(h, "h")
    T, hidden = h.shape
    width = W1.shape[0]
    cuh, ckh = _host_i32(cu_seqlens_host), _host_i32(cu_kept_host)
    batch = cuh.numel() - 1
    dev = h.device
    ds_out = torch.empty(T, dtype=torch.float32, device=dev) if ds_out is None else ds_out
    dW1 = torch.empty((width, hidden), dtype=torch.float32, device=dev) if dW1 is None else dW1
    dw2 = torch.empty(width, dtype=torch.float32, device=dev) if dw2 is None else dw2
    if dnorm_w is None and norm_w is not None:
        dnorm_w = torch.empty(hidden, dtype=torch.float32, device=dev)
    if workspace is None:
        need = tg_gate_score_backward_workspace_size(T, hidden, width, batch)
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    rc = lib.tg_gate_score_backward(
        _ptr(h), ld_h, T, hidden, _ptr(norm_w), _ptr(W1), width, _ptr(w2), float(eps_norm),
        _ptr(s), _ptr(cu_seqlens), _ptr(cuh), batch, float(eps_seq), _ptr(prunable),
        _ptr(cu_kept), _ptr(ckh), _ptr(kept_idx), _ptr(d_kept_bias), _ptr(ds_out), _ptr(dW1),
        _ptr(dnorm_w), _ptr(dw2), _ptr(workspace), workspace.numel(), _ptr(status),
        _stream(stream))
    _check(rc, "tg_gate_score_backward")
    if T > 0:
        _count(6 + (1 if int(ckh[-1]) > 0 else 0) + (1 if norm_w is not None else 0))
    return ds_out, dW1, dw2, dnorm_w

def tg_gemm_workspace_size() -> int:
    """Bytes of the stream-K workspace the CTA-pair GEMMs may use (see the header)."""
    return int(lib.tg_gemm_workspace_size())


def _ws(workspace):
    if workspace is None or workspace.numel() == 0:
        return None, 0
    return _ptr(workspace), workspace.numel() * workspace.element_size()


def tg_linear(a, w, c=None, rmsnorm=False, eps=1e-6, residual=None, row_ssq=None, status=None,
              stream=None, workspace=None):
    """c = (RMSNorm(a)) w^T (+ residual).  `workspace`: a zero-filled uint8 tensor of
    tg_gemm_workspace_size() bytes lets the CTA-pair GEMM split its last round of tiles
    along K (left zeroed by every call)."""
    lda, ldw = _mat(a, "a"), _mat(w, "w")
    M, K = a.shape
    N = w.shape[0]
    if c is None:
        c = torch.empty((M, N), dtype=a.dtype, device=a.device)
    ldc = _mat(c, "c")
    ldr = _mat(residual, "residual") if residual is not None else 0
    ld_ssq = _mat(row_ssq, "row_ssq") if row_ssq is not None else 0
    ws_ptr, ws_bytes = _ws(workspace)
    rc = lib.tg_linear(_ptr(a), lda, _ptr(w), ldw, _ptr(c), ldc, M, N, K, 1 if rmsnorm else 0,
                       float(eps), _ptr(residual), ldr, _ptr(row_ssq), ld_ssq, ws_ptr, ws_bytes,
                       _ptr(status), _stream(stream))
    _check(rc, "tg_linear")
    _count()
    return c


def tg_qkv_rope_cache(x, w_qkv, pos, cos_sin, cache_k, cache_v, n_q_heads, n_kv_heads,
                      q_out=None, head_dim=128, eps=1e-6, slot_offset=0, row_ssq=None,
                      status=None, stream=None, q_norm_w=None, k_norm_w=None, workspace=None):
    """Fused QKV projection (RMSNorm folded) + RoPE at `pos` + compacted KV-cache write
    (pos=None: cos_sin is the per-row table of tg_rope_rows);
    with q_norm_w / k_norm_w (float32 [head_dim]) also QK-norm before RoPE
    (tg_qkv_qknorm_rope_cache)."""
    ld_x, ld_w = _mat(x, "x"), _mat(w_qkv, "w_qkv")
    M, hidden = x.shape
    if q_out is None:
        q_out = torch.empty((M, n_q_heads * head_dim), dtype=x.dtype, device=x.device)
    ld_q = _mat(q_out, "q_out")
    ld_c = _mat(cache_k, "cache_k")
    if _mat(cache_v, "cache_v") != ld_c:
        raise ValueError("cache_k and cache_v must share a row stride")
    ld_ssq = _mat(row_ssq, "row_ssq") if row_ssq is not None else 0
    ws_ptr, ws_bytes = _ws(workspace)
    if q_norm_w is not None or k_norm_w is not None:
        rc = lib.tg_qkv_qknorm_rope_cache(_ptr(x), ld_x, _ptr(w_qkv), ld_w, M, hidden, n_q_heads,
                                          n_kv_heads, head_dim, float(eps), _ptr(q_norm_w),
                                          _ptr(k_norm_w), _ptr(pos), _ptr(cos_sin),
                                          _rope_rows_arg(pos, cos_sin), _ptr(q_out), ld_q,
                                          _ptr(cache_k),
                                          _ptr(cache_v), ld_c, int(slot_offset), _ptr(row_ssq),
                                          ld_ssq, ws_ptr, ws_bytes, _ptr(status),
                                          _stream(stream))
        _check(rc, "tg_qkv_qknorm_rope_cache")
    else:
        rc = lib.tg_qkv_rope_cache(_ptr(x), ld_x, _ptr(w_qkv), ld_w, M, hidden, n_q_heads,
                                   n_kv_heads, head_dim, float(eps), _ptr(pos), _ptr(cos_sin),
                                   _rope_rows_arg(pos, cos_sin), _ptr(q_out), ld_q,
                                   _ptr(cache_k),
                                   _ptr(cache_v), ld_c, int(slot_offset), _ptr(row_ssq), ld_ssq,
                                   ws_ptr, ws_bytes, _ptr(status), _stream(stream))
        _check(rc, "tg_qkv_rope_cache")
    _count()
    return q_out


def tg_swiglu(x, w_gu, row_ssq, h_out=None, eps=1e-6, status=None, stream=None):
    """h = SiLU(b W_gate^T) * (b W_up^T), b = RMSNorm(x) from its row sums of squares;
    w_gu from tg_pack_gate_up (norm weight folded, rows interleaved)."""
    ld_x, ld_w, ld_ssq = _mat(x, "x"), _mat(w_gu, "w_gu"), _mat(row_ssq, "row_ssq")
    M, hidden = x.shape
    ffn = w_gu.shape[0] // 2
    if h_out is None:
        h_out = torch.empty((M, ffn), dtype=x.dtype, device=x.device)
    ld_h = _mat(h_out, "h_out")
    rc = lib.tg_swiglu(_ptr(x), ld_x, _ptr(w_gu), ld_w, M, hidden, ffn, float(eps),
                       _ptr(row_ssq), ld_ssq, _ptr(h_out), ld_h, _ptr(status), _stream(stream))
    _check(rc, "tg_swiglu")
    _count()
    return h_out


def tg_fold_norm_weight(w, norm_w, out=None, stream=None):
    """out[r, c] = bf16(w[r, c] * norm_w[c]): an RMSNorm weight folded into the projection."""
    ld_w = _mat(w, "w")
    if out is None:
        out = torch.empty_like(w)
    rc = lib.tg_fold_norm_weight(_ptr(w), ld_w, w.shape[0], w.shape[1], _ptr(norm_w), _ptr(out),
                                 _mat(out, "out"), _stream(stream))
    _check(rc, "tg_fold_norm_weight")
    _count()
    return out


def tg_pack_gate_up(w_gate, w_up, norm_w=None, out=None, stream=None):
    """[2 F, H] weight for tg_swiglu: gate and up rows interleaved in blocks of 64, columns
    scaled by the MLP's RMSNorm weight."""
    ffn, hidden = w_gate.shape
    if out is None:
        out = torch.empty((2 * ffn, hidden), dtype=w_gate.dtype, device=w_gate.device)
    rc = lib.tg_pack_gate_up(_ptr(w_gate), _mat(w_gate, "w_gate"), _ptr(w_up), _mat(w_up, "w_up"),
                             ffn, hidden, _ptr(norm_w), _ptr(out), _mat(out, "out"),
                             _stream(stream))
    _check(rc, "tg_pack_gate_up")
    _count()
    return out


def tg_out_proj_qkv_workspace_size(M: int) -> int:
    return int(lib.tg_out_proj_qkv_workspace_size(int(M)))


def tg_out_proj_qkv_next(o, w_o, x, row_ssq, w_qkv, pos, cos_sin, cache_k, cache_v, n_q_heads,
                         n_kv_heads, q_out, workspace, head_dim=128, eps=1e-6, slot_offset=0,
                         status=None, stream=None):
    """x <- x + o w_o^T (row sums of squares into row_ssq), then the next layer's fused
    QKV + RoPE + KV-cache write from the new x, in one launch.  `workspace` is a
    zero-filled uint8 tensor of tg_out_proj_qkv_workspace_size(M) bytes (left zeroed)."""
    ld_o, ld_wo, ld_x = _mat(o, "o"), _mat(w_o, "w_o"), _mat(x, "x")
    ld_ssq, ld_wqkv, ld_q = _mat(row_ssq, "row_ssq"), _mat(w_qkv, "w_qkv"), _mat(q_out, "q_out")
    ld_c = _mat(cache_k, "cache_k")
    if _mat(cache_v, "cache_v") != ld_c:
        raise ValueError("cache_k and cache_v must share a row stride")
    M, hidden = x.shape
    rc = lib.tg_out_proj_qkv_next(_ptr(o), ld_o, _ptr(w_o), ld_wo, _ptr(x), ld_x, _ptr(row_ssq),
                                  ld_ssq, M, hidden, o.shape[1], _ptr(w_qkv), ld_wqkv, n_q_heads,
                                  n_kv_heads, head_dim, float(eps), _ptr(pos), _ptr(cos_sin),
                                  _rope_rows_arg(pos, cos_sin), _ptr(q_out), ld_q,
                                  _ptr(cache_k),
                                  _ptr(cache_v), ld_c, int(slot_offset), _ptr(workspace),
                                  workspace.numel(), _ptr(status), _stream(stream))
    _check(rc, "tg_out_proj_qkv_next")
    _count()
    return x


# ----------------------------------------------------------------------------- pipeline

@dataclass
class LayerWeights:
    Wqkv: torch.Tensor   # bf16 [(Hq + 2 Hkv) d, H] (a weighted attention norm folded in)
    Wo: torch.Tensor     # bf16 [H, Hq d]
    gamma: torch.Tensor = None  # fp32 [Hq] (layers above the gate)
    beta: float = 1.0
    q_norm: torch.Tensor = None  # fp32 [d]: QK-norm weights (full layer body)
    k_norm: torch.Tensor = None
    W_gu: torch.Tensor = None    # bf16 [2 F, H]: packed SwiGLU gate/up (tg_pack_gate_up)
    W_down: torch.Tensor = None  # bf16 [H, F]

    @property
    def ffn(self):
        return 0 if self.W_gu is None else self.W_gu.shape[0] // 2


def prepare_layer(layer) -> LayerWeights:
    """LayerWeights from a weight dict: Wqkv, Wo (+ gamma, beta above the gate), and for
    a full layer body attn_norm, q_norm, k_norm and mlp = {norm_w, W_gate, W_up, W_down}.
    The norm weights that multiply a projection's input are folded into it here, once
    (tg_fold_norm_weight, tg_pack_gate_up)."""
    if isinstance(layer, LayerWeights):
        return layer
    d = dict(layer)
    Wqkv = d["Wqkv"]
    if d.get("attn_norm") is not None:
        Wqkv = tg_fold_norm_weight(Wqkv, d["attn_norm"])
    W_gu = W_down = None
    mlp = d.get("mlp")
    if mlp is not None:
        W_gu = tg_pack_gate_up(mlp["W_gate"], mlp["W_up"], mlp.get("norm_w"))
        W_down = mlp["W_down"]
    return LayerWeights(Wqkv=Wqkv, Wo=d["Wo"], gamma=d.get("gamma"), beta=d.get("beta", 1.0),
                        q_norm=d.get("q_norm"), k_norm=d.get("k_norm"), W_gu=W_gu,
                        W_down=W_down)


def _mlp(L, x, P, eps, status, stream, mark):
    """The SwiGLU MLP of a full layer body, in place on x (nothing without one)."""
    if L.W_gu is None:
        return
    h = P["ffn"][:, :L.ffn]
    tg_swiglu(x, L.W_gu, P["ssq"], h_out=h, eps=eps, status=status, stream=stream)
    mark("mlp_gate_up")
    tg_linear(h, L.W_down, x, residual=x, row_ssq=P["ssq"], status=status, stream=stream,
              workspace=P.get("gemm_ws"))
    mark("mlp_down")


class FullContextLayers:
    """Layers below the gate: every token of every request, ordinary causal GQA
    attention on the same kernels as the gated layers (gamma = 0, every token kept,
    so tau = beta = 1 and no key bias).  Also the full-context reference of a gated
    stack: the same weights without pruning.

    ``plan`` allocates full-length buffers and caches; ``run`` leaves the residual
    stream after the last layer in ``planned["x"]`` (the gate's input) and each
    layer's post-RoPE K/V in ``planned["caches"]``; ``trim`` copies the kept rows of
    those caches into compacted ones.
    """

    def __init__(self, layers: list, n_q_heads=16, n_kv_heads=8, head_dim=128,
                 rope_theta=1.0e6, norm_eps=1e-6, device="cuda"):
        self.device = torch.device(device)
        self.layers = [prepare_layer(l) for l in layers]
        self.hq, self.hkv, self.d = n_q_heads, n_kv_heads, head_dim
        self.theta, self.norm_eps = rope_theta, norm_eps
        self.status = torch.zeros(1, dtype=torch.int32, device=self.device)
        self.cos_sin = None
        self.planned = None
        self.marker = None
        self.stage_prefix = ""

    def _mark(self, name):
        if self.marker is not None:
            self.marker(self.stage_prefix + name)

    def plan(self, lengths, hidden):
        lengths = [int(x) for x in lengths]
        cu = [0]
        for n in lengths:
            cu.append(cu[-1] + n)
        cu_h = _host_i32(cu)
        T = cu[-1]
        dev = self.device
        max_pos = max(lengths) if lengths else 1
        if self.cos_sin is None or self.cos_sin.shape[0] < max_pos:
            self.cos_sin = tg_rope_table(max_pos, self.d, self.theta, device=dev)
        pos = torch.cat([torch.arange(n, dtype=torch.int32) for n in lengths]) if T else \
            torch.zeros(0, dtype=torch.int32)
        bf = dict(dtype=torch.bfloat16, device=dev)
        nqkv = (self.hq + 2 * self.hkv) * self.d
        self.planned = dict(
            T=T, cu_h=cu_h, cu=cu_h.to(dev), pos=pos.to(dev),
            bias=torch.zeros(T, dtype=torch.float32, device=dev),
            gamma=torch.zeros(self.hq, dtype=torch.float32, device=dev),
            x=torch.empty((T, hidden), **bf),
            ssq=torch.empty((T, hidden // 128), dtype=torch.float32, device=dev),
            qkv=torch.empty((T, nqkv), **bf),
            o=torch.empty((T, self.hq * self.d), **bf),
            attn_ws=torch.zeros(tg_gated_attention_workspace_size(cu_h, self.hq, self.hkv,
                                                                  self.d),
                                dtype=torch.uint8, device=dev),
            caches=[(torch.empty((T, self.hkv * self.d), **bf),
                     torch.empty((T, self.hkv * self.d), **bf)) for _ in self.layers],
            ffn=torch.empty((T, max([L.ffn for L in self.layers] + [0])), **bf),
            gemm_ws=torch.zeros(tg_gemm_workspace_size(), dtype=torch.uint8, device=dev),
        )
        return self.planned

    def run(self, h, stream=None):
        """All layers on all rows of h (left untouched); returns the final residual."""
        P = self.planned
        if P["T"] == 0:
            return P["x"]
        nq = self.hq * self.d
        qkv, o, x = P["qkv"], P["o"], P["x"]
        tg_gather_rope(h, x, row_ssq=P["ssq"], status=self.status, stream=stream)
        for L, (ck, cv) in zip(self.layers, P["caches"]):
            tg_qkv_rope_cache(x, L.Wqkv, P["pos"], self.cos_sin, ck, cv, self.hq, self.hkv,
                              q_out=qkv[:, :nq], head_dim=self.d, eps=self.norm_eps,
                              row_ssq=P["ssq"], status=self.status, stream=stream,
                              q_norm_w=L.q_norm, k_norm_w=L.k_norm, workspace=P["gemm_ws"])
            self._mark("qkv_rope_cache")
            tg_gated_attention(qkv[:, :nq], ck, cv, P["cu"], P["cu_h"], self.hq, self.hkv,
                               P["pos"], P["bias"], P["gamma"], 1.0, o=o, head_dim=self.d,
                               workspace=P["attn_ws"], status=self.status, stream=stream)
            self._mark("attention")
            tg_linear(o, L.Wo, x, residual=x, row_ssq=P["ssq"], status=self.status,
                      stream=stream,
                      workspace=P["gemm_ws"])
            self._mark("out_proj")
            _mlp(L, x, P, self.norm_eps, self.status, stream, self._mark)
        return x

    def trim(self, kept_idx, out=None, stream=None):
        """Keep only the kept rows of every layer's cache (lower-layer KV trimming).
        `out`: list of (k, v) [K, Hkv d] bf16 pairs to fill, else allocated."""
        P = self.planned
        K = kept_idx.numel()
        if out is None:
            out = [(torch.empty((K, self.hkv * self.d), dtype=torch.bfloat16,
                                device=self.device),
                    torch.empty((K, self.hkv * self.d), dtype=torch.bfloat16,
                                device=self.device)) for _ in self.layers]
        if K:
            for (ck, cv), (tk, tv) in zip(P["caches"], out):
                tg_kv_compact(ck, cv, tk, tv, row_idx=kept_idx, status=self.status,
                              stream=stream)
        return out


class GatedPrefill:
    """Buffers and call sequence of one gated prefill step on one device.

    ``plan`` fixes the request layout (host work: lengths, question sizes, budgets ->
    cu_kept) and allocates the device buffers; ``run`` then only launches kernels on
    the stream, with no host synchronisation.
    """

    def __init__(self, gate: dict, layers: list, n_q_heads=16, n_kv_heads=8, head_dim=128,
                 rope_theta=1.0e6, norm_eps=1e-6, seq_eps=1e-6, device="cuda", lower=None,
                 trim_lower_kv=True):
        """`lower`: optional FullContextLayers below the gate.  The gate then scores
        their output (the residual at the gate layer), the kept rows of that output go
        up, and with `trim_lower_kv` their caches are trimmed to the kept rows."""
        self.device = torch.device(device)
        self.lower = lower
        self.trim_lower_kv = trim_lower_kv
        self.gate = gate
        # the scorer's RMSNorm weight, folded into W1 once (the same bf16 products
        # tg_gate_score would form on every call)
        self._w1 = (tg_fold_norm_weight(gate["W1"], gate["norm_w"])
                    if gate.get("norm_w") is not None else gate["W1"])
        self.layers = [prepare_layer(l) for l in layers]
        self.hq, self.hkv, self.d = n_q_heads, n_kv_heads, head_dim
        self.theta = rope_theta
        self.norm_eps, self.seq_eps = norm_eps, seq_eps
        self.hidden = gate["W1"].shape[1]
        self.width = gate["W1"].shape[0]
        self.cos_sin = None
        self.status = torch.zeros(1, dtype=torch.int32, device=self.device)
        if lower is not None:
            lower.status = self.status  # one status word for the whole step
            lower.stage_prefix = "lower_"
        self.planned = None
        # optional callable(stage_name) invoked after each launch (e.g. to record events)
        self.marker = None
        # QKV projection, RoPE and KV-cache write as one fused kernel (else three)
        self.fused_qkv = True
        # optional: while layer i's attention runs, a side stream pulls that layer's Wo
        # and the next layer's Wqkv into L2 (measured slower on the 16k and 128k steps:
        # off by default)
        self.prefetch_weights = False
        self._side = None
        # optional: one launch per layer boundary, layer i's output projection and layer
        # i+1's QKV (tg_out_proj_qkv_next).  Measured 0.9% slower at the 16k step (2.260
        # against 2.239 ms) and 0.8% faster at 128k (27.56 against 27.78 ms): off by
        # default.
        self.fuse_boundaries = False
        # share the projections' last round of tiles along K over all CTA pairs (stream-K):
        # measured slower at the 16k kept count (QKV 45 -> 53 us, output projection 29 ->
        # 39 us), so off by default
        self.split_gemm = False
        # RoPE in the QKV epilogue from a per-row table built once per step
        # (tg_rope_rows), whose blocks are contiguous across a warp's rows: the same bits
        # as the position table; with the first half's blocks loaded before the
        # accumulator wait, the 16k step takes 2.27 instead of 2.34 ms (one more launch)
        self.rope_rows = True
        self._qkv_done = -1  # index of the layer whose QKV already ran in a fused launch
        self._graph = None   # CUDA graph of the layers above the gate (upper_layers(graph=True))
        self._graph_key_cur = None
        self.graph_captures = 0  # graphs captured by upper_layers(graph=True)
        self._upper_gen = 0

    def _mark(self, name):
        if self.marker is not None:
            self.marker(name)

    def plan(self, lengths, n_question, budgets, k_pad=None):
        """Fix the request layout and allocate the step's buffers.

        `k_pad`: rows of the layers above the gate (>= the kept total K).  The layers then
        run on a fixed row count whatever K a call keeps: rows [K, k_pad) are padding that
        the last request takes as extra trailing rows (see `padded_layout`), so one CUDA
        graph of those layers (`upper_layers(..., graph=True)`) serves every later plan
        with the same padded layout.  A re-plan with the same padded layout keeps the
        upper buffers (and the graph); only the gate's buffers follow the new lengths."""
        lengths = [int(x) for x in lengths]
        cu = [0]
        for n in lengths:
            cu.append(cu[-1] + n)
        cu_h = _host_i32(cu)
        ck_h = tg_plan_kept(cu_h, n_question, budgets)
        T, K = cu[-1], int(ck_h[-1])
        up_h = padded_layout(ck_h, k_pad)
        R = int(up_h[-1])
        dev = self.device
        max_pos = max(lengths) if lengths else 1
        if self.cos_sin is None or self.cos_sin.shape[0] < max_pos:
            self.cos_sin = tg_rope_table(max_pos, self.d, self.theta, device=dev)
        f32 = dict(dtype=torch.float32, device=dev)
        up_key = (tuple(up_h.tolist()), k_pad is not None)
        prev = self.planned
        if k_pad is not None and prev is not None and prev.get("up_key") == up_key:
            upper = {k: prev[k] for k in self._UPPER_KEYS}
        else:
            upper = self._upper_buffers(up_h)
        upper["up_key"] = up_key
        if R > K:  # padding rows: h row 0 at position 0 with zero bias (finite, unused)
            for k in ("kept_idx", "kept_pos", "kept_bias"):
                upper[k][K:].zero_()
        self.planned = dict(
            T=T, K=K, R=R, cu_h=cu_h, ck_h=ck_h,
            cu=cu_h.to(dev), ck=ck_h.to(dev),
            s=torch.empty(T, **f32), z=torch.empty(T, **f32), bias=torch.empty(T, **f32),
            ws=torch.empty(tg_gate_score_workspace_size(T, self.hidden, self.width,
                                                        len(lengths)), dtype=torch.uint8,
                           device=dev),
            **upper,
        )
        if self.lower is not None:
            bf = dict(dtype=torch.bfloat16, device=dev)
            self.lower.plan(lengths, self.hidden)
            if self.trim_lower_kv:
                self.planned["lower_caches"] = [
                    (torch.empty((K, self.hkv * self.d), **bf),
                     torch.empty((K, self.hkv * self.d), **bf)) for _ in self.lower.layers]
        return self.planned

    _UPPER_KEYS = ("up_gen", "up_h", "up", "kept_idx", "kept_pos", "kept_bias", "rot", "x",
                   "ssq", "qkv", "o", "attn_ws", "caches", "chain_ws", "gemm_ws", "ffn")

    def _upper_buffers(self, up_h):
        """Buffers of the layers above the gate for the row layout `up_h` (R rows)."""
        R = int(up_h[-1])
        dev = self.device
        f32 = dict(dtype=torch.float32, device=dev)
        bf = dict(dtype=torch.bfloat16, device=dev)
        nqkv = (self.hq + 2 * self.hkv) * self.d
        self._upper_gen += 1
        return dict(
            up_gen=self._upper_gen,  # which allocation these are (a graph is tied to one)
            up_h=up_h, up=up_h.to(dev),
            kept_idx=torch.zeros(R, dtype=torch.int32, device=dev),
            kept_pos=torch.zeros(R, dtype=torch.int32, device=dev),
            kept_bias=torch.zeros(R, **f32),
            rot=torch.empty((self.d // 4, max(R, 1), 4), **f32),
            x=torch.empty((R, self.hidden), **bf),
            ssq=torch.empty((R, self.hidden // 128), **f32),
            qkv=torch.empty((R, nqkv), **bf),
            o=torch.empty((R, self.hq * self.d), **bf),
            attn_ws=torch.zeros(tg_gated_attention_workspace_size(up_h, self.hq, self.hkv,
                                                                  self.d),
                                dtype=torch.uint8, device=dev),
            caches=[(torch.empty((R, self.hkv * self.d), **bf),
                     torch.empty((R, self.hkv * self.d), **bf)) for _ in self.layers],
            chain_ws=torch.zeros(max(16, tg_out_proj_qkv_workspace_size(R)), dtype=torch.uint8,
                                 device=dev),
            # stream-K tail of the projections (zero-filled; empty = unsplit)
            gemm_ws=torch.zeros(tg_gemm_workspace_size() if self.split_gemm else 0,
                                dtype=torch.uint8, device=dev),
            ffn=torch.empty((R, max([L.ffn for L in self.layers] + [0])), **bf),
        )

    def score(self, h, prunable, stream=None):
        P = self.planned
        g = self.gate
        tg_gate_score(h, self._w1, g["w2"], P["cu"], P["cu_h"], prunable, norm_w=None,
                      eps_norm=self.norm_eps, eps_seq=self.seq_eps, s_out=P["s"], z_out=P["z"],
                      bias_out=P["bias"], workspace=P["ws"], status=self.status, stream=stream)
        self._mark("gate_score")

    def select(self, prunable, z=None, stream=None):
        P = self.planned
        tg_topk_compact(P["z"] if z is None else z, prunable, P["cu"], P["cu_h"], P["ck"],
                        P["ck_h"], P["kept_idx"], P["kept_pos"], P["kept_bias"],
                        status=self.status, stream=stream)
        self._mark("topk_compact")

    def gather(self, h, stream=None):
        """x = h[kept_idx]: the kept rows go up, pruned rows stop here."""
        P = self.planned
        if P["K"]:
            tg_gather_rope(h, P["x"], row_idx=P["kept_idx"], row_ssq=P["ssq"], status=self.status,
                           stream=stream)
            self._mark("gather")
            if self.rope_rows:
                tg_rope_rows(P["kept_pos"], self.cos_sin, out=P["rot"], status=self.status,
                             stream=stream)
                self._mark("rope_rows")

    def _rope(self):
        """(pos, table) arguments of the QKV entry points for the kept rows."""
        P = self.planned
        return (None, P["rot"]) if self.rope_rows else (P["kept_pos"], self.cos_sin)

    def _fusable(self):
        nq, nkv = self.hq * self.d, self.hkv * self.d
        plain = all(L.q_norm is None and L.W_gu is None for L in self.layers)
        return (self.fused_qkv and self.hidden % 256 == 0 and nq % 256 == 0 and nkv % 256 == 0
                and self.d == 128 and plain)

    def layer(self, i, stream=None, fuse_next=False):
        """Upper layer i on the kept rows, in place on x; K/V land in cache i.  With
        `fuse_next`, layer i's output projection and layer i+1's QKV run as one launch
        (then layer i+1 skips its QKV)."""
        P = self.planned
        if P["K"] == 0:
            return
        L = self.layers[i]
        ck, cv = P["caches"][i]
        nq, nk = self.hq * self.d, self.hkv * self.d
        qkv, o, x = P["qkv"], P["o"], P["x"]
        if self._qkv_done == i:
            pass  # ran with the previous layer's output projection
        elif self.fused_qkv or L.q_norm is not None:
            rpos, rtab = self._rope()
            tg_qkv_rope_cache(x, L.Wqkv, rpos, rtab, ck, cv, self.hq, self.hkv,
                              q_out=qkv[:, :nq], head_dim=self.d, eps=self.norm_eps,
                              row_ssq=P["ssq"], status=self.status, stream=stream,
                              q_norm_w=L.q_norm, k_norm_w=L.k_norm, workspace=P["gemm_ws"])
            self._mark("qkv_rope_cache")
        else:
            tg_linear(x, L.Wqkv, qkv, rmsnorm=True, eps=self.norm_eps, status=self.status,
                      stream=stream)
            self._mark("qkv_proj")
            tg_gather_rope(qkv, qkv, rope_pos=P["kept_pos"], rope_cols=(0, nq + nk),
                           head_dim=self.d, cos_sin=self.cos_sin, status=self.status,
                           stream=stream)
            self._mark("rope")
            tg_kv_compact(qkv[:, nq:nq + nk], qkv[:, nq + nk:], ck, cv, status=self.status,
                          stream=stream)
            self._mark("kv_compact")
        if self.prefetch_weights:
            main = stream if stream is not None else torch.cuda.current_stream(self.device)
            if self._side is None:
                self._side = torch.cuda.Stream(device=self.device)
            self._side.wait_stream(main)
            tg_prefetch_l2(L.Wo, stream=self._side)
            if i + 1 < len(self.layers):
                tg_prefetch_l2(self.layers[i + 1].Wqkv, stream=self._side)
        tg_gated_attention(qkv[:, :nq], ck, cv, P["up"], P["up_h"], self.hq, self.hkv,
                           P["kept_pos"], P["kept_bias"], L.gamma, L.beta, o=o,
                           head_dim=self.d, workspace=P["attn_ws"], status=self.status,
                           stream=stream)
        self._mark("attention")
        if fuse_next and i + 1 < len(self.layers) and self._fusable():
            Ln = self.layers[i + 1]
            ckn, cvn = P["caches"][i + 1]
            rpos, rtab = self._rope()
            tg_out_proj_qkv_next(o, L.Wo, x, P["ssq"], Ln.Wqkv, rpos, rtab, ckn,
                                 cvn, self.hq, self.hkv, qkv[:, :nq], P["chain_ws"],
                                 head_dim=self.d, eps=self.norm_eps, status=self.status,
                                 stream=stream)
            self._qkv_done = i + 1
            self._mark("out_proj_qkv")
        else:
            tg_linear(o, L.Wo, x, residual=x, row_ssq=P["ssq"], status=self.status, stream=stream,
                      workspace=P["gemm_ws"])
            self._mark("out_proj")
        _mlp(L, x, P, self.norm_eps, self.status, stream, self._mark)

    def _layers(self, stream=None):
        self._qkv_done = -1
        for i in range(len(self.layers)):
            self.layer(i, stream=stream, fuse_next=self.fuse_boundaries)
        self._qkv_done = -1
        if self._side is not None:  # join the prefetch stream (a captured graph needs it)
            main = stream if stream is not None else torch.cuda.current_stream(self.device)
            main.wait_stream(self._side)

    def _graph_key(self):
        P = self.planned
        # the position table is read inside the layers only without the per-row table
        table = 0 if self.rope_rows else self.cos_sin.data_ptr()
        return (P["up_key"], P["up_gen"], table, self.rope_rows, self.fuse_boundaries,
                self.fused_qkv, self.prefetch_weights, tg_get_launch_overlap())

    def upper_layers(self, h, stream=None, graph=False):
        """The kept rows' way up: the gather, then every layer above the gate.

        With `graph`, the layers (not the gather, whose source rows change from call to
        call) run as one CUDA graph captured for the planned row layout.  The first such
        call runs them eagerly and captures the graph; later calls with the same layout
        (the same `k_pad` bucket and the same buffers) replay it."""
        self.gather(h, stream=stream)
        if not graph or self.planned["K"] == 0:
            self._layers(stream)
            return
        main = stream if stream is not None else torch.cuda.current_stream(self.device)
        key = self._graph_key()
        if self._graph is not None and self._graph_key_cur == key:
            with torch.cuda.stream(main):
                self._graph.replay()
            return
        self._graph = None
        self._layers(main)  # this call's result, and the kernels' one-time set-up
        side = torch.cuda.Stream(device=self.device)
        side.wait_stream(main)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=side):
            self._layers(side)
        main.wait_stream(side)
        self._graph, self._graph_key_cur = g, key
        self.graph_captures += 1

    def run(self, h, prunable, scores=None, stream=None, graph=False):
        """One gated prefill step.  With lower layers, h is the model's input rows and
        the lower layers run first on all of them.  The scorer always runs on the
        gate layer's residual; with `scores` (raw per-token scores, fp32 [T]) selection
        uses the sequence-normalised `scores` instead of the scorer's own (the drawn
        planted-cluster workload)."""
        if self.lower is not None:
            self.lower.marker = self.marker
            h = self.lower.run(h, stream=stream)
            self.lower.marker = None
        self.score(h, prunable, stream=stream)
        if scores is not None:
            P = self.planned
            tg_seq_rmsnorm(scores, P["cu"], P["cu_h"], prunable, self.seq_eps, P["z"],
                           P["bias"], stream=stream)
            self._mark("seq_rmsnorm")
        self.select(prunable, stream=stream)
        if self.lower is not None and self.trim_lower_kv:
            P = self.planned
            self.lower.trim(P["kept_idx"][:P["K"]], out=P["lower_caches"], stream=stream)
            self._mark("lower_kv_trim")
        self.upper_layers(h, stream=stream, graph=graph)
        return self.planned
