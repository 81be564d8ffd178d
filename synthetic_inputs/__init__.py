"""Seeded synthetic workloads for the TokenGate gate layer and token-gated attention.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic (no normalisation, selection, attention or budget rule).
Both the CPU oracle and the CUDA path take their inputs from here, so that the two
see bit-identical tensors.

Shapes follow the Qwen3-1.7B-sized setting the pages evaluate on (hidden 2048,
16 query heads, 8 KV heads, head_dim 128, RoPE theta 1e6), with a 2048 -> 256 -> 1
scoring MLP.  The pages' own workloads are long-document prompts (NIAH, 2Wiki,
RepoBench-P, MultiNews, BioDEX); none of their items are used: every tensor here
is drawn from a seeded generator.

Recipe (all draws on the CPU with ``torch.Generator``):
  * residual rows h ~ N(0, 1), rounded to bf16, one generator per request seed;
  * gate weights: RMSNorm weight = 1, W1 [F, H] ~ N(0, 0.02) bf16, w2 [F] ~ N(0, 0.02) fp32;
  * layer l weights: Wqkv [Hq*d + 2*Hkv*d, H] ~ N(0, 0.02) bf16 (rows: Wq, then Wk,
    then Wv), Wo [H, Hq*d] ~ N(0, 0.02) bf16, gamma [Hq] ~ U(0.5, 2) fp32, beta = 1;
  * layers below the gate (full context): Wqkv and Wo drawn the same way from their
    own stream, no gamma or beta;
  * full layer body (optional): attention-norm weight [H], QK-norm weights [d] and the
    MLP norm weight [H] ~ U(0.8, 1.2) fp32; W_gate, W_up [F, H] and W_down [H, F]
    ~ N(0, 0.02) bf16 with F = 6144, from their own stream;
  * prunable mask: the first D_b tokens of each request are the document (prunable),
    the last Q_b tokens are the question (never pruned);
  * drawn scores (planted-cluster workload): s ~ N(0, 1) fp32 with +4 added on 64
    consecutive document tokens at a seeded offset.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

HIDDEN = 2048
SCORER_WIDTH = 256
N_Q_HEADS = 16
N_KV_HEADS = 8
HEAD_DIM = 128
ROPE_THETA = 1.0e6
NORM_EPS = 1.0e-6
SEQ_EPS = 1.0e-6

# Generator seeds for weight streams are derived from the workload's weight seed so
# that weights do not depend on how many residual rows were drawn before them.
_GATE_STREAM = 1_000_001
_LAYER_STREAM = 2_000_003
_LAYOUT_STREAM = 3_000_017
_SCORE_STREAM = 4_000_037
_LOWER_STREAM = 5_000_011
_BODY_STREAM = 6_000_023
FFN = 6144  # SwiGLU width of the Qwen3-1.7B-shaped layer


@dataclass(frozen=True)
class Workload:
    """One synthetic prefill batch: per-request lengths, question sizes, budgets."""

    name: str
    lengths: tuple            # N_b, tokens per request
    questions: tuple          # Q_b, non-prunable tokens per request (at the end)
    budgets: tuple            # max kept prefill tokens per request
    n_layers: int
    seeds: tuple              # residual-row seed per request
    weight_seed: int = 0
    planted_cluster: bool = False
    dense: bool = False       # gamma = 0 and beta = 1 for every layer
    hidden: int = HIDDEN
    scorer_width: int = SCORER_WIDTH
    n_q_heads: int = N_Q_HEADS
    n_kv_heads: int = N_KV_HEADS
    head_dim: int = HEAD_DIM
    rope_theta: float = ROPE_THETA
    notes: str = field(default="", compare=False)

    @property
    def batch(self) -> int:
        return len(self.lengths)

    @property
    def total_tokens(self) -> int:
        return int(sum(self.lengths))

    def cu_seqlens(self) -> list:
        out = [0]
        for n in self.lengths:
            out.append(out[-1] + int(n))
        return out


def pr1_ref() -> Workload:
    """N=1024 (960 document + 64 question), budget 256, one gated layer, seed 0."""
    return Workload("n1k_k256_l1", (1024,), (64,), (256,), 1, (0,))


def n16k() -> Workload:
    """N=16384 (16320 + 64), budget floor(0.1 N)=1638, 28 stacked gated layers."""
    return Workload("n16k_k1638_l28", (16384,), (64,), (1638,), 28, (0,))


def n32k_sweep(ratio: float) -> Workload:
    """N=32768 (32704 + 64), budget floor(ratio N); ratio 1.0 is the dense point."""
    n = 32768
    budget = int(math.floor(ratio * n))
    dense = ratio >= 1.0
    return Workload(f"n32k_r{ratio:g}_l1", (n,), (64,), (budget,), 1, (0,), dense=dense)


N32K_RATIOS = (0.01, 0.05, 0.25, 1.0)


def n128k() -> Workload:
    """N=131072 (131008 + 64), budget 13107, 28 layers, drawn scores with a planted cluster."""
    return Workload("n128k_k13107_l28", (131072,), (64,), (13107,), 28, (0,),
                    planted_cluster=True)


def ragged8(layout_seed: int = 0) -> Workload:
    """8 packed requests: N_b ~ U{4096..32768}, Q_b ~ U{16..256},
    keep ratio ~ log-uniform in [0.02, 0.5], budget max(Q_b, floor(ratio N_b)); seeds 0..7."""
    g = torch.Generator().manual_seed(_LAYOUT_STREAM + layout_seed)
    lengths, questions, budgets = [], [], []
    for _ in range(8):
        n = int(torch.randint(4096, 32769, (1,), generator=g))
        q = int(torch.randint(16, 257, (1,), generator=g))
        u = float(torch.rand((1,), generator=g, dtype=torch.float64))
        ratio = math.exp(math.log(0.02) + u * (math.log(0.5) - math.log(0.02)))
        lengths.append(n)
        questions.append(q)
        budgets.append(max(q, int(math.floor(ratio * n))))
    return Workload("ragged8_varlen_l1", tuple(lengths), tuple(questions), tuple(budgets),
                    1, tuple(range(8)))


def custom(lengths, questions, budgets, n_layers=1, seeds=None, **kw) -> Workload:
    """Small ad-hoc workloads for tests (any lengths, questions at the end)."""
    seeds = tuple(seeds) if seeds is not None else tuple(range(len(lengths)))
    return Workload(kw.pop("name", "custom"), tuple(int(x) for x in lengths),
                    tuple(int(x) for x in questions), tuple(int(x) for x in budgets),
                    n_layers, seeds, **kw)


def all_workloads() -> dict:
    out = {"n1k": pr1_ref(), "n16k": n16k(), "n128k": n128k(), "ragged8": ragged8()}
    for r in N32K_RATIOS:
        out[f"n32k_r{r:g}"] = n32k_sweep(r)
    return out


# ----------------------------------------------------------------------------- draws

def hidden_rows(wl: Workload) -> torch.Tensor:
    """Packed residual rows [T, hidden] bf16, request b drawn from generator seed wl.seeds[b]."""
    parts = []
    for n, seed in zip(wl.lengths, wl.seeds):
        g = torch.Generator().manual_seed(int(seed))
        parts.append(torch.randn((int(n), wl.hidden), generator=g, dtype=torch.float32)
                     .to(torch.bfloat16))
    return parts[0] if len(parts) == 1 else torch.cat(parts, 0)


def gate_weights(wl: Workload) -> dict:
    g = torch.Generator().manual_seed(_GATE_STREAM + wl.weight_seed)
    norm_w = torch.ones(wl.hidden, dtype=torch.float32)
    W1 = (torch.randn((wl.scorer_width, wl.hidden), generator=g) * 0.02).to(torch.bfloat16)
    w2 = (torch.randn((wl.scorer_width,), generator=g) * 0.02).to(torch.float32)
    return {"norm_w": norm_w, "W1": W1, "w2": w2}


def layer_weights(wl: Workload, layer: int) -> dict:
    g = torch.Generator().manual_seed(_LAYER_STREAM + 7919 * wl.weight_seed + layer)
    hq, hkv, d, H = wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.hidden
    Wqkv = (torch.randn(((hq + 2 * hkv) * d, H), generator=g) * 0.02).to(torch.bfloat16)
    Wo = (torch.randn((H, hq * d), generator=g) * 0.02).to(torch.bfloat16)
    gamma = (0.5 + 1.5 * torch.rand((hq,), generator=g)).to(torch.float32)
    beta = 1.0
    if wl.dense:
        gamma = torch.zeros_like(gamma)
    return {"Wqkv": Wqkv, "Wo": Wo, "gamma": gamma, "beta": beta}


def lower_layer_weights(wl: Workload, n_layers: int) -> list:
    """Weights of `n_layers` full-context layers below the gate: Wqkv, Wo only."""
    hq, hkv, d, H = wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.hidden
    out = []
    for layer in range(n_layers):
        g = torch.Generator().manual_seed(_LOWER_STREAM + 7919 * wl.weight_seed + layer)
        Wqkv = (torch.randn(((hq + 2 * hkv) * d, H), generator=g) * 0.02).to(torch.bfloat16)
        Wo = (torch.randn((H, hq * d), generator=g) * 0.02).to(torch.bfloat16)
        out.append({"Wqkv": Wqkv, "Wo": Wo})
    return out


def layer_body_parts(wl: Workload, layer: int, lower: bool = False, ffn: int = FFN) -> dict:
    """The optional parts of a full layer body for layer `layer` (above the gate, or
    below it with `lower`): attn_norm, q_norm, k_norm and mlp (norm_w, W_gate, W_up,
    W_down)."""
    H, d = wl.hidden, wl.head_dim
    g = torch.Generator().manual_seed(_BODY_STREAM + 7919 * wl.weight_seed + 104729 * int(lower)
                                      + layer)

    def gain(n):
        return (0.8 + 0.4 * torch.rand((n,), generator=g)).to(torch.float32)

    attn_norm, q_norm, k_norm = gain(H), gain(d), gain(d)
    mlp_norm = gain(H)
    W_gate = (torch.randn((ffn, H), generator=g) * 0.02).to(torch.bfloat16)
    W_up = (torch.randn((ffn, H), generator=g) * 0.02).to(torch.bfloat16)
    W_down = (torch.randn((H, ffn), generator=g) * 0.02).to(torch.bfloat16)
    return {"attn_norm": attn_norm, "q_norm": q_norm, "k_norm": k_norm,
            "mlp": {"norm_w": mlp_norm, "W_gate": W_gate, "W_up": W_up, "W_down": W_down}}


def prunable_mask(wl: Workload) -> torch.Tensor:
    """uint8 [T]: 1 on document tokens (first N_b - Q_b of each request), 0 on the question."""
    parts = []
    for n, q in zip(wl.lengths, wl.questions):
        m = torch.ones(int(n), dtype=torch.uint8)
        if q:
            m[int(n) - int(q):] = 0
        parts.append(m)
    return parts[0] if len(parts) == 1 else torch.cat(parts, 0)


def drawn_scores(wl: Workload) -> torch.Tensor:
    """fp32 [T] raw scores ~N(0,1) with a +4 cluster of 64 tokens at a seeded document offset."""
    parts = []
    for n, q, seed in zip(wl.lengths, wl.questions, wl.seeds):
        g = torch.Generator().manual_seed(_SCORE_STREAM + int(seed))
        s = torch.randn((int(n),), generator=g, dtype=torch.float32)
        doc = int(n) - int(q)
        if doc >= 64:
            o = int(torch.randint(0, doc - 64 + 1, (1,), generator=g))
            s[o:o + 64] += 4.0
        parts.append(s)
    return parts[0] if len(parts) == 1 else torch.cat(parts, 0)


def random_like_scores(n: int, seed: int, ties: bool = False) -> torch.Tensor:
    """fp32 scores for selection tests; with ties=True values repeat on a coarse grid."""
    g = torch.Generator().manual_seed(seed)
    s = torch.randn((n,), generator=g, dtype=torch.float32)
    if ties:
        s = torch.round(s * 4.0) / 4.0
    return s


def uniform_rows(rows: int, cols: int, seed: int, scale: float = 1.0,
                 dtype=torch.bfloat16) -> torch.Tensor:
    """N(0, scale) rows of any shape (test tensors for Q/K/V and projections)."""
    g = torch.Generator().manual_seed(seed)
    return (torch.randn((rows, cols), generator=g) * scale).to(dtype)
