"""fp64 forward of a Llama-architecture decoder stack and the layer-wise
sensitivity scores built on it.

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``: only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py``'s CPU legs may import it, and
the CUDA library shares no code with it.

Layer-wise sensitivity [TS §2.1 "Laaggewijze Sensitiviteit"]: the L2 error at
the model's final output when one linear layer alone is quantised.  The
pages name the measure, not the model code, so the readings are:
  * the model is the random-init decoder stack of the workload (no embedding
    table or LM head: synthetic hidden states go in, the final-normed hidden
    states come out); each block is the Llama block -- pre-norm RMSNorm
    (weight 1), q/k/v projections, rotary position embedding (rotate-half
    form, base theta), causal grouped-query softmax attention, o projection
    and residual, RMSNorm, SwiGLU MLP (silu(gate) * up, then down) and
    residual; a final RMSNorm gives the output;
  * "quantised" is the W4A4 MXINT4 linear of the library: the layer's input
    activations and weight both in the uniform 4-bit layout {0, 0, K}
    (blocks of 32 along K), their fp64 product rounded once to bf16 (the
    library's output type);
  * the score is the Frobenius norm of (output with that layer quantised)
    minus (output of the unquantised stack), over all tokens and features.
Everything else is plain fp64.

Weights are given per block as a 7-tuple in the order q, k, v, o, gate, up,
down, each an (out x in) array; layer index = 7 * block + position.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

import oracle

LINEARS = ("q", "k", "v", "o", "gate", "up", "down")


@dataclass
class StackConfig:
    hidden: int
    n_heads: int
    n_kv_heads: int
    mlp: int
    rms_eps: float = 1e-5
    rope_theta: float = 500000.0

    @property
    def head_dim(self) -> int:
        return self.hidden // self.n_heads


def rms_norm(x: np.ndarray, eps: float) -> np.ndarray:
    """x / sqrt(mean(x^2) + eps), per row (weight 1)."""
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)


def rope(x: np.ndarray, n_heads: int, theta: float) -> np.ndarray:
    """Rotary embedding of a (T x n_heads*d) projection, token t at position
    t: within each head, pair (i, i + d/2) turns by the angle t * theta^(-2i/d)."""
    T, width = x.shape
    d = width // n_heads
    half = d // 2
    out = x.copy()
    inv = theta ** (-2.0 * np.arange(half) / d)
    for t in range(T):
        ang = t * inv
        c, s = np.cos(ang), np.sin(ang)
        for h in range(n_heads):
            a = x[t, h * d:h * d + half]
            b = x[t, h * d + half:(h + 1) * d]
            out[t, h * d:h * d + half] = a * c - b * s
            out[t, h * d + half:(h + 1) * d] = a * s + b * c
    return out


def causal_attention(q, k, v, n_heads: int, n_kv_heads: int) -> np.ndarray:
    """Causal softmax attention, query head h on kv head h // (n_heads / n_kv_heads);
    scores scaled by 1/sqrt(d)."""
    T = q.shape[0]
    d = q.shape[1] // n_heads
    rep = n_heads // n_kv_heads
    out = np.zeros_like(q)
    for h in range(n_heads):
        g = h // rep
        qh = q[:, h * d:(h + 1) * d]
        kh = k[:, g * d:(g + 1) * d]
        vh = v[:, g * d:(g + 1) * d]
        for t in range(T):
            s = kh[:t + 1] @ qh[t] / math.sqrt(d)
            p = np.exp(s - s.max())
            p /= p.sum()
            out[t, h * d:(h + 1) * d] = p @ vh[:t + 1]
    return out


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Nearest bf16 value (8 significant bits, ties to even) of each element."""
    m, e = np.frexp(x)                      # x = m 2^e, |m| in [0.5, 1)
    return np.ldexp(np.rint(m * 256.0), e - 8)


def quantized_linear(x: np.ndarray, W: np.ndarray) -> np.ndarray:
    """W4A4 MXINT4 product of the library: both operands in the uniform 4-bit
    layout, fp64 product of the decoded values, rounded once to bf16."""
    K = x.shape[1]
    counts = (0, 0, K)
    ac, as_ = oracle.quantize_rows(x, None, counts)
    wc, ws = oracle.quantize_rows(W, None, counts)
    return round_bf16(oracle.gemm(ac, as_, wc, ws, counts))


def block_forward(h: np.ndarray, Ws, cfg: StackConfig, quant: int = -1) -> np.ndarray:
    """One block; linear `quant` (0..6) runs quantised, the others in fp64."""
    lin = lambda i, x: quantized_linear(x, Ws[i]) if i == quant else x @ Ws[i].T
    a = rms_norm(h, cfg.rms_eps)
    q = rope(lin(0, a), cfg.n_heads, cfg.rope_theta)
    k = rope(lin(1, a), cfg.n_kv_heads, cfg.rope_theta)
    v = lin(2, a)
    h = h + lin(3, causal_attention(q, k, v, cfg.n_heads, cfg.n_kv_heads))
    a = rms_norm(h, cfg.rms_eps)
    g = lin(4, a)
    u = lin(5, a)
    return h + lin(6, g / (1.0 + np.exp(-g)) * u)


def stack_output(x: np.ndarray, blocks, cfg: StackConfig, quant_layer: int = -1) -> np.ndarray:
    h = np.asarray(x, dtype=np.float64)
    for b, Ws in enumerate(blocks):
        h = block_forward(h, Ws, cfg, quant_layer - 7 * b if quant_layer // 7 == b else -1)
    return rms_norm(h, cfg.rms_eps)


def layer_scores(x: np.ndarray, blocks, cfg: StackConfig, layers=None) -> np.ndarray:
    """Score of every linear layer (or of the listed ones): ||F_l - F||_2."""
    ref = stack_output(x, blocks, cfg)
    idx = range(7 * len(blocks)) if layers is None else layers
    return np.array([np.sqrt(np.sum((stack_output(x, blocks, cfg, l) - ref) ** 2)) for l in idx])
