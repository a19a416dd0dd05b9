"""fp64 CPU oracle for the forward pass of a quantised top-k routed MoE FFN layer.

TEST INFRASTRUCTURE ONLY.  Nothing in the library's product path may import,
call or link this module: only the tests, the smoke check and the bench's
CPU-baseline leg use it.  It shares no code with the CUDA path (no kernels,
headers, helpers, tables or pre/post-processing); both sides are fed the same
bytes by the seeded input generator, which holds none of the arithmetic below.

Every step is the plain definition, written out in float64 with no
intermediate rounding, in the order the sources state it:

1. Router logits ``z[t,e] = sum_i x[t,i] * Wr[e,i] (+ b[e])``.
   ("Quantized Mixture of Experts (Q-MoE)", section 3 "Components": the gating
   network picks the experts to activate from the input.)
2. Top-k by logit, descending, lower expert index first on ties.
   (Same row: top-k routing, e.g. top-2.)
3. Gates: softmax over all E logits, then the k selected probabilities are
   renormalised to sum to 1.  ("FineRMoE", the paragraph on the Sparse Sum
   Layer: the mixing weights are the router's softmax probabilities.)
4. Expert-centric schedule: every (token, slot) routing decision becomes one
   task; tasks are grouped by expert id (contiguous, ascending) and sorted by
   token id inside each group.  ("OmniMoE: An Efficient MoE by Orchestrating
   Atomic Experts at Scale", section 2.2, "Expert-Centric Scheduling", task
   collection and grouping/sorting.)
5. Expert FFN: gate, up and down matrices with an activation between
   (``h = silu(W1 x) * (W3 x)``, ``y = W2 h``).  ("FineRMoE" architecture
   paragraph: an expert is Up, Gate and Down matrices with an activation.)
6. Combine: ``out[t] = sum_j g[t,j] * y[t,j] + sum_s y_shared[s,t]``; shared
   experts are always active with weight 1.  ("OmniMoE", section 2.1, the
   shared dense MLP that every input activates.)

Dequantisation ("Quantized Mixture of Experts (Q-MoE)", sections 3 and 4:
per-expert INT8 / FP8 / INT4 precision) is the closed form ``q * scale``:
INT8 per output channel, INT4 with one bf16 scale per 128 consecutive K,
FP8 e4m3 per output channel with the e4m3 code decoded from the format
definition (bias 7, 3 mantissa bits, subnormals m * 2^-9, S.1111.111 = NaN,
no infinities).

Readings where the sources are silent (each also listed in the design notes):
selection is on logits (same order as on probabilities in exact arithmetic);
ties go to the lower expert index; the router bias is added to the logits
and so affects both selection and gate values; shared experts use weight 1.
"""
from __future__ import annotations

import math
from typing import Dict, List, Optional, Sequence

import numpy as np

FMT_INT8 = 1
FMT_INT4 = 2
FMT_FP8 = 3


# ---------------------------------------------------------------------------
# input decoding
# ---------------------------------------------------------------------------
def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> float64 (exact: bf16 is the top half of an fp32)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def decode_e4m3(codes: np.ndarray) -> np.ndarray:
    """e4m3 byte codes -> float64, from the format definition.

    sign = bit 7, exponent = bits 6..3 (bias 7), mantissa = bits 2..0.
    exponent 0: subnormal, value m * 2^-9.  exponent 15 with mantissa 7: NaN.
    There are no infinities.
    """
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = (c >> 7) & 1
    e = (c >> 3) & 0xF
    m = c & 0x7
    mag = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.power(2.0, e - 7))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return np.where(sign == 1, -mag, mag)


def unpack_int4(packed: np.ndarray, K: int) -> np.ndarray:
    """[N][K/2] bytes -> [N][K] int64; low nibble is the even k, two's complement."""
    p = np.asarray(packed, dtype=np.uint8).astype(np.int64)
    lo = p & 0xF
    hi = (p >> 4) & 0xF
    lo = np.where(lo >= 8, lo - 16, lo)
    hi = np.where(hi >= 8, hi - 16, hi)
    N = p.shape[0]
    q = np.empty((N, K), dtype=np.int64)
    q[:, 0::2] = lo
    q[:, 1::2] = hi
    return q


def dequantize(fmt: int, w: np.ndarray, s: np.ndarray, N: int, K: int) -> np.ndarray:
    """Closed form q * scale in float64, shape [N][K]."""
    if fmt == FMT_INT8:
        q = np.asarray(w).view(np.int8).reshape(N, K).astype(np.float64)
        return q * np.asarray(s, dtype=np.float32).astype(np.float64)[:, None]
    if fmt == FMT_INT4:
        q = unpack_int4(np.asarray(w).reshape(N, K // 2), K).astype(np.float64)
        sc = bf16_to_f64(np.asarray(s).reshape(N, K // 128))
        return q * np.repeat(sc, 128, axis=1)
    if fmt == FMT_FP8:
        v = decode_e4m3(np.asarray(w).reshape(N, K))
        return v * np.asarray(s, dtype=np.float32).astype(np.float64)[:, None]
    raise ValueError(f"unknown weight format {fmt}")


# ---------------------------------------------------------------------------
# stage 1: router
# ---------------------------------------------------------------------------
def router_logits(x_bits: np.ndarray, router_w: np.ndarray,
                  router_b: Optional[np.ndarray]) -> np.ndarray:
    """z[t,e] = sum_i x[t,i] Wr[e,i] + b[e], float64."""
    x = bf16_to_f64(x_bits)
    z = x @ np.asarray(router_w, dtype=np.float32).astype(np.float64).T
    if router_b is not None:
        z = z + np.asarray(router_b, dtype=np.float32).astype(np.float64)[None, :]
    return z


def topk(z: np.ndarray, k: int) -> np.ndarray:
    """Brute force: order all experts by (logit descending, index ascending), keep k."""
    z = np.asarray(z, dtype=np.float64)
    T, E = z.shape
    out = np.empty((T, k), dtype=np.int32)
    for t in range(T):
        row = z[t]
        order = sorted(range(E), key=lambda e: (-row[e], e))
        out[t] = order[:k]
    return out


def topk_margin(z: np.ndarray, k: int) -> np.ndarray:
    """Gap between the k-th and (k+1)-th largest logit per token (inf when k == E)."""
    z = np.asarray(z, dtype=np.float64)
    T, E = z.shape
    if k >= E:
        return np.full(T, np.inf)
    srt = -np.sort(-z, axis=1)
    return srt[:, k - 1] - srt[:, k]


def gates(z: np.ndarray, idx: np.ndarray) -> np.ndarray:
    """Softmax over all E logits, then renormalise the selected k probabilities."""
    z = np.asarray(z, dtype=np.float64)
    m = z.max(axis=1, keepdims=True)
    ez = np.exp(z - m)
    p = ez / ez.sum(axis=1, keepdims=True)
    sel = np.take_along_axis(p, np.asarray(idx, dtype=np.int64), axis=1)
    return sel / sel.sum(axis=1, keepdims=True)


# ---------------------------------------------------------------------------
# stage 2: expert-centric schedule
# ---------------------------------------------------------------------------
def schedule(idx: np.ndarray, E: int) -> Dict[str, np.ndarray]:
    """Flatten (t, j) decisions into tasks, group by expert, sort by token.

    Returns counts[E], offsets[E+1], sorted_token[T*k] (token of each task in
    grouped order) and inv_pos[T][k] (where task (t, j) landed).
    """
    idx = np.asarray(idx, dtype=np.int64)
    T, k = idx.shape
    tasks = [(int(idx[t, j]), t, j) for t in range(T) for j in range(k)]
    tasks.sort(key=lambda task: (task[0], task[1]))
    counts = np.zeros(E, dtype=np.int32)
    for e, _, _ in tasks:
        counts[e] += 1
    offsets = np.zeros(E + 1, dtype=np.int32)
    for e in range(E):
        offsets[e + 1] = offsets[e] + counts[e]
    sorted_token = np.empty(T * k, dtype=np.int32)
    inv_pos = np.empty((T, k), dtype=np.int32)
    for pos, (_, t, j) in enumerate(tasks):
        sorted_token[pos] = t
        inv_pos[t, j] = pos
    return dict(counts=counts, offsets=offsets, sorted_token=sorted_token, inv_pos=inv_pos)


# ---------------------------------------------------------------------------
# stages 3-4: one expert's gated FFN
# ---------------------------------------------------------------------------
def silu(a: np.ndarray) -> np.ndarray:
    return a / (1.0 + np.exp(-a))


def expert_ffn(xr: np.ndarray, w13: np.ndarray, w2: np.ndarray, I: int) -> np.ndarray:
    """Rows xr [n][d] through one expert: y = W2 (silu(W1 x) * (W3 x)).

    w13 is the dequantised [2I][d] matrix (rows 0..I-1 gate W1, I..2I-1 up W3),
    w2 the dequantised [d][I] down matrix.
    """
    a = xr @ w13[:I].T
    u = xr @ w13[I:].T
    h = silu(a) * u
    return h @ w2.T


def dequantize_expert(ex, d: int, I: int):
    w13 = dequantize(ex.fmt, ex.w13, ex.s13, 2 * I, d)
    w2 = dequantize(ex.fmt, ex.w2, ex.s2, d, I)
    return w13, w2


# ---------------------------------------------------------------------------
# the whole forward
# ---------------------------------------------------------------------------
def route(layer, tokens: Optional[Sequence[int]] = None,
          logits: Optional[np.ndarray] = None) -> Dict[str, np.ndarray]:
    """Stages 1-2 for the given tokens (default all).  ``logits`` (fp32 [T][E])
    replaces the computed logits when given."""
    tok = np.arange(layer.T) if tokens is None else np.asarray(tokens, dtype=np.int64)
    if logits is not None:
        z = np.asarray(logits, dtype=np.float32)[tok].astype(np.float64)
    else:
        z = router_logits(layer.x[tok], layer.router_w, layer.router_b)
    idx = topk(z, layer.k)
    out = dict(logits=z, idx=idx, gates=gates(z, idx), margin=topk_margin(z, layer.k))
    if tokens is None:
        out.update(schedule(idx, layer.E))
    return out


def forward(layer, tokens: Optional[Sequence[int]] = None,
            logits: Optional[np.ndarray] = None,
            idx_override: Optional[np.ndarray] = None) -> Dict[str, np.ndarray]:
    """Layer output (float64) for the given tokens (default: all of them).

    Each expert's weights are dequantised once and applied to every row routed
    to it; each (token, slot) output is still its own definition.
    ``idx_override`` replaces the top-k selection (gates then follow from it),
    used to evaluate the layer on another router's choice of experts.
    """
    tok = np.arange(layer.T) if tokens is None else np.asarray(tokens, dtype=np.int64)
    r = route(layer, tokens=tok, logits=logits)
    if idx_override is not None:
        r["idx"] = np.asarray(idx_override, dtype=np.int32)
        r["gates"] = gates(r["logits"], r["idx"])
    idx, g = r["idx"], r["gates"]
    d, I, k = layer.d, layer.I, layer.k
    x = bf16_to_f64(layer.x[tok])
    y = np.zeros((len(tok), k, d))
    for e in sorted(set(int(v) for v in idx.ravel())):
        rows, slots = np.nonzero(idx == e)
        w13, w2 = dequantize_expert(layer.experts[e], d, I)
        y[rows, slots] = expert_ffn(x[rows], w13, w2, I)
        del w13, w2
    out = np.einsum("tj,tjd->td", g, y)
    for s in range(layer.S):
        w13, w2 = dequantize_expert(layer.experts[layer.E + s], d, I)
        out = out + expert_ffn(x, w13, w2, I)
        del w13, w2
    r["out"] = out
    r["tokens"] = tok
    return r


def margin_safe(margin: np.ndarray, threshold: float = 1e-4) -> np.ndarray:
    """Tokens whose k-th/(k+1)-th logit gap exceeds the threshold."""
    return np.asarray(margin) > threshold


def rel_l2(a: np.ndarray, b: np.ndarray) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    den = math.sqrt(float((b * b).sum()))
    return math.sqrt(float(((a - b) ** 2).sum())) / max(den, 1e-300)


def layer_flops(T: int, d: int, E: int, k: int, I: int, S: int) -> float:
    """Algorithmic FLOPs of one forward: router plus 3 matmuls per routed/shared pair."""
    return 2.0 * T * d * E + 6.0 * T * (k + S) * d * I


__all__: List[str] = [
    "bf16_to_f64", "decode_e4m3", "unpack_int4", "dequantize", "router_logits", "topk",
    "topk_margin", "gates", "schedule", "silu", "expert_ffn", "dequantize_expert", "route",
    "forward", "margin_safe", "rel_l2", "layer_flops",
]
