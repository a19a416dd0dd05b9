"""Seeded synthetic inputs for the quantised top-k MoE FFN layer.

This module only *makes inputs*: activations, router weights, an optional
per-expert router bias, and expert weights quantised to the byte formats the
library accepts.  It holds none of the layer's own arithmetic (no routing, no
softmax, no dequantisation, no expert FFN), so that both the fp64 oracle and
the CUDA path can be fed from it without sharing any of the computation they
are compared on.

Workloads (the five shapes the pages' layer is measured on):

=========  =====  ====  ===  ==  =====  =  ============  =========
name       T      d     E    k   I      S  weights       router
=========  =====  ====  ===  ==  =====  =  ============  =========
tiny       64     256   8    2   512    0  INT8 per-ch   N(0,1/d)
decode     1..256 2048  128  8   768    0  INT4 g128     N(0,1/d)
prefill    8192   4096  8    2   14336  0  FP8 e4m3 pc   N(0,1/d)
fine       4096   2048  64   6   1408   2  INT4 g128     + Zipf 1.2
mixed      16384  4096  64   4   2048   0  INT8 / INT4   + Zipf 1.0
=========  =====  ====  ===  ==  =====  =  ============  =========

Quantisers (symmetric, no zero point; the Q-MoE page, "Expert Quantizer"
and "INT4/INT8 Quantization" rows, names the formats but not the recipe, so
the plainest symmetric recipe is used):

* INT8 per output channel: ``s = max|w_row| / 127`` (fp32),
  ``q = clamp(rint(w / s), -127, 127)``.
* INT4 group 128 along K: ``s = bf16_rne(max|w_group| / 7)``,
  ``q = clamp(rint(w / s), -7, 7)`` with ``s`` taken as the bf16 value.
  Packed two per byte, low nibble = even k, two's complement.
* FP8 e4m3 per output channel: ``s = max|w_row| / 448`` (fp32),
  ``q = e4m3_rne(clamp(w / s, -448, 448))``.

A row or group that is all zero gets ``s = 1`` and ``q = 0``.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional

import numpy as np

FMT_INT8 = 1      # int8 [N][K], fp32 scale [N]
FMT_INT4 = 2      # packed u8 [N][K/2], bf16 scale [N][K/128]
FMT_FP8 = 3       # e4m3 u8 [N][K], fp32 scale [N]

FMT_NAMES = {FMT_INT8: "int8_pc", FMT_INT4: "int4_g128", FMT_FP8: "fp8_e4m3_pc"}

# name -> shape parameters.  "fmt" is a format id or "mixed" (experts below
# E/2 INT8 per channel, the rest INT4 group 128).
CONFIGS = {
    "tiny": dict(T=64, d=256, E=8, k=2, I=512, S=0, fmt=FMT_INT8, zipf=None),
    "decode": dict(T=256, d=2048, E=128, k=8, I=768, S=0, fmt=FMT_INT4, zipf=None),
    "prefill": dict(T=8192, d=4096, E=8, k=2, I=14336, S=0, fmt=FMT_FP8, zipf=None),
    "fine": dict(T=4096, d=2048, E=64, k=6, I=1408, S=2, fmt=FMT_INT4, zipf=1.2),
    "mixed": dict(T=16384, d=4096, E=64, k=4, I=2048, S=0, fmt="mixed", zipf=1.0),
}
DECODE_SWEEP = (1, 8, 32, 128, 256)


@dataclasses.dataclass
class Expert:
    fmt: int
    w13: np.ndarray   # [2I][d] codes (int8 / u8 packed / u8 e4m3); rows 0..I-1 gate, I..2I-1 up
    s13: np.ndarray   # fp32 [2I] or bf16 bits u16 [2I][d/128]
    w2: np.ndarray    # [d][I] codes
    s2: np.ndarray    # fp32 [d] or bf16 bits u16 [d][I/128]


@dataclasses.dataclass
class LayerInputs:
    name: str
    T: int
    d: int
    E: int
    k: int
    I: int
    S: int
    x: np.ndarray                 # bf16 bits, u16 [T][d]
    router_w: np.ndarray          # fp32 [E][d]
    router_b: Optional[np.ndarray]  # fp32 [E] or None
    experts: List[Expert]         # E routed, then S shared
    seed: int = 0

    @property
    def n_experts_total(self) -> int:
        return self.E + self.S


# --------------------------------------------------------------------------
# value encoders (input preparation only)
# --------------------------------------------------------------------------
def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (round to nearest, ties to even); return the bits."""
    b = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (b + 0x7FFF + ((b >> 16) & 1)) >> 16
    return r.astype(np.uint16)


def bf16_bits_as_f32(u: np.ndarray) -> np.ndarray:
    """Widen bf16 bits to fp32 (exact)."""
    return (np.asarray(u, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def f32_to_e4m3_codes(a: np.ndarray) -> np.ndarray:
    """Encode fp32 values (already inside [-448, 448]) as e4m3 codes, RNE.

    Uses torch's CPU float8_e4m3fn cast, a library encoder.
    """
    import torch

    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy().copy()


# --------------------------------------------------------------------------
# host quantisers
# --------------------------------------------------------------------------
def quantize_int8_pc(w: np.ndarray):
    w = np.asarray(w, dtype=np.float32)
    amax = np.abs(w).max(axis=1)
    s = np.where(amax > 0, amax / np.float32(127.0), np.float32(1.0)).astype(np.float32)
    q = np.clip(np.rint(w / s[:, None]), -127, 127).astype(np.int8)
    return q, s


def quantize_fp8_pc(w: np.ndarray):
    w = np.asarray(w, dtype=np.float32)
    amax = np.abs(w).max(axis=1)
    s = np.where(amax > 0, amax / np.float32(448.0), np.float32(1.0)).astype(np.float32)
    v = np.clip(w / s[:, None], -448.0, 448.0).astype(np.float32)
    return f32_to_e4m3_codes(v), s


def pack_int4(q: np.ndarray) -> np.ndarray:
    """[N][K] int values in [-8, 7] -> [N][K/2] bytes, low nibble = even k."""
    q = np.asarray(q, dtype=np.int8)
    lo = (q[:, 0::2].astype(np.uint8) & 0xF)
    hi = (q[:, 1::2].astype(np.uint8) & 0xF)
    return (lo | (hi << 4)).astype(np.uint8)


def quantize_int4_g128(w: np.ndarray):
    w = np.asarray(w, dtype=np.float32)
    N, K = w.shape
    assert K % 128 == 0
    g = w.reshape(N, K // 128, 128)
    amax = np.abs(g).max(axis=2)
    s_bits = f32_to_bf16_bits(amax / np.float32(7.0))
    s_bits = np.where(amax > 0, s_bits, np.uint16(0x3F80)).astype(np.uint16)
    s = bf16_bits_as_f32(s_bits)
    q = np.clip(np.rint(g / s[:, :, None]), -7, 7).astype(np.int8).reshape(N, K)
    return pack_int4(q), s_bits


def quantize(fmt: int, w: np.ndarray):
    if fmt == FMT_INT8:
        return quantize_int8_pc(w)
    if fmt == FMT_INT4:
        return quantize_int4_g128(w)
    if fmt == FMT_FP8:
        return quantize_fp8_pc(w)
    raise ValueError(f"unknown weight format {fmt}")


# --------------------------------------------------------------------------
# generators
# --------------------------------------------------------------------------
def _streams(seed: int):
    ss = np.random.SeedSequence(seed)
    x_ss, r_ss, b_ss, e_ss = ss.spawn(4)
    return x_ss, r_ss, b_ss, e_ss


def make_x(T: int, d: int, seed: int = 0) -> np.ndarray:
    """Activations ~ N(0, 1) rounded to bf16; row t is the same for every T."""
    x_ss, _, _, _ = _streams(seed)
    rng = np.random.Generator(np.random.PCG64(x_ss))
    return f32_to_bf16_bits(rng.standard_normal((T, d), dtype=np.float32))


def zipf_bias(E: int, s: float, seed: int = 0) -> np.ndarray:
    """Per-expert router bias for a Zipf(s) load skew.

    Expert e gets target share pi_e proportional to r_e**(-s), where r is a
    seeded permutation of 1..E; the bias is log(pi_e) minus its mean.  The
    pages only say the load should follow Zipf; this is the plainest bias
    that ranks the experts that way.  The realised load is measured, not
    assumed.
    """
    _, _, b_ss, _ = _streams(seed)
    rng = np.random.Generator(np.random.PCG64(b_ss))
    r = rng.permutation(E) + 1
    logpi = -s * np.log(r.astype(np.float64))
    logpi -= np.log(np.exp(logpi).sum())
    return (logpi - logpi.mean()).astype(np.float32)


def expert_format(cfg: dict, e: int) -> int:
    if cfg["fmt"] == "mixed":
        return FMT_INT8 if e < cfg["E"] // 2 else FMT_INT4
    if cfg["fmt"] == "mixed_fp8":            # FP8 beside INT4: the layer computes in bf16
        return FMT_FP8 if e < cfg["E"] // 2 else FMT_INT4
    return cfg["fmt"]


def make_expert(d: int, I: int, fmt: int, e: int, seed: int = 0) -> Expert:
    """Expert e: W13 [2I][d] and W2 [d][I], each ~ N(0, 1/d) in fp32, quantised."""
    _, _, _, e_ss = _streams(seed)
    child = np.random.SeedSequence(entropy=e_ss.entropy, spawn_key=e_ss.spawn_key + (e,))
    rng = np.random.Generator(np.random.PCG64(child))
    sd = np.float32(1.0 / np.sqrt(d))
    w13 = rng.standard_normal((2 * I, d), dtype=np.float32) * sd
    q13, s13 = quantize(fmt, w13)
    del w13
    w2 = rng.standard_normal((d, I), dtype=np.float32) * sd
    q2, s2 = quantize(fmt, w2)
    return Expert(fmt=fmt, w13=q13, s13=s13, w2=q2, s2=s2)


def _config(name: str, T: Optional[int], overrides: dict) -> dict:
    cfg = dict(CONFIGS[name]) if name in CONFIGS else {}
    cfg.update(overrides)
    if T is not None:
        cfg["T"] = T
    return cfg


def make_router_inputs(name: str, T: Optional[int] = None, seed: int = 0, **overrides):
    """The named workload's x (bf16 bits), router weights and bias, without
    the experts: the same arrays make_layer returns for them."""
    cfg = _config(name, T, overrides)
    T_, d, E = cfg["T"], cfg["d"], cfg["E"]
    _, r_ss, _, _ = _streams(seed)
    rng = np.random.Generator(np.random.PCG64(r_ss))
    router_w = (rng.standard_normal((E, d), dtype=np.float32) * np.float32(1.0 / np.sqrt(d))).astype(np.float32)
    router_b = zipf_bias(E, cfg["zipf"], seed) if cfg.get("zipf") else None
    return make_x(T_, d, seed), router_w, router_b


def make_layer(name: str, T: Optional[int] = None, seed: int = 0, **overrides) -> LayerInputs:
    """Build the named workload (``CONFIGS``) with optional shape overrides."""
    cfg = _config(name, T, overrides)
    T_, d, E, k, I, S = (cfg[key] for key in ("T", "d", "E", "k", "I", "S"))
    x, router_w, router_b = make_router_inputs(name, T, seed, **overrides)
    experts = [make_expert(d, I, expert_format(cfg, e), e, seed) for e in range(E + S)]
    return LayerInputs(name=name, T=T_, d=d, E=E, k=k, I=I, S=S, x=x,
                       router_w=router_w, router_b=router_b, experts=experts, seed=seed)


def weight_bytes(ex: Expert) -> int:
    """Bytes of codes plus scales an expert's three matrices occupy."""
    return int(ex.w13.nbytes + ex.s13.nbytes + ex.w2.nbytes + ex.s2.nbytes)
