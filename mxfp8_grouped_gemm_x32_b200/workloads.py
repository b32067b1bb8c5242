"""Seeded synthetic inputs for the grouped MXFP8 MoE expert MLP.

This module is shared by the CUDA path's tests and benchmark and by the CPU
oracle's tests.  It holds only the input recipe: random draws, rounding of
those draws to bf16 (the storage format of every input tensor), and the
routing used to synthesise the expert MLP's top-k inputs.  It contains none
of the expert MLP's arithmetic (no quantisation, no GEMM, no activation).
The router step itself (moe_router_topk) is checked against its own oracle
(oracle/router.py) on the raw `router_logits`; neither side uses `route`.

Recipe (the workloads of "Efficient MoE Training for Biological Foundation
Models", Challenge 1-3, and the MoE table of the NeMo Automodel page, with the
shapes of the Mixtral-8x7B, Qwen3-MoE-30B and GPT-OSS-20B expert layers):

* x ~ N(0, 1), W_gate_up[e] in R^{2I x H} ~ N(0, 1/H), W_down[e] in
  R^{H x I} ~ N(0, 1/I), dY ~ N(0, 1); every draw is float32, rounded to
  bf16 with round-to-nearest-even.
* Router logits ~ N(0, 1) (plus a fixed per-expert bias ~ N(0, 1.5^2) for
  the skewed 128-expert layer).  "softmax_topk": softmax over all E experts
  in float64, the k largest (ties to the lower expert id), renormalised by
  their sum.  "topk_softmax": the k largest logits, softmax over those k.
  Probabilities are stored as float32.
* Every tensor is drawn in fixed chunks, each from its own counter-derived
  PCG64 stream, so the values do not depend on the thread count.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

__all__ = ["LayerConfig", "CONFIGS", "get_config", "make_inputs",
           "bf16_bits_from_f32", "bf16_bits_to_f32", "route"]


@dataclass(frozen=True)
class LayerConfig:
    """Shape of one MoE expert layer: T tokens, hidden H, intermediate I,
    E experts, top-k routing."""
    name: str
    T: int
    H: int
    I: int
    E: int
    k: int
    router: str = "softmax_topk"      # or "topk_softmax"
    expert_bias_std: float = 0.0      # skew of the router (per-expert bias)
    backward: bool = True
    note: str = field(default="", compare=False)

    @property
    def R(self) -> int:
        """Routed rows (token, k) pairs."""
        return self.T * self.k

    def fwd_flops(self) -> float:
        """Algorithmic forward FLOPs: gate_up (2*R*H*2I) + down (2*R*I*H)."""
        return 6.0 * self.R * self.H * self.I

    def bwd_flops(self) -> float:
        """Algorithmic backward FLOPs: two dgrad + two wgrad GEMMs."""
        return 12.0 * self.R * self.H * self.I


CONFIGS = {
    # parity-size layer: several tiles and ragged tails, seconds on the CPU
    "tiny": LayerConfig("tiny", T=512, H=256, I=512, E=4, k=2,
                        note="T512 H256 I512 E4 top2"),
    "mixtral_8x7b": LayerConfig("mixtral_8x7b", T=8192, H=4096, I=14336, E=8, k=2,
                                note="Mixtral-8x7B expert layer, 2x4096 tokens"),
    # Mixtral expert shapes with 2 of the 8 experts and the same 2048 rows per
    # expert: a profiler-sized slice of the Mixtral layer
    "mixtral_profile": LayerConfig("mixtral_profile", T=4096, H=4096, I=14336, E=2, k=1,
                                   note="Mixtral-8x7B expert shapes, 2 experts x 2048 rows"),
    "qwen3_30b_ragged": LayerConfig("qwen3_30b_ragged", T=16384, H=2048, I=768, E=128, k=8,
                                    expert_bias_std=1.5,
                                    note="Qwen3-MoE-30B-shaped, skewed routing"),
    # Qwen3 shapes and routing with a quarter of the tokens: a profiler-sized
    # slice of the ragged layer (about 32 rows per expert instead of 128)
    "qwen3_profile": LayerConfig("qwen3_profile", T=4096, H=2048, I=768, E=128, k=8, expert_bias_std=1.5,
                                 note="Qwen3-MoE-30B-shaped, skewed routing, T=4096"),
    "gpt_oss_20b": LayerConfig("gpt_oss_20b", T=8192, H=2880, I=2880, E=32, k=4,
                               router="topk_softmax",
                               note="GPT-OSS-20B-shaped, K=2880 not a multiple of 128"),
}


def get_config(name: str, **overrides) -> LayerConfig:
    base = CONFIGS[name]
    if not overrides:
        return base
    d = {f: getattr(base, f) for f in base.__dataclass_fields__}
    d.update(overrides)
    return LayerConfig(**d)


# ----------------------------------------------------------------------------
# bf16 storage helpers (bit manipulation only)
# ----------------------------------------------------------------------------

def bf16_bits_from_f32(a: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns (uint16), round-to-nearest-even.
    NaN inputs map to a quiet NaN."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    b = a.view(np.uint32)
    r = ((b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)).astype(np.uint16)
    nan = np.isnan(a)
    if nan.any():
        r[nan] = np.uint16(0x7FC0)
    return r


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> exact float32 values."""
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


# ----------------------------------------------------------------------------
# chunked, thread-count-independent normal draws
# ----------------------------------------------------------------------------

_CHUNK = 1 << 24


def _normal_f32(seed: int, stream: int, n: int, std: float) -> np.ndarray:
    out = np.empty(n, np.float32)
    nchunks = (n + _CHUNK - 1) // _CHUNK

    def fill(c):
        lo, hi = c * _CHUNK, min(n, (c + 1) * _CHUNK)
        g = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, stream, c])))
        g.standard_normal(hi - lo, dtype=np.float32, out=out[lo:hi])
        if std != 1.0:
            out[lo:hi] *= np.float32(std)

    if nchunks == 1:
        fill(0)
    else:
        workers = max(1, min(nchunks, len(os.sched_getaffinity(0))))
        with ThreadPoolExecutor(workers) as ex:
            list(ex.map(fill, range(nchunks)))
    return out


def _normal_bf16(seed, stream, shape, std) -> np.ndarray:
    n = int(np.prod(shape))
    return bf16_bits_from_f32(_normal_f32(seed, stream, n, std)).reshape(shape)


# stream ids: one per tensor so each can be regenerated on its own
_S_X, _S_W1, _S_W2, _S_LOGITS, _S_BIAS, _S_DY = range(6)


def route(logits: np.ndarray, k: int, kind: str):
    """Router used to build the inputs: returns (topk_idx int32 [T,k],
    topk_prob float32 [T,k]).  Ties go to the lower expert id."""
    lg = logits.astype(np.float64)
    order = np.argsort(-lg, axis=1, kind="stable")[:, :k]
    if kind == "softmax_topk":
        z = lg - lg.max(axis=1, keepdims=True)
        p = np.exp(z)
        p /= p.sum(axis=1, keepdims=True)
        top = np.take_along_axis(p, order, axis=1)
        top = top / top.sum(axis=1, keepdims=True)
    elif kind == "topk_softmax":
        top = np.take_along_axis(lg, order, axis=1)
        top = np.exp(top - top.max(axis=1, keepdims=True))
        top = top / top.sum(axis=1, keepdims=True)
    else:
        raise ValueError(kind)
    return order.astype(np.int32), top.astype(np.float32)


def make_inputs(cfg: LayerConfig, seed: int = 0, *, weights: bool = True,
                grad: bool = True, topk_idx: np.ndarray | None = None) -> dict:
    """Draw one layer's inputs.

    Returns a dict of numpy arrays:
      x      uint16 bf16 bits [T, H]
      w1     uint16 bf16 bits [E, 2I, H]   (gate rows 0..I-1, up rows I..2I-1)
      w2     uint16 bf16 bits [E, H, I]
      topk_idx int32 [T, k], topk_prob float32 [T, k]
      router_logits float32 [T, E]           (the logits the routing was drawn from)
      dy     uint16 bf16 bits [T, H]        (when grad)
    ``topk_idx`` may be given to force a routing pattern (edge cases); the
    probabilities are then drawn from the same router over those experts.
    """
    T, H, I, E, k = cfg.T, cfg.H, cfg.I, cfg.E, cfg.k
    out = {"x": _normal_bf16(seed, _S_X, (T, H), 1.0)}
    if weights:
        out["w1"] = _normal_bf16(seed, _S_W1, (E, 2 * I, H), 1.0 / np.sqrt(H))
        out["w2"] = _normal_bf16(seed, _S_W2, (E, H, I), 1.0 / np.sqrt(I))
    logits = _normal_f32(seed, _S_LOGITS, T * E, 1.0).reshape(T, E).astype(np.float64)
    if cfg.expert_bias_std:
        logits = logits + _normal_f32(seed, _S_BIAS, E, cfg.expert_bias_std).astype(np.float64)[None, :]
    out["router_logits"] = logits.astype(np.float32)
    if topk_idx is None:
        idx, prob = route(logits, k, cfg.router)
    else:
        idx = np.ascontiguousarray(topk_idx, dtype=np.int32)
        g = np.take_along_axis(logits, idx.astype(np.int64), axis=1)
        g = np.exp(g - g.max(axis=1, keepdims=True))
        prob = (g / g.sum(axis=1, keepdims=True)).astype(np.float32)
    out["topk_idx"], out["topk_prob"] = idx, prob
    if grad:
        out["dy"] = _normal_bf16(seed, _S_DY, (T, H), 1.0)
    return out
