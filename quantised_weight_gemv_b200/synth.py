"""Seeded synthetic inputs and workload shapes.

This module only draws random numbers and describes shapes.  It holds none of
the GEMV's arithmetic (no quantisation, no packing, no dot products), so both
the oracle side and the CUDA side of the tests, and the benchmark, may take
their inputs from it.

Distributions (stated with the workloads): weights w ~ N(0, 0.02) (0.02 is the
standard deviation) drawn in fp32; activations x ~ N(0, 1) drawn in fp32 and
rounded to fp16 (nearest-even); cached keys and values of decode attention
~ N(0, 1) in fp32 (quantised into the cache per position); routed-expert
indices drawn uniformly without
replacement per token; routing weights are a softmax (fp64, stored as fp32) of
N(0, 1) logits.  Every stream is keyed by
``(seed, workload id, layer, matrix id, kind)``.

Two generators: numpy ``default_rng`` for anything the CPU handles in
seconds, and torch's CUDA Philox generator (seeded from the same key) for the
multi-GB weight sets, which are then quantised on the device.
"""
from __future__ import annotations

import dataclasses
import hashlib
from typing import List, Optional, Sequence, Tuple

import numpy as np

KIND_W, KIND_X, KIND_IDX, KIND_LOGIT, KIND_H, KIND_KEY, KIND_VAL, KIND_LEN = 0, 1, 2, 3, 4, 5, 6, 7
W_STD = 0.02


def key(seed: int, workload: int, layer: int, matrix: int, kind: int) -> List[int]:
    return [int(seed), int(workload), int(layer), int(matrix), int(kind)]


def rng(k: Sequence[int]) -> np.random.Generator:
    return np.random.default_rng(list(k))


def torch_seed(k: Sequence[int]) -> int:
    """63-bit seed for torch.Generator derived from the same key."""
    h = hashlib.sha256((",".join(str(int(v)) for v in k)).encode()).digest()
    return int.from_bytes(h[:8], "little") & ((1 << 63) - 1)


# ------------------------------------------------------------- numpy side ----
def weights_f32(k: Sequence[int], N: int, K: int) -> np.ndarray:
    """fp32 [N, K], N(0, 0.02)."""
    return (rng(k).standard_normal((N, K), dtype=np.float32) * np.float32(W_STD)).astype(np.float32)


def kv_values_f32(k: Sequence[int], *shape: int) -> np.ndarray:
    """fp32 N(0, 1) keys or values of a KV cache (before quantisation)."""
    return rng(k).standard_normal(shape, dtype=np.float32)


def seq_lens(k: Sequence[int], B: int, Tmax: int) -> np.ndarray:
    """int32 [B] sequence lengths drawn uniformly from 1 .. Tmax."""
    return rng(k).integers(1, Tmax + 1, size=B).astype(np.int32)


def activations_f16_bits(k: Sequence[int], *shape: int) -> np.ndarray:
    """fp16 bit patterns (uint16) of N(0,1) fp32 draws rounded to nearest-even."""
    x = rng(k).standard_normal(shape, dtype=np.float32)
    return x.astype(np.float16).view(np.uint16)


def routing(k_idx: Sequence[int], k_logit: Sequence[int], B: int, E: int, topk: int
            ) -> Tuple[np.ndarray, np.ndarray]:
    """(expert_idx int32 [B, topk], route_w float32 [B, topk]).

    Indices: per token a uniform sample without replacement of topk of E.
    Weights: softmax (fp64) over that token's topk N(0,1) logits, stored fp32.
    """
    r = rng(k_idx)
    idx = np.stack([r.choice(E, size=topk, replace=False) for _ in range(B)]).astype(np.int32)
    logits = rng(k_logit).standard_normal((B, topk))
    ex = np.exp(logits - logits.max(axis=1, keepdims=True))
    w = (ex / ex.sum(axis=1, keepdims=True)).astype(np.float32)
    return idx, w


# ------------------------------------------------------------- torch side ----
def weights_f32_torch(k: Sequence[int], N: int, K: int, device):
    """fp32 [N, K] N(0, 0.02) on `device`, from torch's generator for that device."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(torch_seed(k))
    return torch.randn((N, K), generator=g, device=device, dtype=torch.float32).mul_(W_STD)


def activations_f16_torch(k: Sequence[int], shape, device):
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(torch_seed(k))
    return torch.randn(tuple(shape), generator=g, device=device, dtype=torch.float32).to(torch.float16)


# -------------------------------------------------------------- workloads ----
@dataclasses.dataclass(frozen=True)
class Mat:
    """One weight matrix of a decode step: N outputs x K inputs."""
    name: str
    N: int
    K: int
    stage: int          # stages run in order; matrices of one stage are independent


@dataclasses.dataclass(frozen=True)
class DenseWorkload:
    wid: int            # workload id, part of every seed key
    name: str
    fmt: int            # 2, 3, 4, 5, 6 or 8
    layers: int
    mats: Tuple[Mat, ...]   # per-layer matrices, in model order
    B: int = 1
    independent: bool = False   # layers are independent copies (one stage for all)
    verify: bool = False        # a batched-verification step (bq_verify_gemm per matrix)

    def layer_weights(self) -> int:
        return sum(m.N * m.K for m in self.mats)

    def stage_of(self, layer: int, stage: int) -> int:
        """Global stage of a layer's stage: layers run one after another, unless
        they are independent copies (then every layer shares the stages)."""
        n_st = 1 + max(m.stage for m in self.mats)
        return stage if self.independent else layer * n_st + stage


def packed_bytes(fmt: int, N: int, K: int) -> int:
    """Algorithmic bytes of one packed matrix: codes + scales (no padding)."""
    codes = {2: N * K // 4, 3: 3 * N * K // 8, 4: N * K // 2, 5: 5 * N * K // 8,
             6: 3 * N * K // 4, 8: N * K}[fmt]
    return codes + N * (K // 32) * 2


# A single 2048 x 2048 Q8 matrix at batch 1 (the small case).
SINGLE_Q8 = DenseWorkload(1, "q8-2048x2048", 8, 1, (Mat("w", 2048, 2048, 0),))

# 16-layer dense decoder, hidden 2048, FFN 8192, Q4, batch 1.  q|k|v share an
# input, as do gate|up; each group forms one stage.
DENSE_H2048 = DenseWorkload(2, "dense16L-h2048-ffn8192-q4", 4, 16, (
    Mat("q", 2048, 2048, 0), Mat("k", 512, 2048, 0), Mat("v", 512, 2048, 0),
    Mat("o", 2048, 2048, 1),
    Mat("gate", 8192, 2048, 2), Mat("up", 8192, 2048, 2),
    Mat("down", 2048, 8192, 3),
))


def dense_h2048(fmt: int) -> DenseWorkload:
    """The 16-layer hidden-2048 decoder in another format (Q2, Q3, Q5, Q6 or Q8)."""
    return DenseWorkload(8, f"dense16L-h2048-ffn8192-q{fmt}", fmt, 16, DENSE_H2048.mats)


def dense_h4096(fmt: int, B: int) -> DenseWorkload:
    """One layer of a dense decoder, hidden 4096, FFN 12288 (qkv and gate|up
    fused), streamed 36 times as distinct copies."""
    return DenseWorkload(3, f"dense36L-h4096-ffn12288-q{fmt}-b{B}", fmt, 36, (
        Mat("qkv", 6144, 4096, 0), Mat("o", 4096, 4096, 1),
        Mat("gateup", 24576, 4096, 2), Mat("down", 4096, 12288, 3),
    ), B)


def verify_h4096(fmt: int, B: int) -> DenseWorkload:
    """The hidden-4096 layer's matrices (36 distinct copies) as a batched
    verification step of B = 16 or 32 drafted tokens: every matrix through the
    tensor-core GEMM, each with its own seeded batch of activations."""
    return DenseWorkload(9, f"verify36L-h4096-ffn12288-q{fmt}-b{B}", fmt, 36,
                         dense_h4096(fmt, B).mats, B, verify=True)


# 64-layer dense decoder, hidden 5120, FFN 25600, Q4, batch 1 (~16 GB packed).
# Attention shapes: q, o 5120 x 5120; k, v 1024 x 5120 (8 KV heads x 128).
DENSE_H5120 = DenseWorkload(5, "dense64L-h5120-ffn25600-q4", 4, 64, (
    Mat("q", 5120, 5120, 0), Mat("k", 1024, 5120, 0), Mat("v", 1024, 5120, 0),
    Mat("o", 5120, 5120, 1),
    Mat("gate", 25600, 5120, 2), Mat("up", 25600, 5120, 2),
    Mat("down", 5120, 25600, 3),
))

# Matrix-shape sweep (N x K) for achieved bandwidth against matrix size.
SWEEP_SHAPES = ((512, 512), (1024, 1024), (2048, 2048), (4096, 4096), (5120, 5120),
                (1024, 5120), (8192, 5120), (25600, 5120), (5120, 25600))


def sweep_workload(fmt: int, N: int, K: int, B: int = 1, min_bytes: int = 512 << 20,
                   max_copies: int = 256) -> DenseWorkload:
    """Independent copies of one N x K matrix, enough of them (>= min_bytes,
    i.e. several times the L2) that no copy is served from L2 -- at most
    max_copies (the matrices one step plan holds); a set that then stays below
    twice the L2 is timed with the L2 flushed before every step."""
    copies = min(max_copies, max(2, -(-min_bytes // packed_bytes(fmt, N, K))))
    return DenseWorkload(6, f"sweep-q{fmt}-{N}x{K}-b{B}", fmt, copies, (Mat("w", N, K, 0),), B,
                         independent=True)


def verify_sweep_workload(fmt: int, N: int, K: int, B: int, min_bytes: int = 512 << 20) -> DenseWorkload:
    """Independent copies of one N x K matrix (>= min_bytes of packed weights)
    through the batched-verification GEMM: its steady-state rate."""
    copies = min(256, max(2, -(-min_bytes // packed_bytes(fmt, N, K))))
    return DenseWorkload(10, f"verify-sweep-q{fmt}-{N}x{K}-b{B}", fmt, copies, (Mat("w", N, K, 0),),
                         B, independent=True, verify=True)


def single_workload(fmt: int, N: int, K: int, B: int = 1) -> DenseWorkload:
    """One N x K matrix: a single call (its latency, with the L2 flushed)."""
    return DenseWorkload(7, f"single-q{fmt}-{N}x{K}-b{B}", fmt, 1, (Mat("w", N, K, 0),), B)


@dataclasses.dataclass(frozen=True)
class MoEWorkload:
    wid: int
    name: str
    layers: int
    E: int
    topk: int
    hidden: int
    ffn: int
    B: int

    def gateup(self) -> Tuple[int, int]:
        return 2 * self.ffn, self.hidden      # gate|up of one expert fused: N, K

    def down(self) -> Tuple[int, int]:
        return self.hidden, self.ffn


def moe_h2048(B: int) -> MoEWorkload:
    """48 layers, hidden 2048, 128 experts (gate/up 768 x 2048, down 2048 x 768),
    top-8 routing."""
    return MoEWorkload(4, f"moe48L-e128-top8-h2048-b{B}", 48, 128, 8, 2048, 768, B)


@dataclasses.dataclass(frozen=True)
class AttnWorkload:
    """Decode attention of every layer of a decoder over a Q8 KV cache of
    Tmax positions per (sequence, KV head), head dimension 128.  lens None:
    every sequence is full (Tmax positions); else lengths drawn uniformly
    from 1 .. Tmax (seq_lens)."""
    wid: int
    name: str
    layers: int
    B: int
    Hkv: int
    G: int
    Tmax: int
    full: bool = True
    D: int = 128

    def lens(self, seed: int = 0) -> np.ndarray:
        if self.full:
            return np.full(self.B, self.Tmax, dtype=np.int32)
        return seq_lens(key(seed, self.wid, 0, 0, KIND_LEN), self.B, self.Tmax)


def attn_h5120(B: int, Tmax: int, layers: int = 64) -> AttnWorkload:
    """The hidden-5120 decoder's attention (40 query heads on 8 KV heads),
    every sequence at Tmax positions: all 64 layers, or the first `layers`
    (a cache small enough for a many-pass profile)."""
    return AttnWorkload(11, f"attn{layers}L-kv8-g5-t{Tmax}-b{B}", layers, B, 8, 5, Tmax)


def attn_h2048(B: int, Tmax: int) -> AttnWorkload:
    """The 16-layer hidden-2048 decoder's attention (16 query heads on 4 KV
    heads), sequence lengths drawn uniformly from 1 .. Tmax."""
    return AttnWorkload(12, f"attn16L-kv4-g4-t{Tmax}-b{B}-mixed", 16, B, 4, 4, Tmax, full=False)
