"""Seeded synthetic inputs for the sigmoid-routed mixture-of-experts FFN.

This module holds the workload shapes and the random-input recipe and nothing of
the method's arithmetic (no routing, no SwiGLU, no gates).  Both the CUDA path's
tests/benchmark and the CPU oracle's tests draw their inputs from here.

Shapes follow the two model families the pages describe:
  * GLM-4.7-Flash (nnterp encyclopedia, "Config"): hidden_size 2048,
    moe_intermediate_size 1536, n_routed_experts 64, num_experts_per_tok 4,
    n_shared_experts 1;
  * GLM-5 (config.json on the atlas projection page, and the nnterp GLM-5
    "Config"): hidden_size 6144, moe_intermediate_size 2048, n_routed_experts 256,
    num_experts_per_tok 8, n_shared_experts 1, routed_scaling_factor 2.5.

Recipe (the same for every workload; seed = 1000 + workload number):
  x    [T, H]  bf16   N(0, 1)     NumPy PCG64 (default_rng(seed)), fp32 -> bf16 RNE
  W_r  [E, H]  fp32   N(0, 0.02)  same generator, drawn after x
  b    [E]     fp32   N(0, 0.1)   same generator, drawn after W_r
  W1, W3 [E, I, H], W2 [E, H, I], shared Ws1, Ws3 [I, H], Ws2 [H, I]:
               bf16   N(0, 0.02)  torch generator on the target device seeded with
                                  seed, drawn expert by expert (W1, W3, W2), shared last.
The skewed workload additionally sets feature 0 of every token to 1.0 (exact in
bf16) and W_r[e, 0] = 1.5 * ln(rank_e ** -1.2) with rank a seeded permutation of
1..E, which adds exactly that per-expert offset to every router logit.
"""
from __future__ import annotations

import dataclasses

import numpy as np


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    T: int          # tokens
    H: int          # hidden size
    I: int          # expert (and shared expert) intermediate size
    E: int          # routed experts
    K: int          # experts per token
    scale: float    # routed scaling factor
    seed: int
    skew: bool = False
    has_shared: bool = True

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "tiny": Workload("tiny", T=64, H=256, I=128, E=16, K=4, scale=2.5, seed=1000),
    "glm47flash": Workload("glm47flash", T=4096, H=2048, I=1536, E=64, K=4, scale=2.5, seed=1001),
    "glm5_decode": Workload("glm5_decode", T=64, H=6144, I=2048, E=256, K=8, scale=2.5, seed=1002),
    "glm5_prefill": Workload("glm5_prefill", T=16384, H=6144, I=2048, E=256, K=8, scale=2.5,
                             seed=1003),
    "glm5_skewed": Workload("glm5_skewed", T=8192, H=6144, I=2048, E=256, K=8, scale=2.5,
                            seed=1004, skew=True),
    # GLM-5 expert shapes with 32 experts: 2.5 GB of weights, small enough for
    # multi-pass profiler captures, still far larger than the 126 MB L2
    "glm5_e32": Workload("glm5_e32", T=8192, H=6144, I=2048, E=32, K=8, scale=2.5, seed=1005),
    # dense SwiGLU MLP of the first blocks (E = K = 0; I = intermediate_size)
    "glm5_dense": Workload("glm5_dense", T=16384, H=6144, I=12288, E=0, K=0, scale=1.0, seed=1007),
    "glm47flash_dense": Workload("glm47flash_dense", T=4096, H=2048, I=10240, E=0, K=0, scale=1.0,
                                 seed=1008),
    "glm5_decode_e32": Workload("glm5_decode_e32", T=64, H=6144, I=2048, E=32, K=8, scale=2.5,
                                seed=1006),
}


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to the nearest bf16 (ties to even); returns uint16 bit patterns."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    b = a.view(np.uint32).astype(np.uint64)
    b = (b + 0x7FFF + ((b >> 16) & 1)) >> 16
    return b.astype(np.uint16)


def bf16_bits_to_f32(a: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp32."""
    return (np.ascontiguousarray(a, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def router_inputs(w: Workload):
    """(x uint16 [T,H] bf16 bits, W_r float32 [E,H], b float32 [E]) for a workload."""
    rng = np.random.default_rng(w.seed)
    x = f32_to_bf16_bits(rng.standard_normal((w.T, w.H), dtype=np.float32))
    w_r = (rng.standard_normal((w.E, w.H), dtype=np.float32) * np.float32(0.02)).astype(np.float32)
    b = (rng.standard_normal((w.E,), dtype=np.float32) * np.float32(0.1)).astype(np.float32)
    if w.skew:
        rank = rng.permutation(w.E).astype(np.float64) + 1.0
        x[:, 0] = f32_to_bf16_bits(np.ones((w.T,), dtype=np.float32))
        w_r[:, 0] = (1.5 * np.log(rank ** -1.2)).astype(np.float32)
    return x, w_r, b


def norm_weight(w: Workload):
    """Pre-FFN RMSNorm weight gamma [H] (bf16 bits): 1 + N(0, 0.1), seeded by (seed, 7)."""
    rng = np.random.default_rng([w.seed, 7])
    return f32_to_bf16_bits(1.0 + 0.1 * rng.standard_normal((w.H,), dtype=np.float32))


def expert_weights(w: Workload, device="cpu"):
    """Expert weights as torch bf16 tensors on ``device``:
    dict(w1 [E,I,H], w3 [E,I,H], w2 [E,H,I], ws1 [I,H], ws3 [I,H], ws2 [H,I])."""
    import torch

    dev = torch.device(device)
    gen = torch.Generator(device=dev)
    gen.manual_seed(w.seed)
    w1 = torch.empty((w.E, w.I, w.H), dtype=torch.bfloat16, device=dev)
    w3 = torch.empty((w.E, w.I, w.H), dtype=torch.bfloat16, device=dev)
    w2 = torch.empty((w.E, w.H, w.I), dtype=torch.bfloat16, device=dev)

    def draw(shape):
        return (torch.randn(shape, generator=gen, device=dev, dtype=torch.float32) * 0.02).to(
            torch.bfloat16)

    for e in range(w.E):
        w1[e] = draw((w.I, w.H))
        w3[e] = draw((w.I, w.H))
        w2[e] = draw((w.H, w.I))
    ws1 = draw((w.I, w.H))
    ws3 = draw((w.I, w.H))
    ws2 = draw((w.H, w.I))
    return dict(w1=w1, w3=w3, w2=w2, ws1=ws1, ws3=ws3, ws2=ws2)


def torch_bf16_to_bits(t) -> np.ndarray:
    """Host uint16 bit patterns of a torch bf16 tensor (copied to the CPU)."""
    import torch

    return t.detach().to("cpu").contiguous().view(torch.int16).numpy().view(np.uint16)


# ------------------------------------------------- sparse-attention key selection
# Shapes of the GLM-5 indexer (config.json: index_n_heads 32, index_head_dim 128,
# index_topk 2048).  Recipe (seed as listed): q [B, T, NH, D] and k [B, S, D] bf16
# N(0, 1) (the keys leave a LayerNorm, the queries a normalised latent's
# projection), w [B, T, NH] fp32 N(0, 1), drawn in that order from NumPy
# default_rng(seed), fp32 -> bf16 RNE.  Prefill: T == S (4 sequences of 4096
# tokens, the block's 16384-token batch); decode: one query per sequence over a
# 32768-key cache.

@dataclasses.dataclass(frozen=True)
class DsaWorkload:
    name: str
    B: int
    T: int
    S: int
    n_heads: int = 32
    head_dim: int = 128
    topk: int = 2048
    seed: int = 2000

    def replace(self, **kw) -> "DsaWorkload":
        return dataclasses.replace(self, **kw)


DSA_WORKLOADS = {
    "dsa_tiny": DsaWorkload("dsa_tiny", B=2, T=300, S=300, topk=64, seed=2001),
    "dsa_prefill": DsaWorkload("dsa_prefill", B=4, T=4096, S=4096, seed=2002),
    "dsa_decode": DsaWorkload("dsa_decode", B=64, T=1, S=32768, seed=2003),
}


def dsa_inputs(w: DsaWorkload):
    """(q bf16 bits [B,T,NH,D], k bf16 bits [B,S,D], w fp32 [B,T,NH]) on the host."""
    rng = np.random.default_rng(w.seed)
    q = f32_to_bf16_bits(rng.standard_normal((w.B, w.T, w.n_heads, w.head_dim), dtype=np.float32))
    k = f32_to_bf16_bits(rng.standard_normal((w.B, w.S, w.head_dim), dtype=np.float32))
    wt = rng.standard_normal((w.B, w.T, w.n_heads), dtype=np.float32)
    return q, k, wt
