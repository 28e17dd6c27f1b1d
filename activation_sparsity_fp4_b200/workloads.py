"""Seeded synthetic inputs shaped like the layers the SharQ pages evaluate.

This module holds input generation only -- no step of the method.  Both the
CUDA path and the CPU oracle take their inputs from here, so they see the same
values.  Activations and weights that the layer receives in bf16 are returned
as fp32 arrays whose values are exactly representable in bf16 (round to
nearest even), together with the dtype name the caller should hand to the GPU.

Workloads (SharQ abstract: Llama-3.1-8B, Qwen3-30B-A3B, Wan2.2; the Huawei
problem statement: LLaMa3.1-8B down_proj, 2:4 / 8:16, 50% pruned, seq 2048).
The pages use real checkpoints and datasets; these seeded tensors stand in for
them by shape and value distribution only:

* ``tiny``       X 16x256 fp32 ~N(0,1), channels 3 and 77 scaled x40; W 256x256 ~N(0, 0.02^2);
                 MXFP4, 2:4, no norm.
* ``q_proj``     X 2048x4096 bf16 = 0.5 * Student-t(3), 8 outlier channels x100 (the first 8
                 entries of a seeded permutation of K); RMSNorm gamma ~U(0.5, 1.5) bf16, eps 1e-6;
                 W 4096x4096 ~N(0, 0.02^2); NVFP4, 4:8 pair.
* ``down_proj``  X T x 14336 bf16 = SiLU(a) * b with a, b ~N(0,1) (computed in fp32);
                 W 4096x14336 ~N(0, 0.01^2); MXFP4, 2:4; T in {1, 16, 64, 256, 2048}; also
                 gate = a and up = b rounded to bf16, the inputs of the SwiGLU form.
* ``wan``        X 32768x5120 bf16 ~N(0,1), 16 outlier channels x50; RMSNorm gamma ~U(0.5, 1.5);
                 W 5120x5120 ~N(0, 0.02^2); NVFP4, 4:8 pair (and 8:16).
* ``qwen_moe``   4096 tokens, hidden 2048, 0.5 * Student-t(3) bf16; router logits 4096x128 ~N(0,1),
                 softmax, top-8 (ties to the lower expert); routed rows gathered in expert order,
                 each expert's segment padded with zero rows to a multiple of 128; per expert
                 gate/up W 1536x2048 and down W 2048x768 ~N(0, 0.02^2); down input 0.5 * t(3)
                 of shape (routed rows) x 768; NVFP4, 4:8 pair, no norm.
"""
from __future__ import annotations

import numpy as np

SEED = 0


def to_bf16_values(a: np.ndarray) -> np.ndarray:
    """fp32 array rounded (nearest even) to values representable in bfloat16."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32)


def _outlier_channels(rng: np.random.Generator, k: int, count: int) -> np.ndarray:
    return rng.permutation(k)[:count]


def tiny(seed: int = SEED) -> dict:
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((16, 256)).astype(np.float32)
    x[:, [3, 77]] *= 40.0
    w = (rng.standard_normal((256, 256)) * 0.02).astype(np.float32)
    return dict(name="tiny", x=x, x_dtype="f32", gamma=None, eps=1e-6, w=w, w_dtype="f32",
                fmt="mxfp4", pat="2:4")


def q_proj(seed: int = SEED, t: int = 2048) -> dict:
    rng = np.random.default_rng(seed)
    k, n = 4096, 4096
    x = 0.5 * rng.standard_t(3, size=(t, k))
    ch = _outlier_channels(rng, k, 8)
    x[:, ch] *= 100.0
    x = to_bf16_values(x.astype(np.float32))
    gamma = to_bf16_values(rng.uniform(0.5, 1.5, size=k).astype(np.float32))
    w = to_bf16_values(rng.standard_normal((n, k), dtype=np.float32) * np.float32(0.02))
    return dict(name="q_proj", x=x, x_dtype="bf16", gamma=gamma, eps=1e-6, w=w, w_dtype="bf16",
                fmt="nvfp4", pat="4:8pair")


def down_proj(seed: int = SEED, t: int = 2048) -> dict:
    rng = np.random.default_rng(seed)
    k, n = 14336, 4096
    a = rng.standard_normal((t, k), dtype=np.float32)
    b = rng.standard_normal((t, k), dtype=np.float32)
    x = (a / (np.float32(1.0) + np.exp(-a))) * b
    x = to_bf16_values(x.astype(np.float32))
    w = to_bf16_values(rng.standard_normal((n, k), dtype=np.float32) * np.float32(0.01))
    # the gate and up projections as a bf16 model hands them over, for the form of the
    # preprocessing that builds the down projection's input itself
    return dict(name="down_proj", x=x, x_dtype="bf16", gamma=None, eps=1e-6, w=w, w_dtype="bf16",
                fmt="mxfp4", pat="2:4", gate=to_bf16_values(a), up=to_bf16_values(b))


def wan(seed: int = SEED, t: int = 32768, pat: str = "4:8pair") -> dict:
    rng = np.random.default_rng(seed)
    k, n = 5120, 5120
    x = rng.standard_normal((t, k), dtype=np.float32)
    ch = _outlier_channels(rng, k, 16)
    x[:, ch] *= np.float32(50.0)
    x = to_bf16_values(x)
    gamma = to_bf16_values(rng.uniform(0.5, 1.5, size=k).astype(np.float32))
    w = to_bf16_values(rng.standard_normal((n, k), dtype=np.float32) * np.float32(0.02))
    return dict(name="wan" if pat == "4:8pair" else "wan_8_16", x=x, x_dtype="bf16", gamma=gamma, eps=1e-6,
                w=w, w_dtype="bf16", fmt="nvfp4", pat=pat)


def route_top_k(logits: np.ndarray, top_k: int) -> np.ndarray:
    """Indices of the top_k experts per token by softmax probability, ties to the lower index."""
    z = logits - logits.max(axis=1, keepdims=True)
    p = np.exp(z)
    p /= p.sum(axis=1, keepdims=True)
    # stable sort on -p keeps the lower index first among equal probabilities
    order = np.argsort(-p, axis=1, kind="stable")
    return order[:, :top_k]


def expert_rows(experts: np.ndarray, n_experts: int, align: int = 128):
    """Routed-row layout of a top-k assignment: each expert's rows contiguous, in token
    order, padded to a multiple of align.  Returns (counts, offsets (n_experts+1),
    gather = token index per routed row, -1 for a padding row)."""
    counts = np.bincount(experts.ravel(), minlength=n_experts)
    padded = ((counts + align - 1) // align) * align
    offsets = np.zeros(n_experts + 1, np.int64)
    offsets[1:] = np.cumsum(padded)
    gather = np.full(int(offsets[-1]), -1, np.int64)
    fill = offsets[:-1].copy()
    for tok in range(experts.shape[0]):
        for e in experts[tok]:
            gather[fill[e]] = tok
            fill[e] += 1
    return counts, offsets, gather


def qwen_moe(seed: int = SEED, tokens: int = 4096, n_experts: int = 128, top_k: int = 8,
             hidden: int = 2048, inter: int = 768, align: int = 128) -> dict:
    rng = np.random.default_rng(seed)
    x_tok = to_bf16_values((0.5 * rng.standard_t(3, size=(tokens, hidden))).astype(np.float32))
    logits = rng.standard_normal((tokens, n_experts))
    experts = route_top_k(logits, top_k)
    counts, offsets, gather = expert_rows(experts, n_experts, align)
    rows = int(offsets[-1])
    x_routed = np.zeros((rows, hidden), np.float32)
    valid = gather >= 0
    x_routed[valid] = x_tok[gather[valid]]
    x_down = to_bf16_values((0.5 * rng.standard_t(3, size=(rows, inter))).astype(np.float32))
    x_down[~valid] = 0.0
    w_gu = to_bf16_values(rng.standard_normal((n_experts, 2 * inter, hidden), dtype=np.float32) * np.float32(0.02))
    w_d = to_bf16_values(rng.standard_normal((n_experts, hidden, inter), dtype=np.float32) * np.float32(0.02))
    return dict(name="qwen_moe", x=x_routed, x_down=x_down, x_dtype="bf16", gamma=None, eps=1e-6,
                w_gu=w_gu, w_d=w_d, w_dtype="bf16", fmt="nvfp4", pat="4:8pair", counts=counts,
                offsets=offsets, gather=gather, n_experts=n_experts, x_tok=x_tok)


CONFIGS = {
    "tiny": tiny,
    "q_proj": q_proj,
    "down_proj": down_proj,
    "wan": wan,
    "qwen_moe": qwen_moe,
}
