"""Seeded synthetic inputs for the NVFP4 verify GEMM.

This module only draws random numbers and rounds them to the storage type of
each input. It holds none of the method's arithmetic: no quantisation, no
decoding, no products. Both the CPU oracle (through the tests) and the GPU
library (through the tests and the benchmark) take their inputs from here, so
the two sides see the same bytes without sharing any code.

Workloads (one dense ~27B model checked on a draft tree of 8/16/24/32 rows,
TandemLLM docs v0.12.0, "What TandemLLM is", section 1.2, and the StairCut
research page): every weight matrix W[N, K] is drawn as fp32 from N(0, 0.02),
or 0.02 * Student-t(4) for the heavy-tailed MLP-down case; the activations
X[M, K] are N(0, 1) rounded to bf16.

Two generators exist:
  * numpy (PCG64, keyed by (seed, tensor_id)) for the CPU side: tests and the
    oracle's inputs;
  * torch on a CUDA device (Philox, keyed the same way) for the multi-GB
    layer stack, where drawing 21 G values on the host would take minutes.
They produce different streams; each is deterministic for its key.
"""

from __future__ import annotations

import numpy as np

# tensor_id conventions for the 64-layer stack: W of (layer, matrix) has id
# layer*4 + matrix and its X has id X_ID_BASE + layer*4 + matrix.
X_ID_BASE = 1_000_000

# (name, K, N) of the four projections of one layer of the stack.
LAYER_SHAPES = (
    ("qkv", 5120, 7168),
    ("o", 5120, 5120),
    ("gate_up", 5120, 34816),
    ("down", 17408, 5120),
)

# Weight distribution of each projection: the MLP down projection is heavy tailed.
LAYER_DISTS = {"qkv": "normal", "o": "normal", "gate_up": "normal", "down": "t4"}

W_STD = 0.02


def _rng(seed: int, tensor_id: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(seed), int(tensor_id)])))


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (round to nearest, ties to even); return the uint16 bit patterns.

    Storage-type rounding of generated inputs; NaN is not expected here.
    """
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = (u + 0x7FFF + lsb) >> 16
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to fp32 (exact)."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def x_bf16(M: int, K: int, seed: int = 0, tensor_id: int = X_ID_BASE) -> np.ndarray:
    """Activations X[M, K] ~ N(0, 1), returned as bf16 bit patterns (uint16, row-major)."""
    g = _rng(seed, tensor_id)
    return f32_to_bf16_bits(g.standard_normal((M, K), dtype=np.float32))


def w_f32(N: int, K: int, seed: int = 0, tensor_id: int = 0, dist: str = "normal",
          std: float = W_STD) -> np.ndarray:
    """Weights W[N, K] in fp32: N(0, std) or std * Student-t(nu=4) (dist='t4')."""
    g = _rng(seed, tensor_id)
    if dist == "normal":
        w = g.standard_normal((N, K), dtype=np.float32) * np.float32(std)
    elif dist == "t4":
        w = (g.standard_t(4.0, size=(N, K)) * std).astype(np.float32)
    else:
        raise ValueError(f"unknown weight distribution {dist!r}")
    return np.ascontiguousarray(w, dtype=np.float32)


# ---------------------------------------------------------------------------
# Device-side generators (torch, CUDA). Only draw and round; no method arithmetic.

def _torch_gen(seed: int, tensor_id: int, device):
    import torch
    g = torch.Generator(device=device)
    g.manual_seed((int(seed) * 1_000_003 + int(tensor_id)) & 0x7FFF_FFFF_FFFF_FFFF)
    return g


def x_bf16_torch(M: int, K: int, seed: int, tensor_id: int, device):
    """Activations X[M, K] ~ N(0, 1) as a bf16 tensor on `device`."""
    import torch
    g = _torch_gen(seed, tensor_id, device)
    return torch.randn((M, K), generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)


def w_f32_torch(N: int, K: int, seed: int, tensor_id: int, device, dist: str = "normal",
                std: float = W_STD):
    """Weights W[N, K] as an fp32 tensor on `device`: N(0, std) or std * t(4).

    t(4) is drawn as Z / sqrt(V / 4) with V the sum of four squared normals (chi-square, 4 dof).
    """
    import torch
    g = _torch_gen(seed, tensor_id, device)
    z = torch.randn((N, K), generator=g, device=device, dtype=torch.float32)
    if dist == "normal":
        return z.mul_(std)
    if dist == "t4":
        v = torch.zeros_like(z)
        for _ in range(4):
            e = torch.randn((N, K), generator=g, device=device, dtype=torch.float32)
            v.addcmul_(e, e)
            del e
        return z.div_(v.mul_(0.25).sqrt_()).mul_(std)
    raise ValueError(f"unknown weight distribution {dist!r}")


# ---------------------------------------------------------------------------
# Gated DeltaNet commit inputs: per-head states and per-node key/value/gate/step of a draft tree.

def gdn_inputs(H: int, d_k: int, d_v: int, n_nodes: int, seed: int = 0):
    """(S0 [H, d_v, d_k], K [n_nodes, H, d_k], V [n_nodes, H, d_v], alpha [n_nodes, H], beta [n_nodes, H]),
    all float32: S0 ~ N(0, 0.1); keys N(0, 1) scaled to unit length (as the layer normalises them);
    V ~ N(0, 1); gates alpha ~ U(0.9, 1); steps beta ~ U(0, 1)."""
    g = _rng(seed, 2_000_000 + H)
    S0 = (g.standard_normal((H, d_v, d_k), dtype=np.float32) * np.float32(0.1)).astype(np.float32)
    K = g.standard_normal((n_nodes, H, d_k), dtype=np.float32)
    K = (K / np.linalg.norm(K, axis=2, keepdims=True)).astype(np.float32)
    V = g.standard_normal((n_nodes, H, d_v), dtype=np.float32)
    alpha = g.uniform(0.9, 1.0, (n_nodes, H)).astype(np.float32)
    beta = g.uniform(0.0, 1.0, (n_nodes, H)).astype(np.float32)
    return S0, K, V, alpha, beta


def gdn_inputs_torch(H: int, d_k: int, d_v: int, n_nodes: int, seed: int, device):
    """The same recipe drawn on `device` with torch (for the bench's 1,536 heads)."""
    import torch
    gen = _torch_gen(seed, 2_000_000 + H, device)
    S0 = torch.randn((H, d_v, d_k), generator=gen, device=device) * 0.1
    K = torch.randn((n_nodes, H, d_k), generator=gen, device=device)
    K = K / K.norm(dim=2, keepdim=True)
    V = torch.randn((n_nodes, H, d_v), generator=gen, device=device)
    alpha = torch.rand((n_nodes, H), generator=gen, device=device) * 0.1 + 0.9
    beta = torch.rand((n_nodes, H), generator=gen, device=device)
    return S0, K.contiguous(), V, alpha, beta
