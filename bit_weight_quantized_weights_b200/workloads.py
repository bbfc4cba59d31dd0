"""Seeded synthetic inputs and the workload table (no quantization arithmetic).

Both the CUDA path and the CPU oracle consume exactly the tensors produced
here. The recipe: a CPU torch.Generator seeded per workload; weights
W ~ N(0, 0.02) fp32 [N, K]; activations x ~ N(0, 1) fp32 [M, K] drawn after W,
a set of outlier channels (round(frac * K) columns chosen by randperm on the
same generator) multiplied by a constant, then x is rounded once to bf16.
The shapes are the Llama / Qwen linear-layer shapes the quantized-kernel pages
evaluate on (synthetic stand-ins: no trained weights are involved).
"""

import torch

# (name, kind, shapes, extra) for each workload family.
GEMV_TINY = dict(name="gemv_tiny_int4_g64", M=1, N=1024, K=1024, group=64)
NF4_DEQUANT_SHAPES = [(28672, 8192), (8192, 8192), (5120, 25600)]
DECODE_SHAPES = [(4096, 4096), (11008, 4096), (4096, 11008)]
DECODE_M = [1, 4, 8, 16]
PREFILL_SHAPES = [(4096, 4096), (14336, 4096), (4096, 14336)]
PREFILL_M = [512, 2048, 8192]
MSD_SHAPES = [(5120, 5120), (25600, 5120), (5120, 25600)]
MSD_M = [1, 16, 128, 1024]

DECODE_OUTLIERS = (0.01, 20.0)
MSD_OUTLIERS = (0.005, 50.0)


def generator(seed=0):
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def weights(n, k, seed=0, gen=None):
    """fp32 [N, K] ~ N(0, 0.02), CPU."""
    g = gen if gen is not None else generator(seed)
    return torch.randn(n, k, generator=g, dtype=torch.float32) * 0.02


def activations(m, k, seed=0, gen=None, outliers=None):
    """bf16 [M, K]: N(0, 1) with optional (fraction, scale) outlier channels, CPU."""
    g = gen if gen is not None else generator(seed)
    x = torch.randn(m, k, generator=g, dtype=torch.float32)
    if outliers is not None:
        frac, scale = outliers
        cnt = max(1, round(frac * k))
        idx = torch.randperm(k, generator=g)[:cnt]
        x[:, idx] *= scale
    return x.to(torch.bfloat16)


def layer(m, n, k, seed=0, outliers=None):
    """(W fp32 [N, K], x bf16 [M, K]) drawn in that order from one generator."""
    g = generator(seed)
    w = weights(n, k, gen=g)
    x = activations(m, k, gen=g, outliers=outliers)
    return w, x


def flat_weights(n, k, seed=0):
    """fp32 [N, K] weights for the standalone NF4 dequantization workload."""
    return weights(n, k, seed=seed)


def scaled_weights(n, k, seed=0, row_exp=None, block_exp=None, factor=1.0):
    """fp32 [N, K] ~ N(0, 0.02) x `factor`, with rows and/or 64-element blocks
    (of the flattened row-major matrix) scaled by powers of ten, CPU:

    row_exp (lo, hi): row n is multiplied by 10^(lo + n mod (hi - lo + 1));
    block_exp (lo, hi): each block is multiplied by 10^u, u drawn uniformly
    from [lo, hi] on the same generator after W.

    Layers whose weights span many orders of magnitude, for the NF4 paths
    whose block absmax enters a narrower floating-point type."""
    g = generator(seed)
    w = weights(n, k, gen=g) * factor
    if block_exp is not None:
        lo, hi = block_exp
        u = torch.rand(n * k // 64, generator=g, dtype=torch.float64) * (hi - lo) + lo
        w = (w.reshape(-1, 64).double() * torch.pow(10.0, u)[:, None]).float().reshape(n, k)
    if row_exp is not None:
        lo, hi = row_exp
        e = lo + torch.arange(n) % (hi - lo + 1)
        w = (w.double() * torch.pow(10.0, e.double())[:, None]).float()
    return w


# Decode attention over a quantized KV cache: Qwen3-32B's attention heads
# (64 query heads sharing 8 KV heads, head dimension 128).
ATTN_HEADS = dict(Hq=64, Hkv=8, D=128)
KV_K_OUTLIERS = (0.04, 8.0)


def decode_attention(b, hq, hkv, length, d=128, seed=0, k_outliers=KV_K_OUTLIERS):
    """(q bf16 [B, Hq, D], K fp32 [B, Hkv, L, D], V fp32 [B, Hkv, L, D]), CPU,
    drawn in that order from one generator: q ~ N(0, 1) rounded once to bf16,
    K ~ N(0, 0.5) with a few channels (the same for every token of a head,
    chosen by randperm) scaled up, as keys carry per-channel outliers, and
    V ~ N(0, 1)."""
    g = generator(seed)
    q = torch.randn(b, hq, d, generator=g, dtype=torch.float32).to(torch.bfloat16)
    k = torch.randn(b, hkv, length, d, generator=g, dtype=torch.float32) * 0.5
    if k_outliers is not None:
        frac, scale = k_outliers
        cnt = max(1, round(frac * d))
        for h in range(hkv):
            idx = torch.randperm(d, generator=g)[:cnt]
            k[:, h, :, idx] *= scale
    v = torch.randn(b, hkv, length, d, generator=g, dtype=torch.float32)
    return q, k, v
