"""Seeded synthetic inputs for the blockwise-FP8 linear layer.

Shared by the tests, the smoke check and the benchmark.  This module holds
input generation only — none of the method's arithmetic — so that the CUDA
library and the CPU oracle are both fed the same bf16 bytes.

The workloads stand in for the pages' models (Llama 3.1 8B and
Qwen3-30B-A3B, "NVIDIA NeMo RL erreicht 48% ..." sections "Der technische
Durchbruch" and "Leistungsgewinne in der Praxis"; "NeMo-RL v0.3 mit
Megatron-Core ..."): shapes only, random values, no weights or datasets.

All values are drawn in fp32 from a seeded torch generator and rounded to
bf16 (round-to-nearest-even).  ``device`` selects where they are drawn; a
given (seed, device) pair always yields the same bytes.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch

# Llama-3.1-8B-like dense linear layers: (name, K = in_features, N = out_features)
LLAMA8B_LAYERS = [
    ("qkv", 4096, 6144),
    ("o_proj", 4096, 4096),
    ("gate_up", 4096, 28672),
    ("down", 14336, 4096),
]
LLAMA8B_TOKENS = 8192

# Qwen3-30B-A3B-like MoE expert layers
MOE_HIDDEN = 2048
MOE_EXPERTS = 128
MOE_TOPK = 8
MOE_INTER = 768
MOE_TOKENS = 16384
MOE_ZIPF = 1.1

PACKED_TOKENS = 32768
PACKED_NSEQ = 4
# generation (decode) batch over an FP8 KV cache: rollouts of Llama-3.1-8B
# ("NeMo-RL v0.3 mit Megatron-Core ...": 16K-token contexts)
DECODE_BATCH = 64
DECODE_LMAX = 16384


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def normal_bf16(shape, std: float, seed: int, device="cpu") -> torch.Tensor:
    g = _gen(seed, device)
    return (torch.randn(shape, generator=g, device=device, dtype=torch.float32) * std).to(torch.bfloat16)


def activations_with_outliers(M: int, K: int, seed: int, device="cpu",
                              frac: float = 0.001, factor: float = 50.0) -> torch.Tensor:
    """X ~ N(0,1) with round(frac*K) seeded outlier channels multiplied by `factor`."""
    g = _gen(seed, device)
    x = torch.randn((M, K), generator=g, device=device, dtype=torch.float32)
    n_out = int(round(frac * K))
    gc = _gen(seed + 7919, "cpu")
    ch = torch.randperm(K, generator=gc)[:n_out].to(device)
    if n_out:
        x[:, ch] *= factor
    return x.to(torch.bfloat16)


def outlier_channels(K: int, seed: int, frac: float = 0.001):
    n_out = int(round(frac * K))
    gc = _gen(seed + 7919, "cpu")
    return torch.randperm(K, generator=gc)[:n_out].tolist()


# ------------------------------------------------------------------ tiny ---
def tiny(seed: int = 0, device="cpu"):
    """X [256,512] ~N(0,1), W [512,512] ~N(0,0.02), dY [256,512] ~N(0,1)*1e-3."""
    X = normal_bf16((256, 512), 1.0, seed, device)
    W = normal_bf16((512, 512), 0.02, seed + 100, device)
    dY = normal_bf16((256, 512), 1e-3, seed + 1, device)
    return X, W, dY


# ------------------------------------------------------- llama-8B layers ---
def llama_layer(name: str, seed: int = 0, device="cpu", M: int = LLAMA8B_TOKENS):
    """One Llama-8B-like linear layer: X [M,K] (0.1% outlier channels x50),
    W [N,K] ~N(0,0.02), dY [M,N] ~N(0,1)*1e-3."""
    idx = [l[0] for l in LLAMA8B_LAYERS].index(name)
    _, K, N = LLAMA8B_LAYERS[idx]
    base = seed * 1000 + idx * 10
    X = activations_with_outliers(M, K, base + 1, device)
    W = normal_bf16((N, K), 0.02, base + 2, device)
    dY = normal_bf16((M, N), 1e-3, base + 3, device)
    return X, W, dY


def llama_weight(name: str, layer: int, seed: int = 0, device="cpu"):
    idx = [l[0] for l in LLAMA8B_LAYERS].index(name)
    _, K, N = LLAMA8B_LAYERS[idx]
    return normal_bf16((N, K), 0.02, seed * 100003 + layer * 17 + idx, device)


def requant_update_(W: torch.Tensor, step: int, layer: int, idx: int, seed: int = 0,
                    std: float = 1e-4) -> None:
    """Adam-like perturbation of one weight in place: W <- bf16(fp32(W) + N(0, std^2))."""
    g = _gen(seed * 7777 + step * 1009 + layer * 13 + idx, W.device)
    upd = torch.randn(W.shape, generator=g, device=W.device, dtype=torch.float32) * std
    W.copy_((W.float() + upd).to(torch.bfloat16))


# -------------------------------------------------------------------- MoE --
@dataclass
class MoERouting:
    offsets: list          # padded segment offsets, length G+1, multiples of 128
    counts: list           # unpadded rows per expert
    row_token: torch.Tensor  # [M_total_pad] int64 token index of each row, -1 = padding
    m_total_pad: int


def moe_routing(seed: int = 0, tokens: int = MOE_TOKENS, experts: int = MOE_EXPERTS,
                topk: int = MOE_TOPK, zipf: float = MOE_ZIPF) -> MoERouting:
    """Seeded Zipf(1.1) expert popularity; each token takes `topk` distinct
    experts (Gumbel-top-k); rows grouped by expert, stable by token, each
    segment zero-padded to a multiple of 128."""
    g = _gen(seed + 424242, "cpu")
    ranks = torch.randperm(experts, generator=g) + 1          # expert -> Zipf rank
    logp = -zipf * torch.log(ranks.double())
    u = torch.rand((tokens, experts), generator=g, dtype=torch.float64).clamp_(1e-300, 1.0)
    gumbel = -torch.log(-torch.log(u))
    choice = torch.topk(logp[None, :] + gumbel, topk, dim=1).indices   # [T, topk]
    tok = torch.arange(tokens).repeat_interleave(topk)
    exp = choice.reshape(-1)
    order = torch.argsort(exp * tokens + tok)   # by expert, then by token (stable)
    tok_sorted, exp_sorted = tok[order], exp[order]
    counts = torch.bincount(exp_sorted, minlength=experts).tolist()
    offsets = [0]
    for c in counts:
        offsets.append(offsets[-1] + ((c + 127) // 128) * 128)
    row_token = torch.full((offsets[-1],), -1, dtype=torch.int64)
    pos = 0
    for e in range(experts):
        c = counts[e]
        row_token[offsets[e]:offsets[e] + c] = tok_sorted[pos:pos + c]
        pos += c
    return MoERouting(offsets, counts, row_token, offsets[-1])


def moe_permuted(routing: MoERouting, width: int, std: float, seed: int, device="cpu"):
    """Token matrix [tokens, width] ~N(0,std) gathered into expert order, with
    zero rows in the padding."""
    T = int(routing.row_token.max().item()) + 1 if routing.row_token.numel() else 0
    T = max(T, MOE_TOKENS)
    base = normal_bf16((T, width), std, seed, device)
    rt = routing.row_token.to(device)
    out = torch.zeros((routing.m_total_pad, width), dtype=torch.bfloat16, device=device)
    valid = rt >= 0
    out[valid] = base[rt[valid]]
    return out


def moe_experts(G: int, N: int, K: int, seed: int, device="cpu"):
    return normal_bf16((G, N, K), 0.02, seed, device)


# ------------------------------------------------------ long packed batch --
def packed_lengths(seed: int = 0, nseq: int = PACKED_NSEQ, total: int = PACKED_TOKENS):
    g = _gen(seed + 31337, "cpu")
    lens = torch.randint(1024, 16385, (nseq,), generator=g).tolist()
    return lens


def student_t_bf16(shape, nu: int, scale: float, seed: int, device="cpu") -> torch.Tensor:
    """Student-t with integer nu: Z / sqrt(chi2_nu / nu), chi2 as a sum of squares."""
    g = _gen(seed, device)
    z = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    chi = torch.zeros(shape, device=device, dtype=torch.float32)
    for _ in range(nu):
        chi += torch.randn(shape, generator=g, device=device, dtype=torch.float32) ** 2
    return (z / torch.sqrt(chi / nu) * scale).to(torch.bfloat16)


def packed_rows_mask(seed: int = 0, total: int = PACKED_TOKENS):
    """Boolean [total]: True for real tokens, False for zero padding.  Each
    sequence is padded to a multiple of 128; the batch is padded (or the
    last sequence truncated) to `total`."""
    lens = packed_lengths(seed, total=total)
    mask = torch.zeros(total, dtype=torch.bool)
    pos = 0
    for L in lens:
        if pos >= total:
            break
        n = min(L, total - pos)
        mask[pos:pos + n] = True
        pos += ((L + 127) // 128) * 128
    return mask


def packed_segments(seed: int = 0, total: int = PACKED_TOKENS):
    """(offsets, lengths) of the packing drawn by packed_rows_mask: segment s
    covers tokens [off[s], off[s+1]) (each sequence padded to a multiple of
    128, the last one cut at `total`), of which the first len[s] are real."""
    lens = packed_lengths(seed, total=total)
    off, ln = [0], []
    pos = 0
    for L in lens:
        if pos >= total:
            break
        ln.append(min(L, total - pos))
        pos += min(((L + 127) // 128) * 128, total - pos)
        off.append(pos)
    return off, ln


def packed_activations(K: int, seed: int = 0, device="cpu", total: int = PACKED_TOKENS,
                       scale: float = 1.0, mask_seed: int = 0):
    """[total, K] Student-t (nu=3) values times `scale`, zero on the padding
    rows of the packing drawn with `mask_seed` (shared by X and dY)."""
    mask = packed_rows_mask(mask_seed, total).to(device)
    x = student_t_bf16((total, K), 3, scale, seed * 97 + K, device)
    x[~mask] = 0
    return x


def decode_lengths(seed: int = 0, batch: int = DECODE_BATCH, lmax: int = DECODE_LMAX):
    """(cache lengths [batch], Lmax) of a generation step: each rollout's
    cached tokens (prompt plus tokens generated so far), uniform in
    [256, lmax]."""
    g = _gen(seed + 4242, "cpu")
    return torch.randint(256, lmax + 1, (batch,), generator=g).tolist(), lmax


def padded_shape(n: int, mult: int = 128) -> int:
    return int(math.ceil(n / mult) * mult)
