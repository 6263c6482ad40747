"""Seeded synthetic inputs for Reduced Matrix Multiplication (RMM) workloads.

This module only draws random numbers and rounds them to bfloat16.  It holds
none of RMM's arithmetic (no norms, no selection, no products), so both the
CPU oracle and the CUDA path may take their inputs from it without sharing any
of the method's code.

Recipes (all shapes follow the five workloads the RMM pages benchmark or
describe: a single linear layer, Llama-3.1-8B prefill projections, a
Llama-3.1-70B MLP-up decode GEMV, GQA attention scores and long-context PV):

* Every draw comes from ``numpy.random.Generator(PCG64(seed))`` in float32 and
  is rounded once to bfloat16 with round-to-nearest-even (``torch.bfloat16``).
* Workload ``c`` uses the base seed ``20260814 + c``; head ``h`` of an attention
  workload uses its own sub-stream ``base * 1000 + h``.
* "Outlier channels": activation column ``j`` is scaled by ``c_j = exp(sigma *
  N(0,1))`` (a LogNormal(0, sigma) draw), which gives the heavy-tailed column
  norms RMM's selection reacts to.
* Weights are ``N(0, 1/d)`` with ``d`` the contraction length.
* The full-size PV attention matrix (32 heads of 16384 x 16384) is too large to
  draw on host cores in reasonable time, so ``pv_inputs_device`` draws it with
  torch's seeded device generator instead; parity tests then copy the very same
  array to the host for the oracle.
"""
from __future__ import annotations

import math

import numpy as np
import torch

BASE_SEED = 20260814


def seed_for(workload: int) -> int:
    """Base seed of workload ``workload`` (1..5)."""
    return BASE_SEED + int(workload)


def head_seed(base: int, h: int) -> int:
    """Per-head sub-stream seed."""
    return int(base) * 1000 + int(h)


def rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(int(seed)))


def to_bf16(x: np.ndarray) -> torch.Tensor:
    """Round a float array to bfloat16 (round-to-nearest-even), CPU tensor."""
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)


def widen(t: torch.Tensor) -> np.ndarray:
    """Exact widening of a bfloat16 (or float) tensor to a float64 numpy array."""
    return t.detach().to("cpu", torch.float64).numpy()


def lognormal_scales(g: np.random.Generator, count: int, sigma: float) -> np.ndarray:
    """c_j = exp(sigma * z_j), z_j ~ N(0,1): LogNormal(0, sigma) column scales."""
    return np.exp(sigma * g.standard_normal(count, dtype=np.float32)).astype(np.float32)


def outlier_activations(g: np.random.Generator, n: int, d: int, sigma: float) -> np.ndarray:
    """A[i,j] = z_ij * c_j with z ~ N(0,1) and c_j ~ LogNormal(0, sigma), float32."""
    c = lognormal_scales(g, d, sigma)
    z = g.standard_normal((n, d), dtype=np.float32)
    z *= c[None, :]
    return z


def gaussian_weight(g: np.random.Generator, d: int, m: int) -> np.ndarray:
    """W[d, m] ~ N(0, 1/d), float32, row-major with the contraction index as row."""
    w = g.standard_normal((d, m), dtype=np.float32)
    w *= np.float32(1.0 / math.sqrt(d))
    return w


# ---------------------------------------------------------------- workload 1
def linear_small(seed: int | None = None, n: int = 128, d: int = 1024, m: int = 1024):
    """Single linear layer: A n x d = N(0,1) * LogNormal(0,1) columns, B d x m ~ N(0,1/d).

    Returns bfloat16 CPU tensors (A, B)."""
    g = rng(seed_for(1) if seed is None else seed)
    A = outlier_activations(g, n, d, 1.0)
    B = gaussian_weight(g, d, m)
    return to_bf16(A), to_bf16(B)


def tiny_bruteforce_set(seed: int | None = None, draws: int = 100, n: int = 16, d: int = 12, m: int = 8):
    """Small float64 draws (n x d activations with LogNormal(0,1) columns, d x m weights)
    for exhaustive subset checks at d = 12."""
    g = rng((seed_for(1) if seed is None else seed) * 7 + 1)
    out = []
    for _ in range(draws):
        c = np.exp(g.standard_normal(d))
        A = g.standard_normal((n, d)) * c[None, :]
        B = g.standard_normal((d, m)) / math.sqrt(d)
        out.append((A, B))
    return out


# ---------------------------------------------------------------- workload 2
PREFILL_SHAPES = {
    # name: (d, m)  with the activation operand n x d and the weight d x m
    "q_proj": (4096, 4096),
    "gate_proj": (4096, 14336),
    "up_proj": (4096, 14336),
    "down_proj": (14336, 4096),
}


def _silu(x: np.ndarray) -> np.ndarray:
    return x / (1.0 + np.exp(-x))


def down_proj_sigma(g0: np.ndarray, u0: np.ndarray, c: np.ndarray, target: float = 0.70,
                    thresh: float = 0.05, iters: int = 60) -> float:
    """Bisection for sigma so that a fraction ``target`` of x = c * silu(sigma g0) * sigma u0
    has |x| < thresh, evaluated on the given (already seeded) draws."""
    lo, hi = 1e-3, 20.0
    for _ in range(iters):
        mid = 0.5 * (lo + hi)
        x = c * _silu(mid * g0) * (mid * u0)
        frac = float(np.mean(np.abs(x) < thresh))
        if frac > target:
            lo = mid  # too many small entries: grow sigma
        else:
            hi = mid
    return 0.5 * (lo + hi)


def prefill_projection(name: str, seed: int | None = None, n: int = 4096):
    """Llama-3.1-8B-shaped prefill projection inputs.

    q_proj, gate_proj, up_proj: A = N(0,1) * LogNormal(0,1.5) columns (n x 4096).
    down_proj: A = c_j * silu(g) * u with g, u ~ N(0, sigma^2), c_j ~ LogNormal(0, 1.5),
    sigma chosen by bisection so that 70% of entries have |x| < 0.05 (the
    post-SiLU-times-up activation statistics the workload names).
    Weights N(0, 1/d).  Returns bfloat16 CPU tensors (A [n, d], W [d, m])."""
    d, m = PREFILL_SHAPES[name]
    base = seed_for(2) if seed is None else seed
    idx = list(PREFILL_SHAPES).index(name)
    g = rng(base * 10 + idx)
    if name == "down_proj":
        c = lognormal_scales(g, d, 1.5)
        g0 = g.standard_normal((n, d), dtype=np.float32)
        u0 = g.standard_normal((n, d), dtype=np.float32)
        sub = slice(0, min(n, 64))
        sigma = down_proj_sigma(g0[sub].astype(np.float64), u0[sub].astype(np.float64),
                                np.broadcast_to(c[None, :], g0[sub].shape).astype(np.float64))
        A = (c[None, :] * _silu(np.float32(sigma) * g0) * (np.float32(sigma) * u0)).astype(np.float32)
        del g0, u0
    else:
        A = outlier_activations(g, n, d, 1.5)
    W = gaussian_weight(g, d, m)
    return to_bf16(A), to_bf16(W)


# ---------------------------------------------------------------- workload 3
def decode_gemv(n: int, seed: int | None = None, d: int = 8192, m: int = 28672, weight: bool = True):
    """Llama-3.1-70B MLP-up decode shape: A n x d with N(0,1) * LogNormal(0,1.5) columns,
    W d x m ~ N(0, 1/d).  Returns bfloat16 CPU tensors (A, W or None)."""
    base = seed_for(3) if seed is None else seed
    ga = rng(base * 10 + n)
    A = outlier_activations(ga, n, d, 1.5)
    W = None
    if weight:
        gw = rng(base * 10)
        W = to_bf16(gaussian_weight(gw, d, m))
    return to_bf16(A), W


# ---------------------------------------------------------------- workload 4
def qk_inputs(seed: int | None = None, batch: int = 1, hq: int = 32, hkv: int = 8, n: int = 4096,
              dh: int = 128):
    """GQA attention-score operands: Q [batch, hq, n, dh], K [batch, hkv, n, dh], entries
    N(0,1) times a per-head LogNormal(0,1) scale per head dimension (independent draws
    for every query head and every key/value head).  bfloat16 CPU tensors."""
    base = seed_for(4) if seed is None else seed
    Q = np.empty((batch, hq, n, dh), dtype=np.float32)
    K = np.empty((batch, hkv, n, dh), dtype=np.float32)
    for b in range(batch):
        for h in range(hq):
            Q[b, h] = outlier_activations(rng(head_seed(base, b * 4096 + h)), n, dh, 1.0)
        for h in range(hkv):
            K[b, h] = outlier_activations(rng(head_seed(base, b * 4096 + 2048 + h)), n, dh, 1.0)
    return to_bf16(Q), to_bf16(K)


# ---------------------------------------------------------------- workload 5
def causal_softmax_rows(logits: np.ndarray, offset: int = 0) -> np.ndarray:
    """Row softmax over the entries j <= i + offset (float32); entries above are 0.
    This builds the attention-probability INPUT of PV; it is not part of RMM."""
    n, nk = logits.shape
    j = np.arange(nk)[None, :]
    i = np.arange(n)[:, None]
    mask = j <= i + offset
    x = np.where(mask, logits, -np.inf).astype(np.float32)
    x = x - x.max(axis=1, keepdims=True)
    e = np.exp(x, dtype=np.float32)
    e = np.where(mask, e, 0.0).astype(np.float32)
    return (e / e.sum(axis=1, keepdims=True, dtype=np.float32)).astype(np.float32)


def pv_inputs(seed: int | None = None, batch: int = 1, heads: int = 32, n: int = 16384, dh: int = 128,
              kv_heads: int | None = None):
    """Host-side PV operands for small n: P [batch, heads, n, n] = causal softmax of
    2 * N(0,1) logits (float32, rounded to bfloat16), V [batch, kv_heads, n, dh] ~ N(0,1)."""
    base = seed_for(5) if seed is None else seed
    hkv = heads if kv_heads is None else kv_heads
    P = np.empty((batch, heads, n, n), dtype=np.float32)
    V = np.empty((batch, hkv, n, dh), dtype=np.float32)
    for b in range(batch):
        for h in range(heads):
            g = rng(head_seed(base, b * 4096 + h))
            logits = 2.0 * g.standard_normal((n, n), dtype=np.float32)
            P[b, h] = causal_softmax_rows(logits)
        for h in range(hkv):
            g = rng(head_seed(base, b * 4096 + 2048 + h))
            V[b, h] = g.standard_normal((n, dh), dtype=np.float32)
    return to_bf16(P), to_bf16(V)


def pv_inputs_device(device, seed: int | None = None, batch: int = 1, heads: int = 32, n: int = 16384,
                     dh: int = 128, kv_heads: int | None = None):
    """Device-side PV operands at full size, same recipe as ``pv_inputs`` but drawn with
    torch's seeded generator on ``device`` (one head at a time, float32 softmax, then
    bfloat16).  Returns device tensors (P, V)."""
    base = seed_for(5) if seed is None else seed
    hkv = heads if kv_heads is None else kv_heads
    P = torch.empty((batch, heads, n, n), dtype=torch.bfloat16, device=device)
    V = torch.empty((batch, hkv, n, dh), dtype=torch.bfloat16, device=device)
    gen = torch.Generator(device=device)
    upper = torch.ones((n, n), dtype=torch.bool, device=device).triu_(1)
    for b in range(batch):
        for h in range(heads):
            gen.manual_seed(head_seed(base, b * 4096 + h))
            logits = torch.randn((n, n), generator=gen, device=device, dtype=torch.float32)
            logits.mul_(2.0).masked_fill_(upper, float("-inf"))
            P[b, h] = torch.softmax(logits, dim=1).to(torch.bfloat16)
            del logits
        for h in range(hkv):
            gen.manual_seed(head_seed(base, b * 4096 + 2048 + h))
            V[b, h] = torch.randn((n, dh), generator=gen, device=device, dtype=torch.float32).to(torch.bfloat16)
    del upper
    return P, V


# ------------------------------------------------------------------ decode attention
DECODE_ATTN_SEED = 6  # workload number of the decode-attention inputs


def decode_attention_inputs(seed: int | None = None, batch: int = 2, hq: int = 8, hkv: int = 2, dh: int = 128,
                            nk: int = 1000, L: int | None = None):
    """Decode-attention operands on the host (small sizes): one query row per head.

    Q  [batch, hq, dh]       N(0,1) times a per-head LogNormal(0,1) scale per head dim
    Kt [batch, hkv, dh, L]   the key cache stored dim-major, N(0,1)
    P  [batch, hq, L]        softmax over the first nk positions of 2 N(0,1) logits
                             (float32, then bfloat16), zero past nk
    V  [batch, hkv, L, dh]   the value cache, token-major, N(0,1)
    L defaults to nk rounded up to a multiple of 8 (cache capacity).  bfloat16 CPU tensors."""
    base = seed_for(DECODE_ATTN_SEED) if seed is None else seed
    L = (nk + 7) // 8 * 8 if L is None else L
    Q = np.empty((batch, hq, dh), dtype=np.float32)
    Kt = np.zeros((batch, hkv, dh, L), dtype=np.float32)
    P = np.zeros((batch, hq, L), dtype=np.float32)
    V = np.zeros((batch, hkv, L, dh), dtype=np.float32)
    for b in range(batch):
        for h in range(hq):
            g = rng(head_seed(base, b * 4096 + h))
            Q[b, h] = g.standard_normal(dh, dtype=np.float32) * np.exp(g.standard_normal(dh)).astype(np.float32)
            x = 2.0 * g.standard_normal(nk, dtype=np.float32)
            e = np.exp(x - x.max(), dtype=np.float32)
            P[b, h, :nk] = e / e.sum(dtype=np.float32)
        for h in range(hkv):
            g = rng(head_seed(base, b * 4096 + 2048 + h))
            Kt[b, h, :, :nk] = g.standard_normal((dh, nk), dtype=np.float32)
            V[b, h, :nk] = g.standard_normal((nk, dh), dtype=np.float32)
    return to_bf16(Q), to_bf16(Kt), to_bf16(P), to_bf16(V)


def decode_attention_inputs_device(device, seed: int | None = None, batch: int = 8, hq: int = 32, hkv: int = 8,
                                   dh: int = 128, nk: int = 32768):
    """Full-size decode-attention operands drawn on the device with torch's seeded
    generator, same recipe as ``decode_attention_inputs`` (cache capacity = nk)."""
    base = seed_for(DECODE_ATTN_SEED) if seed is None else seed
    gen = torch.Generator(device=device)
    gen.manual_seed(base)
    f32 = torch.float32
    Q = (torch.randn((batch, hq, dh), generator=gen, device=device, dtype=f32)
         * torch.randn((batch, hq, dh), generator=gen, device=device, dtype=f32).exp()).to(torch.bfloat16)
    Kt = torch.randn((batch, hkv, dh, nk), generator=gen, device=device, dtype=f32).to(torch.bfloat16)
    P = torch.softmax(2.0 * torch.randn((batch, hq, nk), generator=gen, device=device, dtype=f32), dim=-1)
    P = P.to(torch.bfloat16)
    V = torch.randn((batch, hkv, nk, dh), generator=gen, device=device, dtype=f32).to(torch.bfloat16)
    return Q, Kt, P, V


# ------------------------------------------------------------------ MLP block
MLP_SEED = 7  # workload number of the MLP-block inputs


def mlp_block(seed: int | None = None, n: int = 4096, d: int = 4096, f: int = 14336, m: int | None = None):
    """Gated-MLP operands (Llama-3.1-8B shape by default): X [n, d] with N(0,1) entries
    times LogNormal(0, 1.5) column scales; Wg, Wu [d, f] ~ N(0, 1/d); Wd [f, m] ~ N(0, 1/f)
    with m = d.  bfloat16 CPU tensors."""
    base = seed_for(MLP_SEED) if seed is None else seed
    m = d if m is None else m
    g = rng(base)
    X = outlier_activations(g, n, d, 1.5)
    Wg = gaussian_weight(g, d, f)
    Wu = gaussian_weight(g, d, f)
    Wd = gaussian_weight(g, f, m)
    return to_bf16(X), to_bf16(Wg), to_bf16(Wu), to_bf16(Wd)


def int8_weight(g: np.random.Generator, d: int, m: int):
    """A N(0, 1/d) weight quantized to int8 with one scale per output column:
    scale_c = max_j |W[j, c]| / 127, Wq = round(W / scale) clipped to [-127, 127].
    Returns (Wq int8 CPU tensor [d, m], scale float32 CPU tensor [m])."""
    w = gaussian_weight(g, d, m)
    scale = np.maximum(np.abs(w).max(axis=0), np.float32(1e-30)) / np.float32(127.0)
    q = np.clip(np.rint(w / scale[None, :]), -127, 127).astype(np.int8)
    return torch.from_numpy(q), torch.from_numpy(scale.astype(np.float32))
