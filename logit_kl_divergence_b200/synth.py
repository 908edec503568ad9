"""Seeded synthetic logit workloads.

This module only draws inputs. It holds none of the statistic's arithmetic and
imports neither the CUDA binding nor the oracle, so both sides can be fed the
same tensors from it.

The shapes stand in for the evaluation runs the pages describe: contexts of
8192 tokens ("Qwen3.6 27B Quantization Benchmark", "Measurement method": the
BF16 model's logits are saved, then every quantized model is scored against
them over the same text) and chunked scoring of held-out text
("Mistral-Small-4-119B-2603 GSQ-RCO IQ3_S GGUF", "Quality": 100 chunks of 512
tokens per domain). Vocabulary sizes span 32000 to 262144 entries. No dataset
or model weights are used: logits are random with the structure below.

Recipes (all draws from one ``torch.Generator`` seeded per workload, rows
generated in fixed chunks of ``CHUNK_ROWS`` so the values depend only on the
seed and the device):

``small``      base ~ N(0, 2.0^2) plus +8.0 at one uniform index per row;
               quant = base + N(0, 0.25^2); token ids uniform in [0, V).
``ctx``        base ~ N(0, 2.5^2) plus a Zipf(s=1.1) boost: the vocabulary
               entry of rank r in one random permutation (shared by all rows of
               the tensor) gets +12 * r^-1.1; quant = base + N(0, sigma_i^2)
               with sigma_i drawn per row from {0.05, 0.15, 0.4}; token ids
               sampled from softmax(base) by the Gumbel-max trick. The bf16
               variant rounds both tensors to bf16 (round to nearest even);
               token ids come from the fp32 values before rounding.
``splitrow``   base ~ N(0, 3.0^2) plus +15 at one uniform index per row;
               quant = base + N(0, 0.2^2); token ids uniform.
``edge``       rows split into four equal groups by a seeded permutation:
               (i) one logit +40 in base (near one-hot), quant = base + noise;
               (ii) exact ties: k in [2, 8] random indices set to rowmax + 1.0
               in base only, quant only, or both (one third each);
               (iii) the last 1024 entries -inf in both rows (padding mask);
               (iv) quant = base + 1000.0 (a constant shift, rounded to fp32).
               Base N(0, 2.5^2), noise N(0, 0.15^2); token ids sampled from
               softmax(base).
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch

CHUNK_ROWS = 512

F32, BF16, F16 = 0, 1, 2
_TORCH_DTYPE = {F32: torch.float32, BF16: torch.bfloat16, F16: torch.float16}
_DTYPE_NAME = {F32: "f32", BF16: "bf16", F16: "f16"}


@dataclass
class Workload:
    name: str
    base: torch.Tensor        # [N, V] logits of the reference (BF16) model
    quant: torch.Tensor       # [N, V] logits of the quantized model
    token_ids: torch.Tensor   # [N] int32 next-token ids, or None
    dtype: int                # F32 / BF16 / F16 code

    @property
    def n(self) -> int:
        return self.base.shape[0]

    @property
    def v(self) -> int:
        return self.base.shape[1]

    @property
    def bytes_per_elem(self) -> int:
        return self.base.element_size()


# Named workloads: (recipe, rows, vocab, dtype, seed)
WORKLOADS = {
    "small_64x32000_f32": ("small", 64, 32000, F32, 0),
    "ctx8192_v151936_f32": ("ctx", 8192, 151936, F32, 1),
    "ctx8192_v151936_bf16": ("ctx", 8192, 151936, BF16, 1),
    "ctx4x8192_v151936_bf16": ("ctx", 32768, 151936, BF16, 2),
    "splitrow1_v262144_f32": ("splitrow", 1, 262144, F32, 3),
    "splitrow4_v262144_f32": ("splitrow", 4, 262144, F32, 3),
    "splitrow16_v262144_f32": ("splitrow", 16, 262144, F32, 3),
    "splitrow32_v262144_f32": ("splitrow", 32, 262144, F32, 3),
    "edge_16384x131072_f32": ("edge", 16384, 131072, F32, 4),
}


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _normal(shape, std, g, device):
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32) * std


def _gumbel_argmax(logits: torch.Tensor, g, device) -> torch.Tensor:
    """Sample one index per row from softmax(logits) (Gumbel-max trick)."""
    u = torch.rand(logits.shape, generator=g, device=device, dtype=torch.float32)
    u = u.clamp_(min=1e-20, max=1.0 - 1e-7)
    gumbel = -torch.log(-torch.log(u))
    return torch.argmax(logits + gumbel, dim=1).to(torch.int32)


def _round_store(t: torch.Tensor, dtype: int) -> torch.Tensor:
    return t.to(_TORCH_DTYPE[dtype])


def _alloc(n, v, dtype, device):
    return torch.empty((n, v), dtype=_TORCH_DTYPE[dtype], device=device)


def _small(n, v, dtype, seed, device, peak=8.0, std=2.0, noise=0.25):
    g = _gen(device, seed)
    base, quant = _alloc(n, v, dtype, device), _alloc(n, v, dtype, device)
    tok = torch.empty(n, dtype=torch.int32, device=device)
    for r0 in range(0, n, CHUNK_ROWS):
        r1 = min(n, r0 + CHUNK_ROWS)
        m = r1 - r0
        b = _normal((m, v), std, g, device)
        idx = torch.randint(0, v, (m,), generator=g, device=device)
        b[torch.arange(m, device=device), idx] += peak
        q = b + _normal((m, v), noise, g, device)
        tok[r0:r1] = torch.randint(0, v, (m,), generator=g, device=device).to(torch.int32)
        base[r0:r1] = _round_store(b, dtype)
        quant[r0:r1] = _round_store(q, dtype)
    return base, quant, tok


def _ctx(n, v, dtype, seed, device):
    g = _gen(device, seed)
    # One Zipf-ranked boost vector for the whole tensor.
    perm = torch.randperm(v, generator=g, device=device)
    ranks = torch.arange(1, v + 1, device=device, dtype=torch.float64)
    boost_by_rank = (12.0 * ranks.pow(-1.1)).to(torch.float32)
    boost = torch.empty(v, dtype=torch.float32, device=device)
    boost[perm] = boost_by_rank
    sigmas = torch.tensor([0.05, 0.15, 0.4], dtype=torch.float32, device=device)
    base, quant = _alloc(n, v, dtype, device), _alloc(n, v, dtype, device)
    tok = torch.empty(n, dtype=torch.int32, device=device)
    for r0 in range(0, n, CHUNK_ROWS):
        r1 = min(n, r0 + CHUNK_ROWS)
        m = r1 - r0
        b = _normal((m, v), 2.5, g, device) + boost
        sig = sigmas[torch.randint(0, 3, (m,), generator=g, device=device)]
        q = b + _normal((m, v), 1.0, g, device) * sig[:, None]
        tok[r0:r1] = _gumbel_argmax(b, g, device)
        base[r0:r1] = _round_store(b, dtype)
        quant[r0:r1] = _round_store(q, dtype)
    return base, quant, tok


def _edge(n, v, dtype, seed, device):
    g = _gen(device, seed)
    group = torch.empty(n, dtype=torch.int64, device=device)
    group[torch.randperm(n, generator=g, device=device)] = (
        torch.arange(n, device=device) * 4 // max(n, 1))
    base, quant = _alloc(n, v, dtype, device), _alloc(n, v, dtype, device)
    tok = torch.empty(n, dtype=torch.int32, device=device)
    mask_len = min(1024, v - 1) if v > 1 else 0
    for r0 in range(0, n, CHUNK_ROWS):
        r1 = min(n, r0 + CHUNK_ROWS)
        m = r1 - r0
        rows = torch.arange(m, device=device)
        gr = group[r0:r1]
        b = _normal((m, v), 2.5, g, device)
        noise = _normal((m, v), 0.15, g, device)
        # (i) near one-hot base
        hot = torch.randint(0, v, (m,), generator=g, device=device)
        b[rows, hot] += torch.where(gr == 0, 40.0, 0.0)
        q = b + noise
        # (ii) exact ties at k indices in base only / quant only / both
        which = torch.randint(0, 3, (m,), generator=g, device=device)
        k = torch.randint(2, 9, (m,), generator=g, device=device)
        cand = torch.argsort(torch.rand((m, v), generator=g, device=device), dim=1)[:, :8]
        sel = torch.arange(8, device=device)[None, :] < k[:, None]
        tie_rows = gr == 1
        tb = (tie_rows & (which != 1))[:, None] & sel
        tq = (tie_rows & (which != 0))[:, None] & sel
        bval = (b.max(dim=1).values + 1.0)[:, None].expand(m, 8)
        qval = (q.max(dim=1).values + 1.0)[:, None].expand(m, 8)
        b.scatter_(1, cand, torch.where(tb, bval, b.gather(1, cand)))
        q.scatter_(1, cand, torch.where(tq, qval, q.gather(1, cand)))
        # (iii) padding mask on the last entries of both rows
        pad = gr == 2
        if mask_len > 0:
            b[pad, v - mask_len:] = -math.inf
            q[pad, v - mask_len:] = -math.inf
        # (iv) constant shift of the whole quant row
        shift = gr == 3
        q[shift] = b[shift] + 1000.0
        tok[r0:r1] = _gumbel_argmax(b, g, device)
        base[r0:r1] = _round_store(b, dtype)
        quant[r0:r1] = _round_store(q, dtype)
    return base, quant, tok


_RECIPES = {
    "small": _small,
    "ctx": _ctx,
    "splitrow": lambda n, v, d, s, dev: _small(n, v, d, s, dev, peak=15.0, std=3.0, noise=0.2),
    "edge": _edge,
}


def make(name: str, device="cpu", n: int | None = None, v: int | None = None,
         dtype: int | None = None, seed: int | None = None) -> Workload:
    """Build a named workload; ``n``/``v``/``dtype``/``seed`` override the
    named sizes (same recipe, e.g. fewer rows for a CPU-checkable case)."""
    recipe, n0, v0, d0, s0 = WORKLOADS[name]
    n = n0 if n is None else int(n)
    v = v0 if v is None else int(v)
    d = d0 if dtype is None else int(dtype)
    s = s0 if seed is None else int(seed)
    with torch.no_grad():
        base, quant, tok = _RECIPES[recipe](n, v, d, s, torch.device(device))
    return Workload(name, base.contiguous(), quant.contiguous(), tok.contiguous(), d)


def make_recipe(recipe: str, n: int, v: int, dtype: int = F32, seed: int = 0,
                device="cpu") -> Workload:
    """Any recipe at any size (used for ragged / tiny parity cases)."""
    with torch.no_grad():
        base, quant, tok = _RECIPES[recipe](int(n), int(v), int(dtype), int(seed),
                                            torch.device(device))
    return Workload(f"{recipe}_{n}x{v}_{_DTYPE_NAME[dtype]}", base.contiguous(),
                    quant.contiguous(), tok.contiguous(), int(dtype))
