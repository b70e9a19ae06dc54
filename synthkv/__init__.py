"""Seeded synthetic K caches and decode queries for the Fathom key scan.

This module only draws inputs.  It holds none of the scan's arithmetic
(no bit planes, no allocation, no scores, no top-k); both the CPU oracle and
the CUDA library consume what it returns.

What it draws (Fathom, "Fathom Makes KV-Cache Scans Query-Adaptive...",
method paragraphs; arXiv 2609.17652 abstract): the 4-bit K cache that a
quantised serving stack keeps anyway, shaped like Qwen3-8B GQA layers (8 KV heads of
d = 128 channels, 32 query heads), with contexts up to 1M tokens.  The pages
use real models and sessions that are not available here, so every input is
synthetic, with this recipe per (session, KV head):

* channel means  mu_c ~ N(0, 1); channel spreads sigma_c log-uniform in
  [0.1, 10]; four outlier channels per head (drawn without replacement) have
  mu_c and sigma_c multiplied by 10;
* keys k_{i,c} ~ N(mu_c, sigma_c) in fp32;
* the serving stack's per-channel asymmetric min-max 4-bit quantiser:
  m_c = min_i k, M_c = max_i k, s_c = (M_c - m_c) / 15 (fp64, stored fp32),
  u = clamp(floor((k - m_c) / s_c + 0.5), 0, 15) in fp64 from the stored
  fp32 m_c, s_c (u = 0 when s_c = 0), packed token-major, two channels per
  byte, low nibble = even channel;
* each query head h of KV head g = h // G mixes four key directions plus
  noise: q = sum_l a_l * sqrt(d) * k_{r_l} / |k_{r_l}| / 2 + N(0, I_d), with
  r_l uniform over the context and a_l ~ N(0, 1); rounded to bf16 (RNE) or
  kept fp32.

The allocator's sigma_c input is the generator's population sigma_c
(outliers included): it stands for calibrated channel statistics.

Quantiser variant (token_group > 0): the same min-max quantiser applied to
each run of token_group consecutive tokens on its own, so m and s are
[h_kv, ceil(n / token_group), d] (the pages give no group size; per-channel
statistics over the whole context are the default).

Draws use a torch.Generator on the requested device, so a given seed gives
the same case on the same device type and torch build.  Small cases are drawn
on the CPU; the 1M-token cases are drawn on the GPU (the CPU draw of 1G
normals takes minutes).
"""

from __future__ import annotations

import dataclasses
import math
from typing import List, Optional

import torch

__all__ = ["KVCase", "make_case", "make_ragged", "CONFIGS", "pack_nibbles"]


@dataclasses.dataclass
class KVCase:
    """One session's quantised K cache and one decode step's queries."""

    n: int
    d: int
    h_kv: int
    h_q: int
    codes: torch.Tensor        # uint8 [h_kv, n, d/2], low nibble = even channel
    qmin: torch.Tensor         # float32 [h_kv, d] (m_c), or [h_kv, groups, d] per token group
    qscale: torch.Tensor       # float32 [h_kv, d] (s_c), or [h_kv, groups, d] per token group
    sigma: torch.Tensor        # float32 [h_kv, d]   (population sigma_c)
    q: torch.Tensor            # float32 [h_q, d] holding the exact query values
    q_dtype: str               # "bf16" or "f32": the storage type handed to the library
    keys: Optional[torch.Tensor] = None  # float32 [h_kv, n, d] (kept for small cases)
    token_group: int = 0       # tokens per quantiser group (0: the whole context)

    @property
    def group(self) -> int:
        return self.h_q // self.h_kv

    def q_storage(self) -> torch.Tensor:
        """The query tensor in its storage type (bf16 or f32)."""
        return self.q.to(torch.bfloat16) if self.q_dtype == "bf16" else self.q

    def to(self, device) -> "KVCase":
        f = lambda t: None if t is None else t.to(device)
        return dataclasses.replace(
            self, codes=f(self.codes), qmin=f(self.qmin), qscale=f(self.qscale),
            sigma=f(self.sigma), q=f(self.q), keys=f(self.keys))


def pack_nibbles(u: torch.Tensor) -> torch.Tensor:
    """[.., n, d] uint8 codes in [0, 15] -> [.., n, d/2], low nibble = even channel."""
    return (u[..., 0::2] | (u[..., 1::2] << 4)).contiguous()


def _quantise_head(k: torch.Tensor):
    """Per-channel asymmetric min-max 4-bit quantiser of one head's keys [n, d]."""
    m32 = k.min(dim=0).values
    M32 = k.max(dim=0).values
    s32 = ((M32.double() - m32.double()) / 15.0).float()
    m = m32.double()
    s = s32.double()
    u = torch.empty(k.shape, dtype=torch.uint8, device=k.device)
    step = 1 << 20  # bounded fp64 temporaries
    safe = torch.where(s == 0, torch.ones_like(s), s)
    for i0 in range(0, k.shape[0], step):
        x = (k[i0:i0 + step].double() - m) / safe
        x = torch.floor(x + 0.5).clamp_(0.0, 15.0)
        x = torch.where(s == 0, torch.zeros_like(x), x)
        u[i0:i0 + step] = x.to(torch.uint8)
    return u, m32, s32


def make_case(seed: int, n: int, h_kv: int, h_q: int, d: int = 128,
              q_dtype: str = "bf16", device="cpu", keep_keys: Optional[bool] = None,
              outliers: int = 4, token_group: int = 0) -> KVCase:
    """Draw one session: K cache of n tokens x h_kv heads x d channels and h_q queries.

    token_group > 0 quantises every run of token_group tokens with its own
    min-max statistics (the draws are the same as for token_group = 0)."""
    if h_q % h_kv:
        raise ValueError("h_q must be a multiple of h_kv")
    if keep_keys is None:
        keep_keys = n * h_kv * d <= (1 << 24)
    dev = torch.device(device)
    gen = torch.Generator(device=dev).manual_seed(int(seed))
    G = h_q // h_kv

    mu = torch.randn(h_kv, d, generator=gen, device=dev, dtype=torch.float32)
    lo, hi = math.log(0.1), math.log(10.0)
    sigma = torch.exp(lo + (hi - lo) * torch.rand(h_kv, d, generator=gen, device=dev,
                                                   dtype=torch.float32))
    for g in range(h_kv):
        out = torch.randperm(d, generator=gen, device=dev)[:outliers]
        mu[g, out] *= 10.0
        sigma[g, out] *= 10.0

    codes = torch.empty(h_kv, n, d // 2, dtype=torch.uint8, device=dev)
    ng = (n + token_group - 1) // token_group if token_group > 0 else 0
    shape = (h_kv, ng, d) if token_group > 0 else (h_kv, d)
    qmin = torch.empty(shape, dtype=torch.float32, device=dev)
    qscale = torch.empty(shape, dtype=torch.float32, device=dev)
    q = torch.empty(h_q, d, dtype=torch.float32, device=dev)
    keys = torch.empty(h_kv, n, d, dtype=torch.float32, device=dev) if keep_keys else None

    for g in range(h_kv):
        k = torch.randn(n, d, generator=gen, device=dev, dtype=torch.float32)
        k.mul_(sigma[g]).add_(mu[g])
        if token_group > 0:
            for j in range(ng):
                t0, t1 = j * token_group, min(n, (j + 1) * token_group)
                u, m32, s32 = _quantise_head(k[t0:t1])
                codes[g, t0:t1] = pack_nibbles(u)
                qmin[g, j] = m32
                qscale[g, j] = s32
            del u
        else:
            u, m32, s32 = _quantise_head(k)
            codes[g] = pack_nibbles(u)
            del u
            qmin[g] = m32
            qscale[g] = s32
        for hh in range(G):
            h = g * G + hh
            r = torch.randint(0, n, (4,), generator=gen, device=dev)
            a = torch.randn(4, generator=gen, device=dev, dtype=torch.float32)
            rows = k[r]
            dirs = rows / rows.norm(dim=1, keepdim=True)
            qv = (a[:, None] * math.sqrt(d) * dirs / 2.0).sum(0)
            qv = qv + torch.randn(d, generator=gen, device=dev, dtype=torch.float32)
            if q_dtype == "bf16":
                qv = qv.to(torch.bfloat16).float()
            q[h] = qv
        if keep_keys:
            keys[g] = k
        del k

    return KVCase(n=n, d=d, h_kv=h_kv, h_q=h_q, codes=codes, qmin=qmin, qscale=qscale,
                  sigma=sigma, q=q, q_dtype=q_dtype, keys=keys, token_group=token_group)


def make_ragged(seed: int, sessions: int, n_lo: int, n_hi: int, h_kv: int, h_q: int,
                d: int = 128, q_dtype: str = "bf16", device="cpu") -> List[KVCase]:
    """Sessions with context lengths uniform in [n_lo, n_hi] and their own sigma_c."""
    lgen = torch.Generator().manual_seed(int(seed))
    lengths = torch.randint(n_lo, n_hi + 1, (sessions,), generator=lgen).tolist()
    seeds = torch.randint(0, 2**31 - 1, (sessions,), generator=lgen).tolist()
    return [make_case(s, n, h_kv, h_q, d, q_dtype, device) for s, n in zip(seeds, lengths)]


# The five workloads, named by what they are (sizes as in the pages' settings:
# Qwen3-8B GQA layers, contexts up to 1M tokens, budgets 68/92/136 bits).
CONFIGS = {
    "tiny_4k": dict(seed=0, n=4096, h_kv=1, h_q=1, d=128, q_dtype="f32",
                    budgets=[92], k=64),
    "qwen3_8b_layer_131k": dict(seed=1, n=131072, h_kv=8, h_q=32, d=128, q_dtype="bf16",
                                budgets=[68, 92, 136], k=2048),
    "decode_1m": dict(seed=2, n=1048576, h_kv=8, h_q=32, d=128, q_dtype="bf16",
                      budgets=[92, 136], k=2048),
    "ragged_32_sessions": dict(seed=3, sessions=32, n_lo=65536, n_hi=262144, h_kv=8,
                               h_q=32, d=128, q_dtype="bf16", budgets=[92], k=1024),
    "host_resident_1m": dict(seed=4, n=1048576, h_kv=8, h_q=32, d=128, q_dtype="bf16",
                             budgets=[32, 68, 92, 136, 256, 512], k=2048),
}
