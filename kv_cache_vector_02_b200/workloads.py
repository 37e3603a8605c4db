"""Seeded synthetic workloads (shapes and value laws only; none of the method).

The five workload families follow the statement of the problem:
  tiny        1 sequence, 1 kv head, 1 query head, 1024 tokens; K, V ~ N(0,1) per
              coordinate, key channels 0, 32, 64, 96 scaled x10 (READING: the four
              fixed outlier channels are not named; these are evenly spaced).
  llama8b     Llama-3-8B single layer: 8 kv heads, 32 query heads, 4096-token
              context, then decode steps each appending one token.  Per (K/V,
              kv head, channel) std = exp(0.5 * N(0,1)); round(2% of 128) = 3
              outlier channels per (K/V, kv head) scaled x8.
  batched     32 sequences x 4096 tokens in the llama8b layout and law, physical
              blocks a seeded random permutation.
  long70b     1 sequence x 131072 tokens, 8 kv heads, 64 query heads; std =
              exp(0.7 * N(0,1)), round(1% of 128) = 1 channel x12.
  prefill80   80 layers x 8 kv heads x 32768 tokens (flattened into the token
              axis, one context), llama8b law drawn per layer.
Queries are N(0, 1/128) per coordinate.  fp16 everywhere.

Random numbers: per-channel scales and outlier picks come from numpy's
PCG64 (small arrays); bulk normals from torch generators on the target device,
seeded per (seed, tag, chunk).  The same call on the same device is
bit-reproducible; tests that compare the GPU with the CPU oracle generate once
and hand the very same fp16 tensor to both.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

PAGE = 16
D = 128


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int                 # sequences
    T: int                 # context tokens per sequence (compressed prefill)
    Hkv: int
    Hq: int
    bits: int = 4
    rotation: int = 0      # 0 Haar, 1 Hadamard
    key_mode: int = 0      # 0 prod (QJL), 1 MSE
    law: str = "llama8b"   # "tiny" | "llama8b" | "long70b"
    layers: int = 1        # prefill80: layers flattened into the token axis
    decode_steps: int = 0  # appended tokens, one decode each
    param_seed: int = 0
    data_seed: int = 1

    @property
    def tokens(self) -> int:
        """Tokens compressed by the prefill (all sequences, all layers)."""
        return self.B * self.T * self.layers

    @property
    def max_seq_len(self) -> int:
        return self.T + self.decode_steps

    @property
    def max_blocks(self) -> int:
        return (self.max_seq_len + PAGE - 1) // PAGE

    @property
    def num_blocks(self) -> int:
        return self.B * self.max_blocks if self.layers == 1 else (self.tokens + PAGE - 1) // PAGE

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "tiny": Workload("tiny", B=1, T=1024, Hkv=1, Hq=1, law="tiny", decode_steps=0),
    "llama8b": Workload("llama8b", B=1, T=4096, Hkv=8, Hq=32, decode_steps=64),
    "batched": Workload("batched", B=32, T=4096, Hkv=8, Hq=32),
    "long70b": Workload("long70b", B=1, T=131072, Hkv=8, Hq=64, law="long70b"),
    "prefill80": Workload("prefill80", B=1, T=32768, Hkv=8, Hq=32, layers=80),
}


# ---------------------------------------------------------------- per-channel law
def channel_scales(w: Workload, kind: int, layer: int = 0) -> np.ndarray:
    """std per (kv head, channel) for kind 0 = K, 1 = V: float32 [Hkv, 128]."""
    rng = np.random.default_rng([w.data_seed, 7919, kind, layer])
    if w.law == "tiny":
        s = np.ones((w.Hkv, D), np.float32)
        if kind == 0:
            s[:, [0, 32, 64, 96]] = 10.0
        return s
    sig, frac, mult = (0.5, 0.02, 8.0) if w.law == "llama8b" else (0.7, 0.01, 12.0)
    s = np.exp(sig * rng.standard_normal((w.Hkv, D))).astype(np.float32)
    n_out = int(round(frac * D))
    for h in range(w.Hkv):
        ch = rng.choice(D, size=n_out, replace=False)
        s[h, ch] *= mult
    return s


def _gen(shape, seed_parts, device):
    import torch
    seed = int(np.random.SeedSequence(list(seed_parts)).generate_state(1, np.uint64)[0] & ((1 << 63) - 1))
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32)


def gen_kv(w: Workload, kind: int, device="cpu", token_offset: int = 0, n_tokens: int | None = None):
    """K (kind 0) or V (kind 1) prefill tensor, fp16 [n_tokens, Hkv, 128].

    Tokens are generated in chunks of 32768 so that any sub-range is
    reproducible on its own (chunk c uses seed (data_seed, kind, c)).
    """
    import torch
    if n_tokens is None:
        n_tokens = w.tokens - token_offset
    out = torch.empty((n_tokens, w.Hkv, D), dtype=torch.float16, device=device)
    CH = 32768
    t = token_offset
    end = token_offset + n_tokens
    while t < end:
        c = t // CH
        c0, c1 = c * CH, min((c + 1) * CH, w.tokens)
        layer = c0 // (w.B * w.T) if w.layers > 1 else 0
        z = _gen((c1 - c0, w.Hkv, D), (w.data_seed, 11, kind, c), device)
        sc = torch.as_tensor(channel_scales(w, kind, layer), device=device)
        z.mul_(sc)
        lo, hi = max(t, c0), min(end, c1)
        out[lo - token_offset:hi - token_offset] = z[lo - c0:hi - c0].to(torch.float16)
        t = hi
    return out


def gen_step_kv(w: Workload, kind: int, step: int, device="cpu"):
    """The token appended at decode step `step` for every sequence: fp16 [B, Hkv, 128]."""
    import torch
    z = _gen((w.B, w.Hkv, D), (w.data_seed, 13, kind, step), device)
    z.mul_(torch.as_tensor(channel_scales(w, kind), device=device))
    return z.to(torch.float16)


def gen_q(w: Workload, step: int = 0, device="cpu"):
    """Decode queries, fp16 [B, Hq, 128], N(0, 1/128) per coordinate."""
    import torch
    z = _gen((w.B, w.Hq, D), (w.data_seed, 17, step), device)
    return (z / math.sqrt(D)).to(torch.float16)


def block_table(w: Workload) -> np.ndarray:
    """[B, max_blocks] int32: a seeded random permutation of the physical blocks."""
    rng = np.random.default_rng([w.data_seed, 23])
    perm = rng.permutation(w.B * w.max_blocks).astype(np.int32)
    return perm.reshape(w.B, w.max_blocks)


def prefill_slots(w: Workload, bt: np.ndarray) -> np.ndarray:
    """slot_mapping of the prefill (token-major over sequences): [B*T] int32."""
    t = np.arange(w.T)
    return np.concatenate([bt[b][t // PAGE] * PAGE + t % PAGE for b in range(w.B)]).astype(np.int32)


def step_slots(w: Workload, bt: np.ndarray, step: int) -> np.ndarray:
    """slot of the token appended at decode step `step` for each sequence: [B] int32."""
    pos = w.T + step
    return (bt[:, pos // PAGE] * PAGE + pos % PAGE).astype(np.int32)


def flat_slots(n_tokens: int, perm_seed: int | None = None) -> np.ndarray:
    """Slots for a flat token axis (prefill80): page-aligned, blocks optionally permuted."""
    nb = (n_tokens + PAGE - 1) // PAGE
    blocks = np.arange(nb, dtype=np.int64)
    if perm_seed is not None:
        blocks = np.random.default_rng([perm_seed, 29]).permutation(nb)
    t = np.arange(n_tokens)
    return (blocks[t // PAGE] * PAGE + t % PAGE).astype(np.int32)
