"""Seeded synthetic decode-step inputs shared by the oracle and the CUDA path.

This module only draws random numbers and lays them out; it contains none of
the method's arithmetic (no scoring, softmax, voting, selection or attention).
Both sides of every parity test consume the exact bf16 bits produced here.

Workloads (shapes follow the attention layers of the models the TokenSelect
README evaluates -- Qwen2-7B-Instruct and Llama-3-8B -- and its 1M-token
context length):

  tiny         B=1,  h_q=4,  h_kv=2, d=64,  n=4096;     K,V ~ N(0,1); 16 planted keys;
               k=256, sink 4, local 64; no selection cache
  qwen7b_32k   B=1,  h_q=28, h_kv=4, d=128, n=32768;    K ~ N(0,1) * lognormal(0,0.5)
               per-channel scale; V ~ N(0,1); 1% planted; k=2048, 4, 512
  llama8b_b4   B=4,  h_q=32, h_kv=8, d=128, n=131072;   K,V ~ N(0,1); 64 AR(1)
               queries (rho 0.95); k=2048, 4, 512; selection cache theta 0.9
  ragged_b32   B=32, h_q=32, h_kv=8, d=128, n_b ~ U[8192, 65536]; K,V ~ N(0,1);
               0.5% planted; k=1024, 4, 256
  qwen7b_1m    B=1,  h_q=28, h_kv=4, d=128, n=1048576, 28 layers; lognormal K
               scales; 0.1% planted (aligned to each layer's first query);
               k=4096, 4, 1024; selection cache theta 0.9 over 16 AR(1) queries

A planted ("needle") key for kv head g is 3 * qbar_g / |qbar_g| * sqrt(d) plus
N(0, 0.1) noise, where qbar_g is the mean of g's query heads (float64 from the
bf16 query); planted keys carry no channel scale.
"""
from __future__ import annotations

import dataclasses
import hashlib
import math

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Config:
    name: str
    batch: int
    h_q: int
    h_kv: int
    head_dim: int
    n: int                      # tokens per sequence (fixed n) or max of the ragged range
    k: int
    n_sink: int
    n_local: int
    n_min: int = 0              # ragged: n_b ~ U[n_min, n] inclusive; 0 = fixed n
    layers: int = 1
    steps: int = 1              # decode queries per layer
    theta: float | None = None  # selection-cache threshold (None = no cache)
    ar_rho: float | None = None  # AR(1) queries when set
    k_lognormal_sigma: float = 0.0
    planted_frac: float = 0.0
    planted_count: int = 0      # fixed planted count (overrides planted_frac)
    seed: int = 0

    @property
    def group(self) -> int:
        return self.h_q // self.h_kv

    @property
    def capacity(self) -> int:
        return self.k + self.n_sink + self.n_local


CONFIGS = {
    "tiny": Config("tiny", 1, 4, 2, 64, 4096, 256, 4, 64,
                   planted_count=16, seed=101),
    "qwen7b_32k": Config("qwen7b_32k", 1, 28, 4, 128, 32768, 2048, 4, 512,
                         k_lognormal_sigma=0.5, planted_frac=0.01, seed=202),
    "llama8b_b4": Config("llama8b_b4", 4, 32, 8, 128, 131072, 2048, 4, 512,
                         steps=64, theta=0.9, ar_rho=0.95, seed=303),
    "ragged_b32": Config("ragged_b32", 32, 32, 8, 128, 65536, 1024, 4, 256,
                         n_min=8192, planted_frac=0.005, seed=404),
    "qwen7b_1m": Config("qwen7b_1m", 1, 28, 4, 128, 1048576, 4096, 4, 1024,
                        layers=28, steps=16, theta=0.9, ar_rho=0.95,
                        k_lognormal_sigma=0.5, planted_frac=0.001, seed=505),
}
ORDER = ["tiny", "qwen7b_32k", "llama8b_b4", "ragged_b32", "qwen7b_1m"]


def subseed(*tags) -> int:
    """Deterministic 63-bit seed from a tuple of tags (config seed, layer, ...)."""
    h = hashlib.sha256(repr(tags).encode()).digest()
    return int.from_bytes(h[:8], "little") & ((1 << 63) - 1)


def _gen(device, *tags) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(subseed(*tags))
    return g


def seq_lengths(cfg: Config) -> np.ndarray:
    if cfg.n_min:
        rng = np.random.default_rng(subseed(cfg.seed, "lengths"))
        return rng.integers(cfg.n_min, cfg.n + 1, size=cfg.batch).astype(np.int64)
    return np.full(cfg.batch, cfg.n, np.int64)


def seq_offsets(lengths) -> np.ndarray:
    off = np.zeros(len(lengths) + 1, np.int64)
    off[1:] = np.cumsum(np.asarray(lengths, np.int64))
    return off


def queries(cfg: Config, layer: int = 0) -> torch.Tensor:
    """Decode queries [steps, B, h_q, d] bf16 (CPU).

    AR(1) when cfg.ar_rho is set: q_0 = e_0, q_t = rho*q_{t-1} + e_t with unit
    normal innovations per element, kept in float64 and rounded to bf16 per
    step; otherwise independent N(0,1)."""
    rng = np.random.default_rng(subseed(cfg.seed, "q", layer))
    shape = (cfg.batch, cfg.h_q, cfg.head_dim)
    out = np.empty((cfg.steps,) + shape, np.float64)
    state = np.zeros(shape, np.float64)
    for t in range(cfg.steps):
        e = rng.standard_normal(shape)
        if cfg.ar_rho is not None:
            state = (cfg.ar_rho * state + e) if t else e
        else:
            state = e
        out[t] = state
    return torch.from_numpy(out).to(torch.bfloat16)


def _planted_count(cfg: Config, n: int) -> int:
    if cfg.planted_count:
        return min(cfg.planted_count, n)
    return int(math.floor(cfg.planted_frac * n))


def planted_keys(cfg: Config, q0: torch.Tensor, count: int, tags) -> torch.Tensor:
    """[count, h_kv, d] bf16 planted keys aligned to query q0 [h_q, d] (CPU)."""
    d, G = cfg.head_dim, cfg.group
    qd = q0.to(torch.float64).reshape(cfg.h_kv, G, d).mean(dim=1)       # qbar_g
    unit = qd / qd.norm(dim=1, keepdim=True)
    rng = np.random.default_rng(subseed(*tags, "planted-noise"))
    noise = torch.from_numpy(rng.normal(0.0, 0.1, size=(count, cfg.h_kv, d)))
    return (3.0 * math.sqrt(d) * unit.unsqueeze(0) + noise).to(torch.bfloat16)


@dataclasses.dataclass
class LayerInputs:
    k: torch.Tensor            # [sum_n, h_kv, d] bf16 (device)
    v: torch.Tensor            # [sum_n, h_kv, d] bf16 (device)
    seq_offsets: np.ndarray    # [B+1] int64
    q: torch.Tensor            # [steps, B, h_q, d] bf16 (CPU)
    planted: list              # per sequence: int64 array of planted positions


def layer_inputs(cfg: Config, layer: int = 0, device="cpu", *, n_override=None,
                 chunk_tokens: int = 1 << 18) -> LayerInputs:
    """All inputs of one layer.  n_override replaces every sequence length
    (small parity cases that keep the workload's structure)."""
    lengths = seq_lengths(cfg) if n_override is None else np.full(cfg.batch, n_override, np.int64)
    off = seq_offsets(lengths)
    total = int(off[-1])
    d, hk = cfg.head_dim, cfg.h_kv
    q = queries(cfg, layer)
    k = torch.empty((total, hk, d), dtype=torch.bfloat16, device=device)
    v = torch.empty((total, hk, d), dtype=torch.bfloat16, device=device)
    scale = None
    if cfg.k_lognormal_sigma > 0:
        sg = _gen("cpu", cfg.seed, "kscale", layer)
        scale = torch.exp(torch.randn((hk, d), generator=sg, dtype=torch.float32)
                          * cfg.k_lognormal_sigma).to(device)
    gk = _gen(device, cfg.seed, "K", layer)
    gv = _gen(device, cfg.seed, "V", layer)
    for a in range(0, total, chunk_tokens):
        b = min(total, a + chunk_tokens)
        kk = torch.randn((b - a, hk, d), generator=gk, device=device, dtype=torch.float32)
        if scale is not None:
            kk.mul_(scale)
        k[a:b].copy_(kk)
        v[a:b].copy_(torch.randn((b - a, hk, d), generator=gv, device=device, dtype=torch.float32))
        del kk
    planted = []
    for bi in range(cfg.batch):
        n_b = int(lengths[bi])
        cnt = _planted_count(cfg, n_b)
        if cnt == 0:
            planted.append(np.zeros(0, np.int64))
            continue
        rng = np.random.default_rng(subseed(cfg.seed, "planted-pos", layer, bi))
        pos = np.sort(rng.choice(n_b, size=cnt, replace=False)).astype(np.int64)
        keys = planted_keys(cfg, q[0, bi], cnt, (cfg.seed, layer, bi))
        idx = torch.from_numpy(pos + off[bi]).to(device)
        k[idx] = keys.to(device)
        planted.append(pos)
    return LayerInputs(k, v, off, q, planted)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """Host uint16 array of a bf16 tensor's bits, with the tensor's strides.

    Strided (padded) device tensors are copied with their whole underlying
    span, so the host array has the same element strides as the device one."""
    t = t.detach()
    if t.is_contiguous():
        return t.to("cpu").view(torch.int16).numpy().view(np.uint16)
    span = 1 + sum((s - 1) * st for s, st in zip(t.shape, t.stride()))
    base = torch.as_strided(t, (span,), (1,), t.storage_offset()).to("cpu")
    arr = base.view(torch.int16).numpy().view(np.uint16)
    return np.lib.stride_tricks.as_strided(
        arr, shape=tuple(t.shape), strides=tuple(2 * s for s in t.stride()))


def random_kv(n: int, h_kv: int, d: int, seed: int, device="cpu", *, dist="normal",
              stride_tok: int | None = None, stride_head: int | None = None):
    """Small ad-hoc K/V pair for edge-case tests.

    dist: "normal" (N(0,1)), "const" (every element 1.0), "int" (small
    integers in [-3, 3]).  A padded layout (stride_tok / stride_head larger than
    the dense ones, in elements) is built as a view into a larger buffer whose
    gaps hold large junk values, so that a wrong stride reads junk."""
    st = stride_tok if stride_tok is not None else h_kv * d
    sh = stride_head if stride_head is not None else d
    assert sh >= d and st >= (h_kv - 1) * sh + d
    g = _gen("cpu", seed, "kv", n, h_kv, d, dist)

    def one():
        if dist == "normal":
            x = torch.randn((n, h_kv, d), generator=g)
        elif dist == "const":
            x = torch.ones((n, h_kv, d))
        elif dist == "int":
            x = torch.randint(-3, 4, (n, h_kv, d), generator=g).float()
        else:
            raise ValueError(dist)
        buf = torch.full((max(n, 1) * st + 8,), 1.0e4, dtype=torch.bfloat16)
        view = buf.as_strided((n, h_kv, d), (st, sh, 1))
        view.copy_(x.to(torch.bfloat16))
        if device != "cpu":
            view = buf.to(device).as_strided((n, h_kv, d), (st, sh, 1))
        return view
    return one(), one()
