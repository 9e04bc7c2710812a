"""Seeded synthetic workloads for the compressed-KV hot path.

This module only draws random numbers and names shapes.  It holds none of the
method's arithmetic: no normalisation, rotation, bucketization, packing or
attention.  Both the CUDA path's harness (tests, bench) and the CPU oracle take
their inputs from here, and from nowhere else.

Random quantities the method itself draws (the rotation Pi and the QJL matrix
S) are produced here too and handed to both sides as plain data, as the pages
describe them: a fixed, seeded, data-oblivious random orthogonal rotation and
an i.i.d. Gaussian d x d sketch matrix ("turboquant/audit_claims.py", AUDIT 1:
Pi and S are each D*D fp32 per layer; TurboQuant explainer (troisinh.com),
"Ý tưởng cốt lõi": a fixed random rotation, Johnson-Lindenstrauss style).

Workload shapes follow the pages' models: a Llama-3-8B-shaped layer
(H_kv=8, H_q=32), a Qwen2.5-1.5B-shaped layer (H_kv=2, H_q=12, the model of
"03. Results & Benchmarks", turboquant_cutile) and batched / long-context
variants.  There are no model weights in this build, so K, V and q are
synthetic tensors with those head shapes.
"""

from __future__ import annotations

import dataclasses
import zlib

import numpy as np
import torch

TOKEN_CHUNK = 8192  # K/V are drawn per (sequence, 8192-token chunk)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    h_kv: int
    h_q: int
    d: int
    key_bits: int      # total key bits: (key_bits - 1) Lloyd-Max bits + 1 QJL bit
    value_bits: int
    group: int
    capacity: int      # tokens per sequence the cache holds
    lengths: tuple     # cached tokens per sequence at decode time
    kv_dtype: str      # "f32" or "bf16"
    channel_scale: str  # "lognormal0.5" | "unit" | "lognormal1"
    outliers: int      # outlier channels per head (scaled x20)
    seed: int
    n_queries: int = 1  # decode calls per workload (tiny case runs 4)

    @property
    def gqa(self) -> int:
        return self.h_q // self.h_kv

    @property
    def mse_bits(self) -> int:
        return self.key_bits - 1


def _round_up(x: int, m: int) -> int:
    return (x + m - 1) // m * m


def _ragged_lengths(batch: int, lo: int, hi: int, seed: int) -> tuple:
    rng = np.random.default_rng(seed * 7919 + 17)
    return tuple(int(x) for x in rng.integers(lo, hi + 1, size=batch))


def tiny() -> Workload:
    """One layer, batch 1, H_kv=2, H_q=2, N=256; fp32 K/V with per-channel
    lognormal(0.5) scales; 2+1-bit keys, 2-bit values; 4 queries; seed 0."""
    return Workload("tiny", 1, 2, 2, 128, 3, 2, 32, 256, (256,), "f32",
                    "lognormal0.5", 0, 0, n_queries=4)


def llama8b() -> Workload:
    """Llama-3-8B-shaped layer: batch 1, H_kv=8, H_q=32, N=4096, bf16 K/V
    ~N(0,1) with 4 outlier channels per head scaled x20; seed 1."""
    return Workload("llama8b", 1, 8, 32, 128, 3, 2, 32, 4096, (4096,), "bf16",
                    "unit", 4, 1)


def qwen15b(n: int = 16384) -> Workload:
    """Qwen2.5-1.5B-shaped layer: batch 1, H_kv=2, H_q=12, bf16 K/V with
    lognormal(1) channel scales; 3-bit keys (2+1) and 3-bit values; seed 2."""
    return Workload(f"qwen15b_{n}", 1, 2, 12, 128, 3, 3, 32, _round_up(n, 128),
                    (n,), "bf16", "lognormal1", 0, 2)


QWEN_SWEEP = (512, 1024, 2048, 4096, 8192, 16384)


def batched() -> Workload:
    """Batched decode: batch 32, H_kv=8, H_q=32, capacity 32768, ragged
    lengths uniform in [16384, 32768]; lognormal(1) channel scales plus
    round(0.02*128)=3 outlier channels x20 per head; seed 3."""
    return Workload("batched", 32, 8, 32, 128, 3, 2, 32, 32768,
                    _ragged_lengths(32, 16384, 32768, 3), "bf16",
                    "lognormal1", 3, 3)


def longctx() -> Workload:
    """Long context: batch 4, H_kv=8, H_q=32, 131072 tokens appended in
    8192-token bf16 chunks; 3+1-bit keys, 2-bit values; seed 4."""
    return Workload("longctx", 4, 8, 32, 128, 4, 2, 32, 131072,
                    (131072,) * 4, "bf16", "lognormal1", 3, 4)


def by_name(name: str) -> Workload:
    if name.startswith("qwen15b"):
        n = int(name.split("_")[1]) if "_" in name else 16384
        return qwen15b(n)
    return {"tiny": tiny, "llama8b": llama8b, "batched": batched,
            "longctx": longctx}[name]()


def scaled(wl: Workload, batch: int | None = None, lengths: tuple | None = None,
           capacity: int | None = None, name: str | None = None) -> Workload:
    """Same distribution, smaller shape (for parity cases the oracle can finish)."""
    b = batch if batch is not None else wl.batch
    ls = lengths if lengths is not None else wl.lengths[:b]
    cap = capacity if capacity is not None else _round_up(max(ls), 128)
    return dataclasses.replace(wl, batch=b, lengths=tuple(ls), capacity=cap,
                               name=name or wl.name + "_scaled")


# ---------------------------------------------------------------------------
# Random matrices the method draws (passed to both sides as data)
# ---------------------------------------------------------------------------

def rotation_and_sketch(d: int, seed: int):
    """Haar-random orthogonal Pi (float64) and Gaussian S (float64 holding
    float32-representable values), drawn from numpy's default_rng(seed).

    Pi = Q * diag(sign(diag(R))) for the QR factorisation of a standard
    Gaussian d x d matrix, which is Haar-distributed.  S has i.i.d. N(0,1)
    entries, rounded to float32 so that the GPU copy is exact.
    """
    rng = np.random.default_rng(seed)
    g = rng.standard_normal((d, d))
    q, r = np.linalg.qr(g)
    pi = q * np.sign(np.diag(r))[None, :]
    s = rng.standard_normal((d, d)).astype(np.float32).astype(np.float64)
    return pi, s


def layer_matrices(wl: Workload):
    """(Pi64, Pi32, S) for the workload's layer; Pi32 is what both the GPU and
    the parity oracle consume (the oracle upcasts it to float64)."""
    pi, s = rotation_and_sketch(wl.d, 1000 + wl.seed)
    return pi, pi.astype(np.float32), s.astype(np.float32)


# ---------------------------------------------------------------------------
# K / V / q draws
# ---------------------------------------------------------------------------

def _channel_scales(wl: Workload, which: str) -> np.ndarray:
    """Per (kv-head, channel) multiplicative scales, float32 [H_kv, d]."""
    tag = zlib.crc32(which.encode()) & 0xFFFF
    rng = np.random.default_rng(wl.seed * 65537 + tag)
    if wl.channel_scale == "unit":
        c = np.ones((wl.h_kv, wl.d))
    elif wl.channel_scale == "lognormal0.5":
        c = np.exp(0.5 * rng.standard_normal((wl.h_kv, wl.d)))
    elif wl.channel_scale == "lognormal1":
        c = np.exp(1.0 * rng.standard_normal((wl.h_kv, wl.d)))
    else:
        raise ValueError(wl.channel_scale)
    for h in range(wl.h_kv):
        if wl.outliers:
            idx = rng.choice(wl.d, size=wl.outliers, replace=False)
            c[h, idx] *= 20.0
    return c.astype(np.float32)


def _torch_dtype(name: str):
    return {"f32": torch.float32, "bf16": torch.bfloat16}[name]


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) & 0x7FFFFFFFFFFFFFFF)
    return g


def kv_chunk(wl: Workload, b: int, chunk: int, device="cpu"):
    """K and V for sequence b, tokens [chunk*8192, (chunk+1)*8192): each
    [8192, H_kv, d] in the workload's dtype.  Values depend on the device the
    generator runs on (CPU and CUDA Philox streams differ); harnesses that
    compare against the oracle copy the same tensor to the host."""
    device = torch.device(device)
    t = min(TOKEN_CHUNK, wl.capacity)
    out = []
    for which in ("k", "v"):
        scale = torch.from_numpy(_channel_scales(wl, which)).to(device)
        seed = wl.seed * 1_000_003 + b * 4099 + chunk * 131 + (0 if which == "k" else 7)
        x = torch.randn((t, wl.h_kv, wl.d), generator=_gen(device, seed),
                        device=device, dtype=torch.float32)
        x = x * scale[None]
        out.append(x.to(_torch_dtype(wl.kv_dtype)))
    return out[0], out[1]


def kv_tokens(wl: Workload, b: int, t0: int, t1: int, device="cpu"):
    """K, V for sequence b, tokens [t0, t1): [t1 - t0, H_kv, d] each."""
    ks, vs = [], []
    c0, c1 = t0 // TOKEN_CHUNK, (t1 - 1) // TOKEN_CHUNK
    for c in range(c0, c1 + 1):
        k, v = kv_chunk(wl, b, c, device)
        lo = max(t0, c * TOKEN_CHUNK) - c * TOKEN_CHUNK
        hi = min(t1, (c + 1) * TOKEN_CHUNK) - c * TOKEN_CHUNK
        ks.append(k[lo:hi])
        vs.append(v[lo:hi])
    return torch.cat(ks, 0), torch.cat(vs, 0)


def queries(wl: Workload, call: int = 0, device="cpu"):
    """Decode queries [B, H_q, d] ~ N(0, 1) in the workload's dtype."""
    device = torch.device(device)
    seed = wl.seed * 7_777_777 + 999 + call
    q = torch.randn((wl.batch, wl.h_q, wl.d), generator=_gen(device, seed),
                    device=device, dtype=torch.float32)
    return q.to(_torch_dtype(wl.kv_dtype))
