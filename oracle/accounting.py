"""Storage accounting of the compressed cache.

Test infrastructure only (see oracle/__init__.py).

"turboquant/audit_claims.py", AUDIT 1, counts the quantized data of N tokens x
H_kv heads, then adds per-layer overhead (Pi and S, each d*d fp32, and the
codebook tensors at 4 bytes an entry) and a 128-token bf16 ring buffer of
recent tokens, and compares with an fp16 K+V cache of N*H_kv*d*2*2 bytes.

Reading for the record size: fp16 norms and fp16 scale+zero per value group
(the only layout that gives the audit's printed ratios, see
tests/test_oracle_accounting.py); codebook = centroids + decision boundaries
(a few dozen bytes, below the printed precision).

TurboQuant-MSE values ("03. Results & Benchmarks", "At a Glance ->
Compression": 3 bits per coordinate for keys and values, 1,288 KB -> 257 KB,
5.02x): 3-bit value cells plus one fp16 value norm, 102 bytes per (token,
head) at 3-bit keys, so the data-only ratio is 512 / 102.
"""

from __future__ import annotations

from .layout import record_bytes


def data_bytes(n_tokens, h_kv, d, key_bits, value_bits, group, value_mode="group") -> int:
    return n_tokens * h_kv * record_bytes(d, key_bits, value_bits, group, value_mode)


def fp16_kv_bytes(n_tokens, h_kv, d) -> int:
    return n_tokens * h_kv * d * 2 * 2


def per_layer_overhead(d, key_bits) -> int:
    levels = 2 ** (key_bits - 1)
    return 2 * d * d * 4 + levels * 4 + (levels - 1) * 4


def ring_bytes(h_kv, d, ring_tokens=128) -> int:
    return ring_tokens * h_kv * d * 2


def ratios(n_tokens, h_kv, d, key_bits, value_bits, group, value_mode="group") -> dict:
    fp16 = fp16_kv_bytes(n_tokens, h_kv, d)
    data = data_bytes(n_tokens, h_kv, d, key_bits, value_bits, group, value_mode)
    over = per_layer_overhead(d, key_bits)
    ring = ring_bytes(h_kv, d)
    return {"data_only": fp16 / data,
            "with_overhead": fp16 / (data + over),
            "all_in": fp16 / (data + over + ring)}
