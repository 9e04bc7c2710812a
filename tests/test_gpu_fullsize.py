"""GPU parity at the full sizes and launch plans the benchmark runs.

* Quantize-append in its steady state: one 8192-token chunk of the long-context
  workload (4 sequences x 8 heads, 4-bit keys: 2048 tiles, about 14 per
  persistent CTA) with every record compared against the oracle, and one
  8192-token chunk of the batched workload (32 sequences, 3-bit keys) on 16
  (sequence, head) pairs spread over the CTAs.
* Decode at the batched workload's own split plan (32 sequences, ragged
  16K-32K contexts: two splits of 128 tiles per (sequence, head)), with
  sequences whose second split is empty, holds one token, or is full; the
  oracle decodes the library's own records of sampled (sequence, head) pairs.
* Decode of the long-context workload at 131,072 tokens on sampled heads of
  two sequences.
Bars as elsewhere: codes, signs and value codes exact outside the bands (band
fraction <= 1e-4), norms and outputs within 1e-3 relative per row.
"""

import numpy as np
import pytest
import torch

from kv_cache_quantization_turboquantprod_b200 import tq, workloads
from oracle import layout

import parity_util as pu

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _built():
    from kv_cache_quantization_turboquantprod_b200 import build
    build.build()
    tq.load()


def _setup(wl):
    _, pi32, s32 = workloads.layer_matrices(wl)
    glayer = pu.gpu_layer(pi32, s32, wl.key_bits, wl.value_bits)
    olayer = pu.OracleLayer(pi32, s32, wl.key_bits, wl.value_bits)
    spec = layout.CacheSpec(wl.batch, wl.h_kv, wl.capacity, wl.d, wl.key_bits,
                            wl.value_bits, wl.group)
    return glayer, olayer, spec


def _chunk_parity(wl, pairs):
    """Append chunk 0 (8192 tokens) of every sequence in one call; compare the
    records of the given (b, h) pairs with the oracle."""
    n = workloads.TOKEN_CHUNK
    wl = workloads.scaled(wl, lengths=(n,) * wl.batch, capacity=n)
    glayer, olayer, spec = _setup(wl)
    cache = tq.CompressedCache(glayer, wl.batch, wl.h_kv, n)
    kv = [workloads.kv_chunk(wl, b, 0, DEV) for b in range(wl.batch)]
    k = torch.stack([x[0] for x in kv]).contiguous()
    v = torch.stack([x[1] for x in kv]).contiguous()
    tq.tq_quantize_append(glayer, cache, k, v, [0] * wl.batch)
    torch.cuda.synchronize()
    buf = cache.buffer.cpu().numpy()
    stats = None
    for b, h in pairs:
        kk = k[b, :, h].float().cpu().numpy()
        vv = v[b, :, h].float().cpu().numpy()
        ke, ve = olayer.encode(kk, vv)
        stats = pu.compare_records(spec, buf, b, h, 0, ke, ve, stats, olayer, kk)
    pu.check_band_fraction(stats)
    return stats


def test_quantize_steady_state_longctx_chunk_every_record():
    wl = workloads.longctx()
    pairs = [(b, h) for b in range(wl.batch) for h in range(wl.h_kv)]
    stats = _chunk_parity(wl, pairs)
    assert stats["coords"] == wl.batch * wl.h_kv * workloads.TOKEN_CHUNK * wl.d
    print("longctx chunk", stats)


def test_quantize_steady_state_batched_chunk_sampled():
    wl = workloads.batched()
    rng = np.random.default_rng(21)
    pairs = sorted({(int(b), int(h)) for b, h in zip(rng.integers(0, 32, 40), rng.integers(0, 8, 40))})[:16]
    stats = _chunk_parity(wl, pairs)
    print("batched chunk", stats)


def test_decode_at_the_benchmark_split_plan():
    wl = workloads.batched()
    lengths = list(wl.lengths)
    # second split (tokens 16384 ..) empty, one token, and a tile short of full
    lengths[3], lengths[7], lengths[11] = 16384, 16000, 16385
    lengths[20] = wl.capacity
    glayer, olayer, spec = _setup(wl)
    cache = tq.CompressedCache(glayer, wl.batch, wl.h_kv, wl.capacity)
    pu.fill_cache_gpu(glayer, cache, wl, lengths)
    max_len = max(lengths)
    ntile = (max_len + 127) // 128
    assert ntile == 256     # the plan: 256 (b, h) units, two splits of 128 tiles each
    q = workloads.queries(wl, 0, device=DEV)
    len_dev = torch.tensor(lengths, dtype=torch.int32, device=DEV)
    ws = tq.workspace_for(glayer, cache, wl.h_q, max_len)
    out = torch.empty((wl.batch, wl.h_q, wl.d), dtype=torch.float32, device=DEV)
    tq.tq_decode_attention(glayer, cache, q, len_dev, max_len, out, ws)
    torch.cuda.synchronize()
    assert tq.decode_status(ws) == 0
    got = out.cpu().numpy()
    buf = cache.buffer.cpu().numpy()
    qf = q.float().cpu().numpy()
    G = wl.gqa
    worst = 0.0
    for b, h in [(3, 0), (7, 5), (11, 2), (20, 7), (0, 1), (31, 4), (16, 3), (25, 6)]:
        ref = pu.oracle_decode_head(olayer, spec, buf, b, h, lengths[b], qf[b, h * G:(h + 1) * G])
        err = pu.row_rel_err(got[b, h * G:(h + 1) * G], ref)
        worst = max(worst, err)
        assert err <= pu.REL_TOL, (b, h, err)
    print("batched plan decode max row rel err", worst)


def test_decode_longctx_131072():
    wl = workloads.longctx()
    glayer, olayer, spec = _setup(wl)
    cache = tq.CompressedCache(glayer, wl.batch, wl.h_kv, wl.capacity)
    lengths = list(wl.lengths)
    pu.fill_cache_gpu(glayer, cache, wl, lengths)
    q = workloads.queries(wl, 0, device=DEV)
    len_dev = torch.tensor(lengths, dtype=torch.int32, device=DEV)
    ws = tq.workspace_for(glayer, cache, wl.h_q, wl.capacity)
    out = torch.empty((wl.batch, wl.h_q, wl.d), dtype=torch.float32, device=DEV)
    tq.tq_decode_attention(glayer, cache, q, len_dev, wl.capacity, out, ws)
    torch.cuda.synchronize()
    assert tq.decode_status(ws) == 0
    got = out.cpu().numpy()
    buf = cache.buffer.cpu().numpy()
    qf = q.float().cpu().numpy()
    G = wl.gqa
    for b, h in [(0, 0), (0, 5), (3, 2), (3, 7)]:
        ref = pu.oracle_decode_head(olayer, spec, buf, b, h, lengths[b], qf[b, h * G:(h + 1) * G])
        assert pu.row_rel_err(got[b, h * G:(h + 1) * G], ref) <= pu.REL_TOL, (b, h)
