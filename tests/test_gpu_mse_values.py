"""GPU parity of TurboQuant-MSE values (3-bit Lloyd-Max cells of the rotated
unit value plus an fp16 norm; "03. Results & Benchmarks", "At a Glance ->
Compression" and "Live Generation"), called through the C ABI.

* Quantize-append (SIMT kernel, bf16 and fp32 inputs, ragged appends): key
  records as for group-quantized values; value cells bit-exact outside the
  1e-6 band of the values' boundaries (band count <= 1e-4), value norms
  within 1e-3 relative.
* Decode over an oracle-packed cache (accumulated in the rotated space,
  rotated back in the combine step): outputs within 1e-3 relative per row,
  ragged lengths and GQA 1/4/6; with a recent-token window; chunked prefill.
* Dequantize: v_hat = ||v|| Pi^T c[cell].
"""

import dataclasses

import numpy as np
import pytest
import torch

from kv_cache_quantization_turboquantprod_b200 import tq, workloads
from oracle import attention, layout, quant

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
    glayer = pu.gpu_layer(pi32, s32, wl.key_bits, wl.value_bits, value_mode="mse")
    olayer = pu.OracleLayer(pi32, s32, wl.key_bits, wl.value_bits, value_mode="mse")
    spec = layout.CacheSpec(wl.batch, wl.h_kv, wl.capacity, wl.d, wl.key_bits,
                            wl.value_bits, wl.group, value_mode="mse")
    return glayer, olayer, spec


def _oracle_cache(wl, olayer, spec, lengths):
    buf = spec.empty()
    encs = []
    for b in range(wl.batch):
        n = lengths[b]
        if n == 0:
            encs.append(([], []))
            continue
        k, v = workloads.kv_tokens(wl, b, 0, n)
        kes, ves = pu.oracle_records_for(olayer, k.float().numpy(), v.float().numpy())
        for h in range(wl.h_kv):
            spec.write_sequence(buf, b, h, 0, kes[h], ves[h])
        encs.append((kes, ves))
    return buf, encs


@pytest.mark.parametrize("name,vb,chunks", [
    ("qwen15b_512", 3, [(0, 512)]),
    ("qwen15b_512", 3, [(0, 100), (100, 101), (101, 512)]),
    ("qwen15b_512", 2, [(0, 512)]),
    ("tiny", 3, [(0, 256)]),          # fp32 inputs
])
def test_mse_quantize_append_parity(name, vb, chunks):
    wl = dataclasses.replace(workloads.by_name(name), value_bits=vb, name=f"mse_{name}_{vb}")
    glayer, olayer, spec = _setup(wl)
    cache = tq.CompressedCache(glayer, wl.batch, wl.h_kv, wl.capacity)
    assert glayer.record_bytes() == layout.record_bytes(128, wl.key_bits, vb, 32, "mse")
    n = wl.lengths[0]
    k, v = workloads.kv_tokens(wl, 0, 0, n)
    kd, vd = k.to(DEV), v.to(DEV)
    lens = [0]
    for t0, t1 in chunks:
        tq.tq_quantize_append(glayer, cache, kd[None, t0:t1].contiguous(), vd[None, t0:t1].contiguous(), lens)
        lens = [lens[0] + t1 - t0]
    torch.cuda.synchronize()
    buf = cache.buffer.cpu().numpy()
    kf, vf = k.float().numpy(), v.float().numpy()
    stats = None
    for h in range(wl.h_kv):
        ke, ve = olayer.encode(kf[:, h], vf[:, h])
        stats = pu.compare_records(spec, buf, 0, h, 0, ke, ve, stats, olayer, kf[:, h])
    pu.check_band_fraction(stats)
    print(name, vb, chunks, stats)


@pytest.mark.parametrize("h_kv,h_q,lengths", [
    (2, 12, (4096, 512)),             # the Qwen-shaped layer, GQA 6
    (2, 8, (1, 127, 129, 300, 0)),     # GQA 4, ragged, an empty sequence
    (2, 2, (700, 256)),                # GQA 1
])
def test_mse_decode_parity(h_kv, h_q, lengths):
    wl = dataclasses.replace(workloads.qwen15b(4096), batch=len(lengths), h_kv=h_kv, h_q=h_q,
                             lengths=lengths, capacity=4096, name=f"mse_dec_{h_kv}_{h_q}")
    glayer, olayer, spec = _setup(wl)
    buf, encs = _oracle_cache(wl, olayer, spec, lengths)
    cache = tq.CompressedCache(glayer, wl.batch, wl.h_kv, wl.capacity)
    cache.buffer.copy_(torch.from_numpy(buf))
    q = workloads.queries(wl, 0)
    len_dev = torch.tensor(lengths, dtype=torch.int32, device=DEV)
    ml = max(lengths)
    ws = tq.workspace_for(glayer, cache, h_q, ml)
    out = torch.empty((wl.batch, h_q, 128), dtype=torch.float32, device=DEV)
    tq.tq_decode_attention(glayer, cache, q.to(DEV).contiguous(), len_dev, ml, out, ws)
    torch.cuda.synchronize()
    got = out.cpu().numpy()
    for b in range(wl.batch):
        if lengths[b] == 0:
            assert np.all(got[b] == 0.0)
            continue
        kes, ves = encs[b]
        ref = pu.oracle_decode(olayer, q[b].float().numpy(), kes, ves, lengths[b])
        assert pu.row_rel_err(got[b], ref) <= pu.REL_TOL, b


def test_mse_decode_with_window_and_prefill():
    lengths = (0, 129, 300)
    wlens = (5, 128, 64)
    wl = dataclasses.replace(workloads.qwen15b(512), batch=3, lengths=lengths, capacity=384,
                             name="mse_win")
    glayer, olayer, spec = _setup(wl)
    buf, encs = _oracle_cache(wl, olayer, spec, lengths)
    cache = tq.CompressedCache(glayer, wl.batch, wl.h_kv, wl.capacity)
    cache.buffer.copy_(torch.from_numpy(buf))
    wk = torch.zeros((3, wl.h_kv, 128, 128), dtype=torch.bfloat16)
    wv = torch.zeros_like(wk)
    for b in range(3):
        k, v = workloads.kv_tokens(wl, b, lengths[b], lengths[b] + wlens[b])
        wk[b, :, :wlens[b]] = k.transpose(0, 1)
        wv[b, :, :wlens[b]] = v.transpose(0, 1)
    q = workloads.queries(wl, 0)
    len_dev = torch.tensor(lengths, dtype=torch.int32, device=DEV)
    wlen_dev = torch.tensor(wlens, dtype=torch.int32, device=DEV)
    ws = tq.workspace_for(glayer, cache, wl.h_q, max(lengths))
    out = torch.empty((3, wl.h_q, 128), device=DEV)
    tq.tq_decode_attention_window(glayer, cache, q.to(DEV).contiguous(), len_dev, max(lengths),
                                  wk.to(DEV).contiguous(), wv.to(DEV).contiguous(), wlen_dev, out, ws)
    torch.cuda.synchronize()
    got = out.cpu().numpy()
    for b in range(3):
        n, w = lengths[b], wlens[b]
        rec = None
        if n:
            kes, ves = encs[b]
            rec = attention.stack_heads([pu.logical(ke, ve) for ke, ve in zip(kes, ves)])
        ref = attention.decode_with_window(q[b].float().numpy(), rec,
                                           wk[b, :, :w].transpose(0, 1).float().numpy(),
                                           wv[b, :, :w].transpose(0, 1).float().numpy(),
                                           olayer.pi, olayer.s, olayer.cent, 32,
                                           value_centroids=olayer.vcent)
        assert pu.row_rel_err(got[b], ref) <= pu.REL_TOL, b
    # chunked prefill of the last 3 tokens of sequences 1 and 2
    t_chunk = 3
    g = torch.Generator().manual_seed(8)
    qp = torch.randn((3, t_chunk, wl.h_q, 128), generator=g).to(torch.bfloat16)
    lp = (3, 129, 300)
    len_dev = torch.tensor(lp, dtype=torch.int32, device=DEV)
    cache2 = tq.CompressedCache(glayer, 3, wl.h_kv, wl.capacity)
    buf2, encs2 = _oracle_cache(wl, olayer, spec, lp)
    cache2.buffer.copy_(torch.from_numpy(buf2))
    wsp = tq.prefill_workspace_for(glayer, cache2, wl.h_q, t_chunk, max(lp))
    outp = torch.empty((3, t_chunk, wl.h_q, 128), dtype=torch.float32, device=DEV)
    tq.tq_prefill_attention(glayer, cache2, qp.to(DEV).contiguous(), len_dev, max(lp), outp, wsp)
    torch.cuda.synchronize()
    gotp = outp.cpu().numpy()
    for b in range(3):
        kes, ves = encs2[b]
        rec = attention.stack_heads([pu.logical(ke, ve) for ke, ve in zip(kes, ves)])
        ref = attention.prefill_one_sequence(qp[b].float().numpy(), rec, olayer.pi, olayer.s,
                                             olayer.cent, 32, value_centroids=olayer.vcent)
        assert pu.row_rel_err(gotp[b], ref) <= pu.REL_TOL, b


def test_mse_dequantize_parity():
    wl = dataclasses.replace(workloads.qwen15b(512), name="mse_deq")
    glayer, olayer, spec = _setup(wl)
    buf, encs = _oracle_cache(wl, olayer, spec, wl.lengths)
    cache = tq.CompressedCache(glayer, 1, wl.h_kv, wl.capacity)
    cache.buffer.copy_(torch.from_numpy(buf))
    start, count = 37, 150
    ko = torch.empty((count, wl.h_kv, 128), device=DEV)
    vo = torch.empty_like(ko)
    tq.tq_dequantize(glayer, cache, 0, start, count, ko, vo)
    torch.cuda.synchronize()
    kes, ves = encs[0]
    for h in range(wl.h_kv):
        sl = slice(start, start + count)
        vref = quant.dequantize_values_mse(ves[h]["vidx"][sl], ves[h]["nv16"][sl], olayer.pi, olayer.vcent)
        assert pu.row_rel_err(vo[:, h].cpu().numpy(), vref) <= 1e-5
