"""GPU parity at head dims 64 and 256 (the SIMT kernels; the tensor-core
kernels are built for d = 128), called through the C ABI.

* Quantize-append (bf16 and fp32 inputs, ragged appends from mid-tile
  positions, a 1-token append): key codes and signs bit-exact outside the
  1e-6 bands, value codes exact outside the value band, norms within 1e-3.
* Decode over an oracle-packed cache at GQA 1 and 4, ragged lengths and an
  empty sequence, with group-quantized and TurboQuant-MSE values, and with a
  recent-token window: outputs within 1e-3 relative per row.
* Dequantize: explicit K and V reconstruction.
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


def _wl(d, **kw):
    base = dataclasses.replace(workloads.qwen15b(512), d=d, value_bits=2, name=f"d{d}")
    return dataclasses.replace(base, **kw)


def _setup(wl, value_mode="group"):
    pi, s = workloads.rotation_and_sketch(wl.d, 1000 + wl.seed)
    pi32, s32 = pi.astype(np.float32), s.astype(np.float32)
    glayer = pu.gpu_layer(pi32, s32, wl.key_bits, wl.value_bits, value_mode=value_mode)
    olayer = pu.OracleLayer(pi32, s32, wl.key_bits, wl.value_bits, value_mode=value_mode)
    spec = layout.CacheSpec(wl.batch, wl.h_kv, wl.capacity, wl.d, wl.key_bits, wl.value_bits,
                            wl.group, value_mode=value_mode)
    return glayer, olayer, spec


@pytest.mark.parametrize("d", [64, 256])
@pytest.mark.parametrize("kv_dtype,chunks,mode", [
    ("bf16", [(0, 512)], "group"),
    ("bf16", [(0, 100), (100, 101), (101, 512)], "group"),
    ("f32", [(0, 300)], "group"),
    ("bf16", [(0, 77), (77, 512)], "mse"),
])
def test_quantize_append_parity(d, kv_dtype, chunks, mode):
    wl = _wl(d, kv_dtype=kv_dtype, value_bits=3 if mode == "mse" else 2)
    glayer, olayer, spec = _setup(wl, mode)
    assert glayer.record_bytes() == layout.record_bytes(d, wl.key_bits, wl.value_bits, 32, mode)
    cache = tq.CompressedCache(glayer, 1, wl.h_kv, wl.capacity)
    n = chunks[-1][1]
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
    print(d, kv_dtype, chunks, mode, stats)


@pytest.mark.parametrize("d", [64, 256])
@pytest.mark.parametrize("h_kv,h_q,mode", [(2, 8, "group"), (2, 2, "group"), (2, 8, "mse")])
def test_decode_parity(d, h_kv, h_q, mode):
    lengths = (1, 127, 300, 0)
    wl = _wl(d, batch=4, h_kv=h_kv, h_q=h_q, lengths=lengths, capacity=384,
             value_bits=3 if mode == "mse" else 2)
    glayer, olayer, spec = _setup(wl, mode)
    buf = spec.empty()
    encs = []
    for b in range(wl.batch):
        if lengths[b] == 0:
            encs.append(None)
            continue
        k, v = workloads.kv_tokens(wl, b, 0, lengths[b])
        kes, ves = pu.oracle_records_for(olayer, k.float().numpy(), v.float().numpy())
        for h in range(h_kv):
            spec.write_sequence(buf, b, h, 0, kes[h], ves[h])
        encs.append((kes, ves))
    cache = tq.CompressedCache(glayer, wl.batch, h_kv, wl.capacity)
    cache.buffer.copy_(torch.from_numpy(buf))
    q = torch.randn((wl.batch, h_q, d), generator=torch.Generator().manual_seed(d + h_q)).to(torch.bfloat16)
    len_dev = torch.tensor(lengths, dtype=torch.int32, device=DEV)
    ml = max(lengths)
    ws = tq.workspace_for(glayer, cache, h_q, ml)
    out = torch.empty((wl.batch, h_q, d), dtype=torch.float32, device=DEV)
    tq.tq_decode_attention(glayer, cache, q.to(DEV).contiguous(), len_dev, ml, out, ws)
    # the same call with a recent-token window of 5 exact tokens per sequence
    wk = torch.randn((wl.batch, h_kv, 8, d), generator=torch.Generator().manual_seed(1)).to(torch.bfloat16)
    wv = torch.randn_like(wk.float()).to(torch.bfloat16)
    wlen = torch.full((wl.batch,), 5, dtype=torch.int32, device=DEV)
    outw = torch.empty_like(out)
    tq.tq_decode_attention_window(glayer, cache, q.to(DEV).contiguous(), len_dev, ml, wk.to(DEV), wv.to(DEV),
                                  wlen, outw, ws)
    torch.cuda.synchronize()
    got, gotw = out.cpu().numpy(), outw.cpu().numpy()
    for b in range(wl.batch):
        qb = q[b].float().numpy()
        rec = None
        if encs[b] is None:
            assert np.all(got[b] == 0.0)
        else:
            kes, ves = encs[b]
            ref = pu.oracle_decode(olayer, qb, kes, ves, lengths[b])
            assert pu.row_rel_err(got[b], ref) <= pu.REL_TOL, b
            rec = attention.stack_heads([pu.logical(ke, ve) for ke, ve in zip(kes, ves)])
        refw = attention.decode_with_window(qb, rec, wk[b, :, :5].transpose(0, 1).float().numpy(),
                                            wv[b, :, :5].transpose(0, 1).float().numpy(), olayer.pi,
                                            olayer.s, olayer.cent, 32, value_centroids=olayer.vcent)
        assert pu.row_rel_err(gotw[b], refw) <= pu.REL_TOL, b


@pytest.mark.parametrize("d", [64, 256])
def test_dequantize_parity(d):
    wl = _wl(d, lengths=(256,), capacity=256)
    glayer, olayer, spec = _setup(wl)
    k, v = workloads.kv_tokens(wl, 0, 0, 256)
    kes, ves = pu.oracle_records_for(olayer, k.float().numpy(), v.float().numpy())
    buf = spec.empty()
    for h in range(wl.h_kv):
        spec.write_sequence(buf, 0, h, 0, kes[h], ves[h])
    cache = tq.CompressedCache(glayer, 1, wl.h_kv, 256)
    cache.buffer.copy_(torch.from_numpy(buf))
    start, count = 37, 150
    ko = torch.empty((count, wl.h_kv, d), device=DEV)
    vo = torch.empty_like(ko)
    tq.tq_dequantize(glayer, cache, 0, start, count, ko, vo)
    torch.cuda.synchronize()
    sl = slice(start, start + count)
    for h in range(wl.h_kv):
        ke, ve = kes[h], ves[h]
        kref = quant.dequantize_keys(ke["idx"][sl], ke["sign"][sl], ke["nk16"][sl], ke["rn16"][sl],
                                     olayer.pi, olayer.s, olayer.cent)
        vref = quant.dequantize_values(ve["codes"][sl], ve["scale16"][sl], ve["zero16"][sl], 32)
        assert pu.row_rel_err(ko[:, h].cpu().numpy(), kref) <= 1e-5
        assert pu.row_rel_err(vo[:, h].cpu().numpy(), vref) <= 1e-6
