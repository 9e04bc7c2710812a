"""GPU parity: the CUDA path, called through the C ABI, against the oracle on
the same seeded inputs.

Quantize-append: codes and signs bit-exact outside the 1e-6 bands, value
codes and scales outside the value band (band counts <= 1e-4 of the
coordinates), zeros exact, norms within 1e-3 relative.
Decode: the oracle's own encoding is packed (by the oracle's layout writer)
into the device cache, so the CUDA decode and the oracle decode read the same
records; outputs within 1e-3 relative per (b, h_q) row.
"""

import numpy as np
import pytest
import torch

from kv_cache_quantization_turboquantprod_b200 import tq, workloads
from oracle import attention, layout

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


def _kv_cpu(wl, b, t0, t1):
    k, v = workloads.kv_tokens(wl, b, t0, t1, device="cpu")
    return k, v


def _append_all(glayer, cache, wl, chunks, device_tensors):
    """Append per-sequence token ranges [(t0, t1), ...] in calls."""
    lens = [0] * wl.batch
    for (t0, t1) in chunks:
        T = t1 - t0
        ks = torch.stack([device_tensors[b][0][t0:t1] for b in range(wl.batch)])
        vs = torch.stack([device_tensors[b][1][t0:t1] for b in range(wl.batch)])
        tq.tq_quantize_append(glayer, cache, ks.contiguous(), vs.contiguous(), lens)
        lens = [x + T for x in lens]
    torch.cuda.synchronize()
    return lens


# ---------------------------------------------------------------------------
# quantize-append parity
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("name,chunks", [
    ("tiny", [(0, 256)]),
    ("tiny", [(0, 100), (100, 101), (101, 256)]),      # ragged tails, mid-tile starts
    ("llama8b", [(0, 4096)]),
    ("llama8b", [(0, 40), (40, 1000), (1000, 4096)]),  # short append (SIMT), then tiles mid-way
])
def test_quantize_append_parity(name, chunks):
    wl = workloads.by_name(name)
    glayer, olayer, spec = _setup(wl)
    cache = tq.CompressedCache(glayer, wl.batch, wl.h_kv, wl.capacity)
    n = wl.lengths[0]
    dev = {}
    for b in range(wl.batch):
        k, v = _kv_cpu(wl, b, 0, n)
        dev[b] = (k.to(DEV), v.to(DEV))
    _append_all(glayer, cache, wl, chunks, dev)
    buf = cache.buffer.cpu().numpy()
    stats = None
    for b in range(wl.batch):
        k = pu.to_np(dev[b][0])
        v = dev[b][1].float().cpu().numpy()
        for h in range(wl.h_kv):
            ke, ve = olayer.encode(k[:, h], v[:, h])
            stats = pu.compare_records(spec, buf, b, h, 0, ke, ve, stats, olayer, k[:, h])
    pu.check_band_fraction(stats)
    print(name, chunks, stats)


def test_quantize_append_ragged_batch_and_zero_key():
    """Three sequences at different lengths, different n_new, a zero key,
    positions crossing tile boundaries."""
    wl = workloads.scaled(workloads.llama8b(), batch=3, lengths=(300, 300, 300),
                          capacity=384, name="ragged")
    glayer, olayer, spec = _setup(wl)
    cache = tq.CompressedCache(glayer, 3, wl.h_kv, 384, zero=True)
    lens0 = [0, 120, 127]
    T = 140
    nnew = [140, 9, 129]
    k = torch.empty((3, T, wl.h_kv, 128), dtype=torch.bfloat16)
    v = torch.empty_like(k)
    for b in range(3):
        kb, vb = workloads.kv_tokens(wl, b, 0, T)
        k[b], v[b] = kb, vb
    k[1, 3, 2] = 0.0          # a zero key vector
    tq.tq_quantize_append(glayer, cache, k.to(DEV), v.to(DEV), lens0, nnew)
    torch.cuda.synchronize()
    buf = cache.buffer.cpu().numpy()
    stats = None
    for b in range(3):
        kk = k[b, :nnew[b]].float().numpy()
        vv = v[b, :nnew[b]].float().numpy()
        for h in range(wl.h_kv):
            ke, ve = olayer.encode(kk[:, h], vv[:, h])
            stats = pu.compare_records(spec, buf, b, h, lens0[b], ke, ve, stats, olayer, kk[:, h])
        # slots before lens0 and after lens0 + nnew stay untouched (zeroed buffer)
        if lens0[b] > 0:
            assert not spec.read(buf, b, 0, 0, lens0[b])["nk16"].any()
        end = lens0[b] + nnew[b]
        assert not spec.read(buf, b, 0, end, 384 - end)["nk16"].any()
    pu.check_band_fraction(stats)
    zero_rec = spec.read(buf, 1, 2, lens0[1] + 3, 1)
    assert zero_rec["nk16"][0] == 0 and zero_rec["rn16"][0] == 0
    assert not zero_rec["idx"].any() and not zero_rec["sign"].any()


@pytest.mark.parametrize("kb,vb", [(2, 2), (4, 2), (3, 3), (4, 4)])
def test_quantize_append_bit_widths(kb, vb):
    import dataclasses
    wl = dataclasses.replace(workloads.tiny(), key_bits=kb, value_bits=vb, name=f"bits{kb}{vb}")
    glayer, olayer, spec = _setup(wl)
    cache = tq.CompressedCache(glayer, 1, wl.h_kv, 256)
    k, v = _kv_cpu(wl, 0, 0, 256)
    tq.tq_quantize_append(glayer, cache, k[None].to(DEV).contiguous(),
                          v[None].to(DEV).contiguous(), [0])
    torch.cuda.synchronize()
    buf = cache.buffer.cpu().numpy()
    stats = None
    for h in range(wl.h_kv):
        ke, ve = olayer.encode(k[:, h].numpy(), v[:, h].numpy())
        stats = pu.compare_records(spec, buf, 0, h, 0, ke, ve, stats, olayer, k[:, h].numpy())
    pu.check_band_fraction(stats)


@pytest.mark.parametrize("kb", [3, 4])
def test_prepared_operands_give_the_same_records(kb):
    """The tensor-core append with operand images prepared once per layer
    (tq_prepare_operands, the default of tq.Layer) writes the same bytes as
    with tc_operands = NULL (every CTA building them itself), and the
    prepared images match a second preparation; 20 tiles of bf16 keys per
    sequence (several tiles per CTA)."""
    import ctypes
    import dataclasses
    wl = dataclasses.replace(workloads.llama8b(), batch=2, key_bits=kb, value_bits=2,
                             capacity=2560, lengths=(2560, 2560), name=f"ops{kb}")
    glayer, olayer, spec = _setup(wl)
    assert glayer.tc_operands is not None
    again = torch.empty_like(glayer.tc_operands)
    st = tq.load().tq_prepare_operands(ctypes.byref(glayer.params), again.data_ptr(), None)
    assert st == 0
    torch.cuda.synchronize()
    assert torch.equal(again, glayer.tc_operands)
    T = 2560
    k = torch.stack([workloads.kv_tokens(wl, b, 0, T)[0] for b in range(2)]).to(DEV).contiguous()
    v = torch.stack([workloads.kv_tokens(wl, b, 0, T)[1] for b in range(2)]).to(DEV).contiguous()
    bufs = []
    for prepared in (True, False):
        glayer.params.tc_operands = glayer.tc_operands.data_ptr() if prepared else None
        cache = tq.CompressedCache(glayer, 2, wl.h_kv, T, zero=True)
        tq.tq_quantize_append(glayer, cache, k, v, [0, 0], [T, T - 100])
        torch.cuda.synchronize()
        bufs.append(cache.buffer.cpu().numpy())
    glayer.params.tc_operands = glayer.tc_operands.data_ptr()
    assert np.array_equal(bufs[0], bufs[1])


@pytest.mark.parametrize("kb,vb", [(2, 2), (4, 2), (3, 3), (4, 4)])
def test_quantize_append_bit_widths_bf16_tiles(kb, vb):
    """bf16 appends of 300 tokens (the tensor-core kernel) at every key and
    value width, into a sequence that already holds 77 tokens."""
    import dataclasses
    wl = dataclasses.replace(workloads.llama8b(), batch=2, key_bits=kb, value_bits=vb,
                             capacity=384, lengths=(377, 377), name=f"tcbits{kb}{vb}")
    glayer, olayer, spec = _setup(wl)
    cache = tq.CompressedCache(glayer, 2, wl.h_kv, 384, zero=True)
    T = 300
    k = torch.stack([workloads.kv_tokens(wl, b, 0, T)[0] for b in range(2)])
    v = torch.stack([workloads.kv_tokens(wl, b, 0, T)[1] for b in range(2)])
    tq.tq_quantize_append(glayer, cache, k.to(DEV).contiguous(), v.to(DEV).contiguous(), [77, 0],
                          [T, 250])
    torch.cuda.synchronize()
    buf = cache.buffer.cpu().numpy()
    stats = None
    for b, (start, n) in enumerate([(77, T), (0, 250)]):
        for h in range(wl.h_kv):
            ke, ve = olayer.encode(k[b, :n, h].float().numpy(), v[b, :n, h].float().numpy())
            stats = pu.compare_records(spec, buf, b, h, start, ke, ve, stats, olayer,
                                       k[b, :n, h].float().numpy())
    pu.check_band_fraction(stats)
    print(kb, vb, stats)


@pytest.mark.parametrize("d", [64, 128, 256])
def test_sketch_product_is_float64_s_pi_t(d):
    """W = S Pi^T (the append kernels' float64 refinement reads it) equals
    the float64 product of the float32 matrices to a few ulps."""
    pi, s = workloads.rotation_and_sketch(d, 77)
    pi32, s32 = pi.astype(np.float32), s.astype(np.float32)
    layer = pu.gpu_layer(pi32, s32, 3, 2)
    torch.cuda.synchronize()
    got = layer.s_pit.cpu().numpy()
    ref = s32.astype(np.float64) @ pi32.astype(np.float64).T
    assert got.shape == (d, d)
    assert np.max(np.abs(got - ref)) <= 1e-13 * max(1.0, np.max(np.abs(ref)))


def _tie_values(n_tok, h_kv, d, vb, seed):
    """bf16 values whose groups put many channels exactly on rounding
    thresholds z + (k + 1/2) s (ties) and on the levels z + k s: per group
    the minimum o = m 2^e (m a small integer), the maximum o + L 2^e
    (L = 2^vb - 1), so zero = o and scale = 2^e exactly, and the other
    channels drawn from o + 2^e {k + 1/2, k, k + 1/2 +- 1/8}: at most 8
    significant bits, exact in bf16."""
    rng = np.random.default_rng(seed)
    L = (1 << vb) - 1
    v = np.empty((n_tok, h_kv, d), dtype=np.float64)
    ks = np.arange(L, dtype=np.float64)
    cands = np.concatenate([ks + 0.5, ks, ks + 0.5 + 0.125, ks + 0.5 - 0.125, [L]])
    for t in range(n_tok):
        for h in range(h_kv):
            for g in range(d // 32):
                e = 2.0 ** int(rng.integers(-4, 3))
                o = e * int(rng.integers(-3, 4))
                grp = o + e * rng.choice(cands, size=32)
                grp[rng.integers(0, 32)] = o
                grp[rng.integers(0, 32)] = o + e * L
                grp[:] = np.where(grp < o, o, grp)
                v[t, h, 32 * g:32 * g + 32] = grp
    vt = torch.from_numpy(v).to(torch.bfloat16)
    assert np.array_equal(vt.double().numpy(), v), "tie values must be exact in bf16"
    return vt


@pytest.mark.parametrize("vb", [2, 3, 4])
@pytest.mark.parametrize("T", [128, 8])  # the tensor-core path and the SIMT path
def test_value_codes_exact_ties(vb, T):
    """Group-quantized value codes on exact rounding ties (half to even) and
    exact levels: bit-exact against the oracle with no band, on both append
    kernels."""
    import dataclasses
    wl = dataclasses.replace(workloads.llama8b(), batch=1, key_bits=3, value_bits=vb, capacity=256,
                             lengths=(T,), name=f"ties{vb}")
    glayer, olayer, spec = _setup(wl)
    cache = tq.CompressedCache(glayer, 1, wl.h_kv, 256, zero=True)
    k = workloads.kv_tokens(wl, 0, 0, T)[0]
    v = _tie_values(T, wl.h_kv, 128, vb, seed=vb * 100 + T)
    tq.tq_quantize_append(glayer, cache, k[None].to(DEV).contiguous(), v[None].to(DEV).contiguous(), [0])
    torch.cuda.synchronize()
    buf = cache.buffer.cpu().numpy()
    ties = 0
    for h in range(wl.h_kv):
        ke, ve = olayer.encode(k[:, h].float().numpy(), v[:, h].float().numpy())
        got = spec.read(buf, 0, h, 0, T)
        assert np.array_equal(got["scale16"], ve["scale16"])
        assert np.array_equal(got["zero16"], ve["zero16"])
        assert np.array_equal(got["codes"], ve["codes"]), np.argwhere(got["codes"] != ve["codes"])[:5]
        ties += int(np.sum(ve["t"] == np.floor(ve["t"]) + 0.5))
    assert ties > 100, ties


# ---------------------------------------------------------------------------
# decode parity (oracle-encoded cache uploaded to the device)
# ---------------------------------------------------------------------------

def _oracle_cache(wl, olayer, spec, lengths, dtype_cpu_kv=None):
    """Encode every sequence with the oracle and pack it; returns (buf,
    per-sequence (kes, ves))."""
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


def _run_decode(glayer, wl, buf, lengths, q, max_len=None):
    cache = tq.CompressedCache(glayer, wl.batch, wl.h_kv, wl.capacity)
    cache.buffer.copy_(torch.from_numpy(buf))
    len_dev = torch.tensor(lengths, dtype=torch.int32, device=DEV)
    ml = max(lengths) if max_len is None else max_len
    ws = tq.workspace_for(glayer, cache, wl.h_q, ml)
    out = torch.empty((wl.batch, wl.h_q, wl.d), dtype=torch.float32, device=DEV)
    tq.tq_decode_attention(glayer, cache, q.to(DEV).contiguous(), len_dev, ml, out, ws)
    torch.cuda.synchronize()
    return out.cpu().numpy()


@pytest.mark.parametrize("name", ["tiny", "llama8b", "qwen15b_512", "qwen15b_4096", "qwen15b_8192",
                                  "qwen15b_16384"])
def test_decode_parity(name):
    wl = workloads.by_name(name)
    glayer, olayer, spec = _setup(wl)
    buf, encs = _oracle_cache(wl, olayer, spec, wl.lengths)
    worst = 0.0
    for call in range(wl.n_queries):
        q = workloads.queries(wl, call)
        got = _run_decode(glayer, wl, buf, list(wl.lengths), q)
        for b in range(wl.batch):
            kes, ves = encs[b]
            ref = pu.oracle_decode(olayer, q[b].float().numpy(), kes, ves, wl.lengths[b])
            err = pu.row_rel_err(got[b], ref)
            worst = max(worst, err)
    print(name, "max row rel err", worst)
    assert worst <= pu.REL_TOL


@pytest.mark.parametrize("h_kv,h_q", [(2, 2), (2, 8), (1, 6), (3, 18)])
def test_decode_ragged_lengths_and_gqa(h_kv, h_q):
    """Lengths 1, a tile minus one, a tile plus one, a partial last tile and
    an empty sequence; GQA 1, 4 and 6."""
    base = workloads.qwen15b(512)
    import dataclasses
    lengths = (1, 127, 129, 300, 0)
    wl = dataclasses.replace(base, batch=5, h_kv=h_kv, h_q=h_q, lengths=lengths,
                             capacity=384, name=f"ragged_{h_kv}_{h_q}")
    glayer, olayer, spec = _setup(wl)
    buf, encs = _oracle_cache(wl, olayer, spec, lengths)
    q = workloads.queries(wl, 0)
    got = _run_decode(glayer, wl, buf, list(lengths), q)
    for b in range(wl.batch):
        if lengths[b] == 0:
            assert np.all(got[b] == 0.0)
            continue
        kes, ves = encs[b]
        ref = pu.oracle_decode(olayer, q[b].float().numpy(), kes, ves, lengths[b])
        assert pu.row_rel_err(got[b], ref) <= pu.REL_TOL, b


def test_decode_max_len_bounds_the_read():
    """max_len below a sequence's length: tokens at or beyond max_len are not
    read, so the result equals decode over the first max_len tokens."""
    wl = workloads.scaled(workloads.tiny(), name="maxlen")
    glayer, olayer, spec = _setup(wl)
    buf, encs = _oracle_cache(wl, olayer, spec, wl.lengths)
    q = workloads.queries(wl, 0)
    got = _run_decode(glayer, wl, buf, list(wl.lengths), q, max_len=200)
    kes, ves = encs[0]
    ref = pu.oracle_decode(olayer, q[0].float().numpy(), kes, ves, 200)
    assert pu.row_rel_err(got[0], ref) <= pu.REL_TOL


def test_workspace_too_small_is_rejected():
    wl = workloads.tiny()
    glayer, _, _ = _setup(wl)
    cache = tq.CompressedCache(glayer, 1, wl.h_kv, wl.capacity)
    n = tq.tq_decode_workspace_size(glayer, cache, wl.h_q, 256)
    assert n > 0
    ws = torch.empty(n - 256, dtype=torch.uint8, device=DEV)
    out = torch.empty((1, wl.h_q, 128), device=DEV)
    len_dev = torch.tensor([256], dtype=torch.int32, device=DEV)
    with pytest.raises(tq.TQError) as e:
        tq.tq_decode_attention(glayer, cache, workloads.queries(wl).to(DEV), len_dev, 256, out, ws)
    assert e.value.status == 4


# ---------------------------------------------------------------------------
# dequantize parity and end to end
# ---------------------------------------------------------------------------

def test_dequantize_parity():
    wl = workloads.tiny()
    glayer, olayer, spec = _setup(wl)
    buf, encs = _oracle_cache(wl, olayer, spec, wl.lengths)
    cache = tq.CompressedCache(glayer, 1, wl.h_kv, wl.capacity)
    cache.buffer.copy_(torch.from_numpy(buf))
    start, count = 37, 150
    ko = torch.empty((count, wl.h_kv, 128), device=DEV)
    vo = torch.empty_like(ko)
    tq.tq_dequantize(glayer, cache, 0, start, count, ko, vo)
    torch.cuda.synchronize()
    from oracle import quant
    kes, ves = encs[0]
    for h in range(wl.h_kv):
        ke, ve = kes[h], ves[h]
        sl = slice(start, start + count)
        kref = quant.dequantize_keys(ke["idx"][sl], ke["sign"][sl], ke["nk16"][sl],
                                     ke["rn16"][sl], olayer.pi, olayer.s, olayer.cent)
        vref = quant.dequantize_values(ve["codes"][sl], ve["scale16"][sl], ve["zero16"][sl], 32)
        assert pu.row_rel_err(ko[:, h].cpu().numpy(), kref) <= 1e-5
        assert pu.row_rel_err(vo[:, h].cpu().numpy(), vref) <= 1e-6


@pytest.mark.parametrize("name", ["tiny", "llama8b"])
def test_end_to_end_quantize_then_decode(name):
    """GPU quantize -> GPU decode, held to 1e-3 in two steps: the GPU's records
    equal the oracle's encoding outside the bands (checked here), and the GPU
    decode of those records equals the oracle's decode of the same records.
    When no record differs at all (no banded code took the other cell, no norm
    differs in its last fp16 bit), the GPU result is also held to 1e-3 against
    the oracle's own quantize -> decode chain."""
    wl = workloads.by_name(name)
    glayer, olayer, spec = _setup(wl)
    cache = tq.CompressedCache(glayer, wl.batch, wl.h_kv, wl.capacity)
    n = wl.lengths[0]
    k, v = workloads.kv_tokens(wl, 0, 0, n)
    tq.tq_quantize_append(glayer, cache, k[None].to(DEV).contiguous(),
                          v[None].to(DEV).contiguous(), [0])
    q = workloads.queries(wl, 0)
    len_dev = torch.tensor([n], dtype=torch.int32, device=DEV)
    ws = tq.workspace_for(glayer, cache, wl.h_q, n)
    out = torch.empty((1, wl.h_q, 128), device=DEV)
    tq.tq_decode_attention(glayer, cache, q.to(DEV), len_dev, n, out, ws)
    torch.cuda.synchronize()
    got = out[0].cpu().numpy()
    buf = cache.buffer.cpu().numpy()
    kf, vf = k.float().numpy(), v.float().numpy()
    kes, ves = pu.oracle_records_for(olayer, kf, vf)
    stats = None
    identical = True
    for h in range(wl.h_kv):
        stats = pu.compare_records(spec, buf, 0, h, 0, kes[h], ves[h], stats, olayer, kf[:, h])
        rec = spec.read(buf, 0, h, 0, n)
        identical &= all(np.array_equal(rec[f], pu.logical(kes[h], ves[h])[f]) for f in rec)
    pu.check_band_fraction(stats)
    rec = attention.stack_heads([spec.read(buf, 0, h, 0, n) for h in range(wl.h_kv)])
    ref_dev = attention.decode_one_sequence(q[0].float().numpy(), rec, olayer.pi, olayer.s,
                                            olayer.cent, olayer.group)
    assert pu.row_rel_err(got, ref_dev) <= pu.REL_TOL
    ref = pu.oracle_decode(olayer, q[0].float().numpy(), kes, ves, n)
    err = pu.row_rel_err(got, ref)
    print(name, "records identical:", identical, "end-to-end row rel err", err, stats)
    if identical:
        assert err <= pu.REL_TOL


@pytest.mark.parametrize("kb,vb", [(2, 2), (4, 2), (3, 4), (4, 3)])
def test_decode_bit_widths(kb, vb):
    """1-, 2- and 3-bit Lloyd-Max keys and 2-4-bit values at GQA 4 (tensor-core
    kernel where built, the general SIMT kernel otherwise)."""
    import dataclasses
    lengths = (700, 256)
    wl = dataclasses.replace(workloads.llama8b(), batch=2, key_bits=kb, value_bits=vb,
                             lengths=lengths, capacity=768, name=f"dec_bits{kb}{vb}")
    glayer, olayer, spec = _setup(wl)
    buf, encs = _oracle_cache(wl, olayer, spec, lengths)
    q = workloads.queries(wl, 0)
    got = _run_decode(glayer, wl, buf, list(lengths), q)
    for b in range(wl.batch):
        kes, ves = encs[b]
        ref = pu.oracle_decode(olayer, q[b].float().numpy(), kes, ves, lengths[b])
        assert pu.row_rel_err(got[b], ref) <= pu.REL_TOL, (kb, vb, b)


@pytest.mark.parametrize("h_kv,h_q", [(2, 2), (2, 4), (2, 8), (1, 8)])
def test_decode_ragged_packed_values_gqa(h_kv, h_q):
    """2-bit packed values (the tensor-core kernel) at GQA 1, 2, 4 and 8, with
    lengths 1, a tile minus one, a tile plus one, a partial last tile and an
    empty sequence."""
    import dataclasses
    lengths = (1, 127, 129, 300, 0)
    wl = dataclasses.replace(workloads.llama8b(), batch=5, h_kv=h_kv, h_q=h_q, lengths=lengths,
                             capacity=384, name=f"ragged_packed_{h_kv}_{h_q}")
    glayer, olayer, spec = _setup(wl)
    buf, encs = _oracle_cache(wl, olayer, spec, lengths)
    q = workloads.queries(wl, 0)
    got = _run_decode(glayer, wl, buf, list(lengths), q)
    for b in range(wl.batch):
        if lengths[b] == 0:
            assert np.all(got[b] == 0.0)
            continue
        kes, ves = encs[b]
        ref = pu.oracle_decode(olayer, q[b].float().numpy(), kes, ves, lengths[b])
        assert pu.row_rel_err(got[b], ref) <= pu.REL_TOL, (h_kv, h_q, b)


@pytest.mark.parametrize("kb", [2, 3, 4])
def test_decode_asymmetric_codebook(kb):
    """A caller-supplied codebook that is not symmetric about zero (shifted and
    stretched Lloyd-Max levels): decode must use every level as given, so the
    constant and even-order terms of its expansion in the code bits matter."""
    import dataclasses
    lengths = (700, 256)
    wl = dataclasses.replace(workloads.llama8b(), batch=2, key_bits=kb, lengths=lengths,
                             capacity=768, name=f"asym{kb}")
    glayer, olayer, spec = _setup(wl)
    buf, encs = _oracle_cache(wl, olayer, spec, lengths)
    n = len(olayer.cent)
    cent = np.asarray(olayer.cent, np.float64) * (1.0 + 0.1 * np.arange(n) / n) + 0.02
    cent = np.asarray(cent.astype(np.float32), np.float64)
    olayer.cent = cent
    glayer.centroids.copy_(torch.tensor(cent, dtype=torch.float32))
    q = workloads.queries(wl, 0)
    got = _run_decode(glayer, wl, buf, list(lengths), q)
    for b in range(wl.batch):
        kes, ves = encs[b]
        ref = pu.oracle_decode(olayer, q[b].float().numpy(), kes, ves, lengths[b])
        assert pu.row_rel_err(got[b], ref) <= pu.REL_TOL, (kb, b)


@pytest.mark.parametrize("name,kb,vb,h_kv,h_q", [
    ("llama8b", 3, 2, 2, 8),     # tensor-core kernel, GQA 4
    ("qwen15b_512", 3, 3, 1, 6),  # tensor-core kernel, 3-bit values, GQA 6
    ("llama8b", 3, 4, 2, 4),     # SIMT split-K kernel
])
def test_decode_with_recent_window(name, kb, vb, h_kv, h_q):
    """Compressed history plus an exact window of the next tokens of each
    sequence, one softmax: lengths 0, 1, a tile plus one, 300; window
    lengths 5, 0, 128, 64 (capacity 128), and a sequence with neither."""
    import dataclasses
    lengths = (0, 1, 129, 300, 0)
    wlens = (5, 0, 128, 64, 0)
    base = workloads.by_name(name)
    wl = dataclasses.replace(base, batch=5, h_kv=h_kv, h_q=h_q, key_bits=kb, value_bits=vb,
                             lengths=lengths, capacity=384, name=f"win_{name}_{kb}{vb}")
    glayer, olayer, spec = _setup(wl)
    buf, encs = _oracle_cache(wl, olayer, spec, lengths)
    cap = 128
    dt = torch.bfloat16 if wl.kv_dtype == "bf16" else torch.float32
    wk = torch.zeros((wl.batch, h_kv, cap, 128), dtype=dt)
    wv = torch.zeros_like(wk)
    for b in range(wl.batch):
        if wlens[b]:
            k, v = workloads.kv_tokens(wl, b, lengths[b], lengths[b] + wlens[b])
            wk[b, :, :wlens[b]] = k.transpose(0, 1).to(dt)
            wv[b, :, :wlens[b]] = v.transpose(0, 1).to(dt)
    q = workloads.queries(wl, 0)
    cache = tq.CompressedCache(glayer, wl.batch, wl.h_kv, wl.capacity)
    cache.buffer.copy_(torch.from_numpy(buf))
    len_dev = torch.tensor(lengths, dtype=torch.int32, device=DEV)
    wlen_dev = torch.tensor(wlens, dtype=torch.int32, device=DEV)
    ml = max(lengths)
    ws = tq.workspace_for(glayer, cache, wl.h_q, ml)
    out = torch.empty((wl.batch, wl.h_q, 128), device=DEV)
    tq.tq_decode_attention_window(glayer, cache, q.to(DEV).contiguous(), len_dev, ml,
                                  wk.to(DEV).contiguous(), wv.to(DEV).contiguous(), wlen_dev, out, ws)
    torch.cuda.synchronize()
    got = out.cpu().numpy()
    from oracle import attention
    for b in range(wl.batch):
        n, w = lengths[b], wlens[b]
        rec = None
        if n:
            kes, ves = encs[b]
            rec = attention.stack_heads([pu.logical(ke, ve) for ke, ve in zip(kes, ves)])
        wkb = wk[b, :, :w].transpose(0, 1).float().numpy()
        wvb = wv[b, :, :w].transpose(0, 1).float().numpy()
        ref = attention.decode_with_window(q[b].float().numpy(), rec, wkb, wvb, olayer.pi, olayer.s,
                                           olayer.cent, 32)
        if n + w == 0:
            assert np.all(got[b] == 0.0)
            continue
        assert pu.row_rel_err(got[b], ref) <= pu.REL_TOL, (name, b)


@pytest.mark.gpu
@pytest.mark.parametrize("h_kv,h_q,kb,t_chunk", [(2, 8, 3, 3), (2, 4, 3, 5), (2, 2, 3, 8), (2, 8, 4, 3), (1, 1, 3, 11)])
def test_prefill_parity(h_kv, h_q, kb, t_chunk):
    """Causal chunked prefill over the compressed cache: passes of 4 / G
    query tokens (GQA 1 -> 4 tokens, GQA 2 -> 2) plus smaller last passes,
    single-token passes at GQA 4; ragged lengths, a sequence holding exactly
    the chunk."""
    import dataclasses
    lengths = (t_chunk, 127, 129, 300)
    wl = dataclasses.replace(workloads.llama8b(), batch=4, h_kv=h_kv, h_q=h_q, key_bits=kb,
                             lengths=lengths, capacity=384, name=f"prefill_{h_kv}_{h_q}_{kb}_{t_chunk}")
    glayer, olayer, spec = _setup(wl)
    buf, encs = _oracle_cache(wl, olayer, spec, lengths)
    g = torch.Generator().manual_seed(5)
    q = torch.randn((wl.batch, t_chunk, h_q, wl.d), generator=g).to(torch.bfloat16)
    cache = tq.CompressedCache(glayer, wl.batch, wl.h_kv, wl.capacity)
    cache.buffer.copy_(torch.from_numpy(buf))
    len_dev = torch.tensor(lengths, dtype=torch.int32, device=DEV)
    ml = max(lengths)
    ws = tq.prefill_workspace_for(glayer, cache, h_q, t_chunk, ml)
    out = torch.full((wl.batch, t_chunk, h_q, wl.d), float("nan"), dtype=torch.float32, device=DEV)
    tq.tq_prefill_attention(glayer, cache, q.to(DEV).contiguous(), len_dev, ml, out, ws)
    torch.cuda.synchronize()
    got = out.cpu().numpy()
    for b in range(wl.batch):
        kes, ves = encs[b]
        for t in range(t_chunk):
            m = lengths[b] - (t_chunk - 1 - t)
            ref = pu.oracle_decode(olayer, q[b, t].float().numpy(), kes, ves, m)
            assert pu.row_rel_err(got[b, t], ref) <= pu.REL_TOL, (b, t)


@pytest.mark.parametrize("kb,vb,h_q", [(3, 2, 64), (2, 2, 64), (4, 2, 32), (3, 3, 48), (3, 2, 32)])
def test_decode_long_splits_every_kernel_shape(kb, vb, h_q):
    """Every tensor-core decode shape with many tiles per CTA (32 sequences x
    8 KV heads x 4096 tokens: the split plan gives each CTA 16 tiles, four per
    worker group): the call finishes well inside the kernels' 2 s wait
    bound, and sampled rows match the oracle run on the device's own records."""
    import dataclasses
    import time
    from oracle import attention
    n, B, hkv = 4096, 32, 8
    wl = dataclasses.replace(workloads.batched(), batch=B, h_kv=hkv, h_q=h_q, key_bits=kb,
                             value_bits=vb, lengths=(n,) * B, capacity=n, name=f"long{kb}{vb}{h_q}")
    glayer, olayer, spec = _setup(wl)
    cache = tq.CompressedCache(glayer, B, hkv, n)
    g = torch.Generator(device=DEV).manual_seed(9)
    for b0 in range(0, B, 8):
        k = torch.randn((8, n, hkv, 128), generator=g, device=DEV).to(torch.bfloat16)
        v = torch.randn((8, n, hkv, 128), generator=g, device=DEV).to(torch.bfloat16)
        # sequences b0 .. b0 + 7 take n tokens, the others none
        ks = torch.zeros((B, n, hkv, 128), dtype=torch.bfloat16, device=DEV)
        vs = torch.zeros_like(ks)
        ks[b0:b0 + 8], vs[b0:b0 + 8] = k, v
        nnew = [n if b0 <= b < b0 + 8 else 0 for b in range(B)]
        tq.tq_quantize_append(glayer, cache, ks, vs, [0] * B, nnew)
        del ks, vs, k, v
    q = torch.randn((B, h_q, 128), generator=g, device=DEV).to(torch.bfloat16)
    len_dev = torch.full((B,), n, dtype=torch.int32, device=DEV)
    ws = tq.workspace_for(glayer, cache, h_q, n)
    out = torch.empty((B, h_q, 128), dtype=torch.float32, device=DEV)
    tq.tq_decode_attention(glayer, cache, q, len_dev, n, out, ws)
    torch.cuda.synchronize()
    t0 = time.time()
    tq.tq_decode_attention(glayer, cache, q, len_dev, n, out, ws)
    torch.cuda.synchronize()
    assert time.time() - t0 < 0.5
    buf = cache.buffer.cpu().numpy()
    got = out.cpu().numpy()
    for b in (0, B - 1):
        rec = attention.stack_heads([spec.read(buf, b, h, 0, n) for h in range(hkv)])
        ref = attention.decode_one_sequence(q[b].float().cpu().numpy(), rec, olayer.pi, olayer.s,
                                            olayer.cent, olayer.group)
        assert pu.row_rel_err(got[b], ref) <= pu.REL_TOL, b
