"""tq_decode_attention_noalloc: decode for callers that cannot allocate.

Callers such as a plain C host without a device allocator, a decode loop
that must not call cudaMalloc, or an engine that has reserved all free device
memory cannot pass the library a workspace.  The no-allocation entry point
keeps its scratch in a fixed device array inside the library instead.  This
test calls it through the C ABI twice in a row (different queries and
lengths, so the second call runs on scratch the first call left behind) and
checks each result against the workspace entry point's within the parity
tolerance.  It also checks that a request larger than the fixed scratch is
rejected before any launch.

The file is named so that pytest collects it last.
"""

import numpy as np
import pytest
import torch

from kv_cache_quantization_turboquantprod_b200 import tq, workloads

pytestmark = pytest.mark.gpu

DEV = "cuda"
REL_TOL = 1e-3


def _row_rel_err(got, ref):
    g = got.reshape(-1, got.shape[-1])
    r = ref.reshape(-1, ref.shape[-1])
    num = np.abs(g - r).max(axis=1)
    den = np.abs(r).max(axis=1)
    return float(np.max(np.where(den > 0, num / np.maximum(den, 1e-300), num)))


@pytest.fixture(scope="module")
def filled_cache():
    from kv_cache_quantization_turboquantprod_b200 import build
    build.build()
    tq.load()
    wl = workloads.scaled(workloads.llama8b(), batch=3, lengths=(4096, 1000, 2500),
                          capacity=4096, name="noalloc")
    _, pi32, s32 = workloads.layer_matrices(wl)
    layer = tq.Layer(pi32, s32, wl.key_bits, wl.value_bits, device=DEV)
    cache = tq.CompressedCache(layer, wl.batch, wl.h_kv, wl.capacity, device=DEV)
    ks, vs = [], []
    for b in range(wl.batch):
        k, v = workloads.kv_tokens(wl, b, 0, wl.capacity, device=DEV)
        ks.append(k)
        vs.append(v)
    k = torch.stack(ks).contiguous()
    v = torch.stack(vs).contiguous()
    tq.tq_quantize_append(layer, cache, k, v, [0] * wl.batch, list(wl.lengths))
    torch.cuda.synchronize()
    return wl, layer, cache


def _with_workspace(layer, cache, q, lengths, max_len):
    len_dev = torch.tensor(lengths, dtype=torch.int32, device=DEV)
    ws = tq.workspace_for(layer, cache, q.shape[1], max_len, device=DEV)
    out = torch.empty((q.shape[0], q.shape[1], 128), dtype=torch.float32, device=DEV)
    tq.tq_decode_attention(layer, cache, q, len_dev, max_len, out, ws)
    return out


def _no_alloc(layer, cache, q, lengths, max_len):
    len_dev = torch.tensor(lengths, dtype=torch.int32, device=DEV)
    out = torch.full((q.shape[0], q.shape[1], 128), float("nan"), dtype=torch.float32, device=DEV)
    tq.tq_decode_attention_noalloc(layer, cache, q, len_dev, max_len, out)
    return out


def test_no_alloc_matches_workspace_entry_point_twice(filled_cache):
    wl, layer, cache = filled_cache
    calls = [
        (workloads.queries(wl, 0, device=DEV), list(wl.lengths), max(wl.lengths)),
        (workloads.queries(wl, 1, device=DEV), [17, 1000, 129], 1000),
    ]
    for q, lengths, max_len in calls:
        got = _no_alloc(layer, cache, q, lengths, max_len)
        ref = _with_workspace(layer, cache, q, lengths, max_len)
        torch.cuda.synchronize()
        g, r = got.cpu().numpy(), ref.cpu().numpy()
        assert np.all(np.isfinite(g))
        assert _row_rel_err(g, r) <= REL_TOL


def test_no_alloc_rejects_oversized_requests(filled_cache):
    wl, layer, _ = filled_cache
    # a batch large enough that the rotated queries alone exceed the scratch
    big_batch = 1024
    cache = tq.CompressedCache(layer, big_batch, 8, 128, device=DEV)
    need = tq.tq_decode_workspace_size(layer, cache, 32, 128)
    assert need > tq.NOALLOC_SCRATCH_BYTES
    q = torch.zeros((big_batch, 32, 128), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(tq.TQError) as e:
        _no_alloc(layer, cache, q, [1] * big_batch, 128)
    assert e.value.status == 4
