"""Helpers shared by the GPU parity tests: run the oracle on the same seeded
inputs, read the library's cache bytes back with the oracle's layout reader,
and compare with the bands and tolerances the parity bar fixes.

Parity bar:
* key codes and sign bits bit-exact except coordinates within 1e-6 of a
  decision boundary (|y - t| < 1e-6, oracle y) or of zero (|S r| < 1e-6);
  the band count is reported and must be <= 1e-4 of all coordinates;
* value codes bit-exact except in the value band (a code whose exact quotient
  t = (v - zero16) / scale16 lies within 1e-6 of a half-integer without being
  one; an exact half-integer is a tie that both sides resolve half-to-even),
  counted, <= 1e-4 of all coordinates; scales and zeros bit-exact;
* norms and attention outputs within 1e-3 relative: per row,
  max |gpu - oracle| / max |oracle|.
"""

from __future__ import annotations

import numpy as np
import torch

from kv_cache_quantization_turboquantprod_b200 import tq, workloads
from oracle import attention, codebook, layout, quant

BAND = 1e-6
BAND_FRACTION_MAX = 1e-4
REL_TOL = 1e-3


class OracleLayer:
    """The oracle's view of one layer: the same Pi (float32 values), S and
    codebooks from the oracle's own Lloyd-Max (keys: key_bits - 1 bits;
    TurboQuant-MSE values: value_bits bits)."""

    def __init__(self, pi32: np.ndarray, s32: np.ndarray, key_bits: int, value_bits: int,
                 group: int = 32, value_mode: str = "group"):
        self.pi = np.asarray(pi32, np.float64)
        self.s = np.asarray(s32, np.float64)
        self.key_bits, self.value_bits, self.group = key_bits, value_bits, group
        self.value_mode = value_mode
        self.cent, self.bnd, _ = codebook.lloyd_max_gaussian(key_bits - 1, self.pi.shape[0])
        self.vcent = self.vbnd = None
        if value_mode == "mse":
            self.vcent, self.vbnd, _ = codebook.lloyd_max_gaussian(value_bits, self.pi.shape[0])

    def encode(self, k: np.ndarray, v: np.ndarray):
        ke = quant.encode_keys(k, self.pi, self.s, self.cent, self.bnd)
        if self.value_mode == "mse":
            ve = quant.encode_values_mse(v, self.pi, self.vcent, self.vbnd)
        else:
            ve = quant.encode_values(v, self.value_bits, self.group)
        return ke, ve


def gpu_layer(pi32, s32, key_bits, value_bits, device="cuda", value_mode="group"):
    return tq.Layer(pi32, s32, key_bits, value_bits, device=device, value_mode=value_mode)


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy()


def compare_records(spec: layout.CacheSpec, buf: np.ndarray, b: int, h: int, pos0: int,
                    ke: dict, ve: dict, stats: dict | None = None, layer=None,
                    keys: np.ndarray | None = None) -> dict:
    """Compare the library's records of tokens [pos0, pos0+n) of (b, h) with
    the oracle's encoding (ke, ve of n vectors).  Raises AssertionError on a
    mismatch outside the bands; returns accumulated band statistics.
    layer / keys (the oracle layer and the n key vectors) let a vector whose
    banded code took the other cell be checked against that cell's residual."""
    n = len(ke["nk16"])
    got = spec.read(buf, b, h, pos0, n)
    stats = stats if stats is not None else {"coords": 0, "code_band": 0, "sign_band": 0,
                                             "value_band": 0, "max_norm_rel": 0.0}
    bnd = np.asarray(codebook.lloyd_max_gaussian(spec.key_bits - 1, spec.d)[1])
    # codes: band where y is within 1e-6 of a boundary
    near = np.zeros_like(ke["y"], dtype=bool)
    for t in bnd:
        near |= np.abs(ke["y"] - t) < BAND
    zero = ke["nk"] == 0
    near[zero] = False
    bad = (got["idx"] != ke["idx"]) & ~near
    assert not bad.any(), f"code mismatch outside band at (b={b}, h={h}): {np.argwhere(bad)[:5]}"
    if layer is not None:
        layer_pi, layer_s, layer_cent = layer.pi, layer.s, layer.cent
    elif (got["idx"] != ke["idx"]).any():
        raise AssertionError("banded code mismatch: pass layer= and keys= to check its residual")
    # a vector whose banded code went to the other cell has the residual,
    # signs and ||r|| of the cell the library chose: take those from the
    # oracle's steps 4-5 on the library's codes
    z_ref, sign_ref, rn16_ref = ke["z"], ke["sign"], ke["rn16"]
    alt = np.flatnonzero((got["idx"] != ke["idx"]).any(axis=1) & ~zero)
    if alt.size:
        res = quant.residual_sketch(quant.unit_keys(keys[alt]), got["idx"][alt], layer_pi, layer_s,
                                    layer_cent)
        z_ref, sign_ref, rn16_ref = z_ref.copy(), sign_ref.copy(), rn16_ref.copy()
        z_ref[alt], sign_ref[alt], rn16_ref[alt] = res["z"], res["sign"], quant.fp16(res["rn"])
    snear = np.abs(z_ref) < BAND
    snear[zero] = False
    bad = (got["sign"] != sign_ref) & ~snear
    assert not bad.any(), f"sign mismatch outside band at (b={b}, h={h}): {np.argwhere(bad)[:5]}"
    stats["alt_cell_vectors"] = stats.get("alt_cell_vectors", 0) + int(alt.size)
    if "vidx" in ve:
        # TurboQuant-MSE values: cells exact outside |y - t| < 1e-6 of the
        # values' boundaries (oracle y), the norm within the norm tolerance
        vb = codebook.lloyd_max_gaussian(spec.value_bits, spec.d)[1]
        vnear = np.zeros_like(ve["vy"], dtype=bool)
        for tb in vb:
            vnear |= np.abs(ve["vy"] - tb) < BAND
        vnear[ve["nv"] == 0] = False
        bad = (got["vidx"] != ve["vidx"]) & ~vnear
        assert not bad.any(), f"value cell mismatch at (b={b}, h={h}): {np.argwhere(bad)[:5]}"
        rel = np.abs(got["nv16"] - ve["nv16"]) / np.maximum(np.abs(ve["nv16"]), 1e-30)
        rel[(ve["nv16"] == 0) & (got["nv16"] == 0)] = 0.0
        assert rel.max(initial=0.0) <= REL_TOL, f"nv16 rel err {rel.max()}"
    else:
        vnear = value_band(ve)
        bad = (got["codes"] != ve["codes"]) & ~vnear
        assert not bad.any(), f"value code mismatch at (b={b}, h={h}): {np.argwhere(bad)[:5]}"
        assert np.array_equal(got["scale16"], ve["scale16"]), "value scale mismatch"
        assert np.array_equal(got["zero16"], ve["zero16"]), "value zero mismatch"
    for key in ("nk16", "rn16"):
        ref = ke[key] if key == "nk16" else rn16_ref
        rel = np.abs(got[key] - ref) / np.maximum(np.abs(ref), 1e-30)
        rel[(ref == 0) & (got[key] == 0)] = 0.0
        assert rel.max(initial=0.0) <= REL_TOL, f"{key} rel err {rel.max()}"
        stats["max_norm_rel"] = max(stats["max_norm_rel"], float(rel.max(initial=0.0)))
    stats["coords"] += n * spec.d
    stats["code_band"] += int(near.sum())
    stats["sign_band"] += int(snear.sum())
    stats["value_band"] += int(vnear.sum())
    vkey = "vidx" if "vidx" in ve else "codes"
    stats["value_mismatch_in_band"] = stats.get("value_mismatch_in_band", 0) + int(
        (got[vkey] != ve[vkey]).sum())
    return stats


def value_band(ve: dict):
    """Per-element value band mask [n, d] of the oracle's value encoding
    ``ve``: quotients within 1e-6 of a half-integer, exact ties excluded."""
    t = ve["t"]
    half = np.floor(t) + 0.5
    return (np.abs(t - half) < BAND) & (t != half)


def check_band_fraction(stats: dict) -> None:
    for key in ("code_band", "sign_band", "value_band"):
        frac = stats[key] / max(stats["coords"], 1)
        assert frac <= BAND_FRACTION_MAX, f"{key} fraction {frac}"


def row_rel_err(got: np.ndarray, ref: np.ndarray) -> float:
    """max over rows of max|got - ref| / max|ref| (rows = last axis)."""
    g = got.reshape(-1, got.shape[-1])
    r = ref.reshape(-1, ref.shape[-1])
    num = np.abs(g - r).max(axis=1)
    den = np.abs(r).max(axis=1)
    rel = np.where(den > 0, num / np.maximum(den, 1e-300), num)
    return float(rel.max(initial=0.0))


def oracle_records_for(layer: OracleLayer, k: np.ndarray, v: np.ndarray):
    """Encode [n, H_kv, d] keys/values head by head; returns per-head lists."""
    kes, ves = [], []
    for h in range(k.shape[1]):
        ke, ve = layer.encode(k[:, h], v[:, h])
        kes.append(ke)
        ves.append(ve)
    return kes, ves


def logical(ke: dict, ve: dict) -> dict:
    if "vidx" in ve:
        return {"idx": ke["idx"], "sign": ke["sign"], "nk16": ke["nk16"], "rn16": ke["rn16"],
                "vidx": ve["vidx"], "nv16": ve["nv16"]}
    return {"idx": ke["idx"], "sign": ke["sign"], "nk16": ke["nk16"], "rn16": ke["rn16"],
            "codes": ve["codes"], "scale16": ve["scale16"], "zero16": ve["zero16"]}


def oracle_decode(layer: OracleLayer, q: np.ndarray, kes: list, ves: list, length: int,
                  start: int = 0) -> np.ndarray:
    """Oracle decode for one sequence from per-head encodings, using tokens
    [start, start + length) of the encodings."""
    recs = []
    for ke, ve in zip(kes, ves):
        r = logical(ke, ve)
        recs.append({k2: v2[start:start + length] for k2, v2 in r.items()})
    rec = attention.stack_heads(recs)
    return attention.decode_one_sequence(q, rec, layer.pi, layer.s, layer.cent, layer.group,
                                         value_centroids=layer.vcent)


def fill_cache_gpu(glayer, cache, wl, lengths, device="cuda") -> None:
    """Quantize-append every sequence's synthetic K/V (the workload's 8192-token
    chunks drawn on the device) up to lengths[b] tokens, one call per chunk."""
    chunk = workloads.TOKEN_CHUNK
    lens = [0] * wl.batch
    for c in range((max(lengths) + chunk - 1) // chunk):
        t0 = c * chunk
        nnew = [max(0, min(lengths[b] - t0, chunk)) for b in range(wl.batch)]
        if max(nnew) == 0:
            break
        T = max(nnew)
        ks, vs = [], []
        for b in range(wl.batch):
            k, v = workloads.kv_chunk(wl, b, c, device)
            ks.append(k[:T])
            vs.append(v[:T])
        k = torch.stack(ks).contiguous()
        v = torch.stack(vs).contiguous()
        tq.tq_quantize_append(glayer, cache, k, v, lens, nnew)
        lens = [lens[b] + nnew[b] for b in range(wl.batch)]
        del k, v, ks, vs
    torch.cuda.synchronize()


def oracle_decode_head(layer: OracleLayer, spec, buf: np.ndarray, b: int, h: int, n: int,
                       q_heads: np.ndarray) -> np.ndarray:
    """Oracle decode of the G query heads of KV head h of sequence b over the
    first n records of the library's cache bytes (read with the oracle's own
    layout reader): [G, d]."""
    rec = attention.stack_heads([spec.read(buf, b, h, 0, n)])
    return attention.decode_one_sequence(q_heads, rec, layer.pi, layer.s, layer.cent, layer.group,
                                         value_centroids=layer.vcent)
