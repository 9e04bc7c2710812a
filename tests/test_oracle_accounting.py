"""Pin the storage accounting against the ratios the audit script prints
("turboquant/audit_claims.py", AUDIT 1 and its SUMMARY; fixture
tests/golden/audit1_compression.json)."""

import json
import os

from oracle import accounting


def test_audit1_ratios(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "audit1_compression.json")))
    st = g["setup"]
    tol = g["printed_precision"]
    args = (st["h_kv"], st["d"], st["key_bits"], st["value_bits"], st["group"])
    r4096 = accounting.ratios(4096, *args)
    assert abs(r4096["data_only"] - g["printed"]["data_only"]) <= tol
    for n, want in g["printed"]["all_in"].items():
        got = accounting.ratios(int(n), *args)["all_in"]
        assert abs(got - want) <= tol, (n, got, want)
    r_big = accounting.ratios(g["approaches_5x_at"], *args)["all_in"]
    assert 4.95 <= r_big < r4096["data_only"]


def test_fp16_record_is_512_bytes_per_token_head():
    assert accounting.fp16_kv_bytes(1, 1, 128) == 512
    assert accounting.data_bytes(1, 1, 128, 3, 2, 32) == 100
