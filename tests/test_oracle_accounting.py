"""The oracle's accounting functions reproduce the numbers the pages print
(tests/golden/accounting_pages.txt gives each number and where it appears)."""
import os

import pytest

from conftest import GOLDEN
from oracle import accounting as acc


def golden():
    vals = {}
    with open(os.path.join(GOLDEN, "accounting_pages.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                k, v = line.split("=")
                vals[k.strip()] = float(v)
    return vals


G = golden()
P7B = 7e9
GB = 1e9


def test_sixteen_bytes_per_param():
    assert acc.bytes_per_param_mixed_adamw() == G["bytes_per_param"]
    assert acc.optimizer_state_bytes_per_param() == 12


def test_7b_ledger():
    assert acc.ddp_bytes_per_card(P7B) / GB == G["ddp_7b_gb"]
    # the page's figures are rounded to 0.1 GB (ZeRO-3: "about 1.7")
    assert acc.zero1_bytes_per_card(P7B, 64) / GB == pytest.approx(29.3125)
    assert round(acc.zero1_bytes_per_card(P7B, 64) / GB, 1) == G["zero1_7b_64_gb"]
    assert round(acc.zero2_bytes_per_card(P7B, 64) / GB, 1) == G["zero2_7b_64_gb"]
    assert acc.zero3_bytes_per_card(P7B, 64) / GB == pytest.approx(1.75)
    assert abs(acc.zero3_bytes_per_card(P7B, 64) / GB - G["zero3_7b_64_gb"]) <= 0.05 + 1e-9


def test_fits_table_at_twelve_bytes():
    mem = 80e9
    got = [acc.largest_model_that_fits(mem, 8, s, k=8) / 1e9 for s in range(4)]
    want = [G["fits_ddp_b"], G["fits_zero1_b"], G["fits_zero2_b"], G["fits_zero3_b"]]
    for g, w in zip(got, want):
        assert round(g, 2 if w < 10 else 1) == pytest.approx(w), (got, want)


def test_communication_volumes():
    N = 1_000_000
    # ring: 2 (W-1)/W of the buffer per rank, approaching 2x as W grows
    assert acc.ring_allreduce_bytes_per_rank(N, 2, 1) == N
    assert acc.ring_allreduce_bytes_per_rank(N, 1000, 1) == pytest.approx(2 * N, rel=1e-3)
    # ZeRO-1: reduce-scatter + all-gather moves exactly what the all-reduce moves
    for W in (2, 8, 64):
        assert acc.reduce_scatter_bytes_per_rank(N, W, 2) + acc.all_gather_bytes_per_rank(N, W, 2) \
            == acc.ring_allreduce_bytes_per_rank(N, W, 2)
    assert acc.zero1_comm_elems(N) == G["zero1_comm_factor"] * N
    assert acc.zero3_comm_elems(N) == G["zero3_comm_factor"] * N
    assert acc.zero3_comm_elems(N) / acc.zero1_comm_elems(N) == 1.5
    # 7B: 14 GB of bf16 gradient, ~28 GB moved per card per step
    assert acc.ring_allreduce_bytes_per_rank(P7B, 10**6, 2) / GB == pytest.approx(G["ddp_7b_sync_gb"], rel=1e-5)
