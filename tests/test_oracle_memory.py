"""Pin the oracle's per-rank model-state accounting to the figures the pages
print (tests/golden/memory_pages.txt) and to the stage reduction factors."""
import os

import oracle as O


def rows(path):
    out = []
    for line in open(path):
        line = line.strip()
        if line and not line.startswith("#"):
            t = line.split()
            out.append((t[0], int(t[1]), float(t[2]), float(t[3]), t[4], float(t[5]), " ".join(t[6:])))
    return out


def test_pages_figures(golden_dir):
    got_any = 0
    for what, stage, psi, N, relation, value, cite in rows(os.path.join(golden_dir, "memory_pages.txt")):
        b = O.fp32_weight_bytes(psi) if what == "fp32w" else O.model_state_bytes(stage, psi, N)
        if relation == "approx":
            assert abs(b / value - 1) <= 0.01, (cite, b)
        elif relation == "gt":
            assert b > value, (cite, b)
        elif relation == "lt":
            assert b < value, (cite, b)
        got_any += 1
    assert got_any == 5


def test_stage_factors_limit():
    # The stage bullets (inferensys legal and genomic pages): up to 4x for
    # ZeRO-1, up to 8x for ZeRO-2, N x for ZeRO-3, relative to plain DP.
    psi = 1e9
    dp = O.model_state_bytes(0, psi, 1)
    big = 1e12
    assert abs(dp / O.model_state_bytes(1, psi, big) - 4) < 1e-6
    assert abs(dp / O.model_state_bytes(2, psi, big) - 8) < 1e-6
    for N in (2, 8, 64, 1000):
        assert abs(dp / O.model_state_bytes(3, psi, N) - N) < 1e-9
        # stages are monotone and a single rank gains nothing
        assert dp > O.model_state_bytes(1, psi, N) > O.model_state_bytes(2, psi, N) > O.model_state_bytes(3, psi, N)
    for stage in range(4):
        assert O.model_state_bytes(stage, psi, 1) == dp


def test_optimizer_state_divided_by_degree():
    # ZeRO-1 "Memory Reduction" (inferensys instruction-tuning page): the
    # optimizer state alone shrinks by the data-parallel degree (8x on 8 GPUs).
    psi = 3e9
    opt_dp = O.model_state_bytes(0, psi, 1) - O.model_state_bytes(1, psi, 1e30)
    opt_z1 = O.model_state_bytes(1, psi, 8) - O.model_state_bytes(1, psi, 1e30)
    assert abs(opt_dp / opt_z1 - 8) < 1e-9


def test_ten_billion_needs_eleven_ranks_under_15GB():
    # 10B at ZeRO-3: 160 GB / N < 15 GB  <=>  N >= 11
    assert O.model_state_bytes(3, 10e9, 10) >= 15e9
    assert O.model_state_bytes(3, 10e9, 11) < 15e9
