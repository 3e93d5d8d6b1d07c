"""Pin the oracle's loss-scale state machine against hand-written sequences
(tests/golden/fsm_sequences.txt), and the skip semantics of a whole step."""
import os

import numpy as np

import oracle as O

MODES = {"NONE": O.SCALE_NONE, "STATIC": O.SCALE_STATIC, "DYNAMIC": O.SCALE_DYNAMIC}


def parse(path):
    seqs, cur = [], None
    for line in open(path):
        line = line.split("#")[0].strip()
        if not line:
            continue
        tok = line.split()
        if tok[0] == "seq":
            cur = dict(name=tok[1], mode=MODES[tok[2]], init=float(tok[3]),
                       interval=int(tok[4]), min_scale=float(tok[5]), ovf=set(), rows=[])
        elif tok[0] == "ovf":
            cur["ovf"] = {int(x) for x in tok[1:]}
        elif tok[0] == "end":
            seqs.append(cur)
        else:
            cur["rows"].append([float(x) for x in tok])
    return seqs


def test_sequences(golden_dir):
    seqs = parse(os.path.join(golden_dir, "fsm_sequences.txt"))
    assert len(seqs) == 4
    for s in seqs:
        fsm = O.make_fsm(s["mode"], scale=s["init"], interval=s["interval"],
                         min_scale=s["min_scale"])
        want = {int(r[0]): r for r in s["rows"]}
        last = max(want)
        for step in range(1, last + 1):
            skipped = O.fsm_update(fsm, step in s["ovf"])
            if step in want:
                _, ovf, skp, scale, good, t = want[step]
                got = (fsm.last_overflow, int(skipped), fsm.last_skipped, fsm.scale, fsm.good, fsm.t)
                assert got == (ovf, skp, skp, scale, good, t), (s["name"], step, got)


def test_skipped_step_leaves_state_untouched():
    rng = np.random.default_rng(1)
    P, R = 300, 4
    x = rng.normal(0, 0.02, P).astype(np.float32)
    st = O.State(x, O.FP16)
    fsm = O.make_fsm(O.SCALE_DYNAMIC, scale=1024.0, interval=100)
    g = O.float_to_half((rng.normal(0, 1e-3, (R, P)) * 1024).astype(np.float32), O.FP16)
    O.step(st, g, O.AdamW(1e-3, 0.9, 0.999, 1e-8, 0.01), fsm)
    before = st.copy()
    g2 = g.copy()
    g2[2, 17] = 0x7C00  # +inf in one replica
    skipped = O.step(st, g2, O.AdamW(1e-3, 0.9, 0.999, 1e-8, 0.01), fsm)
    assert skipped and fsm.last_overflow == 1 and fsm.t == 1 and fsm.scale == 512.0
    for a in ("master", "m", "v", "param"):
        assert np.array_equal(getattr(st, a), getattr(before, a))
    assert not np.isfinite(fsm.grad_norm_sq)


def test_nan_and_sum_overflow_count_as_overflow():
    # a NaN replica value, and two finite bf16 values whose fp32 sum overflows
    big = O.float_to_half(np.array([3.0e38], np.float32), O.BF16)[0]
    g = np.zeros((2, 4), np.uint16)
    g[0, 1] = big
    g[1, 1] = big
    acc, ovf = O.allreduce_sum(g, O.BF16)
    assert ovf and np.isinf(acc[1])
    g = np.zeros((3, 4), np.uint16)
    g[1, 3] = 0x7E00  # fp16 NaN
    acc, ovf = O.allreduce_sum(g, O.FP16)
    assert ovf and np.isnan(acc[3])
    g = np.zeros((3, 4), np.uint16)
    acc, ovf = O.allreduce_sum(g, O.FP16)
    assert not ovf
