"""Run a cross-section of the hot path through the bounds-checking debug
build of the library (selected with ZERO_B200_LIB), comparing each step with
the oracle, then print the debug build's record of skipped out-of-range
accesses as one JSON line. Launched by tests/test_gpu_debug_bounds.py."""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(HERE))
sys.path.insert(0, HERE)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import oracle as O  # noqa: E402
import zero_partitioned_mixed_reduce_b200 as Z  # noqa: E402
from gpu_harness import Case  # noqa: E402


def main():
    assert os.environ.get("ZERO_B200_LIB"), "run with ZERO_B200_LIB pointing at the debug build"
    count, _, _ = Z.zero_debug_bounds(reset=True)
    assert count == 0, "expected the debug build (the release build reports -1)"
    numels = [70_001, 13, 4096, 7, 999, 3]
    layers = [0, 0, 1, 1, 2, 2]
    runs = 0
    for R in (1, 2, 3, 4, 8, 16):
        for path, mode, dtype in (("pingpong", O.SCALE_DYNAMIC, O.FP16), ("inplace", O.SCALE_NONE, O.BF16),
                                  ("twopass", O.SCALE_STATIC, O.FP16), ("twopass_pp", O.SCALE_DYNAMIC, O.FP16),
                                  ("fused_acc", O.SCALE_DYNAMIC, O.FP16)):
            c = Case(numels, R, dtype, 8 if R != 3 else 1, mode, init_scale=256.0, interval=2, path=path,
                     bucket_elems=5000, layer_ids=layers, seed=R)
            try:
                if path in ("pingpong", "inplace"):
                    c.step()
                    c.step_fused_ex(1.0, 1e-3)  # clipping on the fused path
                elif path == "fused_acc":
                    c.step_fused_accum(3, 3.0)
                else:
                    c.step_ex(2, 2.0, 1e-3)
                    c.compare()
                    c.step_ex(2, 2.0, 1e-3, rs_norm=True)  # the norm from the reduce-scatters
                    c.compare()
                    c.step_ex(1, 1.0, 1e-3, rs_norm=True, whole=True)
                c.compare()
                splits = [(o, o + 1) for o in range(R)]
                if path == "fused_acc":
                    c.step_sharded_ex(splits, 2, 2.0)
                else:
                    c.step_sharded_ex(splits, 1 if not path.startswith("twopass") else 2, 1.0, 1e-3)
                c.compare()
                outs = [torch.empty(hi - lo, dtype=torch.int16, device="cuda") for lo, hi in c.lay.layers]
                Z.zero_gather_layers(c.ctx, 0, outs, c.handle)
                torch.cuda.synchronize()
                runs += 1
            finally:
                c.close()
    # the static-scratch step (zero_step_noalloc): R = 3 with packed tensors
    # and a skipped step, and R = 16
    for R, align, mode, dtype in ((3, 1, O.SCALE_DYNAMIC, O.FP16), (16, 8, O.SCALE_STATIC, O.BF16)):
        c = Case(numels, R, dtype, align, mode, init_scale=256.0, interval=2, path="inplace",
                 layer_ids=layers, seed=R + 100)
        try:
            for s in range(3):
                c.step_noalloc(inject=[(1, 5, 0x7C00)] if (s == 1 and mode == O.SCALE_DYNAMIC) else None)
                c.compare(fsm=c.noalloc_ls)
            runs += 1
        finally:
            c.close()
    # the parameter push (fused ping-pong and two-pass), R = 3 with packed tensors
    for path in ("pingpong", "twopass"):
        c = Case(numels, 3, O.FP16, 1, O.SCALE_STATIC, init_scale=64.0, path=path, layer_ids=layers, seed=300)
        try:
            full = [[c.g.half(c.plan.T, c.dtype) for _ in range(c.R)] for _ in range(c.sets)]
            Z.zero_ctx_set_param_push(c.ctx, full[0], full[1] if c.sets == 2 else None)
            for _ in range(2):
                c.step_no += 1
                g = c.make_grads()
                for r in range(c.R):
                    gp = np.zeros(c.plan.T, np.uint16)
                    gp[c.idx] = g[r]
                    c.grads[r].view(torch.int16).copy_(torch.from_numpy(gp.view(np.int16)))
                if path == "twopass":
                    Z.zero_reduce_scatter_bucket(c.ctx, -1, c.grads, c.acc)
                Z.zero_step_ex(c.ctx, c.hp, c.handle, c.grads if path == "pingpong" else None,
                               flags=Z.ZERO_STEP_PUSH_PARAMS)
                O.step(c.ostate, g, O.AdamW(**{k: c.hp[k] for k in ("lr", "beta1", "beta2", "eps",
                                                                    "weight_decay")}), c.ofsm)
                c.g.check()
                c.compare()
            cur = c.gpu_fsm()["cur"] if c.sets == 2 else 0
            want = np.zeros(c.plan.T, np.uint16)
            want[c.idx] = c.ostate.param
            from gpu_harness import u16
            assert all(np.array_equal(u16(full[cur][r]), want) for r in range(c.R))
            runs += 1
        finally:
            c.close()
    count, site, index = Z.zero_debug_bounds()
    print(json.dumps({"cases": runs, "count": count, "first_site": site, "first_index": index}))


if __name__ == "__main__":
    main()
