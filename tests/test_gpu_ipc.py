"""Buffers shared between processes through CUDA IPC (zero_ipc_export,
zero_ipc_open, zero_ipc_close), the way DistributedZero maps its peers'
gradient replicas and parameter shards. Two processes on one GPU: the
exporter fills a parameter shard that sits at a non-zero offset inside a
larger allocation; the importer maps it and gathers it through the library's
gather kernel, which must copy the exporter's bytes exactly. A second open of
the same handle shares the mapping, closing both unmaps it, and a third close
is refused. No kernel of one process waits on the other: the processes meet
on the host, through queues."""
import multiprocessing as mp
import os
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
N = 100_008  # a multiple of 8


def _pattern(n):
    import torch
    return ((torch.arange(n, dtype=torch.int64) * 7919 + 13) % 65536 - 32768).to(torch.int16)


def _exporter(to_importer, from_importer, res):
    sys.path.insert(0, ROOT)
    import torch
    import zero_partitioned_mixed_reduce_b200 as Z
    torch.cuda.set_device(0)
    big = torch.zeros(1 << 20, dtype=torch.int16, device="cuda")  # the allocation holds more
    shard = big[4096:4096 + N]  # 8192 bytes in
    shard.copy_(_pattern(N).cuda())
    torch.cuda.synchronize()
    blob = Z.zero_ipc_export(shard)
    offset = int.from_bytes(blob[64:72], "little", signed=True)
    alloc = int.from_bytes(blob[72:80], "little", signed=True)
    res.put(("exporter", offset % 16 == 0 and offset >= 8192 and alloc >= offset + 2 * N))
    to_importer.put(blob)
    from_importer.get(timeout=180)  # the importer has unmapped: the buffer may go
    del shard, big


def _importer(from_exporter, to_exporter, res):
    sys.path.insert(0, ROOT)
    import torch
    import zero_partitioned_mixed_reduce_b200 as Z
    torch.cuda.set_device(0)
    blob = from_exporter.get(timeout=180)
    ok = False
    try:
        ptr = Z.zero_ipc_open(blob)
        same = Z.zero_ipc_open(blob) == ptr  # one mapping per allocation
        plan = Z.Plan([N], None, 1, Z.ZERO_BF16, 8, 0)
        ctx = Z.zero_ctx_create(plan.handle)
        handle = Z.StateHandle([dict(master=[None], m=[None], v=[None], param=[ptr])])
        out = torch.empty(N, dtype=torch.bfloat16, device="cuda")
        Z.zero_gather_layer(ctx, 0, handle, out)
        torch.cuda.synchronize()
        equal = torch.equal(out.view(torch.int16).cpu(), _pattern(N))
        Z.zero_ctx_destroy(ctx)
        Z.zero_ipc_close(blob)
        Z.zero_ipc_close(blob)
        try:
            Z.zero_ipc_close(blob)
            refused = False
        except Z.ZeroError as e:
            refused = e.status == Z.ZERO_ERR_STATE
        ok = same and equal and refused
    finally:
        res.put(("importer", ok))
        to_exporter.put("done")


def test_two_processes_share_a_shard_through_ipc():
    ctx = mp.get_context("spawn")
    a2b, b2a, res = ctx.Queue(), ctx.Queue(), ctx.Queue()
    pa = ctx.Process(target=_exporter, args=(a2b, b2a, res))
    pb = ctx.Process(target=_importer, args=(a2b, b2a, res))
    pa.start()
    pb.start()
    pb.join(240)
    pa.join(240)
    for p in (pa, pb):
        if p.is_alive():
            p.kill()
    assert pa.exitcode == 0 and pb.exitcode == 0
    got = dict(res.get(timeout=10) for _ in range(2))
    assert got == {"exporter": True, "importer": True}
