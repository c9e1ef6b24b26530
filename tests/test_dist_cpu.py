"""The one exchange step of the sharded NVFP4 path, on 2 CPU ranks (gloo).

Each rank holds row shards of two sibling groups, reduces its shard amax with
the oracle, and all-reduces the vector of group amaxes with the library's
helper.  The result must be the oracle amax of the unsharded groups on both
ranks, and the oracle quantisation of each shard with it must equal the
matching rows of the unsharded quantisation (max is exact and order-free).
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

GROUPS = [[(96, 64), (40, 64)], [(130, 32)]]   # ragged row counts: uneven shards


def _port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    import torch
    import torch.distributed as dist
    from oracle import oracle as O
    import workloads as W
    from precision_weight_quantization_b200.dist import allreduce_group_amax, row_shard

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        full = [[W.bits(W.random_bf16(s, seed=900 + 10 * g + i, std=0.5)) for i, s in enumerate(grp)]
                for g, grp in enumerate(GROUPS)]
        full[1][0][7, 3] = 0x4480   # a large value on rank 0's rows only
        shards = [[row_shard(torch.from_numpy(x.astype(np.int32)), rank, world).numpy().astype(np.uint16)
                   for x in grp] for grp in full]
        local = torch.tensor([np.float32(O.nvfp4_group_amax([s for s in grp if s.size])) if any(s.size for s in grp)
                              else np.float32(0) for grp in shards], dtype=torch.float32)
        glob = allreduce_group_amax(local.clone())
        ok = True
        for g, grp in enumerate(full):
            A = np.float32(O.nvfp4_group_amax(grp))
            ok &= bool(np.float32(glob[g].item()) == A)
            for x, s in zip(grp, shards[g]):
                if s.size == 0:
                    continue
                pk_full, sb_full, _ = O.nvfp4_quant(x, A)
                pk, sb, _ = O.nvfp4_quant(s, np.float32(glob[g].item()))
                r0 = row_shard(torch.arange(x.shape[0])[:, None], rank, world)[0, 0].item()
                ok &= bool(np.array_equal(pk, pk_full[r0:r0 + s.shape[0]]))
                ok &= bool(np.array_equal(sb, sb_full[r0:r0 + s.shape[0]]))
        with open(os.path.join(out_dir, "rank%d" % rank), "w") as f:
            f.write("ok" if ok else "mismatch")
    finally:
        dist.destroy_process_group()


def test_sharded_group_amax_two_ranks(tmp_path):
    sys.path.insert(0, ROOT)
    import __graft_entry__
    __graft_entry__._load_build_script().build()   # once, before the ranks import the package
    ctx = mp.get_context("spawn")
    port = _port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, str(tmp_path))) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(300)
        assert p.exitcode == 0
    for r in range(2):
        assert (tmp_path / ("rank%d" % r)).read_text() == "ok", r


def test_row_shard_covers_rows_once():
    import torch
    sys.path.insert(0, ROOT)
    from precision_weight_quantization_b200.dist import row_shard
    for M in (1, 5, 127, 128, 129, 1000):
        for world in (1, 2, 3, 8):
            for mult in (1, 128):
                x = torch.arange(M)[:, None]
                parts = [row_shard(x, r, world, mult) for r in range(world)]
                got = torch.cat(parts).flatten().tolist()
                assert got == list(range(M))
                for p in parts[:-1]:
                    if p.shape[0] and mult > 1:
                        assert p[0, 0].item() % mult == 0
