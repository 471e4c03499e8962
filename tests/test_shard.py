"""The (stream, head) partition of a layer over ranks, on CPU.

Streams and heads are independent in every step of the layer, so a partition is correct when
its shards cover every (stream, head) pair exactly once; and because the method's result for one
pair depends on that pair's rows only, per-rank results reassemble into the single-process
result bit for bit.  The second part runs two gloo ranks, each feeding its shard's rows to the
oracle, and compares the reassembled output with the oracle run on the whole layer in one
process."""
import os
import socket

import numpy as np
import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

from causal_video_diffusion_b200 import shard as S


@pytest.mark.parametrize("B,H", [(1, 12), (4, 12), (2, 3), (3, 5), (8, 1), (1, 1)])
@pytest.mark.parametrize("world", [1, 2, 3, 4, 6, 8])
def test_shards_cover_every_stream_head_once(B, H, world):
    if world > B * H:
        with pytest.raises(ValueError):
            S.plan(B, H, world)
        return
    shards = S.plan(B, H, world)
    assert len(shards) == world
    cells = [c for sh in shards for c in sh.cells()]
    assert sorted(cells) == [(b, h) for b in range(B) for h in range(H)]
    assert len(cells) == len(set(cells))
    for sh in shards:
        assert sh.nb >= 1 and sh.nh >= 1
        assert 0 <= sh.b0 and sh.b0 + sh.nb <= B and 0 <= sh.h0 and sh.h0 + sh.nh <= H
        # streams first: a rank holds whole streams, or part of exactly one stream
        assert sh.nh == H or sh.nb == 1


def test_streams_go_whole_before_heads_split():
    assert S.plan(4, 12, 4) == [S.Shard(b, 1, 0, 12) for b in range(4)]
    assert S.plan(4, 12, 2) == [S.Shard(0, 2, 0, 12), S.Shard(2, 2, 0, 12)]
    assert S.plan(1, 12, 8) == [S.Shard(0, 1, 0, 2), S.Shard(0, 1, 2, 2), S.Shard(0, 1, 4, 2),
                                S.Shard(0, 1, 6, 2), S.Shard(0, 1, 8, 1), S.Shard(0, 1, 9, 1),
                                S.Shard(0, 1, 10, 1), S.Shard(0, 1, 11, 1)]
    # 6 ranks over 4 streams: two streams split in two, two whole
    assert S.plan(4, 12, 6) == [S.Shard(0, 1, 0, 6), S.Shard(0, 1, 6, 6), S.Shard(1, 1, 0, 6),
                                S.Shard(1, 1, 6, 6), S.Shard(2, 1, 0, 12), S.Shard(3, 1, 0, 12)]


def test_split_is_contiguous_and_balanced():
    for n in range(1, 40):
        for k in range(1, n + 1):
            parts = S.split(n, k)
            assert parts[0][0] == 0
            assert all(a + c == b for (a, c), (b, _) in zip(parts, parts[1:]))
            assert sum(c for _, c in parts) == n
            assert max(c for _, c in parts) - min(c for _, c in parts) <= 1
    with pytest.raises(ValueError):
        S.split(2, 3)


# --------------------------------------------------------------------------------------------
# two gloo ranks, each computing its shard with the oracle
# --------------------------------------------------------------------------------------------

CASES = [dict(B=2, H=3), dict(B=1, H=3)]   # a stream split, then a head split


def _layer_inputs(B, H, seed):
    """A tiny layer: D = 64 (24/20/20), 4x6 tokens per frame, three chunks of three frames
    through a six-frame ring (it evicts once)."""
    from causal_video_diffusion_b200 import workloads as W
    shape = W.LayerShape(B=B, H=H, D=64, Hg=4, Wg=6, d_t=24, d_h=20, d_w=20)
    chunks = [W.gen_qkv(W.qkv_seed(seed, chunk=c), shape) for c in range(3)]
    return shape, [tuple(W.bits(t) for t in qkv) for qkv in chunks]


def _oracle_shard(shape, chunks, sh):
    """The last chunk's output rows of one shard, [nb][L][nh][D], from the oracle fed only
    that shard's streams (and keeping only its heads)."""
    import oracle
    ol = oracle.OracleLayer(sh.nb, shape.H, shape.Hg, shape.Wg,
                            oracle.RopeSpec(shape.d_t, shape.d_h, shape.d_w, shape.theta), 6,
                            heads=list(range(sh.h0, sh.h0 + sh.nh)))
    bs = slice(sh.b0, sh.b0 + sh.nb)
    for c, (q, k, v) in enumerate(chunks):
        q_rot = ol.append(q[bs], k[bs], v[bs], 3 * c, 3)
    o = ol.attend(q_rot, 6)                       # rows (b, h, l) in that order
    return o.reshape(sh.nb, sh.nh, shape.L, shape.D).transpose(0, 2, 1, 3)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        for i, case in enumerate(CASES):
            shape, chunks = _layer_inputs(case["B"], case["H"], seed=70 + i)
            sh = S.plan(shape.B, shape.H, world)[rank]
            part = _oracle_shard(shape, chunks, sh)
            got = [None] * world
            dist.all_gather_object(got, (sh, part))
            if rank == 0:
                q.put((i, got))
    finally:
        dist.destroy_process_group()


def test_two_ranks_reassemble_the_single_process_result():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = dict(q.get(timeout=300) for _ in CASES)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    for i, case in enumerate(CASES):
        shape, chunks = _layer_inputs(case["B"], case["H"], seed=70 + i)
        whole = _oracle_shard(shape, chunks, S.Shard(0, shape.B, 0, shape.H))
        out = np.full_like(whole, np.nan)
        seen = np.zeros((shape.B, shape.H), dtype=int)
        for sh, part in results[i]:
            out[sh.b0:sh.b0 + sh.nb, :, sh.h0:sh.h0 + sh.nh] = part
            seen[sh.b0:sh.b0 + sh.nb, sh.h0:sh.h0 + sh.nh] += 1
        assert (seen == 1).all()
        assert np.array_equal(out, whole)          # bit for bit
