"""The multi-GPU path shards by image with no data exchange; its host logic
(image shards, per-rank coding, max-over-ranks timing, the sharded
container's index) runs here as two gloo ranks on the CPU, coding with the
oracle."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import oracle as O
import workloads as WL
from rans_entropy_coding_b200 import shard


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ids = bench.shard_images(rank, images=1)
        w = WL.y_batch(n_images=1, first_image=ids[0], cg=4, th=64, tw=64)
        c, l, o = O.build_cdfs_from_scales(w["scales"], w["tail_mass"])
        sym = np.asarray(w["symbols"]).reshape(-1)
        streams = list(range(8))            # a few streams of this rank's image
        data, offs = O.encode_with_indexes(sym, w["indexes"], c, l, o, w["chunking"], W=32,
                                           streams=streams)
        t = float(rank + 1)                  # a per-rank "time"
        tmax = bench.max_over_ranks(t, world)
        gathered = [None] * world
        dist.all_gather_object(gathered, (ids, int(sym.sum()), data.tobytes()[:64]))
        # the sharded container: rank r codes 8 + r streams of its image
        offs = O.encode_with_indexes(sym, w["indexes"], c, l, o, w["chunking"], W=32,
                                     streams=list(range(8 + rank)))[1]
        gidx, base, counts = shard.global_index(torch.from_numpy(offs.astype(np.int64)))
        streams_data = O.encode_with_indexes(sym, w["indexes"], c, l, o, w["chunking"], W=32,
                                             streams=list(range(8 + rank)))[0]
        got = shard.gather_container(torch.from_numpy(streams_data.copy()),
                                     torch.from_numpy(offs.astype(np.int64)), dst=0)
        whole = None if got is None else (got[0].numpy().tobytes(), got[1].numpy().tolist())
        out[rank] = (tmax, gathered, gidx.numpy().tolist(), base, counts,
                     offs.astype(np.int64).tolist(), whole, streams_data.tobytes())
    finally:
        dist.destroy_process_group()


def test_two_ranks_shard_by_image():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 2.0                     # max over ranks
    shards = [g[0] for g in res[0][1]]
    assert shards == [[0], [1]]                              # disjoint, covering
    # each rank coded its own image: different data, different streams
    assert res[0][1][0][1] != res[0][1][1][1]
    assert res[0][1][0][2] != res[0][1][1][2]
    # rank 1's shard equals image 1 of a two-image batch coded in one process
    w = WL.y_batch(n_images=2)
    assert int(np.asarray(w["symbols"])[1].sum()) == res[0][1][1][1]


def test_sharded_container_index():
    """Each rank keeps its own streams' bytes; the all-gathered index places
    rank 1's streams after rank 0's, as one container of both."""
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    g0, g1 = res[0][2], res[1][2]
    assert g0 == g1                                          # every rank has the index
    o0, o1 = res[0][5], res[1][5]
    assert res[0][4] == [8, 9] and len(g0) == 8 + 9 + 1
    assert res[0][3] == 0 and res[1][3] == o0[-1]            # rank bases
    assert g0 == o0 + [v + o0[-1] for v in o1[1:]]


def test_gathered_container_is_both_ranks_bytes_in_rank_order():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[1][6] is None                                 # only the destination gets it
    data, offsets = res[0][6]
    assert data == res[0][7] + res[1][7]
    assert offsets == res[0][2]



def _sweep_rank(rank, world, port, out):
    """Rank ``rank`` codes its stream block of a small sweep with the oracle
    and joins the container index."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = bench.shard_streams(WL.sweep(log2_n=16, n_streams=7), world, rank)
        c, l = O.build_cdfs_from_pmfs(w["pmfs"], w["pmf_lengths"], w["tail"])
        data, offs = O.encode_with_indexes(w["symbols"], w["indexes"], c, l, w["offsets"],
                                           w["chunking"], W=32, index_block=w["index_block"])
        gidx, base, counts = shard.global_index(torch.from_numpy(offs.astype(np.int64)))
        out[rank] = (w["stream_block"], w["chunking"]["kind"], gidx.numpy().tolist(), base,
                     counts, data.tobytes())
    finally:
        dist.destroy_process_group()


def test_two_ranks_split_the_sweep_by_stream_range():
    """The sweep split by stream range: rank 0 codes streams 0-3 and rank 1
    streams 4-6 (stream 4 starts inside an index block and the last stream
    is short, so rank 1 reads from the block's start and needs explicit
    boundaries); the all-gathered index and the ranks' bytes in rank order
    are the container one process codes from the whole sweep."""
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_sweep_rank, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    n = 1 << 16
    assert res[0][0] == (0, 4, n, 7) and res[1][0] == (4, 3, n, 7)
    assert res[0][1] == "contig" and res[1][1] == "explicit"
    assert res[0][2] == res[1][2] and res[0][4] == [4, 3]
    w = WL.sweep(log2_n=16, n_streams=7)
    c, l = O.build_cdfs_from_pmfs(w["pmfs"], w["pmf_lengths"], w["tail"])
    data, offs = O.encode_with_indexes(w["symbols"], w["indexes"], c, l, w["offsets"],
                                       w["chunking"], W=32, index_block=w["index_block"])
    assert res[0][2] == offs.astype(np.int64).tolist()
    assert res[1][3] == int(offs[4])
    assert res[0][5] + res[1][5] == data.tobytes()
