"""A container sharded over ranks: every rank codes its own streams (images;
streams never cross an image, so coding needs no exchange -- "kompressor"
README, Why: no cross-chunk dependency) and keeps its bytes; one all-gather
of the ranks' stream offsets gives every rank the global index of the
container that the concatenation of all ranks' bytes (rank order) forms.

The only collective is that all-gather of (S_r + 1) uint64 offsets per
rank; it runs on whatever backend the process group has (NCCL on GPUs,
gloo in the CPU tests).  Payload never moves between ranks here: a rank
that writes the container at byte ``base`` needs only its own bytes.
"""
import torch
import torch.distributed as dist


def global_index(local_offsets, group=None):
    """local_offsets: this rank's int64 tensor of S_r + 1 stream offsets
    (offsets[0] = 0, offsets[S_r] = the rank's byte total), as the encoders
    return them.  Returns (global_offsets, base, counts): the int64 offsets
    of all ranks' streams in rank order (sum(S_r) + 1 entries, on the
    offsets' device), this rank's first byte in the container, and each
    rank's stream count."""
    world = dist.get_world_size(group)
    dev = local_offsets.device
    n_local = torch.tensor([local_offsets.numel() - 1], dtype=torch.int64, device=dev)
    counts = [torch.zeros_like(n_local) for _ in range(world)]
    dist.all_gather(counts, n_local, group=group)
    counts = [int(c.item()) for c in counts]
    width = max(counts) + 1
    padded = torch.zeros(width, dtype=torch.int64, device=dev)
    padded[:local_offsets.numel()] = local_offsets
    parts = [torch.zeros_like(padded) for _ in range(world)]
    dist.all_gather(parts, padded, group=group)
    out, base, run = [torch.zeros(1, dtype=torch.int64, device=dev)], 0, 0
    me = dist.get_rank(group)
    for r in range(world):
        offs = parts[r][:counts[r] + 1]
        if r == me:
            base = run
        out.append(offs[1:] + run)
        run += int(offs[counts[r]].item())
    return torch.cat(out), base, counts


def gather_container(data, local_offsets, dst=0, group=None):
    """The other exchange the sharded container allows: every rank's bytes
    sent to rank ``dst`` (point to point, rank order), which returns
    (data, global_offsets) of the whole container; the other ranks return
    None.  data: this rank's uint8 tensor of at least local_offsets[-1]
    bytes, on the device the process group moves."""
    gidx, base, counts = global_index(local_offsets, group)
    me, world = dist.get_rank(group), dist.get_world_size(group)
    mine = int(local_offsets[-1].item())
    if me != dst:
        if mine:
            dist.send(data[:mine].contiguous(), dst=dst, group=group)
        return None
    total = int(gidx[-1].item())
    out = torch.empty(total, dtype=torch.uint8, device=data.device)
    bounds, run = [], 0
    ends = gidx.tolist()
    first = 0
    for r in range(world):
        n_r = counts[r]
        size = int(ends[first + n_r]) - int(ends[first])
        bounds.append((run, size))
        run += size
        first += n_r
    for r in range(world):
        start, size = bounds[r]
        if size == 0:
            continue
        if r == me:
            out[start:start + size] = data[:size]
        else:
            dist.recv(out[start:start + size], src=r, group=group)
    return out, gidx


def stream_block(n, n_streams, world, rank, index_block=1):
    """Rank ``rank``'s share of a contiguous chunking of n elements into
    n_streams streams (stream k covers [k*per, min((k+1)*per, n)),
    per = ceil(n / n_streams)): a contiguous block of whole streams, the
    blocks of ranks 0 .. world-1 covering all streams in order, their sizes
    differing by at most one stream.  Streams are independent ("kompressor"
    README, Why), so each rank codes its block with no exchange and the
    ranks' bytes in rank order are the single-GPU container.

    Returns a dict: ``first`` and ``count`` (the rank's streams),
    ``elems`` (the element range [a0, b) the rank reads: its streams' range
    [a, b) widened down to the start of the index block holding a, so that
    its row indexes are a plain slice), ``index_range`` ([a0 // index_block,
    ceil(b / index_block))) and ``chunking`` (the rank's chunking of its
    b - a0 elements: contiguous when that reproduces the global stream
    boundaries, else explicit with those boundaries)."""
    if n_streams < 1 or world < 1 or not 0 <= rank < world or index_block < 1:
        raise ValueError("bad stream block request")
    per = -(-n // n_streams) if n else 0
    base, extra = divmod(n_streams, world)
    first = rank * base + min(rank, extra)
    count = base + (1 if rank < extra else 0)
    a = min(first * per, n)
    b = min((first + count) * per, n)
    a0 = a - a % index_block
    bounds = [min((first + k) * per, n) - a0 for k in range(count + 1)]
    local_per = -(-(b - a0) // count) if count else 0
    if count and a0 == a and all(min(k * local_per, b - a) == bounds[k]
                                 for k in range(count + 1)):
        chunking = dict(kind="contig", n_streams=count)
    else:
        chunking = dict(kind="explicit", starts=bounds)
    return dict(first=first, count=count, elems=(a0, b),
                index_range=(a0 // index_block, -(-b // index_block)), chunking=chunking)
