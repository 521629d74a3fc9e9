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
