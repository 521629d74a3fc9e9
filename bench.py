#!/usr/bin/env python
"""Throughput of librans_b200 on the 16-image 1080p latent batch.

One step = the whole coding path over one batch: the 64 Gaussian CDF rows
built from the scale table, the coder's tables rebuilt from them, every
stream encoded (with compaction) and decoded, on one GPU per rank.  Workload: 16 synthetic
y latents [16, 192, 68, 120] int32 (25,067,520 symbols), one stream per
64 x 64 spatial tile per group of 4 channels (3,072 streams), 32 interleaved
states per stream.  Ranks shard by image (weak scaling: every rank codes its
own 16 images; no collective on the data path).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

--workload picks one of the other synthetic configurations instead (one
GPU, for the per-configuration table): tiny (4,096 int32, 8 rows, W=1),
z (128x17x30 int32, 128 pmf rows, 32 contiguous streams, W=1),
y (192x68x120 int32, 24 contiguous streams, --interleave 1 or 32) and
sweep (2^28 uint8, 16 Zipf rows, one index per 4,096 symbols, 8,192
streams, W=32) and float (the batch as float latents: y, means and scales
per element in, rows and symbols computed inside the coders, float values
out).

Prints one JSON line (rank 0).  Inputs (200 MB of symbols and indexes) are
larger than the 126 MB L2, so no flush is needed between steps.
"""
import argparse
import concurrent.futures as cf
import json
import os
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as WL  # noqa: E402

METRIC = ("rANS encode & decode Gsymbol/s and HBM GB/s (fraction of B200 roofline), 1 GPU")
UNIT = "Gsymbol/s"
WORKLOAD = "batch16_y1080p: 16x192x68x120 int32, 64 Gaussian rows, tiles 64x64 x 4 channels, W=32"
N_IMAGES = 16
CLOCK_FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--group", type=int, default=4, help="channels per stream")
    ap.add_argument("--images", type=int, default=N_IMAGES, help="images per GPU")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--traffic-file", default=os.path.join(ROOT, "profiles", "dram_traffic.txt"))
    ap.add_argument("--workload", choices=["batch", "tiny", "z", "y", "sweep", "float", "r16"],
                    default="batch")
    ap.add_argument("--interleave", type=int, default=None, help="W for --workload y")
    ap.add_argument("--log2n", type=int, default=28,
                    help="--workload sweep: 2^log2n symbols (28 is the configuration; smaller "
                         "sizes serve profiling)")
    ap.add_argument("--format", choices=["rans64", "rans32_16"], default=None,
                    help="coder format (default: rans32_16 for --workload r16, else rans64)")
    ap.add_argument("--alias", action="store_true",
                    help="alias-coded streams (rows of power-of-two bucket counts, W <= 8)")
    ap.add_argument("--eager", action="store_true",
                    help="call the entry points every step instead of replaying the step "
                         "(its phases and their timing events) from a CUDA graph")
    return ap.parse_args()


# The sources the measured coders (encode_kernel, decode_kernel and the
# compaction kernels) are compiled from.
MEASURED_SOURCES = ("rans_entropy_coding_b200/csrc/encode.cu",
                    "rans_entropy_coding_b200/csrc/decode.cu",
                    "rans_entropy_coding_b200/csrc/rans_common.cuh",
                    "rans_entropy_coding_b200/csrc/rans_internal.h",
                    "include/rans_b200.h")


def kernel_sources_digest():
    """sha256 over the coders' CUDA sources, so a DRAM-traffic figure taken
    with ncu is only reported while the kernels it measured are unchanged."""
    import hashlib
    h = hashlib.sha256()
    for rel in MEASURED_SOURCES:
        h.update(os.path.basename(rel).encode())
        h.update(open(os.path.join(ROOT, rel), "rb").read())
    return h.hexdigest()


def measured_traffic(path, kernel, workload):
    """Per-launch dram__bytes_read.sum + dram__bytes_write.sum for `kernel`
    from the committed ncu summary, or None when the summary is missing, was
    taken on another workload or on other kernel sources."""
    if not os.path.exists(path):
        return None
    kv = {}
    for line in open(path):
        if ":" in line and not line.startswith("#"):
            k, v = line.split(":", 1)
            kv[k.strip()] = v.strip()
    if kv.get("workload") != workload or kv.get("sources_sha256") != kernel_sources_digest():
        return None
    v = kv.get(kernel + "_bytes_per_launch")
    return int(v) if v else None


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        backend = "gloo" if args.impl == "reference" else "nccl"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v, world, device=None):
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while running."""

    def __init__(self, gpu_index, enabled=True):
        self.gpu = gpu_index
        self.enabled = enabled
        self.proc = None

    def __enter__(self):
        if self.enabled:
            self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            try:
                self.proc = subprocess.Popen(
                    ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + CLOCK_FIELDS,
                     "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.f,
                    stderr=subprocess.DEVNULL)
                time.sleep(0.3)
            except OSError:
                self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None:
            return None
        self.f.flush()
        rows = []
        with open(self.f.name) as fh:
            for line in fh:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.f.name)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        return {"sm_mhz": float(np.median(sm)) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


def shard_images(rank, images=N_IMAGES):
    """Image ids coded by `rank`: every rank codes its own `images` images
    (weak scaling; streams never cross images, so no exchange is needed)."""
    return list(range(images * rank, images * (rank + 1)))


def shard_streams(w, world, rank):
    """Rank ``rank``'s block of a contiguously chunked workload (the sweep):
    a contiguous range of whole streams with its symbols and row indexes
    (strong scaling: the ranks split one fixed workload; streams are
    independent, so no exchange is needed).  Returns the rank's workload dict
    with "stream_block" = (first stream, count, global symbol count, global
    stream count)."""
    from rans_entropy_coding_b200 import shard
    sym = np.asarray(w["symbols"]).reshape(-1)
    blk = int(w["index_block"])
    b = shard.stream_block(sym.size, int(w["chunking"]["n_streams"]), world, rank, blk)
    (a, e), (i0, i1) = b["elems"], b["index_range"]
    return dict(w, symbols=sym[a:e], indexes=np.asarray(w["indexes"])[i0:i1],
                chunking=b["chunking"],
                stream_block=(b["first"], b["count"], sym.size, int(w["chunking"]["n_streams"])))


def load_inputs(rank, group, images=N_IMAGES, workload="batch", interleave=None, world=1,
                log2n=28):
    if workload == "tiny":
        w = WL.tiny()
    elif workload == "z":
        w = WL.z_latent()
    elif workload == "y":
        w = WL.y_latent(W=interleave or 32)
    elif workload == "sweep":
        w = WL.sweep(log2_n=log2n)
        if world > 1:  # split by stream range
            w = shard_streams(w, world, rank)
    elif workload == "r16":
        w = WL.r16_rows()
    elif workload == "float":
        ids = shard_images(rank, images)
        w = WL.y_float(seed=6000 + ids[0], n_images=len(ids), cg=group)
    else:
        ids = shard_images(rank, images)
        w = WL.y_batch(n_images=len(ids), first_image=ids[0], cg=group)
        w["W"] = 32
    if interleave is not None:
        w["W"] = interleave
    return w


def apply_format(w, fmt, alias=False):
    """Sets the coder format (and its row precision) on a workload dict."""
    fmt = fmt or w.get("fmt", "rans64")
    w["fmt"] = fmt
    w["precision"] = 15 if fmt == "rans32_16" else 16
    w["alias"] = bool(alias)
    return w


def workload_name(w, args):
    if w.get("fmt", "rans64") != "rans64" or w.get("alias"):
        return "%s [%s%s, precision %d]" % (
            workload_name(dict(w, fmt="rans64", alias=False), args), w["fmt"],
            " alias" if w.get("alias") else "", w["precision"])
    if args.workload == "batch":
        return WORKLOAD if w["W"] == 32 else WORKLOAD.replace("W=32", "W=%d" % w["W"])
    if args.workload == "float":
        return ("float_batch%d: %dx192x68x120 float32 y, means and scales per element, "
                "64-entry scale table, tiles 64x64 x %d channels, W=32" %
                (args.images, args.images, args.group))
    n = int(np.asarray(w["symbols"]).size)
    rows = len(w["scales"]) if "scales" in w else len(w["pmf_lengths"])
    n_streams = w["chunking"].get("n_streams", 0)
    split = w.get("stream_block")
    if split:  # the whole workload, then the ranks' split
        n, n_streams = split[2], split[3]
    name = "%s: %d %s symbols, %d %s rows, %s %d streams, W=%d, index block %d" % (
        args.workload, n, np.asarray(w["symbols"]).dtype, rows,
        "Gaussian" if "scales" in w else "pmf", "contig" if split else w["chunking"]["kind"],
        n_streams, w["W"], w["index_block"])
    return name + (", split by stream range over the ranks" if split else "")


# --------------------------------------------------------- CPU oracle leg --
def oracle_sample(w, max_streams, workers):
    """Oracle encode + decode of the first max_streams streams of the
    workload, one stream per call, spread over `workers` threads (the C
    oracle runs without the GIL).  Returns (symbols coded, seconds)."""
    import oracle as O
    fmt, prec, alias = w.get("fmt", "rans64"), w.get("precision", 16), w.get("alias", False)
    if "scales" in w:
        c, l, o = O.build_cdfs_from_scales(w["scales"], w["tail_mass"], precision=prec)
    else:
        c, l = O.build_cdfs_from_pmfs(w["pmfs"], w["pmf_lengths"], w["tail"], precision=prec)
        o = np.asarray(w["offsets"], dtype=np.int32)
    flat = np.asarray(w["symbols"]).reshape(-1)
    pos = O.stream_positions(flat.size, w["chunking"])[:max_streams]
    idx = np.asarray(w["indexes"], dtype=np.int32)
    blk = int(w.get("index_block", 1))
    W = int(w.get("W", 32))

    def one(p):
        s = flat[p].astype(np.int64)
        r = idx[p // blk]
        b = O.encode_stream(s, r, c, l, o, W=W, fmt=fmt, precision=prec, alias=alias)
        back = O.decode_stream(b, r, c, l, o, W=W, fmt=fmt, precision=prec, alias=alias)
        assert np.array_equal(back, s)
        return p.size

    t = time.perf_counter()
    with cf.ThreadPoolExecutor(max_workers=workers) as ex:
        n = sum(ex.map(one, pos))
    return n, time.perf_counter() - t


def run_reference(args, world, rank):
    """--impl reference: the oracle as it stands on the host cores."""
    if rank != 0:
        return
    w = apply_format(load_inputs(0, args.group, workload=args.workload,
                                 interleave=args.interleave, log2n=args.log2n), args.format,
                     args.alias)
    if args.workload == "float":  # the oracle codes rows and symbols computed first
        import oracle as O
        w = dict(w, symbols=O.quantize(w["y"], w["means"]), W=32,
                 indexes=O.build_indexes(w["fscales"], w["scales"],
                                         w["scale_bound"]).reshape(-1))
    workers = os.cpu_count() or 1
    max_streams = 768     # batch: 4 of the 16 images per step, a bounded sample
    for _ in range(args.warmup):
        oracle_sample(w, 48, workers)
    tot_n, tot_t = 0, 0.0
    for _ in range(args.steps):
        n, t = oracle_sample(w, max_streams, workers)
        tot_n += n
        tot_t += t
    value = tot_n / tot_t / 1e9
    sample = ("oracle encode+decode of streams 0..767 (images 0-3, %d symbols) per step, "
              "one stream per call over %d threads" % (tot_n // max(args.steps, 1), workers))
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot_t / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "u64" if w["fmt"] == "rans64" else "u32",
        "data": "synthetic", "config": {"workload": workload_name(w, args),
                                        "streams_per_step": max_streams},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": workers, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


# --------------------------------------------------------------- GPU leg --
def run_ours(args, world, rank, local):
    import torch

    import rans_entropy_coding_b200 as rb

    rb.lib()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    w = apply_format(load_inputs(rank, args.group, args.images, args.workload, args.interleave,
                                 world, args.log2n), args.format, args.alias)
    fmt, prec = w["fmt"], w["precision"]
    sym_np = np.ascontiguousarray(np.asarray(w["symbols"]).reshape(-1))
    idx_np = np.ascontiguousarray(w["indexes"], dtype=np.int32)
    n = sym_np.size
    sym = torch.from_numpy(sym_np).to(dev)
    idx = torch.from_numpy(idx_np).to(dev)
    ch = rb.Chunking.from_spec(w["chunking"], w["W"], w["index_block"], device=dev, fmt=fmt,
                               alias=w["alias"])
    S = rb.rans_num_streams(ch, n)

    # tables: sized once; rebuilt inside every step (from the scale table, or
    # from the pmfs)
    if "scales" in w:
        scales = torch.from_numpy(w["scales"]).to(dev)
        tail = w["tail_mass"]
        cdfs, lengths, offsets = rb.Tables.build_from_scales(scales, tail, precision=prec)

        def build_rows():
            rb.check(rb.rans_build_cdfs_from_scales(scales, tail, cdfs, lengths, offsets,
                                                    precision=prec), "cdfs")

        def rebuild_tables():  # the rows and the prepared tables in one launch
            rb.check(rb.rans_tables_refresh_from_scales(scales, tail, cdfs, lengths, offsets,
                                                        tables), "tables")
    else:
        pmfs = torch.from_numpy(np.ascontiguousarray(w["pmfs"])).to(dev)
        plen = torch.from_numpy(np.asarray(w["pmf_lengths"], np.int32)).to(dev)
        ptail = torch.from_numpy(np.asarray(w["tail"], np.float32)).to(dev)
        cdfs, lengths = rb.Tables.build_from_pmfs(pmfs, plen, ptail, precision=prec)
        offsets = torch.from_numpy(np.asarray(w["offsets"], np.int32)).to(dev)

        def build_rows():
            rb.check(rb.rans_build_cdfs_from_pmfs(pmfs, plen, ptail, cdfs, lengths,
                                                  precision=prec), "cdfs")

        def rebuild_tables():
            build_rows()
            rb.check(rb.rans_tables_refresh(cdfs, lengths, offsets, tables), "refresh")
    K, Lmax = cdfs.shape
    tables = rb.Tables(cdfs, lengths, offsets, precision=prec)
    if w["alias"]:  # built once, before timing: the rows do not change between steps
        tables.prepare_alias()
    blob = tables.blob
    ws = rb.Workspaces(ch, n, dev)
    dec = torch.empty_like(sym)
    stream = torch.cuda.current_stream()
    # inputs smaller than L2: flush it (a 256 MB write) before every step,
    # outside the phase events
    in_bytes = n * (sym.element_size() + 4)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev) if in_bytes < (126 << 20) \
        else None

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]

    def phase_tables():
        rebuild_tables()

    def phase_encode():
        rb.check(rb.rans_encode_with_indexes(sym, idx, n, tables, ch, ws.out, ws.offsets,
                                             ws.enc), "encode")

    def phase_decode():
        rb.check(rb.rans_decode_with_indexes(ws.out, ws.offsets, idx, n, tables, ch, dec,
                                             ws.dec), "decode")

    phases = [phase_tables, phase_encode, phase_decode]

    def step_body(e=None):
        cur = torch.cuda.current_stream()
        if flush is not None:
            flush.fill_(1)
        for k, ph in enumerate(phases):
            if e: e[k].record(cur)
            ph()
        if e: e[3].record(cur)

    for _ in range(max(args.warmup, 0)):
        step_body()
    torch.cuda.synchronize()
    steps = [lambda e=e: step_body(e) for e in ev]
    if not args.eager:
        # a step (the L2 flush if any, then the three phases) captured into
        # one CUDA graph, its phase events recorded as graph nodes between
        # them; one graph per timed step, so that each keeps its own events:
        # a step is one host launch
        ev = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(4)]
              for _ in range(args.steps)]
        cap = torch.cuda.Stream(dev)

        def capture(e):
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr, stream=cap):
                step_body(e)
            return gr

        warm = capture(None)
        graphs = [capture(e) for e in ev]
        steps = [gr.replay for gr in graphs]
        for _ in range(max(args.warmup, 0)):
            warm.replay()
        torch.cuda.synchronize()
    rb.check(rb.rans_get_status(ws.enc), "encode status")
    rb.check(rb.rans_get_status(ws.dec), "decode status")
    rb.check(rb.rans_get_status(blob), "tables status")
    assert torch.equal(dec, sym), "round trip failed"
    barrier(world)

    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with ClockSampler(local, enabled=not args.no_clocks) as clk:
        torch.cuda.synchronize()
        barrier(world)
        t0.record(stream)
        for i in range(args.steps):
            steps[i]()
        t1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
    elapsed_ms = max_over_ranks(t0.elapsed_time(t1), world, dev)
    clocks = clk.summary()
    rb.check(rb.rans_get_status(ws.enc), "encode status")
    rb.check(rb.rans_get_status(ws.dec), "decode status")
    assert torch.equal(dec, sym), "round trip failed"
    # N > 1: the ranks' streams form one sharded container; its index is one
    # all-gather of every rank's stream offsets (after the timed region)
    container = None
    if world > 1:
        from rans_entropy_coding_b200 import shard
        gidx, base, counts = shard.global_index(ws.offsets)
        container = {"streams": int(sum(counts)), "bytes": int(gidx[-1].item()),
                     "rank0_base": base if rank == 0 else None}

    tab_t = [e[0].elapsed_time(e[1]) for e in ev]
    enc_t = [e[1].elapsed_time(e[2]) for e in ev]
    dec_t = [e[2].elapsed_time(e[3]) for e in ev]
    tab_ms, enc_ms, dec_ms = (float(np.mean(t)) for t in (tab_t, enc_t, dec_t))
    comp = int(ws.offsets[-1].item())
    sym_b = sym.element_size()
    alg_enc = n * (sym_b + 4) + comp     # symbols + indexes read, bytes written
    alg_dec = n * (sym_b + 4) + comp     # bytes + indexes read, symbols written
    peaks = {}
    pk_path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(pk_path):
        peaks = json.load(open(pk_path))
    peak = peaks.get("hbm_gbs")
    peak_src = "measured" if peak else "fallback"
    peak = peak or 6650.0
    enc_gbs = alg_enc / (enc_ms * 1e-3) / 1e9
    dec_gbs = alg_dec / (dec_ms * 1e-3) / 1e9
    dominant = "decode" if dec_ms >= enc_ms else "encode"
    traffic = (measured_traffic(args.traffic_file, dominant,
                                "images=%d group=%d" % (args.images, args.group))
               if args.workload == "batch" else None)
    ach = dec_gbs if dominant == "decode" else enc_gbs
    # strong scaling when the ranks split one workload's streams (the
    # sweep), weak when each rank codes its own images
    split = w.get("stream_block")
    total_syms = split[2] if split else n * world
    ms_per_step = elapsed_ms / args.steps
    if flush is not None:  # the steps' coding time, without the L2 flushes
        ms_per_step = tab_ms + enc_ms + dec_ms
    value = total_syms / (ms_per_step * 1e-3) / 1e9

    # end to end through the public API with host buffers: every step copies
    # its symbols and indexes in from pinned host memory and reads the coded
    # bytes, the stream offsets and the decoded symbols back.  Two buffer sets
    # and three streams let step i+1's input copy and step i's result read run
    # on the copy engines while the coders run.
    e2e = None
    if not args.no_e2e:
        h_sym = torch.from_numpy(sym_np).pin_memory()
        h_idx = torch.from_numpy(idx_np).pin_memory()
        s_in, s_run, s_out = (torch.cuda.Stream(dev) for _ in range(3))
        bufs = []
        for _ in range(2):
            bufs.append(dict(
                sym=torch.empty_like(sym), idx=torch.empty_like(idx),
                ws=ws if not bufs else rb.Workspaces(ch, n, dev), dec=torch.empty_like(sym),
                h_out=torch.empty(ws.out.numel(), dtype=torch.uint8).pin_memory(),
                h_off=torch.empty(S + 1, dtype=torch.int64).pin_memory(),
                h_tot=torch.empty(1, dtype=torch.int64).pin_memory(),
                h_dec=torch.empty(n, dtype=sym.dtype).pin_memory(),
                ev_in=torch.cuda.Event(), ev_used=torch.cuda.Event(),
                ev_enc=torch.cuda.Event(), ev_dec=torch.cuda.Event(),
                ev_tot=torch.cuda.Event(), ev_out=torch.cuda.Event()))
        moved = {"h2d": 0, "d2h": 0}

        def copy_in(b):
            # the input buffers are free once the step that used them decoded
            s_in.wait_event(b["ev_used"])
            with torch.cuda.stream(s_in):
                b["sym"].copy_(h_sym, non_blocking=True)
                b["idx"].copy_(h_idx, non_blocking=True)
            b["ev_in"].record(s_in)
            moved["h2d"] += n * sym_b + n * 4

        def run_steps(k):
            copy_in(bufs[0])
            for i in range(k):
                b, nb = bufs[i % 2], bufs[(i + 1) % 2]
                bw = b["ws"]
                s_run.wait_event(b["ev_in"])
                s_run.wait_event(b["ev_out"])      # this set's last result read is done
                with torch.cuda.stream(s_run):
                    build_rows()
                    rb.check(rb.rans_tables_refresh(cdfs, lengths, offsets, tables))
                    rb.check(rb.rans_encode_with_indexes(b["sym"], b["idx"], n, tables, ch,
                                                         bw.out, bw.offsets, bw.enc))
                    b["ev_enc"].record(s_run)
                    b["h_tot"].copy_(bw.offsets[-1:], non_blocking=True)
                    b["ev_tot"].record(s_run)
                    rb.check(rb.rans_decode_with_indexes(bw.out, bw.offsets, b["idx"], n, tables,
                                                         ch, b["dec"], bw.dec))
                    b["ev_dec"].record(s_run)
                    b["ev_used"].record(s_run)
                if i + 1 < k:
                    copy_in(nb)
                b["ev_tot"].synchronize()          # the coded size, once the encoder is done
                total = int(b["h_tot"][0])
                s_out.wait_event(b["ev_enc"])
                with torch.cuda.stream(s_out):
                    b["h_out"][:total].copy_(bw.out[:total], non_blocking=True)
                    b["h_off"].copy_(bw.offsets, non_blocking=True)
                s_out.wait_event(b["ev_dec"])
                with torch.cuda.stream(s_out):
                    b["h_dec"].copy_(b["dec"], non_blocking=True)
                b["ev_out"].record(s_out)
                moved["d2h"] += total + 8 * (S + 1) + n * sym_b
            return total

        torch.cuda.synchronize()
        run_steps(2)
        torch.cuda.synchronize()
        barrier(world)
        a = torch.cuda.Event(enable_timing=True)
        z = torch.cuda.Event(enable_timing=True)
        ke = max(3, min(args.steps, 10))
        moved = {"h2d": 0, "d2h": 0}
        a.record(s_in)
        total = run_steps(ke)
        s_in.wait_event(bufs[0]["ev_out"])
        s_in.wait_event(bufs[1]["ev_out"])
        z.record(s_in)
        torch.cuda.synchronize()
        e_ms = max_over_ranks(a.elapsed_time(z), world, dev) / ke
        for b in bufs:
            assert torch.equal(b["h_dec"], torch.from_numpy(sym_np)), "e2e round trip failed"
        lb = bufs[(ke - 1) % 2]
        assert int(lb["h_off"][-1]) == total
        assert torch.equal(lb["h_out"][:total], lb["ws"].out[:total].cpu())
        e2e = {"value": total_syms / (e_ms * 1e-3) / 1e9, "unit": UNIT,
               "h2d_bytes_per_step": moved["h2d"] // ke, "d2h_bytes_per_step": moved["d2h"] // ke,
               "overlap": "double-buffered: next step's input copy and this step's result "
                          "read run beside the coders"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        workers = os.cpu_count() or 1
        ms = {"batch": 768, "sweep": 64, "r16": 256}.get(args.workload, S)
        ns, ts = oracle_sample(w, ms, workers)
        ms1 = max(1, ms // workers)           # one thread: about the same wall time
        ns1, ts1 = oracle_sample(w, ms1, 1)
        cpu = {"value": ns / ts / 1e9, "unit": UNIT, "cores": workers, "kind": "oracle",
               "sample": "oracle encode+decode of the first %d streams (%d symbols), "
                         "one stream per call over %d threads" % (ms, ns, workers),
               "single_thread": {"value": ns1 / ts1 / 1e9, "unit": UNIT,
                                 "sample": "the first %d streams on one thread" % ms1}}

    # our kernels per step: the table rebuild (one fused kernel for a scale
    # table; rows + refresh for pmfs), the coder and its compaction (one
    # kernel up to 65,536 streams, scan + copy above), the decoder
    launches_per_step = (1 if "scales" in w else 2) + (2 if S <= 65536 else 3) + 1
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "strong" if split else "weak",
            "vs_baseline": None, "dtype": "u64" if fmt == "rans64" else "u32",
            "data": "synthetic",
            "config": {"workload": workload_name(w, args), "symbols_per_gpu": n,
                       "streams_per_gpu": S, "channel_group": args.group,
                       "interleave": w["W"], "rows": K,
                       "lmax": Lmax,
                       "launch": "eager calls" if args.eager else
                                 "each step one CUDA graph (its phases and their events)",
                       "parallelism": ("shard-by-stream-range x%d" if split else
                                       "shard-by-image x%d") % world,
                       "l2": ("inputs larger than L2 (%d MB read per encode)" %
                              (n * (sym_b + 4) // 2**20)) if flush is None else
                             "L2 flushed before every step (256 MB write, not timed)"},
            "encode": {"ms": enc_ms, "ms_median": float(np.median(enc_t)),
                       "ms_best": float(np.min(enc_t)), "gsym_s": n / enc_ms / 1e6,
                       "GBps": enc_gbs, "frac_hbm": enc_gbs / peak, "alg_bytes": alg_enc},
            "decode": {"ms": dec_ms, "ms_median": float(np.median(dec_t)),
                       "ms_best": float(np.min(dec_t)), "gsym_s": n / dec_ms / 1e6,
                       "GBps": dec_gbs, "frac_hbm": dec_gbs / peak, "alg_bytes": alg_dec},
            "tables": {"ms": tab_ms, "ms_median": float(np.median(tab_t))},
            "compressed_bytes": comp, "bits_per_symbol": 8.0 * comp / n,
            "roofline": {"bound": "hbm", "achieved": ach, "peak": peak, "unit": "GB/s",
                         "frac": ach / peak, "traffic": traffic, "kernel": dominant,
                         "peak_source": peak_src},
            "cpu_baseline": cpu,
            "e2e": e2e,
            "clocks": clocks,
            "gpu_launches": launches_per_step * args.steps,
        }
        if container is not None:
            line["config"]["container"] = container
        print(json.dumps(line), flush=True)


def run_float(args, world, rank, local):
    """--workload float: the batch as float latents through
    rans_encode_from_scales / rans_decode_to_values."""
    import torch

    import rans_entropy_coding_b200 as rb

    rb.lib()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    w = load_inputs(rank, args.group, args.images, "float")
    flat = lambda a: torch.from_numpy(np.ascontiguousarray(a).reshape(-1)).to(dev)
    y, sc, mu = flat(w["y"]), flat(w["fscales"]), flat(w["means"])
    n = y.numel()
    table = torch.from_numpy(np.asarray(w["scales"], np.float32)).to(dev)
    bound, tail = w["scale_bound"], w["tail_mass"]
    ch = rb.Chunking.from_spec(w["chunking"], 32, 1, device=dev)
    S = rb.rans_num_streams(ch, n)
    cdfs, lengths, offsets = rb.Tables.build_from_scales(table, tail)
    K, Lmax = cdfs.shape
    tables = rb.Tables(cdfs, lengths, offsets)
    ws = rb.Workspaces(ch, n, dev)
    vals = torch.empty_like(y)
    want = torch.round(y - mu).to(torch.int32).to(torch.float32) + mu
    stream = torch.cuda.current_stream()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]

    def step_body(e=None):
        cur = torch.cuda.current_stream()
        if e: e[0].record(cur)
        rb.check(rb.rans_tables_refresh_from_scales(table, tail, cdfs, lengths, offsets, tables),
                 "tables")
        if e: e[1].record(cur)
        rb.check(rb.rans_encode_from_scales(y, mu, sc, n, table, bound, tables, ch, ws.out,
                                            ws.offsets, ws.enc), "encode")
        if e: e[2].record(cur)
        rb.check(rb.rans_decode_to_values(ws.out, ws.offsets, sc, mu, n, table, bound, tables,
                                          ch, vals, ws.dec), "decode")
        if e: e[3].record(cur)

    for _ in range(max(args.warmup, 0)):
        step_body()
    torch.cuda.synchronize()
    steps = [lambda e=e: step_body(e) for e in ev]
    if not args.eager:
        # one CUDA graph per timed step, its phase events graph nodes (as the
        # integer workloads)
        ev = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(4)]
              for _ in range(args.steps)]
        cap = torch.cuda.Stream(dev)

        def capture(e):
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr, stream=cap):
                step_body(e)
            return gr

        warm = capture(None)
        graphs = [capture(e) for e in ev]
        steps = [gr.replay for gr in graphs]
        for _ in range(max(args.warmup, 0)):
            warm.replay()
        torch.cuda.synchronize()
    for what, b in (("encode", ws.enc), ("decode", ws.dec), ("tables", tables.blob)):
        rb.check(rb.rans_get_status(b), what + " status")
    assert torch.equal(vals, want), "round trip failed"
    barrier(world)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with ClockSampler(local, enabled=not args.no_clocks) as clk:
        torch.cuda.synchronize()
        barrier(world)
        t0.record(stream)
        for i in range(args.steps):
            steps[i]()
        t1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
    elapsed_ms = max_over_ranks(t0.elapsed_time(t1), world, dev)
    assert torch.equal(vals, want), "round trip failed"
    tab_ms = float(np.mean([e[0].elapsed_time(e[1]) for e in ev]))
    enc_ms = float(np.mean([e[1].elapsed_time(e[2]) for e in ev]))
    dec_ms = float(np.mean([e[2].elapsed_time(e[3]) for e in ev]))
    comp = int(ws.offsets[-1].item())
    alg_enc = n * 12 + comp      # y, scale, mean read; bytes written
    alg_dec = n * 12 + comp      # bytes, scale, mean read; values written
    peak = (json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json"))).get("hbm_gbs")
            if os.path.exists(os.path.join(ROOT, "MEASURED_PEAKS.json")) else None) or 6650.0
    enc_gbs = alg_enc / (enc_ms * 1e-3) / 1e9
    dec_gbs = alg_dec / (dec_ms * 1e-3) / 1e9
    ms_per_step = elapsed_ms / args.steps
    value = n * world / (ms_per_step * 1e-3) / 1e9
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle as O
        wi = dict(w, symbols=O.quantize(w["y"], w["means"]),
                  indexes=O.build_indexes(w["fscales"], w["scales"], bound).reshape(-1), W=32)
        workers = os.cpu_count() or 1
        ns, ts = oracle_sample(wi, 768, workers)
        cpu = {"value": ns / ts / 1e9, "unit": UNIT, "cores": workers, "kind": "oracle",
               "sample": "oracle encode+decode of the first 768 streams (%d symbols), rows "
                         "and symbols computed beforehand" % ns}
    if rank == 0:
        dominant = "decode" if dec_ms >= enc_ms else "encode"
        ach = dec_gbs if dominant == "decode" else enc_gbs
        print(json.dumps({
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "u64",
            "data": "synthetic",
            "config": {"workload": workload_name(w, args), "symbols_per_gpu": n,
                       "streams_per_gpu": S, "channel_group": args.group, "interleave": 32,
                       "rows": K, "lmax": Lmax, "parallelism": "shard-by-image x%d" % world,
                       "launch": "eager calls" if args.eager else
                                 "each step one CUDA graph (its phases and their events)",
                       "l2": "inputs larger than L2 (%d MB read per encode)" % (n * 12 >> 20)},
            "encode": {"ms": enc_ms, "gsym_s": n / enc_ms / 1e6, "GBps": enc_gbs,
                       "frac_hbm": enc_gbs / peak, "alg_bytes": alg_enc},
            "decode": {"ms": dec_ms, "gsym_s": n / dec_ms / 1e6, "GBps": dec_gbs,
                       "frac_hbm": dec_gbs / peak, "alg_bytes": alg_dec},
            "tables": {"ms": tab_ms}, "compressed_bytes": comp,
            "bits_per_symbol": 8.0 * comp / n,
            "roofline": {"bound": "hbm", "achieved": ach, "peak": peak, "unit": "GB/s",
                         "frac": ach / peak, "traffic": None, "kernel": dominant},
            "cpu_baseline": cpu, "e2e": None, "clocks": clk.summary(),
            "gpu_launches": (1 + (2 if S <= 65536 else 3) + 1) * args.steps,
        }), flush=True)


def main():
    args = parse()
    world, rank, local = dist_setup(args)
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        elif args.workload == "float":
            run_float(args, world, rank, local)
        else:
            run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
