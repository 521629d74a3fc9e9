"""Seeded synthetic inputs for the five coding workloads.

Shared by the oracle side and the CUDA side of every test and of the bench:
both code exactly these arrays.  This module holds none of the coder's
arithmetic (no CDF quantisation, no rANS step); it only draws symbols, row
indexes and the model-side inputs the coder starts from (a scale table or
float pmfs).

The pages measure on the latents of one 1920x1080 image run through CompressAI's
mbt2018_mean model ("kompressor" README, Getting Started and Benchmarks: the y
latent has 1,566,720 symbols and 64 CDF rows, the z latent 65,280 symbols).
Those latents need trained weights that are not available, so the generators
below stand in for them with the same shapes and row structure:

  tiny   4,096 int32; 8 Gaussian rows (scales log-spaced 0.11..8); uniform
         row per symbol; symbol = round(N(0, row scale)); about 1% forced far
         past every row's coded range (|s| >= 65, so the bypass path carries
         1-8 raw nibbles) plus INT32_MIN / INT32_MAX; 1 stream, W = 1.
  z      128 x 17 x 30 int32 (NCHW, batch 1); one Laplace pmf row per channel,
         b ~ U[0.3, 3]; symbols drawn from the channel's pmf; 32 contiguous
         streams, W = 1.
  y      192 x 68 x 120 int32; 64-row Gaussian scale table
         exp(linspace(ln 0.11, ln 256, 64)); per-element scale log-uniform on
         [0.11, 256]; row = the nearest table entry in log space; symbol =
         round(N(0, element scale)); 24 contiguous streams, W = 1 or 32.
  batch  16 y latents (image b drawn with seed 3000 + b), NCHW
         [16, 192, 68, 120]; one stream per 64 x 64 spatial tile per group of
         4 channels (3,072 streams), W = 32.
  sweep  2^28 uint8 symbols; 16 Zipf rows p(k) ~ (k+1)^-s, s in
         linspace(0.8, 1.6, 16), over 256 symbols with no tail; one row per
         4,096-symbol block; 8,192 contiguous streams, W = 32.

Seeds: numpy Generator(PCG64(1000 * workload_number + image)).
"""
import math

import numpy as np

SCALE_MIN = 0.11
SCALE_MAX_Y = 256.0
N_ROWS_Y = 64
Y_SHAPE = (192, 68, 120)
Z_SHAPE = (128, 17, 30)


def _rng(seed):
    return np.random.Generator(np.random.PCG64(seed))


def log_spaced_scales(lo, hi, k):
    """k scales log-spaced from lo to hi, as float32."""
    return np.exp(np.linspace(math.log(lo), math.log(hi), k)).astype(np.float32)


def _sample_from_pmfs(rng, cum, rows):
    """Draws one value per entry of ``rows`` from that row's distribution;
    ``cum`` holds each row's running sum of probabilities (float64)."""
    u = rng.random(rows.size)
    out = np.empty(rows.size, dtype=np.int64)
    for r in np.unique(rows):
        sel = np.nonzero(rows == r)[0]
        c = cum[r]
        out[sel] = np.minimum(np.searchsorted(c, u[sel] * c[-1], side="right"), c.size - 1)
    return out


def tiny(seed=0, n=4096):
    rng = _rng(seed)
    scales = log_spaced_scales(SCALE_MIN, 8.0, 8)
    idx = rng.integers(0, 8, size=n).astype(np.int32)
    sym = np.rint(rng.standard_normal(n) * scales[idx].astype(np.float64))
    force = rng.random(n) < 0.01
    sign = np.where(rng.random(n) < 0.5, -1.0, 1.0)
    k = np.floor(2.0 ** rng.uniform(0.0, 30.0, size=n))
    sym = np.where(force, sign * (65.0 + k), sym)
    sym = sym.astype(np.int64)
    if n > 2:
        sym[1] = np.iinfo(np.int32).min
        sym[2] = np.iinfo(np.int32).max
    return dict(name="tiny", symbols=sym.astype(np.int32), indexes=idx, scales=scales,
                tail_mass=1e-9, chunking=dict(kind="contig", n_streams=1), W=1,
                index_block=1)


def z_latent(seed=1000):
    rng = _rng(seed)
    C, H, Wd = Z_SHAPE
    b = rng.uniform(0.3, 3.0, size=C)
    centers = np.ceil(b * math.log(1e9) - 0.5).astype(np.int64)
    S = int(2 * centers.max() + 1)
    pmfs = np.zeros((C, S), dtype=np.float32)
    pmf_lengths = (2 * centers + 1).astype(np.int32)
    tails = np.zeros(C, dtype=np.float32)
    cum = []
    for c in range(C):
        k = np.arange(-centers[c], centers[c] + 1, dtype=np.float64)
        lap = lambda x: np.where(x < 0, 0.5 * np.exp(x / b[c]), 1.0 - 0.5 * np.exp(-x / b[c]))
        p = lap(k + 0.5) - lap(k - 0.5)
        pmfs[c, :p.size] = p.astype(np.float32)
        tails[c] = np.float32(2.0 * lap(np.array(-centers[c] - 0.5)))
        cum.append(np.cumsum(p))
    rows = np.repeat(np.arange(C, dtype=np.int32), H * Wd)
    v = _sample_from_pmfs(rng, cum, rows)
    sym = (v - centers[rows]).astype(np.int32)
    return dict(name="z", symbols=sym.reshape(1, C, H, Wd), indexes=rows, pmfs=pmfs,
                pmf_lengths=pmf_lengths, tail=tails,
                offsets=(-centers).astype(np.int32),
                chunking=dict(kind="contig", n_streams=32), W=1, index_block=1)


def _y_image(seed):
    rng = _rng(seed)
    n = int(np.prod(Y_SHAPE))
    lo, hi = math.log(SCALE_MIN), math.log(SCALE_MAX_Y)
    u = rng.uniform(lo, hi, size=n)
    step = (hi - lo) / (N_ROWS_Y - 1)
    idx = np.clip(np.rint((u - lo) / step), 0, N_ROWS_Y - 1).astype(np.int32)
    sym = np.rint(rng.standard_normal(n) * np.exp(u))
    sym = np.clip(sym, np.iinfo(np.int32).min, np.iinfo(np.int32).max).astype(np.int32)
    return sym, idx


def many_rows(seed=5000, n=1 << 18, n_rows=256, n_streams=64, W=32):
    """The y recipe over a finer scale table (n_rows rows from 0.11 to 256):
    about 0.4 MB of bucket words, more than one CUDA block's shared memory holds."""
    rng = _rng(seed)
    lo, hi = math.log(SCALE_MIN), math.log(SCALE_MAX_Y)
    u = rng.uniform(lo, hi, size=n)
    step = (hi - lo) / (n_rows - 1)
    idx = np.clip(np.rint((u - lo) / step), 0, n_rows - 1).astype(np.int32)
    sym = np.rint(rng.standard_normal(n) * np.exp(u)).astype(np.int32)
    return dict(name="many_rows", symbols=sym, indexes=idx,
                scales=log_spaced_scales(SCALE_MIN, SCALE_MAX_Y, n_rows), tail_mass=1e-9,
                chunking=dict(kind="contig", n_streams=n_streams), W=W, index_block=1)


def y_float(seed=6000, n_images=2, cg=4, th=64, tw=64, W=32, with_means=True,
            n_rows=N_ROWS_Y):
    """Float latents of a mean-scale model, [n_images, 192, 68, 120]: per
    element a scale exp(U(ln 0.11, ln 256)), a mean U(-8, 8) (or none) and
    y = mean + N(0, scale), all float32; the n_rows-entry scale table (64 by
    default) and its lower bound 0.11.  Rows and symbols come from the scales
    and y - mean."""
    rng = _rng(seed)
    shape = (n_images,) + Y_SHAPE
    n = int(np.prod(shape))
    scales = np.exp(rng.uniform(math.log(SCALE_MIN), math.log(SCALE_MAX_Y), n)).astype(np.float32)
    means = rng.uniform(-8.0, 8.0, n).astype(np.float32) if with_means else None
    y = (rng.standard_normal(n) * scales.astype(np.float64)).astype(np.float32)
    if means is not None:
        y = (y + means).astype(np.float32)
    return dict(name="y_float", y=y.reshape(shape), means=None if means is None else
                means.reshape(shape), fscales=scales.reshape(shape),
                scales=log_spaced_scales(SCALE_MIN, SCALE_MAX_Y, n_rows), tail_mass=1e-9,
                scale_bound=SCALE_MIN,
                chunking=dict(kind="tiled", shape=shape, cg=cg, th=th, tw=tw), W=W,
                index_block=1)


def y_latent(seed=2000, W=1):
    sym, idx = _y_image(seed)
    return dict(name="y", symbols=sym.reshape((1,) + Y_SHAPE), indexes=idx,
                scales=log_spaced_scales(SCALE_MIN, SCALE_MAX_Y, N_ROWS_Y), tail_mass=1e-9,
                chunking=dict(kind="contig", n_streams=24), W=W, index_block=1)


def y_batch(n_images=16, first_image=0, cg=4, th=64, tw=64):
    """Images first_image .. first_image + n_images - 1 of the batch."""
    syms, idxs = [], []
    for b in range(first_image, first_image + n_images):
        s, i = _y_image(3000 + b)
        syms.append(s)
        idxs.append(i)
    C, H, Wd = Y_SHAPE
    return dict(name="batch", symbols=np.concatenate(syms).reshape(n_images, C, H, Wd),
                indexes=np.concatenate(idxs),
                scales=log_spaced_scales(SCALE_MIN, SCALE_MAX_Y, N_ROWS_Y), tail_mass=1e-9,
                chunking=dict(kind="tiled", shape=(n_images, C, H, Wd), cg=cg, th=th, tw=tw),
                W=32, index_block=1)


def sweep(log2_n=28, seed=4000, n_streams=None, block=4096, n_rows=16):
    n = 1 << log2_n
    rng = _rng(seed)
    s = np.linspace(0.8, 1.6, n_rows)
    k = np.arange(1, 257, dtype=np.float64)
    pmfs = np.zeros((n_rows, 256), dtype=np.float32)
    cum = []
    for r in range(n_rows):
        p = k ** (-s[r])
        p /= p.sum()
        pmfs[r] = p.astype(np.float32)
        cum.append(np.cumsum(p))
    nblk = -(-n // block)
    idx = rng.integers(0, n_rows, size=nblk).astype(np.int32)
    sym = np.empty(n, dtype=np.uint8)
    chunk = 1 << 22
    for a in range(0, n, chunk):
        b = min(a + chunk, n)
        rows = np.repeat(idx[a // block: -(-b // block)], block)[: b - a]
        sym[a:b] = _sample_from_pmfs(rng, cum, rows).astype(np.uint8)
    if n_streams is None:
        n_streams = max(1, n // 32768)
    return dict(name="sweep", symbols=sym, indexes=idx, pmfs=pmfs,
                pmf_lengths=np.full(n_rows, 256, dtype=np.int32),
                tail=np.zeros(n_rows, dtype=np.float32),
                offsets=np.zeros(n_rows, dtype=np.int32),
                chunking=dict(kind="contig", n_streams=n_streams), W=32, index_block=block)


def r16_rows(seed=7000, n_streams=1024, per_stream=4096, n_dists=256, alphabet=255):
    """The rans32_16 benchmark shape of "torch_ans 0.3.0" (Performance
    Tuning, GPU table): n_streams streams of per_stream int32 symbols coded
    32-way, alphabet 255 with bypass coding (cdf rows of 257 entries),
    n_dists distributions.  The page gives no distributions; here each row's
    pmf is a Dirichlet(1) draw over the alphabet (about 7.4 bits of entropy),
    every symbol takes a row uniformly at random and is drawn from it, and the
    tail mass is 0 (the escape bucket gets its unit by stealing)."""
    rng = _rng(seed)
    pmfs = rng.gamma(1.0, size=(n_dists, alphabet))
    pmfs = (pmfs / pmfs.sum(axis=1, keepdims=True)).astype(np.float32)
    n = n_streams * per_stream
    idx = rng.integers(0, n_dists, size=n).astype(np.int32)
    cum = [np.cumsum(pmfs[r].astype(np.float64)) for r in range(n_dists)]
    sym = _sample_from_pmfs(rng, cum, idx).astype(np.int32)
    return dict(name="r16", symbols=sym, indexes=idx, pmfs=pmfs,
                pmf_lengths=np.full(n_dists, alphabet, dtype=np.int32),
                tail=np.zeros(n_dists, dtype=np.float32),
                offsets=np.zeros(n_dists, dtype=np.int32),
                chunking=dict(kind="contig", n_streams=n_streams), W=32, index_block=1,
                fmt="rans32_16", precision=15)

