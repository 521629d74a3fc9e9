"""The seeded synthetic inputs have the shapes, sizes and structure their
recipes state (the pages' y / z latents, the 16-image batch, the uint8
sweep, the rans32_16 benchmark shape), and are reproducible."""
import numpy as np

import oracle as O
import workloads as WL


def test_y_latent_and_batch_shapes():
    y = WL.y_latent()
    assert np.asarray(y["symbols"]).shape == (1, 192, 68, 120)            # 1,566,720 symbols
    assert np.asarray(y["symbols"]).size == 1566720
    assert len(y["scales"]) == 64 and y["chunking"] == dict(kind="contig", n_streams=24)
    b = WL.y_batch(n_images=2)
    assert np.asarray(b["symbols"]).shape == (2, 192, 68, 120)
    pos = O.stream_positions(np.asarray(b["symbols"]).size, b["chunking"])
    # 2 images x 48 channel groups x 2 tile rows x 2 tile columns
    assert len(pos) == 2 * 48 * 2 * 2
    assert sorted({p.size for p in pos}) == [896, 1024, 14336, 16384]


def test_batch_images_are_the_per_image_seeds():
    one = WL.y_batch(n_images=1, first_image=1)
    two = WL.y_batch(n_images=2)
    assert np.array_equal(np.asarray(two["symbols"])[1], np.asarray(one["symbols"])[0])


def test_z_latent_shape_and_rows():
    z = WL.z_latent()
    assert np.asarray(z["symbols"]).size == 128 * 17 * 30 == 65280
    assert len(z["pmf_lengths"]) == 128 and z["chunking"]["n_streams"] == 32
    # every symbol inside its channel's coded range (Laplace sampling)
    rows = np.asarray(z["indexes"])
    v = np.asarray(z["symbols"]).reshape(-1) - np.asarray(z["offsets"])[rows]
    assert (v >= 0).all() and (v < np.asarray(z["pmf_lengths"])[rows]).all()


def test_tiny_has_escapes_and_extremes():
    t = WL.tiny()
    s = t["symbols"]
    assert s.size == 4096 and s[1] == np.iinfo(np.int32).min and s[2] == np.iinfo(np.int32).max
    far = np.abs(s.astype(np.int64)) >= 65
    assert 0.005 < far.mean() < 0.02                         # ~1% forced escapes


def test_sweep_uint8_with_index_blocks():
    w = WL.sweep(log2_n=16, n_streams=8)
    assert w["symbols"].dtype == np.uint8 and w["symbols"].size == 1 << 16
    assert w["index_block"] == 4096 and w["indexes"].size == (1 << 16) // 4096
    assert (np.asarray(w["pmf_lengths"]) == 256).all()


def test_r16_shape():
    w = WL.r16_rows(n_streams=16, per_stream=4096)
    assert w["symbols"].size == 16 * 4096 and w["fmt"] == "rans32_16" and w["precision"] == 15
    c, l = O.build_cdfs_from_pmfs(w["pmfs"], w["pmf_lengths"], w["tail"], precision=15)
    assert (l == 257).all()                                   # 255 symbols + escape: 256 buckets
    assert w["symbols"].min() >= 0 and w["symbols"].max() <= 254


def test_generators_are_reproducible():
    for make in (lambda: WL.tiny(seed=3), lambda: WL.z_latent(seed=4),
                 lambda: WL.r16_rows(n_streams=2, per_stream=100)):
        a, b = make(), make()
        assert np.array_equal(np.asarray(a["symbols"]), np.asarray(b["symbols"]))
        assert np.array_equal(np.asarray(a["indexes"]), np.asarray(b["indexes"]))
