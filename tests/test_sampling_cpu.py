"""Host logic of the full-size parity tests: the token sample that covers every
128-row band, checked on CPU against routings whose bands are known."""
import numpy as np

from combine_overlap_b200 import synth
import gpu_util as gu


def _perm_of(idx, E):
    # stable counting sort of the slots by expert (what the permutation computes)
    p = np.argsort(idx.reshape(-1), kind="stable").astype(np.int32)
    counts = np.bincount(idx.reshape(-1), minlength=E)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    return offsets, p


def test_band_covering_sample_hits_every_band():
    rng = np.random.default_rng(7)
    for T, E, k in ((1000, 8, 2), (4096, 64, 6), (333, 5, 3), (1, 4, 2)):
        wl = synth.small("s", T, 256, 128, E, k)
        idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
        offsets, perm = _perm_of(idx, E)
        toks = gu.band_covering_tokens(offsets, perm, wl, n_random=5)
        assert gu.bands_covered(offsets, perm, wl, toks)
        assert toks.min() >= 0 and toks.max() < T and 0 in toks and T - 1 in toks
        n_bands = sum(-(-(offsets[e + 1] - offsets[e]) // 128) for e in range(E))
        assert len(toks) <= n_bands + 2 + 5


def test_bands_covered_detects_a_gap():
    wl = synth.small("s", 512, 256, 128, 2, 1)
    idx = np.zeros((512, 1), np.int32)
    idx[256:] = 1
    offsets, perm = _perm_of(idx, 2)
    # tokens 0..127 cover band 0 of expert 0 only
    assert not gu.bands_covered(offsets, perm, wl, np.arange(128))
    assert gu.bands_covered(offsets, perm, wl, np.arange(0, 512, 128))


def test_combine_bound_is_one_bf16_ulp():
    one = np.array([0x3F80], np.uint16)          # 1.0
    nxt = np.array([0x3F81], np.uint16)          # 1.0 + 2^-7
    gu.assert_combine_close(nxt, one)
    two_ulp = np.array([0x3F82], np.uint16)
    try:
        gu.assert_combine_close(two_ulp, one)
    except AssertionError:
        pass
    else:
        raise AssertionError("two ulps accepted")


def test_sweep_cell_spec():
    import sys
    sys.argv = ["bench.py"]
    import bench
    cells = bench._sweep_cells("seq,0,2/2,0+0x400,seq+0x800")
    assert cells == [("seq", None, 0, 1, 0), ("0", "ovl", 0, 1, 0), ("2/2", "ovl", 2, 2, 0),
                     ("0+0x400", "ovl", 0, 1, 0x400), ("seq+0x800", None, 0, 1, 0x800)]
