"""Parity of coarse-to-fine matching on the GPU (needs a B200) against the
oracle's ``c2f`` (coarse reciprocal set, crop table, FRM per crop pair, map
back).  Descriptor values are multiples of 1/64 (smooth unit maps rounded to
k/64, or the quantised generator), so every score is exact and the pairs and
the crop table must agree bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
import reciprocal_nearest_neighbour_b200 as rnn
from reciprocal_nearest_neighbour_b200 import synth
from parity import dev

pytestmark = pytest.mark.gpu


def _q64(F):
    return np.clip(np.round(F * 64.0), -127, 127) / 64.0


def _maps(seed, H1, W1, H2, W2, d, s, dt="f16"):
    """Rounded smooth pair (image 2 cut or padded to its size) and coarse
    maps read from them at cells of s x s pixels."""
    Hm, Wm = max(H1, H2), max(W1, W2)
    A, B = synth.smooth_pair(seed, Hm, Wm, d)
    F1, F2 = _q64(A[:H1, :W1]), _q64(B[:H2, :W2])
    C1 = synth.coarse_map(F1, H1 // s, W1 // s)
    C2 = synth.coarse_map(F2, H2 // s, W2 // s)
    return [synth.to_storage(x, dt) for x in (C1, C2, F1, F2)]


def _check(maps, crop, S, max_iter, min_coarse=1, metric="dot"):
    C1, C2, F1, F2 = maps
    r = rnn.c2f_match(dev(C1), dev(C2), dev(F1), dev(F2), crop=crop, seed_stride=S,
                      max_iter=max_iter, min_coarse=min_coarse, metric=metric)
    ref = oracle.c2f(C1, C2, F1, F2, crop=crop, seed_stride=S, max_iter=max_iter,
                     min_coarse=min_coarse, metric=metric)
    assert np.array_equal(r.crops.cpu().numpy()[: len(ref.crops)], ref.crops)
    assert np.array_equal(r.trimmed().cpu().numpy(), ref.pairs)
    return r, ref


@pytest.mark.parametrize("dt", ["f16", "bf16"])
def test_c2f_grid_of_crops_bitexact(dt):
    r, ref = _check(_maps(1, 72, 100, 72, 100, 16, 4, dt), (32, 40), 4, 10)
    assert ref.crops[:, 5].sum() >= 5 and len(ref.pairs) > 100


def test_c2f_unequal_sizes_min_coarse_and_l2():
    maps = _maps(2, 60, 84, 52, 96, 24, 4)
    _check(maps, (24, 30), 3, 6, min_coarse=3)
    _check(maps, (24, 30), 3, 6, metric="l2")


def test_c2f_crops_off_and_tiny_crops():
    # a high min_coarse turns most crops off; 8x8 crops with stride 4 seed 4 a crop
    maps = _maps(3, 40, 48, 40, 48, 8, 2)
    r, ref = _check(maps, (8, 8), 4, 10, min_coarse=14)
    assert 0 < ref.crops[:, 5].sum() < len(ref.crops)


def test_c2f_one_crop_equals_frm():
    C1, C2, F1, F2 = _maps(4, 48, 64, 48, 64, 16, 4)
    r = rnn.c2f_match(dev(C1), dev(C2), dev(F1), dev(F2), crop=(100, 100), seed_stride=4)
    f = rnn.frm_match_ex(dev(F1), dev(F2), seed_stride=4)
    assert r.crops.shape[0] == 1
    assert np.array_equal(r.trimmed().cpu().numpy(), f.trimmed().cpu().numpy())


def test_c2f_large_maps_bitexact():
    """1024x768 maps, d = 32, coarse 80x64 cells, crops of 384x512 (2 x 2)."""
    A, B = synth.smooth_pair(5, 768, 1024, 32, outliers=0.02)
    F1, F2 = _q64(A), _q64(B)
    C1, C2 = synth.coarse_map(F1, 64, 80), synth.coarse_map(F2, 64, 80)
    maps = [synth.to_storage(x, "f16") for x in (C1, C2, F1, F2)]
    r, ref = _check(maps, (384, 512), 8, 10)
    assert len(ref.crops) == 4 and len(ref.pairs) > 5000


def test_c2f_all_crops_off_gives_no_pairs():
    C1, C2, F1, F2 = _maps(6, 32, 40, 32, 40, 16, 4)
    r = rnn.c2f_match(dev(C1), dev(C2), dev(F1), dev(F2), crop=(16, 16), seed_stride=4,
                      min_coarse=10 ** 6)
    ref = oracle.c2f(C1, C2, F1, F2, crop=(16, 16), seed_stride=4, min_coarse=10 ** 6)
    assert int(r.count.item()) == 0 and len(ref.pairs) == 0
    assert np.array_equal(r.crops.cpu().numpy(), ref.crops)
    assert not ref.crops[:, 5].any()


@pytest.mark.parametrize("metric", ["dot", "l2"])
def test_c2f_bf16_unequal_coarse_ratio(metric):
    # coarse cells of 3 x 5 pixels (not a divisor of the crops), bf16 maps
    C1, C2, F1, F2 = _maps(7, 45, 70, 51, 65, 24, 1, "bf16")
    C1 = synth.to_storage(synth.coarse_map(F1.float().numpy().astype(np.float64), 15, 14), "bf16")
    C2 = synth.to_storage(synth.coarse_map(F2.float().numpy().astype(np.float64), 17, 13), "bf16")
    _check([C1, C2, F1, F2], (20, 24), 3, 8, metric=metric)
