"""The seeded input generators produce the input recipe the measurements are quoted on:
shapes, value distributions, outlier channels, bf16 exactness, signs, weights and HARP draws.
CPU only; every workload is drawn with 256 rows here (same recipe, any M)."""
import math

import numpy as np
import pytest

import workloads as W

# name: (K, outlier fraction, outlier scale, bf16, quant pairs, N)
RECIPE = {
    "pr1": (2048, 0.01, 20.0, False, [(4, 128), (4, 32)], 512),
    "llama32_1b": (2048, 0.005, 100.0, True, [(4, 32)], None),
    "down_proj": (8192, 0.005, 50.0, True, [(4, 128), (2, 64)], None),
    "harp11008": (11008, 0.01, 20.0, True, [(4, 128), (2, 64)], None),
    "q_proj_prefill": (4096, 0.01, 20.0, True, [(4, 128)], 4096),
    "q_proj_decode": (4096, 0.01, 20.0, True, [(4, 128)], 4096),
    "up_proj_prefill": (4096, 0.01, 20.0, True, [(4, 128)], 11008),
    "up_proj_decode": (4096, 0.01, 20.0, True, [(4, 128)], 11008),
}
FULL_M = {"pr1": 16, "llama32_1b": 8192, "down_proj": 4096, "harp11008": 4096, "q_proj_prefill": 2048,
          "q_proj_decode": 16, "up_proj_prefill": 2048, "up_proj_decode": 16}


def test_recipe_table_is_the_generators_table():
    assert set(RECIPE) == set(W.WORKLOADS)
    for name, (K, frac, scale, bf16, quant, N) in RECIPE.items():
        cfg = W.WORKLOADS[name]
        assert (cfg["M"], cfg["K"], cfg["frac"], cfg["scale"], cfg["bf16"]) == (FULL_M[name], K, frac, scale, bf16)
        assert [tuple(q) for q in cfg["quant"]] == quant
        assert cfg.get("N") == N
    assert W.WORKLOADS["harp11008"]["radices"] == [2] * 8 + [43]
    assert int(np.prod(W.WORKLOADS["harp11008"]["radices"])) == 11008
    assert W.WORKLOADS["llama32_1b"]["dist"] == "student_t" and W.WORKLOADS["llama32_1b"]["t_scale"] == 0.5


@pytest.mark.parametrize("name", sorted(RECIPE))
def test_outlier_channels_and_precision(name):
    K, frac, scale, bf16, quant, N = RECIPE[name]
    M = 256   # the recipe does not depend on M; enough rows for stable per-channel statistics
    wl = W.make_workload(name, M=M)
    assert wl.A.shape == (M, K) and wl.A.dtype == np.float32
    # exactly ceil(frac * K) channels carry the outlier scale (per-channel median |a|: robust to
    # the single large draws of the heavy-tailed workload)
    n_out = math.ceil(frac * K)
    mag = np.median(np.abs(wl.A.astype(np.float64)), axis=0)
    order = np.argsort(mag)[::-1]
    base = np.median(mag)
    top = mag[order[:n_out]] / base
    assert np.all(top > scale / 3), (name, top.min())
    assert mag[order[n_out]] / base < 2.0
    assert abs(np.median(top) / scale - 1.0) < 0.35
    if bf16:
        bits = wl.A.view(np.uint32)
        assert np.all(bits & 0xFFFF == 0), "bf16 workloads hold exact bfloat16 values"
    for bits_, G in wl.quant:
        assert K % G == 0 and bits_ in (2, 4)
    if N is not None:
        assert wl.W.shape == (K, N)
        assert abs(float(np.std(wl.W)) - 0.02) < 0.002


def test_student_t_tails_and_normal_body():
    inl = W.make_workload("llama32_1b", M=256).A.astype(np.float64)
    nor = W.make_workload("down_proj", M=64).A.astype(np.float64)
    def excess_kurtosis(a):
        rms = np.sqrt(np.mean(a ** 2, axis=0))
        body = a[:, rms < 3 * np.median(rms)].ravel()
        body = body - body.mean()
        return np.mean(body ** 4) / np.mean(body ** 2) ** 2 - 3.0
    assert excess_kurtosis(inl) > 1.0          # Student-t(4): heavy tails
    assert abs(excess_kurtosis(nor)) < 0.2     # N(0, 1)
    body = inl[:, np.sqrt(np.mean(inl ** 2, axis=0)) < 3 * np.median(np.sqrt(np.mean(inl ** 2, axis=0)))]
    # Student-t(4) * 0.5 has standard deviation 0.5 * sqrt(2)
    assert abs(body.std() / (0.5 * math.sqrt(2.0)) - 1.0) < 0.1


def test_signs_and_determinism():
    a = W.make_workload("q_proj_decode")
    b = W.make_workload("q_proj_decode")
    assert np.array_equal(a.A, b.A) and np.array_equal(a.signs, b.signs) and np.array_equal(a.W, b.W)
    c = W.make_workload("q_proj_decode", seed=1)
    assert not np.array_equal(a.A, c.A)
    s = W.make_workload("llama32_1b", M=4).signs
    assert s.dtype == np.int8 and set(np.unique(s)) == {-1, 1}
    assert abs(float(np.mean(s))) < 0.1


def test_harp_draws():
    radices = [2] * 8 + [43]
    d = W.harp_draws(2, radices)
    K = 11008
    assert len(d.angles) == len(d.gaussians) == len(d.perms) == len(radices)
    for t, b in enumerate(radices):
        if b == 2:
            assert d.angles[t].shape == (K // 2,) and d.gaussians[t] is None
            assert d.angles[t].min() >= -np.pi and d.angles[t].max() < np.pi
        else:
            assert d.angles[t] is None and d.gaussians[t].shape == (1, b, b)
        if t < len(radices) - 1:
            assert np.array_equal(np.sort(d.perms[t]), np.arange(K))
        else:
            assert d.perms[t] is None
    e = W.harp_draws(2, radices)
    assert all(np.array_equal(x, y) for x, y in zip(d.perms[:-1], e.perms[:-1]))
    pb = W.harp_draws(2, [2, 43], per_block_gaussian=True)
    assert pb.gaussians[1].shape == (2, 43, 43)
