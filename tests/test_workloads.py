"""Host synthetic-input generator: determinism, addressing and distributions."""

import numpy as np

from workloads import FORM_GDN, FORM_KDA, FORM_MAMBA2, CONFIGS, config, philox


def test_counter_addressing_is_deterministic_and_independent():
    cfg = config(1)
    a = philox.normals(cfg, np.arange(10), 3, philox.F_K, 1, 128)
    b = philox.normals(cfg, np.arange(10), 3, philox.F_K, 1, 128)
    assert np.array_equal(a, b)
    # any single element can be regenerated alone
    one = philox.normals(cfg, 7, 3, philox.F_K, 1, 128)
    assert np.array_equal(one, a[7])
    # different unit / step / field / phase / workload give different streams
    for other in (philox.normals(cfg, np.arange(10) + 1, 3, philox.F_K, 1, 128),
                  philox.normals(cfg, np.arange(10), 4, philox.F_K, 1, 128),
                  philox.normals(cfg, np.arange(10), 3, philox.F_V, 1, 128),
                  philox.normals(cfg, np.arange(10), 3, philox.F_K, 0, 128),
                  philox.normals(config(2), np.arange(10), 3, philox.F_K, 1, 128)):
        assert not np.any(other == a)


def test_uniform_and_normal_moments():
    cfg = config(0)
    u = philox.uniforms(cfg, np.arange(4000), 0, philox.F_ALPHA, 1, 64)
    assert u.min() > 0 and u.max() < 1
    assert abs(u.mean() - 0.5) < 3e-3 and abs(u.var() - 1 / 12) < 2e-3
    z = philox.normals(cfg, np.arange(4000), 0, philox.F_K, 1, 64)
    assert abs(z.mean()) < 5e-3 and abs(z.std() - 1) < 5e-3
    assert abs(np.mean(z ** 4) - 3) < 0.05


def test_batched_generation_equals_per_unit_generation():
    cfg = config(4, batch=3, layers=2, heads=2)
    b, l, h = np.meshgrid(np.arange(3), np.arange(2), np.arange(2), indexing="ij")
    batch = philox.token_inputs(cfg, b, l, h, 5, philox.PHASE_DECODE)
    for key in batch:
        for idx in np.ndindex(b.shape):
            single = philox.token_inputs(cfg, b[idx], l[idx], h[idx], 5, philox.PHASE_DECODE)
            assert np.array_equal(batch[key][idx], single[key])


def test_value_distributions_per_form():
    n = 2000
    b = np.arange(n) % 64
    h = np.arange(n) % 48
    for cid in (0, 1, 2):
        x = philox.token_inputs(config(cid), b % config(cid).batch, 0, h % config(cid).heads,
                                np.arange(n), 1)
        np.testing.assert_allclose(np.linalg.norm(x["k"], axis=-1), 1, atol=1e-6)
        np.testing.assert_allclose(np.linalg.norm(x["q"], axis=-1), 1, atol=1e-6)
        assert np.all((x["beta"] > 0) & (x["beta"] < 1))
        assert np.all((x["alpha"] > 0) & (x["alpha"] < 1))
        assert abs(np.median(x["alpha"]) - np.exp(-np.log1p(np.exp(-3.0)))) < 5e-3
    kda = config(4)
    x = philox.token_inputs(kda, b % kda.batch, 0, h % kda.heads, np.arange(n), 1)
    assert x["alpha"].shape == (n, kda.d_k)
    assert np.all((x["alpha"] > 0.85) & (x["alpha"] < 1))
    m2 = config(3)
    x = philox.token_inputs(m2, b % m2.batch, 0, h % m2.heads, np.arange(n), 1)
    assert x["v"].shape == (n, 64) and x["k"].shape == (n, 128)
    assert np.all(x["beta"] > 0)
    assert abs(np.median(x["beta"]) - np.log1p(np.exp(-2.0))) < 0.01
    assert abs(np.mean(np.sum(x["k"].astype(np.float64) ** 2, -1)) - 1) < 0.02
    A = philox.mamba2_A(m2, np.arange(40)[:, None], np.arange(64)[None, :])
    assert A.min() > 1 and A.max() < 16


def test_vbar_norms():
    vb0 = philox.vbar_table(config(0))
    np.testing.assert_allclose(np.linalg.norm(vb0, axis=-1), 1, atol=1e-6)
    vb = philox.vbar_table(config(2))
    nrm = np.linalg.norm(vb, axis=-1)
    assert vb.shape == (36, 48, 128) and nrm.min() > 1 and nrm.max() < 4


def test_configs_are_the_five_workloads():
    assert sorted(CONFIGS) == [0, 1, 2, 3, 4]
    assert CONFIGS[2].units == 256 * 36 * 48
    assert [CONFIGS[i].form for i in range(5)] == [FORM_GDN] * 3 + [FORM_MAMBA2, FORM_KDA]


def test_philox_matches_published_known_answer_vectors(golden_dir):
    """The host generator against the published Philox4x32-10 known-answer vectors
    (tests/golden/philox4x32_10_kat.txt); the device generator is tested equal to
    the host one value by value, so this pins both."""
    import os
    rows = []
    with open(os.path.join(golden_dir, "philox4x32_10_kat.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                rows.append([int(x, 16) for x in line.split()])
    assert len(rows) == 3
    for r in rows:
        out = philox.philox4x32_10(*r[:4], *r[4:6])
        assert [int(x) for x in out] == r[6:10]
