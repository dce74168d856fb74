"""The seeded input generator that both the GPU path and the oracle consume,
pinned to things outside itself: the SplitMix64 reference outputs, the
Box-Muller relation between its uniforms and normals, the moments of the
normals, and the geometry of the sink construction."""
import math
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workload  # noqa: E402


def test_splitmix64_reference_outputs():
    # the first five outputs of SplitMix64 (Steele, Lea and Flood, OOPSLA 2014)
    # from state 1234567, as printed by the algorithm's reference implementation
    expected = [6457827717110365317, 3203168211198807973, 9817491932198370423,
                4593380528125082431, 16408922859458223821]
    assert [int(x) for x in workload.splitmix64(1234567, 5)] == expected


def test_box_muller_pairs():
    # elements 2t, 2t+1 are r cos(2 pi u2), r sin(2 pi u2) with r^2 = -2 ln u1,
    # (u1, u2) the stream's uniforms 2t and 2t+1
    seed, stream, n = 11, 3, 4096
    x = workload.normals(seed, stream, 0, n).astype(np.float64)
    u = workload.uniforms(seed, stream, 0, n)
    u1, u2 = u[0::2], u[1::2]
    r2 = x[0::2] ** 2 + x[1::2] ** 2
    np.testing.assert_allclose(r2, -2.0 * np.log(u1), rtol=2e-6, atol=1e-9)
    ang = np.mod(np.arctan2(x[1::2], x[0::2]), 2 * np.pi)
    d = np.abs(ang - 2 * np.pi * u2)
    d = np.minimum(d, 2 * np.pi - d)
    assert d.max() < 1e-4
    # any slice regenerates the same values
    np.testing.assert_array_equal(workload.normals(seed, stream, 1001, 50), x[1001:1051].astype(np.float32))


def test_uniforms_and_normals_moments():
    u = workload.uniforms(5, 1, 0, 1 << 20)
    assert u.min() > 0.0 and u.max() <= 1.0
    assert abs(u.mean() - 0.5) < 3e-3 and abs(u.var() - 1.0 / 12) < 2e-3
    x = workload.normals(5, 2, 0, 1 << 20).astype(np.float64)
    # N(0, 1): mean 0, variance 1, fourth moment 3 (sampling error ~ 1/sqrt(n) = 1e-3)
    assert abs(x.mean()) < 5e-3 and abs(x.var() - 1.0) < 1e-2 and abs((x ** 4).mean() - 3.0) < 5e-2
    # distinct streams and seeds are not the same sequence
    assert not np.array_equal(workload.normals(5, 2, 0, 64), workload.normals(5, 3, 0, 64))
    assert not np.array_equal(workload.normals(5, 2, 0, 64), workload.normals(6, 2, 0, 64))


@pytest.mark.parametrize("delta", [0.0, 8.0])
def test_sink_construction_geometry(delta):
    B, H, Hkv, N, d, ns = 2, 4, 2, 64, 128, 4
    W = workload.make_sink_workload(B, H, Hkv, N, d, ns, delta, seed=9)
    group = H // Hkv
    u = workload._unit_vectors(9, B, Hkv, d)          # the construction's unit vectors
    np.testing.assert_allclose(np.linalg.norm(u, axis=-1), 1.0, rtol=1e-12)
    beta = delta * math.sqrt(d) / 8.0
    for b in range(B):
        for g in range(Hkv):
            qs = W.q[b, g * group:(g + 1) * group].astype(np.float64).reshape(-1, d)
            k = W.k[b, g].astype(np.float64)
            # non-sink keys have u projected out (up to FP32 rounding of the rows)
            assert np.abs(k[ns:] @ u[b, g]).max() < 1e-4
            # queries: N(0, I) plus 8u, so the component along u averages 8
            assert abs((qs @ u[b, g]).mean() - 8.0) < 0.3
            # sink keys: N(0, I) plus beta u, so the component along u averages beta
            assert abs((k[:ns] @ u[b, g]).mean() - beta) < 1.6
    # the scaled logit gap sink - non-sink is delta on average
    s = np.einsum("bhnd,bhmd->bhnm", W.q.astype(np.float64),
                  np.repeat(W.k.astype(np.float64), group, axis=1)) / math.sqrt(d)
    gap = s[..., :ns].mean() - s[..., ns:].mean()
    assert abs(gap - delta) < 0.5
    # values are N(0, 1) and untouched by the construction
    assert abs(W.v.mean()) < 0.05 and abs(W.v.var() - 1.0) < 0.05


def test_kv_head_slice_matches_full_problem():
    full = workload.make_sink_workload(1, 8, 4, 96, 64, 4, 8.0, seed=13)
    part = workload.make_sink_workload(1, 8, 4, 96, 64, 4, 8.0, seed=13, kv_heads=(1, 3))
    np.testing.assert_array_equal(part.q, full.q[:, 2:6])
    np.testing.assert_array_equal(part.k, full.k[:, 1:3])
    np.testing.assert_array_equal(part.v, full.v[:, 1:3])
