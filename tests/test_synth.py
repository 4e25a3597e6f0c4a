"""The seeded input recipe (CPU only): what the generator promises its callers, the oracle tests and the GPU
path alike."""
import numpy as np
import pytest
import torch

from residual_kv_cache_delta_b200 import synth


def test_streams_are_reproducible_and_keyed():
    w = synth.workload(1, seq_len=256)
    a = synth.raw_kv_np(w, 0, 0, 0, 0, 0, 256)
    assert np.array_equal(a, synth.raw_kv_np(w, 0, 0, 0, 0, 0, 256))
    # a row does not depend on how the positions are split into calls
    assert np.array_equal(a[100:200], synth.raw_kv_np(w, 0, 0, 0, 0, 100, 200))
    others = [synth.raw_kv_np(w, *key, 0, 256) for key in ((1, 0, 0, 0), (0, 1, 0, 0), (0, 0, 1, 0), (0, 0, 0, 1))]
    assert all(not np.array_equal(a, o) for o in others)  # layer, sequence, kv head, K/V each change the stream
    assert not np.array_equal(a, synth.raw_kv_np(synth.workload(1, seq_len=256, seed=7), 0, 0, 0, 0, 0, 256))


def test_tokens_follow_the_stated_model():
    w = synth.workload(1, seq_len=4096)
    x = synth.raw_kv_np(w, 0, 0, 0, 0, 0, 4096)
    mu = synth.shared_mu(w, 0, 0, 0)
    assert np.linalg.norm(mu) == pytest.approx(w.mu_norm, rel=1e-5)
    c = synth.centers(w, 0, 0, 0)
    cid = synth.cluster_ids(np.arange(4096), w.hash_mod, w.clusters)
    noise = (x - mu[None, :] - c[cid]) / w.sigma
    assert abs(noise.mean()) < 0.02 and noise.std() == pytest.approx(1.0, abs=0.02)
    # tokens of one cluster recur at distant positions: the long-range similarity the search exploits
    same = np.nonzero(cid == cid[4000])[0]
    assert same.min() < 2000 < 4000 <= same.max()


def test_basis_is_orthonormal_with_positive_r_diagonal():
    w = synth.workload(1)
    b = synth.basis(w, 0, 0, 0)
    assert b.shape == (w.head_dim, w.rank)
    assert np.allclose(b.T @ b, np.eye(w.rank), atol=1e-12)
    g = synth._rng(w.seed, synth.ROLE_BASIS, 0, 0, 0, 0).standard_normal((w.head_dim, w.rank))
    assert np.all(np.diag(b.T @ g) > 0)  # R = Q^T G has a positive diagonal
    mu, bs = synth.params(w, 0)
    assert mu.dtype == torch.float32 and mu.shape == (w.num_kv_heads, 2, w.head_dim)
    assert bs.dtype == torch.bfloat16 and bs.shape == (w.num_kv_heads, 2, w.head_dim, w.rank)


def test_serving_mix_lengths_and_random_block_placement():
    w = synth.workload(4)
    lens = synth.seq_lengths(w)
    assert len(lens) == w.batch and lens.min() >= w.min_len and lens.max() <= w.seq_len
    assert np.array_equal(lens, synth.seq_lengths(w))
    # log-uniform: about half the sequences lie below the geometric mean of the bounds
    assert 0.25 < np.mean(lens < np.sqrt(w.min_len * w.seq_len)) < 0.75
    bt, nb = synth.block_tables(w, lens, extra_tokens=1)
    used = bt[bt >= 0]
    assert len(used) == nb and np.array_equal(np.sort(used), np.arange(nb))  # every block once
    assert not np.array_equal(used, np.arange(nb))                           # not in order
    for s, L in enumerate(lens):
        assert np.sum(bt[s] >= 0) == -(-(int(L) + 1) // w.ref_stride)
    bt1, nb1 = synth.block_tables(synth.workload(2), [32768] * 8)
    assert np.array_equal(bt1.reshape(-1), np.arange(nb1))                 # contiguous workloads: identity
