"""Pins of the oracle's streaming causal conv (one chunk with a [K-1, C] cache), against
formulations that are not the oracle's own code:

- chunked processing from a zero cache equals the causal conv (im2col formulation, in numpy) of
  each stream's concatenated valid frames, with masked frames exactly zero and the final cache
  equal to the stream's last K-1 frames (zeros before the stream's start);
- the direct numpy statement of one chunk, with a non-zero cache.

The operation follows parakeet.cpp PR #102, "What changes": the streaming encoder keeps its own
depthwise conv with a cache; a causal conv over a stream only needs the K-1 previous frames.
"""
import numpy as np
import pytest

import oracle
from pinlib import np_stream_fwd, rel_err, stream_chunked_vs_whole


@pytest.mark.parametrize("K", [1, 2, 3, 4, 5, 7, 9, 15])
@pytest.mark.parametrize("T", [1, 3, 8, 17])
def test_chunks_equal_whole_stream(K, T):
    rng = np.random.default_rng(1000 * K + T)
    fails = stream_chunked_vs_whole(oracle.default(), rng, B=3, C=5, K=K, T=T, n_chunks=7,
                                    bias=(K % 2 == 1))
    assert not fails, fails


@pytest.mark.parametrize("K", [1, 3, 9])
def test_direct_statement_with_cache(K):
    rng = np.random.default_rng(K)
    x = rng.standard_normal((4, 7, 6)); w = rng.standard_normal((K, 6)); bias = rng.standard_normal(6)
    cache = rng.standard_normal((4, K - 1, 6))
    L = np.array([7, 0, 3, 1], np.int32)
    y, c = oracle.dwconv1d_stream_fwd(x, w, bias, cache, L)
    ry, rc = np_stream_fwd(x, w, bias, cache, L)
    assert rel_err(y, ry) <= 1e-12
    assert np.array_equal(c, rc)


def test_empty_chunk_keeps_cache_and_lengths_clamp():
    rng = np.random.default_rng(7)
    x = rng.standard_normal((2, 4, 3)); w = rng.standard_normal((5, 3))
    cache = rng.standard_normal((2, 4, 3))
    y, c = oracle.dwconv1d_stream_fwd(x, w, None, cache, np.array([0, -3], np.int32))
    assert np.all(y == 0.0) and np.array_equal(c, cache)
    y2, c2 = oracle.dwconv1d_stream_fwd(x, w, None, cache, np.array([99, 4], np.int32))
    y3, c3 = oracle.dwconv1d_stream_fwd(x, w, None, cache, None)
    assert np.array_equal(y2, y3) and np.array_equal(c2, c3)


def test_impulse_in_cache_reads_weights_backwards():
    """A unit impulse in cached frame j (zero chunk, zero bias) gives y[t] = w[j - t] for
    t <= j: the stored taps, read backwards along t, as for the forward impulse identity."""
    K, C = 6, 2
    w = np.arange(1.0, K * C + 1).reshape(K, C)
    for j in range(K - 1):
        cache = np.zeros((1, K - 1, C)); cache[0, j] = 1.0
        y, _ = oracle.dwconv1d_stream_fwd(np.zeros((1, K, C)), w, None, cache, None)
        for t in range(K):
            expect = w[j - t] if t <= j else np.zeros(C)
            assert np.array_equal(y[0, t], expect)
