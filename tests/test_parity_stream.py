"""GPU parity of the streaming causal conv1d with a cache (dwconv1d_stream_fwd) against the fp64
CPU oracle, element by element, through the C ABI.

Each test feeds a sequence of chunks to the GPU op and to the oracle, each from its own zero
cache, and compares every chunk's output (bf16 bar or float32 bar) and the cache after every chunk
(bitwise: the cache holds copies of input values).  Streaming workload: 64 streams, C=512, K=9,
bf16, chunks of 1, 4 and 16 frames with random valid lengths; edge cases cover every K with a
compiled window and runtime widths, C not a multiple of any vector, misaligned buffers (narrow
path), T below K-1, zero lengths and no lengths.
"""
import numpy as np
import pytest
import torch

import oracle
import speech_encoder_depthwise_b200 as dw
from gpuhelp import Guarded, assert_bf16_close, assert_f32_close, bf16_ulp, dev
from synth import bf16_round

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    from speech_encoder_depthwise_b200 import build
    build.build()
    dw.lib()


def run_stream(B, T, C, K, chunks, dtype, seed, offset=0, with_lengths=True, bias=True):
    """Feeds `chunks` random chunks through the GPU op and the oracle; checks every chunk."""
    rng = np.random.default_rng(seed)
    td = torch.bfloat16 if dtype == "bf16" else torch.float32
    rnd = bf16_round if dtype == "bf16" else (lambda a: a.astype(np.float32))
    w = rnd(rng.standard_normal((K, C)) / np.sqrt(K))
    b = rnd(rng.standard_normal(C) * np.sqrt(0.1)) if bias else None
    gw, gb = dev(w), dev(b)
    cache_g = Guarded((B, K - 1, C), td, offset=offset)
    cache_g.t.zero_()
    cache_o = np.zeros((B, K - 1, C))
    for i in range(chunks):
        x = rnd(rng.standard_normal((B, T, C)))
        L = rng.integers(0, T + 1, size=B).astype(np.int32) if with_lengths else None
        if with_lengths and B > 1:
            L[0] = T
        xg = Guarded((B, T, C), td, offset=offset)
        xg.t.copy_(torch.from_numpy(x).to(td))
        y = Guarded((B, T, C), td, offset=offset)
        dw.dwconv1d_stream_fwd(xg.t, gw, gb, y.t, cache_g.t if K > 1 else None,
                               dev(L) if L is not None else None)
        torch.cuda.synchronize()
        y.check_slack()
        cache_g.check_slack()
        ry, cache_o = oracle.dwconv1d_stream_fwd(x, w, b, cache_o, L)
        got = y.numpy()
        if dtype == "bf16":
            assert_bf16_close(got, ry)
        else:
            assert_f32_close(got, ry)
        Lc = np.full(B, T) if L is None else L
        for s in range(B):
            tail = got[s, Lc[s]:]
            assert np.all(tail == 0.0) and not np.any(np.signbit(tail)), "masked frames must be +0.0"
        assert np.array_equal(cache_g.numpy(), cache_o), f"cache differs after chunk {i}"


@pytest.mark.parametrize("T", [1, 4, 16])
def test_streaming_workload(T):
    run_stream(64, T, 512, 9, chunks=6, dtype="bf16", seed=T)


@pytest.mark.parametrize("K", [1, 2, 3, 4, 5, 6, 7, 9, 15, 20])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_widths(K, dtype):
    run_stream(3, 7, 24, K, chunks=5, dtype=dtype, seed=100 + K)


@pytest.mark.parametrize("C", [1, 3, 130, 520])
def test_channel_counts(C):
    run_stream(2, 5, C, 9, chunks=4, dtype="bf16", seed=C)


@pytest.mark.parametrize("K", [4, 9, 20])
def test_misaligned_buffers_take_the_narrow_path(K):
    run_stream(2, 6, 64, K, chunks=4, dtype="bf16", seed=7 + K, offset=1)


def test_no_lengths_and_no_bias():
    run_stream(3, 5, 16, 9, chunks=4, dtype="f32", seed=9, with_lengths=False, bias=False)


def test_chunks_shorter_than_the_cache():
    run_stream(4, 2, 32, 15, chunks=12, dtype="bf16", seed=11)


def test_stream_equals_whole_sequence_forward():
    """Chunked GPU outputs against the GPU's own whole-sequence causal dwconv1d_fwd: both within
    the bf16 bar of the oracle, and within two bf16 ulps of each other."""
    rng = np.random.default_rng(5)
    B, C, K, T, n = 8, 256, 9, 8, 10
    w = bf16_round(rng.standard_normal((K, C)) / 3.0)
    b = bf16_round(rng.standard_normal(C) * 0.3)
    xs = bf16_round(rng.standard_normal((B, n * T, C)))
    cache = torch.zeros(B, K - 1, C, dtype=torch.bfloat16, device="cuda")
    parts = []
    for i in range(n):
        x = dev(xs[:, i * T:(i + 1) * T], torch.bfloat16)
        y = torch.empty_like(x)
        dw.dwconv1d_stream_fwd(x, dev(w), dev(b), y, cache, None)
        parts.append(y.float().cpu().numpy())
    chunked = np.concatenate(parts, axis=1)
    whole = torch.empty(B, n * T, C, dtype=torch.bfloat16, device="cuda")
    dw.dwconv1d_fwd(dev(xs, torch.bfloat16), dev(w), dev(b), whole, None, K - 1)
    torch.cuda.synchronize()
    whole = whole.float().cpu().numpy()
    ref = oracle.dwconv1d_fwd(xs, w, b, None, K - 1)
    assert_bf16_close(chunked, ref)
    assert_bf16_close(whole, ref)
    assert np.all(np.abs(chunked - whole) <= 2 * bf16_ulp(ref) + 1e-5)
