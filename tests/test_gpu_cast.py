"""Bit-exactness of the device E4M3 cast (the routine the attention kernel
applies to S*P) against the oracle's codec: every FP32 bit pattern for S = 1,
every non-negative pattern for S = 16, 256, 448 (P is never negative in the
kernel), and a sample of negative ones.  NaN inputs compare by NaN-ness."""
import numpy as np
import pytest

import oracle

pytestmark = pytest.mark.gpu

CHUNK = 1 << 26


def _patterns(torch, start, n, dev):
    x = torch.arange(start, start + n, dtype=torch.int64, device=dev)
    x = torch.where(x >= 2 ** 31, x - 2 ** 32, x).to(torch.int32)
    return x.view(torch.float32)


def _check_range(torch, S, lo, hi):
    from online_softmax_tcgen05_b200 import fp8_e4m3_scale_cast
    dev = torch.device("cuda")
    out = torch.empty(CHUNK, dtype=torch.uint8, device=dev)
    for start in range(lo, hi, CHUNK):
        n = min(CHUNK, hi - start)
        x = _patterns(torch, start, n, dev)
        fp8_e4m3_scale_cast(x, out[:n], S)
        got = out[:n].cpu().numpy()
        want = oracle.e4m3_encode_bits(start, n, S)
        bits = np.arange(start, start + n, dtype=np.uint64).astype(np.uint32)
        isnan = np.isnan(bits.view(np.float32))
        bad = (got != want) & ~isnan
        assert not bad.any(), (S, hex(start + int(np.flatnonzero(bad)[0])))
        assert np.all((got[isnan] & 0x7F) == 0x7F)


def test_cast_exhaustive_S1():
    import torch
    _check_range(torch, 1.0, 0, 1 << 32)


@pytest.mark.parametrize("S", [16.0, 256.0, 448.0])
def test_cast_nonnegative_patterns(S):
    import torch
    _check_range(torch, S, 0, 1 << 31)


@pytest.mark.parametrize("S", [16.0, 256.0, 448.0])
def test_cast_negative_sample(S):
    import torch
    # negative patterns from -2^-20 to -2^10 in magnitude, whole binades
    _check_range(torch, S, 0x80000000 | (107 << 23), 0x80000000 | (137 << 23))


def test_cast_ragged_lengths():
    import torch
    from online_softmax_tcgen05_b200 import fp8_e4m3_scale_cast
    rng = np.random.default_rng(0)
    for n in (1, 7, 8, 9, 15, 17, 1023, 4097):
        x = (rng.standard_normal(n) * 100).astype(np.float32)
        g = torch.empty(n, dtype=torch.uint8, device="cuda")
        fp8_e4m3_scale_cast(torch.from_numpy(x).cuda(), g, 3.0)
        assert np.array_equal(g.cpu().numpy(), oracle.e4m3_encode(x, S=3.0)), n
