"""The device Philox4x32-10 that sv_accept draws its uniforms from, pinned
directly (B200): the published known-answer vectors, and word-for-word
agreement with the oracle's independent implementation on 10^6 counters under
keys with both words set (Salmon, Moraes, Dror and Shaw, SC'11)."""
import os

import numpy as np
import pytest
import torch

import oracle
import speculative_decoding_rl_b200 as sv

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "philox4x32_10_kat.txt")


def _device_words(key: int, ctrs: np.ndarray) -> np.ndarray:
    c = torch.from_numpy(np.ascontiguousarray(ctrs, dtype=np.uint32).view(np.int32)).cuda()
    out = torch.full_like(c, -1)
    sv.sv_testing_philox4x32_10(key, c, out, c.shape[0])
    torch.cuda.synchronize()
    return out.cpu().numpy().view(np.uint32)


def test_device_philox_known_answers():
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        v = [int(x, 16) for x in line.split()]
        ctr, key, want = v[0:4], v[4:6], v[6:10]
        got = _device_words(key[0] | (key[1] << 32), np.array([ctr], dtype=np.uint32))
        assert [int(x) for x in got[0]] == want


@pytest.mark.parametrize("key", [0, 0x00000000FFFFFFFF, 0xFFFFFFFF00000000, 0x0123456789ABCDEF,
                                 0xDEADBEEFCAFEF00D])
def test_device_philox_matches_oracle_on_a_million_counters(key):
    n = 1_000_000
    rng = np.random.default_rng(key & 0xFFFF)
    ctrs = rng.integers(0, 2**32, size=(n, 4), dtype=np.uint64).astype(np.uint32)
    # the counters sv_accept uses: {sequence, node, tag, 0}
    ctrs[: 4096, 3] = 0
    ctrs[: 4096, 2] = np.arange(4096) & 1
    got = _device_words(key, ctrs)
    want = oracle.philox4x32_10_many(ctrs, [key & 0xFFFFFFFF, key >> 32])
    bad = np.nonzero((got != want).any(axis=1))[0]
    assert bad.size == 0, f"{bad.size} counters differ, first {bad[:5]}"
