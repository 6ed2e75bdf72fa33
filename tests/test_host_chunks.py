"""User chunking of the host-to-host forward (host logic, no GPU)."""
import torch

from prototype_sketch_attention_b200 import binding


def check_cover(off, parts):
    R = len(off) - 1
    assert parts[0][0] == 0 and parts[-1][1] == R
    for (a, b), (c, _) in zip(parts, parts[1:]):
        assert a < b == c
    # no part without tokens unless the whole batch has none
    if off[-1] > 0:
        assert all(off[b] > off[a] for a, b in parts)


def test_user_chunks_cover_and_balance():
    gen = torch.Generator().manual_seed(3)
    for trial in range(200):
        R = int(torch.randint(1, 60, (1,), generator=gen))
        n = torch.randint(0, 5000, (R,), generator=gen)
        n[torch.rand(R, generator=gen) < 0.2] = 0
        off = torch.cat([torch.zeros(1, dtype=torch.int64), torch.cumsum(n, 0)])
        for chunks in (1, 2, 4, 7):
            parts = binding.user_chunks(off, chunks)
            assert 1 <= len(parts) <= chunks
            check_cover(off.tolist(), parts)


def test_user_chunks_equal_users():
    off = torch.arange(0, 4001, 1000, dtype=torch.int64)
    assert binding.user_chunks(off, 4) == [(0, 1), (1, 2), (2, 3), (3, 4)]
    assert binding.user_chunks(off, 2) == [(0, 2), (2, 4)]
    assert binding.user_chunks(off, 1) == [(0, 4)]
    assert binding.user_chunks(torch.zeros(1, dtype=torch.int64), 4) == []
