"""Pins of the seeded input generators (usp_inputs) against exact integer arithmetic."""
import math

import torch

from usp_inputs import GAMMA, normal_bf16, peaky_positions, splitmix64, uniform_f32, workload

M64 = (1 << 64) - 1


def _splitmix64_exact(seed, k):
    """k-th output (0-based) of SplitMix64, in exact Python integers."""
    z = (seed + (k + 1) * GAMMA) & M64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & M64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & M64
    return z ^ (z >> 31)


def test_splitmix64_published_first_outputs_seed0():
    # first outputs of SplitMix64 seeded with 0, as published with the reference C code
    got = [v & M64 for v in splitmix64(0, 0, 3).tolist()]
    assert got[0] == 0xE220A8397B1DCDAF
    assert got == [_splitmix64_exact(0, k) for k in range(3)]


def test_splitmix64_matches_exact_integers():
    for seed in (0, 1, 3000, 2**63 + 12345, M64):
        start = 1_000_003
        got = [v & M64 for v in splitmix64(seed, start, 64).tolist()]
        assert got == [_splitmix64_exact(seed, start + k) for k in range(64)]


def test_normal_bf16_statistics_and_determinism():
    x = normal_bf16(77, (1 << 20,)).double()
    assert abs(x.mean().item()) < 5e-3
    assert abs(x.std().item() - 1.0) < 5e-3
    assert torch.equal(normal_bf16(77, (1 << 20,)), normal_bf16(77, (1024, 1024)).flatten())
    assert not torch.equal(normal_bf16(78, (64,)), normal_bf16(77, (64,)))


def test_uniform_range():
    u = uniform_f32(5, (100000,))
    assert u.min() >= 0 and u.max() < 1 and abs(u.mean().item() - 0.5) < 5e-3


def test_peaky_positions_and_workload():
    S = 262144
    pos = peaky_positions(5004, S)
    assert len(pos) == math.floor(0.01 * S) == 2621
    assert len(set(pos)) == len(pos) and 0 <= min(pos) and max(pos) < S
    w = workload(5, which=("k",), S=4096, Hq=2, Hkv=2)
    base = workload(5, which=("k",), S=4096, Hq=2, Hkv=2, peaky=False)
    pos = w["peaky_positions"]
    assert len(pos) == 40
    ratio = w["k"][:, pos].float() / base["k"][:, pos].float().where(base["k"][:, pos] != 0, torch.ones(()))
    nz = base["k"][:, pos] != 0
    assert torch.all(ratio[nz] == 8.0)
    mask = torch.ones(4096, dtype=torch.bool)
    mask[pos] = False
    assert torch.equal(w["k"][:, mask], base["k"][:, mask])
