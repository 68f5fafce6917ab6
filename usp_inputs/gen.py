"""Counter-based seeded generators (SplitMix64 + Box-Muller) and the workload table.

SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom number
generators", OOPSLA 2014): the k-th output of a stream with seed s mixes the
state s + (k+1)*GAMMA (mod 2^64) with two xor-shift-multiply rounds. Normals use
the Box-Muller transform on two consecutive outputs (their top 53 bits as
uniforms); the cosine branch is kept and the sine branch dropped, so element e
of a tensor consumes stream outputs 2e and 2e+1.

Everything is written with torch int64 / float64 ops so the same code runs on
the CPU and on the GPU. int64 multiplication wraps modulo 2^64 on both
devices; tests pin this against exact Python integers. Each test generates a
tensor once and hands the same bytes to both sides, so a one-ulp difference in
a float64 log/cos between devices can never split them.
"""
from __future__ import annotations

import math

import torch

M64 = (1 << 64) - 1
GAMMA = 0x9E3779B97F4A7C15
_C1 = 0xBF58476D1CE4E5B9
_C2 = 0x94D049BB133111EB
_CHUNK = 1 << 24


def _i64(x: int) -> int:
    """Reinterpret an unsigned 64-bit Python int as the signed int64 value."""
    x &= M64
    return x - (1 << 64) if x >= (1 << 63) else x


def _srl(x: torch.Tensor, s: int) -> torch.Tensor:
    """Logical right shift of an int64 tensor holding uint64 bit patterns."""
    return (x >> s) & ((1 << (64 - s)) - 1)


def splitmix64(seed: int, start: int, n: int, device="cpu") -> torch.Tensor:
    """Outputs start..start+n-1 of the SplitMix64 stream `seed`, as int64 bit patterns."""
    k1 = torch.arange(start + 1, start + n + 1, dtype=torch.int64, device=device)
    z = k1 * _i64(GAMMA) + _i64(seed)
    z = (z ^ _srl(z, 30)) * _i64(_C1)
    z = (z ^ _srl(z, 27)) * _i64(_C2)
    return z ^ _srl(z, 31)


def _normal_f64(seed: int, e0: int, n: int, device) -> torch.Tensor:
    z = splitmix64(seed, 2 * e0, 2 * n, device).view(n, 2)
    u1 = (_srl(z[:, 0], 11) + 1).to(torch.float64) * (2.0 ** -53)   # (0, 1]
    u2 = _srl(z[:, 1], 11).to(torch.float64) * (2.0 ** -53)         # [0, 1)
    return torch.sqrt(-2.0 * torch.log(u1)) * torch.cos((2.0 * math.pi) * u2)


def normal_bf16(seed: int, shape, device="cpu") -> torch.Tensor:
    """N(0,1) samples rounded to bf16, element e from stream outputs 2e, 2e+1."""
    n = 1
    for s in shape:
        n *= int(s)
    out = torch.empty(n, dtype=torch.bfloat16, device=device)
    for e0 in range(0, n, _CHUNK):
        m = min(_CHUNK, n - e0)
        out[e0:e0 + m] = _normal_f64(seed, e0, m, device).to(torch.bfloat16)
    return out.view(*shape)


def uniform_f32(seed: int, shape, device="cpu") -> torch.Tensor:
    """Uniform [0,1) samples (top 24 bits of each output) as float32."""
    n = 1
    for s in shape:
        n *= int(s)
    out = torch.empty(n, dtype=torch.float32, device=device)
    for e0 in range(0, n, _CHUNK):
        m = min(_CHUNK, n - e0)
        z = splitmix64(seed, e0, m, device)
        out[e0:e0 + m] = (_srl(z, 40).to(torch.float64) * (2.0 ** -24)).to(torch.float32)
    return out.view(*shape)


def peaky_positions(seed: int, S: int, frac: float = 0.01) -> list[int]:
    """floor(frac*S) distinct token positions by a partial Fisher-Yates shuffle of 0..S-1.

    Step a swaps slot a with slot a + (x_a mod (S-a)), x_a the a-th SplitMix64
    output of `seed`; the first m slots are the chosen positions.
    """
    m = int(math.floor(frac * S))
    xs = [int(v) & M64 for v in splitmix64(seed, 0, m, "cpu").tolist()]
    perm = list(range(S))
    for a in range(m):
        j = a + xs[a] % (S - a)
        perm[a], perm[j] = perm[j], perm[a]
    return sorted(perm[:m])


# The five workloads, each with the tensor shapes and structure of the long-context
# regime on the pages (16K to 256K tokens, causal LLM attention, GQA, peaky keys).
WORKLOADS = {
    1: dict(name="tiny_causal_fwd_s256_usp2x2", B=1, S=256, Hq=2, Hkv=2, D=64,
            causal=True, P_u=2, P_r=2, seed=0, peaky=False),
    2: dict(name="causal_fwd_s16k_ring8", B=1, S=16384, Hq=32, Hkv=32, D=128,
            causal=True, P_u=1, P_r=8, seed=2000, peaky=False),
    3: dict(name="gqa_causal_fwd_s128k_usp4x2", B=1, S=131072, Hq=32, Hkv=8, D=128,
            causal=True, P_u=4, P_r=2, seed=3000, peaky=False),
    4: dict(name="causal_bwd_s32k_ring4", B=2, S=32768, Hq=16, Hkv=16, D=128,
            causal=True, P_u=1, P_r=4, seed=4000, peaky=False),
    5: dict(name="noncausal_peaky_s256k_ring16", B=1, S=262144, Hq=16, Hkv=16, D=128,
            causal=False, P_u=1, P_r=16, seed=5000, peaky=True),
}

PEAKY_SCALE = 8.0


def workload(cfg, device="cpu", which=("q", "k", "v", "do"), **override) -> dict:
    """Global-layout [B, S, H, D] bf16 tensors of a workload.

    Seeds: q = base+0, k = base+1, v = base+2, dO = base+3, peaky positions = base+4.
    With peaky=True every head of K at the chosen positions is scaled by 8 (exact in bf16).
    `override` replaces shape fields (used for reduced-size parity cases).
    """
    w = dict(WORKLOADS[cfg]) if isinstance(cfg, int) else dict(cfg)
    w.update(override)
    B, S, Hq, Hkv, D = w["B"], w["S"], w["Hq"], w["Hkv"], w["D"]
    base = w["seed"]
    out = {"spec": w}
    shapes = {"q": (B, S, Hq, D), "k": (B, S, Hkv, D), "v": (B, S, Hkv, D), "do": (B, S, Hq, D)}
    offs = {"q": 0, "k": 1, "v": 2, "do": 3}
    for name in which:
        out[name] = normal_bf16(base + offs[name], shapes[name], device)
    if w.get("peaky") and "k" in out:
        pos = peaky_positions(base + 4, S)
        idx = torch.tensor(pos, dtype=torch.int64, device=device)
        out["k"][:, idx] = (out["k"][:, idx].float() * PEAKY_SCALE).to(torch.bfloat16)
        out["peaky_positions"] = pos
    return out
