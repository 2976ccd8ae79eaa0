"""SplitMix64, written from its published definition (oracle side).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

The OrbitQuant page ([OQ] Methodology, "Randomized Permuted Block-Hadamard
(RPBH) Rotation") says the permutation is drawn once per dimension and the
signs are Rademacher, but names no generator.  Reading taken: SplitMix64
(Steele, Lea & Flood, "Fast Splittable Pseudorandom Number Generators",
OOPSLA 2014) with its state initialised to the seed.  Each draw adds the
golden-ratio increment to the state and returns a bijective mix of it.

Pure-Python integers with explicit 64-bit masking: slow and obvious.
"""

MASK64 = (1 << 64) - 1
GOLDEN_GAMMA = 0x9E3779B97F4A7C15


class SplitMix64:
    """Sequential SplitMix64 stream: state_{n+1} = state_n + gamma; out = mix(state_{n+1})."""

    def __init__(self, seed: int):
        self.state = seed & MASK64

    def next(self) -> int:
        self.state = (self.state + GOLDEN_GAMMA) & MASK64
        z = self.state
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK64
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK64
        return z ^ (z >> 31)
