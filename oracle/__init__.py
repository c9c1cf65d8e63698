"""Oracle — plain, slow, obviously-correct CPU restatement of the denoise path.

TEST INFRASTRUCTURE ONLY.  Only `tests/`, `__graft_entry__.smoke()` and the
CPU-baseline leg of `bench.py` may import anything under `oracle/`; the CUDA
product path never does, and the two share no code (only the seeded input
generators in `synth/`).

Modules:
  model     fp64 numpy forward: prefill, canvas forward, LM-head entropy, the
            self-conditioning signal z = FFW(p0 E) and the block loops that carry it
  sampler   Entropy-Bound sampler step and block loop (integer decisions)
  anneal    the Report's default sampler: annealed entropy-bounded refinement over a
            uniform-noise canvas, adaptive stop, SplitMix64 draws
  absorbing absorbing forward process (invariant checks)

Every function is pinned by `tests/test_oracle_*.py` against closed forms,
brute force or library routines it does not use.  The whole-model composition
beyond its pinned parts is "parity unpinned": no logits, weights or
trajectories for it are published.
"""
