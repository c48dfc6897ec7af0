"""The five synthetic workloads, each named by what it is and its sizes.

Shapes follow the ParaChromo paper (mdpi.com/2079-9292/15/13/2750): 64-bead
regions with 12-bead overlaps (§3.2), chromosome-scale chains of 32 tiles (§5.5),
2658 regions x 2 guidance settings x up to 1000 samples (§3.1, §3.2), DDIM step
sweeps from 50 to 1000 (§5.4.3).  The pages publish no dataset for this path, so
every input is drawn by :mod:`synth`.
"""
from __future__ import annotations

from dataclasses import dataclass, field


@dataclass(frozen=True)
class Workload:
    name: str
    C: int                    # chains (or regions)
    T: int                    # tiles per chain (1 = untiled)
    B: int                    # samples per tile
    S: int = 50               # DDIM steps
    eta: float = 0.0
    w: float = 0.0            # guidance weight
    s_c: float = 0.1          # conditional-stream noise scale of the stand-in
    s_u: float = 0.3          # unconditional-stream noise scale
    overlap: int = 12
    sync_every: int = 1       # K (0: never project)
    sigma: str = "unit"       # walk step sigma mode for x0
    seed: int = 0
    extra: dict = field(default_factory=dict)

    @property
    def n_maps(self) -> int:
        return self.C * self.T * self.B

    @property
    def map_steps(self) -> int:
        return self.n_maps * self.S


WORKLOADS = {
    # 1 chain x 4 tiles x 8 samples, 50 steps, eta 0, w 0, eps_c noise 0.1,
    # projection after every step, recovery at the end, seed 0
    "chain4_b8_s50": Workload("chain4_b8_s50", C=1, T=4, B=8, S=50, w=0.0, s_c=0.1),
    # chromosome-scale chain: 32 tiles x 1000 samples, CFG w=1 with eps_c
    # (noise 0.1) and eps_u (noise 0.3), 50 steps, eta 0, projection every
    # step, x0 walk sigma ~ U(0.8, 1.2) per tile
    "chain32_b1000_cfg": Workload("chain32_b1000_cfg", C=1, T=32, B=1000, S=50, w=1.0,
                                  s_c=0.1, s_u=0.3, sigma="tile_uniform"),
    # step-count sweep on the 32-tile chain, 100 samples, w 0, eps_c noise 0.1
    "chain32_b100_sweep": Workload("chain32_b100_sweep", C=1, T=32, B=100, S=50, w=0.0,
                                   extra={"S": (50, 100, 250, 500, 1000),
                                          "eta": (0.0, 1.0)}),
    # genome-wide untiled: 2658 regions x {w=0, w=1} x 256 samples, 50 steps
    "genome2658_b256_untiled": Workload("genome2658_b256_untiled", C=2658, T=1, B=256,
                                        S=50, sync_every=0,
                                        extra={"w": (0.0, 1.0), "chunk_maps": 1 << 16}),
    # recovery at scale: 1,000,000 noisy point-cloud maps viewed as
    # 31,250 chains x 32 tiles x 1 sample
    "recovery_1m": Workload("recovery_1m", C=31250, T=32, B=1, S=0, sync_every=0),
}
