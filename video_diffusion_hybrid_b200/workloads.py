"""Named workloads of the hybrid attention core (shapes and modes only).

* tiny      : T=10, N=16 (4x4), H=2, d=32, L=8, fp32 -- two chunks, every
              pair on the softmax path, the linear branch reads text only.
* tiny_scan : T=30 variant of tiny, fp32, so that the scans carry video.
* small     : T=20 (4 chunks), N=240 (12x20), H=8, d=64, L=64, bf16;
              anchors 0 and 19.
* 768p      : T=90 latent frames (18 chunks), N=1008 (24x42 latent grid),
              H=24, d=128, L=512, B=1, bf16 inputs, fp32 state/accumulation;
              90,720 video tokens per head.
* long      : T=180, N=1008, H=24, d=128, L=512, B=2 (two seeds), bf16.
* sweep_N{n}_d{d} : VDA-only shapes at T=90, H=24, bf16.
* prof_d128 : the 768p shape cut to T=30 (about 1 GB of inputs, still larger
              than L2) for detailed profiler captures of the same kernels.

Each workload has its own seed (listed below); batch
element b draws from PCG64(seed * 1000 + b).
"""
from __future__ import annotations

from dataclasses import dataclass

from .synth import Shape


@dataclass(frozen=True)
class Workload:
    name: str
    shape: Shape
    dtype: str
    seed: int

    @property
    def tokens(self) -> int:
        return self.shape.B * self.shape.T * self.shape.N


def _w(name, B, T, N, H, d, L, dtype, seed):
    return Workload(name, Shape(B=B, T=T, N=N, H=H, d_k=d, d_v=d, L=L), dtype, seed)


WORKLOADS = {w.name: w for w in [
    _w("tiny", 1, 10, 16, 2, 32, 8, "f32", 1),
    _w("tiny_scan", 1, 30, 16, 2, 32, 8, "f32", 1),
    _w("small", 1, 20, 240, 8, 64, 64, "bf16", 2),
    _w("768p", 1, 90, 1008, 24, 128, 512, "bf16", 3),
    _w("long", 2, 180, 1008, 24, 128, 512, "bf16", 4),
    _w("prof_d128", 1, 30, 1008, 24, 128, 512, "bf16", 6),
] + [_w(f"sweep_N{n}_d{d}", 1, 90, n, 24, d, 512, "bf16", 5) for n in (256, 1008, 4032) for d in (64, 128, 256)]}
