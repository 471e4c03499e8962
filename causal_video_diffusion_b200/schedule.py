"""The clip's denoising schedule: which forwards a 5-s clip runs and at which noise levels.

UnStep paper (arXiv 2609.32518):
* Table 4 -- Self Forcing's four denoising steps, raw u in {1000, 750, 500, 250}, after the
  shift-5 mapping sigma = 5 u' / (1 + 4 u') with u' = u / 1000 (sigma = 1, 15/16, 5/6, 5/8),
  DiT label t = 1000 sigma; the clean-cache pass runs at sigma = 0 (Self Forcing) or the
  near-clean sigma* = 0.02 (UnStep), label 0.
* Table 3 -- seven chunks of three latent frames; the first chunk takes four denoising steps,
  each later chunk four (Self Forcing) or two (UnStep); every chunk adds one clean-cache forward
  (35 and 23 forwards per clip).
The pages do not list the two timesteps of UnStep's later chunks; the reading taken here is the
two-step grid of the same mapping, raw u in {1000, 500} (the four-step grid is u = 1000 (1 - i/4),
the two-step one u = 1000 (1 - i/2)).
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Tuple

SHIFT = 5.0
FOUR_STEPS = (1000, 750, 500, 250)
TWO_STEPS = (1000, 500)
CLEAN_SIGMA = {"self_forcing": 0.0, "unstep": 0.02}


def shifted_sigma(u: float, shift: float = SHIFT) -> float:
    """Noise level of raw timestep u (0..1000) after the shift mapping."""
    x = u / 1000.0
    return shift * x / (1.0 + (shift - 1.0) * x)


@dataclass(frozen=True)
class Forward:
    chunk: int
    step: int          # denoising step within the chunk; -1 for the clean-cache pass
    sigma: float       # noise level of the latent this forward sees
    label: float       # DiT timestep label
    next_sigma: float  # noise level the latent is renoised to after this forward

    @property
    def clean(self) -> bool:
        return self.step < 0


def clip_schedule(kind: str = "unstep", chunks: int = 7) -> List[Forward]:
    """Every DiT forward of one clip, in order."""
    if kind not in CLEAN_SIGMA:
        raise ValueError(kind)
    out: List[Forward] = []
    clean = CLEAN_SIGMA[kind]
    for c in range(chunks):
        steps = FOUR_STEPS if (c == 0 or kind == "self_forcing") else TWO_STEPS
        sig = [shifted_sigma(u) for u in steps]
        for i, s in enumerate(sig):
            nxt = sig[i + 1] if i + 1 < len(sig) else clean   # last step -> clean-cache level
            out.append(Forward(c, i, s, 1000.0 * s, nxt))
        out.append(Forward(c, -1, clean, 0.0, clean))
    return out


def forwards_per_chunk(kind: str = "unstep", chunks: int = 7) -> Tuple[int, ...]:
    counts = [0] * chunks
    for f in clip_schedule(kind, chunks):
        counts[f.chunk] += 1
    return tuple(counts)
