"""Seeded synthetic inputs shared by the tests, the oracle checks and the bench.

This module draws random numbers and rounds them to the storage types; it
holds none of the method's arithmetic (no kurtosis, no quantiser, no layout),
so the CUDA path and the CPU oracle can both be fed from it.

Workload recipe (the stand-in for trained checkpoints, which the pages measure
on): for every matrix, drawn in this order from one seeded generator,
  1. W = 0.02 * N(0, 1)  [n, k];
  2. n_t distinct input columns chosen uniformly, sorted;
  3. those columns replaced by 0.02 * Student-t(nu=3), built as
     Z / sqrt((Z1^2 + Z2^2 + Z3^2) / 3) from four independent normals;
  4. W rounded to BF16 (round to nearest even from float32).
The norm gain is g = 1 + 0.1 * N(0, 1) [k] in float32, one draw per norm:
q/k/v share the attention input norm, gate/up the post-attention norm, the LM
head uses the final norm, and o/down have no norm in front (g = 1, passed as
None).  Activations are x = N(0, 1) [m, k] rounded to BF16.

Shapes follow the decoder layers of the pages' models: 1.5B-class (hidden 1536,
intermediate 8960, 28 layers, 2 KV heads of 128) and 4B-class (hidden 2560,
intermediate 9728, KV width 1024); the LM head is 131072 x 3072.  The number of
Student-t columns is round(0.015 * k) unless a workload says otherwise.

Seeds: every matrix gets its own generator seeded from
numpy.random.SeedSequence([seed, layer, slot]).  CPU and CUDA generators give
different streams for the same seed; a test that compares two implementations
draws once and hands the same tensors to both.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

# slot numbers inside a layer (also the seed component)
PROJ = ("q", "k", "v", "o", "gate", "up", "down")
_GAIN_OF = {"q": "attn", "k": "attn", "v": "attn", "o": None,
            "gate": "mlp", "up": "mlp", "down": None, "lm_head": "final", "single": "single"}
_GAIN_SLOT = {"attn": 100, "mlp": 101, "final": 102, "single": 103}
_X_SLOT = 200


@dataclass(frozen=True)
class MatrixSpec:
    name: str
    n: int          # out_features (rows of W)
    k: int          # in_features (columns, input channels)
    n_t: int        # heavy-tailed (Student-t) columns

    @property
    def gain_group(self):
        return _GAIN_OF.get(self.name, "single")


def _nt(k: int) -> int:
    return int(round(0.015 * k))


def layer_specs(hidden: int, inter: int, kv: int):
    return [MatrixSpec("q", hidden, hidden, _nt(hidden)),
            MatrixSpec("k", kv, hidden, _nt(hidden)),
            MatrixSpec("v", kv, hidden, _nt(hidden)),
            MatrixSpec("o", hidden, hidden, _nt(hidden)),
            MatrixSpec("gate", inter, hidden, _nt(hidden)),
            MatrixSpec("up", inter, hidden, _nt(hidden)),
            MatrixSpec("down", hidden, inter, _nt(inter))]


SINGLE_512 = MatrixSpec("single", 512, 512, 10)
LAYER_1P5B = layer_specs(1536, 8960, 256)
LAYER_4B = layer_specs(2560, 9728, 1024)
N_LAYERS_1P5B = 28
LM_HEAD_N, LM_HEAD_K = 131072, 3072
LM_HEAD_FRACTIONS = (0.0, 0.01, 0.05, 0.10)
BATCH_SWEEP = (1, 2, 4, 8, 16, 32)


def lm_head_spec(frac: float) -> MatrixSpec:
    return MatrixSpec("lm_head", LM_HEAD_N, LM_HEAD_K, int(round(frac * LM_HEAD_K)))


def _seed(*key: int) -> int:
    return int(np.random.SeedSequence(list(key)).generate_state(1, dtype=np.uint64)[0] >> 1)


def _gen(device, *key: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(_seed(*key))
    return g


def student_t3(shape, gen: torch.Generator, device) -> torch.Tensor:
    z = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    c = torch.randn((3,) + tuple(shape), generator=gen, device=device, dtype=torch.float32)
    return z / torch.sqrt((c * c).sum(0) / 3.0)


def weight(spec: MatrixSpec, seed: int = 0, layer: int = 0, device="cpu",
           slot: int | None = None) -> torch.Tensor:
    """BF16 weight [n, k] with spec.n_t Student-t columns."""
    if slot is None:
        slot = PROJ.index(spec.name) if spec.name in PROJ else 50
    gen = _gen(device, seed, layer, slot)
    w = torch.randn((spec.n, spec.k), generator=gen, device=device, dtype=torch.float32) * 0.02
    if spec.n_t > 0:
        cols = torch.randperm(spec.k, generator=gen, device=device)[: spec.n_t].sort().values
        w[:, cols] = 0.02 * student_t3((spec.n, spec.n_t), gen, device)
    return w.to(torch.bfloat16)


def gain(spec: MatrixSpec, seed: int = 0, layer: int = 0, device="cpu"):
    """float32 gain [k] of the norm in front of this matrix, or None (g = 1)."""
    grp = spec.gain_group
    if grp is None:
        return None
    gen = _gen(device, seed, layer, _GAIN_SLOT[grp])
    return 1.0 + 0.1 * torch.randn(spec.k, generator=gen, device=device, dtype=torch.float32)


def activations(k: int, m: int = 1, seed: int = 0, layer: int = 0, slot: int = 0,
                device="cpu") -> torch.Tensor:
    """BF16 activations [m, k] ~ N(0, 1)."""
    gen = _gen(device, seed, layer, _X_SLOT + slot)
    return torch.randn((m, k), generator=gen, device=device, dtype=torch.float32).to(torch.bfloat16)


def bits(t: torch.Tensor) -> np.ndarray:
    """Raw uint16 bits of a BF16 tensor as a host NumPy array."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def from_bits(a: np.ndarray, device="cpu") -> torch.Tensor:
    """BF16 tensor from raw uint16 bits."""
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint16).view(np.int16)).view(
        torch.bfloat16).to(device)
