"""Seeded synthetic inputs for the FP8 linear layer and NestedFP workloads.

This module only draws random numbers with the shapes, value distributions
and outlier structure of the workloads; it holds none of the method's
arithmetic (no scaling, no FP8 conversion, no products).  Both the CUDA path
(tests, benchmark) and the CPU oracle take their inputs from here.

Generator: numpy ``Generator(PCG64)`` seeded with a ``SeedSequence`` built from
(workload id, shape index, M index, role), so every tensor of every case is
reproducible on any machine and independent of the others.

Workloads (activations x [M, K], weights w [N, K]; shapes are K -> N):

==========  ==========================================  =======================  =====================================  ==============
workload    shapes (K -> N)                             M                        activations                            weights (fp16)
==========  ==========================================  =======================  =====================================  ==============
small       512->512                                    16                       f32 N(0,1); 1% of entries x20          N(0, 0.02)
decode7b    4096->12288, 4096->4096, 4096->22016,       1, 4, 8                  f32 N(0,1); 0.5% of entries x30        N(0, 0.02)
            11008->4096  (QKV, O, gate+up, down)
prefill7b   same four                                   512, 1024, 2048          f32 Student-t(4) / sqrt(2)             N(0, 0.02)
nested7b    4096->12288, 11008->4096                    1, 16, 128, 1024         f16 N(0,1)                             N(0, 0.02)
llama70b    8192->10240, 8192->8192, 8192->57344,       1, 2, 4, ..., 4096       f32 Student-t(3), unscaled             N(0, 0.01)
            28672->8192
==========  ==========================================  =======================  =====================================  ==============
"""
from __future__ import annotations

import dataclasses

import numpy as np


@dataclasses.dataclass(frozen=True)
class Workload:
    wid: int
    name: str
    shapes: tuple          # ((K, N, label), ...)
    ms: tuple              # token counts
    act: str               # activation recipe key
    w_sigma: float
    out: str               # output dtype of the layer ("bf16" or "f16")


WORKLOADS = {
    "small": Workload(1, "small", ((512, 512, "proj"),), (16,), "normal_outl_1pct_x20", 0.02, "bf16"),
    "decode7b": Workload(2, "decode7b",
                         ((4096, 12288, "qkv"), (4096, 4096, "o"), (4096, 22016, "gate_up"),
                          (11008, 4096, "down")),
                         (1, 4, 8), "normal_outl_0p5pct_x30", 0.02, "bf16"),
    "prefill7b": Workload(3, "prefill7b",
                          ((4096, 12288, "qkv"), (4096, 4096, "o"), (4096, 22016, "gate_up"),
                           (11008, 4096, "down")),
                          (512, 1024, 2048), "student_t4_unit", 0.02, "bf16"),
    "nested7b": Workload(4, "nested7b", ((4096, 12288, "qkv"), (11008, 4096, "down")),
                         (1, 16, 128, 1024), "normal_f16", 0.02, "f16"),
    "llama70b": Workload(5, "llama70b",
                         ((8192, 10240, "qkv"), (8192, 8192, "o"), (8192, 57344, "gate_up"),
                          (28672, 8192, "down")),
                         (1, 2, 4, 8, 16, 32, 64, 128, 256, 512, 1024, 2048, 4096),
                         "student_t3", 0.01, "bf16"),
}

ROLE_ACT = 1
ROLE_W = 2


def rng(wid: int, shape_idx: int, m_idx: int, role: int, extra: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([wid, shape_idx, m_idx, role, extra])))


def activations(recipe: str, M: int, K: int, g: np.random.Generator) -> np.ndarray:
    """Activation matrix [M, K] drawn by recipe name."""
    if recipe == "normal_outl_1pct_x20":
        x = g.standard_normal((M, K), dtype=np.float32)
        mask = g.random((M, K)) < 0.01
        return np.where(mask, x * np.float32(20.0), x).astype(np.float32)
    if recipe == "normal_outl_0p5pct_x30":
        x = g.standard_normal((M, K), dtype=np.float32)
        mask = g.random((M, K)) < 0.005
        return np.where(mask, x * np.float32(30.0), x).astype(np.float32)
    if recipe == "student_t4_unit":
        return (g.standard_t(4.0, size=(M, K)) / np.sqrt(2.0)).astype(np.float32)
    if recipe == "student_t3":
        return g.standard_t(3.0, size=(M, K)).astype(np.float32)
    if recipe == "normal_f16":
        return g.standard_normal((M, K), dtype=np.float32).astype(np.float16)
    raise KeyError(recipe)


def weights_f16(N: int, K: int, sigma: float, g: np.random.Generator) -> np.ndarray:
    """fp16 weights ~ N(0, sigma), [N, K] row-major (K contiguous)."""
    w = g.standard_normal((N, K), dtype=np.float32)
    w *= np.float32(sigma)
    return w.astype(np.float16)


def case(workload: str, shape_idx: int, m_idx: int, m_override: int | None = None,
         k_override: int | None = None, n_override: int | None = None):
    """Inputs of one (shape, M) case of a workload: (x, w_f16).

    The overrides shrink a case (for instance to a few tiles plus a ragged
    tail) while keeping the workload's distributions."""
    wl = WORKLOADS[workload]
    K, N, _ = wl.shapes[shape_idx]
    M = wl.ms[m_idx] if m_override is None else m_override
    K = K if k_override is None else k_override
    N = N if n_override is None else n_override
    x = activations(wl.act, M, K, rng(wl.wid, shape_idx, m_idx, ROLE_ACT))
    w = weights_f16(N, K, wl.w_sigma, rng(wl.wid, shape_idx, 0, ROLE_W))
    return x, w


def weights(workload: str, shape_idx: int, copy: int = 0, k_override=None, n_override=None):
    """Weights of one shape; ``copy`` > 0 draws an independent copy of the same
    distribution (used to rotate weights so that no copy is L2 resident)."""
    wl = WORKLOADS[workload]
    K, N, _ = wl.shapes[shape_idx]
    K = K if k_override is None else k_override
    N = N if n_override is None else n_override
    return weights_f16(N, K, wl.w_sigma, rng(wl.wid, shape_idx, 0, ROLE_W, copy))


def acts(workload: str, shape_idx: int, m_idx: int, M: int | None = None, K: int | None = None):
    wl = WORKLOADS[workload]
    K0, _, _ = wl.shapes[shape_idx]
    M = wl.ms[m_idx] if M is None else M
    K = K0 if K is None else K
    return activations(wl.act, M, K, rng(wl.wid, shape_idx, m_idx, ROLE_ACT))
