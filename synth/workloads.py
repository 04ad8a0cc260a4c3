"""Synthetic workloads shaped like the pages' (no trained weights exist here).

Each workload lists its tensors as (name, rows, cols, tensor_id), with the generator seed,
sigma and storage dtype.  Weights are row-major [rows, cols] (out x in for linear layers)
and groups run along cols.

* small_fp32       -- one fp32 256x512 matrix, N(0, 0.02^2), seed 0 (1024 groups).
* outlier_sweep    -- fp32 4096x4096, N(0, 1), seed 1, 1% of columns (41) replaced by
                      10 * Student-t(3) values; swept over ternary / 2 / 3 / 4 bits.
* needle_45m       -- bf16 stand-in for the ~45M-parameter model of page "How Needle 2
                      Compresses to a Single Binary" ("Stage 1": attention with GQA, an
                      MLP), seed 2: embedding 8192x768; 8 layers of q/o 768x768, k/v
                      768x256, up 768x2048, down 2048x768; one 768x1000 tensor (padding).
* llama7b          -- bf16 7B-scale weight set ("standard 7B parameter models", page
                      "Performance Differences Between 2-Bit and 4-Bit Quantization in
                      Needle", "Inference Speed and Computational Overhead"), seed 3:
                      32 layers of q/k/v/o 4096x4096, gate/up 11008x4096, down 4096x11008.
* gemv_7b          -- the two MLP shapes 11008x4096 and 4096x11008, seed 4, 2-bit, with
                      bf16 N(0,1) activations at batch 1 and 8.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np


@dataclass(frozen=True)
class Tensor:
    name: str
    rows: int
    cols: int
    tensor_id: int

    @property
    def numel(self) -> int:
        return self.rows * self.cols

    @property
    def groups(self) -> int:
        return self.rows * (-(-self.cols // 128))


@dataclass(frozen=True)
class Workload:
    name: str
    dtype: str  # "f32" or "bf16"
    seed: int
    sigma: float
    tensors: tuple
    bits: tuple
    extra: dict = field(default_factory=dict)

    @property
    def numel(self) -> int:
        return sum(t.numel for t in self.tensors)

    @property
    def groups(self) -> int:
        return sum(t.groups for t in self.tensors)


SMALL_FP32 = Workload("small_fp32_256x512", "f32", 0, 0.02, (Tensor("w", 256, 512, 0),), (2,))

OUTLIER_SWEEP = Workload("outlier_sweep_4096x4096", "f32", 1, 1.0, (Tensor("w", 4096, 4096, 0),),
                         (0, 2, 3, 4), {"outlier_frac": 0.01, "outlier_scale": 10.0,
                                        "perm_id": 1, "student_id": 2})


def _needle_tensors():
    out = [("embed", 8192, 768)]
    for layer in range(8):
        out += [(f"l{layer}.q", 768, 768), (f"l{layer}.o", 768, 768),
                (f"l{layer}.k", 768, 256), (f"l{layer}.v", 768, 256),
                (f"l{layer}.up", 768, 2048), (f"l{layer}.down", 2048, 768)]
    out.append(("head", 768, 1000))
    return tuple(Tensor(n, r, c, i) for i, (n, r, c) in enumerate(out))


NEEDLE_45M = Workload("needle_45m_bf16", "bf16", 2, 0.02, _needle_tensors(), (2,))


def _llama_tensors(layers: int = 32):
    out = []
    for layer in range(layers):
        out += [(f"l{layer}.q", 4096, 4096), (f"l{layer}.k", 4096, 4096),
                (f"l{layer}.v", 4096, 4096), (f"l{layer}.o", 4096, 4096),
                (f"l{layer}.gate", 11008, 4096), (f"l{layer}.up", 11008, 4096),
                (f"l{layer}.down", 4096, 11008)]
    return tuple(Tensor(n, r, c, i) for i, (n, r, c) in enumerate(out))


LLAMA_7B = Workload("llama7b_bf16", "bf16", 3, 0.02, _llama_tensors(), (2, 4))

GEMV_7B = Workload("gemv_7b_mlp", "bf16", 4, 0.02,
                   (Tensor("gate", 11008, 4096, 0), Tensor("down", 4096, 11008, 1)), (2,),
                   {"x_ids": (100, 101), "x_sigma": 1.0, "batches": (1, 8)})

ALL = (SMALL_FP32, OUTLIER_SWEEP, NEEDLE_45M, LLAMA_7B, GEMV_7B)


def outlier_columns(cols: int, seed: int, perm_id: int, frac: float) -> np.ndarray:
    """First round(frac*cols) entries of a Fisher-Yates shuffle of range(cols), driven by
    word x0 of Philox counters 0, 1, ... of stream (seed, perm_id): j = i + w_i mod (n-i)."""
    from synth import philox_words
    k = int(round(frac * cols))
    words = philox_words(cols, seed, perm_id)
    a = np.arange(cols)
    for i in range(cols - 1):
        j = i + int(words[i] % np.uint64(cols - i))
        a[i], a[j] = a[j], a[i]
    return np.sort(a[:k])


def outlier_sweep_host() -> np.ndarray:
    """The fp32 4096x4096 outlier matrix, generated on the host."""
    from synth import normal_f64
    wl = OUTLIER_SWEEP
    t = wl.tensors[0]
    w = (wl.sigma * normal_f64(t.numel, wl.seed, t.tensor_id)).astype(np.float32).reshape(t.rows, t.cols)
    cols = outlier_columns(t.cols, wl.seed, wl.extra["perm_id"], wl.extra["outlier_frac"])
    n_out = t.rows * cols.size
    z = normal_f64(4 * n_out, wl.seed, wl.extra["student_id"]).reshape(n_out, 4)
    t3 = z[:, 0] / np.sqrt((z[:, 1] ** 2 + z[:, 2] ** 2 + z[:, 3] ** 2) / 3.0)
    w[:, cols] = (wl.extra["outlier_scale"] * t3).astype(np.float32).reshape(t.rows, cols.size)
    return w
