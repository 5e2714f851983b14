"""Seeded synthetic inputs shaped like the pages' workloads.

This module holds no arithmetic of the method (no quantiser, no contraction):
it only draws random numbers.  Both the CPU oracle and the CUDA path are fed
the arrays it returns, so they always see identical inputs.

Recipe (numpy PCG64 via ``default_rng(seed)``; substreams from ``spawn`` in the
order weight tensors, then activations, then masks):
  * weights  W ~ N(0, 0.02^2), fp32, [out_features][in_features]
    ("bitnetv2-model" README, "Technical Details": initializer range 0.02);
  * activations X ~ N(0, 1), fp32 (bf16 where the workload is bf16 I/O);
  * H-BitLinear FFN activations carry element-wise Bernoulli(0.01) outliers
    scaled by 10.

Workload shapes follow the pages' models: the 256/512 tiny model
("BitNet TinyDialogues 1.58b", "Arquitetura"), the 512/2048 H-BitLinear model
("bitnetv2-model", "Architecture Overview") and the 2B model's 2560/6912
projections (nnterp encyclopedia "bitnet", "Printout" and "Config").
"""
from dataclasses import dataclass, field

import numpy as np

W_STD = 0.02


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str                    # "linear" | "decode" | "prefill" | "ffn" | "hffn"
    dims: dict = field(default_factory=dict)
    description: str = ""


WORKLOADS = {
    "tiny": Workload("tiny", "linear", {"M": 8, "K": 256, "N": 512},
                     "single BitLinear of the 256/512 tiny model, fp32 in/out"),
    "hffn": Workload("hffn", "hffn", {"M": 1024, "D": 512, "F": 2048},
                     "H-BitLinear FFN 512->2048->512 with SiLU, 8 seqs x 128 tokens"),
    "decode": Workload("decode", "decode",
                       {"M": (1, 4, 16), "KN": ((2560, 2560), (2560, 6912), (6912, 2560))},
                       "decode GEMV sweep at 2B-model projection shapes, bf16 out"),
    "prefill": Workload("prefill", "prefill", {"M": 4096, "KN": ((2560, 6912), (6912, 2560))},
                        "prefill GEMM, RMSNorm(N(0,1)) activations, bf16 out"),
    "ffn": Workload("ffn", "ffn", {"M": 2048, "H": 2560, "I": 6912},
                    "W1.58A8 FFN block with ffn_sub_norm and residual, bf16 I/O"),
}


def streams(seed, n):
    """n independent PCG64 generators spawned from one seed."""
    return np.random.default_rng(seed).spawn(n)


def weight(rng, n_out, n_in, std=W_STD):
    return (rng.standard_normal((n_out, n_in), dtype=np.float32) * np.float32(std))


def activations(rng, M, K):
    return rng.standard_normal((M, K), dtype=np.float32)


def outliers(rng, X, p=0.01, factor=10.0):
    """Multiply a Bernoulli(p) element mask of X by ``factor``."""
    mask = rng.random(X.shape) < p
    out = X.copy()
    out[mask] *= np.float32(factor)
    return out


def to_bf16_bits(x):
    """Round fp32 to bf16 bit patterns (ties to even); input generation only."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def bf16_bits_to_f32(b):
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


# ----------------------------------------------------------- per workload

def linear_inputs(M, K, N, seed=0):
    """W [N][K] and X [M][K] for one BitLinear."""
    rw, rx = streams(seed, 2)
    return {"W": weight(rw, N, K), "X": activations(rx, M, K)}


def hffn_inputs(M=1024, D=512, F=2048, seed=0):
    r1, r2, rx, rm = streams(seed, 4)
    W1 = weight(r1, F, D)
    W2 = weight(r2, D, F)
    X = outliers(rm, activations(rx, M, D))
    return {"W1": W1, "W2": W2, "X": X}


def ffn_inputs(M=2048, H=2560, I=6912, seed=0):
    """Gate, up, down weights and a bf16 residual input (returned as bits and
    as its exact fp32 widening)."""
    rg, ru, rd, rx = streams(seed, 4)
    Wg = weight(rg, I, H)
    Wu = weight(ru, I, H)
    Wd = weight(rd, H, I)
    xb = to_bf16_bits(activations(rx, M, H))
    return {"Wg": Wg, "Wu": Wu, "Wd": Wd, "x_bf16": xb, "x": bf16_bits_to_f32(xb)}
