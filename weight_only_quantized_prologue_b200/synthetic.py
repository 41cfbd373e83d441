"""Seeded synthetic inputs shared by the tests, the bench and the smoke run.

This module only draws random numbers; it holds none of the quantization or
GEMM arithmetic.  The shapes and distributions are those of the pages' toy
models: ``x = torch.randn(M, K)`` in bf16 and ``nn.Linear``'s default
initialisation U(-1/sqrt(fan_in), 1/sqrt(fan_in)) for the weight and the bias
("Define a linear model..." sections of the quantized-Linear pages).

Draw order from one ``torch.Generator("cpu")`` seeded with ``seed``: x, W, bias.
"""

import numpy as np
import torch


def _uniform(gen, shape, bound):
    return (torch.rand(shape, generator=gen, dtype=torch.float32) * 2.0 - 1.0) * bound


def linear_inputs(M, K, N, seed=0, bias=True):
    """Returns (x bf16 [M, K], W fp32 [N, K], bias bf16 [N] or None) as CPU
    torch tensors."""
    gen = torch.Generator("cpu").manual_seed(int(seed))
    x = torch.randn((M, K), generator=gen, dtype=torch.float32).to(torch.bfloat16)
    bound = 1.0 / float(np.sqrt(K))
    w = _uniform(gen, (N, K), bound)
    b = _uniform(gen, (N,), bound).to(torch.bfloat16) if bias else None
    return x, w, b


def activations(M, K, seed):
    """x ~ N(0, 1) in bf16, [M, K] (calibration and input batches)."""
    gen = torch.Generator("cpu").manual_seed(int(seed))
    return torch.randn((M, K), generator=gen, dtype=torch.float32).to(torch.bfloat16)


def mlp_weights(in_features=256, hidden=512, out_features=128, seed=0):
    """Weights of the static-FP8 page's two-layer model (no bias), drawn in
    fp32 and stored in the model dtype bf16: (W1 [hidden, in], W2 [out, hidden])."""
    gen = torch.Generator("cpu").manual_seed(int(seed))
    w1 = _uniform(gen, (hidden, in_features), 1.0 / float(np.sqrt(in_features))).to(torch.bfloat16)
    w2 = _uniform(gen, (out_features, hidden), 1.0 / float(np.sqrt(hidden))).to(torch.bfloat16)
    return w1, w2
