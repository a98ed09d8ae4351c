"""Pins for the oracle's QKV projection (out = bf16_RNE(x w^T), fp64 sums),
the producer of q, k_new and v_new that the fused projection kernel feeds
into RoPE and the append ("Scaling TensorRT-LLM: Kernel Fusion and Inflight
Batching in Production", section "What Gets Fused").

Pins from outside the oracle's loop: exact integer arithmetic (small-integer
bf16 inputs, whose fp64 sums are exact) against an integer matmul; identity
and one-hot weights; a numpy fp64 matmul on random data (an independent
implementation), rounded by the pinned bf16 codec."""
import numpy as np
import torch

import oracle
from tests._util import bits16


def _b16(a):
    return bits16(torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16))


def _f(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def test_small_integers_are_exact():
    rng = np.random.default_rng(0)
    x = rng.integers(-2, 3, size=(5, 48))
    w = rng.integers(-2, 3, size=(7, 48))
    out = oracle.project_bf16(_b16(x), _b16(w))
    ref = x @ w.T                        # |sum| <= 48 * 4 < 2^8: exact in bf16 as well
    assert np.array_equal(_f(out), ref.astype(np.float64))
    # larger integers: the fp64 sum is still exact, the output is its single bf16 rounding
    x = rng.integers(-64, 65, size=(5, 48))
    w = rng.integers(-64, 65, size=(7, 48))
    out = oracle.project_bf16(_b16(x), _b16(w))
    assert np.array_equal(out, oracle.bf16_encode((x @ w.T).astype(np.float64)))


def test_identity_and_one_hot_weights():
    rng = np.random.default_rng(1)
    x = _b16(rng.standard_normal((6, 32)))
    eye = _b16(np.eye(32))
    assert np.array_equal(oracle.project_bf16(x, eye), x)
    sel = np.zeros((3, 32), np.float32)
    sel[0, 5] = 1.0
    sel[1, 0] = 1.0
    sel[2, 31] = -1.0
    out = oracle.project_bf16(x, _b16(sel))
    assert np.array_equal(out[:, 0], x[:, 5]) and np.array_equal(out[:, 1], x[:, 0])
    assert np.array_equal(out[:, 2], x[:, 31] ^ np.uint16(0x8000))


def test_random_against_a_numpy_fp64_matmul():
    rng = np.random.default_rng(2)
    x = _b16(rng.standard_normal((9, 256)))
    w = _b16(rng.standard_normal((40, 256)) / 16.0)
    out = oracle.project_bf16(x, w)
    ref = _f(x) @ _f(w).T
    assert np.array_equal(out, oracle.bf16_encode(ref))
