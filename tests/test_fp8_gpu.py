"""E4M3 (FP8) inputs through the C ABI against the fp64 oracle.

The oracle computes the exact attention of the dequantized inputs (E4M3
values are exact in bf16, so they go to the oracle as bf16 with the softmax
scale times descale_q * descale_k, and its O is multiplied by descale_v).
The kernel rounds the probabilities to E4M3 before P V, so O is checked
element by element against the bound derived in tests/fp8_bound.py; lse,
which the kernel takes from the unrounded sum, keeps the bf16 tolerance.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_52_b200 import _binding as fb
from exact_io_aware_52_b200 import workloads
from tests import fp8_bound
from tests.gpu_util import TOL_LSE, run_gpu

pytestmark = pytest.mark.gpu
D = 128
SCALE = 1.0 / math.sqrt(D)


def e4m3_inputs(B, H, N, seed, std=1.0, H_kv=None, Nk=None, vstd=1.0):
    g = torch.Generator().manual_seed(seed)
    H_kv = H if H_kv is None else H_kv
    Nk = N if Nk is None else Nk
    q = (torch.randn(B, H, N, D, generator=g) * std).to(torch.float8_e4m3fn)
    k = (torch.randn(B, H_kv, Nk, D, generator=g) * std).to(torch.float8_e4m3fn)
    v = (torch.randn(B, H_kv, Nk, D, generator=g) * vstd).to(torch.float8_e4m3fn)
    return q, k, v


def check_e4m3(q, k, v, causal, scale, descale=(0.0, 0.0, 0.0), k_len=None, rows=None, out_dtype=torch.float32,
               num_splits=0, flags=0):
    dq, dk, dv = (x if x > 0 else 1.0 for x in descale)
    o, lse = run_gpu(q, k, v, causal, scale, k_len=k_len, out_dtype=out_dtype, num_splits=num_splits,
                     descale=descale, flags=flags)
    sig = float(np.float32(scale * dq * dk))
    kl = None if k_len is None else list(k_len)
    o_ref, lse_ref = oracle.attention_f64(q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16), causal,
                                          sig, k_len=kl, rows=rows)
    o_ref = o_ref * dv
    bound = fp8_bound.bound_rows(q.double().numpy(), k.double().numpy(), v.double().numpy() * dv, causal, sig,
                                 k_len=kl, rows=rows)
    if out_dtype == torch.bfloat16:
        bound = bound + 2.0 ** -8 * np.abs(o_ref) + 1e-6  # bf16 rounding of O
    d = q.shape[-1]
    o_rows = o.reshape(-1, d).double().numpy()
    l_rows = lse.reshape(-1).double().numpy()
    if rows is not None:
        o_rows, l_rows = o_rows[rows], l_rows[rows]
    o_ref = o_ref.reshape(o_rows.shape)
    lse_ref = lse_ref.reshape(l_rows.shape)
    empty = np.isneginf(lse_ref)
    assert np.all(np.isneginf(l_rows[empty])) and np.all(o_rows[empty] == 0.0)
    assert np.all(np.isfinite(o_rows))
    err = np.abs(o_rows - o_ref)
    worst = np.unravel_index(np.argmax(err - bound), err.shape)
    assert np.all(err <= bound), (float(err[worst]), float(bound[worst]), worst)
    live = ~empty
    rel = np.abs(l_rows[live] - lse_ref[live]) / np.maximum(np.abs(lse_ref[live]), 1.0)
    assert rel.size == 0 or rel.max() <= TOL_LSE, float(rel.max())
    use = err[live] / bound[live]
    return {"max_dO": float(err.max()), "mean_dO": float(err.mean()), "max_bound_use": float(use.max()) if use.size else 0.0,
            "max_rel_lse": float(rel.max()) if rel.size else 0.0}


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 127, 128, 129, 383, 640])
def test_ragged_shapes(N, causal):
    q, k, v = e4m3_inputs(2, 3, N, seed=3000 + N + causal)
    check_e4m3(q, k, v, causal, SCALE)


@pytest.mark.parametrize("causal", [False, True])
def test_key_padding_edges(causal):
    N = 300
    k_len = [0, 1, N - 1, N, N + 50, -5, 128, 129]
    q, k, v = e4m3_inputs(len(k_len), 2, N, seed=3001 + causal)
    check_e4m3(q, k, v, causal, SCALE, k_len=k_len)


def test_grouped_heads_and_more_units_than_sms():
    q, k, v = e4m3_inputs(2, 32, 700, seed=3002, H_kv=8)
    check_e4m3(q, k, v, True, SCALE, k_len=[700, 333])


def test_descale_factors():
    """Scaled E4M3 tensors: values q * 0.5, k * 2, v * 0.25."""
    q, k, v = e4m3_inputs(1, 4, 500, seed=3003, std=2.0, vstd=4.0)
    for causal in (False, True):
        check_e4m3(q, k, v, causal, SCALE, descale=(0.5, 2.0, 0.25))


@pytest.mark.parametrize("flags", [0, fb.FA_FLAG_EAGER_RESCALE])
@pytest.mark.parametrize("std", [2.0, 4.0])
def test_large_logits(std, flags):
    """Peaked rows: a few keys carry the weight, the bound's worst case."""
    q, k, v = e4m3_inputs(1, 4, 2048, seed=3004 + int(std), std=std)
    print(check_e4m3(q, k, v, True, SCALE, flags=flags))


@pytest.mark.parametrize("flags", [0, fb.FA_FLAG_EAGER_RESCALE])
def test_slowly_growing_maximum(flags):
    """Scores that grow along the keys by about 0.8 (head 0) and 1.6 (head 1)
    natural units per key tile (1.2 and 2.3 binary orders): the row maximum
    moves on most tiles, often by less than the rescale threshold 1.75
    (weights then reach up to 2^8.75 before rounding) and often by more."""
    B, H, N = 1, 2, 1024
    g = torch.Generator().manual_seed(3010 + flags)
    q = torch.zeros(B, H, N, D)
    k = torch.zeros(B, H, N, D)
    q[..., 0] = 1.0
    q[..., 1] = 0.5
    k[0, 0, :, 0] = torch.linspace(0.0, 0.8 * N / 128, N)
    k[0, 1, :, 0] = torch.linspace(0.0, 1.6 * N / 128, N)
    k[..., 1] = torch.randn(B, H, N, generator=g)
    v = torch.randn(B, H, N, D, generator=g)
    q, k, v = (t.to(torch.float8_e4m3fn) for t in (q, k, v))
    for causal in (False, True):
        print(check_e4m3(q, k, v, causal, 1.0, flags=flags))


@pytest.mark.parametrize("splits", [3, 8])
def test_split_kv(splits):
    q, k, v = e4m3_inputs(2, 3, 200, seed=3005 + splits, Nk=1500)
    for causal in (False, True):
        check_e4m3(q, k, v, causal, SCALE, num_splits=splits)


def test_bf16_output():
    q, k, v = e4m3_inputs(2, 4, 555, seed=3006)
    check_e4m3(q, k, v, True, SCALE, out_dtype=torch.bfloat16)


def test_deterministic():
    q, k, v = e4m3_inputs(1, 8, 1000, seed=3007)
    o1, l1 = run_gpu(q, k, v, True, SCALE)
    o2, l2 = run_gpu(q, k, v, True, SCALE)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_long_context_workload():
    w = workloads.WORKLOADS[9]
    q, k, v, _ = workloads.make_inputs(w)
    assert q.dtype == torch.float8_e4m3fn
    print("workload 9:", check_e4m3(q, k, v, w.causal, w.scale, rows=workloads.sample_rows(w)))
