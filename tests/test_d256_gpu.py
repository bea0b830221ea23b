"""Head dimension 256 (its own kernel: one 128-row query tile per work unit,
two score buffers in TMEM) through the C ABI against the fp64 oracle, at the
parity tolerances of tests/gpu_util.py."""
import math

import pytest
import torch

from exact_io_aware_52_b200 import _binding as fb
from exact_io_aware_52_b200 import workloads
from tests.gpu_util import check_case, check_workload, run_gpu

pytestmark = pytest.mark.gpu
D = 256
SCALE = 1.0 / math.sqrt(D)


def rand_inputs(B, H, N, seed, std=1.0, H_kv=None, Nk=None):
    g = torch.Generator().manual_seed(seed)
    H_kv = H if H_kv is None else H_kv
    Nk = N if Nk is None else Nk
    q = (torch.randn(B, H, N, D, generator=g) * std).to(torch.bfloat16)
    k = (torch.randn(B, H_kv, Nk, D, generator=g) * std).to(torch.bfloat16)
    v = torch.randn(B, H_kv, Nk, D, generator=g).to(torch.bfloat16)
    return q, k, v


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 7, 127, 128, 129, 200, 383, 640])
def test_ragged_shapes(N, causal):
    q, k, v = rand_inputs(2, 3, N, seed=2000 + N * 7 + causal)
    check_case(q, k, v, causal, SCALE)


def test_more_units_than_sms():
    """2 * 20 * 9 = 360 units on the persistent grid; one key tile (N = 100)
    and two (N = 129, 256) exercise the short pipelines."""
    q, k, v = rand_inputs(2, 20, 1100, seed=2001)
    for causal in (False, True):
        check_case(q, k, v, causal, SCALE)
    for N in (100, 129, 256):
        q, k, v = rand_inputs(3, 60, N, seed=2002 + N)
        check_case(q, k, v, True, SCALE)


@pytest.mark.parametrize("causal", [False, True])
def test_key_padding_edges(causal):
    N = 300
    k_len = [0, 1, N - 1, N, N + 50, -5, 128, 129]
    q, k, v = rand_inputs(len(k_len), 2, N, seed=2003 + causal)
    check_case(q, k, v, causal, SCALE, k_len=k_len)


@pytest.mark.parametrize("H_kv", [1, 2])
def test_grouped_kv_heads(H_kv):
    q, k, v = rand_inputs(2, 4, 333, seed=2004 + H_kv, H_kv=H_kv)
    check_case(q, k, v, True, SCALE, k_len=[333, 250])


def test_monotone_logits_force_rescale_every_tile():
    """The row maximum moves on every key tile: every tile rescales O while the
    previous tile's P V product may still be running."""
    B, H, N = 1, 2, 1024
    q = torch.zeros(B, H, N, D)
    k = torch.zeros(B, H, N, D)
    q[..., 0] = 1.0
    k[..., 0] = torch.linspace(-20, 60, N)
    g = torch.Generator().manual_seed(2005)
    v = torch.randn(B, H, N, D, generator=g).to(torch.bfloat16)
    for flags in (0, fb.FA_FLAG_EAGER_RESCALE):
        for causal in (False, True):
            check_case(q.to(torch.bfloat16), k.to(torch.bfloat16), v, causal, 1.0, flags=flags)


@pytest.mark.parametrize("std", [4.0, 8.0])
@pytest.mark.parametrize("flags", [0, fb.FA_FLAG_EAGER_RESCALE])
def test_large_logits(std, flags):
    q, k, v = rand_inputs(1, 4, 2048, seed=2006 + int(std) + flags, std=std)
    check_case(q, k, v, True, SCALE, flags=flags)


def test_bf16_output():
    q, k, v = rand_inputs(2, 4, 555, seed=2007)
    check_case(q, k, v, True, SCALE, out_dtype=torch.bfloat16, tol_max=2e-2, tol_mean=2e-3)


@pytest.mark.parametrize("splits", [3, 8])
def test_split_kv(splits):
    q, k, v = rand_inputs(2, 3, 200, seed=2008 + splits, Nk=1500)
    for causal in (False, True):
        check_case(q, k, v, causal, SCALE, num_splits=splits)
    check_case(q, k, v, True, SCALE, k_len=[1500, 130], num_splits=splits, out_dtype=torch.bfloat16,
               tol_max=2e-2, tol_mean=2e-3)


def test_fewer_queries_than_keys():
    q, k, v = rand_inputs(1, 4, 100, seed=2009, Nk=2000)
    check_case(q, k, v, True, SCALE)


def test_deterministic():
    q, k, v = rand_inputs(1, 8, 1000, seed=2010)
    o1, l1 = run_gpu(q, k, v, True, SCALE)
    o2, l2 = run_gpu(q, k, v, True, SCALE)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_long_context_workload():
    stats = check_workload(workloads.WORKLOADS[8])
    print(f"workload 8: {stats}")
