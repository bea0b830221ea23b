"""Queries against a longer (cached) key sequence, and the key-split forward
with its log-sum-exp merge, through the C ABI against the fp64 oracle.

With N_q queries and N_k keys, query i sits at key position i + N_k - N_q, so
the causal mask allows keys j <= i + N_k - N_q.  With S > 1 splits each row's
keys are cut into S contiguous ranges, each range gives a partial O and lse,
and a second kernel merges them; the result must meet the same tolerances as
the single-pass kernel.  The workspace starts as NaN so a partial that the
split pass fails to write reaches the output.
"""
import math

import pytest
import torch

from exact_io_aware_52_b200 import _binding as fb
from tests.gpu_util import check_case, run_gpu

pytestmark = pytest.mark.gpu


def rect_inputs(B, H, H_kv, Nq, Nk, d, seed, std=1.0):
    g = torch.Generator().manual_seed(seed)
    q = (torch.randn(B, H, Nq, d, generator=g) * std).to(torch.bfloat16)
    k = (torch.randn(B, H_kv, Nk, d, generator=g) * std).to(torch.bfloat16)
    v = torch.randn(B, H_kv, Nk, d, generator=g).to(torch.bfloat16)
    return q, k, v


# ------------------------------------------------------------ N_q != N_k, one pass
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Nq,Nk", [(1, 1000), (100, 777), (256, 1024), (129, 4000), (300, 129)])
def test_fewer_or_more_queries_than_keys(Nq, Nk, d, causal):
    """Unequal query and key counts without splitting; with N_q > N_k under the
    causal mask the first N_q - N_k rows have no key (O = 0, lse = -inf)."""
    q, k, v = rect_inputs(2, 2, 2, Nq, Nk, d, seed=Nq * 7 + Nk + d + causal)
    check_case(q, k, v, causal, 1.0 / math.sqrt(d))


# ------------------------------------------------------------ the split forward
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("splits", [2, 3, 8, 1000])
def test_split_parity(splits, d, causal):
    """S = 2, 3, 8 and more splits than key tiles (one tile per split)."""
    q, k, v = rect_inputs(2, 3, 3, 200, 1500, d, seed=splits + d + 10 * causal)
    check_case(q, k, v, causal, 1.0 / math.sqrt(d), num_splits=splits)


@pytest.mark.parametrize("causal", [False, True])
def test_split_square_problem(causal):
    """Splits on an N_q = N_k problem: under the causal mask the early query
    blocks have no key in the late splits."""
    q, k, v = rect_inputs(1, 4, 4, 1000, 1000, 128, seed=21 + causal)
    check_case(q, k, v, causal, 1.0 / math.sqrt(128), num_splits=4)


@pytest.mark.parametrize("d", [64, 128])
def test_split_key_padding_empty_splits(d):
    """Key lengths that leave whole splits (and whole rows) without a key."""
    k_len = [0, 1, 127, 128, 130, 900, 2000, -3]
    q, k, v = rect_inputs(len(k_len), 2, 2, 64, 2000, d, seed=22 + d)
    check_case(q, k, v, True, 1.0 / math.sqrt(d), k_len=k_len, num_splits=8)
    check_case(q, k, v, False, 1.0 / math.sqrt(d), k_len=k_len, num_splits=5)


@pytest.mark.parametrize("causal", [False, True])
def test_split_grouped_heads(causal):
    """Grouped key/value heads (H = 8, H_kv = 2) with splits."""
    q, k, v = rect_inputs(2, 8, 2, 130, 3000, 128, seed=23 + causal)
    check_case(q, k, v, causal, 1.0 / math.sqrt(128), k_len=[3000, 1777], num_splits=5)


def test_split_bf16_output():
    q, k, v = rect_inputs(2, 4, 4, 333, 2222, 128, seed=24)
    check_case(q, k, v, True, 1.0 / math.sqrt(128), num_splits=6, out_dtype=torch.bfloat16, tol_max=2e-2,
               tol_mean=2e-3)


@pytest.mark.parametrize("std", [4.0, 8.0])
def test_split_large_logits(std):
    """Near one-hot rows: the merge weights span many orders of magnitude."""
    q, k, v = rect_inputs(1, 4, 4, 256, 4096, 128, seed=25 + int(std), std=std)
    check_case(q, k, v, True, 1.0 / math.sqrt(128), num_splits=7)


def test_split_close_to_single_pass_and_deterministic():
    q, k, v = rect_inputs(1, 4, 4, 256, 5000, 128, seed=26)
    o1, l1 = run_gpu(q, k, v, True, 0.088)
    o2, l2 = run_gpu(q, k, v, True, 0.088, num_splits=9)
    o3, l3 = run_gpu(q, k, v, True, 0.088, num_splits=9)
    assert torch.equal(o2, o3) and torch.equal(l2, l3)
    assert (o1 - o2).abs().max().item() <= 1e-2
    assert ((l1 - l2).abs() / l1.abs().clamp_min(1.0)).max().item() <= 1e-4


def test_one_effective_split_is_the_single_pass():
    """Keys within one 128-key tile: any split count runs the single pass,
    bit-identical, and needs no workspace."""
    q, k, v = rect_inputs(1, 2, 2, 300, 100, 64, seed=27)
    dev = torch.device("cuda:0")
    assert fb.workspace_bytes(q.to(dev), k.to(dev), 8) == 0
    o1, l1 = run_gpu(q, k, v, True, 0.125)
    o2, l2 = run_gpu(q, k, v, True, 0.125, num_splits=8)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_suggested_splits():
    """The suggestion fills the GPU for few query blocks and long keys, and is 1
    when the single pass already has enough work units."""
    dev = torch.device("cuda:0")
    q = torch.empty(1, 32, 256, 128, dtype=torch.bfloat16, device=dev)
    k = torch.empty(1, 8, 131072, 128, dtype=torch.bfloat16, device=dev)
    s = fb.suggest_splits(q, k)
    assert 2 <= s <= 1024
    q2 = torch.empty(1, 32, 16384, 128, dtype=torch.bfloat16, device=dev)
    k2 = torch.empty(1, 32, 16384, 128, dtype=torch.bfloat16, device=dev)
    assert fb.suggest_splits(q2, k2) == 1
    q3, k3, v3 = rect_inputs(1, 4, 4, 64, 6000, 64, seed=28)
    check_case(q3, k3, v3, True, 0.125, num_splits=-1)


def test_split_host_entry_point():
    """fa_fwd_host with a split workspace equals fa_fwd_ex with the same splits."""
    B, H, Nq, Nk, d = 1, 4, 128, 3000, 128
    q, k, v = rect_inputs(B, H, H, Nq, Nk, d, seed=29)
    dev = torch.device("cuda:0")
    qh, kh, vh = q.pin_memory(), k.pin_memory(), v.pin_memory()
    oh = torch.empty(B, H, Nq, d).pin_memory()
    lh = torch.empty(B, H, Nq).pin_memory()
    qd, kd, vd = (torch.empty_like(t, device=dev) for t in (q, k, v))
    od = torch.empty(B, H, Nq, d, device=dev)
    ld = torch.empty(B, H, Nq, device=dev)
    ws = torch.empty(fb.workspace_bytes(qd, kd, 6), dtype=torch.uint8, device=dev)
    fb.fa_fwd_host(qh, kh, vh, oh, lh, qd, kd, vd, od, ld, True, 1 / math.sqrt(d), num_splits=6, workspace=ws)
    o2, l2 = run_gpu(q, k, v, True, 1 / math.sqrt(d), num_splits=6)
    assert torch.equal(oh, o2) and torch.equal(lh, l2)


def test_split_rejects_small_workspace():
    dev = torch.device("cuda:0")
    q, k, v = (t.to(dev) for t in rect_inputs(1, 2, 2, 64, 1000, 64, seed=30))
    o = torch.empty(1, 2, 64, 64, device=dev)
    lse = torch.empty(1, 2, 64, device=dev)
    need = fb.workspace_bytes(q, k, 4)
    ws = torch.empty(need - 16, dtype=torch.uint8, device=dev)
    with pytest.raises(RuntimeError, match="INVALID_ARGUMENT"):
        fb.fa_fwd_ex(q, k, v, o, lse, True, 0.125, num_splits=4, workspace=ws)
