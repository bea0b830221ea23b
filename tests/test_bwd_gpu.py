"""The backward kernels (fa_bwd) against the fp64 backward oracle.

O and lse are the forward oracle's (rounded to fp32), so that the check
covers the backward kernels alone; dq, dk, dv must lie within the bound
derived in tests/bwd_bound.py element by element.  An end-to-end case takes
O and lse from the forward kernel instead, and the full-size case checks
properties that hold at any size."""
import math

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_52_b200 import _binding as fb
from exact_io_aware_52_b200 import workloads
from tests import bwd_bound
from tests.gpu_util import Guarded, run_gpu

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


def inputs(B, H, N, d, seed, H_kv=None, Nk=None, std=1.0):
    g = torch.Generator().manual_seed(seed)
    H_kv = H if H_kv is None else H_kv
    Nk = N if Nk is None else Nk
    q = (torch.randn(B, H, N, d, generator=g) * std).to(torch.bfloat16)
    k = (torch.randn(B, H_kv, Nk, d, generator=g) * std).to(torch.bfloat16)
    v = torch.randn(B, H_kv, Nk, d, generator=g).to(torch.bfloat16)
    do = torch.randn(B, H, N, d, generator=g).to(torch.bfloat16)
    return q, k, v, do


def run_bwd(q, k, v, do, o, lse, causal, scale, k_len=None):
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    qd, kd, vd, dod = (t.to(DEV) for t in (q, k, v, do))
    od, lsed = o.to(DEV), lse.to(DEV)
    # gradients and the D workspace between guard regions (tests.gpu_util.Guarded)
    gq = Guarded(tuple(q.shape), torch.float32, DEV, fill=float("nan"))
    gk = Guarded(tuple(k.shape), torch.float32, DEV, fill=float("nan"))
    gv = Guarded(tuple(v.shape), torch.float32, DEV, fill=float("nan"))
    gw = Guarded((max(fb.bwd_workspace_bytes(q), 16),), torch.uint8, DEV)
    dq, dk, dv, ws = gq.t, gk.t, gv.t, gw.t
    kl = None if k_len is None else torch.tensor(k_len, dtype=torch.int32, device=DEV)
    fb.fa_bwd(qd, kd, vd, od, lsed, dod, dq, dk, dv, causal, scale, ws, k_len=kl, dev_status=st)
    assert fb.read_device_status(st) == fb.FA_OK
    for g, name in ((gq, "dq"), (gk, "dk"), (gv, "dv"), (gw, "workspace")):
        g.check(name)
    return dq.cpu().double().numpy(), dk.cpu().double().numpy(), dv.cpu().double().numpy()


def check_bwd(q, k, v, do, causal, scale, k_len=None):
    B, H, N, d = q.shape
    o_ref, lse_ref = oracle.attention_f64(q, k, v, causal, scale, k_len=k_len)
    o = torch.from_numpy(o_ref.reshape(B, H, N, d)).float()
    lse = torch.from_numpy(lse_ref.reshape(B, H, N)).float()
    got = run_bwd(q, k, v, do, o, lse, causal, scale, k_len)
    ref = oracle.attention_bwd_f64(q, k, v, do, causal, scale, k_len=k_len)
    bnd = bwd_bound.bounds(*(t.double().numpy() for t in (q, k, v, do)), causal, float(np.float32(scale)), k_len)
    stats = {}
    for name, a, b, c in zip(("dq", "dk", "dv"), got, ref, bnd):
        assert np.all(np.isfinite(a)), name
        err = np.abs(a - b)
        worst = np.unravel_index(np.argmax(err / c), err.shape)
        assert np.all(err <= c), (name, float(err[worst]), float(c[worst]), worst)
        stats[name] = (float(err.max()), float((err / c).max()))
    return stats


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 127, 128, 129, 300])
def test_ragged_shapes(N, d, causal):
    q, k, v, do = inputs(2, 2, N, d, seed=4000 + N + d + causal)
    check_bwd(q, k, v, do, causal, 1.0 / math.sqrt(d))


@pytest.mark.parametrize("Nq,Nk", [(100, 300), (300, 129), (1, 700)])
@pytest.mark.parametrize("causal", [False, True])
def test_fewer_or_more_queries_than_keys(Nq, Nk, causal):
    q, k, v, do = inputs(1, 2, Nq, 128, seed=4001 + Nq + Nk + causal, Nk=Nk)
    check_bwd(q, k, v, do, causal, 1.0 / math.sqrt(128))


@pytest.mark.parametrize("causal", [False, True])
def test_key_padding(causal):
    k_len = [0, 1, 127, 128, 129, 300, 400, -2]
    q, k, v, do = inputs(len(k_len), 2, 300, 64, seed=4002 + causal)
    check_bwd(q, k, v, do, causal, 0.125, k_len=k_len)


@pytest.mark.parametrize("H_kv", [1, 2])
def test_grouped_heads(H_kv):
    q, k, v, do = inputs(2, 4, 333, 128, seed=4003 + H_kv, H_kv=H_kv)
    check_bwd(q, k, v, do, True, 1.0 / math.sqrt(128), k_len=[333, 200])


def test_more_units_than_sms():
    q, k, v, do = inputs(2, 16, 1200, 64, seed=4004)
    check_bwd(q, k, v, do, True, 0.125)


def test_large_logits():
    q, k, v, do = inputs(1, 2, 1024, 128, seed=4005, std=3.0)
    print(check_bwd(q, k, v, do, True, 1.0 / math.sqrt(128)))


def test_end_to_end_with_forward_kernel():
    """O and lse from the forward kernel: the gradients stay within 1% of the
    exact ones in max norm (D inherits the forward's O error)."""
    q, k, v, do = inputs(1, 4, 777, 128, seed=4006)
    scale = 1.0 / math.sqrt(128)
    o, lse = run_gpu(q, k, v, True, scale)
    got = run_bwd(q, k, v, do, o, lse, True, scale)
    ref = oracle.attention_bwd_f64(q, k, v, do, True, scale)
    for name, a, b in zip(("dq", "dk", "dv"), got, ref):
        assert np.abs(a - b).max() <= 1e-2 * np.abs(b).max(), name


def test_full_size_invariants():
    """The long-context shape (B1 H32 N16384 d128 causal): every row of dS
    sums to zero, so dK sums to zero over the keys of each head; P's rows sum
    to one, so dV sums to the sum of dO over the rows (all rows have a key)."""
    w = workloads.WORKLOADS[4]
    q, k, v, _ = workloads.make_inputs(w)
    g = torch.Generator().manual_seed(4007)
    do = torch.randn(q.shape, generator=g).to(torch.bfloat16)
    o, lse = run_gpu(q, k, v, True, w.scale)
    dq, dk, dv = run_bwd(q, k, v, do, o, lse, True, w.scale)
    assert np.all(np.isfinite(dq)) and np.all(np.isfinite(dk)) and np.all(np.isfinite(dv))
    col = np.abs(dk).sum(2)
    assert np.all(np.abs(dk.sum(2)) <= 1e-3 * col + 1e-3)
    dsum = do.double().numpy().sum(2)
    assert np.all(np.abs(dv.sum(2) - dsum) <= 1e-3 * np.abs(do.double().numpy()).sum(2) + 1e-3)


def test_full_size_two_heads_element_wise():
    """The full long-context shape (B1 H32 N16384 d128 causal, the backward
    benchmark's launch configuration: banded unit order, 128-tile query loops),
    compared element by element with the fp64 backward oracle on two of its
    heads under the derived bound.  Heads are independent in the definition,
    so the oracle runs on those heads alone; their O and lse are the forward
    oracle's (the other heads keep the forward kernel's, which cannot reach
    the checked heads' gradients)."""
    w = workloads.WORKLOADS[10]
    q, k, v, _ = workloads.make_inputs(w)
    do = workloads.make_dout(w)
    heads = [0, w.H - 1]
    sub = [t[:, heads].contiguous() for t in (q, k, v, do)]
    o, lse = run_gpu(q, k, v, True, w.scale)
    o_ref, lse_ref = oracle.attention_f64(sub[0], sub[1], sub[2], True, w.scale)
    o[:, heads] = torch.from_numpy(o_ref.reshape(1, 2, w.N, w.d)).float()
    lse[:, heads] = torch.from_numpy(lse_ref.reshape(1, 2, w.N)).float()
    got = run_bwd(q, k, v, do, o, lse, True, w.scale)
    ref = oracle.attention_bwd_f64(*sub, True, w.scale, nthreads=2)
    bnd = bwd_bound.bounds(*(t.double().numpy() for t in sub), True, float(np.float32(w.scale)))
    for name, a, b, c in zip(("dq", "dk", "dv"), got, ref, bnd):
        a = a[:, heads]
        assert np.all(np.isfinite(a)), name
        err = np.abs(a - b)
        worst = np.unravel_index(np.argmax(err / c), err.shape)
        assert np.all(err <= c), (name, float(err[worst]), float(c[worst]), worst)


def test_deterministic_dk_dv():
    q, k, v, do = inputs(1, 4, 600, 128, seed=4008)
    o_ref, lse_ref = oracle.attention_f64(q, k, v, True, 0.088)
    o = torch.from_numpy(o_ref.reshape(q.shape)).float()
    lse = torch.from_numpy(lse_ref.reshape(q.shape[:3])).float()
    a = run_bwd(q, k, v, do, o, lse, True, 0.088)
    b = run_bwd(q, k, v, do, o, lse, True, 0.088)
    assert np.array_equal(a[1], b[1]) and np.array_equal(a[2], b[2])
