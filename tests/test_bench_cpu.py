"""Host-side arithmetic of the benchmark's JSON line, checked on the CPU against
closed forms and brute-force counts: the nominal FLOP counts, the algorithmic
HBM bytes of one launch, the choice of the tensor peak, and the rule that a
committed DRAM-traffic record is reported only for the device sources it was
taken on."""
import os

import numpy as np
import pytest

import bench
from exact_io_aware_52_b200 import workloads


def _allowed_pairs(N, Nk, causal, k_len=None):
    """Brute force: (query, key) pairs the mask allows (bottom-right causal alignment)."""
    i = np.arange(N)[:, None]
    j = np.arange(Nk)[None, :]
    m = np.ones((N, Nk), dtype=bool)
    if causal:
        m &= j <= i + (Nk - N)
    if k_len is not None:
        m &= j < k_len
    return int(m.sum())


def test_flops_square_is_the_nominal_count():
    w = workloads.custom(2, 3, 300, 64, causal=False)
    assert w.flops() == 4.0 * 2 * 3 * 300 * 300 * 64
    wc = workloads.custom(2, 3, 300, 64, causal=True)
    assert wc.flops() == w.flops() / 2


@pytest.mark.parametrize("N,Nk,causal", [(100, 900, True), (256, 131072, True), (37, 50, False), (5, 3, True)])
def test_flops_rectangular_counts_allowed_pairs(N, Nk, causal):
    w = workloads.custom(1, 2, N, 128, causal=causal, Nk=Nk)
    assert w.flops() == 4.0 * 1 * 2 * 128 * _allowed_pairs(N, Nk, causal)


def test_backward_flops_are_two_and_a_half_forward():
    f = workloads.WORKLOADS[4]
    b = workloads.WORKLOADS[10]
    assert (b.B, b.H, b.N, b.d, b.causal) == (f.B, f.H, f.N, f.d, f.causal)
    assert b.flops() == 2.5 * f.flops()


def test_algorithmic_bytes_long_context():
    w = workloads.WORKLOADS[4]  # B1 H32 N16384 d128, bf16 in, fp32 O
    n = 1 * 32 * 16384 * 128
    expect = 2 * n + 2 * 2 * n + 4 * n + 4 * 32 * 16384
    assert bench.algorithmic_bytes(w, None) == expect


def test_algorithmic_bytes_key_padding_and_groups():
    w = workloads.custom(3, 8, 200, 64, causal=False, H_kv=2, Nk=500)
    k_len = [500, 0, 777]  # clamped to [0, N_k]
    n = 3 * 8 * 200 * 64
    kv_rows = 2 * (500 + 0 + 500)
    expect = 2 * n + 2 * 2 * kv_rows * 64 + 4 * n + 4 * 3 * 8 * 200
    assert bench.algorithmic_bytes(w, k_len) == expect


def test_algorithmic_bytes_e4m3_inputs_are_one_byte():
    w = workloads.WORKLOADS[9]
    n = w.B * w.H * w.N * w.d
    assert bench.algorithmic_bytes(w, None) == n + 2 * n + 4 * n + 4 * w.B * w.H * w.N


def test_tensor_peak_sustained_only_for_long_regions():
    peaks = {"bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0}
    peak, label, burst, sustained = bench.tensor_peak(peaks, 999.9)
    assert (peak, burst, sustained) == (1600.0, 1600.0, 1400.0) and "burst" in label
    peak, label, _, _ = bench.tensor_peak(peaks, 1000.0)
    assert peak == 1400.0 and "sustained" in label
    peak, _, burst, sustained = bench.tensor_peak(peaks, 5000.0, ratio=2.0)
    assert (peak, burst, sustained) == (2800.0, 3200.0, 2800.0)
    # without a sustained figure the burst one stands in
    assert bench.tensor_peak({"bf16_tflops": 1500.0}, 2000.0)[0] == 1500.0


def _fake_tree(root, body=b"kernel v1"):
    csrc = os.path.join(root, "exact_io_aware_52_b200", "csrc")
    os.makedirs(csrc, exist_ok=True)
    os.makedirs(os.path.join(root, "profiles"), exist_ok=True)
    for name in ("a.cuh", "b.cuh"):
        with open(os.path.join(csrc, name), "wb") as f:
            f.write(body + name.encode())


def _record(root, workload, source_hash, total):
    with open(os.path.join(root, "profiles", "k_traffic.txt"), "w") as f:
        f.write("# a comment line\n")
        f.write("sources a.cuh b.cuh\n")
        f.write(f"source_hash {source_hash}\nworkload {workload}\n")
        f.write(f"dram_bytes_read 1\ndram_bytes_write 2\ndram_bytes_per_launch {total}\n")


def test_traffic_record_follows_the_device_sources(tmp_path, monkeypatch):
    root = str(tmp_path)
    _fake_tree(root)
    monkeypatch.setattr(bench, "ROOT", root)
    h = bench.kernel_source_hash(["a.cuh", "b.cuh"])
    _record(root, 4, h, 123456)
    assert bench.measured_traffic(4) == 123456.0
    assert bench.measured_traffic(8) is None  # another workload
    _fake_tree(root, body=b"kernel v2")  # the kernel changed since the capture
    assert bench.measured_traffic(4) is None
    _record(root, 4, "0000000000000000", 5)
    assert bench.measured_traffic(4) is None


def test_committed_records_name_existing_sources():
    """Every committed traffic record lists device sources that exist and a
    16-hex-digit hash (whether it matches is decided at run time)."""
    import glob
    paths = glob.glob(os.path.join(bench.ROOT, "profiles", "*traffic.txt"))
    assert paths
    for path in paths:
        rec = {}
        for line in open(path):
            if line.startswith("#") or not line.strip():
                continue
            k, _, v = line.partition(" ")
            rec[k] = v.strip()
        for name in rec["sources"].split():
            assert os.path.isfile(os.path.join(bench.ROOT, "exact_io_aware_52_b200", "csrc", name)), (path, name)
        assert len(rec["source_hash"]) == 16 and int(rec["source_hash"], 16) >= 0
        assert float(rec["dram_bytes_per_launch"]) == float(rec["dram_bytes_read"]) + float(rec["dram_bytes_write"])


def test_clock_peak_is_sms_times_8192_per_clock():
    # 148 SMs at 1965 MHz: 148 * 8192 * 1.965e9 = 2382.4 TFLOP/s
    assert abs(bench.clock_peak_tflops(148, 1965.0) - 148 * 8192 * 1.965e9 / 1e12) < 1e-9
    assert abs(bench.clock_peak_tflops(148, 1000.0, ratio=2.0) - 2 * 148 * 8192 * 1e9 / 1e12) < 1e-9


def test_percentiles_match_numpy_linear_interpolation():
    rng = np.random.default_rng(3)
    xs = rng.exponential(size=37).tolist()
    st = bench.percentiles(xs)
    for key, q in (("median", 50), ("p10", 10), ("p90", 90)):
        assert abs(st[key] - float(np.percentile(xs, q))) < 1e-12
    assert abs(st["mean"] - float(np.mean(xs))) < 1e-12 and st["n"] == 37
    assert bench.percentiles([2.5]) == {"median": 2.5, "p10": 2.5, "p90": 2.5, "mean": 2.5, "n": 1}


@pytest.mark.parametrize("causal", [False, True])
def test_effective_flops_count_keys_inside_each_length(causal):
    w = workloads.custom(3, 2, 40, 64, causal=causal, Nk=56)
    k_len = [56, 0, 23]
    expect = sum(4.0 * 2 * 64 * _allowed_pairs(40, 56, causal, k_len=L) for L in k_len)
    assert bench.effective_flops(w, k_len) == expect
    assert bench.effective_flops(w, None) == w.flops()


def test_bert_shaped_effective_flops_follow_the_drawn_lengths():
    w = workloads.WORKLOADS[3]
    _, _, _, k_len = workloads.make_inputs(w)
    L = k_len.tolist()
    assert all(256 <= x <= 512 for x in L)
    assert bench.effective_flops(w, L) == 4.0 * w.H * w.N * w.d * sum(L)
    assert bench.effective_flops(w, L) < w.flops()


def test_guard_regions_catch_writes_past_either_end():
    """The guard helper the GPU tests wrap every output buffer in, exercised on
    CPU tensors: untouched guards pass; one byte changed on either side fails."""
    import torch

    from tests.gpu_util import GUARD_BYTES, Guarded
    g = Guarded((3, 5), torch.float32, "cpu", fill=float("nan"))
    assert g.t.shape == (3, 5) and bool(torch.isnan(g.t).all())
    g.t.fill_(1.0)
    g.check("ok")
    g.buf[GUARD_BYTES + g.nbytes] = 0  # one byte past the end
    with pytest.raises(AssertionError, match="after"):
        g.check("tail")
    g2 = Guarded((7,), torch.float32, "cpu")
    g2.buf[GUARD_BYTES - 1] = 1  # one byte before the start
    with pytest.raises(AssertionError, match="1 guard bytes changed before"):
        g2.check("head")


def test_memory_footprint_against_the_definition():
    """The memory restatement: the fused path holds Q, K, V, O, lse; the plain
    definition adds one fp32 score matrix per head (B*H*N*N_k values)."""
    w = workloads.WORKLOADS[4]  # B1 H32 N16384 d128 causal
    m = bench.memory_footprint(w)
    io = 3 * 2 * 32 * 16384 * 128 + 4 * 32 * 16384 * 128 + 4 * 32 * 16384
    assert m["fused_bytes"] == io == bench.algorithmic_bytes(w, None)
    assert m["score_matrix_bytes"] == 4 * 32 * 16384 * 16384
    assert m["definition_bytes"] == io + 4 * 32 * 16384 * 16384
    assert abs(m["ratio"] - (io + 4 * 32 * 16384 ** 2) / io) < 1e-9 and m["ratio"] > 50
    # a key-split workspace counts on the fused side; E4M3 inputs take one byte
    m2 = bench.memory_footprint(w, workspace_bytes=1 << 20)
    assert m2["fused_bytes"] == io + (1 << 20)
    w9 = workloads.WORKLOADS[9]
    assert bench.memory_footprint(w9)["fused_bytes"] == 3 * 32 * 16384 * 128 + 4 * 32 * 16384 * 128 + 4 * 32 * 16384
