"""Host-side pieces of bench.py's measurement contract, on CPU: the algorithmic
byte count of the decode step, the rule that ties the recorded ncu traffic to
the kernel source it was taken on, and the L2 flush helper."""
import json
import os

import pytest
import torch

import bench
from sparse_linear_layers_bitnet_b200 import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_decode_step_bytes():
    """A fused projection moves its bf16 activations in, its packed weights at
    2 bits per weight, gamma and its bf16 outputs.  For the 2B shapes
    (hidden 2560, FFN 6912) at T = 1 a layer is 69.47 M weights = 17.37 MB of
    codes plus 74.8 KB of bf16 activations in and out and the gammas:
    17,441,808 bytes, 523,254,240 for the
    30-layer step the benchmark times."""
    mats = synth.DECODE_2B_MATRICES
    assert sum(N * K for _, K, N in mats) == 69_468_160
    per_layer = sum(bench.decode_bytes_fused(1, K, N) for _, K, N in mats)
    assert per_layer == 17_441_808
    assert 30 * per_layer == 523_254_240
    # unfused: the int8 activations (K bytes) and the absmax (4 bytes) are
    # written by the quantisation and read again by the GEMV
    q, g = zip(*(bench.decode_bytes(1, K, N) for _, K, N in mats))
    assert sum(q) + sum(g) - per_layer == sum(2 * K + 8 for _, K, _ in mats)


def test_traffic_record_follows_the_source():
    """ncu_traffic returns the recorded DRAM bytes only while the kernel's
    source still hashes to the value recorded with them."""
    with open(os.path.join(ROOT, "profiles", "ncu_traffic.json")) as f:
        rec = json.load(f)["k_decode_chain"]
    files = ["chain.cu", "frag.cuh"]
    expect = float(rec["dram_bytes_per_launch"]) if rec["source_sha"] == bench.source_sha(*files) else None
    assert bench.ncu_traffic("k_decode_chain", files) == expect
    assert bench.ncu_traffic("k_decode_chain", ["gemv.cu"]) is None   # another source: no record
    assert bench.ncu_traffic("no_such_kernel", files) is None


def test_recorded_chain_traffic_is_near_algorithmic():
    """The recorded chain traffic (one 4-layer launch scaled by 30/4) is within
    a few percent of the algorithmic bytes: every weight byte crosses HBM once."""
    with open(os.path.join(ROOT, "profiles", "ncu_traffic.json")) as f:
        rec = json.load(f)["k_decode_chain"]
    ratio = rec["dram_bytes_per_launch"] / 523_254_240
    assert 0.98 <= ratio <= 1.05


@pytest.mark.parametrize("n", [8, 1000])
def test_flush_writes_one_half_and_reads_the_other(n):
    buf = torch.zeros(2 * n)
    bench.flush_l2(torch, buf)
    assert torch.equal(buf[:n], torch.ones(n))
    assert torch.equal(buf[n:], torch.zeros(n))
