"""bench.py's host-side plumbing, without a GPU: every workload kind has a JSON config,
the algorithmic byte / flop counts follow their formulas, and the committed ncu traffic
is used only while the kernel sources it was taken on are unchanged."""
import os
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
import workloads as W  # noqa: E402

ALL = (list(W.CONFIGS) + list(W.CONV_CONFIGS) + list(W.VARLEN_CONFIGS) + list(W.BACKWARD_CONFIGS)
       + list(W.LAYER_CONFIGS))


@pytest.mark.parametrize("name", ALL)
def test_every_workload_has_a_config(name):
    dtype, cfg = bench.workload_config(name, 1)
    assert dtype in (torch.bfloat16, torch.float32)
    assert cfg["workload"] == name and "parallelism" in cfg and "l2" in cfg


def test_prefill_algorithmic_counts():
    w = W.CONFIGS["gated_bf16_b8h16t8192"]
    b, f = bench.prefill_algorithmic(w)
    th = w.B * w.H * w.T
    assert b == th * (2 * (2 * 128 + 2 * 128) + 4) + w.B * w.H * 128 * 128 * 4
    assert f == th * (2 * 64 * 128 * 2 + 4 * 128 * 128)
    # the constant-decay mode reads no gate stream and does the scalar-gate flops
    r = W.CONFIGS["retnet_bf16_b8h16t8192"]
    br, fr = bench.prefill_algorithmic(r)
    assert br == b - th * 4 and fr == f
    # per-channel gates: d_k floats per token-head
    kd = W.CONFIGS["kda_bf16_b2h16t32768"]
    gd = W.CONFIGS["gdn_bf16_b2h16t32768"]
    assert bench.prefill_algorithmic(kd)[0] - bench.prefill_algorithmic(gd)[0] == \
        kd.B * kd.H * kd.T * 4 * (128 - 1)


def test_decode_algorithmic_counts():
    w = W.CONFIGS["gdn_decode_n256h32"]
    b, f = bench.decode_algorithmic(w)
    nh = w.B * w.H
    assert b == nh * (2 * 128 * 128 * 4 + 2 * (2 * 128 + 2 * 128) + 8)
    assert f == nh * 8 * 128 * 128


def test_committed_traffic_is_keyed_to_sources():
    """Each traffic.json entry records the hashes of the sources its kernels were built from
    (their translation units, every header, the C ABI); bench.py uses an entry only while
    all of them are unchanged (otherwise roofline.traffic is null)."""
    import json
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        t = json.load(f)
    assert bench.DEFAULT_WORKLOAD in t["workloads"]
    now = bench.source_file_shas()
    for name, entry in t["workloads"].items():
        rec = entry.get("sources") or t.get("sources")
        assert rec, name
        if "sources" in entry:   # its kernels' own files, every header and the C ABI
            assert "abi.cu" in rec and all(fn in rec for fn in now if fn.endswith(".cuh")), name
        same = all(now.get(fn) == sha for fn, sha in rec.items())
        got = bench.ncu_traffic(name)
        assert (got is not None) == same, name
        if got is not None:
            assert got["kernels"][-1]["dram_bytes_per_launch"] > 0
