"""Host-side helpers of bench.py (no GPU): which decode kernel a workload's
roofline is attributed to, and when a committed traffic figure applies."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_decode_kernel_key_follows_the_library_dispatch():
    # per-head kernel for plain multi-head attention and odd large groups
    assert bench.decode_kernel_key(128, 1, False) == "fa_decode_split_kernel<128>"
    assert bench.decode_kernel_key(128, 20, False) == "fa_decode_split_kernel<128>"
    assert bench.decode_kernel_key(64, 1, True) == "fa_decode_split_kernel<64,paged>"
    # grouped kernel: the whole group up to 16, else 16 or 8 heads per CTA
    assert bench.decode_kernel_key(128, 4, False) == "fa_decode_group_mma_kernel<128,4>"
    assert bench.decode_kernel_key(128, 16, True) == "fa_decode_group_mma_kernel<128,16,paged>"
    assert bench.decode_kernel_key(128, 32, False) == "fa_decode_group_mma_kernel<128,16>"
    assert bench.decode_kernel_key(64, 24, False) == "fa_decode_group_mma_kernel<64,8>"
    assert bench.decode_kernel_key(128, 3, False) == "fa_decode_group_mma_kernel<128,3>"


def test_traffic_reported_only_for_its_workload_and_sources():
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        table = json.load(f)
    key = "fa_fwd_kernel<128,true>"
    ent = table[key]
    got = bench.profiled_traffic(key, "fwd", ent["workload"])
    if ent["source_sha"] == bench.kernel_sources_sha("fwd"):
        assert got == ent["dram_bytes_per_launch"]
    else:
        assert got is None
    # another workload of the same kernel gets no figure
    assert bench.profiled_traffic(key, "fwd", "fwd_causal_B1_H32_N32768_d128") is None
    assert bench.profiled_traffic("no_such_kernel", "fwd", ent["workload"]) is None
