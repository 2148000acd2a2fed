"""Host-side pieces of bench.py (no GPU): the algorithmic counts behind the
roofline fractions, and the reading of the committed ncu traffic record."""
import json
import os
import tempfile

import bench


def test_headline_algorithmic_counts():
    # B4 H8 L8192 dk256 dv512 C128: q, k, v read once, y written once (bf16),
    # fp32 state out; causal intra-block pairs, cross-block term, state update
    assert bench.chunk_bytes(4, 8, 8192, 256, 512) == 805_306_368 + 16_777_216
    per_token = bench.chunk_flops_per_head_token(128, 256, 512)
    assert per_token == 129 * 768 + 4 * 256 * 512 == 623_360
    assert 4 * 8 * 8192 * per_token == 163_410_083_840


def test_parallel_flops_counts_causal_pairs():
    # L(L+1)/2 pairs per head, 2 (dk + dv) flops each
    assert bench.parallel_flops(1, 1, 4, 2, 3) == 10 * 2 * 5
    assert bench.parallel_flops(2, 8, 2048, 64, 128) == 12_891_193_344


def test_traffic_is_read_only_for_the_current_kernel_source():
    digest = bench.kernel_source_digest()
    assert len(digest) == 16
    rec = {"kernel_source_sha256_16": digest, "dram_bytes_per_launch": 123456}
    stale = dict(rec, kernel_source_sha256_16="0" * 16)
    orig = bench.TRAFFIC_FILE
    try:
        with tempfile.TemporaryDirectory() as d:
            for body, want in ((rec, 123456.0), (stale, None), ({}, None)):
                p = os.path.join(d, "s.json")
                with open(p, "w") as f:
                    json.dump(body, f)
                bench.TRAFFIC_FILE = p
                assert bench.measured_traffic() == want
            bench.TRAFFIC_FILE = os.path.join(d, "missing.json")
            assert bench.measured_traffic() is None
    finally:
        bench.TRAFFIC_FILE = orig


def test_digest_regions_are_found_in_the_kernel_source():
    # every region marker must be present, or the digest silently covers the
    # whole file and any edit elsewhere voids the traffic record
    path = os.path.join(bench.ROOT, "retnet_retention_chunkwise_b200", "csrc", "chunkwise_tc.cuh")
    with open(path, "rb") as f:
        src = f.read()
    for start, end in bench.HEADLINE_SOURCE_REGIONS:
        i, j = src.find(start), src.find(end)
        assert 0 <= i < j, (start[:40], end[:40])
    assert b"chunkwise_tc256_kernel(" in src[src.find(bench.HEADLINE_SOURCE_REGIONS[1][0]):]
