"""The arithmetic behind bench.py's roofline figures (no GPU needed): the
algorithmic flops and bytes of each workload, pinned to values worked out by
hand from the shapes, and the fractions computed from them."""
import pytest

import bench


def test_flops_per_token_and_head_is_the_triangle_aware_count():
    # 5 C d + 6 d^2 at C = 64, d = 128: KK^T and QK^T (C^2 d each per chunk), T [bV | bgK]
    # (2 C^2 d), (M o QK^T) U (C^2 d), three d x d x C state products (6 C d^2); per token
    assert bench.prefill_flops_per_token_head() == 5 * 64 * 128 + 6 * 128 * 128 == 139_264
    assert bench.prefill_flops_per_token_head(C=16, d=16) == 5 * 16 * 16 + 6 * 16 * 16


def test_prefill_bytes_of_the_4096_token_layer():
    # q, k 2 x 16.78 MB; v, o 16.78 MB each; g, beta 0.52 MB; state_out 1.05 MB; cu_seqlens 8 B
    b = bench.prefill_bytes(4096, 16, 16, 128, 1, False)
    assert b == 2 * 16_777_216 + 16_777_216 + 16_777_216 + 524_288 + 1_048_576 + 8 == 68_681_736
    # a state read in adds one more copy of the states
    assert bench.prefill_bytes(4096, 16, 16, 128, 1, True) == b + 1_048_576


def test_prefill_bytes_and_flops_of_the_long_prompts():
    assert bench.prefill_bytes(32768, 16, 32, 128, 1, False) == pytest.approx(815.8e6, rel=1e-4)
    assert bench.prefill_bytes(81920, 16, 32, 128, 1, False) == pytest.approx(2.036e9, rel=1e-3)
    assert 32768 * 32 * bench.prefill_flops_per_token_head() == pytest.approx(146.0e9, rel=1e-3)
    assert 4096 * 16 * bench.prefill_flops_per_token_head() == pytest.approx(9.13e9, rel=1e-3)


def test_decode_bytes_per_step():
    # 64 sequences x 32 v heads: the fp32 state read and written (2 x 134.2 MB) dominates
    assert bench.decode_bytes(64, 16, 32, 128) == 2 * 134_217_728 + 524_288 + 1_048_576 + 16_384 == 270_024_704
    assert bench.decode_bytes(64, 16, 32, 128, state_bytes=2) == 2 * 67_108_864 + 524_288 + 1_048_576 + 16_384
    assert bench.decode_bytes(1, 16, 32, 128) == 2 * 2_097_152 + 8192 + 16_384 + 256


def test_roofline_fractions():
    pk = {"bf16_tflops": 1663.7, "hbm_gbs": 6557.8}
    flops = 4096 * 16 * bench.prefill_flops_per_token_head()
    nbytes = bench.prefill_bytes(4096, 16, 16, 128, 1, False)
    ms = 0.1030
    t = bench.roofline_tensor(flops, ms, pk, "measured")
    assert t["achieved"] == pytest.approx(flops / 0.103e-3 / 1e12, abs=0.01)
    assert t["frac"] == pytest.approx(t["achieved"] / 1663.7, abs=1e-4) and t["unit"] == "TFLOP/s"
    h = bench.roofline_hbm(nbytes, ms, pk, "measured")
    assert h["achieved"] == pytest.approx(nbytes / 0.103e-3 / 1e9, abs=0.1) and h["unit"] == "GB/s"
    # the binding roofline is the HBM one here: 68.68 MB at 6557.8 GB/s = 10.47 us
    assert bench.binding_frac(flops, nbytes, ms, pk) == pytest.approx(nbytes / 6557.8e9 / 0.103e-3, abs=1e-4)
    assert bench.binding_frac(flops, nbytes, ms, pk) == h["frac"]
    # decode at 48.9 us per step: 270.02 MB / 48.9 us = 5522 GB/s = 84 % of the copy peak
    d = bench.roofline_hbm(bench.decode_bytes(64, 16, 32, 128), 0.0489, pk, "measured")
    assert d["frac"] == pytest.approx(0.842, abs=1e-3)


def test_aggregate_rate_counts_every_rank_at_the_slowest_time():
    assert bench.aggregate_rate(4096, 0.1, 1) == pytest.approx(40.96e6)
    assert bench.aggregate_rate(4096, 0.1, 8) == pytest.approx(8 * 40.96e6)


def test_traffic_records_are_keyed_by_kernel_source():
    """Each committed ncu traffic record names the kernel source it was taken on:
    it is served while that source is unchanged (comments aside) and dropped
    once the code differs; an unknown kernel has no record."""
    import json
    import os
    with open(os.path.join(bench.ROOT, "profiles", "traffic.json")) as f:
        recs = json.load(f)
    for kernel in ("prefill_pc", "prefill_pc_long", "decode"):
        assert kernel in recs and kernel in bench.KERNEL_SOURCES
        rec = recs[kernel]
        assert rec["bytes_per_launch"] == rec["dram_read_bytes"] + rec["dram_write_bytes"]
        current = rec["source_hash"] == bench.kernel_source_hash(kernel)
        assert bench.traffic_record(kernel) == (rec if current else None)
    assert bench.traffic_record("no_such_kernel") is None
    src = "int a = 1; // note\n/* block */ int b = 2;"
    assert bench._code_only(src) == bench._code_only(src.replace("note", "other note"))
    assert bench._code_only(src) != bench._code_only(src.replace("b = 2", "b = 3"))


def test_long_prompt_traffic_stays_below_its_algorithmic_bytes():
    """The 32768-token capture's DRAM bytes are at most the prompt's algorithmic
    bytes (inputs once, outputs once): the package ring stays in L2."""
    import json
    import os
    with open(os.path.join(bench.ROOT, "profiles", "traffic.json")) as f:
        rec = json.load(f)["prefill_pc_long"]
    alg = bench.prefill_bytes(32768, 16, 32, 128, 1, True)
    assert rec["bytes_per_launch"] <= alg
