"""The work counts behind the reported throughput (CPU).

bench.py divides each workload's algorithmic flops (or, for the decode, its
K/V/Q/O/LSE bytes) by the measured time.  These tests hold fa_inputs' counts
to the figures the scope table states for the named workloads, and the
generic counting (causal halving, windows, varlen, seqused_k) to a brute-force
count of admitted (row, key) pairs written out from the distance rule.
"""
import itertools

import pytest

import fa_inputs


def brute_pairs(q_len, k_len, causal, window):
    """Admitted (i, j) pairs of one sequence: d = i + k_len - q_len - j; causal
    drops d < 0; a window masks d > left (left >= 0) and -d > right (right >= 0)."""
    left, right = window
    n = 0
    for i, j in itertools.product(range(q_len), range(k_len)):
        d = i + k_len - q_len - j
        if causal and d < 0:
            continue
        if left >= 0 and d > left:
            continue
        if right >= 0 and -d > right:
            continue
        n += 1
    return n


def test_named_small_workloads_match_the_stated_counts():
    # 4 * 257^2 * 128 * 8 = 0.2705 GFLOP
    assert fa_inputs.make("dense_257").flops() == 4 * 257 * 257 * 128 * 8
    # seqused_k = 968 of 1024 padded keys: 4 * 1024 * 968 * 256 * 8 * 2 = 16.24 GFLOP
    p = fa_inputs.make("encoder_d256_seqused")
    assert p.flops() == 4 * 1024 * 968 * 256 * 8 * 2
    # main: sum over the 4 seeded sequences of 4 L^2 D Hq / 2
    p = fa_inputs.make("varlen_gqa_bias")
    assert p.flops() == sum(4 * L * L * 128 * 32 / 2 for L in p.meta["lens"])
    # its bytes: Q, O (bf16), K, V (8 heads), LSE (fp32) and the bias tensor, once each
    T = sum(p.meta["lens"])
    assert p.hbm_bytes() == 2 * T * 32 * 128 * 2 + 2 * T * 8 * 128 * 2 + 4 * T * 32 + T * 32 * 256 * 2


def test_decode_bytes_scale_to_the_stated_figure():
    # the decode workload at 1024 keys; its K+V bytes grow linearly to 4.295 GB at 131072
    p = fa_inputs.make("decode_splitkv", decode_sk=1024)
    B, Hq, Hkv, D = 8, 32, 8, 128
    kv_1024 = 2 * B * 1024 * Hkv * D * 2
    assert p.hbm_bytes() == kv_1024 + 2 * B * Hq * D * 2 + 4 * B * Hq
    assert kv_1024 * 128 == 4_294_967_296  # K + V at 131072 keys


def test_long_dense_count_formula():
    # the S=20480 workload is counted as 4 S^2 D H: 12.026 TFLOP
    assert 4 * 20480 ** 2 * 128 * 56 == 12_025_908_428_800
    p = fa_inputs.random_dense(1, 1, 96, 96, 4, 4, 64)
    assert p.flops() == 4 * 96 * 96 * 64 * 4


@pytest.mark.parametrize("q_len,k_len,causal,window", [
    (40, 40, True, (-1, -1)),
    (30, 55, True, (-1, -1)),     # k longer: bottom-right diagonal
    (55, 30, True, (-1, -1)),     # k shorter: early rows see nothing
    (40, 40, True, (9, -1)),      # causal sliding window
    (33, 50, False, (7, 4)),      # two-sided window
    (50, 33, False, (-1, 0)),     # right bound only
    (20, 20, False, (0, 0)),      # the diagonal key only
])
def test_admitted_pairs_match_brute_force(q_len, k_len, causal, window):
    p = fa_inputs.random_dense(3, 1, q_len, k_len, 2, 2, 16, causal=causal)
    p.window = window
    n = brute_pairs(q_len, k_len, causal, window)
    assert sum(p.admitted_keys(q_len, k_len, i) for i in range(q_len)) == n
    if window != (-1, -1):
        assert p.flops() == 4.0 * 16 * 2 * n
    elif not causal:
        assert p.flops() == 4.0 * q_len * k_len * 16 * 2


def test_local_window_workload_counts_admitted_pairs():
    # the local-window workload's count equals the brute-force pairs on a
    # shortened copy of its window rule (the full one has 32768 rows)
    p = fa_inputs.random_dense(4, 1, 300, 300, 2, 2, 16, causal=True)
    p.window = (63, -1)
    n = brute_pairs(300, 300, True, (63, -1))
    assert p.flops() == 4.0 * 16 * 2 * n
    full = fa_inputs.make("local_window_softcap")
    S, W = 32768, 4095
    exact = sum(min(i, W) + 1 for i in range(S))  # keys max(0, i - W) .. i
    assert full.flops() == 4.0 * 128 * 16 * exact
