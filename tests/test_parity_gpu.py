"""GPU parity: the CUDA path through the C ABI against the CPU fp64 oracle.

Every case draws seeded inputs from fa_inputs, runs the library on cuda:0 and
compares element by element (tests/parity_util.py states the gates).  Sizes
span several tiles and a ragged tail.  The workloads are checked on their
whole output, except the S=20480 one (12 TFLOP), which is checked on sampled
rows that the oracle computes one by one exactly.  Outputs are pre-filled
with NaN, so an element that no kernel writes fails the comparison.
"""

import numpy as np
import pytest
import torch

import fa_inputs
import oracle
import exact_attention_forward_flash_b200 as fa
from parity_util import compare, compare_relative

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    fa.load_library()
    yield
    assert fa.check_device_error() == 0, "a kernel wait timed out"


def nan_outputs(q, lse_shape):
    """Output buffers full of NaN: whatever the kernels leave unwritten shows."""
    return (torch.full_like(q, float("nan")),
            torch.full(lse_shape, float("nan"), dtype=torch.float32, device=q.device))


def run_dense(p, **kw):
    g = p.to(DEV)
    out, lse = nan_outputs(g.q, (p.B, p.Hq, g.q.shape[1]))
    fa.fa_fwd(g.q, g.k, g.v, causal=p.causal, softmax_scale=p.softmax_scale,
              seqused_k=g.seqused_k, rel_bias=g.rel_bias, out=out, lse=lse, **kw)
    torch.cuda.synchronize()
    return out, lse


def ref_dense(p, window=(-1, -1), softcap=0.0):
    return oracle.attention(p.q, p.k, p.v, causal=p.causal, softmax_scale=p.softmax_scale,
                            seqused_k=p.seqused_k, rel_bias=p.rel_bias, window=window,
                            softcap=softcap)


def run_varlen(p, **kw):
    g = p.to(DEV)
    out, lse = nan_outputs(g.q, (p.Hq, g.q.shape[0]))
    fa.fa_fwd_varlen(g.q, g.k, g.v, g.cu_seqlens_q, g.cu_seqlens_k,
                     p.max_seqlen_q, p.max_seqlen_k, seqused_k=g.seqused_k,
                     causal=p.causal, softmax_scale=p.softmax_scale,
                     rel_bias=g.rel_bias, out=out, lse=lse, **kw)
    torch.cuda.synchronize()
    return out, lse


def ref_varlen(p, window=(-1, -1), softcap=0.0):
    return oracle.attention(p.q, p.k, p.v, cu_seqlens_q=p.cu_seqlens_q,
                            cu_seqlens_k=p.cu_seqlens_k, seqused_k=p.seqused_k,
                            causal=p.causal, softmax_scale=p.softmax_scale,
                            rel_bias=p.rel_bias, window=window, softcap=softcap)


# ---------------------------------------------------------------------------
# the small dense workload, both 16-bit types
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_dense_257(dtype):
    p = fa_inputs.make("dense_257", dtype=dtype)
    out, lse = run_dense(p)
    ro, rl = ref_dense(p)
    compare(out, lse, ro, rl, what=f"dense_257 {dtype}")


# ---------------------------------------------------------------------------
# dense shapes: causal, Sq != Sk both ways, GQA groups, D = 64 / 128 / 256
# ---------------------------------------------------------------------------
CASES = [
    # B, Sq, Sk, Hq, Hkv, D, causal
    (2, 300, 300, 4, 4, 128, True),
    (1, 300, 200, 4, 2, 128, True),    # k shorter: first rows see no key
    (1, 100, 333, 8, 2, 128, True),    # k longer: bottom-right diagonal
    (2, 129, 390, 6, 2, 128, False),   # group of 3: heads not packed
    (1, 257, 257, 16, 2, 128, True),   # group of 8 packed
    (2, 200, 300, 8, 8, 256, False),
    (1, 300, 300, 8, 1, 256, True),    # D=256, group of 8 packed
    (1, 70, 600, 4, 4, 256, True),
    (2, 300, 300, 4, 4, 64, True),     # D=64
    (1, 129, 390, 8, 2, 64, False),    # D=64, group of 4 packed
    # narrow head dims (16-column chunks, 32-byte swizzle; 72 padded to 80)
    (2, 300, 300, 4, 4, 16, True),
    (1, 129, 390, 8, 1, 16, False),    # D=16, MQA group of 8 packed
    (1, 257, 300, 6, 2, 48, True),     # D=48, group of 3: heads not packed
    (1, 300, 300, 8, 8, 72, True),     # D=72 MHA
    (2, 129, 390, 8, 2, 72, False),
    (1, 200, 333, 4, 2, 80, True),
]


@pytest.mark.parametrize("case", CASES)
def test_dense_shapes(case):
    B, Sq, Sk, Hq, Hkv, D, causal = case
    p = fa_inputs.random_dense(100 + Sq + Sk, B, Sq, Sk, Hq, Hkv, D, causal=causal)
    out, lse = run_dense(p)
    ro, rl = ref_dense(p)
    compare(out, lse, ro, rl, what=str(case))


@pytest.mark.parametrize("D", [16, 48, 64, 72, 128, 256])
def test_fp16_causal_gqa(D):
    p = fa_inputs.random_dense(7, 2, 260, 270, 8, 2, D, dtype=torch.float16, causal=True)
    out, lse = run_dense(p)
    ro, rl = ref_dense(p)
    compare(out, lse, ro, rl, what=f"fp16 D{D}")


# ---------------------------------------------------------------------------
# varlen with empty / one-token / multi-tile sequences, causal, GQA, bias
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("D", [16, 48, 64, 72, 128, 256])
@pytest.mark.parametrize("causal", [False, True])
def test_varlen_bias(D, causal):
    q_lens = [0, 1, 130, 257, 513, 64]
    k_lens = [3, 1, 130, 300, 513, 0]
    p = fa_inputs.random_varlen(11 + D, q_lens, k_lens, Hq=8, Hkv=2, D=D, causal=causal,
                                bias_extent=256)
    out, lse = run_varlen(p)
    ro, rl = ref_varlen(p)
    compare(out, lse, ro, rl, what=f"varlen D{D} causal={causal}")


def test_varlen_seqused():
    p = fa_inputs.random_varlen(12, [100, 200], [300, 250], Hq=4, Hkv=4, D=128, causal=True,
                                seqused=[260, 250], bias_extent=128)
    out, lse = run_varlen(p)
    ro, rl = ref_varlen(p)
    compare(out, lse, ro, rl, what="varlen seqused")


def test_bias_extent_512_far_band():
    # rel_extent larger than one KV tile and q_len < k_len
    p = fa_inputs.random_varlen(13, [200, 333], [700, 333], Hq=4, Hkv=1, D=128, causal=True,
                                bias_extent=512, bias_std=0.5)
    out, lse = run_varlen(p)
    ro, rl = ref_varlen(p)
    compare(out, lse, ro, rl, what="bias 512")
    # a strong bias (std 2) sharpens the rows: gate on relative error
    p = fa_inputs.random_varlen(14, [200, 333], [700, 333], Hq=4, Hkv=1, D=128, causal=True,
                                bias_extent=512, bias_std=2.0)
    out, lse = run_varlen(p)
    ro, rl = ref_varlen(p)
    compare(None, lse, ro, rl, max_abs=1.0, mean_abs=1.0, rel_rms=1.0, what="bias 512 std 2 lse")
    compare_relative(out, ro, what="bias 512 std 2")


# ---------------------------------------------------------------------------
# the padded D=256 encoder workload (seqused_k, padding holds 1e4), in full
# ---------------------------------------------------------------------------
def test_encoder_d256_seqused():
    p = fa_inputs.make("encoder_d256_seqused")
    out, lse = run_dense(p)
    ro, rl = ref_dense(p)
    compare(out, lse, ro, rl, what="encoder_d256_seqused")


# ---------------------------------------------------------------------------
# full-size workloads on sampled rows
# ---------------------------------------------------------------------------
def _sample_rows(rng, B, Hq, lens, n):
    rows = []
    for _ in range(n):
        b = int(rng.integers(B))
        L = lens[b]
        i = int(rng.choice([0, L - 1, int(rng.integers(L)), min(L - 1, 127), min(L - 1, 128)]))
        rows.append((b, int(rng.integers(Hq)), i))
    return np.array(rows, dtype=np.int32)


def test_varlen_gqa_bias_workload_full():
    # the main workload, every row of every head ("mgoin/tml-fa4", argument
    # contract: every row i of every sequence b)
    p = fa_inputs.make("varlen_gqa_bias")
    out, lse = run_varlen(p)
    ro, rl = ref_varlen(p)
    compare(out, lse, ro, rl, what="varlen_gqa_bias full")


def test_video_dit_20480_sampled():
    # 12 TFLOP: the oracle checks sampled rows; every element must be written
    p = fa_inputs.make("video_dit_20480")
    out, lse = run_dense(p)
    assert torch.isfinite(out).all() and torch.isfinite(lse).all()
    rows = _sample_rows(np.random.default_rng(1), 1, 56, [20480], 256)
    ro, rl = oracle.attention_rows(p.q, p.k, p.v, rows, softmax_scale=p.softmax_scale)
    o = out.float().cpu()
    l = lse.cpu()
    go = np.stack([o[b, i, h].numpy() for b, h, i in rows])
    gl = np.array([float(l[b, h, i]) for b, h, i in rows])
    compare(go, gl, ro, rl, what="video_dit sampled")


@pytest.mark.parametrize("name", ["dense_d64", "tabpfn_d16", "vision_d72", "dense_d256"])
def test_dense_workloads_full(name):
    p = fa_inputs.make(name)
    out, lse = run_dense(p)
    ro, rl = ref_dense(p)
    compare(out, lse, ro, rl, what=f"{name} full")


# ---------------------------------------------------------------------------
# split-KV
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("ns", [0, 1, 3, 7])
@pytest.mark.parametrize("D", [16, 64, 72, 128, 256])
def test_splitkv_small(ns, D):
    p = fa_inputs.random_dense(21 + D, 3, 1, 1000, 8, 2, D)
    g = p.to(DEV)
    out, lse = fa.fa_fwd_splitkv(g.q, g.k, g.v, num_splits=ns)
    torch.cuda.synchronize()
    ro, rl = ref_dense(p)
    compare(out, lse, ro, rl, what=f"splitkv ns={ns} D={D}")


def test_splitkv_causal_multi_query_seqused():
    p = fa_inputs.random_dense(22, 2, 5, 900, 8, 2, 128, causal=True, seqused=[700, 900],
                               pad_value=1e4, bias_extent=128)
    g = p.to(DEV)
    out, lse = fa.fa_fwd_splitkv(g.q, g.k, g.v, num_splits=5, causal=True,
                                 seqused_k=g.seqused_k, rel_bias=g.rel_bias)
    torch.cuda.synchronize()
    ro, rl = ref_dense(p)
    compare(out, lse, ro, rl, what="splitkv causal seqused bias")


def test_decode_splitkv_workload():
    p = fa_inputs.make("decode_splitkv")
    g = p.to(DEV)
    out, lse = fa.fa_fwd_splitkv(g.q, g.k, g.v, softmax_scale=p.softmax_scale)
    torch.cuda.synchronize()
    del g
    o = out.float().cpu()
    l = lse.cpu()
    for b in range(p.B):  # one batch entry at a time keeps host memory small
        ro, rl = oracle.attention(p.q[b:b + 1], p.k[b:b + 1], p.v[b:b + 1],
                                  softmax_scale=p.softmax_scale)
        compare(o[b:b + 1], l[b:b + 1], ro, rl, what=f"decode b={b}")


# ---------------------------------------------------------------------------
# edge cases and invariants
# ---------------------------------------------------------------------------
def test_no_keys_gives_zero_and_minus_inf():
    p = fa_inputs.random_dense(30, 2, 40, 50, 4, 2, 128, seqused=[0, 50])
    out, lse = run_dense(p)
    ro, rl = ref_dense(p)
    compare(out, lse, ro, rl, what="seqused 0")
    assert (out[0] == 0).all() and torch.isneginf(lse[0]).all()


def test_zero_length_keys_everywhere():
    p = fa_inputs.random_dense(31, 1, 10, 0, 2, 2, 128)
    g = p.to(DEV)
    out, lse = fa.fa_fwd(g.q, g.k, g.v)
    torch.cuda.synchronize()
    assert (out == 0).all() and torch.isneginf(lse).all()


def test_empty_batch_is_a_no_op():
    q = torch.empty((0, 5, 2, 128), dtype=torch.bfloat16, device=DEV)
    out, lse = fa.fa_fwd(q, q, q)
    torch.cuda.synchronize()
    assert out.numel() == 0


def test_bias_none_equals_bias_zero():
    # tiles that meet the bias band take the half-tile softmax path, so a zero
    # bias need not reproduce the bias-free path bit for bit; both must meet
    # the oracle's gates and agree closely with each other
    p = fa_inputs.random_dense(32, 1, 300, 300, 4, 4, 128, causal=True)
    g = p.to(DEV)
    o1, l1 = fa.fa_fwd(g.q, g.k, g.v, causal=True)
    zb = torch.zeros((300, 4, 128), dtype=torch.bfloat16, device=DEV)
    o2, l2 = fa.fa_fwd(g.q, g.k, g.v, causal=True, rel_bias=zb)
    torch.cuda.synchronize()
    ro, rl = ref_dense(p)
    compare(o1, l1, ro, rl, what="no bias")
    compare(o2, l2, ro, rl, what="zero bias")
    assert (o1.float() - o2.float()).abs().max().item() <= 8e-3
    assert (l1 - l2).abs().max().item() <= 1e-4


def test_deterministic_run_to_run():
    p = fa_inputs.random_varlen(33, [500, 129], [700, 129], Hq=8, Hkv=2, D=128, causal=True,
                                bias_extent=256)
    o1, l1 = run_varlen(p)
    o2, l2 = run_varlen(p)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_stress_peaked_and_offset_values():
    # sharp softmax (q * 8) and values far from zero (V + 4): bf16 rounding of
    # O near 4 is ~0.016, so this case is gated on relative error
    p = fa_inputs.random_dense(34, 1, 256, 384, 4, 2, 128, causal=True, q_std=8.0,
                               v_offset=4.0)
    out, lse = run_dense(p)
    ro, rl = ref_dense(p)
    compare(None, lse, ro, rl, max_abs=1.0, mean_abs=1.0, rel_rms=1.0, what="stress lse")
    compare_relative(out, ro, what="stress")


def test_many_batches_beyond_grid_y_limit():
    # batch x heads well past 65535 (the grid-dimension limit a kernel that
    # put them in gridDim.y would hit)
    # 40 keys keep |O| small, so that the output's bf16 rounding stays below
    # the mean-abs gate
    B = 70000
    p = fa_inputs.random_dense(35, B, 2, 40, 1, 1, 128)
    out, lse = run_dense(p)
    rows = np.array([[b, 0, i] for b in (0, 1, 65535, 65536, B - 1) for i in (0, 1)],
                    dtype=np.int32)
    ro, rl = oracle.attention_rows(p.q, p.k, p.v, rows)
    o = out.float().cpu()
    l = lse.cpu()
    go = np.stack([o[b, i, h].numpy() for b, h, i in rows])
    gl = np.array([float(l[b, h, i]) for b, h, i in rows])
    compare(go, gl, ro, rl, what="B=70000")


def test_invalid_arguments_raise_and_write_nothing():
    q = torch.randn(1, 16, 4, 100, device=DEV, dtype=torch.bfloat16)  # not a multiple of 8
    with pytest.raises(fa.FAError) as e:
        fa.fa_fwd(q, q, q)
    assert e.value.name == "FA_ERR_UNSUPPORTED"
    q = torch.randn(1, 16, 4, 128, device=DEV, dtype=torch.bfloat16)
    k = torch.randn(1, 16, 3, 128, device=DEV, dtype=torch.bfloat16)
    out = torch.full_like(q, 7.0)
    with pytest.raises(fa.FAError):
        fa.fa_fwd(q, k, k, out=out)
    torch.cuda.synchronize()
    assert (out == 7.0).all()



# ---------------------------------------------------------------------------
# score and mask modifiers: sliding window, soft-cap (fa_mods)
# ---------------------------------------------------------------------------
WINDOW_CASES = [
    # B, Sq, Sk, Hq, Hkv, D, causal, (left, right)
    (2, 700, 700, 4, 2, 128, True, (200, -1)),    # causal sliding window
    (1, 500, 900, 8, 2, 128, False, (128, 64)),   # two-sided, k longer
    (1, 900, 400, 4, 4, 128, False, (-1, 0)),     # right bound only = causal
    (1, 300, 300, 8, 1, 256, True, (63, -1)),     # D = 256
    (2, 400, 650, 4, 2, 64, False, (300, 10)),    # D = 64
    (1, 260, 100, 4, 4, 128, False, (0, 0)),      # diagonal key only; early rows see none
    (1, 500, 500, 4, 1, 16, True, (100, -1)),     # D = 16
    (1, 400, 600, 4, 2, 72, False, (200, 50)),    # D = 72
]


@pytest.mark.parametrize("case", WINDOW_CASES)
def test_window(case):
    B, Sq, Sk, Hq, Hkv, D, causal, win = case
    p = fa_inputs.random_dense(200 + Sq + Sk, B, Sq, Sk, Hq, Hkv, D, causal=causal)
    out, lse = run_dense(p, window=win)
    ro, rl = ref_dense(p, window=win)
    compare(out, lse, ro, rl, what=f"window {case}")


@pytest.mark.parametrize("D", [16, 64, 72, 128, 256])
@pytest.mark.parametrize("causal", [False, True])
def test_softcap(D, causal):
    # q sharpened so that the cap matters (scaled scores well beyond it)
    p = fa_inputs.random_dense(300 + D, 2, 333, 410, 8, 2, D, causal=causal, q_std=4.0)
    out, lse = run_dense(p, softcap=5.0)
    ro, rl = ref_dense(p, softcap=5.0)
    compare(out, lse, ro, rl, what=f"softcap D{D} causal={causal}")


@pytest.mark.parametrize("D", [128, 256])
def test_varlen_window_softcap_bias(D):
    q_lens = [0, 1, 130, 513, 257, 64]
    k_lens = [3, 1, 200, 513, 300, 0]
    p = fa_inputs.random_varlen(41 + D, q_lens, k_lens, Hq=8, Hkv=2, D=D, causal=True,
                                bias_extent=256)
    out, lse = run_varlen(p, window=(150, -1), softcap=10.0)
    ro, rl = ref_varlen(p, window=(150, -1), softcap=10.0)
    compare(out, lse, ro, rl, what=f"varlen window+softcap+bias D{D}")


def test_splitkv_window_softcap():
    p = fa_inputs.random_dense(51, 3, 2, 3000, 8, 2, 128, q_std=3.0)
    g = p.to(DEV)
    out, lse = fa.fa_fwd_splitkv(g.q, g.k, g.v, num_splits=5, window=(1200, -1), softcap=8.0)
    torch.cuda.synchronize()
    ro, rl = ref_dense(p, window=(1200, -1), softcap=8.0)
    compare(out, lse, ro, rl, what="splitkv window+softcap")


def test_window_off_matches_no_modifiers():
    # the window encoding of "no bound" gives bit-identical results
    p = fa_inputs.random_dense(61, 1, 300, 300, 4, 2, 128, causal=True)
    a, la = run_dense(p)
    b, lb = run_dense(p, window=(-1, -1), softcap=0.0)
    assert torch.equal(a, b) and torch.equal(la, lb)


def test_local_window_softcap_workload_full():
    p = fa_inputs.make("local_window_softcap")
    out, lse = run_dense(p, window=p.window, softcap=p.softcap)
    ro, rl = ref_dense(p, window=p.window, softcap=p.softcap)
    compare(out, lse, ro, rl, what="local_window_softcap full")


def test_watchdog_timeout_is_reported_and_the_device_stays_usable():
    # a bounded wait that nothing completes must give up, record the timeout
    # code (1) and leave the context usable
    assert fa.check_device_error() == 0
    fa.watchdog_selftest(0.05)
    assert fa.check_device_error(clear=True) == 1
    assert fa.check_device_error() == 0
    p = fa_inputs.random_dense(71, 1, 130, 200, 4, 2, 128, causal=True)
    out, lse = run_dense(p)
    ro, rl = ref_dense(p)
    compare(out, lse, ro, rl, what="after the watchdog self-test")


# ---------------------------------------------------------------------------
# CUDA graphs: the library allocates nothing and never synchronises, so a
# forward captured once replays on new inputs with the same bits as a call
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("D", [16, 64, 128])
def test_cuda_graph_capture_replays_the_forward(D):
    p = fa_inputs.random_dense(400 + D, 2, 200, 333, 8, 2, D, causal=True)
    g = p.to(DEV)
    q = g.q.clone()
    out = torch.empty_like(q)
    lse = torch.empty((2, 8, 200), dtype=torch.float32, device=DEV)
    fa.fa_fwd(q, g.k, g.v, causal=True, out=out, lse=lse)  # one-time setup outside capture
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        fa.fa_fwd(q, g.k, g.v, causal=True, out=out, lse=lse)
    p2 = fa_inputs.random_dense(500 + D, 2, 200, 333, 8, 2, D, causal=True)
    q.copy_(p2.q.to(DEV))
    graph.replay()
    torch.cuda.synchronize()
    ref_o, ref_l = fa.fa_fwd(q, g.k, g.v, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(out, ref_o) and torch.equal(lse, ref_l)
    ro, rl = oracle.attention(p2.q, p.k, p.v, causal=True, softmax_scale=p.softmax_scale)
    compare(out, lse, ro, rl, what=f"graph replay D{D}")
    del graph


def test_cuda_graph_capture_of_splitkv_with_a_workspace():
    p = fa_inputs.random_dense(600, 2, 1, 3000, 8, 2, 128)
    g = p.to(DEV)
    ns = 5
    ws = torch.empty(fa.splitkv_workspace_bytes(2, 1, 8, 128, ns), dtype=torch.uint8, device=DEV)
    out = torch.empty_like(g.q)
    lse = torch.empty((2, 8, 1), dtype=torch.float32, device=DEV)
    fa.fa_fwd_splitkv(g.q, g.k, g.v, num_splits=ns, out=out, lse=lse, workspace=ws)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        fa.fa_fwd_splitkv(g.q, g.k, g.v, num_splits=ns, out=out, lse=lse, workspace=ws)
    out.zero_()
    graph.replay()
    torch.cuda.synchronize()
    ro, rl = ref_dense(p)
    compare(out, lse, ro, rl, what="graph replay split-KV")
    del graph


# ---------------------------------------------------------------------------
# every head dim the library serves: multiples of 8 from 16 to 256, each in
# the kernel of the next width up (padding columns read as zeros, never stored)
# ---------------------------------------------------------------------------
SWEEP_D = [16, 24, 32, 40, 48, 56, 64, 72, 88, 96, 104, 120, 128, 136, 192, 248, 256]


@pytest.mark.parametrize("D", SWEEP_D)
def test_head_dim_sweep_dense_causal_gqa(D):
    p = fa_inputs.random_dense(700 + D, 1, 200, 333, 8, 2, D, causal=True)
    out, lse = run_dense(p)
    ro, rl = ref_dense(p)
    compare(out, lse, ro, rl, what=f"sweep dense D{D}")


@pytest.mark.parametrize("D", [24, 40, 56, 88, 120, 136])
def test_head_dim_sweep_varlen_bias_and_splitkv(D):
    p = fa_inputs.random_varlen(800 + D, [0, 130, 257, 1], [5, 300, 257, 1], Hq=8, Hkv=2, D=D,
                                causal=True, bias_extent=128)
    out, lse = run_varlen(p)
    ro, rl = ref_varlen(p)
    compare(out, lse, ro, rl, what=f"sweep varlen bias D{D}")
    q = fa_inputs.random_dense(900 + D, 2, 1, 1500, 8, 2, D)
    g = q.to(DEV)
    out, lse = fa.fa_fwd_splitkv(g.q, g.k, g.v, num_splits=3)
    torch.cuda.synchronize()
    ro, rl = ref_dense(q)
    compare(out, lse, ro, rl, what=f"sweep split-KV D{D}")


# ---------------------------------------------------------------------------
# problem size picks the kernel: fewer two-tile units than SMs run one Q tile
# per CTA (most cases above); these shapes have enough units for two tiles
# ---------------------------------------------------------------------------
TWO_TILE_CASES = [
    # B, Sq, Sk, Hq, Hkv, D, causal  -> >= 148 units of two 128-row tiles
    (2, 300, 300, 48, 48, 128, True),
    (2, 300, 333, 64, 16, 64, False),
    (2, 260, 260, 40, 40, 128, False),
    (2, 300, 300, 48, 48, 16, True),   # width 16: three tiles (96 units, 1 wave)
    (2, 300, 333, 64, 16, 72, False),
    (2, 260, 260, 40, 40, 48, True),
]


@pytest.mark.parametrize("case", TWO_TILE_CASES)
def test_two_tile_kernel_at_moderate_sizes(case):
    B, Sq, Sk, Hq, Hkv, D, causal = case
    p = fa_inputs.random_dense(1000 + Hq + D, B, Sq, Sk, Hq, Hkv, D, causal=causal)
    out, lse = run_dense(p)
    ro, rl = ref_dense(p)
    compare(out, lse, ro, rl, what=f"two-tile {case}")


def test_two_tile_kernel_varlen_bias():
    p = fa_inputs.random_varlen(1100, [300, 513, 129], [300, 513, 129], Hq=64, Hkv=8, D=128,
                                causal=True, bias_extent=256)
    out, lse = run_varlen(p)
    ro, rl = ref_varlen(p)
    compare(out, lse, ro, rl, what="two-tile varlen bias")


def test_two_tile_kernel_fp16_varlen_bias():
    p = fa_inputs.random_varlen(1200, [300, 513, 129], [300, 513, 129], Hq=64, Hkv=8, D=128,
                                dtype=torch.float16, causal=True, bias_extent=256)
    out, lse = run_varlen(p)
    ro, rl = ref_varlen(p)
    compare(out, lse, ro, rl, what="two-tile fp16 varlen bias")


@pytest.mark.parametrize("D", [64, 128])
def test_one_tile_kernel_fp16_varlen_bias(D):
    p = fa_inputs.random_varlen(1300 + D, [0, 77, 300], [5, 200, 300], Hq=8, Hkv=2, D=D,
                                dtype=torch.float16, causal=True, bias_extent=128)
    out, lse = run_varlen(p)
    ro, rl = ref_varlen(p)
    compare(out, lse, ro, rl, what=f"one-tile fp16 varlen bias D{D}")


# ---------------------------------------------------------------------------
# widths 16 to 96: three Q tiles per CTA (64-key tiles from 48 up) when the
# problem has no relative bias and the three-tile units fill the waves about
# as well (30 x waves(3) <= 22 x waves(2)); two tiles with a bias or when they
# fill them better
# ---------------------------------------------------------------------------
THREE_TILE_CASES = [
    # B, Sq, Sk, Hq, Hkv, D, causal, dtype -> units of 2 / 3 tiles (waves of 148)
    (2, 700, 650, 32, 8, 32, False, torch.bfloat16),   # 176 / 128 (2 / 1 waves)
    (1, 1000, 1000, 40, 40, 24, True, torch.bfloat16),  # 160 / 120 (2 / 1), width 32
    (2, 700, 650, 32, 8, 16, True, torch.float16),     # 176 / 128 (2 / 1)
    (1, 2000, 1800, 24, 24, 16, False, torch.float16),  # 192 / 144 (2 / 1)
    (2, 700, 650, 32, 8, 64, False, torch.bfloat16),   # 176 / 128, width 64
    (1, 1000, 1000, 40, 40, 48, True, torch.float16),   # 160 / 120, width 48
    (1, 2000, 1800, 24, 24, 40, False, torch.bfloat16),  # 192 / 144, width 48
    (2, 700, 650, 32, 8, 64, True, torch.float16),     # 176 / 128, width 64
    (2, 700, 650, 32, 8, 72, False, torch.bfloat16),   # 176 / 128, width 80
    (1, 1000, 1000, 40, 40, 96, True, torch.float16),   # 160 / 120, width 96
    (1, 2000, 1800, 24, 24, 88, False, torch.bfloat16),  # 192 / 144, width 96
]


@pytest.mark.parametrize("case", THREE_TILE_CASES)
def test_three_tile_kernel(case):
    B, Sq, Sk, Hq, Hkv, D, causal, dt = case
    p = fa_inputs.random_dense(1500 + Sq + D, B, Sq, Sk, Hq, Hkv, D, causal=causal, dtype=dt)
    out, lse = run_dense(p)
    ro, rl = ref_dense(p)
    compare(out, lse, ro, rl, what=f"three-tile {case}")


@pytest.mark.parametrize("D", [32, 64, 80])
def test_three_tile_kernel_varlen_ragged(D):
    # 4 heads packed per K/V head; the launch is sized by the longest sequence
    # (4800 packed rows: 608 two-tile, 416 three-tile units, 5 / 3 waves); a
    # one-token sequence among them
    p = fa_inputs.random_varlen(1600 + D, [700, 1, 385, 1200], [650, 9, 385, 1200], Hq=32, Hkv=8,
                                D=D, causal=True)
    out, lse = run_varlen(p)
    ro, rl = ref_varlen(p)
    compare(out, lse, ro, rl, what=f"three-tile varlen D{D}")


@pytest.mark.parametrize("D", [16, 32, 64, 96])
def test_three_tile_modifier_kernel(D):
    p = fa_inputs.random_dense(1700 + D, 2, 700, 700, 32, 32, D, causal=True, q_std=3.0)
    out, lse = run_dense(p, window=(150, -1), softcap=6.0)
    ro, rl = ref_dense(p, window=(150, -1), softcap=6.0)
    compare(out, lse, ro, rl, what=f"three-tile window+softcap D{D}")


@pytest.mark.parametrize("D", [32, 64, 72])
def test_narrow_two_tile_kernel_with_bias(D):
    # 8 heads packed per K/V head: 408 two-tile units, a relative bias -> two tiles
    p = fa_inputs.random_varlen(1800 + D, [300, 513, 129], [300, 513, 129], Hq=64, Hkv=8, D=D,
                                causal=True, bias_extent=128)
    out, lse = run_varlen(p)
    ro, rl = ref_varlen(p)
    compare(out, lse, ro, rl, what=f"narrow two-tile varlen bias D{D}")


@pytest.mark.parametrize("D", [16, 64, 96])
def test_narrow_two_tile_kernel_by_waves(D):
    # 320 units of two tiles and 320 of three (S = 512): three waves either
    # way, so the two-tile kernel runs
    p = fa_inputs.random_dense(1900 + D, 2, 512, 512, 80, 80, D)
    out, lse = run_dense(p)
    ro, rl = ref_dense(p)
    compare(out, lse, ro, rl, what=f"narrow two-tile by waves D{D}")


@pytest.mark.parametrize("D", [64, 128])
def test_two_tile_modifier_kernel(D):
    # >= 148 two-tile units, left window + soft-cap: the two-tile MODS kernel
    # (at D = 64 the units fill one wave of three tiles, so that one runs)
    p = fa_inputs.random_dense(1400 + D, 2, 300, 300, 48, 48, D, causal=True, q_std=3.0)
    out, lse = run_dense(p, window=(90, -1), softcap=6.0)
    ro, rl = ref_dense(p, window=(90, -1), softcap=6.0)
    compare(out, lse, ro, rl, what=f"two-tile window+softcap D{D}")


# ---------------------------------------------------------------------------
# head dim 256 beyond one wave of CTA pairs: the paired-SM kernel (units of
# 256 rows over two SMs); the smaller D=256 cases above take the one-CTA one
# ---------------------------------------------------------------------------
PAIR_CASES = [
    # B, Sq, Sk, Hq, Hkv, D, causal -> > 74 units of 256 packed rows
    (2, 300, 300, 48, 48, 256, True),
    (2, 300, 333, 64, 8, 256, False),    # 8 heads packed per K/V head
    (2, 260, 260, 40, 40, 136, False),   # a head dim padded up to 256
]


@pytest.mark.parametrize("case", PAIR_CASES)
def test_pair_kernel_dense(case):
    B, Sq, Sk, Hq, Hkv, D, causal = case
    p = fa_inputs.random_dense(1500 + Hq + D, B, Sq, Sk, Hq, Hkv, D, causal=causal)
    out, lse = run_dense(p)
    ro, rl = ref_dense(p)
    compare(out, lse, ro, rl, what=f"pair {case}")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_pair_kernel_varlen_bias(dtype):
    p = fa_inputs.random_varlen(1600, [300, 513, 129, 0], [300, 513, 129, 5], Hq=64, Hkv=8, D=256,
                                dtype=dtype, causal=True, bias_extent=256)
    out, lse = run_varlen(p)
    ro, rl = ref_varlen(p)
    compare(out, lse, ro, rl, what=f"pair varlen bias {dtype}")


def test_pair_kernel_window_softcap_seqused():
    p = fa_inputs.random_dense(1700, 2, 300, 400, 48, 48, 256, causal=True, q_std=3.0,
                               seqused=[350, 400], pad_value=1e4)
    out, lse = run_dense(p, window=(90, -1), softcap=6.0)
    ro, rl = ref_dense(p, window=(90, -1), softcap=6.0)
    compare(out, lse, ro, rl, what="pair window+softcap+seqused")
