"""The seeded input recipes (host only): the drawn lengths and sizes that the
documentation, the bench lines and the profiles quote."""
import torch

from exact_io_aware_tmem_b200.workloads import (DECODE_WORKLOADS, WORKLOADS, decode_bytes,
                                                flops, make_inputs)


def test_packed_workload_lengths():
    # 16 lengths drawn with randint(128, 4097) from the workload's generator.
    w = WORKLOADS["bf16_varlen_h16_d128_16seqs"]
    g = torch.Generator("cpu").manual_seed(w.seed)
    lengths = torch.randint(128, 4097, (16,), generator=g).tolist()
    assert sum(lengths) == 33355 and max(lengths) == 4019 and min(lengths) >= 128
    inp = make_inputs(w)
    assert inp.cu_seqlens.tolist()[-1] == 33355 and inp.max_seqlen == 4019
    assert inp.q.shape == (33355, 16, 128)


def test_dense_workloads_shapes_and_flops():
    w = WORKLOADS["bf16_causal_b2_h16_n8192_d128"]
    fl_f, fl_b = flops([w.N] * w.B, w.H, w.D, w.causal)
    assert round(fl_f / 1e9, 1) == 549.8 and abs(fl_b / fl_f - 2.5) < 1e-12
    w = WORKLOADS["bf16_fwd_b4_h16_n2048_d64"]
    fl_f, _ = flops([w.N] * w.B, w.H, w.D, w.causal)
    assert round(fl_f / 1e9, 1) == 68.7
    w = WORKLOADS["bf16_gqa_causal_b1_h32_kv8_n16384_d128"]
    fl_f, fl_b = flops([w.N] * w.B, w.H, w.D, w.causal)
    assert round(fl_f / 1e9, 1) == 2199.0 and round(fl_b / 1e9, 1) == 5497.6
    w = WORKLOADS["bf16_varlen_h16_d128_16seqs"]
    fl_f, fl_b = flops(make_inputs(w).cu_seqlens.diff().tolist(), w.H, w.D, w.causal)
    assert round(fl_f / 1e9, 1) == 685.3 and round(fl_b / 1e9, 1) == 1713.4


def test_inputs_are_reproducible():
    w = WORKLOADS["f32_b1_h2_n128_d64"]
    a, b = make_inputs(w), make_inputs(w)
    for x, y in ((a.q, b.q), (a.k, b.k), (a.v, b.v), (a.do, b.do)):
        assert torch.equal(x, y)


def test_decode_workload_cache_sizes():
    # Cache lengths uniform in [4096, 32768] from the generator seeded with
    # seed + 1000; the totals are the cached tokens the decode lines report.
    want = {
        "bf16_decode_b16_h32_kv8_d128_q1": 312094,
        "bf16_decode_paged64_b16_h32_kv8_d128_q1": 257430,
        "bf16_decode_b16_h32_kv8_d128_q8": 213790,
    }
    for name, tokens in want.items():
        w = DECODE_WORKLOADS[name]
        lengths = w.lengths()
        assert len(lengths) == 16 and all(4096 <= n <= 32768 for n in lengths)
        assert sum(lengths) == tokens
    w = DECODE_WORKLOADS["bf16_decode_b16_h32_kv8_d128_q1"]
    # K and V at 8 kv heads, D = 128, bf16: the algorithmic bytes of one call.
    assert decode_bytes(w.lengths(), 8, 128) == 2 * 312094 * 8 * 128 * 2
