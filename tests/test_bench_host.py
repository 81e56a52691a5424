"""Host-side logic of bench.py (no GPU): the algorithmic flop and byte counts
behind the roofline figures, and the clock record's summary."""
import bench
from mla_latent_kv_write_b200 import inputs as I


def _per_qkh(d):
    # flops that one more key adds to one query row, per head
    return (bench.flops_attention(d, 1, 1, 2) - bench.flops_attention(d, 1, 1, 1)) / d.n_heads


def test_attention_flops_per_query_key_head():
    # absorbed form: scores over d_c + d_rope, then P.C over d_c -> 832 at the Wan shape;
    # the five rank / RoPE sweep points give 448 / 800 / 832 / 896 / 1600
    assert _per_qkh(I.WAN) == 832
    got = [_per_qkh(I.sweep_dims(dc, dr)) for dc, dr in I.SWEEP_POINTS]
    assert got == [448, 800, 832, 896, 1600]


def test_attention_flops_wan_layer_call():
    # 4680 queries x 32760 keys x 12 heads, plus the per-(query, head) absorption and
    # W_uv epilogue: 1.5355 TFLOP per call
    f = bench.flops_attention(I.WAN, 1, 4680, 32760)
    assert abs(f - 1.5355e12) / 1.5355e12 < 1e-4
    per_qh = (bench.flops_attention(I.WAN, 1, 2, 0) - bench.flops_attention(I.WAN, 1, 1, 0)) / I.WAN.n_heads
    assert per_qh == 2 * 96 * 192 + 2 * 192 * 128


def test_cache_write_bytes_and_flops_per_token():
    # x row in (2 d bytes) + one cache row out (2 (d_c + d_rope) bytes) = 3520 B per token
    assert bench.bytes_cache_write(I.WAN, 1, 1) == 3520
    assert bench.flops_cache_write(I.WAN, 1, 1) == 2 * 224 * 1536


def test_clock_summary_decodes_reasons_and_filters_idle_samples():
    c = bench.ClockSampler(0)
    c.thread = object()  # summary reads the NVML rows
    c.source = "fake"
    power_cap = dict(bench.ClockSampler.REASON_BITS)["sw_power_cap"]
    c.rows = [
        (1965.0, 1965.0, 120.0, 0),            # idle sample, dropped from the median
        (1900.0, 1965.0, 650.0, power_cap),
        (1800.0, 1965.0, 700.0, 0),
        (1700.0, 1965.0, 710.0, 0),
    ]
    s = c.summary()
    assert s["sm_mhz"] == 1800.0 and s["samples"] == 3 and s["samples_all"] == 4
    assert s["sm_mhz_range_all"] == [1700.0, 1965.0]
    assert s["reasons"] == ["sw_power_cap"] and s["power_w_max"] == 710.0


def test_clock_summary_without_samples():
    c = bench.ClockSampler(0)
    s = c.summary()
    assert s["sm_mhz"] is None and s["reasons"] == ["no samples"]


def test_both_arms_share_the_workload_config():
    # both arms print the same config object, so their lines compare directly
    c = bench.workload_config(1)
    assert c["flops_per_step"] == bench.flops_attention(I.WAN, 1, 4680, 32760) + bench.flops_cache_write(I.WAN, 1, 4680)
    assert c["keys"] == 32760 and c["query_tokens_per_step"] == 4680 and c["global_batch"] == 1
    assert bench.workload_config(4)["global_batch"] == 4
    import inspect
    for fn in (bench.run_reference, bench.run_gpu):
        assert "workload_config(world)" in inspect.getsource(fn)
