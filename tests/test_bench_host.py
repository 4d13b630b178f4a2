"""Host-side logic of bench.py (no GPU): the source hash that ties the counters
in profiles/traffic.json to the code they were taken on, and the byte / flop
model of the attention."""
import bench
import workloads


def test_code_hash_ignores_comments_and_whitespace(tmp_path):
    a = tmp_path / "a.cu"
    a.write_text("int f(int x) {  // twice\n    return 2 * x;\n}\n/* done */\n")
    b = tmp_path / "b.cu"
    b.write_text("// a comment of its own\nint f(int x) {\n  return 2 * x; }\n")
    c = tmp_path / "c.cu"
    c.write_text("int f(int x) {\n    return 3 * x;\n}\n")
    assert bench.code_sha(str(a)) == bench.code_sha(str(b))
    assert bench.code_sha(str(a)) != bench.code_sha(str(c))


def test_attention_byte_and_flop_model_of_the_512_pool():
    # workload 3 at step 1: shared K/V once per request, the beams' earlier
    # Unshared tokens, this step's k/v read and appended, q and O, LSE
    w = workloads.WORKLOADS[3]
    att_bytes, att_flops, _ = bench.algorithmic(w, 1, True, 0)
    B, BW, Hq, Hkv, D, P = w.B, w.BW, w.Hq, w.Hkv, w.D, w.prompt[0]
    expect = (2 * B * Hkv * P * D * 2 + 2 * B * BW * Hkv * D * 2 + 2 * B * BW * Hkv * D * 4
              + 2 * B * BW * Hq * D * 2 + B * BW * Hq * 4)
    assert att_bytes == expect
    assert att_flops == 4.0 * B * BW * Hq * D * (P + 2)


def test_attention_kernel_named_per_workload():
    # short items (workload 2: 8 prompt chunks) run the one-O variant, long
    # ones (32 or more chunks) the two-accumulator kernel, D = 64 the small-row
    # kernel with the merge
    assert bench.attention_kernel(workloads.WORKLOADS[2]) == "attn_tc_one_o_kernel"
    assert bench.attention_kernel(workloads.WORKLOADS[3]) == "attn_tc_kernel"
    assert bench.attention_kernel(workloads.WORKLOADS[5]) == "attn_tc_kernel"
    assert bench.attention_kernel(workloads.WORKLOADS[1]).startswith("attn_small_kernel")


def test_traffic_is_reported_only_for_the_workload_it_was_taken_on():
    # the committed counters belong to one workload each; another workload's
    # line (or a kernel with no capture) reports none
    w2, w3 = workloads.WORKLOADS[2].name, workloads.WORKLOADS[3].name
    one_o = bench.measured_traffic("attn_tc_one_o_kernel", w2)
    assert one_o is None or one_o > 0
    assert bench.measured_traffic("attn_tc_one_o_kernel", w3) is None
    assert bench.measured_traffic("attn_tc_kernel", w2) is None
    assert bench.measured_traffic("no_such_kernel", w2) is None


def test_step_percentiles_and_secondary_rates():
    xs = [float(i) for i in range(1, 11)]
    assert bench._pct(xs, 10) == 2.0 and bench._pct(xs, 90) == 9.0 and bench._pct([3.0], 50) == 3.0
    # workload 2 over 1 ms: step 0 scores the distinct first tokens of one beam
    # per request, later steps the mask's entries; every live row reads V logits
    w = workloads.WORKLOADS[2]
    import numpy as np
    items = np.array([[1, 2, 3], [1, 5, 6], [7, 2, 3]], dtype=np.int32)
    r = bench.secondary_rates(w, items, [0, 100, 20], 1.0)
    assert r["valid_candidates_per_decode"] == 2 * w.B + 120
    assert r["tokens_scored_per_decode"] == w.B * w.V * (1 + 2 * w.BW)
    assert r["valid_candidates_per_s"] == r["valid_candidates_per_decode"] * 1e3
