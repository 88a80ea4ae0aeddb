"""Host-side arithmetic of bench.py that feeds the reported numbers: the
algorithmic bytes of a decode step, the memory footprint of a concurrency
sweep batch and the throughput-model rows. No GPU needed."""
import bench
import synth

D = 128


def test_algorithmic_bytes_of_the_128k_step():
    # 16 requests x 8 KV heads x 131072 keys; B = 92 bits per key; k = 2048
    # rows per (request, KV head) of K and V in bf16 plus one 32-byte
    # slot-map sector each
    a = bench.algorithmic_bytes(bench.WORKLOADS["qwen3-8b-128k"], 92)
    keys = 16 * 8 * 131072
    assert a["keys"] == keys
    assert a["scan"] == keys * 92 / 8
    assert a["rows"] == 16 * 8 * 2048 * (2 * D * 2 + 32)
    assert a["total"] == a["scan"] + a["rows"]


def test_sweep_footprint_of_one_128k_request():
    # per layer: the 4-plane index of 8 heads x 128 channels (131072 / 32
    # words each), the int32 slot map and the hot K and V buffers of 4096
    # slots; once per request: the full K and V store
    n = 131072
    per_layer = 8 * D * 4 * (n // 32) * 4 + 8 * n * 4 + 2 * 8 * 4096 * D * 2
    full = 2 * 8 * n * D * 2
    fp = bench.sweep_footprint([n])
    assert fp["bytes"] == 36 * per_layer + full
    assert not fp["over_capacity"]


def test_sweep_capacity_flags_follow_the_180_gb_cap():
    # the sweep's own length draws: batches up to 64 fit, 128 and 256 do not
    c = bench.SWEEP
    flags = {}
    for b in c["batches"]:
        nl = synth.ragged_lengths(b, seed=c["seed"] * 1000 + b)
        fp = bench.sweep_footprint(nl)
        flags[b] = fp["over_capacity"]
        assert fp["over_capacity"] == (fp["gb"] > c["cap_gb"])
    assert not any(flags[b] for b in (1, 2, 4, 8, 16, 32, 64))
    assert flags[128] and flags[256]
    # more requests never need less memory
    sizes = [bench.sweep_footprint([65536] * b)["bytes"] for b in (1, 2, 4)]
    assert sizes[0] < sizes[1] < sizes[2]


def test_model_rows_add_the_link_time_and_stop_at_capacity():
    sweep = {"batches": [
        {"batch": 1, "mean_length": 65536, "ms_per_layer_step": 0.05},
        {"batch": 16, "mean_length": 65536, "ms_per_layer_step": 0.2},
        {"batch": 256, "mean_length": 100000, "ms_per_layer_step": None},  # over capacity: no row
    ]}
    m = bench.model_entry(sweep, hbm_budget=150e9, miss=0.2)
    assert [r["batch"] for r in m["rows"]] == [1, 16]
    entry = 8 * 2 * D * 2  # one selected entry of one layer: K and V rows of 8 KV heads
    for r, e in zip(m["rows"], sweep["batches"]):
        tc = 36 * e["ms_per_layer_step"] / 1e3
        assert abs(r["t_compute_ms"] - tc * 1e3) < 1e-12
        assert abs(r["ideal_tokens_per_s"] - e["batch"] / tc) < 1e-6
        for name, link in m["links"].items():
            row = r["links"][name]
            if row["tokens_per_s"] is None:
                assert e["batch"] > row["batch_max"]
                continue
            fetch = e["batch"] * 36 * 2048 * 0.2 * entry / (link["gbs"] * 1e9)
            expect = e["batch"] / (tc + fetch)
            assert abs(row["tokens_per_s"] - expect) <= 1e-9 * expect
            assert row["tokens_per_s"] < r["ideal_tokens_per_s"]
