"""Host logic of bench.py that needs no GPU: the per-configuration table
covers the per-configuration targets (configs 1-3 and 5), and the fused-reduction overhead is
taken against the same workload's unsharded layer at the same batch."""
import bench


def test_config_cases_cover_the_target_configs():
    names = {c[0].split(":")[0] for c in bench.CONFIG_CASES}
    assert {"config 1", "config 2", "config 3", "config 5"} <= names
    c3 = [c for c in bench.CONFIG_CASES if c[0].startswith("config 3")]
    # the 70B layer at t = 4 (both reduction modes) and its unsharded twin
    assert any(c[5] == 4 and c[8] == "fused" for c in c3)
    assert any(c[5] == 4 and c[8] == "separate" for c in c3)
    assert any(c[5] == 1 for c in c3)
    for c in c3:
        assert c[1:5] == (8192, 64, 8, 28672) and c[6:8] == (16, 8192)
    c2 = [c for c in bench.CONFIG_CASES if c[0].startswith("config 2")]
    assert {(c[5], c[6]) for c in c2} == {(t, B) for t in (1, 2, 4) for B in (1, 16)}


def test_overhead_against_the_unsharded_layer():
    rows = [
        {"workload": "w", "t": 1, "batch": 16, "reduce": "fused", "us_per_layer": 100.0},
        {"workload": "w", "t": 4, "batch": 16, "reduce": "fused", "us_per_layer": 103.0},
        {"workload": "w", "t": 4, "batch": 16, "reduce": "separate", "us_per_layer": 110.0},
        {"workload": "w", "t": 4, "batch": 1, "reduce": "fused", "us_per_layer": 50.0},
        {"workload": "v", "t": 2, "batch": 16, "reduce": "fused", "us_per_layer": 10.0},
    ]
    bench.attach_overheads(rows)
    assert abs(rows[1]["overhead_vs_t1"] - 0.03) < 1e-12
    assert "overhead_vs_t1" not in rows[0]
    assert "overhead_vs_t1" not in rows[2]  # separate mode is not the fused overhead
    assert "overhead_vs_t1" not in rows[3]  # no unsharded row at that batch
    assert "overhead_vs_t1" not in rows[4]  # another workload
