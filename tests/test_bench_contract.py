"""The pieces of bench.py's JSON line that do not need a GPU: the roofline record, the op and
byte models behind it, and the workload config both arms report."""
import math

import bench
import workloads as W


def test_roofline_record_has_the_contract_keys():
    cfg = W.CONFIGS[bench.CONFIG_KEY]
    clk = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []}
    r = bench.roofline(cfg, 40, 40 * 0.235, clk, 4, 2.75, 40, 40 * 0.27)
    for k in ("bound", "achieved", "peak", "unit", "frac", "traffic"):
        assert k in r, k
    assert r["bound"] == "alu" and r["unit"] == "Tops (int32)"
    assert math.isclose(r["frac"], r["achieved"] / r["peak"])
    # achieved = algorithmic ops per launch / average launch time
    assert math.isclose(r["achieved"], 4 * bench.ip_row_ops(cfg) / 235e-6 / 1e12)
    assert math.isclose(r["traffic"], 4 * bench.IP_ROW_TRAFFIC_PER_UNIT)
    assert bench.roofline(cfg, 0, 0.0, clk, 4, 2.75, 0, 0.0) is None


def test_alu_peak_and_op_model():
    # 148 SMs x 4 sub-partitions x 32 lanes x 1 instruction per clock
    assert math.isclose(bench.alu_peak_tops(1965.0), 148 * 128 * 1965e6 / 1e12)
    cfg = W.CONFIGS[bench.CONFIG_KEY]
    ops = bench.ip_row_ops(cfg)
    assert 1.1e9 < ops < 1.25e9            # about 1.17 G int32 operations per key switch


def test_both_arms_report_the_same_workload():
    cfg = W.CONFIGS[bench.CONFIG_KEY]
    ours = bench.workload_config(cfg, 8, 1, False, "2 CUDA streams x 4 units")
    ref = bench.workload_config(cfg, 8, 1)
    ours.pop("streams")
    assert ours == ref
    assert ref["workload"].startswith("n16-full: N=2^16") and ref["batch"] == 8
    assert ref["key_switches_per_step"] == 16


def test_compulsory_bytes_per_unit():
    cfg = W.CONFIGS[bench.CONFIG_KEY]
    limb = cfg.n * 4
    b = bench.step_bytes_min(cfg)
    # at least the two input ciphertexts, the two keys' b halves and the output
    na, ext, beta = cfg.level + 1, cfg.level + 1 + cfg.n_p, -(-(cfg.level + 1) // cfg.alpha)
    assert b >= (4 * na + 2 * beta * ext + 2 * na) * limb
