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
    t = bench.ip_row_traffic_per_unit()
    assert r["traffic"] == (None if t is None else 4 * t)
    assert bench.roofline(cfg, 0, 0.0, clk, 4, 2.75, 0, 0.0) is None


def test_traffic_figure_is_tied_to_the_kernel_sources(monkeypatch):
    """A DRAM figure taken on other kernel sources is never reported."""
    monkeypatch.setitem(bench.IP_ROW_TRAFFIC, "sources_sha16", "0" * 16)
    monkeypatch.setitem(bench.IP_ROW_TRAFFIC, "bytes_per_unit", 1.0e8)
    assert bench.ip_row_traffic_per_unit() is None
    monkeypatch.setitem(bench.IP_ROW_TRAFFIC, "sources_sha16", bench.kernel_sources_sha16())
    assert bench.ip_row_traffic_per_unit() == 1.0e8


def test_kernel_roofline_uses_the_measured_peaks():
    """With measured peaks the kernel's floor is the slower of all operations at the general int32
    rate and its ChaCha12 blocks at the measured ChaCha12 rate."""
    cfg = W.CONFIGS[bench.CONFIG_KEY]
    clk = {"sm_mhz": 1965.0}
    peaks = {"int_tops": 30.0, "chacha_tops": 15.0, "int_probe": "mix_lop3_imad", "source": "test"}
    r = bench.roofline(cfg, 10, 10 * 0.2, clk, 4, 2.5, 0, 0.0, peaks)
    ops, blocks = 4 * bench.ip_row_ops(cfg), 4 * bench.chacha_blocks(cfg, cfg.level)
    t_floor = max(ops / 30e12, blocks * 608 / 15e12)
    assert math.isclose(r["peak"], ops / t_floor / 1e12)
    assert math.isclose(r["frac"], t_floor / 200e-6)


def test_path_op_model_matches_the_unit_costs():
    """Per key switch at N=2^16, 36+12 primes, dnum 3, level 35: ModUp 0.83 G, ChaCha12 + inner
    product 0.88 G, ModDown 0.58 G, 2.29 G in all; 144 (digit, limb) pairs of N/8 ChaCha12 blocks."""
    cfg = W.CONFIGS[bench.CONFIG_KEY]
    n, log_n = cfg.n, cfg.log_n
    ntt = n // 2 * log_n * 8
    assert bench.limb_ntt_ops(log_n) == ntt
    assert bench.chacha_blocks(cfg, 35) == 3 * 48 * n // 8
    # 36 inverse NTTs; per digit 36 targets x (12 multiply-adds + 1 reduction) and 36 NTTs
    assert bench.modup_ops(cfg, 35) == 36 * ntt + 3 * 36 * n * (12 * 2 + 8) + 108 * ntt
    # two components of 12 inverse NTTs, 36 x (12 multiply-adds + reduction), 36 NTTs, 36 combines
    assert bench.moddown_ops(cfg, 35) == 2 * (12 * ntt + 36 * n * (12 * 2 + 8) + 36 * ntt + 36 * n * 6)
    assert 2.2e9 < bench.keyswitch_ops(cfg, 35) < 2.4e9
    # at level 20 with dnum 4 (alpha 9): digits of 9, 9, 3 primes
    c5 = W.CONFIGS["n16-stream64"]
    assert bench.digit_sizes(c5, 20) == [9, 9, 3]
    assert bench.key_limbs(c5, 20) == 3 * 33


def test_path_roofline_takes_the_slower_floor():
    peaks = {"int_tops": 20.0, "chacha_tops": 10.0, "source": "test"}
    r = bench.path_roofline(2e9, 1e6, 1e8, 1e-3, peaks)
    t_int = max(2e9 / 20e12, 1e6 * 608 / 10e12)
    t_hbm = 1e8 / (bench.HBM_PEAK_GBS * 1e9)
    assert r["bound"] == ("alu" if t_int >= t_hbm else "hbm")
    assert math.isclose(r["frac"], max(t_int, t_hbm) / 1e-3)
    assert math.isclose(r["hbm_frac"], t_hbm / 1e-3)


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


def test_evalmod_model_counts_the_products_and_the_shared_keystream():
    """EvalMod of degree 2d with r double angles makes d + r ciphertext products (each a tensor, a
    relinearisation and a rescale); items that share the key regenerate its keystream once."""
    cfg = W.CONFIGS["n16-stream64"]
    lvl, r, d = 32, 3, 6
    o1, b1, k1 = bench.evalmod_model(cfg, lvl, r, d, 1)
    o2, b2, k2 = bench.evalmod_model(cfg, lvl, r, d, 2)
    levels = range(lvl - 1, lvl - 1 - (d + r + 1), -1)
    prod_levels = [lvl - 1] + list(range(lvl - 3, lvl - 3 - (d - 1 + r), -1))
    assert len(prod_levels) == d + r and min(levels) >= 0
    assert b1 == b2 == sum(bench.chacha_blocks(cfg, l) for l in prod_levels)
    assert k1 == k2 == sum(bench.key_limbs(cfg, l) for l in prod_levels) * cfg.n * 4
    chacha = b1 * bench.CHACHA_BLOCK
    assert o2 == 2 * o1 - chacha
    assert o1 > sum(bench.keyswitch_ops(cfg, l) for l in prod_levels)
