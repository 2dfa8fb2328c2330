"""CPU tests of bench.py's reporting arithmetic: the algorithmic bytes and flops it divides by
(counted here by brute force over small batches), the error-to-bar ratios it reports beside the
parity tests' bars, the traffic record lookup and the summary strings."""
import numpy as np
import pytest

import bench


def test_conv_work_counts_valid_frames_and_all_outputs():
    B, T, C, K = 3, 10, 8, 3
    lengths = np.array([4, 12, -2])  # clamped into [0, T]
    valid = sum(1 for b in range(B) for t in range(T) if t < min(max(lengths[b], 0), T))
    params = K * C * 4 + C * 4 + B * 4
    work, v = bench.conv_work(lengths, T, C, K)
    assert v == valid == 14
    assert work["fwd"] == (valid * C * 2 + B * T * C * 2 + params, 2 * K * valid * C)
    assert work["dx"][0] == valid * C * 2 + B * T * C * 2 + K * C * 4 + B * 4
    assert work["dw"] == (2 * valid * C * 2 + (K + 1) * C * 4 + B * 4, 2 * K * valid * C + valid * C)


def test_sub_work_counts_valid_mel_h_and_output_pixels():
    B, T, F, C = 2, 13, 9, 4
    lengths = np.array([7, 13])
    s2 = lambda n: (n - 1) // 2 + 1
    T2, F2, T4, F4 = s2(T), s2(F), s2(s2(T)), s2(s2(F))
    mel_valid = sum(1 for b in range(B) for t in range(T) for f in range(F) if t < lengths[b])
    h_valid = sum(1 for b in range(B) for r in range(T2) for c in range(F2) if r < (lengths[b] + 1) // 2)
    o_valid = sum(1 for b in range(B) for i in range(T4) for j in range(F4) if i < ((lengths[b] + 1) // 2 + 1) // 2)
    by, fl, t4, f4 = bench.sub_work(lengths, T, F, C)
    assert (t4, f4) == (T4, F4) == (4, 3)
    assert by == mel_valid * 4 + B * T4 * F4 * C * 2 + 2 * (9 * C * 4 + C * 4) + B * 8
    assert fl == (h_valid + o_valid) * C * 18


def test_bf16_err_over_bar_uses_the_larger_of_2e2_and_one_ulp():
    ref = np.array([0.5, 3.0, 10.0, -12.0])
    assert bench.bf16_err_over_bar(ref, ref) == 0.0
    # |y| < 4: bf16 spacing is below 2e-2, so the bar is 2e-2
    assert bench.bf16_err_over_bar(ref + [0.01, 0.0, 0.0, 0.0], ref) == pytest.approx(0.5)
    assert bench.bf16_err_over_bar(ref + [0.0, 0.02, 0.0, 0.0], ref) == pytest.approx(1.0)
    # [8, 16): one bf16 ulp is 2**-4
    assert bench.bf16_err_over_bar(ref + [0.0, 0.0, 2.0 ** -4, 0.0], ref) == pytest.approx(1.0)
    assert bench.bf16_err_over_bar(ref + [0.0, 0.0, 0.0, 2.0 ** -5], ref) == pytest.approx(0.5)


def test_dw_err_over_bar_takes_the_smaller_bar():
    ref = np.full(16, 100.0)  # RMS 100: 1e-5 * RMS = 1e-3 < 2e-2
    assert bench.dw_err_over_bar(ref + 5e-4, ref) == pytest.approx(0.5)
    small = np.full(16, 1.0e4)  # 1e-5 * RMS = 0.1 > 2e-2: the absolute bar binds
    assert bench.dw_err_over_bar(small + 1e-2, small) == pytest.approx(0.5)


def test_ncu_traffic_requires_the_current_kernel_sources(tmp_path, monkeypatch):
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_sha", lambda: "abc")
    (tmp_path / "profiles" / "traffic.txt").write_text(
        "# header\n"
        "kernel=k1 sha=abc dram_read=100 sm_write=50 l2_write_all=75 l2_write_fabric=25 dram_write=0 launches=1\n"
        "kernel=k2 sha=old dram_read=7 sm_write=1 l2_write_all=1 l2_write_fabric=0 dram_write=0 launches=1\n")
    assert bench.ncu_traffic("k1") == (150.0, 100.0, 50.0)
    assert bench.ncu_traffic("k2") is None  # captured on other kernel sources
    assert bench.ncu_traffic("k3") is None


def test_summary_table_strings():
    row = {"us": 11.54, "hbm_frac_of_measured": 0.596, "err_over_bar": 0.5}
    line = {"rows": {"dwconv1d_fwd": row},
            "configs": {"causal_kernel_width_sweep": {"C1024_K3": {"us": 15.9, "roofline_frac": 0.83}},
                        "subsampler": {"sym_fp32_simt": {"us": 133.3, "fp32_frac": 0.41}}}}
    s = bench.summary_table(line)
    assert s["cfg2_fwd"] == "11.5us hbm 0.60 err/bar 0.50"
    assert s["cfg3_C1024_K3"] == "15.9us roofline 0.83"
    assert s["cfg4_sym_fp32_simt"] == "133.3us fp32 0.41"
