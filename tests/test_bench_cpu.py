"""bench.py's JSON line, built from fabricated timings on the CPU: every key
the benchmark contract names is present, and the derived fractions follow
from the times (no GPU involved)."""
import argparse
import io
import json
from contextlib import redirect_stdout

import bench


def _fake_result():
    mg = {"mg2_ctx2k": dict(B=8, H=16, T=2048, d=64, groups=2, dv=64, layout="bthd", ms=0.115),
          "sg2_ctx2k": dict(B=8, H=16, T=2048, d=64, groups=2, dv=64, layout="bthd", ms=0.19, summed=True),
          "decode_mg4_b64": dict(B=64, H=16, d=64, groups=4, dv=64, P=1024, ms=0.094)}
    grid = [dict(B=1, T=1024, chunked_ms=0.02, quadratic_ms=0.02)]
    long = dict(B=1, H=16, T=131072, p=16, dv=64, chunked_C64_ms=0.235, chunked_C128_ms=0.234, quadratic_ms=29.0,
                sequential_C64_ms=1.25, decode_b64=dict(B=64, H=16, p=16, dv=64, ms=0.03), sweep=grid,
                recall=dict(B=4, H=16, T=8192, p=32, dv=64, chunked_ms=13.8, quadratic_ms=0.51), mg=mg,
                train=dict(B=8, H=16, T=2048, p=16, dv=64, fwd_ms=0.08, bwd_ms=0.36, step_ms=0.43,
                           chunked={"B1_T131072": dict(B=1, H=16, T=131072, fwd_ms=0.25, bwd_ms=1.6, step_ms=1.85)}))
    return dict(step_ms=0.116, eager_step_ms=0.125, graph=True, path_ms=[0.081, 0.035, 0.0088], e2e_ms=11.0,
                h2d=50356224, d2h=67125248, clocks={"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []},
                timed_s=0.5, long=long, status=0, tokens=8 * 2048, BH=128, T=2048, p=16, dv=64, C=64)


def test_report_line_has_the_contract_keys():
    args = argparse.Namespace(workload="layer340m_ctx2k", steps=1000, warmup=10, cpu_baseline=0)
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.report(args, _fake_result(), 0.116, 11.0, 1)
    line = json.loads(buf.getvalue().strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
                "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches", "clocks"):
        assert key in line, key
    assert line["value"] == 8 * 2048 / 0.116e-3
    rf = line["roofline"]
    assert abs(rf["frac"] - rf["achieved"] / rf["peak"]) < 1e-12
    assert rf["achieved"] == bench.flash_flops(128, 2048, 16, 64) / 0.081e-3 / 1e12
    assert set(line["mg"]) == {"mg2_ctx2k", "sg2_ctx2k", "decode_mg4_b64"}
    assert line["mg"]["sg2_ctx2k"]["workload"].startswith("KATA-Sigma-g")
    assert line["mg"]["sg2_ctx2k"]["tensor_frac"] == bench.flash_flops(128, 2048, 128, 64) / 0.19e-3 / 1e12 / 1617.3
    assert "tensor_frac" in line["mg"]["mg2_ctx2k"] and "hbm_frac" in line["mg"]["decode_mg4_b64"]
    tr = line["train"]
    assert tr["tokens_per_s"] == 8 * 2048 / 0.43e-3 and 0 < tr["bwd_tensor_frac"] < 1


def test_report_line_has_per_path_points():
    """Every path of the metric is reported on its own inside `roofline`:
    tokens/s and the fraction of its binding roofline at T = 2048 and at
    T = 131072 (chunked C = 64 and 128, quadratic), and the B = 64 decode."""
    args = argparse.Namespace(workload="layer340m_ctx2k", steps=1000, warmup=10, cpu_baseline=0)
    res = _fake_result()
    res["clocks_by_part"] = {"step": {"sm_mhz": 1965.0}, "long_ctx": {"sm_mhz": 1950.0}, "decode_b64": {}}
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.report(args, res, 0.116, 11.0, 1)
    pts = json.loads(buf.getvalue().strip().splitlines()[-1])["roofline"]["points"]
    key = {(p["path"], p.get("T"), p.get("C")): p for p in pts}
    c131 = key[("chunked", 131072, 64)]
    assert c131["bound"] == "hbm" and c131["clocks"] == {"sm_mhz": 1950.0}
    assert abs(c131["achieved"] - bench.chunked_bytes(16, 131072, 16, 64) / 0.235e-3 / 1e9) < 1e-6
    assert abs(c131["frac"] - c131["achieved"] / c131["peak"]) < 1e-12
    assert c131["tokens_per_s"] == 131072 / 0.235e-3
    assert ("chunked", 131072, 128) in key and ("quadratic", 131072, None) in key
    assert key[("quadratic", 2048, None)]["bound"] == "tensor" and ("chunked", 2048, 64) in key
    assert any(p["path"] == "decode" for p in pts)


def test_backward_passes_are_reported_against_their_rooflines():
    """The chunked backward's HBM fraction counts q, k, v, o, dO, D read and
    dq, dk, dv written once (8p + 8dv + 4 bytes per token-head); the flash
    backward's tensor fraction counts 2(3p + 2dv) flops per causal pair."""
    args = argparse.Namespace(workload="layer340m_ctx2k", steps=1000, warmup=10, cpu_baseline=0)
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.report(args, _fake_result(), 0.116, 11.0, 1)
    line = json.loads(buf.getvalue().strip().splitlines()[-1])
    assert bench.chunked_bwd_bytes(16, 131072, 16, 64) == 16 * 131072 * 644
    c = line["train"]["chunked"]["B1_T131072"]
    assert abs(c["bwd_hbm_frac"] - 16 * 131072 * 644 / 1.6e-3 / 1e9 / 6551.0) < 1e-12
    pts = {(p["path"], p.get("T")): p for p in line["roofline"]["points"]}
    assert pts[("bwd_chunked", 131072)]["bound"] == "hbm"
    assert abs(pts[("bwd_chunked", 131072)]["frac"] - c["bwd_hbm_frac"]) < 1e-12
    bq = pts[("bwd_quadratic", 2048)]
    assert bq["bound"] == "tensor"
    assert abs(bq["achieved"] - 128 * 2048 * 2049 / 2 * 2 * (3 * 16 + 2 * 64) / 0.36e-3 / 1e12) < 1e-6
