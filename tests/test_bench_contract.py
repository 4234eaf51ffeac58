"""The benchmark's JSON contract, checked on CPU through its reference arm (the fp64 oracle on
the host cores) and its multi-rank helpers."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def reference_line():
    env = dict(os.environ, OMP_NUM_THREADS=os.environ.get("OMP_NUM_THREADS", "4"))
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1",
                          "--warmup", "0"], cwd=ROOT, env=env, capture_output=True, text=True,
                         timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, out.stdout
    return json.loads(lines[0])


def test_reference_line_has_the_contract_keys(reference_line):
    d = reference_line
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference"
    assert d["unit"] == "tokens/s" and d["higher_is_better"] is True
    assert d["value"] > 0 and d["cpu_baseline"]["value"] == d["value"]
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
    assert d["config"]["workload"] == "hybrid_bf16_F21_P1560"
    # the same config keys as the GPU arm prints
    sys.path.insert(0, ROOT)
    import bench
    from hybrid_linear_temporal_kta_b200 import synth
    assert d["config"] == bench.hybrid_config(synth.HYBRID_BF16, 1)
    # ms per step is the measured time of one sample; the whole-layer time at the sampled rate
    # is reported apart, as an extrapolation
    assert 0 < d["ms_per_step"] < 60e3
    assert d["full_layer_ms_extrapolated"] == pytest.approx(32760 / d["value"] * 1e3, rel=1e-6)


def test_workload_algebra_matches_the_layer():
    sys.path.insert(0, ROOT)
    import bench
    from hybrid_linear_temporal_kta_b200 import synth
    w = synth.HYBRID_BF16
    # SWA (W = 3): frames 0, 1 see 1, 2 frames, the other 19 see 3 -> 60 frame pairs;
    # DSWA (W = 4, dil = 3): frames 0-2 see 1, 3-5 see 2, 6-8 see 3, 9-20 see 4 -> 66;
    # 8 heads each, P^2 = 1560^2 token pairs per frame pair
    assert bench.visible_pairs(w) == 1560 ** 2 * (8 * 60 + 8 * 66) == 2_453_068_800
    assert bench.softmax_flops(w) == 4 * 128 * 2_453_068_800
    assert bench.gla_bytes(w) == 12 * 128 * 32760 * 8
    d = synth.DELTA_BF16
    assert bench.delta_bytes(d) == pytest.approx(2.164e9, rel=1e-3)


def test_projection_and_backward_algebra():
    sys.path.insert(0, ROOT)
    import bench
    from hybrid_linear_temporal_kta_b200 import synth
    w = synth.HYBRID_BF16
    # stacked q/k/v/alpha projection: 32,760 rows x 3,072 inputs x (3 x 3,072 + 8 x 128 = 10,240)
    # outputs, plus the 3,072 x 3,072 output projection; 2 FLOP per multiply-add
    assert bench.layer_proj_flops(w) == 2 * 32760 * 3072 * 10240 + 2 * 32760 * 3072 * 3072
    assert bench.layer_proj_flops(w) == 2_679_405_281_280
    # fp32 backward: S, dP, dQ (6d) in the query-major kernel, S, dP, dV, dK (8d) key-major
    fl = bench.softmax_bwd_flops(w)
    assert fl["softmax_bwd_q_f32"] == 6 * 128 * 2_453_068_800
    assert fl["softmax_bwd_kv_f32"] == 8 * 128 * 2_453_068_800
    # fp32 FMA peak at 1965 MHz: 148 SMs x 128 lanes x 2 FLOP
    assert bench.fp32_alu_tflops(1965.0) == pytest.approx(74.44992)
