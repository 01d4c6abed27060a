"""Host-side helpers of bench.py on a machine without a GPU: the clock summary keeps only
the samples inside the timed region and reports throttle reasons; the workload line names
the pack and its valid FLOPs; the oracle sample rate is a bounded CPU measurement."""
import importlib.util
import os

import pytest

import workloads

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


class _DoneProcess:
    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0

    def kill(self):
        pass


def _row(ts, sm, power, active=("Not Active",) * 4):
    # [timestamp, index, clocks.sm, clocks.max.sm, power.draw, reasons.active, hw, hw_thermal, sw_thermal, sw_power]
    return [ts, "0", str(sm), "1965", str(power), "0x0"] + list(active)


def test_clock_summary_keeps_the_timed_region(bench):
    cs = bench.ClockSampler(0)
    cs.proc = _DoneProcess()
    cs.rows = [_row(0.5, 1965, 100.0),                       # before the region: idle boost
               _row(1.0, 1740, 900.0), _row(1.5, 1750, 950.0),
               _row(2.0, 1760, 960.0, ("Not Active", "Not Active", "Not Active", "Active")),
               _row(3.5, 1965, 120.0)]                       # after the region
    rec = cs.stop(1.0, 2.0)
    assert rec["sm_mhz"] == 1750.0 and rec["sm_max_mhz"] == 1965.0
    assert rec["samples"] == 3 and rec["reasons"] == ["sw_power_cap"]
    assert rec["power_w_median"] == 950.0
    assert rec["window"] == "samples taken inside the timed region"


def test_clock_summary_short_region_takes_the_nearest_sample(bench):
    cs = bench.ClockSampler(0)
    cs.proc = _DoneProcess()
    cs.rows = [_row(10.0, 1700, 800.0), _row(10.5, 1800, 800.0)]
    rec = cs.stop(10.45, 10.46)
    assert rec["sm_mhz"] == 1800.0 and rec["samples"] == 0
    assert rec["window"].startswith("timed region shorter")
    assert bench.ClockSampler(0).stop(0.0, 1.0) is None       # never started: no record


def test_workload_line(bench):
    cfg = workloads.load_config("mixed")
    desc = bench.workload_desc(cfg)
    assert desc["segments"] == [1024, 4096, 1296] and desc["total_tokens"] == 6416
    assert desc["valid_flops_per_step"] == workloads.valid_flops([1024, 4096, 1296], 24, 128)
    assert desc["workload"].startswith("mixed pack")


def test_oracle_sample_rate_is_bounded(bench):
    cfg = workloads.load_config("tiny")
    p = workloads.make_inputs(cfg)
    rate, rows, secs, threads = bench.oracle_sample_rate(p, cfg, 0.2)
    assert rate > 0 and rows > 0 and threads >= 1 and secs < 30


def test_unique_bytes_of_a_call(bench):
    # q, k, v read and out written in bf16 (4 tensors x 2 bytes), lse written in fp32
    assert bench.unique_bytes(10, 3, 128) == 4.0 * 10 * 3 * 128 * 2 + 4.0 * 10 * 3
    cfg = workloads.load_config("thumbnails")
    T = sum(cfg["segments"])
    assert bench.unique_bytes(T, 24, 128) == pytest.approx(2.408e9, rel=1e-3)


def test_short_segment_packs_follow_their_recipe():
    """The frozen small-image packs are what their documented draw produces (sides multiples of
    16, aspect at most 2, tokens (h/16)(w/16)); every thumbnail fits one 128-row tile."""
    from workloads import freeze_configs as fc
    for name, seed, n, max_patches in (("many_short", 5, 300, 18), ("thumbnails", 6, 2048, 11)):
        cfg = workloads.load_config(name)
        imgs = fc.draw_small_images(seed, n, max_patches)
        assert cfg["images"] == imgs
        assert cfg["segments"] == [workloads.tokens_for_image(h, w) for h, w in imgs]
        assert all(max(h, w) <= 2 * min(h, w) for h, w in imgs)
    assert max(workloads.load_config("thumbnails")["segments"]) <= 128
