"""Host logic of bench.py (CPU): the roofline table covers every kernel the library launches,
the traffic record is honoured only for the sources it was captured on, and the flags parse."""
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from pooled_selective_scan_b200 import build as fvbuild  # noqa: E402
from pooled_selective_scan_b200 import ssm  # noqa: E402
from pooled_selective_scan_b200.configs import CONFIGS  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def _lib():
    fvbuild.build()


def _shape(cfg, axis, path="auto", ln=False):
    s = ssm.LayerShape(cfg.B, cfg.h, cfg.w, cfg.E, cfg.N, cfg.R, axis, cfg.dir_flags, cfg.K, path=path, ln=ln)
    return s


@pytest.mark.parametrize("cfg", CONFIGS, ids=lambda c: c.name)
def test_every_launched_kernel_has_a_bound(cfg):
    for axis in cfg.pool_axes:
        names = set()
        for path in (("auto", "staged", "fused") if not cfg.masked else ("auto",)):
            names |= set(ssm.launch_names(_shape(cfg, axis, path)))
        names |= set(ssm.launch_names(_shape(cfg, axis, "auto", ln=True)))
        if not cfg.masked:
            conv = _shape(cfg, axis)
            conv.d_conv = 4
            names |= set(ssm.launch_names(conv))
        names |= set(ssm.backward_launch_names(_shape(cfg, axis)))
        names |= set(ssm.backward_launch_names(_shape(cfg, axis, ln=True)))
        for n in names:
            bound, amount = bench.kernel_work(n, cfg, axis)
            if n == "mask_bucket_kernel":  # integer bucketing: no roofline of its own
                assert bound is None
                continue
            assert bound in ("hbm", "alu", "fma") and amount > 0, n


def test_streaming_kernels_count_their_algorithmic_bytes():
    cfg = CONFIGS[3]
    tok = cfg.B * cfg.h * cfg.w
    assert bench.kernel_work("fused_layer_kernel", cfg, 0) == ("hbm", 12 * cfg.E * tok)
    assert bench.kernel_work("bwd_gate_dense_kernel", cfg, 0) == ("hbm", 20 * cfg.E * tok)
    assert bench.kernel_work("bwd_pool_dense_kernel", cfg, 0) == ("hbm", 8 * cfg.E * tok)
    assert cfg.algorithmic_bytes_per_call() == 12 * cfg.E * tok


def test_traffic_record_is_void_once_a_source_changes(tmp_path, monkeypatch):
    rec = {"kernels": {"w/k": {"kernel_source_hash": "abc", "dram_bytes_per_full_launch": 123.0}}}
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "ncu_traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda kernel=None: "abc")
    assert bench.recorded_traffic("k", "w") == 123.0
    assert bench.recorded_traffic("other", "w") is None
    monkeypatch.setattr(bench, "kernel_source_hash", lambda kernel=None: "def")
    assert bench.recorded_traffic("k", "w") is None


def test_committed_traffic_records_name_known_kernels():
    with open(os.path.join(ROOT, "profiles", "ncu_traffic.json")) as f:
        j = json.load(f)
    for key, ent in j["kernels"].items():
        cfg_name, kernel = key.split("/")
        assert kernel in bench.KERNEL_SOURCES, kernel
        # a streaming kernel moves at least its algorithmic bytes, less the writes still in L2 at its end
        assert ent["dram_bytes_per_full_launch"] >= 0.85 * ent["algorithmic_bytes_per_full_launch"]
        assert len(ent["kernel_source_hash"]) == 16


def test_flags():
    a = bench.parse(["--grad", "--steps", "2", "--warmup", "3"])
    assert a.grad and a.steps == 2 and a.impl == "ours"
    with pytest.raises(SystemExit):
        bench.parse(["--warmup", "2"])
    with pytest.raises(SystemExit):
        bench.parse(["--steps", "0"])


def test_secondary_workloads_cover_every_config_and_axis():
    """The default run times every workload of the efficiency study: the headline and, under
    'configs', each other config on each of its pool axes."""
    from pooled_selective_scan_b200.configs import by_name
    want = {(c.name, ax) for c in CONFIGS for ax in c.pool_axes} - {(bench.HEADLINE_NAME, 0)}
    assert set(bench.SECONDARY) == want
    assert (bench.HEADLINE_NAME, 0, 4, "auto") in bench.SECONDARY_VARIANTS
    for name, axis, taps, path in bench.SECONDARY_VARIANTS:
        assert axis in by_name(name).pool_axes and path in ("auto", "staged", "fused")
    for name, axis in bench.SECONDARY:
        assert axis in by_name(name).pool_axes
    assert bench.parse(["--no-configs"]).no_configs
    assert not bench.parse([]).no_configs
