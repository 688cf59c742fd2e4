"""Host logic of bench.py's clock record: only samples inside the timed region count, and the
clock-event reason bits decode to the names the JSON line reports (no GPU, no NVML)."""
import importlib.util
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _sampler(rows, t0, t1):
    b = _bench()
    s = b.ClockSampler("0")
    s.kind = "nvml"              # as if the NVML sampler had run
    s.rows = rows
    s.t0, s.t1 = t0, t1
    return s


def test_window_and_reasons():
    rows = [
        (0.0, 1965, 1965, 250.0, 0x0),     # before the timed region: ignored
        (1.0, 1900, 1965, 990.0, 0x4),     # sw_power_cap
        (1.1, 1880, 1965, 995.0, 0x4),
        (1.2, 1920, 1965, 985.0, 0x0),
        (3.0, 1965, 1965, 240.0, 0x40),    # after: ignored (hw_thermal_slowdown not reported)
    ]
    s = _sampler(rows, 0.5, 2.0).summary()
    assert s["samples"] == 3
    assert s["sm_mhz"] == 1900
    assert s["sm_max_mhz"] == 1965
    assert s["power_w"] == 990.0
    assert s["reasons"] == ["sw_power_cap"]


def test_all_reason_bits():
    rows = [(1.0, 1000, 1965, 500.0, 0x8 | 0x20 | 0x40 | 0x4)]
    s = _sampler(rows, 0.0, 2.0).summary()
    assert s["reasons"] == sorted(["hw_slowdown", "sw_thermal_slowdown", "hw_thermal_slowdown",
                                   "sw_power_cap"])


def test_no_samples_in_window():
    s = _sampler([(0.0, 1965, 1965, 250.0, 0)], 1.0, 2.0).summary()
    assert s["reasons"] == ["unsampled"]


def test_sample_file_location(tmp_path, monkeypatch):
    """MLA_BENCH_CLOCKS_CSV names the sample file (rank appended); without it the samples go
    to a temporary file that summary() removes."""
    b = _bench()
    monkeypatch.setenv("MLA_BENCH_CLOCKS_CSV", str(tmp_path / "clk.csv"))
    monkeypatch.setenv("RANK", "3")
    s = b.ClockSampler("0")
    s.__enter__()
    assert s.path == str(tmp_path / "clk_rank3.csv") and not s.tmp
    s._stop()
    monkeypatch.delenv("MLA_BENCH_CLOCKS_CSV")
    s = b.ClockSampler("0")
    s.__enter__()
    assert s.tmp and s.path is not None
    s._stop()
    open(s.path, "a").close()            # as if the sampler had written it
    s.kind, s.rows = "nvml", []
    s.summary()
    assert not os.path.exists(s.path)


def test_traffic_is_keyed_to_the_kernel_source(tmp_path, monkeypatch):
    """roofline.traffic comes from the committed record only while its source hash matches
    the decode kernel's current sources; otherwise it is null."""
    import json
    b = _bench()
    from mla_inputs import CONFIGS
    cfg = CONFIGS["deepseek_v2"]
    prof = tmp_path / "profiles"
    prof.mkdir()
    monkeypatch.setattr(b, "ROOT", str(tmp_path))
    csrc = tmp_path / "head_latent_attention_attn_b200" / "csrc"
    csrc.mkdir(parents=True)
    for f in ("decode_pair.cu", "decode.cu", "decode_sched.cuh", "ptx.cuh"):
        (csrc / f).write_text(f"// {f}\n")
    hdr = "struct WGemmParams {\n  int a;\n};\nstruct DecodeParams {\n  int b;\n};\n"
    (csrc / "kernels.h").write_text(hdr)
    h = b._source_hash(cfg)
    (prof / "decode_traffic.json").write_text(json.dumps(
        {"deepseek_v2": {"source_hash": h, "dram_bytes_per_launch": 123}}))
    assert b._traffic(cfg) == 123
    # another kernel's parameters change: the record still holds
    (csrc / "kernels.h").write_text(hdr.replace("int a;", "int a, c;"))
    assert b._traffic(cfg) == 123
    # the decode kernel's parameters or source change: it does not
    (csrc / "kernels.h").write_text(hdr.replace("int b;", "int b, d;"))
    assert b._traffic(cfg) is None
    (csrc / "kernels.h").write_text(hdr)
    assert b._traffic(cfg) == 123
    (csrc / "decode_pair.cu").write_text("// changed\n")
    assert b._traffic(cfg) is None
