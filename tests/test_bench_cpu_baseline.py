"""bench.py's CPU baselines (no GPU): the fp64 oracle timed in its unabsorbed and absorbed
forms, over a bounded sample or over every sequence of a workload."""
import importlib.util
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_cpu_mod", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_both_forms_over_every_sequence():
    from mla_inputs import CONFIGS, make_workload
    b = _bench()
    cfg = CONFIGS["tiny"]
    wl = make_workload(cfg)
    for absorbed, kind, form in ((False, "oracle", "unabsorbed"),
                                 (True, "oracle_absorbed", "absorbed")):
        r = b.cpu_oracle_sample(cfg, wl, budget_s=None, absorbed=absorbed)
        assert r["kind"] == kind and r["unit"] == "tokens/s" and r["value"] > 0
        assert r["sample"].startswith(f"{cfg.batch} of {cfg.batch} sequences")
        assert f"fp64 {form} form" in r["sample"]
        assert r["cores"] >= 1


def test_bounded_sample_stops_at_max_seqs():
    from mla_inputs import CONFIGS, make_workload
    b = _bench()
    cfg = CONFIGS["qwen25_7b"].with_(batch=3, context=256)
    wl = make_workload(cfg)
    r = b.cpu_oracle_sample(cfg, wl, budget_s=60.0, max_seqs=2, absorbed=True)
    assert r["sample"].startswith("2 of 3 sequences")
