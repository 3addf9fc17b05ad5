"""Host logic that needs no GPU: the benchmark's clock summary and its
traffic key, and the argument checks the Python layer makes before any
library call."""
import importlib.util
import os

import numpy as np
import pytest

import bit_attention_transformers_b200 as fa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_clock_summary_parses_samples_and_reasons():
    b = _bench()
    c = b.Clocks(0)
    c.lines = [
        "0, 1965, 1965, 700.1, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "0, 1905, 1965, 990.3, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1965, 1965, 710.0, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "garbage line",
    ]
    s = c.summary()
    assert s == {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"],
                 "samples": 3}
    c.lines = ["0, 1000, 1965, 500, 0x0, Active, Not Active, Active, Not Active"]
    assert c.summary()["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]
    c.lines = []
    assert c.summary() is None


def test_clock_sampler_stops_once():
    b = _bench()
    c = b.Clocks(0)
    c.proc = None
    c.__exit__(None, None, None)
    c.__exit__(None, None, None)  # the second call (at exit) does nothing
    assert c.lines == []


def test_traffic_key_ignores_comments_only(tmp_path):
    b = _bench()
    src = "int f(int x) {\n  return x + 1;  // one\n}\n/* block */\n"
    p1, p2, p3 = tmp_path / "a.cuh", tmp_path / "b.cuh", tmp_path / "c.cuh"
    p1.write_text(src)
    p2.write_text("// header\n" + src.replace("// one", "// another comment") + "\n\n")
    p3.write_text(src.replace("x + 1", "x + 2"))
    assert b.code_sha256(str(p1)) == b.code_sha256(str(p2))
    assert b.code_sha256(str(p1)) != b.code_sha256(str(p3))
    # the key in bench.py is the current kernel's
    kernel = os.path.join(ROOT, "bit_attention_transformers_b200", "csrc", "attn_fwd.cuh")
    assert b.code_sha256(kernel) == b.ATTN_TRAFFIC["attn_fwd_code_sha256"]


def test_oracle_flags_per_variant():
    b = _bench()
    import oracle
    assert b.oracle_flags("exp") == 0
    assert b.oracle_flags("efq") == oracle.FLAG_EFQ
    assert b.oracle_flags("fp8pv") == oracle.FLAG_FP8PV
    assert b.oracle_flags("smooth") == oracle.FLAG_SMOOTH_K | oracle.FLAG_SMOOTH_Q


def test_binding_rejects_conflicting_variants():
    with pytest.raises(ValueError):
        fa._attn_fn(True, True, False)


def test_sharded_wrappers_check_shapes_first():
    import torch
    q = torch.zeros(6, 8, 64, dtype=torch.bfloat16)
    k = torch.zeros(4, 8, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):  # 6 query heads for 4 key/value heads
        fa.fp4_attn_fwd_sharded(q, k, k)
    with pytest.raises(ValueError):
        fa.fp4_attn_bwd_sharded(q, k, k, q, q, torch.zeros(6 * 8))
    with pytest.raises(ValueError):  # smoothing with another P generation
        fa.fp4_attn_fwd_sharded(q[:4], k, k, smooth=fa.FP4_SMOOTH_Q, efq=True)
    with pytest.raises(ValueError):  # lse with smoothing
        fa.fp4_attn_fwd_sharded(q[:4], k, k, smooth=fa.FP4_SMOOTH_Q, lse=torch.zeros(32))


def test_units_cover_every_head_once():
    seen = np.zeros(3 * 5, int)
    for r in range(4):
        u0, u1 = fa.shard_units(3, 5, 4, r)
        seen[u0:u1] += 1
    assert (seen == 1).all()
