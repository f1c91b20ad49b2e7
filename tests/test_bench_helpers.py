"""Host-side helpers of bench.py (no GPU): the roofline's DRAM traffic per
launch, taken from the committed ncu capture and rescaled by context."""

import importlib.util
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_module", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_traffic_at_capture_context_is_the_capture():
    b = _bench()
    for k, v in b.NCU_TRAFFIC.items():
        assert b.roofline_traffic(k, b.NCU_KEYS) == v


def test_qkv_traffic_grows_with_the_cached_keys():
    b = _bench()
    # one more cached key adds its key and value rows of every kv head (fp16)
    step = b.roofline_traffic("qkv", b.NCU_KEYS + 1) - b.roofline_traffic("qkv", b.NCU_KEYS)
    assert step == 2 * b.HKV * b.HD * 2
    assert b.roofline_traffic("gate_up", 500) == b.NCU_TRAFFIC["gate_up"]
    assert b.roofline_traffic("decode_fused", 192) is None
