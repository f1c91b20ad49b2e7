"""The C-ABI library loads on a machine without a GPU, exports every entry
point the header declares, and validates arguments on the host (no compute
call is made here)."""

import os
import re

import numpy as np
import pytest

import weight_shared_looped_int4_b200 as tl
from weight_shared_looped_int4_b200 import build as tl_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built_library():
    tl_build.build()
    return tl.load_library()


def _declared_functions():
    names = set()
    inc = os.path.join(ROOT, "include")
    for fn in os.listdir(inc):
        if not fn.endswith(".h"):
            continue
        text = open(os.path.join(inc, fn)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        for m in re.finditer(r"\b(tl_\w+)\s*\(", text):
            names.add(m.group(1))
    return names


def test_header_declares_the_exported_set():
    declared = _declared_functions()
    assert declared == set(tl.EXPORTED)


def test_every_declared_symbol_is_exported():
    lib = tl.load_library()
    for name in _declared_functions():
        assert hasattr(lib, name), name


def test_built_for_sm100a():
    assert "arch=compute_100a,code=sm_100a" in tl_build.NVCC_FLAGS


def test_status_strings():
    names = ["TL_OK", "TL_ERR_INVALID_ARG", "TL_ERR_OOM", "TL_ERR_CUDA", "TL_ERR_CONTEXT_FULL",
             "TL_ERR_LOOPS_MISMATCH", "TL_ERR_NOT_PREFILLED", "TL_ERR_DEVICE_FLAG",
             "TL_ERR_UNSUPPORTED"]
    for i, n in enumerate(names):
        assert tl.tl_status_string(i) == n
        assert getattr(tl, n) == i
    assert tl.tl_version().count(".") == 2


def test_null_arguments_rejected_on_host():
    with pytest.raises(tl.TLError) as e:
        tl.tl_op_rmsnorm(0, 0, 4, 256, 1e-5, 0, stream=0)
    assert e.value.status == tl.TL_ERR_INVALID_ARG
    assert "null" in tl.tl_last_error()
    with pytest.raises(tl.TLError) as e:
        tl.tl_op_gqa_prefill(0, 0, 0, 0, 16, 4, 0, 1, 4, 2, 64, 0, stream=0)
    assert e.value.status == tl.TL_ERR_INVALID_ARG


def test_model_controls_reject_a_null_model_on_host():
    for call in (lambda: tl.tl_model_set_trace(None, None, 0),
                 lambda: tl.tl_model_set_decode_path(None, tl.DECODE_LAYERED),
                 lambda: tl.tl_model_set_graphs(None, True),
                 lambda: tl.tl_model_set_clustered_decode(None, True),
                 lambda: tl.tl_model_set_wait_test(None, 0)):
        with pytest.raises(tl.TLError) as e:
            call()
        assert e.value.status == tl.TL_ERR_INVALID_ARG
    assert tl.tl_model_trace_grid(None) == 0


def test_unsupported_shapes_rejected_on_host():
    x = np.zeros(8, np.uint32)
    lin = type("L", (), {"qweight": x, "scales": x, "qzeros": x})
    with pytest.raises(tl.TLError) as e:
        tl.tl_linear_create(lin, 100, 32, 0)      # K not a multiple of 128
    assert e.value.status == tl.TL_ERR_UNSUPPORTED


def test_model_config_validation_on_host():
    import tl_synth
    sh = tl_synth.TINY_LM
    w = tl_synth.make_model_weights(sh, 1)
    tw, keep = tl.make_weights(w)
    bad = [
        dict(max_lanes=17), dict(max_lanes=0), dict(max_loops=0), dict(max_ctx=9000),
    ]
    for kw in bad:
        args = dict(max_loops=4, max_ctx=64, max_lanes=2)
        args.update(kw)
        cfg = tl.make_config(sh, **args)
        with pytest.raises(tl.TLError) as e:
            tl.tl_model_create(cfg, tw, 0)
        assert e.value.status == tl.TL_ERR_INVALID_ARG, kw
    cfg = tl.make_config(sh, 4, 64, 2)
    cfg.head_dim = 96
    with pytest.raises(tl.TLError) as e:
        tl.tl_model_create(cfg, tw, 0)
    assert e.value.status == tl.TL_ERR_UNSUPPORTED
    del keep


def test_no_device_is_an_error_not_a_crash():
    # Without a GPU the library reports the missing device as an error status.
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    import tl_synth
    w = tl_synth.make_model_weights(tl_synth.TINY_LM, 1)
    tw, keep = tl.make_weights(w)
    with pytest.raises(tl.TLError) as e:
        tl.tl_model_create(tl.make_config(tl_synth.TINY_LM, 4, 64, 2), tw, 0)
    assert e.value.status == tl.TL_ERR_INVALID_ARG
    del keep
