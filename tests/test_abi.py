"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every entry point include/gam.h declares, plans lengths like the oracle, and
rejects bad arguments before touching a device."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
from conformer_speech_recognition_b200 import gam, synth
from conftest import ROOT


def _header_functions():
    text = open(os.path.join(ROOT, "include", "gam.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gam_[a-z_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def L():
    from conformer_speech_recognition_b200 import build
    build.build()
    return gam.lib()


def test_library_exports_every_declared_symbol(L):
    declared = _header_functions()
    assert len(declared) >= 15
    for name in declared:
        assert hasattr(L, name), name
    assert set(declared) == set(gam.EXPORTS)


def test_status_strings(L):
    for k, v in gam.STATUS.items():
        assert gam.gam_status_string(k) == v


def test_plan_lengths_matches_oracle(L):
    cfg = synth.workload_config("c2_varlen_b32_d768")
    lens = synth.clip_lengths("c2_varlen_b32_d768")
    fr, el, fmax, tmax = gam.gam_plan_lengths(cfg, lens)
    for n, f, l in zip(lens, fr, el):
        p = oracle.clip_lengths_plan(int(n), cfg)
        assert (f, l) == (p["F"], p["L2"])
    assert fmax == max(oracle.clip_lengths_plan(int(n), cfg)["F"] for n in lens)
    assert tmax == max(oracle.clip_lengths_plan(int(n), cfg)["T2"] for n in lens)
    fr, el, fmax, tmax = gam.gam_plan_lengths(cfg, [16000, 320000])
    assert list(fr) == [99, 1999] and list(el) == [24, 499] and tmax == 500


def test_plan_rejects_empty_batch(L):
    cfg = synth.workload_config("c1_1s_b1_d768")
    with pytest.raises(gam.GamError) as e:
        gam.gam_plan_lengths(cfg, [])
    assert e.value.name == "GAM_ERR_INVALID_ARG"


def test_plan_rejects_short_clip(L):
    cfg = synth.workload_config("c1_1s_b1_d768")
    with pytest.raises(gam.GamError) as e:
        gam.gam_plan_lengths(cfg, [16000, 1279])
    assert e.value.name == "GAM_ERR_SHAPE" and "1280" in str(e.value)
    gam.gam_plan_lengths(cfg, [1280])


@pytest.mark.parametrize("field,value", [("d_model", 700), ("n_heads", 5), ("conv_kernel", 4), ("n_fft", 512),
                                         ("n_classes", 1), ("precision", 7)])
def test_create_rejects_bad_config(L, field, value):
    cfg = dict(synth.workload_config("c1_1s_b1_d768"))
    cfg[field] = value
    with pytest.raises(gam.GamError) as e:
        gam.gam_create(cfg, {"x": np.zeros(1, np.float32)}, 1, 16000)
    assert e.value.name == "GAM_ERR_INVALID_ARG"


def test_create_without_gpu_reports_device(L):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    cfg = synth.workload_config("c1_1s_b1_d768")
    with pytest.raises(gam.GamError) as e:
        gam.gam_create(cfg, {"x": np.zeros(1, np.float32)}, 1, 16000)
    assert e.value.name == "GAM_ERR_UNSUPPORTED_DEVICE"
