"""The C ABI boundary, checked without a GPU: libkd loads, exports every function that
include/kd.h declares, sizes its arena, refuses bad arguments before touching a device, and
its bytes-per-step formula agrees with the bytes the oracle counts as it reads."""

import ctypes
import os
import re

import pytest

import oracle
import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kd.h")


@pytest.fixture(scope="module")
def kd():
    from persistent_monokernel_sm_b200 import build
    build.build()
    import persistent_monokernel_sm_b200 as kd
    kd.load_library()
    return kd


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(kd_[a-z_0-9]+)\s*\(", text)))


def test_every_declared_function_is_exported(kd):
    names = declared_functions()
    assert len(names) >= 15
    lib = ctypes.CDLL(kd.LIB_PATH)
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing


def test_binding_mirrors_the_abi_names(kd):
    for n in declared_functions():
        assert callable(getattr(kd, n)), n


def test_arena_bytes_for_every_workload(kd):
    for name, w in synth.WORKLOADS.items():
        cfg = kd.config_from(w.dims(), w.capacity)
        n = kd.kd_arena_bytes(cfg)
        # weights + KV cache dominate; the rest (activations, control) is small
        kv = 2 * w.n_layers * w.n_kv_heads * w.capacity * w.head_dim * 2
        assert n >= kv
        assert n % 256 == 0


@pytest.mark.parametrize("bad", [dict(head_dim=96), dict(n_heads=6, n_kv_heads=4), dict(d_model=16384),
                                 dict(ffn_dim=0), dict(n_layers=0), dict(vocab=0), dict(n_heads=18, n_kv_heads=2),
                                 dict(rms_eps=-1.0)])
def test_invalid_configs_are_refused(kd, bad):
    dims = dict(synth.get("tiny").dims())
    dims.update(bad)
    cfg = kd.config_from(dims, 64)
    assert kd.kd_arena_bytes(cfg) == 0
    assert kd.kd_step_bytes(cfg, 10, True) < 0
    h = ctypes.c_void_p()
    rc = kd.load_library().kd_create(ctypes.byref(cfg), ctypes.c_void_p(1 << 20), 1 << 30, None, ctypes.byref(h))
    assert rc == -1 and not h.value


def test_create_refuses_null_arena_without_a_device(kd):
    cfg = kd.config_from(synth.get("tiny").dims(), 64)
    h = ctypes.c_void_p()
    assert kd.load_library().kd_create(ctypes.byref(cfg), None, 1 << 30, None, ctypes.byref(h)) == -1
    assert kd.load_library().kd_create(ctypes.byref(cfg), None, 0, None, None) == -1


def test_calls_on_a_null_handle_are_refused(kd):
    lib = kd.load_library()
    assert lib.kd_decode(None, 1, None, None) == -1
    assert lib.kd_sync(None) == -1
    assert lib.kd_reset(None, None, 1, 0) == -1
    assert lib.kd_position(None) == -1
    assert lib.kd_decode_noalloc(None, None, 1, 0, 1, None, None) == -1
    assert kd.kd_strerror(-6).startswith("device-side wait")
    assert lib.kd_set_timeout(None, 1000) == -1
    assert lib.kd_set_sampling(None, 0.5, 1) == -1


def test_step_bytes_equal_the_bytes_the_oracle_reads(kd, tiny, tiny_weights):
    """Two independent computations: a closed form in libkd, and the oracle counting the
    weight and cache elements it touches while it runs a decode step."""
    cfg = kd.config_from(tiny.dims(), 16)
    o = oracle.Oracle(tiny.dims(), tiny_weights, capacity=16)
    for pos in range(6):
        head = pos % 2 == 0
        _, _, counted = o.step(7, pos, head=head)
        assert kd.kd_step_bytes(cfg, pos + 1, head) == counted


def test_step_bytes_reproduce_the_pages_light_speed_arithmetic(kd):
    """Bandwidth / bytes-per-token is the pages' bound; the 2B-class workload moves about
    4 GB of weights per token and 8x H200 at 30.7 TB/s would then allow ~7,700 tokens/s."""
    import json
    gold = json.load(open(os.path.join(ROOT, "tests", "golden", "bandwidth_arithmetic.json")))
    w = synth.get("2b-4k")
    cfg = kd.config_from(w.dims(), w.capacity)
    weights = kd.kd_step_bytes(cfg, 0, True)
    assert 3.5e9 < weights < 4.2e9
    for row in gold["light_speed"]:
        if "bytes_gb" in row and "tokens_per_s" in row and "aggregate_tb_s" in row:
            bound = row["aggregate_tb_s"] * 1e12 / (row["bytes_gb"] * 1e9)
            assert abs(bound - row["tokens_per_s"]) / row["tokens_per_s"] < 0.02, row
    for row in gold["time_budget"]:
        if "us_per_launch" in row:
            us = row["us_per_launch"] * row["kernels_per_layer"] * row["layers"]
            assert abs(us - row["us_per_token"]) <= 1
            assert abs(1e6 / us - row["tokens_per_s"]) / row["tokens_per_s"] < 0.01
        elif "share" in row:
            assert abs(row["layers"] * row["us_per_layer"] / 333.0 - row["share"]) < 0.001
        else:
            assert abs(1e6 / row["tokens_per_s"] - row["us_per_token"]) < 1


def test_package_never_imports_the_oracle():
    pkg = os.path.join(ROOT, "persistent_monokernel_sm_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".h", ".cuh", ".cpp")):
                text = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in text and "oracle.h" not in text and "liboracle" not in text, f


def test_missing_library_fails_loudly(tmp_path):
    import persistent_monokernel_sm_b200 as kd
    saved = kd._lib
    try:
        kd._lib = None
        with pytest.raises(ImportError):
            kd.load_library(str(tmp_path / "nope.so"))
    finally:
        kd._lib = saved
