"""CPU checks of the boundary: the library builds for sm_100a, loads without a GPU, and
exports exactly the entry points include/rtvla.h declares; the binding fails loudly when
the library is absent."""
import os
import re
import subprocess

import pytest

import flow_matching_action_expert_b200 as R
from flow_matching_action_expert_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared():
    names = set()
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", f)).read()
            names |= set(re.findall(r"^[A-Za-z_][\w \*]*?\b(rtvla_\w+)\s*\(", txt, re.M))
    return names


def test_library_builds_and_exports_every_declared_symbol():
    lib = B.build()
    nm = subprocess.run(["nm", "-D", "--defined-only", lib], capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r" T (rtvla_\w+)$", nm, re.M))
    decl = declared()
    assert decl, "no declarations found"
    assert decl <= exported, decl - exported
    assert decl == set(R.EXPORTS)
    R.library()


def test_status_strings_and_kv_bytes_without_gpu():
    B.build()
    assert R.rtvla_status_string(0) == "ok"
    assert "device wait" in R.rtvla_status_string(6)
    cfg = R.make_config(n_layers=18, chunk=63, max_prefix=512)
    assert R.rtvla_kv_bytes(cfg, 1, 512) == 2 * 18 * 512 * 256 * 2
    assert R.rtvla_kv_bytes(cfg, 0, 512) == 0


def test_host_side_argument_errors_without_gpu():
    B.build()
    cfg = R.make_config()
    with pytest.raises(R.RtvlaError) as e:
        R.rtvla_create({}, cfg)          # missing weights -> INVALID_ARG before any CUDA call
    assert e.value.name == "RTVLA_ERR_INVALID_ARG"


def test_vision_host_side_argument_errors_without_gpu():
    B.build()
    lib = R.library()
    with pytest.raises(R.RtvlaError) as e:
        R.rtvla_vision_create({}, R.make_vision_config(n_layers=27))   # no weights
    assert e.value.name == "RTVLA_ERR_INVALID_ARG"
    cfg = R.make_vision_config(n_layers=2)
    cfg.width = 1024
    with pytest.raises(R.RtvlaError) as e:
        R.rtvla_vision_create({}, cfg)                                 # a shape not built
    assert e.value.name == "RTVLA_ERR_UNSUPPORTED"
    cfg = R.make_vision_config(n_layers=2, max_images=0)
    with pytest.raises(R.RtvlaError) as e:
        R.rtvla_vision_create({}, cfg)
    assert e.value.name == "RTVLA_ERR_INVALID_ARG"
    assert R.STATUS[lib.rtvla_encode_images(None, None, 1, 1, None, 256, None)] == "RTVLA_ERR_INVALID_ARG"
    assert R.STATUS[lib.rtvla_vision_sync_status(None, None)] == "RTVLA_ERR_INVALID_ARG"
    assert lib.rtvla_vision_kernels_per_call(None, 1) == -1
    R.rtvla_vision_destroy(0)


def test_binding_fails_loudly_without_the_library(monkeypatch, tmp_path):
    monkeypatch.setattr(R, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(R, "_LIB", None)
    with pytest.raises(RuntimeError, match="not built"):
        R.library()


def test_sources_use_only_sm100a_and_no_closed_calls():
    csrc = os.path.join(ROOT, "flow_matching_action_expert_b200", "csrc")
    txt = "".join(open(os.path.join(csrc, f)).read() for f in os.listdir(csrc))
    assert "multicast::cluster" not in txt.replace("commit.cta_group::1.mbarrier::arrive::one.shared::cluster", "")
    assert "MemcpyBatch" not in txt and "Memcpy3DBatch" not in txt
    assert "arch=compute_100a,code=sm_100a" in " ".join(B.ARCH)
