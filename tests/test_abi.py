"""The C-ABI library loads on a machine without a GPU, exports every symbol
declared in include/h2o.h, and validates configurations on the host."""
import ctypes
import os
import re

import pytest

from kv_cache_sparse_b200 import binding
from kv_cache_sparse_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build()
    return binding.load_library()


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "h2o.h")).read()
    return sorted(set(re.findall(r"^H2O_API\s+[\w\s\*]+?\b(h2o_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_expected_entry_points():
    names = declared_symbols()
    for n in ("h2o_cache_create", "h2o_chunk_step", "h2o_cache_read"):
        assert n in names
    assert set(binding.EXPORTED) <= set(names)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name


def _cfg(**kw):
    base = dict(batch=1, n_q_heads=32, n_kv_heads=8, head_dim=128, capacity=8192,
                max_chunk=1024, recent_window=256, dtype=binding.H2O_BF16, softmax_scale=0.0)
    base.update(kw)
    return binding.Config(**base)


def _req(lib, cfg):
    sz = binding.Sizes()
    return lib.h2o_required_bytes(ctypes.byref(cfg), ctypes.byref(sz)), sz


def test_required_bytes_qwen_shape(lib):
    st, sz = _req(lib, _cfg())
    assert st == 0
    assert sz.k_bytes == 8 * 8192 * 128 * 2 == sz.v_bytes
    assert sz.scores_bytes == sz.pos_bytes == 8 * 8192 * 4
    assert sz.state_bytes == 16
    # row stats + colsum + plan + staging for q, k, v, out
    assert sz.workspace_bytes >= 32 * 1024 * 4 + 8 * (8192 + 1024) * 4 + 1024 * 8 * 128 * 2 * 2


@pytest.mark.parametrize("kw,expect", [
    (dict(n_q_heads=30), 2), (dict(head_dim=96), 2), (dict(recent_window=9000), 2),
    (dict(recent_window=-1), 2), (dict(capacity=49152, max_chunk=2048), 2),
    (dict(dtype=7), 3), (dict(batch=0), 2), (dict(max_chunk=0), 2),
    (dict(dtype=binding.H2O_F32, head_dim=64, n_q_heads=4, n_kv_heads=2, capacity=256,
          max_chunk=64, recent_window=0), 0),
    (dict(policy=1), 0), (dict(policy=2, sink_tokens=4), 0), (dict(policy=3), 1),
    (dict(policy=-1), 1), (dict(policy=2, sink_tokens=-1), 2),
    (dict(policy=2, sink_tokens=8192 - 255), 2), (dict(policy=2, sink_tokens=8192 - 256), 0),
    (dict(policy=1, sink_tokens=9000), 0),  # the sink count matters only to SLR
])
def test_config_validation(lib, kw, expect):
    st, _ = _req(lib, _cfg(**kw))
    assert st == expect


def test_null_arguments_rejected(lib):
    assert lib.h2o_required_bytes(None, None) == 1
    assert lib.h2o_chunk_step(None, None, None, None, 1, None, None, None) == 1
    assert lib.h2o_cache_check(None, None) == 1
    assert lib.h2o_status_string(6) == b"device wait timed out"


def test_missing_library_fails_loudly(tmp_path):
    """No silent fallback: without the built library the binding raises."""
    with pytest.raises(ImportError, match="is missing"):
        binding.load_library(str(tmp_path / "libh2o.so"))


def test_product_package_does_not_import_the_oracle():
    """The oracle is test infrastructure: importing the package and its
    binding, workloads and build modules loads nothing from oracle/."""
    import subprocess
    import sys
    code = ("import sys, kv_cache_sparse_b200, kv_cache_sparse_b200.binding, "
            "kv_cache_sparse_b200.workloads, kv_cache_sparse_b200.build; "
            "bad = [m for m in sys.modules if m == 'oracle' or m.startswith('oracle.')]; "
            "sys.exit(1 if bad else 0)")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    for name in os.listdir(os.path.join(ROOT, "kv_cache_sparse_b200")):
        if name.endswith(".py"):
            text = open(os.path.join(ROOT, "kv_cache_sparse_b200", name)).read()
            assert not re.search(r"^\s*(from|import)\s+oracle\b", text, flags=re.M), name
