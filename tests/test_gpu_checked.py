"""The checked build (libonetrans_checked.so, device bounds checks on the
kernels' plain row-mapped loads and stores against the extents of the
caller's buffers): on correct calls it computes what the release build
computes, bit for bit, and reports no error; with every extent halved (its
OT_CHECK_SHRINK=1 test hook) the checks fire and the calls report
OT_ERR_DEVICE_BOUNDS instead of making the accesses.  Each variant runs in
a child process (a process loads one library)."""

from __future__ import annotations

import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
OT_ERR_DEVICE_BOUNDS = 9


@pytest.fixture(scope="module", autouse=True)
def _build():
    from unified_transformer_recommender_onetrans_b200.build import build
    build()
    build(checked=True)


def _child(tmp_path, name, **env):
    path = str(tmp_path / f"{name}.pt")
    e = dict(os.environ, **env)
    r = subprocess.run([sys.executable, os.path.join(HERE, "checked_child.py"), path], env=e,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    return torch.load(path)


def test_checked_build_matches_release_and_reports_no_error(tmp_path):
    ref = _child(tmp_path, "release", OT_CHECKED="0")
    chk = _child(tmp_path, "checked", OT_CHECKED="1")
    assert ref["status"] == {"bf16": 0, "f32": 0}
    assert chk["status"] == {"bf16": 0, "f32": 0}
    for k, v in ref["out"].items():
        assert torch.equal(v, chk["out"][k]), k


def test_checked_build_reports_out_of_extent_accesses(tmp_path):
    bad = _child(tmp_path, "shrunk", OT_CHECKED="1", OT_CHECK_SHRINK="1")
    assert bad["status"] == {"bf16": OT_ERR_DEVICE_BOUNDS, "f32": OT_ERR_DEVICE_BOUNDS}
