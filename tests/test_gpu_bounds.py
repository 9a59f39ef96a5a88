"""The debug build (device-side index checks, OSP_ERR_BOUNDS): on valid inputs every kernel family
produces the release build's bits and records no error; with the checks' limits shrunk
(OSP_DEBUG_BOUNDS_DIV=2, no access ever leaves its buffer because a failed check skips it) every
family reports OSP_ERR_BOUNDS through osp_check_status.  Runs the debug library in child
processes (a process loads one build)."""

import os
import subprocess
import sys

import pytest
import torch

from spacetime_attention_b200 import build as B
from tests import bounds_cases
from tests.gpu_common import gpu  # noqa: F401

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _child(tmp_path, *extra, env_extra=None):
    env = dict(os.environ, OSP_LIBRARY="debug", **(env_extra or {}))
    out = str(tmp_path / "out.pt")
    r = subprocess.run([sys.executable, "-m", "tests.bounds_cases", out, *extra], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    return torch.load(out)


def test_debug_build_matches_release_bits(gpu, tmp_path):
    B.build(debug_bounds=True)
    debug = _child(tmp_path)
    release = {}
    for name, fn in bounds_cases.calls(gpu).items():
        r = fn()
        rs = r if isinstance(r, tuple) else (r,)
        release[name] = [t.cpu() for t in rs if t is not None]
    assert sorted(debug) == sorted(release)
    for name in release:
        for a, b in zip(debug[name], release[name]):
            assert torch.equal(a, b), name


def test_debug_checks_report_bounds(gpu, tmp_path):
    B.build(debug_bounds=True)
    _child(tmp_path, "expect_bounds", env_extra={"OSP_DEBUG_BOUNDS_DIV": "2"})
