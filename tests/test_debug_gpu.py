"""The index-checking debug build (-DATTN_DEBUG, libattn_sm100_debug.so) on a
B200: every entry point runs a battery of small calls (all head dims, masks,
the pair split, window, key splits with workspace and static scratch, FP8
casts, quantizers and attention, the prologue, the streaming cache, the
host-buffer path). No index check may fail, no wait may run out, and every
output must equal the release build's bit for bit (the checks only guard
accesses; they change no arithmetic). Each build runs in a process of its own
(the binding loads one library per process)."""

from __future__ import annotations

import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
BATTERY = os.path.join(ROOT, "tests", "debug_battery.py")
DEBUG_SO = os.path.join(ROOT, "head_attention_streaming_b200", "libattn_sm100_debug.so")


def _run(debug: bool):
    env = dict(os.environ, PYTHONPATH=ROOT + os.pathsep + os.environ.get("PYTHONPATH", ""))
    env["HASB_DEBUG"] = "1" if debug else "0"
    r = subprocess.run([sys.executable, BATTERY], capture_output=True, text=True, env=env, timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    return json.loads(r.stdout.strip().splitlines()[-1])


def test_debug_library_is_built_and_exports_the_entry_points():
    import ctypes
    assert os.path.exists(DEBUG_SO), "build it with python -m head_attention_streaming_b200.build --debug"
    L = ctypes.CDLL(DEBUG_SO)
    from test_boundary import _declared_functions
    for name in _declared_functions():
        assert hasattr(L, name), name


@pytest.mark.gpu
def test_debug_build_checks_pass_and_outputs_match_release(cuda_ok):
    dbg = _run(True)
    rel = _run(False)
    assert dbg["debug"] is True and rel["debug"] is False
    assert [c["name"] for c in dbg["cases"]] == [c["name"] for c in rel["cases"]]
    for d, r in zip(dbg["cases"], rel["cases"]):
        assert d["site"] == 0 and d["fault"] == 0, d
        assert r["site"] == 0 and r["fault"] == 0, r
        assert d["digest"] == r["digest"], (d["name"], d["digest"], r["digest"])
