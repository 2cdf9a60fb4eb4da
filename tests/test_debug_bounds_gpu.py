"""The debug build (libgdn_tail_replay_debug.so, -DGDN_DEBUG_BOUNDS), on the GPU.

Its kernels compare every global row, head, column and state index they
compute with the extents the plan validated, and report GDN_ERR_BOUNDS
(skipping the access) instead of reading or writing out of range.

* The reporting path works: one check on an index past a stated extent is
  reported through the workspace status (the access is skipped; nothing
  faults).
* The varlen and edge-case parity tests run clean on the debug build: every
  status is GDN_OK and the results still match the oracle.  They run in a
  child process, since a process loads one of the two libraries.
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)


def _child(args, timeout=900):
    env = dict(os.environ, GDN_DEBUG_BOUNDS="1")
    return subprocess.run([sys.executable, *args], cwd=ROOT, env=env, capture_output=True, text=True,
                          timeout=timeout)


def test_debug_build_reports_a_failing_index_check():
    code = (
        "import torch, gated_deltanet_state_tail_b200 as gdn\n"
        "assert gdn.gdn_debug_bounds_enabled(), gdn.LIB_PATH\n"
        "ws = torch.zeros(256, dtype=torch.uint8, device='cuda')\n"
        "gdn.gdn_selftest_index_check(ws)\n"
        "assert gdn.gdn_workspace_status(ws) == gdn.GDN_ERR_BOUNDS\n"
        "from gated_deltanet_state_tail_b200 import inputs\n"
        "t = inputs.draw_tensors(300, 2, 128, 128, 'bf16', 0.9, 0.999, 3, device='cuda', with_q=False)\n"
        "st = gdn.tail_replay_state(t['k'], t['v'], t['alpha'], t['beta'], [0, 300], [300], [100])\n"
        "assert torch.isfinite(st).all() and st.abs().max() > 0\n"
        "print('debug-ok')\n")
    r = _child(["-c", code], timeout=300)
    assert r.returncode == 0 and "debug-ok" in r.stdout, r.stdout[-2000:] + r.stderr[-2000:]


def test_release_build_has_no_index_checks():
    import gated_deltanet_state_tail_b200 as gdn
    if gdn.DEBUG_BOUNDS:
        pytest.skip("this process runs the debug build")
    import torch
    assert not gdn.gdn_debug_bounds_enabled()
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    with pytest.raises(gdn.GdnError) as e:
        gdn.gdn_selftest_index_check(ws)
    assert e.value.status == gdn.GDN_ERR_UNSUPPORTED


def test_varlen_and_edge_cases_clean_on_debug_build():
    sel = ("varlen or edges or gate or window or random or fused or outputs or strided or noalloc "
           "or mismatch or rerun")
    files = ["tests/test_parity_gpu.py", "tests/test_fused_gpu.py", "tests/test_decode_outputs_gpu.py",
             "tests/test_layouts_gpu.py"]
    r = _child(["-m", "pytest", "-q", "-x", "-m", "gpu", "-p", "no:cacheprovider", "-k", sel, *files])
    tail = r.stdout[-3000:] + r.stderr[-2000:]
    assert r.returncode == 0, tail
    assert " passed" in r.stdout and "failed" not in r.stdout, tail
