"""GPU: the index-checked debug library (libsala_debug.so, built with SALA_DEBUG).

The debug build checks, before each access, the indices that data or arithmetic select
(attention block indices, selection buffer slots and output positions, score scratch
slots, decode block indices); a failed check skips the access and raises
SALA_ERR_BOUNDS.  Two checks here, each running the debug library in a child process
(the binding loads it for SALA_LIBRARY=debug):
  * every entry point on ragged shapes: no check fails, and the outputs equal the release
    library's bit for bit (the checks do not change the arithmetic);
  * an attention call whose selection holds block indices outside [-1, key blocks): the
    debug build reports SALA_ERR_BOUNDS with the source line, and its output equals the
    release build's, which skips such entries as not live (so the planted input is safe
    for both builds: no access is ever made with them).
"""
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

sala = pytest.importorskip("sparse_attention_long_lightning_b200")
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _outputs(bad_idx: bool):
    """The calls both builds run, on seeded inputs; returns a dict of CPU tensors plus the
    device error and the first failed check's line after the calls."""
    from sparse_attention_long_lightning_b200 import inputs
    dev = "cuda"
    out = {}
    if not bad_idx:
        x = inputs.lightning_inputs(1, 128 * 5 + 19, 4, 128, seed=51, device=dev)
        y, S = sala.lightning_prefill(x.q, x.k, x.v, x.g)
        out["light_y"], out["light_S"] = y, S
        s = inputs.sparse_inputs(1, 64 * 90 + 21, 16, 2, 128, seed=52, device=dev, gate=True)
        idx = sala.sparse_select(s.q, s.k, topk=64)
        out["sel"] = idx
        out["sel_k100"] = sala.sparse_select(s.q, s.k, topk=100)
        out["sel_hsm"] = sala.sparse_select(s.q, s.k, topk=32, score="head_softmax")
        out["attn"] = sala.sparse_attn(s.q, s.k, s.v, idx, s.g)
        a, b = 1234, 4000
        wi = sala.sparse_select(s.q[:, a:b], s.k, topk=64, q_pos0=a)
        out["win_sel"] = wi
        out["win_attn"] = sala.sparse_attn(s.q[:, a:b], s.k, s.v, wi, s.g[:, a:b], q_pos0=a)
        # sparse-layer decode over a 4096-row cache for two sequences
        B, Tmax, Hq, Hkv, D = 2, 4096, 16, 2, 128
        c = inputs.sparse_inputs(B, Tmax, Hq, Hkv, D, seed=53, device=dev)
        kbar = sala.sparse_block_means(c.k)
        q1 = c.q[:, 0].contiguous()
        pos = torch.tensor([3000, 4095], dtype=torch.int32, device=dev)
        out["dec"] = sala.sparse_decode(q1, c.k, c.v, kbar, pos, topk=16)
    else:
        s = inputs.sparse_inputs(1, 64 * 40 + 7, 16, 2, 128, seed=54, device=dev, gate=True)
        idx = sala.sparse_select(s.q, s.k, topk=16)
        idx[0, 0, 2000, 3] = 1_000_000  # past the key blocks
        idx[0, 1, 2100, 5] = -5         # below -1
        out["attn_bad"] = sala.sparse_attn(s.q, s.k, s.v, idx, s.g)
    torch.cuda.synchronize()
    res = {k: v.detach().cpu() for k, v in out.items()}
    res["device_error"] = sala.get_device_error()
    res["bounds_line"] = sala.debug_bounds_line()
    res["version"] = sala.version()
    return res


def _child(bad_idx: bool, path: str):
    torch.save(_outputs(bad_idx), path)


def _run_debug(bad_idx: bool, tmp_path):
    path = str(tmp_path / f"dbg_{int(bad_idx)}.pt")
    env = dict(os.environ, SALA_LIBRARY="debug")
    code = (f"import sys; sys.path.insert(0, {ROOT!r}); "
            f"import tests.test_gpu_debug_build as t; t._child({bad_idx}, {path!r})")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    return torch.load(path)


def test_debug_build_matches_release_without_failed_checks(tmp_path):
    from sparse_attention_long_lightning_b200 import build as sala_build
    sala_build.build(debug=True)
    dbg = _run_debug(False, tmp_path)
    assert "SALA_DEBUG" in dbg["version"]
    assert dbg["device_error"] == 0 and dbg["bounds_line"] == 0
    rel = _outputs(False)  # this process: the release library
    assert rel["device_error"] == 0 and rel["bounds_line"] == -1
    for k, v in rel.items():
        if isinstance(v, torch.Tensor):
            assert torch.equal(v, dbg[k]), k


def test_debug_build_reports_out_of_range_block_indices(tmp_path):
    from sparse_attention_long_lightning_b200 import build as sala_build
    sala_build.build(debug=True)
    dbg = _run_debug(True, tmp_path)
    assert dbg["device_error"] == 7  # SALA_ERR_BOUNDS
    assert dbg["bounds_line"] > 0
    rel = _outputs(True)
    assert rel["device_error"] == 0  # the release build skips such entries as not live
    assert torch.equal(rel["attn_bad"], dbg["attn_bad"])
