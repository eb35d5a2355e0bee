"""The BSVA_DEVICE_CHECKS build (libbsva_checked.so) on the GPU.

It runs in a child process, so that the checked library is the one the binding
loads there:
- an ordinary Sol call matches the oracle as the default build does, with a clean
  status word;
- a route whose kept list names a key block past the end, or whose kept count
  exceeds the number of key blocks, is caught by the kernels' own index checks.
  They clamp the values before any access, so nothing reads outside its buffer,
  and bsva_check_status reports BSVA_ERR_DEVICE_BOUNDS;
- the next valid call runs clean.

The corrupted route is never given to the default build: it would index past the
kept list's scales there.
"""
import os
import subprocess
import sys
import textwrap

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = textwrap.dedent("""
    import sys
    sys.path.insert(0, {root!r})
    sys.path.insert(0, {tests!r})
    import numpy as np
    import torch
    import block_sparse_video_int8_b200 as bsva
    import oracle
    import workloads
    from parity import Report, assert_within, compare_rows, q_rows, to_np

    lib = bsva.load()
    assert lib.bsva_device_checks() == 1, "the checked build is not the one loaded"
    w = workloads.get("ragged_pe")
    Q, K, V = [x.cuda() for x in workloads.batch_qkv(w)]
    route = bsva.sparse_attn_route(Q, K, 1.0)
    ws = bsva.new_workspace(route.shape, w.centroid_mode)
    out, lse = bsva.sparse_attn_fwd(route, V, w.centroid_mode, workspace=ws, with_lse=True, out_dtype=torch.float32)
    bsva.check_status(ws)
    rep = Report()
    for b in range(w.B):
        for h in range(w.H):
            q, k, v = (t.float().numpy() for t in workloads.head_qkv(w, b, h))
            ref = oracle.route_head(q, k, 1.0)
            keep = to_np(route.kept_mask[b, h]).astype(bool)
            assert np.array_equal(keep, ref["keep"]) or ref["band"].any(), "routing"
            O, L = oracle.sol_attention_head(ref["q8"], ref["q_scale"], ref["k8"], ref["k_scale"], v, keep,
                                             w.centroid_mode, 0.0)
            compare_rows(to_np(out[b, h]), to_np(lse[b, h]), O, L, q_rows(w.Lq, range(w.nQB)), rep)
    assert_within(rep, "checked build, Sol")

    bad = bsva.sparse_attn_route(Q, K, 1.0)
    bad.kept_idx[0, 0, 0, 0] = w.nKB + 7       # a kept block past the last one
    bad.kept_cnt[0, 1, 2] = w.nKB + 3          # more kept blocks than there are
    torch.cuda.synchronize()
    bsva.sparse_attn_fwd(bad, V, w.centroid_mode, workspace=ws)
    try:
        bsva.check_status(ws)
        raise SystemExit("the out-of-range route was not reported")
    except bsva.BsvaError as e:
        assert e.code == 6, e

    out2 = bsva.sparse_attn_fwd(route, V, w.centroid_mode, workspace=ws, out_dtype=torch.float32)
    bsva.check_status(ws)
    assert torch.equal(out2, out), "a valid call after the bad one differs"
    print("checked build ok")
""")


def test_checked_build_matches_the_oracle_and_flags_bad_routes():
    from block_sparse_video_int8_b200 import build
    build.build(checked=True)
    code = CHILD.format(root=ROOT, tests=os.path.join(ROOT, "tests"))
    env = dict(os.environ, BSVA_CHECKED="1")
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    assert "checked build ok" in r.stdout
