"""The failure path of the attention kernel's bounded waits, on the GPU without
a fault: in a child process whose environment shortens the kernel's wait limit
to 200 ms and makes every CTA's builder withhold its first work item
(LYCHEE_TEST_WAIT_LIMIT_MS, LYCHEE_TEST_WITHHOLD_ITEM, read once per process by
the library), the waits on that item run out, the call returns, the device
error word reports the timeout (LYCHEE_ERR_TIMEOUT, bit 8), and the CUDA
context is still usable afterwards.  The parent process never sets either
variable, so no other test is affected."""
import os
import subprocess
import sys
import textwrap

import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = textwrap.dedent("""
    import sys, time, torch
    sys.path.insert(0, {root!r})
    from hybrid_head_sparse_decode_b200 import inputs, ops
    dev = torch.device("cuda")
    p = inputs.make_layer(1, 8, 2, 128, 4096, roles=[1, 0, 0, 0, 0, 0, 0, 1], seed=9,
                          k_frac=0.3, device=dev)
    ws = ops.alloc_workspace(1, 8, 2, 128, 4096, p.k, torch.bfloat16, dev)
    t0 = time.time()
    ops.hybrid_decode_attn(p.q, p.k_cache, p.v_cache, p.seqlens, p.role, p.idx_in, p.k,
                           k_per_seq=p.k_per_seq, workspace=ws)
    st, bits = ops.check_device_error(ws)
    dt = time.time() - t0
    ok = float(torch.ones(1000, device=dev).sum().item()) == 1000.0
    print("RESULT", st, bits, round(dt, 3), ok)
""")


def test_attention_wait_runs_out_and_reports_timeout():
    env = dict(os.environ, LYCHEE_TEST_WAIT_LIMIT_MS="200", LYCHEE_TEST_WITHHOLD_ITEM="1")
    r = subprocess.run([sys.executable, "-c", CHILD.format(root=ROOT)], env=env,
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    line = [x for x in r.stdout.splitlines() if x.startswith("RESULT")][-1].split()
    st, bits, secs, ok = int(line[1]), int(line[2]), float(line[3]), line[4] == "True"
    assert st == 6 and bits & 8, (st, bits)        # LYCHEE_ERR_TIMEOUT, timeout bit
    assert ok, "the CUDA context must stay usable after a wait gave up"
    assert secs < 30, secs                          # the waits gave up after ~0.2 s each
