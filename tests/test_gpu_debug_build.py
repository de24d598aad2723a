"""The debug build (libb200attn_debug.so, -DB2A_DEBUG) on the GPU: every TMA
box and TMEM access of the real kernels passes its bounds check on the small
and ragged parity shapes (status OK after every call), and the results still
match the FP64 oracle.  Runs in a child process with ATTN_DEBUG=1, since a
process loads one build of the library."""
import json
import os
import subprocess
import sys

import pytest

from parity import LSE_ABS, MAX_ABS, REL_FRO, record

pytestmark = pytest.mark.gpu

TESTS = os.path.dirname(os.path.abspath(__file__))


def test_debug_build_checks_pass_and_results_match_the_oracle():
    from long_context_bidirectional_b200 import build as B
    B.build(debug=True)
    env = dict(os.environ, ATTN_DEBUG="1")
    r = subprocess.run([sys.executable, os.path.join(TESTS, "debug_build_cases.py")], env=env,
                       capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-3000:]
    cases = [json.loads(l) for l in r.stdout.splitlines() if l.startswith("{")]
    # 5 sizes x (d=64: 1 kernel, d=128: 2 kernels) x 3 modes + 7 projection cases
    assert len(cases) == 52, r.stdout[-2000:]
    bad = []
    for c in cases:
        record(f"debug build {c['case']}", "max_abs", c["max_abs"], MAX_ABS)
        ok = (c["status"] == "ok" and c["max_abs"] <= MAX_ABS and c["rel_fro"] <= REL_FRO
              and c["dlse"] <= LSE_ABS)
        if not ok:
            bad.append(c)
    assert not bad, json.dumps(bad, indent=1)[:4000]
