"""The library under more than one CUDA context on one device (a child process, so the
test session's own context is untouched; tests/context_child.py does the work).

  * The no-allocation entry point looks its fixed scratch array up in the context current at
    each call: it gives the planned entry point's codes, scales and s_g in the primary
    context, in a second context made through the driver API, and in the primary context
    again after the second one is destroyed.  (An address kept from an earlier call would
    point into the wrong context.)
  * A plan belongs to the context it was made in: in another context its calls return
    FP4Q_ERR_ARG before their shape check and before anything is launched (probed with an
    invalid row count, which no call launches on); in its own context the same probe gets
    FP4Q_ERR_SHAPE.  A plan made in the second context works there."""

import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.mark.parametrize("b", [16, 128])
def test_two_contexts(cuda_device, b):
    from microscaling_fp4_quantization_b200 import fp4q as F
    r = subprocess.run([sys.executable, os.path.join(HERE, "context_child.py"), str(b)], capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    seen = json.loads(r.stdout.strip().splitlines()[-1])
    for k in ("noalloc_primary_first", "noalloc_second_context", "plan_made_in_second_context",
              "noalloc_primary_after", "planned_primary_after"):
        assert seen[k] is True, (k, seen)
    assert all(v == F.FP4Q_ERR_SHAPE for v in seen["checks_in_primary"].values()), seen
    assert all(v == F.FP4Q_ERR_ARG for v in seen["checks_in_second_context"].values()), seen
