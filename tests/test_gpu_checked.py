"""The checked build of the library (STQ_CHECKS) records, in the pool's sticky error
word, stored codes 0 (a slot decoded before it was initialised) and non-finite updated
states; stq_pool_check reports them. Run in a child process that loads the checked
library through STQ_LIBRARY."""
import os
import subprocess
import sys

import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import numpy as np, torch
from quantized_linear_attention_02_b200 import stq
assert b"checked" in stq.lib().stq_version()
D, H = 128, 2
for bits, kind in ((6, "gdn"), (4, "kda")):
    ub = np.full(H if kind == "gdn" else H * D, bits, np.uint8)
    if kind == "kda":
        ub[5] = 2; ub[200] = 16                      # mixed widths and a pivot row
    pool = stq.Pool(kind, 4, ub, np.ones((H, D), np.float32))
    slots = torch.tensor([1, 2], dtype=torch.int32, device="cuda")
    g = torch.Generator(device="cuda").manual_seed(0)
    q, k, v = (torch.randn(2, H, D, device="cuda", generator=g) for _ in range(3))
    k = torch.nn.functional.normalize(k, dim=-1)
    gate = torch.full((2, H) if kind == "gdn" else (2, H, D), 0.9, device="cuda")
    beta = torch.full((2, H), 0.5, device="cuda")
    out = torch.empty(2, H, D, device="cuda")
    # 1. slots never initialised: every code is 0
    pool.decode_step(slots, q, k, v, gate, beta, out)
    try:
        pool.check(); raise SystemExit("uninitialised slot not reported")
    except stq.StqError as e:
        assert "code was 0" in str(e), e
    # 2. initialised slots and finite inputs: nothing to report
    pool.quantize_init(slots, torch.randn(2, H, D, D, device="cuda", generator=g))
    pool.decode_step(slots, q, k, v, gate, beta, out)
    pool.check()
    # 3. a NaN input makes the updated state non-finite
    v[0, 1, 3] = float("nan")
    pool.decode_step(slots, q, k, v, gate, beta, out)
    try:
        pool.check(); raise SystemExit("non-finite state not reported")
    except stq.StqError as e:
        assert "non-finite" in str(e), e
print("checked ok")
"""


def test_checked_build_records_zero_codes_and_nonfinite_states():
    from quantized_linear_attention_02_b200 import build
    lib = build.build(checked=True)
    env = dict(os.environ, STQ_LIBRARY=lib)
    r = subprocess.run([sys.executable, "-c", CHILD], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]
    assert "checked ok" in r.stdout


def test_default_build_has_no_code_checks():
    """The default library does not look at code values: an uninitialised slot decodes
    without a report (only slot indices are always checked)."""
    import numpy as np
    from quantized_linear_attention_02_b200 import build, stq
    build.build()
    assert b"checked" not in stq.lib().stq_version()
    pool = stq.Pool("gdn", 2, np.full(1, 6, np.uint8), np.ones((1, 128), np.float32))
    slots = torch.tensor([0], dtype=torch.int32, device="cuda")
    x = torch.zeros(1, 1, 128, device="cuda")
    pool.decode_step(slots, x, x, x, torch.ones(1, 1, device="cuda"), torch.zeros(1, 1, device="cuda"),
                     torch.empty(1, 1, 128, device="cuda"))
    pool.check()
