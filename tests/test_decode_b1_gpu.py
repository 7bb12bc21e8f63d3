"""Batch-1 bf16 2:4 apply, the path whose rows are fed to shared memory by
bulk copies: parity with the oracle on the layouts that exercise it (several
256-row segments per CTA, an x that is not 16-byte aligned, a group of layers
of different widths), the fallback for rows too wide for shared memory, and
agreement with the register-fed kernel."""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import oracle
from gpu_util import TOL, dev, host
from test_apply_gpu import Case, err_of

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def hsl():
    from sparse_rank_linear_03_b200 import hsl as mod
    return mod


def test_tall_layer_several_segments_per_cta(hsl):
    # 80000 rows over at most 148 CTAs: > 256 rows (several segments) each
    c = Case(hsl, 80000, 64, 4, "nm24", "bf16", 0.5, 71)
    Xb = c.x(1, 72)
    assert err_of(c, c.L.apply(dev(Xb, "bf16")), Xb) <= TOL["bf16"]


def test_x_not_16_byte_aligned(hsl):
    c = Case(hsl, 300, 1024, 8, "nm24", "bf16", 0.5, 73)
    Xb = c.x(1, 74)
    buf = torch.zeros(1 + c.n, dtype=torch.bfloat16, device="cuda")
    buf[1:] = dev(Xb, "bf16").view(-1)
    X = buf[1:].view(1, c.n)          # 2 bytes past an aligned address
    assert X.data_ptr() % 16 != 0
    assert err_of(c, c.L.apply(X), Xb) <= TOL["bf16"]


def test_group_of_different_widths(hsl):
    shapes = [(700, 4096), (333, 1024), (129, 11008), (1, 64)]
    cases = [Case(hsl, m, n, 8, "nm24", "bf16", 0.5, 80 + i) for i, (m, n) in enumerate(shapes)]
    g = hsl.Group([c.L for c in cases])
    Xs = [c.x(1, 90 + i) for i, c in enumerate(cases)]
    Yd = [torch.empty(1, c.m, dtype=torch.bfloat16, device="cuda") for c in cases]
    for _ in range(2):
        g.apply([dev(x, "bf16") for x in Xs], Yd)
        torch.cuda.synchronize()
        for c, x, y in zip(cases, Xs, Yd):
            assert err_of(c, y, x) <= TOL["bf16"]
    g.close()


def test_rows_wider_than_shared_memory_fall_back(hsl):
    c = Case(hsl, 64, 28672, 4, "nm24", "bf16", 0.5, 75)
    Xb = c.x(1, 76)
    assert err_of(c, c.L.apply(dev(Xb, "bf16")), Xb) <= TOL["bf16"]


def _child(tmp_path, name, env_extra, m, n, r, seed):
    out = str(tmp_path / f"{name}.npy")
    env = dict(os.environ, **env_extra)
    env["PYTHONPATH"] = ROOT + os.pathsep + env.get("PYTHONPATH", "")
    subprocess.run([sys.executable, os.path.join(ROOT, "tests", "decode_child.py"), out,
                    str(m), str(n), str(r), str(seed)], check=True, env=env, cwd=ROOT,
                   timeout=600)
    return np.load(out)


@pytest.mark.parametrize("m,n", [(4000, 8192), (777, 1040)])
def test_bulk_fed_and_register_fed_agree(tmp_path, m, n):
    """The two kernels sum the same products in different orders (per
    super-chunk partials vs one running sum per lane): outputs agree to bf16
    rounding."""
    a = _child(tmp_path, "bulk", {}, m, n, 16, 5)
    b = _child(tmp_path, "regs", {"HSL_DECODE_B1": "regs"}, m, n, 16, 5)
    assert a.shape == (1, m)
    fa, fb = oracle.bits_to_f64(a, "bf16"), oracle.bits_to_f64(b, "bf16")
    assert oracle.rel_err(fa, fb) <= 2 ** -8


def test_bounded_wait_gives_up_and_reports_timeout(hsl, monkeypatch):
    """HSL_FAULT_INJECT=zwait gives the batch-1 kernel's wait for z a target no
    CTA count reaches: the wait gives up after its bounded polls, the kernel
    finishes, hsl_check reports HSL_ERR_TIMEOUT, and the context stays usable
    (the next call, without the injection, is correct)."""
    c = Case(hsl, 3000, 2048, 16, "nm24", "bf16", 0.5, 77)
    Xb = c.x(1, 78)
    monkeypatch.setenv("HSL_FAULT_INJECT", "zwait")
    c.L.apply(dev(Xb, "bf16"))
    monkeypatch.delenv("HSL_FAULT_INJECT")
    with pytest.raises(hsl.HslError) as e:
        c.L.check()
    assert e.value.name == "HSL_ERR_TIMEOUT"
    c.L.check()  # the error word was cleared
    for _ in range(2):
        Y = c.L.apply(dev(Xb, "bf16"))
        c.L.check()
        assert err_of(c, Y, Xb) <= TOL["bf16"]
