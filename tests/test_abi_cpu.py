"""Host-only checks of the C ABI library: it builds, loads, exports every
symbol include/moe.h declares, and answers size queries; no compute call is
made (there may be no GPU)."""
import os
import re
import subprocess

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def B():
    from sparse_moe_expert_gemv_b200 import build
    build.build()
    from sparse_moe_expert_gemv_b200 import binding
    return binding


def declared_symbols():
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    return sorted(set(re.findall(r"^MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", src, flags=re.M)))


def test_header_declares_the_boundary():
    syms = declared_symbols()
    for name in ("moe_create", "moe_load_experts", "moe_route", "moe_forward", "moe_prefill"):
        assert name in syms
    assert len(syms) >= 15


def test_library_exports_every_declared_symbol(B):
    out = subprocess.run(["nm", "-D", "--defined-only", B.SO_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT\s+(moe_\w+)", out))
    missing = [s for s in declared_symbols() if s not in exported]
    assert not missing, missing
    assert set(B.EXPORTS) == set(declared_symbols())


def test_size_queries(B):
    assert B.moe_expert_bytes(2048, 768, B.MOE_Q4_SYM_G32_F16) == 3 * 2048 * 768 // 2 + 3 * 2048 * 768 // 32 * 2
    assert B.moe_expert_bytes(2048, 768, B.MOE_Q2_ASYM_G64_F16) == 3 * 2048 * 768 // 4 + 2 * 3 * 2048 * 768 // 64 * 2
    assert B.moe_expert_bytes(100, 768, 1) == -1
    assert B.moe_expert_bytes(2048, 768, 3) == -1
    assert B.moe_status_string(7) == "MOE_ERR_TIMEOUT"


def test_bad_arguments_rejected_before_any_device_work(B):
    for args in [(100, 128, 8, 2, 1), (128, 128, 0, 1, 1), (128, 128, 8, 9, 1),
                 (128, 128, 8, 2, 5), (128, 100, 8, 2, 1)]:
        with pytest.raises(B.MoeError) as ei:
            B.moe_create(*args)
        assert ei.value.status == 1


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU path")
def test_create_without_gpu_fails_cleanly(B):
    with pytest.raises(B.MoeError) as ei:
        B.moe_create(256, 128, 16, 2, 1)
    assert ei.value.status == 3  # MOE_ERR_CUDA, no crash
    assert B.moe_destroy(None) is None


def test_generator_numpy_and_torch_agree():
    from sparse_moe_expert_gemv_b200 import inputs as I
    for fmt in (I.Q4, I.Q2):
        c, s, m = I.experts_torch(3, fmt, 256, 128, 2, 5, 3, "cpu", chunk=2)
        for i in range(3):
            cn, sn, mn = I.expert_np(3, fmt, 256, 128, 2, 5 + i)
            assert np.array_equal(c[i].numpy(), cn)
            assert np.array_equal(s[i].numpy().view(np.uint16), sn)
            if fmt == I.Q2:
                assert np.array_equal(m[i].numpy().view(np.uint16), mn)
