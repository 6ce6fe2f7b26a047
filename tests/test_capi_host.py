"""C ABI checks that need no GPU: the library loads, exports every entry
point include/*.h declares, and its host-side logic (configuration checks,
ceil/floor partition, buffer sizes, argument refusals) agrees with the
oracle.  No call here enqueues device work."""
import glob
import os
import re
import subprocess

import numpy as np
import pytest

from combine_moe_layout_06_b200 import build, capi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return capi.lib()


def _declared():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"^[A-Za-z_][\w \*]*?\b(moe_\w+)\s*\(", text, flags=re.M)
    return names


def test_header_declares_binding_entry_points():
    assert sorted(_declared()) == sorted(capi.ENTRY_POINTS)


def test_every_declared_symbol_is_exported(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", capi.LIB_PATH], check=True,
                         capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for name in _declared():
        assert name in exported, name
        assert hasattr(lib, name)


def test_partition_matches_oracle(lib, oracle_mod):
    for E in range(1, 200):
        for R in range(1, E + 1):
            assert capi.moe_expert_partition(E, R) == oracle_mod.partition(E, R).tolist()
    for E, R in [(384, 5), (384, 7), (1024, 1000), (60, 7), (256, 7)]:
        assert capi.moe_expert_partition(E, R) == oracle_mod.partition(E, R).tolist()


@pytest.mark.parametrize("E,R,code", [(2, 8, capi.MOE_ERR_EMPTY_RANK), (0, 1, capi.MOE_ERR_INVALID_ARG),
                                      (4, 0, capi.MOE_ERR_INVALID_ARG)])
def test_partition_refusals(lib, E, R, code):
    with pytest.raises(capi.MoeError) as ei:
        capi.moe_expert_partition(E, R)
    assert ei.value.status == code


def test_check_config_agrees_with_oracle(lib, oracle_mod):
    rng = np.random.default_rng(1)
    cases = [(4, 8, 8, 2, 2, 1), (4, 8, 2, 1, 8, 1), (4, 8, 8, 9, 2, 1), (4, 8, 8, 2, 4, 3),
             (4, 8, 8, 2, 4, 8), (-1, 8, 8, 2, 2, 1), (4, 0, 8, 2, 2, 1), (4, 8, 8, 0, 2, 1),
             (0, 8, 8, 2, 2, 2), (4, 8, 60, 4, 7, 7), (4, 8, 60, 4, 7, 1)]
    for _ in range(400):
        cases.append(tuple(int(v) for v in (rng.integers(0, 5), rng.integers(1, 9),
                                            rng.integers(1, 40), rng.integers(1, 10),
                                            rng.integers(1, 12), rng.integers(1, 6))))
    for T, H, E, k, R, N in cases:
        want = oracle_mod.validate_config(T, H, E, k, R, N)
        got = capi.moe_check_config(capi.config(T, H, E, k, R, N))
        assert got == want, (T, H, E, k, R, N)


def test_library_limits(lib):
    assert capi.moe_check_config(capi.config(1, 8, capi.MOE_MAX_EXPERTS + 1, 2, 2)) == capi.MOE_ERR_INVALID_ARG
    assert capi.moe_check_config(capi.config(1, 8, 64, capi.MOE_MAX_TOPK + 1, 2)) == capi.MOE_ERR_INVALID_ARG
    assert capi.moe_check_config(capi.config(1 << 28, 8, 64, 8, 2)) == capi.MOE_ERR_INVALID_ARG
    assert capi.moe_check_config(capi.config(1, 8, 64, 8, 64, 64, capi.MOE_FLAG_TWO_LEVEL)) == capi.MOE_ERR_BAD_NODES
    assert capi.moe_check_config(capi.config(1, 8, 64, 8, 64, 32, capi.MOE_FLAG_TWO_LEVEL)) == capi.MOE_OK
    assert capi.moe_check_config(capi.config(1, 8, 8, 2, 2, 1, 0x80)) == capi.MOE_ERR_INVALID_ARG
    both = capi.MOE_FLAG_COPY_BULK | capi.MOE_FLAG_COPY_VECTOR
    assert capi.moe_check_config(capi.config(1, 8, 8, 2, 2, 1, both)) == capi.MOE_ERR_INVALID_ARG


def test_sizes(lib):
    cfg = capi.config(16384, 7168, 256, 8, 8, 2, capi.MOE_FLAG_TWO_LEVEL)
    assert capi.moe_node_staging_rows(cfg) == 16384 * 2
    assert capi.moe_node_staging_rows(capi.config(100, 8, 64, 4, 32, 32, 1)) == 400
    ws_flat = capi.moe_layout_workspace_bytes(capi.config(65536, 2048, 60, 4, 7))
    assert ws_flat >= 60 * (65536 // 256) * 4
    ws_two = capi.moe_layout_workspace_bytes(cfg)
    assert ws_two >= (256 + 2) * (16384 // 256) * 4
    assert capi.moe_layout_workspace_bytes(capi.config(0, 8, 8, 2, 2)) > 0


def test_argument_refusals_touch_no_device(lib):
    cfg = capi.config(4, 8, 8, 2, 2)
    empty = capi.MoeLayout()
    with pytest.raises(capi.MoeError) as ei:
        capi.moe_layout(cfg, 0, empty, stream=0)
    assert ei.value.status == capi.MOE_ERR_INVALID_ARG
    with pytest.raises(capi.MoeError) as ei:
        capi.moe_dispatch(capi.config(4, 8, 2, 1, 8), empty, 0, 0, stream=0)
    assert ei.value.status == capi.MOE_ERR_EMPTY_RANK
    with pytest.raises(capi.MoeError) as ei:
        capi.moe_combine(cfg, empty, 0, 0, 0, stream=0)
    assert ei.value.status == capi.MOE_ERR_INVALID_ARG
    with pytest.raises(capi.MoeError) as ei:   # decoupled needs one node per rank
        capi.moe_dispatch_decoupled(capi.config(4, 8, 8, 2, 2, 1, capi.MOE_FLAG_TWO_LEVEL),
                                    empty, 0, 0, 0, 0, stream=0)
    assert ei.value.status == capi.MOE_ERR_INVALID_ARG
    assert capi.moe_get_error(empty, stream=0) == capi.MOE_ERR_INVALID_ARG
    for s in range(9):
        assert capi.moe_status_string(s).startswith("MOE_")


def test_enable_peer_access_without_a_device(lib):
    """With no GPU visible the host call reports MOE_ERR_CUDA and changes
    nothing (the refusals of bad device pairs are checked on a GPU)."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is visible here")
    with pytest.raises(capi.MoeError) as ei:
        capi.moe_enable_peer_access(0, 1)
    assert ei.value.status == capi.MOE_ERR_CUDA
