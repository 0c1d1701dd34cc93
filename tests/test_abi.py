"""The C-ABI library loads on a machine without a GPU and exports every function that
include/moe.h declares (no compute call is made here)."""
import re
import subprocess
from pathlib import Path

import pytest

ROOT = Path(__file__).resolve().parent.parent


def _declared():
    text = (ROOT / "include" / "moe.h").read_text()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def built():
    from expert_ffn_gemv_b200 import build

    return build.build()


def test_header_declares_the_boundary():
    names = _declared()
    for n in ("moe_create", "moe_load_layer", "moe_forward", "moe_forward_stack", "moe_destroy",
              "moe_status_string", "moe_last_error"):
        assert n in names


def test_library_exports_every_declared_symbol(built):
    out = subprocess.run(["nm", "-D", "--defined-only", str(built)], capture_output=True, text=True, check=True)
    exported = set(re.findall(r"\bT (moe_[a-z0-9_]+)", out.stdout))
    missing = [n for n in _declared() if n not in exported]
    assert not missing, missing


def test_library_loads_and_answers_without_gpu(built):
    import expert_ffn_gemv_b200 as P

    L = P.lib()
    for n in _declared():
        assert hasattr(L, n)
    assert L.moe_status_string(P.MOE_ERR_NOT_LOADED) == b"layer not loaded"
    assert L.moe_last_error(None) == b"no handle"
    assert P.moe_destroy(None) == P.MOE_OK
    assert set(P.EXPORTED) == set(_declared())


def test_binding_names_match_c_names():
    import expert_ffn_gemv_b200 as P

    for n in ("moe_create", "moe_load_layer", "moe_forward", "moe_forward_stack", "moe_check", "moe_destroy"):
        assert callable(getattr(P, n))
