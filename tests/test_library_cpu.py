"""CPU-only checks of the C library: it builds for sm_100a, loads, exports every
symbol the public header declares, and validates arguments on the host."""
import ctypes
import os
import re

import pytest

from quantized_routed_expert_04_b200 import binding, build, synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return binding.load_library()


def header_functions():
    text = open(os.path.join(ROOT, "include", "strata_moe.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(strata_\w+)\s*\(", text)))


def test_header_declares_the_four_named_calls():
    names = header_functions()
    for n in ("strata_moe_create", "strata_moe_bind_slot", "strata_moe_route",
              "strata_moe_forward"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for name in header_functions():
        assert hasattr(lib, name), name
        ctypes.cast(getattr(lib, name), ctypes.c_void_p)


def test_expert_bytes_matches_format(lib):
    for H, I in [(256, 512), (2048, 1408), (4096, 14336), (4096, 1024), (4096, 2048), (384, 256)]:
        assert binding.strata_moe_expert_bytes(H, I) == synth.expert_bytes(H, I)
    assert binding.strata_moe_expert_bytes(100, 64) == 0


@pytest.mark.parametrize("args", [
    (0, 512, 8, 2, 0, 8),        # hidden 0
    (256, 448, 8, 2, 0, 8),      # inter not a multiple of 128
    (256, 512, 0, 1, 0, 1),      # no experts
    (256, 512, 300, 2, 0, 300),  # too many experts
    (256, 512, 8, 9, 0, 8),      # top_k > n_experts
    (256, 512, 8, 2, 5, 8),      # too many shared experts
    (256, 512, 8, 2, 0, 1),      # fewer slots than top_k
    (256, 512, 8, 2, 0, 9),      # more slots than experts
])
def test_create_rejects_bad_shapes_on_host(lib, args):
    h = ctypes.c_void_p()
    st = lib.strata_moe_create(*args, ctypes.byref(h))
    assert st == binding.Status.INVALID_ARG and not h.value


def test_null_handle_calls_fail_cleanly(lib):
    assert lib.strata_moe_bind_slot(None, 0, 0, None) == binding.Status.INVALID_ARG
    assert lib.strata_moe_forward(None, None, 1, None, None) == binding.Status.INVALID_ARG
    assert lib.strata_moe_route(None, None, 1, None, None, None, None) == binding.Status.INVALID_ARG
    assert lib.strata_moe_slot_expert(None, 0) == -2
    assert binding.strata_status_str(4) == "expert already bound to another slot"


def test_library_is_sm100a_only():
    """Every kernel object was compiled for sm_100a (ptxas log)."""
    logs = [f for f in os.listdir(build.BUILD) if f.startswith("ptxas_")]
    assert logs
    for f in logs:
        text = open(os.path.join(build.BUILD, f)).read()
        targets = set(re.findall(r"for '(sm_\w+)'", text))
        assert targets <= {"sm_100a"}, (f, targets)


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    # no fallback: without the built library the binding raises
    monkeypatch.setattr(binding, "_lib", None)
    monkeypatch.setattr(binding, "LIB_PATH", str(tmp_path / "libstrata_moe.so"))
    with pytest.raises(RuntimeError, match="not built"):
        binding.load_library()


def test_product_code_never_uses_the_oracle():
    # the oracle is test infrastructure: the package, its C sources and the
    # header must not import it, load its library or call its functions
    use = re.compile(r"(import\s+oracle|from\s+oracle|liboracle|oracle_\w+\s*\(|oracle\.\w+\()")
    offenders = []
    for base, _, files in os.walk(os.path.join(ROOT, "quantized_routed_expert_04_b200")):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                if use.search(open(os.path.join(base, f)).read()):
                    offenders.append(os.path.relpath(os.path.join(base, f), ROOT))
    assert not offenders, offenders
    assert not use.search(open(os.path.join(ROOT, "include", "strata_moe.h")).read())
