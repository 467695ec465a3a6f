"""The C ABI library loads and exports every symbol include/confkv.h declares;
host-side argument validation works without a GPU (CPU only)."""
import ctypes
import os
import re
import subprocess

import pytest

from confidence_gated_kv_logit_b200 import binding, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return binding.load_library()


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "confkv.h")).read()
    return sorted(set(re.findall(r"CONFKV_API\s+[\w\s\*]+?\b(confkv_\w+)\s*\(", text)))


def test_header_declares_the_documented_entry_points():
    names = declared_symbols()
    for n in ("confkv_create", "confkv_prefill", "confkv_confidence", "confkv_decode_attn",
              "confkv_evict_compact", "confkv_destroy"):
        assert n in names
    assert sorted(binding.EXPORTED) == names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name
    # nothing else leaks: the shared object exports only the confkv_ prefix
    out = os.popen(f"nm -D --defined-only {binding.LIB_PATH}").read()
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    assert {s for s in exported if s.startswith("confkv_")} == set(declared_symbols())


def test_status_strings_and_version(lib):
    for code in range(8):
        assert lib.confkv_status_string(code)
    assert lib.confkv_version() >= 100


def test_default_params(lib):
    p = binding.default_params()
    assert (p.n_low, p.n_high, p.protect_last, p.fp16_window) == (256, 512, 64, 128)
    assert abs(p.tau - 0.6) < 1e-7 and abs(p.alpha - 0.5) < 1e-7 and abs(p.ema_decay - 0.9) < 1e-7
    assert lib.confkv_default_params(None) == 1
    assert (p.score_source, p.seed, p.single_stream) == (binding.SCORE_EMA, 0, 0)


def test_param_struct_matches_the_header():
    # every field of confkv_params in include/confkv.h, in order, is in the ctypes mirror
    text = open(os.path.join(ROOT, "include", "confkv.h")).read()
    body = text[text.index("typedef struct {", text.index("CONFKV_ALL_LAYERS")):text.index("} confkv_params;")]
    fields = re.findall(r"^\s*(?:int32_t|uint32_t|float)\s+(\w+);", body, re.M)
    assert fields == [name for name, _ in binding.Params._fields_]


@pytest.mark.parametrize("shape,kw", [
    ((1, 4, 4, 96), {}),          # head_dim must be 64 or 128
    ((1, 4, 6, 64), {}),          # q_heads not a multiple of kv_heads
    ((1, 1, 16, 128), {}),        # 16 query heads per KV head is beyond the kernels
    ((0, 4, 4, 64), {}),
    ((1, 4, 4, 64), {"alpha": 1.5}),
    ((1, 4, 4, 64), {"fp16_window": 0}),
    ((1, 4, 4, 64), {"mode": 1, "fixed_budget": 10, "n_sink": 8, "protect_last": 8}),
    ((1, 4, 4, 64), {"gate": 7}),
    ((1, 4, 4, 64), {"score_source": 3}),
    ((1, 4, 4, 64), {"compact": 3}),
    ((1, 4, 4, 64), {"compact": 2, "int8_enable": 0}),       # the linear window needs INT8 on
    ((1, 4, 4, 64), {"compact": 2, "mode": 1, "fixed_budget": 64, "protect_last": 16}),   # and confidence mode
])
def test_create_rejects_bad_arguments_before_touching_the_device(lib, shape, kw):
    p = binding.default_params()
    for k, v in kw.items():
        setattr(p, k, v)
    h = ctypes.c_void_p()
    assert lib.confkv_create(*shape, ctypes.byref(p), ctypes.byref(h)) == 1
    assert not h


def test_null_and_foreign_handles_are_rejected(lib):
    assert lib.confkv_destroy(None) == 0
    bogus = ctypes.c_void_p(0x1000)
    assert lib.confkv_destroy(bogus) == 3
    assert lib.confkv_evict_compact(bogus, 0, None) == 3
    assert lib.confkv_last_error(bogus, 0) == 3


def test_binding_refuses_without_library(tmp_path):
    with pytest.raises(RuntimeError):
        binding.load_library.__wrapped__(str(tmp_path / "missing.so")) if hasattr(binding.load_library, "__wrapped__") else _load_missing(tmp_path)


def _load_missing(tmp_path):
    saved = binding._LIB
    binding._LIB = None
    try:
        binding.load_library(str(tmp_path / "missing.so"))
    finally:
        binding._LIB = saved


def test_plain_c_caller_sees_the_binding_layout(lib, tmp_path):
    """Compile tests/abi_check.c against include/confkv.h with gcc, link it to
    the library, run it, and compare the struct layout it prints (offsetof,
    sizeof) with the ctypes mirrors; it also calls the entry points that need
    no device and checks their results itself."""
    exe = tmp_path / "abi_check"
    libdir = os.path.dirname(binding.LIB_PATH)
    cc = subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                         os.path.join(ROOT, "tests", "abi_check.c"), "-o", str(exe), binding.LIB_PATH,
                         f"-Wl,-rpath,{libdir}"], capture_output=True, text=True)
    assert cc.returncode == 0, cc.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0, (run.returncode, run.stdout, run.stderr)
    lines = run.stdout.splitlines()
    assert lines[-1] == "ok"
    layout = {}
    for ln in lines:
        parts = ln.split()
        if ln.startswith("sizeof "):
            layout[parts[1]] = int(parts[2])
        elif "." in parts[0] and parts[0].startswith("confkv_"):
            layout[parts[0]] = (int(parts[1]), int(parts[2]))
    for struct, mirror in (("confkv_params", binding.Params), ("confkv_stats", binding.Stats),
                           ("confkv_profile", binding.Profile)):
        assert layout[struct] == ctypes.sizeof(mirror), struct
        for name, _ in mirror._fields_:
            f = getattr(mirror, name)
            assert layout[f"{struct}.{name}"] == (f.offset, f.size), (struct, name)
    d = next(ln for ln in lines if ln.startswith("default "))
    assert d.split()[1:6] == ["256", "512", "64", "128", "4096"]
    statuses = [ln for ln in lines if ln.startswith("status ")]
    assert len(statuses) == 8
    for code, ln in enumerate(statuses):
        assert ln.split(" ", 2)[2] == lib.confkv_status_string(code).decode()
