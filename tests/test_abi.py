"""The C ABI on the CPU: the library builds for sm_100a, loads, exports every
symbol include/moe.h declares, the ctypes mirror of its structs matches the C
layout, and host-side validation / sizing behave (no compute calls)."""
import ctypes as C
import os
import re
import subprocess

import pytest

from sparsely_gated_mixture_gate_b200 import _lib, build, synth
from sparsely_gated_mixture_gate_b200 import moe as M

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _lib.load()


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", text)))


def test_header_declares_exports():
    assert declared_symbols() == sorted(_lib.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", _lib.LIB_PATH], check=True,
                         capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (moe_\w+)", out))
    for name in declared_symbols():
        assert name in exported, name
        assert hasattr(lib, name)


def test_struct_layout_matches_c(tmp_path):
    src = tmp_path / "layout.c"
    src.write_text(f'''#include <stdio.h>
#include <stddef.h>
#include "{HEADER}"
int main(void) {{
  printf("%zu %zu %zu %zu %zu %zu %zu %zu %zu %zu %zu\\n", sizeof(moe_config), offsetof(moe_config, seed),
         offsetof(moe_config, capacity_factor), offsetof(moe_config, gate_precision),
         sizeof(moe_gate_params), sizeof(moe_expert_params),
         offsetof(moe_config, alpha_aux), offsetof(moe_config, token_base),
         offsetof(moe_gate_params, seed_dev), sizeof(moe_grads), offsetof(moe_grads, dW_g2));
  return 0;
}}
''')
    exe = tmp_path / "layout"
    subprocess.check_call(["gcc", "-std=c11", "-o", str(exe), str(src)])
    vals = [int(v) for v in subprocess.check_output([str(exe)]).split()]
    want = [C.sizeof(_lib.moe_config), _lib.moe_config.seed.offset,
            _lib.moe_config.capacity_factor.offset, _lib.moe_config.gate_precision.offset,
            C.sizeof(_lib.moe_gate_params), C.sizeof(_lib.moe_expert_params),
            _lib.moe_config.alpha_aux.offset, _lib.moe_config.token_base.offset,
            _lib.moe_gate_params.seed_dev.offset, C.sizeof(_lib.moe_grads),
            _lib.moe_grads.dW_g2.offset]
    assert vals == want


def test_strerror(lib):
    for code in (0, -1, -2, -3, -4, -99):
        assert isinstance(lib.moe_strerror(code), bytes)


@pytest.mark.parametrize("name", list(synth.WORKLOADS) + list(synth.VARIANTS))
def test_workloads_validate(lib, name):
    w = synth.WORKLOADS.get(name) or synth.VARIANTS[name]
    cfg = M.Config.from_workload(w)
    assert M.validate(cfg)
    assert M.workspace_size(cfg) > 0


BAD = [
    dict(k=0), dict(k=9), dict(n=2, k=3), dict(d=12), dict(f=20), dict(T=-1), dict(n=8193),
    dict(router=1, k=1, noise=1), dict(router=1, k=2, noise=0), dict(router=2),
    dict(hier_a=4, hier_b=3, hier_k1=2, hier_k2=2, n=13, k=4),
    dict(hier_a=4, hier_b=2, hier_k1=2, hier_k2=2, n=8, k=2),
    dict(hier_a=4, hier_b=2, hier_k1=5, hier_k2=1, n=8, k=5),
    dict(passthrough=2), dict(capacity_factor=float("nan")),
    dict(raw_expert_dtype=3), dict(raw_gate_precision=2),
    dict(raw_backward=2), dict(raw_shared_expert=2), dict(raw_router_stats=-1),
    dict(token_base=-1), dict(token_base=(1 << 32) - 63),
]


@pytest.mark.parametrize("bad", BAD)
def test_validate_rejects(lib, bad):
    base = dict(T=64, d=32, n=8, k=2, f=64)
    base.update({k: v for k, v in bad.items() if not k.startswith("raw_")})
    cfg = M.Config(**base)
    c = cfg.c()
    for k, v in bad.items():
        if k.startswith("raw_"):
            setattr(c, k[4:], v)
    assert lib.moe_validate(C.byref(c)) == _lib.MOE_EINVAL
    sz = C.c_size_t(0)
    assert lib.moe_workspace_size(C.byref(c), C.byref(sz)) == _lib.MOE_EINVAL


def test_capacity_matches_oracle(lib, orc):
    for (T, k, n, cf) in [(32768, 1, 128, 1.25), (3, 1, 2, 0.5), (1000, 4, 37, 1.1), (7, 2, 3, 0.0),
                          (8192, 4, 256, 1.0), (5, 3, 4, 2.7)]:
        cfg = M.Config(T=T, d=32, n=n, k=k, f=32, capacity_factor=cf)
        assert M.capacity(cfg) == orc.capacity(T, k, n, cf)


def test_workspace_grows_with_tokens(lib):
    a = M.workspace_size(M.Config(T=64, d=32, n=8, k=2, f=64))
    b = M.workspace_size(M.Config(T=640, d=32, n=8, k=2, f=64))
    assert b > a


def test_calls_fail_cleanly_without_gpu(lib):
    """Argument errors come back before any device work; with valid
    arguments and no device the call reports MOE_EDEVICE (never crashes)."""
    cfg = M.Config(T=64, d=32, n=8, k=2, f=64, expert_bf16=0)
    c = cfg.c()
    gp = _lib.moe_gate_params()
    ep = _lib.moe_expert_params()
    nul = None
    # NULL status / outputs -> EINVAL
    rc = lib.moe_forward(C.byref(c), nul, C.byref(gp), C.byref(ep), nul, nul, nul, nul, nul, nul, nul,
                         nul, 0, nul, nul)
    assert rc == _lib.MOE_EINVAL
    # too-small workspace -> EWORKSPACE
    buf = (C.c_byte * 4096)()
    fake = C.c_void_p(C.addressof(buf) + (-C.addressof(buf)) % 256)
    rc = lib.moe_gate(C.byref(c), fake, C.byref(gp), fake, fake, fake, nul, fake, 16, fake, nul)
    assert rc == _lib.MOE_EWORKSPACE
    # combine validates then asks for the device
    rc = lib.moe_combine(C.byref(c), fake, fake, fake, fake, fake, fake, nul)
    import torch
    if not torch.cuda.is_available():
        assert rc == _lib.MOE_EDEVICE


def test_backward_workspace_and_refusals_without_gpu(lib):
    """backward = 1 adds the backward's scratch to the workspace; the entry
    point checks its arguments on the host before anything touches a device."""
    cfg = M.Config(T=64, d=32, n=8, k=2, f=64)
    import dataclasses
    bwd = dataclasses.replace(cfg, backward=1)
    assert M.workspace_size(bwd) > M.workspace_size(cfg)
    assert M.workspace_size(dataclasses.replace(bwd, shared_expert=1)) > M.workspace_size(bwd)
    c = cfg.c()
    g = _lib.moe_grads()
    # no backward flag -> EINVAL (before any device work; a NULL workspace is
    # refused first, either way not MOE_OK)
    rc = lib.moe_backward(C.byref(c), None, None, None, None, None, None, None, None, None, None,
                          C.byref(g), None, 0, None, None)
    assert rc in (_lib.MOE_EINVAL, _lib.MOE_EWORKSPACE, _lib.MOE_EDEVICE)
    cb = bwd.c()
    rc = lib.moe_backward(C.byref(cb), None, None, None, None, None, None, None, None, None, None,
                          None, None, 0, None, None)
    assert rc != _lib.MOE_OK


def test_noise_step_and_probe_refuse_bad_arguments(lib):
    """moe_noise_step wants an 8-byte aligned word, moe_fma_probe a buffer
    and positive sizes: both refuse on the host, before any device work."""
    assert lib.moe_noise_step(None, None) == _lib.MOE_EINVAL
    buf = (C.c_uint64 * 2)()
    assert lib.moe_noise_step(C.c_void_p(C.addressof(buf) + 4), None) == _lib.MOE_EINVAL
    assert lib.moe_fma_probe(None, 1, 1, 0, None) == _lib.MOE_EINVAL
    assert lib.moe_fma_probe(C.c_void_p(C.addressof(buf)), 0, 1, 0, None) == _lib.MOE_EINVAL
    assert lib.moe_fma_probe(C.c_void_p(C.addressof(buf)), 1, 0, 1, None) == _lib.MOE_EINVAL
    import torch
    if not torch.cuda.is_available():
        assert lib.moe_noise_step(C.c_void_p(C.addressof(buf)), None) == _lib.MOE_EDEVICE


def test_gate_params_seed_word_must_be_aligned(lib):
    """A misaligned seed word in moe_gate_params is an argument error."""
    cfg = M.Config(T=64, d=32, n=8, k=2, f=64, expert_bf16=0)
    c = cfg.c()
    buf = (C.c_byte * 65536)()
    base = C.addressof(buf) + (-C.addressof(buf)) % 256
    fake = C.c_void_p(base)
    gp = _lib.moe_gate_params(W_g=fake, W_noise=fake, seed_dev=C.c_void_p(base + 4))
    ws = C.c_void_p(base)
    rc = lib.moe_gate(C.byref(c), fake, C.byref(gp), fake, fake, fake, None, ws, 0, fake, None)
    assert rc in (_lib.MOE_EINVAL, _lib.MOE_EWORKSPACE)
    need = C.c_size_t(0)
    assert lib.moe_workspace_size(C.byref(c), C.byref(need)) == _lib.MOE_OK
    if need.value <= 65536 - 256:
        rc = lib.moe_gate(C.byref(c), fake, C.byref(gp), fake, fake, fake, None, ws, need.value,
                          fake, None)
        assert rc == _lib.MOE_EINVAL
