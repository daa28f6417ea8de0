"""The C-ABI library: it loads, exports every entry point include/moe.h
declares, and rejects bad arguments on the host before launching anything
(no GPU needed: every call here returns before touching CUDA)."""

import ctypes
import math
import os
import re

import pytest

import routed_swiglu_experts_b200 as rse
from routed_swiglu_experts_b200 import _abi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")

FAKE = 1 << 20          # a 256-aligned fake device address; never dereferenced
FAKE_UNALIGNED = FAKE + 4


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*MOE_API\s+[\w\s\*]*?\b(moe_\w+)\s*\(", text, flags=re.M)))


@pytest.fixture(scope="module")
def lib():
    return _abi.load_library()


def test_header_declares_the_hot_path(lib):
    names = declared_functions()
    for required in ("moe_router_topk", "moe_permute", "moe_grouped_swiglu_ffn", "moe_combine", "moe_forward"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(lib, n), n
    assert set(_abi.EXPORTED) <= set(names)


def test_status_strings(lib):
    s = _abi.status_strings()
    assert s[0] == "MOE_OK" and s[5] == "MOE_ERR_DEVICE_TIMEOUT"
    assert lib.moe_status_string(99) is not None


def mid_cfg(**kw):
    base = dict(hidden=2048, num_experts=64, top_k=6, expert_inter=1408, shared_inter=2816, swiglu_limit=7.0,
                routed_scaling_factor=2.5, renormalize=True)
    base.update(kw)
    return _abi.make_config(**base)


@pytest.mark.parametrize("kw,status", [
    ({}, _abi.MOE_OK),
    ({"hidden": 2044}, _abi.MOE_ERR_INVALID_ARG),
    ({"hidden": 0}, _abi.MOE_ERR_INVALID_ARG),
    ({"expert_inter": 1404}, _abi.MOE_ERR_INVALID_ARG),
    ({"shared_inter": -8}, _abi.MOE_ERR_INVALID_ARG),
    ({"shared_inter": 0}, _abi.MOE_OK),
    ({"num_experts": 0}, _abi.MOE_ERR_INVALID_ARG),
    ({"num_experts": 2048}, _abi.MOE_ERR_UNSUPPORTED),
    ({"top_k": 0}, _abi.MOE_ERR_INVALID_ARG),
    ({"top_k": 65}, _abi.MOE_ERR_INVALID_ARG),          # k > E
    ({"top_k": 17}, _abi.MOE_ERR_UNSUPPORTED),          # above the 16-entry selection arrays
    ({"top_k": 16}, _abi.MOE_OK),
    ({"swiglu_limit": float("nan")}, _abi.MOE_ERR_INVALID_ARG),
    ({"swiglu_limit": 0.0}, _abi.MOE_ERR_INVALID_ARG),
    ({"swiglu_limit": -1.0}, _abi.MOE_ERR_INVALID_ARG),
    ({"swiglu_limit": math.inf}, _abi.MOE_OK),           # no clamp
    ({"routed_scaling_factor": math.inf}, _abi.MOE_ERR_INVALID_ARG),
    ({"expert_format": 7}, _abi.MOE_ERR_INVALID_ARG),
    ({"expert_format": _abi.MOE_W_INT4_G128}, _abi.MOE_OK),
    ({"expert_format": _abi.MOE_W_INT4_G128, "expert_inter": 1416}, _abi.MOE_ERR_UNSUPPORTED),
    ({"expert_format": _abi.MOE_W_INT4_G128, "expert_inter": 2048}, _abi.MOE_OK),
    # int4 experts compute on fp16 operands: |h| <= L^2 must stay finite in fp16
    ({"expert_format": _abi.MOE_W_INT4_G128, "swiglu_limit": math.inf}, _abi.MOE_ERR_UNSUPPORTED),
    ({"expert_format": _abi.MOE_W_INT4_G128, "swiglu_limit": 256.0}, _abi.MOE_ERR_UNSUPPORTED),
    ({"expert_format": _abi.MOE_W_INT4_G128, "swiglu_limit": 255.0}, _abi.MOE_OK),
    ({"swiglu_limit": 1e30}, _abi.MOE_OK),                # bf16 experts: no such bound
    # NVFP4 experts: the same multiples of 128 and the same fp16 bound on h
    ({"expert_format": _abi.MOE_W_NVFP4}, _abi.MOE_OK),
    ({"expert_format": _abi.MOE_W_NVFP4, "expert_inter": 1416}, _abi.MOE_ERR_UNSUPPORTED),
    ({"expert_format": _abi.MOE_W_NVFP4, "hidden": 2056}, _abi.MOE_ERR_UNSUPPORTED),
    ({"expert_format": _abi.MOE_W_NVFP4, "swiglu_limit": 256.0}, _abi.MOE_ERR_UNSUPPORTED),
    ({"expert_format": _abi.MOE_W_NVFP4, "swiglu_limit": 255.0}, _abi.MOE_OK),
    ({"expert_format": 3}, _abi.MOE_ERR_INVALID_ARG),
])
def test_config_validation(lib, kw, status):
    if kw.get("expert_format") in (_abi.MOE_W_INT4_G128, _abi.MOE_W_NVFP4) and "expert_inter" not in kw:
        kw = dict(kw, expert_inter=1536)
    assert _abi.moe_config_validate(mid_cfg(**kw)) == status


def test_workspace_size(lib):
    cfg = mid_cfg()
    n0 = _abi.moe_workspace_size(cfg, 0)
    n1 = _abi.moe_workspace_size(cfg, 4096)
    assert 0 < n0 < n1
    R, H, I = 4096 * 6, 2048, 1408
    assert n1 >= 2 * R * H * 2 + R * I * 2      # x_perm + y_perm + h at least
    # int4 experts gather their rows while converting them: no x_perm region
    c4 = mid_cfg(expert_format=_abi.MOE_W_INT4_G128, expert_inter=2048, hidden=2048)
    R4, I4 = 4096 * 6, 2048
    bf16_like = R4 * H * 2 + R4 * 2 * I4 * 4 + R4 * H * 2 + R4 * max(H, I4) * 2  # with an x_perm region
    assert _abi.moe_workspace_size(c4, 4096) < bf16_like + (64 << 20)
    # NVFP4 experts run the same two kernels with the same scratch: the same
    # workspace as the int4 layer of the same shape
    cf = mid_cfg(expert_format=_abi.MOE_W_NVFP4, expert_inter=2048, hidden=2048)
    for T in (1, 32, 4096):
        assert _abi.moe_workspace_size(cf, T) == _abi.moe_workspace_size(c4, T)
    with pytest.raises(rse.MoEError):
        _abi.moe_workspace_size(cfg, -1)


def _call_forward(lib, cfg, w, x=FAKE, T=16, out=FAKE, ws=FAKE, ws_bytes=None):
    if ws_bytes is None:
        ok = _abi.moe_config_validate(cfg) == _abi.MOE_OK
        ws_bytes = _abi.moe_workspace_size(cfg, max(T, 0)) if ok else 1 << 40
    return lib.moe_forward(ctypes.byref(cfg), ctypes.byref(w), x, T, out, None, None, ws, ws_bytes, None)


def _fake_weights(**kw):
    base = dict(router_w=FAKE, correction_bias=FAKE, w_gate_up=FAKE, w_down=FAKE, shared_w_gate_up=FAKE,
                shared_w_down=FAKE)
    base.update(kw)
    return _abi.moe_weights(*(base.get(n) for n, _ in _abi.moe_weights._fields_))


def test_forward_argument_checks(lib):
    cfg = mid_cfg()
    w = _fake_weights()
    # T == 0 is a no-op that succeeds
    assert _call_forward(lib, cfg, w, T=0) == _abi.MOE_OK
    assert _call_forward(lib, cfg, w, T=-1) == _abi.MOE_ERR_INVALID_ARG
    assert _call_forward(lib, cfg, w, x=None) == _abi.MOE_ERR_INVALID_ARG
    assert _call_forward(lib, cfg, w, x=FAKE_UNALIGNED) == _abi.MOE_ERR_INVALID_ARG
    assert _call_forward(lib, cfg, w, out=None) == _abi.MOE_ERR_INVALID_ARG
    assert _call_forward(lib, cfg, w, ws=None) == _abi.MOE_ERR_WORKSPACE
    assert _call_forward(lib, cfg, w, ws=FAKE + 16) == _abi.MOE_ERR_INVALID_ARG
    small = _abi.moe_workspace_size(cfg, 16) - 1
    assert _call_forward(lib, cfg, w, ws_bytes=small) == _abi.MOE_ERR_WORKSPACE
    assert _call_forward(lib, cfg, _fake_weights(router_w=None)) == _abi.MOE_ERR_INVALID_ARG
    assert _call_forward(lib, cfg, _fake_weights(w_down=None)) == _abi.MOE_ERR_INVALID_ARG
    assert _call_forward(lib, cfg, _fake_weights(shared_w_down=None)) == _abi.MOE_ERR_INVALID_ARG
    assert _call_forward(lib, mid_cfg(shared_inter=0), _fake_weights(shared_w_down=None, shared_w_gate_up=None),
                         T=0) == _abi.MOE_OK
    # int4 experts need their scales
    c4 = mid_cfg(expert_format=_abi.MOE_W_INT4_G128, expert_inter=2048)
    assert _call_forward(lib, c4, _fake_weights()) == _abi.MOE_ERR_INVALID_ARG
    assert _call_forward(lib, c4, _fake_weights(s_gate_up=FAKE, s_down=FAKE), T=0) == _abi.MOE_OK
    # NVFP4 experts need their block scales and their fp32 tensor scales (4-byte aligned)
    cf = mid_cfg(expert_format=_abi.MOE_W_NVFP4, expert_inter=2048)
    scaled = dict(s_gate_up=FAKE, s_down=FAKE)
    assert _call_forward(lib, cf, _fake_weights(**scaled)) == _abi.MOE_ERR_INVALID_ARG
    assert _call_forward(lib, cf, _fake_weights(g_gate_up=FAKE, g_down=FAKE)) == _abi.MOE_ERR_INVALID_ARG
    assert _call_forward(lib, cf, _fake_weights(**scaled, g_gate_up=FAKE)) == _abi.MOE_ERR_INVALID_ARG
    assert _call_forward(lib, cf, _fake_weights(**scaled, g_gate_up=FAKE, g_down=FAKE + 2)) == \
        _abi.MOE_ERR_INVALID_ARG
    assert _call_forward(lib, cf, _fake_weights(**scaled, g_gate_up=FAKE + 4, g_down=FAKE + 8), T=0) == _abi.MOE_OK
    # the tensor scales are ignored for the other formats
    assert _call_forward(lib, c4, _fake_weights(s_gate_up=FAKE, s_down=FAKE, g_down=FAKE + 2), T=0) == _abi.MOE_OK
    # bad configuration is reported first
    assert _call_forward(lib, mid_cfg(top_k=17), w) == _abi.MOE_ERR_UNSUPPORTED


def test_stage_argument_checks(lib):
    cfg = mid_cfg()
    w = _fake_weights()
    ws_bytes = _abi.moe_workspace_size(cfg, 16)
    r = lib.moe_router_topk(ctypes.byref(cfg), ctypes.byref(w), FAKE, 16, None, FAKE, FAKE, ws_bytes, None)
    assert r == _abi.MOE_ERR_INVALID_ARG
    r = lib.moe_router_topk(ctypes.byref(cfg), ctypes.byref(w), FAKE, 0, FAKE, FAKE, FAKE, ws_bytes, None)
    assert r == _abi.MOE_OK
    r = lib.moe_permute(ctypes.byref(cfg), FAKE, FAKE, FAKE, 16, FAKE, None, FAKE, FAKE, FAKE, FAKE, ws_bytes, None)
    assert r == _abi.MOE_ERR_INVALID_ARG
    r = lib.moe_permute(ctypes.byref(cfg), FAKE, FAKE, FAKE, 16, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0, None)
    assert r == _abi.MOE_ERR_WORKSPACE
    # shared input without a shared output
    r = lib.moe_grouped_swiglu_ffn(ctypes.byref(cfg), ctypes.byref(w), FAKE, FAKE, FAKE, 16, FAKE, FAKE, None,
                                   FAKE, ws_bytes, None)
    assert r == _abi.MOE_ERR_INVALID_ARG
    # permute: x_perm NULL means maps only, and x is then not needed
    r = lib.moe_permute(ctypes.byref(cfg), FAKE, FAKE, None, 0, FAKE, FAKE, FAKE, FAKE, None, FAKE, ws_bytes, None)
    assert r == _abi.MOE_OK
    r = lib.moe_permute(ctypes.byref(cfg), FAKE, FAKE, None, 16, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, ws_bytes, None)
    assert r == _abi.MOE_ERR_INVALID_ARG
    # gathered FFN: x, src, offsets and y_perm are required; shared_out needs a shared expert
    def ffn_gather(x=FAKE, T=16, src=FAKE, offs=FAKE, w_perm=FAKE, y=FAKE, sh=FAKE, c=cfg, ww=w, nbytes=ws_bytes):
        return lib.moe_grouped_swiglu_ffn_gather(ctypes.byref(c), ctypes.byref(ww), x, T, src, offs, w_perm, y, sh,
                                                 FAKE, nbytes, None)
    assert ffn_gather(T=0) == _abi.MOE_OK
    assert ffn_gather(x=None) == _abi.MOE_ERR_INVALID_ARG
    assert ffn_gather(src=None) == _abi.MOE_ERR_INVALID_ARG
    assert ffn_gather(src=FAKE_UNALIGNED) == _abi.MOE_ERR_INVALID_ARG
    assert ffn_gather(offs=None) == _abi.MOE_ERR_INVALID_ARG
    assert ffn_gather(y=None) == _abi.MOE_ERR_INVALID_ARG
    assert ffn_gather(w_perm=FAKE_UNALIGNED) == _abi.MOE_ERR_INVALID_ARG
    assert ffn_gather(c=mid_cfg(shared_inter=0)) == _abi.MOE_ERR_INVALID_ARG
    assert ffn_gather(ww=_fake_weights(shared_w_gate_up=None)) == _abi.MOE_ERR_INVALID_ARG
    assert ffn_gather(ww=_fake_weights(w_gate_up=None)) == _abi.MOE_ERR_INVALID_ARG
    assert ffn_gather(nbytes=ws_bytes - 1) == _abi.MOE_ERR_WORKSPACE
    assert ffn_gather(c=mid_cfg(shared_inter=0), sh=None, T=0) == _abi.MOE_OK
    r = lib.moe_combine(ctypes.byref(cfg), FAKE, FAKE, None, None, 16, FAKE_UNALIGNED, None)
    assert r == _abi.MOE_ERR_INVALID_ARG
    r = lib.moe_combine(ctypes.byref(cfg), FAKE, FAKE, None, None, 0, FAKE, None)
    assert r == _abi.MOE_OK
    code = ctypes.c_int32(0)
    assert lib.moe_read_device_error(None, None, ctypes.byref(code)) == _abi.MOE_ERR_INVALID_ARG


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(RuntimeError, match="no CPU fallback"):
        _load_fresh(str(tmp_path / "nope.so"))


def _load_fresh(path):
    saved = _abi._lib
    _abi._lib = None
    try:
        return _abi.load_library(path)
    finally:
        _abi._lib = saved


def test_selftest_timeout_argument_checks(lib):
    """The timeout test hook validates its scratch before touching the GPU."""
    n = _abi.MOE_SELFTEST_SCRATCH_BYTES
    assert lib.moe_selftest_device_timeout(None, n, None) == _abi.MOE_ERR_WORKSPACE
    assert lib.moe_selftest_device_timeout(FAKE, n - 1, None) == _abi.MOE_ERR_WORKSPACE
    assert lib.moe_selftest_device_timeout(FAKE + 16, n, None) == _abi.MOE_ERR_INVALID_ARG


def test_pair_selftest_argument_checks(lib):
    """The CTA-pair timeout hook validates its scratch and kernel selector
    before touching the GPU."""
    n = _abi.MOE_SELFTEST_SCRATCH_BYTES
    assert lib.moe_selftest_pair_timeout(None, n, _abi.MOE_SELFTEST_PAIR_BF16, None) == _abi.MOE_ERR_WORKSPACE
    assert lib.moe_selftest_pair_timeout(FAKE, n - 1, _abi.MOE_SELFTEST_PAIR_BF16, None) == _abi.MOE_ERR_WORKSPACE
    assert lib.moe_selftest_pair_timeout(FAKE + 16, n, _abi.MOE_SELFTEST_PAIR_INT4, None) == _abi.MOE_ERR_INVALID_ARG
    assert lib.moe_selftest_pair_timeout(FAKE, n, 2, None) == _abi.MOE_ERR_INVALID_ARG
    assert lib.moe_selftest_pair_timeout(FAKE, n, -1, None) == _abi.MOE_ERR_INVALID_ARG


def _call_ep(lib, cfg, w, b, e, T=16, x=FAKE, out=FAKE, ws=FAKE):
    ok = _abi.moe_config_validate(cfg) == _abi.MOE_OK
    nbytes = _abi.moe_workspace_size(cfg, max(T, 0)) if ok else 1 << 40
    return lib.moe_forward_ep(ctypes.byref(cfg), ctypes.byref(w), b, e, x, T, out, None, None, ws, nbytes, None)


def test_forward_ep_argument_checks(lib):
    """The expert range must lie in [0, E]; an empty range needs no routed
    weights; everything is validated before any launch."""
    cfg = mid_cfg()
    w = _fake_weights()
    E = cfg.num_experts
    assert _call_ep(lib, cfg, w, 0, E, T=0) == _abi.MOE_OK
    assert _call_ep(lib, cfg, w, -1, 4) == _abi.MOE_ERR_INVALID_ARG
    assert _call_ep(lib, cfg, w, 0, E + 1) == _abi.MOE_ERR_INVALID_ARG
    assert _call_ep(lib, cfg, w, 5, 4) == _abi.MOE_ERR_INVALID_ARG
    assert _call_ep(lib, cfg, w, 0, E, out=None) == _abi.MOE_ERR_INVALID_ARG
    assert _call_ep(lib, cfg, w, 0, E, ws=None) == _abi.MOE_ERR_WORKSPACE
    # local experts need weights, an empty range does not
    assert _call_ep(lib, cfg, _fake_weights(w_gate_up=None), 0, 4) == _abi.MOE_ERR_INVALID_ARG
    assert _call_ep(lib, cfg, _fake_weights(w_gate_up=None, w_down=None), 4, 4, T=0) == _abi.MOE_OK


def test_header_is_plain_c_and_matches_the_binding(tmp_path):
    """include/moe.h compiles as C99 on its own (no CUDA headers), and the
    struct layouts, enum values and limits it declares are the ones the
    ctypes binding mirrors."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    structs = {"moe_config": _abi.moe_config, "moe_weights": _abi.moe_weights}
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "moe.h"', "int main(void) {"]
    for sname, ct in structs.items():
        lines.append(f'  printf("sizeof {sname} %zu\\n", sizeof({sname}));')
        for f, _ in ct._fields_:
            lines.append(f'  printf("offset {sname}.{f} %zu\\n", offsetof({sname}, {f}));')
    consts = ["MOE_OK", "MOE_ERR_INVALID_ARG", "MOE_ERR_UNSUPPORTED", "MOE_ERR_WORKSPACE", "MOE_ERR_CUDA",
              "MOE_ERR_DEVICE_TIMEOUT", "MOE_W_BF16", "MOE_W_INT4_G128", "MOE_W_NVFP4", "MOE_MAX_TOP_K",
              "MOE_MAX_EXPERTS", "MOE_NO_ALLOC_MAX_ROWS", "MOE_SELFTEST_SCRATCH_BYTES", "MOE_SELFTEST_PAIR_BF16",
              "MOE_SELFTEST_PAIR_INT4"]
    for c in consts:
        lines.append(f'  printf("const {c} %ld\\n", (long)({c}));')
    lines.append('  printf("const MOE_INT4_MAX_SWIGLU_LIMIT %.1f\\n", (double)MOE_INT4_MAX_SWIGLU_LIMIT);')
    lines += ["  return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                    str(src), "-o", str(exe)], check=True, capture_output=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split("\n")
    got = {" ".join(l.split()[:2]): l.split()[2] for l in out if l}
    for sname, ct in structs.items():
        assert int(got[f"sizeof {sname}"]) == ctypes.sizeof(ct), sname
        for f, _ in ct._fields_:
            assert int(got[f"offset {sname}.{f}"]) == getattr(ct, f).offset, f"{sname}.{f}"
    for c in consts:
        assert int(got[f"const {c}"]) == getattr(_abi, c), c
    assert float(got["const MOE_INT4_MAX_SWIGLU_LIMIT"]) == _abi.MOE_INT4_MAX_SWIGLU_LIMIT
