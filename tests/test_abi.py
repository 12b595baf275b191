"""Host-only checks of the C ABI: the library loads, exports every entry point the
header declares, sizes workspaces, and rejects bad arguments before launching
anything (none of these calls touches a GPU)."""
import ctypes
import os
import re

import pytest

from rope_attention_fwd_b200 import binding as rb

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "rope_attn.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(rope_attn_\w+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    names = declared_functions()
    assert len(names) >= 9
    lib = rb.lib()
    for name in names:
        assert hasattr(lib, name), name


def test_status_strings():
    lib = rb.lib()
    for code in range(6):
        assert lib.rope_attn_status_string(code)
    assert lib.rope_attn_status_string(0) == b"ok"


def test_size_limits_are_inclusive():
    """The largest problems inside the limits still get a workspace size, computed without
    overflow (it exceeds the bytes of the rotated Q~ and K~ alone)."""
    for B, H, n, d, dt in [(1 << 8, 1 << 8, 1 << 16, 64, rb.RA_BF16),
                           (1, 1, 1 << 30, 128, rb.RA_BF16), (1, 65535, 1 << 16, 64, rb.RA_F32)]:
        p = rb.problem(B, H, n, d, dt, True, 1e4)
        elems = B * H * n * d
        assert elems <= 1 << 38
        assert rb.rope_attn_workspace_bytes(p) > 2 * elems * (2 if dt == rb.RA_BF16 else 4)


def test_workspace_bytes():
    elems = 2 * 32 * 8192 * 128
    p = rb.problem(2, 32, 8192, 128, rb.RA_BF16, True, 1e4)
    nb = rb.rope_attn_workspace_bytes(p)
    # the two rotated 16-bit tensors dominate
    assert 2 * elems * 2 <= nb < 2 * elems * 2 * 1.1
    assert nb % 1024 == 0


@pytest.mark.parametrize("bad", [
    dict(B=0), dict(H=0), dict(n=0), dict(d=3), dict(d=0), dict(dtype=7), dict(causal=2),
    dict(base=0.0), dict(base=-1.0), dict(base=float("nan")),
])
def test_invalid_problem_has_no_workspace(bad):
    args = dict(B=1, H=1, n=16, d=64, dtype=rb.RA_F32, causal=0, base=1e4)
    args.update(bad)
    p = rb.RaProblem(args["B"], args["H"], args["n"], args["d"], args["dtype"], args["causal"],
                     args["base"])
    assert rb.rope_attn_workspace_bytes(p) == 0


@pytest.mark.parametrize("bad, code", [
    (dict(d=96, dtype=rb.RA_BF16), 2), (dict(d=256), 2), (dict(d=32, dtype=rb.RA_BF16), 2),
    # sizes whose products would overflow, or that no device holds
    (dict(B=1 << 32, H=1 << 32), 2), (dict(B=1 << 31), 2), (dict(n=(1 << 30) + 1), 2),
    (dict(B=1 << 15, H=1 << 15, n=1 << 30), 2), (dict(B=1 << 20, H=1 << 10, n=1 << 12), 2),
    (dict(H=65536, n=64), 2),
])
def test_unsupported_problem(bad, code):
    args = dict(B=1, H=1, n=16, d=64, dtype=rb.RA_F32, causal=0, base=1e4)
    args.update(bad)
    p = rb.RaProblem(args["B"], args["H"], args["n"], args["d"], args["dtype"], args["causal"],
                     args["base"])
    assert rb.rope_attn_workspace_bytes(p) == 0
    lib = rb.lib()
    null = ctypes.c_void_p(0)
    r = lib.rope_attn_fwd(ctypes.byref(p), null, null, null, null, null, null, null, 0, null)
    assert r == code


def test_null_pointers_rejected_before_launch():
    lib = rb.lib()
    p = rb.problem(1, 1, 16, 64, rb.RA_F32, False, 1e4)
    null = ctypes.c_void_p(0)
    fake = ctypes.c_void_p(4096)        # aligned, never dereferenced: validation fails first
    assert lib.rope_attn_fwd(ctypes.byref(p), null, fake, fake, fake, fake, fake, fake,
                             1 << 20, null) == 1
    assert lib.rope_attn_loss(ctypes.byref(p), fake, null, fake, fake, fake, 1 << 20, null) == 1
    assert lib.rope_attn_bwd(ctypes.byref(p), fake, fake, fake, fake, fake, fake, fake,
                             fake, fake, null, fake, fake, 1 << 20, null) == 1
    misaligned = ctypes.c_void_p(4096 + 8)
    assert lib.rope_attn_fwd(ctypes.byref(p), misaligned, fake, fake, fake, fake, fake, fake,
                             1 << 20, null) == 1


def test_workspace_checks_before_launch():
    """The forward needs the leading part of the layout (rope_attn_fwd_workspace_bytes);
    one byte less, a misaligned or a null workspace is rejected before any launch."""
    lib = rb.lib()
    p = rb.problem(1, 1, 16, 64, rb.RA_F32, False, 1e4)
    fake = ctypes.c_void_p(4096)
    need = rb.lib().rope_attn_fwd_workspace_bytes(ctypes.byref(p))
    assert 0 < need <= rb.rope_attn_workspace_bytes(p)
    assert lib.rope_attn_fwd(ctypes.byref(p), fake, fake, fake, fake, fake, fake, fake,
                             need - 1, None) == 3
    assert lib.rope_attn_fwd(ctypes.byref(p), fake, fake, fake, fake, fake, fake,
                             ctypes.c_void_p(4096 + 16), need, None) == 3
    assert lib.rope_attn_fwd(ctypes.byref(p), fake, fake, fake, fake, fake, fake, None,
                             need, None) == 3


def test_kernel_names():
    lib = rb.lib()
    names = [lib.rope_attn_kernel_name(i).decode() for i in range(18)]
    assert {"fwd_sm100", "bwd_dkdv_sm100", "bwd_dq_sm100", "dalpha_final", "proj_gemm",
            "proj_dw_gemm", "proj_dx_gemm", "merge_heads", "spectrum", "alpha_adam"} <= set(names)
    assert "unknown" not in names and len(set(names)) == 18
    assert lib.rope_attn_kernel_name(18) == b"unknown"


def test_fixed_bands_and_reserved_are_validated():
    """fixed_bands must lie in 0..d/2 and reserved must be 0 (checked before any launch)."""
    lib = rb.lib()
    for fb, ok in ((0, True), (64, True), (65, False), (-1, False)):
        p = rb.problem(1, 1, 256, 128, rb.RA_BF16, True, 1e4, fixed_bands=fb)
        assert (rb.rope_attn_workspace_bytes(p) > 0) == ok, fb
    p = rb.problem(1, 1, 256, 128, rb.RA_BF16, True, 1e4)
    p.reserved = 1
    assert lib.rope_attn_workspace_bytes(ctypes.byref(p)) == 0


def test_alpha_adam_rejects_bad_arguments():
    """Invalid optimiser arguments return RA_ERR_INVALID_ARG before any launch."""
    lib = rb.lib()
    buf = ctypes.c_void_p(256)  # never dereferenced: validation fails first
    for kw in (dict(step=0), dict(beta1=1.0), dict(eps=0.0), dict(lr=float("nan"))):
        args = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, clip_norm=1.0, step=1)
        args.update(kw)
        opt = rb.RaAdam(args["lr"], args["beta1"], args["beta2"], args["eps"], args["clip_norm"],
                        args["step"])
        assert lib.rope_attn_alpha_adam(ctypes.byref(opt), 64, buf, buf, buf, buf, None) == 1, kw
    opt = rb.RaAdam(1e-3, 0.9, 0.999, 1e-8, 1.0, 1)
    assert lib.rope_attn_alpha_adam(ctypes.byref(opt), 0, buf, buf, buf, buf, None) == 1


def test_projection_validation_before_any_call():
    """The projection entry points reject bad sizes, pointers and workspaces before they
    launch anything."""
    lib = rb.lib()
    fake = ctypes.c_void_p(4096)
    p = rb.problem(2, 4, 64, 64, rb.RA_BF16, True, 1e4)
    need = rb.rope_attn_proj_workspace_bytes(p)
    # the error word region and three merged [B n, H d] gradients
    assert need == 1024 + 3 * 2 * 64 * 4 * 64 * 2
    # d_model out of range, a null or misaligned operand, a workspace too small
    assert lib.rope_attn_proj_fwd(ctypes.byref(p), 0, *[fake] * 7, fake, 1024, None) == 1
    assert lib.rope_attn_proj_fwd(ctypes.byref(p), 256, None, *[fake] * 6, fake, 1024,
                                  None) == 1
    assert lib.rope_attn_proj_fwd(ctypes.byref(p), 256, ctypes.c_void_p(4096 + 8), *[fake] * 6,
                                  fake, 1024, None) == 1
    assert lib.rope_attn_proj_fwd(ctypes.byref(p), 256, *[fake] * 7, fake, 1023, None) == 3
    # bf16 needs d_model a multiple of 8 (16-byte tensor-map rows)
    assert lib.rope_attn_proj_fwd(ctypes.byref(p), 100, *[fake] * 7, fake, 1024, None) == 2
    # backward: workspace too small or misaligned, then a head row that is not whole
    # 16-byte vectors (d = 2 in fp32) is unsupported
    assert lib.rope_attn_proj_bwd(ctypes.byref(p), 256, *[fake] * 11, fake, need - 1, None) == 3
    assert lib.rope_attn_proj_bwd(ctypes.byref(p), 256, *[fake] * 11,
                                  ctypes.c_void_p(4096 + 8), need, None) == 3
    p2 = rb.problem(1, 1, 8, 2, rb.RA_F32, False, 1e4)
    need2 = rb.rope_attn_proj_workspace_bytes(p2)
    assert lib.rope_attn_proj_bwd(ctypes.byref(p2), 16, *[fake] * 11, fake, need2, None) == 2
    # sizes whose products would overflow get no workspace and are refused
    for B, H, n in [(1 << 40, 1, 1 << 30), (1, 1 << 40, 64), (1 << 20, 1 << 10, 1 << 10),
                    (1 << 15, 1 << 14, 1 << 15)]:
        big = rb.problem(B, H, n, 64, rb.RA_BF16, False, 1e4)
        assert rb.rope_attn_proj_workspace_bytes(big) == 0
        assert lib.rope_attn_proj_fwd(ctypes.byref(big), 256, *[fake] * 7, fake, 1 << 40,
                                      None) == 2


def test_spectrum_validation_before_any_call():
    """The spectrum diagnostic sizes its O(n^2) scratch, caps n and rejects bad pointers and
    workspaces before any launch."""
    lib = rb.lib()
    fake = ctypes.c_void_p(4096)
    p = rb.problem(1, 2, 96, 64, rb.RA_BF16, True, 1e4)
    need = rb.rope_attn_spectrum_workspace_bytes(p)
    assert need >= 2 * 96 * 96 * 4 + 32 * (2 * 96 - 1) * 16
    too_long = rb.problem(1, 1, 32769, 64, rb.RA_BF16, True, 1e4)
    assert rb.rope_attn_spectrum_workspace_bytes(too_long) == 0
    assert rb.rope_attn_spectrum_workspace_bytes(rb.problem(1, 1, 32768, 64, rb.RA_BF16,
                                                            True, 1e4)) > 0
    # q, k, v, o, lse, dO, alpha, g, dalpha, then the workspace
    assert lib.rope_attn_spectrum(ctypes.byref(too_long), *[fake] * 9, fake, 1 << 40,
                                  None) == 1
    assert lib.rope_attn_spectrum(ctypes.byref(p), *[fake] * 7, None, fake, fake, need,
                                  None) == 1
    assert lib.rope_attn_spectrum(ctypes.byref(p), *[fake] * 9, fake, need - 1, None) == 3
    assert lib.rope_attn_spectrum(ctypes.byref(p), *[fake] * 9, ctypes.c_void_p(4096 + 16),
                                  need, None) == 3
    # B and H large enough to overflow their product are refused
    for B, H in [(1 << 32, 1 << 32), (1 << 31, 1), (1 << 16, 1 << 16)]:
        big = rb.problem(B, H, 96, 64, rb.RA_BF16, True, 1e4)
        assert rb.rope_attn_spectrum_workspace_bytes(big) == 0
        assert lib.rope_attn_spectrum(ctypes.byref(big), *[fake] * 9, fake, 1 << 40, None) == 1


def test_header_is_plain_c_and_links(tmp_path):
    """include/rope_attn.h compiles as strict C99 in a C client that links the library and
    drives its host-side checks (no GPU call)."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    libdir = os.path.dirname(rb.LIB_PATH)
    exe = str(tmp_path / "abi_check")
    src = os.path.join(ROOT, "tests", "c_abi", "abi_check.c")
    r = subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                        "-I", os.path.join(ROOT, "include"), src, "-L", libdir, "-lrope_attn",
                        f"-Wl,-rpath,{libdir}", "-o", exe], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "c abi ok" in r.stdout
