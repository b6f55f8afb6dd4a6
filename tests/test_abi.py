"""The C-ABI library loads and exports every symbol include/fathom.h
declares; host-only entry points and argument checks that return before
any CUDA call behave as documented (no GPU needed)."""
import ctypes
import os
import re

import pytest

from long_context_decode_bit_b200 import build, fathom

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fathom.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return fathom.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fathom_\w+)\s*\(", text)))


def test_header_and_binding_agree():
    assert declared_functions() == sorted(fathom.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    raw = ctypes.CDLL(fathom.LIB_PATH)
    for name in declared_functions():
        assert hasattr(raw, name), name


def test_header_is_plain_c_and_links(lib, tmp_path):
    """A C11 program (no C++, -Wall -Wextra -pedantic -Werror) includes the
    header, takes the address of every declared function and links against
    the library; it then runs the host-only calls (no GPU needed)."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    names = declared_functions()
    src = ["#include \"fathom.h\"", "#include <stdio.h>", "int main(void) {",
           "    void (*table[])(void) = {"]
    src += [f"        (void (*)(void)){n}," for n in names]
    src += ["    };",
            "    printf(\"%d %u %s %lld\\n\", fathom_version(), (unsigned)(sizeof table / sizeof table[0]),",
            "           fathom_status_string(FATHOM_ERR_OVERFLOW), (long long)fathom_nb_stride(1025));",
            "    return table[0] == 0;", "}"]
    c_file = tmp_path / "abi.c"
    c_file.write_text("\n".join(src) + "\n")
    exe = tmp_path / "abi"
    libdir = os.path.dirname(fathom.LIB_PATH)
    subprocess.run([cc, "-std=c11", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.join(ROOT, "include"),
                    str(c_file), "-L", libdir, "-lfathom", f"-Wl,-rpath,{libdir}", "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split()
    assert out[0] == "10000" and int(out[1]) == len(names) and out[-1] == "32"


def test_host_only_entry_points(lib):
    assert lib.fathom_version() == 10000
    assert lib.fathom_status_string(0) == b"ok"
    assert b"exact" in lib.fathom_status_string(-6)
    assert lib.fathom_last_cuda_error() == 0
    assert lib.fathom_nb_stride(1) == 16
    assert lib.fathom_nb_stride(1024) == 16
    assert lib.fathom_nb_stride(1025) == 32
    assert lib.fathom_nb_stride(2 ** 20) == 16384
    assert lib.fathom_topk_workspace_bytes(288, 4, 2 ** 20, 512) == 0
    assert lib.fathom_scan_cand_bytes(0, 4, 100, 1) == 0
    assert lib.fathom_scan_cand_bytes(1, 4, 100, 101) == 0   # k > n
    small = lib.fathom_scan_cand_bytes(2, 4, 1000, 64)        # no sample: cap = n
    assert small >= 2 * 4 * (16 + 1000 * 8)
    big = lib.fathom_scan_cand_bytes(288, 4, 2 ** 20, 512)
    # 1152 heads x (16384 survivor slots of 8 B, i.e. 8x the ~2048 expected,
    # spread over the tiles + one count per tile + 16384 sample scores of 4 B:
    # 1 tile in 64 is sampled)
    per_head = 16384 * 8 + 16384 * 4
    assert 1152 * per_head <= big < 1152 * (per_head + 4096 + 16) + 4 * 256
    # calibration scratch: two fp64 sums per (group, channel), plus the
    # fp64 D x D sums with the covariance
    assert lib.fathom_calibrate_workspace_bytes(0, 128, 0) == 0
    assert lib.fathom_calibrate_workspace_bytes(8, 100, 0) == 0              # unsupported D
    assert lib.fathom_calibrate_workspace_bytes(8, 128, 0) == 2 * 8 * 128 * 8
    assert lib.fathom_calibrate_workspace_bytes(8, 128, 1) == 2 * 8 * 128 * 8 + 8 * 128 * 128 * 8
    # attention over the union: (max, weight sum) per (group, 256-row chunk, head) + the chunk outputs
    assert lib.fathom_union_attention_workspace_bytes(288, 4, 128, 2048) == 2 * 288 * 8 * 4 * 4 + 288 * 8 * 4 * 128 * 4
    assert lib.fathom_union_attention_workspace_bytes(1, 4, 128, 0) == 0
    assert lib.fathom_union_attention_workspace_bytes(1, 9, 128, 64) == 0


def test_rejections_before_any_cuda_call(lib):
    n = None
    # unsupported D and G, bad dtype, bad mode, bad budget: rejected on sizes alone
    assert lib.fathom_pack(n, 0, 1, 64, 48, 64 * 48, 48, n, n, 16, n) == fathom.ERR_UNSUPPORTED
    assert lib.fathom_pack(n, 7, 1, 64, 128, 64 * 128, 128, n, n, 16, n) == fathom.ERR_INVALID_ARG
    assert lib.fathom_pack(n, 0, 0, 64, 128, 0, 128, n, n, 16, n) == fathom.OK        # nothing to do
    assert lib.fathom_plan(n, n, 4, 9, 128, n, 48, n, n, n, n, n) == fathom.ERR_UNSUPPORTED
    assert lib.fathom_plan(n, n, 4, 4, 128, n, 513, n, n, n, n, n) == fathom.ERR_INVALID_ARG
    assert lib.fathom_plan(n, n, 4, 4, 128, n, -1, n, n, n, n, n) == fathom.ERR_INVALID_ARG
    assert lib.fathom_plan_fixed(n, 4, 4, 128, 129, 4, n, n, n, n) == fathom.ERR_INVALID_ARG   # r > D
    assert lib.fathom_plan_fixed(n, 4, 4, 128, 32, 0, n, n, n, n) == fathom.ERR_INVALID_ARG    # bits = 0
    assert lib.fathom_plan_fixed(n, 4, 4, 128, 32, 5, n, n, n, n) == fathom.ERR_INVALID_ARG    # bits > 4
    assert lib.fathom_scan(n, n, 1, 128, 100, 2, n, n, n, 4, 5, n, n, 0, 1, n) == fathom.ERR_INVALID_ARG
    assert lib.fathom_scan(n, n, 1, 100, 100, 2, n, n, n, 4, 0, n, n, 0, 1, n) == fathom.ERR_UNSUPPORTED
    assert lib.fathom_topk(n, n, 1, 4, 100, 5, n, n, n, n, 0, n) == fathom.ERR_INVALID_ARG   # neither input
    assert lib.fathom_topk(n, n, 1, 0, 100, 5, n, n, n, n, 0, n) == fathom.ERR_UNSUPPORTED   # G = 0
    assert lib.fathom_calibrate(n, 3, 1, 64, 128, 64 * 128, 128, n, n, n, n, 0, n) == fathom.ERR_INVALID_ARG
    assert lib.fathom_calibrate(n, 0, 1, 64, 48, 64 * 48, 48, n, n, n, n, 0, n) == fathom.ERR_UNSUPPORTED
    assert lib.fathom_calibrate(n, 0, 0, 64, 128, 0, 128, n, n, n, n, 0, n) == fathom.OK     # nothing to do
    fake = ctypes.c_void_p(256)   # never dereferenced: the size check comes first
    assert lib.fathom_calibrate(fake, 0, 2, 64, 128, 64 * 128, 128, n, fake, n, fake, 100, n) == fathom.ERR_WORKSPACE
    assert lib.fathom_calibrate(fake, 0, 2, 64, 128, 64 * 128, 128, n, n, n, fake, 1 << 20, n) == fathom.ERR_INVALID_ARG
    assert lib.fathom_scan_nibbles(n, n, 1, 128, 100, 2, n, n, n, 4, 5, n, n, 0, 1, n) == fathom.ERR_INVALID_ARG
    assert lib.fathom_scan_nibbles(n, n, 1, 100, 100, 2, n, n, n, 4, 0, n, n, 0, 1, n) == fathom.ERR_UNSUPPORTED
    assert lib.fathom_nibbles_from_planes(n, 1, 48, 100, 2, n, n) == fathom.ERR_UNSUPPORTED
    assert lib.fathom_nibbles_from_planes(n, 1, 128, 1000, 15, n, n) == fathom.ERR_INVALID_ARG   # stride < nb
    assert lib.fathom_layer_budgets_workspace_bytes(288, 128) == 288 * 512 * 8 + 288 * 128 * 4
    assert lib.fathom_layer_budgets(n, n, 10, 4, 128, 3, 100, n, n, 0, n) == fathom.ERR_INVALID_ARG   # 3 does not divide 10
    assert lib.fathom_layer_budgets(n, n, 10, 4, 128, 0, 100, n, n, 0, n) == fathom.ERR_INVALID_ARG   # no layer
    assert lib.fathom_layer_budgets(n, n, 10, 4, 100, 5, 100, n, n, 0, n) == fathom.ERR_UNSUPPORTED
    assert lib.fathom_layer_budgets(fake, fake, 10, 4, 128, 5, 100, fake, fake, 64, n) == fathom.ERR_WORKSPACE
    # keys rotated inside pack: the checks of fathom_pack, plus U's alignment
    assert lib.fathom_pack_rotated(n, 0, 1, 64, 48, 64 * 48, 48, n, n, n, 16, n) == fathom.ERR_UNSUPPORTED
    assert lib.fathom_pack_rotated(n, 7, 1, 64, 128, 64 * 128, 128, n, n, n, 16, n) == fathom.ERR_INVALID_ARG
    assert lib.fathom_pack_rotated(n, 0, 0, 64, 128, 0, 128, n, n, n, 16, n) == fathom.OK      # nothing to do
    assert lib.fathom_pack_rotated(n, 0, 1, 1000, 128, 1000 * 128, 128, n, n, n, 15, n) == fathom.ERR_INVALID_ARG
    assert lib.fathom_pack_rotated(fake, 0, 1, 64, 128, 64 * 128, 128, ctypes.c_void_p(258), fake, fake, 16,
                                   n) == fathom.ERR_UNSUPPORTED                                 # U misaligned
    # the token-major comparator: the checks of fathom_scan and of the nibble store
    assert lib.fathom_scan_nibbles_tm(n, n, 1, 128, 100, 2, n, n, n, 4, 5, n, n, 0, 1, n) == fathom.ERR_INVALID_ARG
    assert lib.fathom_scan_nibbles_tm(n, n, 1, 100, 100, 2, n, n, n, 4, 0, n, n, 0, 1, n) == fathom.ERR_UNSUPPORTED
    assert lib.fathom_nibbles_tm_from_planes(n, 1, 48, 100, 2, n, n) == fathom.ERR_UNSUPPORTED
    assert lib.fathom_nibbles_tm_from_planes(n, 1, 128, 1000, 15, n, n) == fathom.ERR_INVALID_ARG   # stride < nb
    assert lib.fathom_nibbles_tm_from_planes(fake, 1, 128, 1000, 16, ctypes.c_void_p(264), n) == fathom.ERR_UNSUPPORTED
    ua = lib.fathom_union_attention
    assert ua(n, n, 0, 1, 64, 128, 64 * 128, 128, n, 4, n, n, 0, 1.0, n, n, 0, n) == fathom.ERR_INVALID_ARG   # M = 0
    assert ua(n, n, 2, 1, 64, 128, 64 * 128, 128, n, 4, n, n, 8, 1.0, n, n, 0, n) == fathom.ERR_INVALID_ARG   # dtype
    assert ua(n, n, 0, 1, 64, 128, 64 * 128, 128, n, 9, n, n, 8, 1.0, n, n, 0, n) == fathom.ERR_UNSUPPORTED   # G = 9
    assert ua(n, n, 0, 1, 64, 128, 64 * 128, 128, n, 4, n, n, 8, float("nan"), n, n, 0, n) == fathom.ERR_INVALID_ARG
    assert ua(fake, fake, 0, 2, 64, 128, 64 * 128, 128, fake, 4, fake, fake, 8, 1.0, fake, fake, 64, n) == \
        fathom.ERR_WORKSPACE


def test_missing_library_fails_loudly(tmp_path):
    saved = fathom._lib
    fathom._lib = None
    try:
        with pytest.raises(FileNotFoundError):
            fathom.load(str(tmp_path / "nope.so"))
    finally:
        fathom._lib = saved


def test_step_repair_raises_on_device_fault_statuses(lib):
    """Step.repair's host decision (no GPU): a TIMEOUT or BOUNDS status in
    union_count raises instead of starting a dense rerun, and a step whose
    groups all proved exact needs no repair."""
    import torch
    H, D, G, n, k = 3, 128, 4, 4096, 64
    planes = torch.zeros((H, D, 4, fathom.nb_stride(n)), dtype=torch.int64)
    scales = torch.zeros((H, D, fathom.nb_stride(n)), dtype=torch.int16)
    sigma2 = torch.ones((H, D))
    st = fathom.Step(planes, scales, n, sigma2, G, k)
    q = torch.zeros((H, G, D))
    st.topk_out[2].copy_(torch.tensor([5, 7, 9], dtype=torch.int32))
    assert st.repair(q) == 0
    for status in (fathom.ERR_TIMEOUT, fathom.ERR_BOUNDS):
        st.topk_out[2].copy_(torch.tensor([status] * H, dtype=torch.int32))
        with pytest.raises(fathom.FathomError) as e:
            st.repair(q)
        assert e.value.status == status
    assert lib.fathom_status_string(fathom.ERR_BOUNDS).decode() != "unknown status"
