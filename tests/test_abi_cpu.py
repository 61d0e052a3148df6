"""The C-ABI library on a machine without a GPU: it builds, loads, exports
every function include/eva_vq.h declares, and rejects bad arguments on the
host before any device work."""
import ctypes
import os
import re
import subprocess

import pytest

from vector_quantized_weight_b200 import build, eva_vq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "eva_vq.h")


def declared_functions():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"EVA_API\s+[\w\s\*]*?\b(eva_\w+)\s*\(", src)))


def test_header_declares_the_binding_functions():
    assert declared_functions() == sorted(eva_vq.ABI_FUNCTIONS)


def test_library_exports_every_declared_symbol():
    lib = eva_vq.load()
    out = subprocess.run(["nm", "-D", "--defined-only", build.LIB], capture_output=True, text=True,
                         check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    for fn in declared_functions():
        assert fn in exported, fn
        assert getattr(lib, fn) is not None
    # nothing beyond the ABI leaks out of the library
    assert exported == set(declared_functions())


def test_status_strings():
    for s in range(7):
        assert eva_vq.eva_vq_status_string(s)
    assert eva_vq.eva_vq_status_string(99) == "unknown status"


def _desc(**kw):
    base = dict(N=256, K=512, d=4, index_bits=8, codebook_rows=0, residual_group=0,
                hadamard_block=0, max_batch=1, out_dtype=0, path=0)
    base.update(kw)
    return eva_vq.eva_vq_desc(*[base[f] for f, _ in eva_vq.eva_vq_desc._fields_])


def _create(desc, wc=0x1000, wi=0x2000, signs=None, alpha=None, hsign=None):
    lib = eva_vq.load()
    h = ctypes.c_void_p()
    return lib.eva_vq_linear_create(ctypes.byref(h), ctypes.byref(desc), wc, wi, signs, alpha, hsign, None)


@pytest.mark.parametrize("kw,expect", [
    (dict(d=3), eva_vq.EVA_ERR_UNSUPPORTED),
    (dict(index_bits=6), eva_vq.EVA_ERR_UNSUPPORTED),
    (dict(index_bits=4, path=2), eva_vq.EVA_ERR_UNSUPPORTED),   # 4-bit: the lookup path only
    (dict(path=2, residual_group=128, codebook_rows=16), eva_vq.EVA_ERR_UNSUPPORTED),  # dequantize: residual and
    (dict(path=2, hadamard_block=128, codebook_rows=16), eva_vq.EVA_ERR_UNSUPPORTED),  # rotation need one codebook
    (dict(index_bits=4, K=516), eva_vq.EVA_ERR_INVALID_ARG),
    (dict(N=0), eva_vq.EVA_ERR_INVALID_ARG),
    (dict(K=510), eva_vq.EVA_ERR_INVALID_ARG),
    (dict(codebook_rows=100), eva_vq.EVA_ERR_INVALID_ARG),
    (dict(codebook_rows=48), eva_vq.EVA_ERR_INVALID_ARG),     # does not divide N=256
    (dict(residual_group=64), eva_vq.EVA_ERR_UNSUPPORTED),
    (dict(hadamard_block=384), eva_vq.EVA_ERR_INVALID_ARG),
    (dict(hadamard_block=1024), eva_vq.EVA_ERR_INVALID_ARG),  # does not divide K=512
    (dict(K=896, hadamard_block=896), eva_vq.EVA_ERR_INVALID_ARG),    # 28 * 32: Paley factor m < 64
    (dict(K=3584, hadamard_block=1792, residual_group=128), eva_vq.EVA_ERR_INVALID_ARG),  # no signs given
    (dict(max_batch=0), eva_vq.EVA_ERR_INVALID_ARG),
    (dict(max_batch=65), eva_vq.EVA_ERR_INVALID_ARG),
    (dict(out_dtype=7), eva_vq.EVA_ERR_INVALID_ARG),
    (dict(path=4), eva_vq.EVA_ERR_INVALID_ARG),
    (dict(path=3, K=520), eva_vq.EVA_ERR_UNSUPPORTED),            # tcgen05 path: K a multiple of 64
    (dict(path=3, codebook_rows=16), eva_vq.EVA_ERR_UNSUPPORTED),  # ... whole 128-row codebook blocks
    (dict(path=3, index_bits=4), eva_vq.EVA_ERR_UNSUPPORTED),      # ... 8-bit indices
])
def test_create_rejects_bad_descriptor(kw, expect):
    assert _create(_desc(**kw)) == expect


def test_create_rejects_bad_pointers():
    assert _create(_desc(), wc=None) == eva_vq.EVA_ERR_INVALID_ARG
    assert _create(_desc(), wi=None) == eva_vq.EVA_ERR_INVALID_ARG
    assert _create(_desc(), wc=0x1004) == eva_vq.EVA_ERR_INVALID_ARG           # misaligned
    assert _create(_desc(residual_group=128)) == eva_vq.EVA_ERR_INVALID_ARG     # residual without signs
    assert _create(_desc(), signs=0x3000, alpha=0x4000) == eva_vq.EVA_ERR_INVALID_ARG  # signs without residual
    assert _create(_desc(hadamard_block=64)) == eva_vq.EVA_ERR_INVALID_ARG      # rotation without signs s
    lib = eva_vq.load()
    assert lib.eva_vq_linear_create(None, ctypes.byref(_desc()), 0x1000, 0x2000, None, None, None,
                                    None) == eva_vq.EVA_ERR_INVALID_ARG


def test_calls_on_null_handle():
    lib = eva_vq.load()
    assert lib.eva_vq_linear_run(None, 0x1000, 1, 0x2000, None) == eva_vq.EVA_ERR_INVALID_ARG
    assert lib.eva_vq_linear_run_host(None, 0x1000, 1, 0x2000, None) == eva_vq.EVA_ERR_INVALID_ARG
    assert lib.eva_vq_unpack_indices(None, 0x1000, None) == eva_vq.EVA_ERR_INVALID_ARG
    assert lib.eva_vq_sync_status(None) == eva_vq.EVA_ERR_INVALID_ARG
    assert lib.eva_vq_linear_info(None, None) == eva_vq.EVA_ERR_INVALID_ARG
    assert lib.eva_vq_linear_destroy(None) == eva_vq.EVA_OK
    assert lib.eva_vq_linear_run_ex(None, 0x1000, 1, 0x2000, None, 0) == eva_vq.EVA_ERR_INVALID_ARG
    assert lib.eva_vq_linear_run_noalloc(None, 0x1000, 1, 0x2000, None) == eva_vq.EVA_ERR_INVALID_ARG
    assert lib.eva_vq_debug_inject_wait_timeout(None, 1024) == eva_vq.EVA_ERR_INVALID_ARG


def test_grouped_call_rejects_bad_arguments():
    """eva_vq_linear_run_group: null arrays or handles, a count outside
    1..16 and unknown flags are rejected before any device work."""
    import ctypes
    lib = eva_vq.load()
    hs = (ctypes.c_void_p * 2)(None, None)
    xs = (ctypes.c_void_p * 2)(0x1000, 0x1000)
    ys = (ctypes.c_void_p * 2)(0x2000, 0x2000)
    bad = eva_vq.EVA_ERR_INVALID_ARG
    assert lib.eva_vq_linear_run_group(hs, xs, ys, 2, 1, None, 0) == bad
    assert lib.eva_vq_linear_run_group(None, xs, ys, 2, 1, None, 0) == bad
    assert lib.eva_vq_linear_run_group(hs, None, ys, 2, 1, None, 0) == bad
    assert lib.eva_vq_linear_run_group(hs, xs, None, 2, 1, None, 0) == bad
    assert lib.eva_vq_linear_run_group(hs, xs, ys, 0, 1, None, 0) == bad
    assert lib.eva_vq_linear_run_group(hs, xs, ys, 17, 1, None, 0) == bad
    assert lib.eva_vq_linear_run_group(hs, xs, ys, 2, 1, None, 4) == bad


def test_create_without_device_reports_no_device():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    assert _create(_desc()) == eva_vq.EVA_ERR_NO_DEVICE


def test_kernels_do_not_spill():
    """ptxas report of every kernel (the lookup instances, the dequantize and
    tcgen05 instances, the rotation, repack and quantizer kernels): no local-memory
    stack frame and no spills (hot loops keep everything in registers)."""
    cmd = [build._nvcc(), *[f for f in build.NVCC_FLAGS if f != "-shared"], "-Xptxas", "-v", "-c",
           "-I", os.path.join(ROOT, "include"), "-o", os.devnull, *build.SOURCES]
    out = subprocess.run(cmd, capture_output=True, text=True, check=True).stderr
    blocks = re.findall(r"Function properties for (\S*eva_\w+_kernel\S*)\n\s*(\d+) bytes stack frame, "
                        r"(\d+) bytes spill stores, (\d+) bytes spill loads", out)
    assert sum("eva_lookup_kernelI" in b[0] for b in blocks) == 32, out     # 16 for 8-bit + 16 for 4-bit indices
    assert sum("eva_lookup_kernel3I" in b[0] for b in blocks) == 4, out     # three CTAs per SM
    assert sum("eva_dequant_kernel" in b[0] for b in blocks) == 12, out     # per-group x tokens x direct push, + residual
    assert sum("eva_dequant_group_kernel" in b[0] for b in blocks) == 4, out   # several layers per launch
    assert sum("eva_tc_kernel" in b[0] for b in blocks) == 2, out           # tcgen05 path, with / without residual
    assert sum("eva_kmeans_assign_kernel" in b[0] for b in blocks) == 2, out
    for name, stack, st, ld in blocks:
        assert (stack, st, ld) == ("0", "0", "0"), (name, stack, st, ld)


def _qdesc(**kw):
    base = dict(N=64, K=256, d=4, index_bits=8, codebook_rows=0, residual_group=128, hadamard_block=0, iters=2)
    base.update(kw)
    return eva_vq.eva_quant_desc(*[base[f] for f, _ in eva_vq.eva_quant_desc._fields_])


@pytest.mark.parametrize("kw,expect", [
    (dict(d=8), eva_vq.EVA_ERR_UNSUPPORTED),
    (dict(index_bits=9), eva_vq.EVA_ERR_UNSUPPORTED),
    (dict(N=0), eva_vq.EVA_ERR_INVALID_ARG),
    (dict(K=258), eva_vq.EVA_ERR_INVALID_ARG),
    (dict(codebook_rows=48), eva_vq.EVA_ERR_INVALID_ARG),      # does not divide N
    (dict(residual_group=100), eva_vq.EVA_ERR_INVALID_ARG),
    (dict(hadamard_block=96), eva_vq.EVA_ERR_INVALID_ARG),     # not a power of two
    (dict(iters=-1), eva_vq.EVA_ERR_INVALID_ARG),
])
def test_quantize_rejects_bad_descriptor(kw, expect):
    lib = eva_vq.load()
    d = _qdesc(**kw)
    rc = lib.eva_vq_quantize(ctypes.byref(d), 0x1000, None, 0x2000, 0x3000, 0x4000, 0x5000, 0x6000, None, None, None)
    assert rc == expect


def test_quantize_and_steps_reject_bad_pointers():
    lib = eva_vq.load()
    d = _qdesc()
    P = 0x1000
    assert lib.eva_vq_quantize(None, P, None, P, P, P, P, P, None, None, None) == eva_vq.EVA_ERR_INVALID_ARG
    assert lib.eva_vq_quantize(ctypes.byref(d), P, None, P, P, P, None, None, None, None, None) == \
        eva_vq.EVA_ERR_INVALID_ARG                                   # residual without outputs
    assert lib.eva_vq_quantize(ctypes.byref(d), P, 0x7000, P, P, P, P, P, None, None, None) == \
        eva_vq.EVA_ERR_INVALID_ARG                                   # signs s without a rotation
    assert lib.eva_vq_kmeans_assign(P, 10, 3, P, 256, 0, P, None) == eva_vq.EVA_ERR_UNSUPPORTED
    assert lib.eva_vq_kmeans_assign(P + 4, 10, 4, P, 256, 0, P, None) == eva_vq.EVA_ERR_INVALID_ARG
    assert lib.eva_vq_kmeans_assign(P, 10, 4, P, 257, 0, P, None) == eva_vq.EVA_ERR_INVALID_ARG
    assert lib.eva_vq_kmeans_update(P, 10, 4, None, 256, 0, P, P, None, None) == eva_vq.EVA_ERR_INVALID_ARG
    assert lib.eva_vq_residual(P, 4, 256, P, 256, P, 0, 100, P, P, None) == eva_vq.EVA_ERR_INVALID_ARG
    assert lib.eva_vq_residual(P, 4, 256, P, 256, P, 3, 128, P, P, None) == eva_vq.EVA_ERR_INVALID_ARG


def test_create_accepts_order_k_rotation_descriptor():
    """K = 3584 = 28 * 128 with b = K passes validation (the CPU machine then has
    no device to create it on)."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    d = _desc(K=3584, hadamard_block=3584, residual_group=128)
    assert _create(d, signs=0x3000, alpha=0x4000, hsign=0x5000) == eva_vq.EVA_ERR_NO_DEVICE


def test_unit_layouts_are_bijections():
    """The repack layouts (host-compilable header): every (row, sub-vector) of
    a unit appears exactly once, for byte indices and for 4-bit indices, and
    the 4-bit inverse undoes the forward map; every (row, input) of a
    dequantize-path sign unit has exactly one bit, and lane (g, q)'s 16 bytes
    hold rows g and g + 8 only, at the inputs of the sub-vectors it reads
    (dq_subvec)."""
    src = r"""
#include <cstdio>
#define __host__
#define __device__
#define __forceinline__ inline
#include "eva_vq_layout.cuh"
using namespace eva;
int main() {
    int bad = 0, seen8[16][64] = {{0}}, seen4[16][64] = {{0}};
    for (int b = 0; b < kUnitBytes; ++b) { int r, j; wi_unit_pos(b, r, j); seen8[r][j]++; }
    for (int n = 0; n < 2 * kUnitBytes4; ++n) {
        int r, j; wi4_unit_pos(n, r, j); seen4[r][j]++;
        if (wi4_unit_nibble(r, j) != n) ++bad;
    }
    for (int r = 0; r < 16; ++r) for (int j = 0; j < 64; ++j) bad += (seen8[r][j] != 1) + (seen4[r][j] != 1);
    static int seen_s[16][256];
    for (int b = 0; b < kDqSignUnitBytes; ++b)
        for (int t = 0; t < 8; ++t) {
            int r, k;
            dq_sign_pos(b, t, r, k);
            if (r < 0 || r >= 16 || k < 0 || k >= 256) { ++bad; continue; }
            seen_s[r][k]++;
            const int lane = b >> 4, g = lane >> 2, q = lane & 3;
            if ((r & 7) != g) ++bad;
            bool read = false;
            for (int beta = 0; beta < 16; ++beta) read |= (k >> 2) == dq_subvec(beta, q);
            if (!read) ++bad;
        }
    for (int r = 0; r < 16; ++r) for (int k = 0; k < 256; ++k) bad += seen_s[r][k] != 1;
    std::printf("%d\n", bad);
    return 0;
}
"""
    import tempfile
    with tempfile.TemporaryDirectory() as d:
        cpp = os.path.join(d, "t.cpp")
        open(cpp, "w").write(src)
        exe = os.path.join(d, "t")
        subprocess.run(["g++", "-std=c++17", "-I", os.path.join(ROOT, "vector_quantized_weight_b200", "csrc"),
                        "-o", exe, cpp], check=True)
        assert subprocess.run([exe], capture_output=True, text=True, check=True).stdout.strip() == "0"


def test_independent_grid_invariants():
    """The grid of independent calls (host-compilable header), over every
    latency plan of up to 148 CTAs and row-tile counts up to 2000, with a
    footprint that grows with the tile count: clusters of at most 8 CTAs (the
    latency plan's Gs when it is at most 8, else half of it), never more CTAs
    than the latency plan, never more tiles per CTA than the layout holds,
    within the footprint budget, and the fewest row groups that satisfy all
    of that (no smaller Gt would do)."""
    src = r"""
#include <cstdio>
#include <cstddef>
#include "eva_vq_plan.h"
using namespace eva;
int main() {
    long long bad = 0, found = 0;
    const int hards[2] = {128, 247}, softs[2] = {64, 128};
    const size_t fits[3] = {70000, 98304, 116736};
    for (int T = 1; T <= 2000; T += (T < 300 ? 1 : 7))
    for (int lgs = 1; lgs <= 16; ++lgs)
    for (int lgt = 1; lgs * lgt <= 148 && lgt <= T; ++lgt)
    for (int hi = 0; hi < 2; ++hi) for (int si = 0; si < 2; ++si) for (int fi = 0; fi < 3; ++fi) {
        const int hard = hards[hi], soft = softs[si];
        const size_t fit = fits[fi];
        auto smem = [](int tiles, int gs) { return (size_t)65536 + 256 * (size_t)tiles + 8 * (size_t)gs; };
        int gs = 0, gt = 0; size_t sm = 0;
        if (!independent_grid(T, lgs, lgt, hard, soft, fit, smem, &gs, &gt, &sm)) continue;
        ++found;
        const int tiles = (T + gt - 1) / gt;
        bad += gs != (lgs > 8 ? (lgs + 1) / 2 : lgs);
        bad += gs > 8 || gt < 1 || gt > T;
        bad += gs * gt > lgs * lgt;
        bad += tiles > hard;
        bad += sm != smem(tiles, gs) || sm > fit;
        // minimal: no smaller row-group count meets the same constraints
        // and the preferred tile count
        for (int g2 = 1; g2 < gt; ++g2) {
            const int t2 = (T + g2 - 1) / g2;
            if (t2 <= hard && t2 <= soft && smem(t2, gs) <= fit) { ++bad; break; }
        }
    }
    std::printf("%lld %lld\n", bad, found);
    return 0;
}
"""
    import tempfile
    with tempfile.TemporaryDirectory() as d:
        cpp = os.path.join(d, "t.cpp")
        open(cpp, "w").write(src)
        exe = os.path.join(d, "t")
        subprocess.run(["g++", "-std=c++17", "-O2", "-I", os.path.join(ROOT, "vector_quantized_weight_b200", "csrc"),
                        "-o", exe, cpp], check=True)
        bad, found = map(int, subprocess.run([exe], capture_output=True, text=True, check=True).stdout.split())
        assert bad == 0 and found > 100_000, (bad, found)

