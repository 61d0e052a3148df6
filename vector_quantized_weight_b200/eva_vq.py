"""Thin ctypes binding of the C ABI in include/eva_vq.h.

Functions carry the C names and only marshal arguments: every step of the
layer runs in the CUDA library.  PyTorch is used for device memory and
streams only (``VQLinear``).  There is no CPU fallback: if the library cannot
be loaded, every call raises.
"""
from __future__ import annotations

import ctypes
import os

from . import build as _build

EVA_OK, EVA_ERR_INVALID_ARG, EVA_ERR_UNSUPPORTED, EVA_ERR_CUDA, EVA_ERR_OOM, \
    EVA_ERR_DEVICE_TIMEOUT, EVA_ERR_NO_DEVICE, EVA_ERR_DEVICE_CHECK, EVA_ERR_SCRATCH_TOO_SMALL = range(9)
EVA_F16, EVA_F32 = 0, 1
EVA_PATH_AUTO, EVA_PATH_OC_LOOKUP, EVA_PATH_DEQUANT_MMA, EVA_PATH_TCGEN05 = 0, 1, 2, 3

# Every function the header declares; the CPU tests check the library exports them.
EVA_RUN_INDEPENDENT = 1

ABI_FUNCTIONS = (
    "eva_vq_linear_create", "eva_vq_linear_run", "eva_vq_linear_run_ex", "eva_vq_linear_run_host",
    "eva_vq_linear_destroy", "eva_vq_unpack_indices", "eva_vq_sync_status",
    "eva_vq_status_string", "eva_vq_linear_info", "eva_vq_device_check_record",
    "eva_vq_debug_timeline", "eva_vq_linear_run_noalloc",
    "eva_vq_quantize", "eva_vq_kmeans_assign", "eva_vq_kmeans_update", "eva_vq_residual",
    "eva_vq_linear_run_group", "eva_vq_debug_inject_wait_timeout",
)


class EvaError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        msg = eva_vq_status_string(status) if _lib is not None else str(status)
        super().__init__(f"{fn} failed: {msg} ({status})")


class eva_vq_desc(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int32), ("K", ctypes.c_int32), ("d", ctypes.c_int32),
                ("index_bits", ctypes.c_int32), ("codebook_rows", ctypes.c_int32),
                ("residual_group", ctypes.c_int32), ("hadamard_block", ctypes.c_int32),
                ("max_batch", ctypes.c_int32), ("out_dtype", ctypes.c_int),
                ("path", ctypes.c_int)]


class eva_quant_desc(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int32), ("K", ctypes.c_int32), ("d", ctypes.c_int32),
                ("index_bits", ctypes.c_int32), ("codebook_rows", ctypes.c_int32),
                ("residual_group", ctypes.c_int32), ("hadamard_block", ctypes.c_int32),
                ("iters", ctypes.c_int32)]


class eva_vq_info(ctypes.Structure):
    _fields_ = [("stream_bytes", ctypes.c_int64), ("wi_bytes", ctypes.c_int64),
                ("sign_bytes", ctypes.c_int64), ("alpha_bytes", ctypes.c_int64),
                ("codebook_bytes", ctypes.c_int64), ("workspace_bytes", ctypes.c_int64),
                ("slices", ctypes.c_int32), ("row_tiles", ctypes.c_int32),
                ("grid", ctypes.c_int32), ("kernels_per_run", ctypes.c_int32),
                ("path", ctypes.c_int32), ("sm_count", ctypes.c_int32),
                ("staged_units", ctypes.c_int32)]


_lib = None


def library_path() -> str:
    """The regular library; EVA_VQ_CHECKED=1 selects the device-check build,
    EVA_VQ_TIMELINE=1 the phase-timeline build, EVA_VQ_NAIVE=1 the build with
    the naive image layout (all three diagnostics only), and
    EVA_VQ_LIBRARY=<path> any other build of the same C ABI."""
    if os.environ.get("EVA_VQ_LIBRARY"):
        return os.environ["EVA_VQ_LIBRARY"]
    if os.environ.get("EVA_VQ_CHECKED") == "1":
        return _build.CHECKED_LIB
    if os.environ.get("EVA_VQ_TIMELINE") == "1":
        return _build.TIMELINE_LIB
    if os.environ.get("EVA_VQ_NAIVE") == "1":
        return _build.NAIVE_LIB
    return _build.LIB


def load(build_if_missing: bool = True) -> ctypes.CDLL:
    """Load libeva_vq.so (building it with nvcc if it is absent)."""
    global _lib
    if _lib is not None:
        return _lib
    path = library_path()
    if not os.path.exists(path):
        if not build_if_missing:
            raise RuntimeError(f"{path} is missing; build it with vector_quantized_weight_b200.build")
        _build.build(checked=path == _build.CHECKED_LIB, timeline=path == _build.TIMELINE_LIB,
                     naive=path == _build.NAIVE_LIB)
    lib = ctypes.CDLL(path)
    P, I32, H = ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p
    lib.eva_vq_linear_create.argtypes = [ctypes.POINTER(H), ctypes.POINTER(eva_vq_desc), P, P, P, P, P, P]
    lib.eva_vq_linear_run.argtypes = [H, P, I32, P, P]
    lib.eva_vq_linear_run_ex.argtypes = [H, P, I32, P, P, ctypes.c_uint32]
    lib.eva_vq_linear_run_noalloc.argtypes = [H, P, I32, P, P]
    lib.eva_vq_linear_run_group.argtypes = [P, P, P, I32, I32, P, ctypes.c_uint32]
    lib.eva_vq_linear_run_host.argtypes = [H, P, I32, P, P]
    lib.eva_vq_linear_destroy.argtypes = [H]
    lib.eva_vq_unpack_indices.argtypes = [H, P, P]
    lib.eva_vq_sync_status.argtypes = [H]
    lib.eva_vq_status_string.argtypes = [ctypes.c_int]
    lib.eva_vq_status_string.restype = ctypes.c_char_p
    lib.eva_vq_linear_info.argtypes = [H, ctypes.POINTER(eva_vq_info)]
    lib.eva_vq_device_check_record.argtypes = [H, P]
    lib.eva_vq_debug_inject_wait_timeout.argtypes = [H, I32]
    lib.eva_vq_debug_timeline.argtypes = [H, P, I32, ctypes.POINTER(I32)]
    I64 = ctypes.c_int64
    lib.eva_vq_quantize.argtypes = [ctypes.POINTER(eva_quant_desc), P, P, P, P, P, P, P, P, P, P]
    lib.eva_vq_kmeans_assign.argtypes = [P, I64, I32, P, I32, I64, P, P]
    lib.eva_vq_kmeans_update.argtypes = [P, I64, I32, P, I32, I64, P, P, P, P]
    lib.eva_vq_residual.argtypes = [P, I32, I32, P, I32, P, I32, I32, P, P, P]
    for fn in ABI_FUNCTIONS:
        if fn != "eva_vq_status_string":
            getattr(lib, fn).restype = ctypes.c_int
    _lib = lib
    return lib


def _check(fn: str, rc: int):
    if rc != EVA_OK:
        raise EvaError(fn, rc)


# ------------------------------------------------------------ the C names

def eva_vq_status_string(status: int) -> str:
    return load().eva_vq_status_string(int(status)).decode()


def eva_vq_linear_create(desc: eva_vq_desc, wc: int, wi: int, signs: int | None, alpha: int | None,
                         hsign: int | None, stream: int | None) -> int:
    h = ctypes.c_void_p()
    rc = load().eva_vq_linear_create(ctypes.byref(h), ctypes.byref(desc), wc, wi, signs, alpha,
                                     hsign, stream)
    _check("eva_vq_linear_create", rc)
    return h.value


def eva_vq_linear_run(h: int, x: int, B: int, y: int, stream: int | None) -> None:
    _check("eva_vq_linear_run", load().eva_vq_linear_run(h, x, int(B), y, stream))


def eva_vq_linear_run_ex(h: int, x: int, B: int, y: int, stream: int | None, flags: int) -> None:
    _check("eva_vq_linear_run_ex", load().eva_vq_linear_run_ex(h, x, int(B), y, stream, int(flags)))


def eva_vq_linear_run_noalloc(h: int, x: int, B: int, y: int, stream: int | None) -> None:
    """eva_vq_linear_run without any device allocation: a rotated layer's
    scratch comes from the library's 4 MiB static device array (see the
    header for who needs this and the sharing rules)."""
    _check("eva_vq_linear_run_noalloc", load().eva_vq_linear_run_noalloc(h, x, int(B), y, stream))


def eva_vq_linear_run_group(hs: list, xs: list, ys: list, B: int, stream: int | None, flags: int = 0) -> None:
    """Independent layers in one launch where their shapes and formats allow
    (see the header); hs, xs, ys are lists of handles and device pointers."""
    n = len(hs)
    ha = (ctypes.c_void_p * n)(*hs)
    xa = (ctypes.c_void_p * n)(*xs)
    ya = (ctypes.c_void_p * n)(*ys)
    _check("eva_vq_linear_run_group", load().eva_vq_linear_run_group(ha, xa, ya, n, int(B), stream, int(flags)))


def eva_vq_linear_run_host(h: int, x_host: int, B: int, y_host: int, stream: int | None) -> None:
    _check("eva_vq_linear_run_host", load().eva_vq_linear_run_host(h, x_host, int(B), y_host, stream))


def eva_vq_linear_destroy(h: int | None) -> None:
    _check("eva_vq_linear_destroy", load().eva_vq_linear_destroy(h))


def eva_vq_unpack_indices(h: int, wi_out: int, stream: int | None) -> None:
    _check("eva_vq_unpack_indices", load().eva_vq_unpack_indices(h, wi_out, stream))


def eva_vq_sync_status(h: int) -> int:
    return int(load().eva_vq_sync_status(h))


def eva_vq_debug_inject_wait_timeout(h: int, rounds: int) -> None:
    _check("eva_vq_debug_inject_wait_timeout", load().eva_vq_debug_inject_wait_timeout(h, rounds))


def eva_vq_device_check_record(h: int) -> list:
    rec = (ctypes.c_int32 * 8)()
    _check("eva_vq_device_check_record", load().eva_vq_device_check_record(h, rec))
    return list(rec)


def eva_vq_debug_timeline(h: int, max_entries: int = 1 << 16) -> list:
    buf = (ctypes.c_uint64 * max_entries)()
    n = ctypes.c_int32()
    _check("eva_vq_debug_timeline", load().eva_vq_debug_timeline(h, buf, max_entries, ctypes.byref(n)))
    return list(buf[:n.value])


def eva_vq_linear_info(h: int) -> eva_vq_info:
    info = eva_vq_info()
    _check("eva_vq_linear_info", load().eva_vq_linear_info(h, ctypes.byref(info)))
    return info


def eva_vq_quantize(desc: eva_quant_desc, w: int, hsign: int | None, init_index: int, wc_out: int, wi_out: int,
                    signs_out: int | None, alpha_out: int | None, wrot_out: int | None, cent_out: int | None,
                    stream: int | None) -> None:
    _check("eva_vq_quantize", load().eva_vq_quantize(ctypes.byref(desc), w, hsign, init_index, wc_out, wi_out,
                                                     signs_out, alpha_out, wrot_out, cent_out, stream))


def eva_vq_kmeans_assign(v: int, M: int, d: int, centroids: int, ncent: int, vecs_per_cb: int, idx_out: int,
                         stream: int | None) -> None:
    _check("eva_vq_kmeans_assign", load().eva_vq_kmeans_assign(v, int(M), int(d), centroids, int(ncent),
                                                               int(vecs_per_cb), idx_out, stream))


def eva_vq_kmeans_update(v: int, M: int, d: int, idx: int, ncent: int, vecs_per_cb: int, old: int, new_out: int,
                         counts_out: int | None, stream: int | None) -> None:
    _check("eva_vq_kmeans_update", load().eva_vq_kmeans_update(v, int(M), int(d), idx, int(ncent),
                                                               int(vecs_per_cb), old, new_out, counts_out, stream))


def eva_vq_residual(wrot: int, N: int, K: int, wc: int, ncent: int, wi: int, codebook_rows: int, group: int,
                    signs_out: int, alpha_out: int, stream: int | None) -> None:
    _check("eva_vq_residual", load().eva_vq_residual(wrot, int(N), int(K), wc, int(ncent), wi,
                                                     int(codebook_rows), int(group), signs_out, alpha_out, stream))


# ------------------------------------------------------- torch convenience

def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(stream=None):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


class VQLinear:
    """One layer held on the device.  Weights are torch CUDA tensors in the
    canonical layouts (see synth.py); they are copied and repacked by the
    library, so the caller may drop them after construction."""

    def __init__(self, wc, wi, *, signs=None, alpha=None, hsign=None, codebook_rows=0,
                 residual_group=0, hadamard_block=0, max_batch=1, out_dtype="float16",
                 path=EVA_PATH_AUTO, index_bits=8, stream=None):
        import torch
        N, J = wi.shape
        if index_bits == 4:          # two indices per byte
            J *= 2
        self.index_bits = int(index_bits)
        self.N, self.K = int(N), int(J) * 4
        self.out_dtype = torch.float32 if out_dtype in ("float32", torch.float32) else torch.float16
        self.max_batch = int(max_batch)
        self.desc = eva_vq_desc(self.N, self.K, 4, self.index_bits, int(codebook_rows), int(residual_group),
                                int(hadamard_block), self.max_batch,
                                EVA_F32 if self.out_dtype == torch.float32 else EVA_F16, int(path))
        tensors = [wc, wi, signs, alpha, hsign]
        for t in tensors:
            if t is not None and (not t.is_cuda or not t.is_contiguous()):
                raise ValueError("weights must be contiguous CUDA tensors")
        self.handle = None
        self.handle = eva_vq_linear_create(self.desc, _ptr(wc), _ptr(wi), _ptr(signs), _ptr(alpha),
                                           _ptr(hsign), _stream_handle(stream))

    def __call__(self, x, out=None, stream=None, independent=False):
        """y = layer(x) on `stream`.  independent=True passes EVA_RUN_INDEPENDENT:
        the caller promises the preceding kernel on the stream neither writes x
        nor touches y; the call then overlaps it and takes the overlap grid."""
        import torch
        if x.dtype != torch.float16 or not x.is_cuda or not x.is_contiguous():
            raise ValueError("x must be a contiguous CUDA float16 tensor [B, K]")
        x2 = x.view(-1, self.K)
        B = x2.shape[0]
        y = out if out is not None else torch.empty((B, self.N), dtype=self.out_dtype, device=x.device)
        eva_vq_linear_run_ex(self.handle, _ptr(x2), B, _ptr(y), _stream_handle(stream),
                             EVA_RUN_INDEPENDENT if independent else 0)
        return y

    def run_host(self, x_host, y_host, stream=None):
        """Host buffers in and out (torch CPU tensors, ideally pinned)."""
        B = x_host.shape[0]
        eva_vq_linear_run_host(self.handle, _ptr(x_host), B, _ptr(y_host), _stream_handle(stream))
        return y_host

    def unpack_indices(self, stream=None):
        """The canonical index matrix back: [N][K/4], or [N][K/8] packed for 4-bit indices."""
        import torch
        cols = self.K // 4 if self.index_bits == 8 else self.K // 8
        out = torch.empty((self.N, cols), dtype=torch.uint8, device="cuda")
        eva_vq_unpack_indices(self.handle, _ptr(out), _stream_handle(stream))
        return out

    def info(self) -> eva_vq_info:
        return eva_vq_linear_info(self.handle)

    def close(self):
        if self.handle is not None:
            eva_vq_linear_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def from_layer(layer, *, max_batch=1, out_dtype="float16", path=EVA_PATH_AUTO, device="cuda"):
    """Build a VQLinear from a synth.LayerData (numpy arrays)."""
    import torch

    def dev(a):
        return None if a is None else torch.from_numpy(a).to(device)
    s = layer.shape
    return VQLinear(dev(layer.wc), dev(layer.wi), signs=dev(layer.signs), alpha=dev(layer.alpha),
                    hsign=dev(layer.hsign), codebook_rows=s.codebook_rows,
                    residual_group=s.residual_group, hadamard_block=s.hadamard_block,
                    max_batch=max_batch, out_dtype=out_dtype, path=path, index_bits=s.index_bits)


def quantize(w, init_index, iters: int, *, hsign=None, hadamard_block: int = 0, codebook_rows: int = 0,
             residual_group: int = 128, index_bits: int = 8, keep_wrot: bool = False, keep_centroids: bool = False,
             stream=None) -> dict:
    """The offline quantizer on the GPU (eva_vq_quantize).  w: CUDA fp16
    [N][K]; init_index: CUDA int32 [G][2^index_bits] starting blocks (see the
    header).  Returns CUDA tensors wc, wi (and signs, alpha with a residual;
    wrot, centroids on request) ready for VQLinear."""
    import torch
    N, K = w.shape
    dev = w.device
    G = N // codebook_rows if codebook_rows else 1
    ncent = 1 << index_bits
    # 4-bit pointers come packed two per byte (the layout VQLinear(index_bits=4) takes)
    out = {"wc": torch.empty((G, ncent, 4), dtype=torch.float16, device=dev),
           "wi": torch.empty((N, K // 8 if index_bits == 4 else K // 4), dtype=torch.uint8, device=dev)}
    if residual_group:
        out["signs"] = torch.empty((N, K // 8), dtype=torch.uint8, device=dev)
        out["alpha"] = torch.empty((N, K // residual_group), dtype=torch.float16, device=dev)
    if keep_wrot:
        out["wrot"] = torch.empty((N, K), dtype=torch.float32, device=dev)
    if keep_centroids:
        out["centroids"] = torch.empty((G, ncent, 4), dtype=torch.float32, device=dev)
    desc = eva_quant_desc(N, K, 4, index_bits, codebook_rows, residual_group, hadamard_block, iters)
    eva_vq_quantize(desc, _ptr(w.contiguous()), _ptr(hsign), _ptr(init_index.contiguous()), _ptr(out["wc"]),
                    _ptr(out["wi"]), _ptr(out.get("signs")), _ptr(out.get("alpha")), _ptr(out.get("wrot")),
                    _ptr(out.get("centroids")), _stream_handle(stream))
    return out


def run_group(layers, xs, outs=None, stream=None, independent=False):
    """Run VQLinear layers on their inputs (CUDA fp16 [B][K] tensors, one B)
    as one grouped call; returns the outputs."""
    import torch
    B = xs[0].shape[0]
    if outs is None:
        outs = [torch.empty((B, l.N), dtype=l.out_dtype, device=x.device) for l, x in zip(layers, xs)]
    eva_vq_linear_run_group([l.handle for l in layers], [x.data_ptr() for x in xs], [y.data_ptr() for y in outs],
                            B, _stream_handle(stream), EVA_RUN_INDEPENDENT if independent else 0)
    return outs
