"""Thin ctypes binding of libuw (include/uw.h): argument marshalling only.

Every step of the compression and matmul path runs inside libuw.so (host
C++ encoder, CUDA kernels for sm_100a).  PyTorch only provides device memory
and streams.  If libuw.so is missing this module raises at import time; there
is no fallback implementation.

BF16 matrices are handled as their raw 16-bit patterns: numpy ``uint16`` on
the host, torch ``int16`` (same bits) on the device.
"""
from __future__ import annotations

import ctypes
import json
import os
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
# the in-tree build; UW_LIBRARY may point at another build of the same library
LIB_PATH = os.environ.get("UW_LIBRARY") or os.path.join(_HERE, "libuw.so")

UW_OK = 0
ERR_INVALID_ARG, ERR_UNSUPPORTED_SHAPE, ERR_CORRUPT, ERR_CUDA, ERR_NOMEM, ERR_TIMEOUT, ERR_WORKSPACE = range(1, 8)
STATUS_NAMES = {0: "UW_OK", 1: "UW_ERR_INVALID_ARG", 2: "UW_ERR_UNSUPPORTED_SHAPE",
                3: "UW_ERR_CORRUPT", 4: "UW_ERR_CUDA", 5: "UW_ERR_NOMEM", 6: "UW_ERR_TIMEOUT",
                7: "UW_ERR_WORKSPACE"}
EMIT_HUFFMAN = 1
EMIT_PALETTE = 2
SEC_SM, SEC_RAWEXP, SEC_FLAGS, SEC_RAWBASE, SEC_STREAM, SEC_CHUNKOFF, SEC_DLUT, SEC_PAL = range(8)
NUM_SECTIONS = 8
PIPE_DECODE_GEMM, PIPE_DECODE_EXP_FUSED, PIPE_TRANSCODE_FUSED, PIPE_DIRECT_PALETTE, PIPE_HUFFMAN_FUSED = 1, 2, 3, 4, 5
KERNEL_FMA, KERNEL_TC, KERNEL_MMA, KERNEL_TC_SK, KERNEL_MMA_SK = 1, 2, 3, 4, 5
DEBUG_NEVER_ARRIVE = 1

# every symbol include/uw.h declares
EXPORTS = ("uw_status_str", "uw_version", "uw_encode", "uw_blob_data", "uw_blob_free",
           "uw_blob_info_get", "uw_matrix_bind", "uw_device_status", "uw_decode_to_bf16",
           "uw_decode_exponents", "uw_transcode_palette", "uw_plan_default", "uw_workspace_size", "uw_fused_matmul",
           "uw_matmul_bf16", "uw_autotune_workspace_size", "uw_plan_autotune",
           "uw_fused_matmul_noalloc", "uw_stack_workspace_size", "uw_stack_run",
           "uw_sm_split_create", "uw_sm_split_get", "uw_sm_split_destroy", "uw_stack_tune_split",
           "uw_fused_matmul_batched")


class UwError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__("%s: %s" % (what, STATUS_NAMES.get(status, status)))


class BlobInfo(ctypes.Structure):
    _fields_ = [("n", ctypes.c_int64), ("k", ctypes.c_int64), ("flags", ctypes.c_uint32),
                ("palette_size", ctypes.c_int32), ("palette", ctypes.c_uint8 * 16),
                ("code_len", ctypes.c_uint8 * 16), ("n_groups", ctypes.c_int64),
                ("n_raw", ctypes.c_int64), ("n_chunks", ctypes.c_int64),
                ("stream_bits", ctypes.c_uint64), ("entropy_bits", ctypes.c_double),
                ("top16_coverage", ctypes.c_double), ("total_bytes", ctypes.c_uint64),
                ("huffman_bytes", ctypes.c_uint64), ("palette_bytes", ctypes.c_uint64),
                ("section_offset", ctypes.c_uint64 * NUM_SECTIONS),
                ("section_bytes", ctypes.c_uint64 * NUM_SECTIONS)]


class DMat(ctypes.Structure):
    _fields_ = [("n", ctypes.c_int64), ("k", ctypes.c_int64), ("flags", ctypes.c_uint32),
                ("palette_size", ctypes.c_int32), ("palette", ctypes.c_uint8 * 16),
                ("code_len", ctypes.c_uint8 * 16), ("n_groups", ctypes.c_int64),
                ("n_raw", ctypes.c_int64), ("n_chunks", ctypes.c_int64),
                ("stream_bits", ctypes.c_uint64), ("stream_words", ctypes.c_uint64),
                ("sm", ctypes.c_void_p), ("rawexp", ctypes.c_void_p), ("flagbits", ctypes.c_void_p),
                ("rawbase", ctypes.c_void_p), ("stream", ctypes.c_void_p),
                ("chunk_off", ctypes.c_void_p), ("dlut", ctypes.c_void_p), ("pal", ctypes.c_void_p),
                ("dev_status", ctypes.c_void_p)]


class Plan(ctypes.Structure):
    _fields_ = [("pipeline", ctypes.c_int32), ("kernel", ctypes.c_int32), ("bn", ctypes.c_int32),
                ("split_k", ctypes.c_int32), ("stages", ctypes.c_int32),
                ("debug_flags", ctypes.c_uint32), ("timeout_ns", ctypes.c_int64)]

    def as_dict(self):
        return {f: getattr(self, f) for f, _ in self._fields_}

    def __repr__(self):
        return "Plan(%s)" % ", ".join("%s=%s" % kv for kv in self.as_dict().items())


class StackStep(ctypes.Structure):
    _fields_ = [("w", ctypes.POINTER(DMat)), ("x_dev", ctypes.c_void_p), ("m", ctypes.c_int64),
                ("y_dev", ctypes.c_void_p), ("plan", Plan), ("pal_dev", ctypes.c_void_p)]


class BatchItem(ctypes.Structure):
    _fields_ = [("w", ctypes.POINTER(DMat)), ("x_dev", ctypes.c_void_p), ("m", ctypes.c_int64),
                ("y_dev", ctypes.c_void_p)]


def make_plan(pipeline=PIPE_DIRECT_PALETTE, kernel=KERNEL_TC, bn=16, split_k=1, stages=0,
              debug_flags=0, timeout_ns=0) -> Plan:
    return Plan(pipeline, kernel, bn, split_k, stages, debug_flags, timeout_ns)


_lib = None


def lib() -> ctypes.CDLL:
    """Load libuw.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError("libuw.so not found at %s; build it with "
                           "`python -m decode_gemm_exponent_b200.build`" % LIB_PATH)
    L = ctypes.CDLL(LIB_PATH)
    P, I64, I32, U32, SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_uint32, ctypes.c_size_t
    sig = {
        "uw_status_str": (ctypes.c_char_p, [ctypes.c_int]),
        "uw_version": (ctypes.c_char_p, []),
        "uw_encode": (ctypes.c_int, [P, I64, I64, U32, ctypes.POINTER(P)]),
        "uw_blob_data": (P, [P, ctypes.POINTER(SZ)]),
        "uw_blob_free": (None, [P]),
        "uw_blob_info_get": (ctypes.c_int, [P, SZ, ctypes.c_int, ctypes.POINTER(BlobInfo)]),
        "uw_matrix_bind": (ctypes.c_int, [P, SZ, P, P, ctypes.c_int, ctypes.POINTER(DMat)]),
        "uw_device_status": (ctypes.c_int, [ctypes.POINTER(DMat), P]),
        "uw_decode_to_bf16": (ctypes.c_int, [ctypes.POINTER(DMat), P, P]),
        "uw_decode_exponents": (ctypes.c_int, [ctypes.POINTER(DMat), P, P]),
        "uw_transcode_palette": (ctypes.c_int, [ctypes.POINTER(DMat), P, P]),
        "uw_plan_default": (ctypes.c_int, [I64, I64, I64, I32, ctypes.POINTER(Plan)]),
        "uw_workspace_size": (ctypes.c_int, [I64, I64, I64, ctypes.POINTER(Plan), ctypes.POINTER(SZ)]),
        "uw_fused_matmul": (ctypes.c_int, [P, I64, ctypes.POINTER(DMat), P, P, ctypes.POINTER(Plan),
                                           P, SZ, P]),
        "uw_matmul_bf16": (ctypes.c_int, [P, I64, P, I64, I64, P, ctypes.POINTER(Plan), P, SZ, P, P]),
        "uw_fused_matmul_noalloc": (ctypes.c_int, [P, I64, ctypes.POINTER(DMat), P, ctypes.POINTER(Plan), P]),
        "uw_fused_matmul_batched": (ctypes.c_int, [ctypes.POINTER(BatchItem), ctypes.c_int, ctypes.POINTER(Plan), P]),
        "uw_stack_workspace_size": (ctypes.c_int, [ctypes.POINTER(StackStep), ctypes.c_int, ctypes.POINTER(SZ)]),
        "uw_stack_run": (ctypes.c_int, [ctypes.POINTER(StackStep), ctypes.c_int, P, SZ, P, P]),
        "uw_sm_split_create": (ctypes.c_int, [ctypes.c_int, ctypes.c_int, ctypes.POINTER(P)]),
        "uw_sm_split_get": (ctypes.c_int, [P, ctypes.POINTER(P), ctypes.POINTER(P), ctypes.POINTER(ctypes.c_int),
                                           ctypes.POINTER(ctypes.c_int)]),
        "uw_sm_split_destroy": (None, [P]),
        "uw_stack_tune_split": (ctypes.c_int, [ctypes.POINTER(StackStep), ctypes.c_int, P, SZ, ctypes.c_int,
                                               ctypes.POINTER(ctypes.c_int), ctypes.c_int, ctypes.c_int,
                                               ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_float), P]),
        "uw_autotune_workspace_size": (ctypes.c_int, [ctypes.POINTER(ctypes.POINTER(DMat)), ctypes.c_int,
                                                      ctypes.POINTER(I64), ctypes.c_int,
                                                      ctypes.POINTER(SZ)]),
        "uw_plan_autotune": (ctypes.c_int, [ctypes.POINTER(ctypes.POINTER(DMat)), ctypes.c_int,
                                            ctypes.POINTER(I64), ctypes.c_int, P, P, P, SZ,
                                            ctypes.c_int, ctypes.POINTER(Plan), ctypes.c_char_p, SZ,
                                            P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _lib = L
    return L


def check(status: int, what: str) -> None:
    if status != UW_OK:
        raise UwError(status, what)


def version() -> str:
    return lib().uw_version().decode()


# ----------------------------------------------------------------------------- host side

def encode(w: np.ndarray, flags: int = 0) -> bytes:
    """uw_encode: BF16 bit patterns uint16[n, k] -> serialized blob bytes."""
    w = np.ascontiguousarray(w)
    if w.dtype != np.uint16:
        w = w.view(np.uint16)
    n, k = w.shape
    out = ctypes.c_void_p()
    check(lib().uw_encode(w.ctypes.data, n, k, flags, ctypes.byref(out)), "uw_encode")
    try:
        size = ctypes.c_size_t()
        ptr = lib().uw_blob_data(out, ctypes.byref(size))
        return ctypes.string_at(ptr, size.value)
    finally:
        lib().uw_blob_free(out)


def blob_info(blob: bytes, verify_payload: bool = False) -> BlobInfo:
    info = BlobInfo()
    buf = np.frombuffer(blob, np.uint8)
    check(lib().uw_blob_info_get(buf.ctypes.data, buf.size, int(verify_payload), ctypes.byref(info)),
          "uw_blob_info_get")
    return info


def section(blob: bytes, sec: int, info: Optional[BlobInfo] = None) -> np.ndarray:
    """uint8 view of one section of a serialized blob."""
    info = info or blob_info(blob)
    off, size = info.section_offset[sec], info.section_bytes[sec]
    return np.frombuffer(blob, np.uint8, count=size, offset=off)


# ----------------------------------------------------------------------------- device side

def _stream_handle(stream=None):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t) -> ctypes.c_void_p:
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


class Matrix:
    """A compressed matrix whose blob lives in device memory (torch-owned)."""

    def __init__(self, blob: bytes, device="cuda", verify_payload: bool = False):
        import torch
        self.blob = blob
        self.host = np.frombuffer(blob, np.uint8)
        self.dev = torch.empty(len(blob), dtype=torch.uint8, device=device)
        self.dev.copy_(torch.from_numpy(self.host.copy()))
        self.status = torch.zeros(4, dtype=torch.int32, device=device)
        self.dmat = DMat()
        check(lib().uw_matrix_bind(self.host.ctypes.data, self.host.size, self.dev.data_ptr(),
                                   self.status.data_ptr(), int(verify_payload), ctypes.byref(self.dmat)),
              "uw_matrix_bind")
        self.info = blob_info(blob)
        self.n, self.k = int(self.dmat.n), int(self.dmat.k)

    # -- preprocessing kernels
    def decode(self, out=None, stream=None):
        import torch
        if out is None:
            out = torch.empty(self.n, self.k, dtype=torch.int16, device=self.dev.device)
        check(lib().uw_decode_to_bf16(ctypes.byref(self.dmat), _ptr(out), _stream_handle(stream)),
              "uw_decode_to_bf16")
        return out

    def decode_exponents(self, out=None, stream=None):
        """Exponent byte of every weight, uint8 [n, k]."""
        import torch
        if out is None:
            out = torch.empty(self.n, self.k, dtype=torch.uint8, device=self.dev.device)
        check(lib().uw_decode_exponents(ctypes.byref(self.dmat), _ptr(out), _stream_handle(stream)),
              "uw_decode_exponents")
        return out

    def transcode(self, out=None, stream=None):
        import torch
        if out is None:
            out = torch.empty(self.n * self.k // 2, dtype=torch.uint8, device=self.dev.device)
        check(lib().uw_transcode_palette(ctypes.byref(self.dmat), _ptr(out), _stream_handle(stream)),
              "uw_transcode_palette")
        return out

    def device_status(self, stream=None) -> int:
        """Synchronize and return (and clear) the kernels' error status."""
        return int(lib().uw_device_status(ctypes.byref(self.dmat), _stream_handle(stream)))

    # -- matmul
    def workspace_bytes(self, m: int, plan: Plan) -> int:
        return workspace_size(m, self.n, self.k, plan)

    def matmul(self, x, plan: Plan, y=None, ws=None, pal=None, stream=None):
        """Y[m, n] (float32) = X[m, k] (BF16 bits, int16) * W^T."""
        import torch
        m = x.shape[0]
        if y is None:
            y = torch.empty(m, self.n, dtype=torch.float32, device=x.device)
        if ws is None:
            ws = new_workspace(self.workspace_bytes(m, plan), x.device)
        check(lib().uw_fused_matmul(_ptr(x), m, ctypes.byref(self.dmat), _ptr(pal), _ptr(y),
                                    ctypes.byref(plan), _ptr(ws), ws.numel() if ws is not None else 0,
                                    _stream_handle(stream)), "uw_fused_matmul")
        return y


def fused_matmul_noalloc(mat: "Matrix", x, plan: Plan, y=None, stream=None):
    """uw_fused_matmul_noalloc: the fused matmul with no caller workspace (the
    split-K partial sums live in a fixed library-owned device array)."""
    import torch
    m = x.shape[0]
    if y is None:
        y = torch.empty(m, mat.n, dtype=torch.float32, device=x.device)
    check(lib().uw_fused_matmul_noalloc(_ptr(x), m, ctypes.byref(mat.dmat), _ptr(y), ctypes.byref(plan),
                                        _stream_handle(stream)), "uw_fused_matmul_noalloc")
    return y


def fused_matmul_batched(items, plan: Plan, stream=None):
    """uw_fused_matmul_batched: items are (Matrix, x [m, k], y [m, n]) with
    0 <= m <= 16 (m = 0: skipped); all run with the warp-MMA plan `plan` in
    as few launches as possible (32 matrices each)."""
    arr = (BatchItem * len(items))()
    for i, (mat, x, y) in enumerate(items):
        m = int(x.shape[0])
        if x.shape[1] != mat.k or tuple(y.shape) != (m, mat.n):
            raise ValueError("item %d: shapes do not match the matrix" % i)
        arr[i] = BatchItem(ctypes.pointer(mat.dmat), x.data_ptr() if m else None, m, y.data_ptr() if m else None)
    check(lib().uw_fused_matmul_batched(arr, len(items), ctypes.byref(plan), _stream_handle(stream)),
          "uw_fused_matmul_batched")


class Stack:
    """A fixed sequence of matmuls run by uw_stack_run: matmuls in order on the
    main stream, the decodes / transcodes of pipeline 1-3 steps on a side
    stream ahead of their matmuls (cross-layer overlap).

    steps: (Matrix, x, y, plan) tuples, or (Matrix, x, y, plan, pal) for a
    pipeline-4 step with its own palette plane.  The tensors are kept alive
    by this object; the workspace is allocated once here."""

    def __init__(self, steps):
        import torch
        self.keep = list(steps)
        arr = (StackStep * len(steps))()
        for i, st in enumerate(steps):
            mat, x, y, plan = st[:4]
            pal = st[4] if len(st) > 4 else None
            if x.shape[1] != mat.k or y.shape != (x.shape[0], mat.n):
                raise ValueError("step %d: shapes do not match the matrix" % i)
            arr[i] = StackStep(ctypes.pointer(mat.dmat), x.data_ptr(), x.shape[0], y.data_ptr(), plan,
                               pal.data_ptr() if pal is not None else None)
        self.steps = arr
        size = ctypes.c_size_t()
        check(lib().uw_stack_workspace_size(arr, len(steps), ctypes.byref(size)), "uw_stack_workspace_size")
        self.ws_bytes = int(size.value)
        dev = steps[0][1].device
        self.ws = new_workspace(max(self.ws_bytes, 256), dev)

    def run(self, stream=None, side_stream=None):
        """Issue the whole stack; side_stream=None runs everything on `stream`."""
        side = ctypes.c_void_p(side_stream.cuda_stream) if side_stream is not None else ctypes.c_void_p(0)
        check(lib().uw_stack_run(self.steps, len(self.steps), _ptr(self.ws), self.ws.numel(),
                                 _stream_handle(stream), side), "uw_stack_run")

    def tune_split(self, candidates, reps: int = 5, stream=None):
        """uw_stack_tune_split: the fastest preprocessing SM count among
        `candidates` (0 = no split) and each candidate's microseconds per run."""
        import torch
        cand = (ctypes.c_int * len(candidates))(*candidates)
        us = (ctypes.c_float * len(candidates))()
        best = ctypes.c_int()
        dev = self.ws.device.index if self.ws.device.index is not None else torch.cuda.current_device()
        check(lib().uw_stack_tune_split(self.steps, len(self.steps), _ptr(self.ws), self.ws.numel(), dev, cand,
                                        len(candidates), reps, ctypes.byref(best), us, _stream_handle(stream)),
              "uw_stack_tune_split")
        return best.value, [float(u) for u in us]


class SmSplit:
    """uw_sm_split: the device's SMs split into a preprocessing and a compute
    partition (green contexts), each with a stream, wrapped as torch external
    streams (`prep_stream`, `compute_stream`) for Stack.run and the matmuls.
    Call close() (or leave a `with` block) once their work has completed."""

    def __init__(self, prep_sms: int, device=None):
        import torch
        dev = torch.cuda.current_device() if device is None else int(device)
        h = ctypes.c_void_p()
        check(lib().uw_sm_split_create(dev, prep_sms, ctypes.byref(h)), "uw_sm_split_create")
        self.handle = h
        ps, cs = ctypes.c_void_p(), ctypes.c_void_p()
        pn, cn = ctypes.c_int(), ctypes.c_int()
        check(lib().uw_sm_split_get(h, ctypes.byref(ps), ctypes.byref(cs), ctypes.byref(pn), ctypes.byref(cn)),
              "uw_sm_split_get")
        self.prep_sms, self.compute_sms = pn.value, cn.value
        self.prep_stream = torch.cuda.ExternalStream(ps.value, device=dev)
        self.compute_stream = torch.cuda.ExternalStream(cs.value, device=dev)

    def close(self):
        if self.handle:
            self.prep_stream.synchronize()
            self.compute_stream.synchronize()
            lib().uw_sm_split_destroy(self.handle)
            self.handle = None

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()


def new_workspace(nbytes: int, device):
    """A zero-filled device workspace of `nbytes` (None for 0).  Zero matters
    for stream-K plans, whose tile counters must start at zero; every call
    that completes leaves them zero, so the buffer can be reused as is."""
    import torch
    return torch.zeros(nbytes, dtype=torch.uint8, device=device) if nbytes else None


def workspace_size(m: int, n: int, k: int, plan: Plan) -> int:
    size = ctypes.c_size_t()
    check(lib().uw_workspace_size(m, n, k, ctypes.byref(plan), ctypes.byref(size)), "uw_workspace_size")
    return int(size.value)


def plan_default(m: int, n: int, k: int, pipeline: int = 0) -> Plan:
    p = Plan()
    check(lib().uw_plan_default(m, n, k, pipeline, ctypes.byref(p)), "uw_plan_default")
    return p


def matmul_bf16(x, w, plan: Plan, y=None, ws=None, status=None, stream=None):
    """The same kernels on plain BF16 weights w[n, k] (int16 bit patterns)."""
    import torch
    m, k = x.shape
    n = w.shape[0]
    if y is None:
        y = torch.empty(m, n, dtype=torch.float32, device=x.device)
    if ws is None:
        ws = new_workspace(workspace_size(m, n, k, plan), x.device)
    check(lib().uw_matmul_bf16(_ptr(x), m, _ptr(w), n, k, _ptr(y), ctypes.byref(plan), _ptr(ws),
                               ws.numel() if ws is not None else 0, _ptr(status), _stream_handle(stream)),
          "uw_matmul_bf16")
    return y


def autotune(mats: Sequence[Matrix], ms: Sequence[int], reps: int = 5, stream=None):
    """uw_plan_autotune over matrices x batch sizes -> (plans[i][j], json text)."""
    import torch
    arr = (ctypes.POINTER(DMat) * len(mats))(*[ctypes.pointer(m.dmat) for m in mats])
    msa = (ctypes.c_int64 * len(ms))(*ms)
    size = ctypes.c_size_t()
    check(lib().uw_autotune_workspace_size(arr, len(mats), msa, len(ms), ctypes.byref(size)),
          "uw_autotune_workspace_size")
    dev = mats[0].dev.device
    ws = torch.empty(max(int(size.value), 256), dtype=torch.uint8, device=dev)
    kmax = max(m.k for m in mats)
    nmax = max(m.n for m in mats)
    x = torch.zeros(max(ms), kmax, dtype=torch.int16, device=dev)
    x.copy_(torch.randn(max(ms), kmax, device=dev).to(torch.bfloat16).view(torch.int16))
    y = torch.empty(max(ms), nmax, dtype=torch.float32, device=dev)
    plans = (Plan * (len(mats) * len(ms)))()
    cap = 1 << 20
    js = ctypes.create_string_buffer(cap)
    check(lib().uw_plan_autotune(arr, len(mats), msa, len(ms), _ptr(x), _ptr(y), _ptr(ws), ws.numel(),
                                 reps, plans, js, cap, _stream_handle(stream)), "uw_plan_autotune")
    out = [[plans[i * len(ms) + j] for j in range(len(ms))] for i in range(len(mats))]
    return out, js.value.decode()


PIPELINE_NAMES = {PIPE_DECODE_GEMM: "decode_gemm", PIPE_DECODE_EXP_FUSED: "decode_exp_fused",
                  PIPE_TRANSCODE_FUSED: "transcode_fused", PIPE_DIRECT_PALETTE: "direct_palette",
                  PIPE_HUFFMAN_FUSED: "huffman_fused"}
KERNEL_NAMES = {KERNEL_FMA: "fma", KERNEL_TC: "tc", KERNEL_MMA: "mma", KERNEL_TC_SK: "tc_sk",
                KERNEL_MMA_SK: "mma_sk"}


def plans_from_json(text: str, ms: Sequence[int]):
    """Reload a plan file written by uw_plan_autotune (the per-model plan of
    Unweight page §九): plans[i][j] for matrix i and batch size ms[j].  Raises
    ValueError when the file lacks a (matrix, m) pair or names an unknown
    pipeline or kernel."""
    doc = json.loads(text)
    pipes = {v: k for k, v in PIPELINE_NAMES.items()}
    kerns = {v: k for k, v in KERNEL_NAMES.items()}
    ms = list(ms)
    n_mats = 1 + max((e["matrix"] for e in doc["plans"]), default=-1)
    plans = [[None] * len(ms) for _ in range(n_mats)]
    for e in doc["plans"]:
        if e["m"] not in ms:
            continue
        b = e["best"]
        if b["pipeline"] not in pipes or b["kernel"] not in kerns:
            raise ValueError("plan file: unknown pipeline or kernel in %r" % (b,))
        plans[e["matrix"]][ms.index(e["m"])] = make_plan(pipes[b["pipeline"]], kerns[b["kernel"]], b["bn"],
                                                         b["split_k"], b.get("stages", 0))
    missing = [(i, ms[j]) for i in range(n_mats) for j in range(len(ms)) if plans[i][j] is None]
    if missing:
        raise ValueError("plan file has no plan for (matrix, m) %s" % missing[:4])
    return plans


lib()   # fail loudly at import when the library is missing
