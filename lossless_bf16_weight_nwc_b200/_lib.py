"""ctypes binding of libnwc (include/nwc.h): argument marshalling only.

Every function of the C ABI is exposed under the same name; each step of the
path runs in libnwc's kernels.  PyTorch supplies device memory and streams.
There is no fallback: if libnwc.so is missing or cannot be loaded, import of
this module raises.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libnwc.so")

NWC_OK = 0
STATUS = {0: "NWC_OK", 1: "NWC_ERR_INVALID_ARG", 2: "NWC_ERR_UNSUPPORTED", 3: "NWC_ERR_CUDA",
          4: "NWC_ERR_CORRUPT", 5: "NWC_ERR_NOMEM", 6: "NWC_ERR_DEVICE_TIMEOUT",
          7: "NWC_ERR_DEVICE_CORRUPT", 8: "NWC_ERR_SCRATCH_LIMIT"}
NWC_ERR_SCRATCH_LIMIT = 8
NWC_NOALLOC_SCRATCH_BYTES = 8 << 20


class NwcError(RuntimeError):
    def __init__(self, status: int, call: str):
        super().__init__(f"{call} failed: {STATUS.get(status, status)}")
        self.status = status


class nwc_schedule_info(ctypes.Structure):
    _fields_ = [("struct_size", ctypes.c_uint32), ("ctas", ctypes.c_int32),
                ("batch_tiles", ctypes.c_int32), ("ring_bytes", ctypes.c_int32),
                ("tiles", ctypes.c_int64), ("batches", ctypes.c_int64),
                ("smem_bytes", ctypes.c_uint64), ("xstage_bytes", ctypes.c_uint32)]


class nwc_tc_schedule_info(ctypes.Structure):
    _fields_ = [("struct_size", ctypes.c_uint32), ("ctas", ctypes.c_int32),
                ("rows", ctypes.c_int32), ("teams", ctypes.c_int32),
                ("batch_tiles", ctypes.c_int32), ("ring_bytes", ctypes.c_int32),
                ("n", ctypes.c_int32), ("x_stages", ctypes.c_int32),
                ("tiles", ctypes.c_int64), ("batches", ctypes.c_int64),
                ("smem_bytes", ctypes.c_uint64), ("a_offset", ctypes.c_uint64),
                ("b_offset", ctypes.c_uint64), ("ring_offset", ctypes.c_uint64),
                ("ksplit", ctypes.c_int32), ("a_stages", ctypes.c_int32)]


NWC_CODE_PREFIX, NWC_CODE_RANK, NWC_CODE_ESCAPE = 0, 1, 2


class nwc_opts(ctypes.Structure):
    _fields_ = [("struct_size", ctypes.c_uint32), ("lmax", ctypes.c_uint32),
                ("tile_rows", ctypes.c_uint32), ("tile_cols", ctypes.c_uint32),
                ("threads", ctypes.c_uint32), ("code", ctypes.c_uint32),
                ("streams", ctypes.c_uint32), ("keep", ctypes.c_uint32)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"libnwc.so not built ({LIB_PATH}); run "
                           "`python -m lossless_bf16_weight_nwc_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    c = ctypes
    vp, u64, i64, i32 = c.c_void_p, c.c_uint64, c.c_int64, c.c_int32
    sig = {
        "nwc_version": ([], c.c_int),
        "nwc_status_string": ([c.c_int], c.c_char_p),
        "nwc_plan": ([vp, i64, i64, c.POINTER(nwc_opts), c.POINTER(vp)], c.c_int),
        "nwc_plan_size": ([vp, c.POINTER(u64), c.POINTER(u64)], c.c_int),
        "nwc_compress": ([vp, vp, vp, u64, vp, c.POINTER(vp)], c.c_int),
        "nwc_compress_host": ([vp, vp, vp, u64], c.c_int),
        "nwc_blob_device_bytes": ([vp, u64, c.POINTER(u64)], c.c_int),
        "nwc_upload_blob": ([vp, u64, vp, u64, vp, c.POINTER(vp)], c.c_int),
        "nwc_handle_from_device": ([vp, u64, c.POINTER(vp)], c.c_int),
        "nwc_decompress": ([vp, vp, vp], c.c_int),
        "nwc_gather_rows": ([vp, vp, i32, vp, vp], c.c_int),
        "nwc_gemv_scratch_bytes": ([vp, i32, c.POINTER(u64)], c.c_int),
        "nwc_gemv": ([vp, vp, vp, i32, vp], c.c_int),
        "nwc_gemv_noalloc": ([vp, vp, vp, i32, vp], c.c_int),
        "nwc_gemv_set_tc_min_batch": ([vp, i32], c.c_int),
        "nwc_gemv_path": ([vp, vp, i32, c.POINTER(i32), c.POINTER(i32)], c.c_int),
        "nwc_handle_info": ([vp, c.POINTER(i64), c.POINTER(i64), c.POINTER(u64),
                             c.POINTER(u64), c.POINTER(u64)], c.c_int),
        "nwc_get_device_error": ([vp, vp, c.POINTER(c.c_uint32)], c.c_int),
        "nwc_test_set_wait_limit": ([c.c_uint32], None),
        "nwc_schedule_describe": ([vp, u64, i32, u64, i32, c.POINTER(nwc_schedule_info), vp, vp,
                                   vp],
                                  c.c_int),
        "nwc_tc_schedule_describe": ([vp, u64, i32, u64, i32, c.POINTER(nwc_tc_schedule_info), vp,
                                      vp, vp, vp], c.c_int),
        "nwc_plan_destroy": ([vp], None),
        "nwc_handle_destroy": ([vp], None),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    return lib


LIB = _load()
EXPORTED = ("nwc_version", "nwc_status_string", "nwc_plan", "nwc_plan_size", "nwc_compress",
            "nwc_compress_host", "nwc_blob_device_bytes", "nwc_upload_blob",
            "nwc_handle_from_device", "nwc_decompress", "nwc_gather_rows",
            "nwc_gemv_scratch_bytes", "nwc_gemv",
            "nwc_gemv_noalloc", "nwc_gemv_set_tc_min_batch", "nwc_gemv_path",
            "nwc_handle_info", "nwc_get_device_error", "nwc_test_set_wait_limit",
            "nwc_schedule_describe", "nwc_tc_schedule_describe",
            "nwc_plan_destroy", "nwc_handle_destroy")


def _check(status: int, call: str) -> None:
    if status != NWC_OK:
        raise NwcError(status, call)


def _stream(stream) -> int | None:
    """A torch.cuda.Stream, a raw handle, or None (the current torch stream)."""
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return getattr(stream, "cuda_stream", stream)


def _ptr(t) -> int:
    return t.data_ptr() if hasattr(t, "data_ptr") else int(t)


# ---- the C ABI, one Python function per entry point ------------------------

def nwc_version() -> int:
    return LIB.nwc_version()


def nwc_plan(w_host: np.ndarray, lmax: int = 0, tile_cols: int = 512, threads: int = 0,
             code: int = NWC_CODE_PREFIX, streams: int = 1, keep: int = 0):
    """code NWC_CODE_RANK: the ranked unary code, lmax = number of ranks (0 = 7);
    code NWC_CODE_ESCAPE: the `keep` (0 = 16) most frequent exponents coded, runs
    of 64 holding another one verbatim; streams 2 or 4: bit streams per lane
    (the kernels read 1 and 2; 4 is host encoder only, nwc_compress_host)."""
    w = np.ascontiguousarray(w_host, dtype=np.uint16)
    rows, cols = w.shape
    opts = nwc_opts(ctypes.sizeof(nwc_opts), lmax, 8, tile_cols, threads, code, streams, keep)
    plan = ctypes.c_void_p()
    _check(LIB.nwc_plan(w.ctypes.data, rows, cols, ctypes.byref(opts), ctypes.byref(plan)),
           "nwc_plan")
    return plan


def nwc_plan_size(plan) -> tuple[int, int]:
    dev, host = ctypes.c_uint64(), ctypes.c_uint64()
    _check(LIB.nwc_plan_size(plan, ctypes.byref(dev), ctypes.byref(host)), "nwc_plan_size")
    return dev.value, host.value


def nwc_compress(plan, w_host: np.ndarray, d_buf, d_bytes: int, stream=None):
    w = np.ascontiguousarray(w_host, dtype=np.uint16)
    h = ctypes.c_void_p()
    _check(LIB.nwc_compress(plan, w.ctypes.data, _ptr(d_buf), d_bytes, _stream(stream),
                            ctypes.byref(h)), "nwc_compress")
    return h


def nwc_compress_host(plan, w_host: np.ndarray) -> np.ndarray:
    w = np.ascontiguousarray(w_host, dtype=np.uint16)
    _, n = nwc_plan_size(plan)
    blob = np.zeros(n, dtype=np.uint8)
    _check(LIB.nwc_compress_host(plan, w.ctypes.data, blob.ctypes.data, n), "nwc_compress_host")
    return blob


def nwc_blob_device_bytes(blob: np.ndarray) -> int:
    blob = np.ascontiguousarray(blob, dtype=np.uint8)
    out = ctypes.c_uint64()
    _check(LIB.nwc_blob_device_bytes(blob.ctypes.data, blob.size, ctypes.byref(out)),
           "nwc_blob_device_bytes")
    return out.value


def nwc_upload_blob(blob: np.ndarray, d_buf, d_bytes: int, stream=None):
    blob = np.ascontiguousarray(blob, dtype=np.uint8)
    h = ctypes.c_void_p()
    _check(LIB.nwc_upload_blob(blob.ctypes.data, blob.size, _ptr(d_buf), d_bytes,
                               _stream(stream), ctypes.byref(h)), "nwc_upload_blob")
    return h


def nwc_handle_from_device(d_buf, d_bytes: int):
    h = ctypes.c_void_p()
    _check(LIB.nwc_handle_from_device(_ptr(d_buf), d_bytes, ctypes.byref(h)),
           "nwc_handle_from_device")
    return h


def nwc_decompress(handle, d_w_out, stream=None) -> None:
    _check(LIB.nwc_decompress(handle, _ptr(d_w_out), _stream(stream)), "nwc_decompress")


def nwc_gather_rows(handle, d_rows, n: int, d_out, stream=None) -> None:
    """out[i] = W[rows[i]] (BF16 bit patterns), decoded from the compressed matrix."""
    _check(LIB.nwc_gather_rows(handle, _ptr(d_rows), n, _ptr(d_out), _stream(stream)),
           "nwc_gather_rows")


def nwc_gemv_scratch_bytes(handle, batch: int) -> int:
    out = ctypes.c_uint64()
    _check(LIB.nwc_gemv_scratch_bytes(handle, batch, ctypes.byref(out)), "nwc_gemv_scratch_bytes")
    return out.value


def nwc_gemv(handle, d_x, d_y, batch: int, stream=None) -> None:
    _check(LIB.nwc_gemv(handle, _ptr(d_x), _ptr(d_y), batch, _stream(stream)), "nwc_gemv")


def nwc_gemv_set_tc_min_batch(handle, min_batch: int) -> None:
    """Batches >= min_batch take the tensor-core kernel (0: never)."""
    _check(LIB.nwc_gemv_set_tc_min_batch(handle, min_batch), "nwc_gemv_set_tc_min_batch")


def nwc_gemv_path(handle, d_x, batch: int) -> tuple[int, bool]:
    """(kernel launches, tensor-core kernel?) of a GEMV of `batch` rows with d_x."""
    n, tc = ctypes.c_int32(), ctypes.c_int32()
    _check(LIB.nwc_gemv_path(handle, _ptr(d_x), batch, ctypes.byref(n), ctypes.byref(tc)),
           "nwc_gemv_path")
    return n.value, bool(tc.value)


def nwc_gemv_noalloc(handle, d_x, d_y, batch: int, stream=None) -> None:
    """nwc_gemv with library-owned scratch, for callers that may not allocate
    device memory (see include/nwc.h)."""
    _check(LIB.nwc_gemv_noalloc(handle, _ptr(d_x), _ptr(d_y), batch, _stream(stream)),
           "nwc_gemv_noalloc")


def nwc_handle_info(handle) -> dict:
    r, c = ctypes.c_int64(), ctypes.c_int64()
    b, d, k = ctypes.c_uint64(), ctypes.c_uint64(), ctypes.c_uint64()
    _check(LIB.nwc_handle_info(handle, ctypes.byref(r), ctypes.byref(c), ctypes.byref(b),
                               ctypes.byref(d), ctypes.byref(k)), "nwc_handle_info")
    return {"rows": r.value, "cols": c.value, "blob_bytes": b.value, "device_bytes": d.value,
            "compressed_bytes": k.value}


def nwc_get_device_error(handle, stream=None) -> tuple[int, int]:
    """(status, raw word) of the handle's device error word, read and cleared in
    order on the stream, which it synchronizes."""
    w = ctypes.c_uint32()
    st = LIB.nwc_get_device_error(handle, _stream(stream), ctypes.byref(w))
    return st, w.value


def nwc_test_set_wait_limit(polls: int) -> None:
    """Test use only: polls before a kernel's bounded wait gives up (0 = default)."""
    LIB.nwc_test_set_wait_limit(polls)


def nwc_schedule_describe(blob: np.ndarray, sm_count: int = 148, smem_limit: int = 232448,
                          rows_of_x: int = 1):
    """Launch shape and schedule for a blob on a device of the given size, for a
    launch with rows_of_x rows of x (0: decompression); host only.  Returns
    (info dict, cta_batch [ctas + 1], batch [batches x 4], tile_ring [tiles])."""
    blob = np.ascontiguousarray(blob, dtype=np.uint8)
    info = nwc_schedule_info(struct_size=ctypes.sizeof(nwc_schedule_info))
    _check(LIB.nwc_schedule_describe(blob.ctypes.data, blob.size, sm_count, smem_limit, rows_of_x,
                                     ctypes.byref(info), None, None, None),
           "nwc_schedule_describe")
    cta = np.zeros(info.ctas + 1, dtype=np.uint32)
    bat = np.zeros((info.batches, 4), dtype=np.uint32)
    ring = np.zeros(info.tiles, dtype=np.uint32)
    _check(LIB.nwc_schedule_describe(blob.ctypes.data, blob.size, sm_count, smem_limit, rows_of_x,
                                     ctypes.byref(info), cta.ctypes.data, bat.ctypes.data,
                                     ring.ctypes.data), "nwc_schedule_describe")
    d = {k: getattr(info, k) for k, _ in nwc_schedule_info._fields_ if k != "struct_size"}
    return d, cta, bat, ring


def nwc_tc_schedule_describe(blob: np.ndarray, sm_count: int = 148, smem_limit: int = 232448,
                             rows_of_x: int = 64):
    """The tensor-core kernel's launch shape and schedule for a blob and a GEMV
    of rows_of_x rows on a device of the given size; host only.  Returns (info
    dict, cta_batch [ctas + 1], batch [batches x 4], tile_ring [tiles],
    tile_batch [tiles])."""
    blob = np.ascontiguousarray(blob, dtype=np.uint8)
    info = nwc_tc_schedule_info(struct_size=ctypes.sizeof(nwc_tc_schedule_info))
    _check(LIB.nwc_tc_schedule_describe(blob.ctypes.data, blob.size, sm_count, smem_limit,
                                        rows_of_x, ctypes.byref(info), None, None, None, None),
           "nwc_tc_schedule_describe")
    cta = np.zeros(info.ctas + 1, dtype=np.uint32)
    bat = np.zeros((info.batches, 4), dtype=np.uint32)
    ring = np.zeros(info.tiles, dtype=np.uint32)
    tb = np.zeros(info.tiles, dtype=np.uint32)
    _check(LIB.nwc_tc_schedule_describe(blob.ctypes.data, blob.size, sm_count, smem_limit,
                                        rows_of_x, ctypes.byref(info), cta.ctypes.data,
                                        bat.ctypes.data, ring.ctypes.data, tb.ctypes.data),
           "nwc_tc_schedule_describe")
    d = {k: getattr(info, k) for k, _ in nwc_tc_schedule_info._fields_ if k != "struct_size"}
    return d, cta, bat, ring, tb


def nwc_plan_destroy(plan) -> None:
    LIB.nwc_plan_destroy(plan)


def nwc_handle_destroy(handle) -> None:
    LIB.nwc_handle_destroy(handle)


# ---- convenience object over the same calls ---------------------------------

def _require(t, what: str, dtypes, shape, device, pinned_host_ok: bool = False) -> None:
    """Host-side checks of a tensor handed to a kernel: a tensor on another
    device, of another type or shape would otherwise be read or written out of
    bounds on the GPU."""
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{what}: expected a torch.Tensor, got {type(t).__name__}")
    if t.dtype not in dtypes:
        raise TypeError(f"{what}: dtype {t.dtype}, expected one of {[str(d) for d in dtypes]}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{what}: shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{what}: must be contiguous")
    if t.device != device and not (pinned_host_ok and t.device.type == "cpu" and t.is_pinned()):
        where = f"{device} or pinned host memory" if pinned_host_ok else str(device)
        raise ValueError(f"{what}: on {t.device}, expected {where}")


class CompressedMatrix:
    """A BF16 matrix held compressed in device memory that torch allocated.

    Owns the device image (a uint8 CUDA tensor, which also holds the GEMV's
    scratch) and the handle.  Calls make the image's device current and run on
    that device's current torch stream (or the stream given); calls on one
    matrix must be ordered."""

    def __init__(self, image, handle, rows: int, cols: int, blob_bytes: int):
        self.image = image
        self.handle = handle
        self.rows, self.cols = rows, cols
        self.blob_bytes = blob_bytes
        self.device_bytes = image.numel()
        self.row_splits = [0, rows]  # first output row of each part, then rows

    @classmethod
    def compress(cls, w_host: np.ndarray, device="cuda", lmax: int = 0, tile_cols: int = 512,
                 threads: int = 0, stream=None, streams: int = 1,
                 code: int = NWC_CODE_PREFIX, keep: int = 0) -> "CompressedMatrix":
        """streams: bit streams per lane and tile (1 or 2; with 2 a lane's
        decoder follows two independent streams).  code NWC_CODE_RANK: the
        ranked unary code, lmax = its number of ranks (0 = 7).  code
        NWC_CODE_ESCAPE: the `keep` (0 = 16) most frequent exponents coded, a
        run of 64 weights holding another one kept verbatim."""
        import torch
        plan = nwc_plan(w_host, lmax=lmax, tile_cols=tile_cols, threads=threads, streams=streams,
                        code=code, keep=keep)
        try:
            dev_bytes, blob_bytes = nwc_plan_size(plan)
            image = torch.empty(dev_bytes, dtype=torch.uint8, device=device)
            with torch.cuda.device(image.device):
                h = nwc_compress(plan, w_host, image, dev_bytes, stream)
        finally:
            nwc_plan_destroy(plan)
        return cls(image, h, w_host.shape[0], w_host.shape[1], blob_bytes)

    @classmethod
    def compress_fused(cls, parts, device="cuda", lmax: int = 0, tile_cols: int = 512,
                       threads: int = 0, stream=None, streams: int = 1,
                       code: int = NWC_CODE_PREFIX, keep: int = 0) -> "CompressedMatrix":
        """Projections that read the same input (q, k, v; gate, up) held as one
        matrix: the parts' rows stacked in order under one code table, so that a
        call is one launch ("NWC — Neural Weight Compression", "Install": fuse
        before convert).  row_splits holds each part's first output row; split()
        cuts a result into the parts' outputs."""
        ws = [np.ascontiguousarray(p, dtype=np.uint16) for p in parts]
        if not ws or any(w.ndim != 2 or w.shape[1] != ws[0].shape[1] for w in ws):
            raise ValueError("parts: one or more 2-D matrices with the same number of columns")
        m = cls.compress(np.concatenate(ws, axis=0), device=device, lmax=lmax,
                         tile_cols=tile_cols, threads=threads, stream=stream, streams=streams,
                         code=code, keep=keep)
        m.row_splits = [int(v) for v in np.cumsum([0] + [w.shape[0] for w in ws])]
        return m

    def split(self, y):
        """The parts' outputs: views of y's last dimension at row_splits."""
        b = self.row_splits
        return [y[..., b[i]:b[i + 1]] for i in range(len(b) - 1)]

    @classmethod
    def from_blob(cls, blob: np.ndarray, device="cuda", stream=None) -> "CompressedMatrix":
        import torch
        n = nwc_blob_device_bytes(blob)
        image = torch.empty(n, dtype=torch.uint8, device=device)
        with torch.cuda.device(image.device):
            h = nwc_upload_blob(blob, image, n, stream)
        info = nwc_handle_info(h)
        return cls(image, h, info["rows"], info["cols"], info["blob_bytes"])

    @property
    def ratio(self) -> float:
        """Uncompressed BF16 bytes / compressed bytes (blob, decode table and
        launch schedules: the device image without its scratch area)."""
        return 2.0 * self.rows * self.cols / self.compressed_bytes

    @property
    def compressed_bytes(self) -> int:
        return nwc_handle_info(self.handle)["compressed_bytes"]

    def device_error(self, stream=None) -> tuple[int, int]:
        """(status, raw word) of this matrix's device error word (read and cleared)."""
        import torch
        with torch.cuda.device(self.image.device):
            return nwc_get_device_error(self.handle, stream)

    def _open(self) -> None:
        if self.handle is None:
            raise ValueError("the compressed matrix is closed")

    def decompress(self, out=None, stream=None):
        """W as BF16 [rows, cols] (out may also be int16 or uint16: the bit patterns)."""
        import torch
        self._open()
        if out is None:
            out = torch.empty((self.rows, self.cols), dtype=torch.bfloat16,
                              device=self.image.device)
        _require(out, "out", (torch.bfloat16, torch.int16, torch.uint16), (self.rows, self.cols),
                 self.image.device)
        with torch.cuda.device(self.image.device):
            nwc_decompress(self.handle, out, stream)
        return out

    def gemv(self, x, y=None, stream=None):
        """y = x @ W^T for x BF16 [..., cols] on the matrix's device -> FP32
        [batch, rows], batch = x.numel() // cols.  y, when given, is FP32
        [batch, rows] on that device or in pinned host memory."""
        import torch
        self._open()
        if not isinstance(x, torch.Tensor) or x.dim() < 1 or x.shape[-1] != self.cols:
            raise ValueError(f"x: expected a tensor [..., {self.cols}]")
        xb = x.reshape(-1, self.cols)
        batch = xb.shape[0]
        if not 1 <= batch <= 64:
            raise ValueError(f"x: {batch} rows; a call takes 1 to 64")
        _require(xb, "x", (torch.bfloat16,), (batch, self.cols), self.image.device)
        if y is None:
            y = torch.empty((batch, self.rows), dtype=torch.float32, device=self.image.device)
        _require(y, "y", (torch.float32,), (batch, self.rows), self.image.device,
                 pinned_host_ok=True)
        with torch.cuda.device(self.image.device):
            nwc_gemv(self.handle, xb, y, batch, stream)
        return y

    def gather_rows(self, rows, stream=None):
        """BF16 rows W[rows] -> [len(rows), cols]; integer ids, moved to the
        matrix's device.  An id outside [0, rows) makes the kernel skip that row
        and set the device error word (see nwc_get_device_error)."""
        import torch
        self._open()
        if not isinstance(rows, torch.Tensor) or rows.dtype.is_floating_point or rows.dim() != 1:
            raise TypeError("rows: expected a 1-D integer tensor")
        ids = rows.to(device=self.image.device, dtype=torch.int32).contiguous()
        out = torch.empty((ids.numel(), self.cols), dtype=torch.bfloat16, device=self.image.device)
        if ids.numel():
            with torch.cuda.device(self.image.device):
                nwc_gather_rows(self.handle, ids, ids.numel(), out, stream)
        return out

    def close(self) -> None:
        if self.handle is not None:
            nwc_handle_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
