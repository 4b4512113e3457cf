"""ctypes binding of librssm (the C ABI declared in include/rssm.h).

Argument marshalling only: every step of the decode path runs in the CUDA
kernels of librssm.so.  PyTorch supplies device memory and streams.  There is
no CPU fallback: if the library is missing or no GPU is present, the calls
raise.

Low level: ``lib()`` returns the loaded ctypes library whose functions carry
the C names (``rssm_create``, ``rssm_decode_step``, ...).  High level:
``ReplayLayer`` allocates the four caller-owned buffers with torch, binds a
handle, and exposes the calls with the same names minus the ``rssm_`` prefix.
"""
from __future__ import annotations

import ctypes as C
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "librssm.so")

RSSM_OK, RSSM_ERR_INVALID_ARG, RSSM_ERR_UNSUPPORTED = 0, 1, 2
RSSM_ERR_CAPACITY, RSSM_ERR_STATE, RSSM_ERR_CUDA, RSSM_ERR_TIMEOUT = 3, 4, 5, 6
RSSM_STATUS_CAPACITY, RSSM_STATUS_STATE, RSSM_STATUS_TIMEOUT = 1, 2, 4
RSSM_MAMBA2, RSSM_GDN, RSSM_KDA = 1, 2, 3
RSSM_F32, RSSM_BF16 = 0, 1
RSSM_READ_FP32, RSSM_READ_FP8_E4M3_ROW, RSSM_READ_NVFP4 = 0, 1, 2

EXPORTED = [
    "rssm_workspace_size", "rssm_create", "rssm_destroy", "rssm_reset", "rssm_set_params",
    "rssm_decode_step", "rssm_verify", "rssm_rollback", "rssm_flush",
    "rssm_quantize_read_copy", "rssm_conventional_step", "rssm_get_bookkeeping",
    "rssm_get_status", "rssm_last_error_string", "rssm_launch_count",
    "rssm_decode_step_static_scratch", "rssm_conventional_step_quantized",
    "rssm_branch", "rssm_restore", "rssm_get_slots",
    "rssm_state_bytes", "rssm_export_state", "rssm_import_state", "rssm_get_lengths",
    "rssm_set_wait_limit", "rssm_arm_timeout_test",
]
RSSM_STATIC_SCRATCH_MAX_BATCH = 65536


class LayerDesc(C.Structure):
    _fields_ = [("kind", C.c_int), ("batch", C.c_int), ("nheads", C.c_int), ("ngroups", C.c_int),
                ("headdim", C.c_int), ("dstate", C.c_int), ("window", C.c_int),
                ("max_draft", C.c_int), ("in_dtype", C.c_int), ("read_fmt", C.c_int),
                ("auto_flush", C.c_int), ("out_scale", C.c_float), ("branching", C.c_int)]


class Layout(C.Structure):
    _fields_ = [("cap", C.c_size_t), ("buf_off", C.c_size_t * 5), ("rc_codes_off", C.c_size_t),
                ("rc_scales_off", C.c_size_t), ("meta_start_off", C.c_size_t),
                ("meta_len_off", C.c_size_t), ("meta_pending_off", C.c_size_t),
                ("meta_flushes_off", C.c_size_t), ("meta_arrivals_off", C.c_size_t),
                ("meta_status_off", C.c_size_t), ("meta_slot_off", C.c_size_t),
                ("meta_dst_off", C.c_size_t), ("meta_seen_off", C.c_size_t),
                ("meta_work_off", C.c_size_t), ("branch_scratch_off", C.c_size_t),
                ("fold_scratch_off", C.c_size_t)]


_LIB = None


def lib():
    """Load librssm.so (built in-tree); raise if it is missing."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m hybrid_ssm_decode_replayssm_b200.build`")
        L = C.CDLL(LIB_PATH)
        vp, i32, sz = C.c_void_p, C.c_int, C.c_size_t
        L.rssm_workspace_size.argtypes = [C.POINTER(LayerDesc), C.POINTER(sz), C.POINTER(sz),
                                          C.POINTER(sz), C.POINTER(sz), C.POINTER(Layout)]
        L.rssm_create.argtypes = [C.POINTER(LayerDesc), vp, vp, vp, vp, C.POINTER(vp)]
        L.rssm_destroy.argtypes = [vp]
        L.rssm_reset.argtypes = [vp, vp]
        L.rssm_set_params.argtypes = [vp, vp, vp]
        L.rssm_decode_step.argtypes = [vp, C.POINTER(vp), vp, vp]
        L.rssm_verify.argtypes = [vp, i32, C.POINTER(vp), vp, vp]
        L.rssm_decode_step_static_scratch.argtypes = [vp, C.POINTER(vp), vp, vp]
        L.rssm_rollback.argtypes = [vp, vp, vp]
        L.rssm_flush.argtypes = [vp, vp, vp]
        L.rssm_quantize_read_copy.argtypes = [vp, vp]
        L.rssm_conventional_step.argtypes = [vp, vp, vp, C.POINTER(vp), vp, vp]
        L.rssm_conventional_step_quantized.argtypes = [vp, vp, vp, vp, vp, C.POINTER(vp), vp, vp]
        L.rssm_get_bookkeeping.argtypes = [vp, vp, vp]
        L.rssm_get_lengths.argtypes = [vp, vp, vp, vp]
        L.rssm_set_wait_limit.argtypes = [vp, C.c_longlong]
        L.rssm_arm_timeout_test.argtypes = [vp]
        L.rssm_branch.argtypes = [vp, vp, vp]
        L.rssm_restore.argtypes = [vp, vp, vp]
        L.rssm_get_slots.argtypes = [vp, vp, vp]
        L.rssm_state_bytes.argtypes = [vp, C.POINTER(sz)]
        L.rssm_export_state.argtypes = [vp, vp, sz, vp]
        L.rssm_import_state.argtypes = [vp, vp, sz, vp]
        L.rssm_get_status.argtypes = [vp, C.POINTER(C.c_uint32), i32, vp]
        for name in EXPORTED:
            getattr(L, name).restype = C.c_int
        L.rssm_last_error_string.restype = C.c_char_p
        L.rssm_last_error_string.argtypes = []
        L.rssm_launch_count.restype = C.c_uint64
        L.rssm_launch_count.argtypes = []
        _LIB = L
    return _LIB


class RSSMError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__(f"rssm error {code}: {msg}")
        self.code = code


def check(code: int):
    if code != RSSM_OK:
        raise RSSMError(code, lib().rssm_last_error_string().decode())


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _ptr_array(tensors):
    arr = (C.c_void_p * len(tensors))()
    for i, t in enumerate(tensors):
        arr[i] = t.data_ptr()
    return arr


def make_desc(kind, batch, nheads, headdim, dstate, ngroups=1, window=16, max_draft=4,
              in_dtype=RSSM_BF16, read_fmt=RSSM_READ_FP32, auto_flush=True, out_scale=1.0,
              branching=False):
    return LayerDesc(kind, batch, nheads, ngroups, headdim, dstate, window, max_draft,
                     in_dtype, read_fmt, int(bool(auto_flush)), float(out_scale), int(bool(branching)))


def workspace_size(desc: LayerDesc):
    L = lib()
    sizes = [C.c_size_t() for _ in range(4)]
    lay = Layout()
    check(L.rssm_workspace_size(C.byref(desc), *[C.byref(s) for s in sizes], C.byref(lay)))
    return [s.value for s in sizes], lay


class ReplayLayer:
    """One SSM layer's ReplaySSM storage on one GPU, with torch-owned buffers.

    ``ckpt`` is the fp32 checkpoint tensor [B, H, R, C] on the device (kept by
    reference: the library folds windows into it in place).  A branching
    layer's checkpoint has 2B slots, [2B, H, R, C]: the caller fills the first
    B, and ``checkpoint_rows()`` gathers the one each sequence reads.
    """

    def __init__(self, desc: LayerDesc, ckpt: torch.Tensor, A=None, D=None, stream=None):
        if not ckpt.is_cuda or ckpt.dtype != torch.float32 or not ckpt.is_contiguous():
            raise ValueError("ckpt must be a contiguous fp32 CUDA tensor")
        self.desc = desc
        (ck, nb, nr, nm), self.layout = workspace_size(desc)
        if ckpt.numel() * 4 != ck:
            raise ValueError(f"ckpt has {ckpt.numel() * 4} bytes, the layer needs {ck}")
        dev = ckpt.device
        self.ckpt = ckpt
        self.buf = torch.zeros(nb, dtype=torch.uint8, device=dev)
        self.read_copy = torch.zeros(max(nr, 256), dtype=torch.uint8, device=dev) if nr else None
        self.meta = torch.zeros(nm, dtype=torch.uint8, device=dev)
        self.A, self.D = A, D
        h = C.c_void_p()
        check(lib().rssm_create(C.byref(desc), ckpt.data_ptr(), self.buf.data_ptr(),
                                _ptr(self.read_copy), self.meta.data_ptr(), C.byref(h)))
        self.handle = h
        check(lib().rssm_reset(self.handle, _stream(stream)))
        if desc.kind == RSSM_MAMBA2:
            if A is None or D is None:
                raise ValueError("Mamba-2 layers need A and D")
            check(lib().rssm_set_params(self.handle, A.data_ptr(), D.data_ptr()))
        if nr:
            check(lib().rssm_quantize_read_copy(self.handle, _stream(stream)))

    def __del__(self):
        h = getattr(self, "handle", None)
        if h is not None and _LIB is not None:
            _LIB.rssm_destroy(h)
            self.handle = None

    # -------------------------------------------------------------- calls
    def decode_step(self, inputs, out, stream=None):
        check(lib().rssm_decode_step(self.handle, _ptr_array(inputs), out.data_ptr(), _stream(stream)))
        return out

    def verify(self, k, inputs, out, stream=None):
        check(lib().rssm_verify(self.handle, int(k), _ptr_array(inputs), out.data_ptr(), _stream(stream)))
        return out

    def rollback(self, n_reject, stream=None):
        check(lib().rssm_rollback(self.handle, n_reject.data_ptr(), _stream(stream)))

    def flush(self, row_mask=None, stream=None):
        check(lib().rssm_flush(self.handle, _ptr(row_mask), _stream(stream)))

    def quantize_read_copy(self, stream=None):
        check(lib().rssm_quantize_read_copy(self.handle, _stream(stream)))

    def conventional_step(self, state_in, state_out, inputs, out, stream=None):
        check(lib().rssm_conventional_step(self.handle, state_in.data_ptr(), state_out.data_ptr(),
                                           _ptr_array(inputs), out.data_ptr(), _stream(stream)))
        return out

    def conventional_step_quantized(self, codes_in, scales_in, codes_out, scales_out, inputs, out,
                                    stream=None):
        """One conventional token on a state kept in the layer's low-precision format
        (buffers from quantized_state_buffers(); in and out may be the same)."""
        check(lib().rssm_conventional_step_quantized(
            self.handle, codes_in.data_ptr(), scales_in.data_ptr(), codes_out.data_ptr(),
            scales_out.data_ptr(), _ptr_array(inputs), out.data_ptr(), _stream(stream)))
        return out

    def quantized_state_buffers(self):
        """(codes uint8, scales) tensors for a state stored in the layer's read format,
        shaped as read_copy_views()."""
        d = self.desc
        B, H, R, Cc = d.batch, d.nheads, d.headdim, d.dstate
        dev = self.ckpt.device
        if d.read_fmt == RSSM_READ_FP8_E4M3_ROW:
            return (torch.zeros((B, H, R, Cc), dtype=torch.uint8, device=dev),
                    torch.zeros((B, H, R), dtype=torch.float32, device=dev))
        if d.read_fmt == RSSM_READ_NVFP4:
            return (torch.zeros((B, H, R, Cc // 2), dtype=torch.uint8, device=dev),
                    torch.zeros((B, H, R, Cc // 16), dtype=torch.uint8, device=dev))
        raise ValueError("layer has no low-precision format")

    def branch(self, parent, stream=None):
        """Sequence b continues from sequence parent[b] (device int32 [B])."""
        check(lib().rssm_branch(self.handle, parent.data_ptr(), _stream(stream)))

    def restore(self, keep, stream=None):
        """Sequence b keeps the first keep[b] committed tokens of its window."""
        check(lib().rssm_restore(self.handle, keep.data_ptr(), _stream(stream)))

    def get_slots(self, stream=None) -> torch.Tensor:
        out = torch.empty(self.desc.batch, dtype=torch.int32, device=self.ckpt.device)
        check(lib().rssm_get_slots(self.handle, out.data_ptr(), _stream(stream)))
        return out

    def checkpoint_rows(self, stream=None) -> torch.Tensor:
        """The checkpoint each sequence reads, [B, H, R, C] (a copy)."""
        if not self.desc.branching:
            return self.ckpt.clone()
        return self.ckpt.index_select(0, self.get_slots(stream).long())

    def state_bytes(self) -> int:
        n = C.c_size_t()
        check(lib().rssm_state_bytes(self.handle, C.byref(n)))
        return n.value

    def export_state(self, host=None, stream=None) -> torch.Tensor:
        """The layer's whole replay state into a pinned host uint8 tensor (synchronised)."""
        n = self.state_bytes()
        if host is None:
            host = torch.empty(n, dtype=torch.uint8, pin_memory=True)
        check(lib().rssm_export_state(self.handle, host.data_ptr(), n, _stream(stream)))
        (torch.cuda.current_stream() if stream is None else stream).synchronize()
        return host

    def import_state(self, host, stream=None):
        check(lib().rssm_import_state(self.handle, host.data_ptr(), host.numel(), _stream(stream)))
        (torch.cuda.current_stream() if stream is None else stream).synchronize()

    def get_bookkeeping(self, stream=None) -> torch.Tensor:
        out = torch.empty((4, self.desc.batch), dtype=torch.int32, device=self.ckpt.device)
        check(lib().rssm_get_bookkeeping(self.handle, out.data_ptr(), _stream(stream)))
        return out

    def get_status(self, clear=False, stream=None) -> int:
        bits = C.c_uint32()
        check(lib().rssm_get_status(self.handle, C.byref(bits), int(bool(clear)), _stream(stream)))
        return bits.value

    def reset(self, stream=None):
        check(lib().rssm_reset(self.handle, _stream(stream)))

    # ------------------------------------------------------ buffer views
    def read_copy_views(self):
        """(codes uint8, scales) views of the read copy, shaped per rssm.h."""
        d, lay = self.desc, self.layout
        B, H, R, Cc = d.batch * (2 if d.branching else 1), d.nheads, d.headdim, d.dstate
        rc = self.read_copy
        if d.read_fmt == RSSM_READ_FP8_E4M3_ROW:
            codes = rc[: B * H * R * Cc].view(B, H, R, Cc)
            scales = rc[lay.rc_scales_off: lay.rc_scales_off + B * H * R * 4].view(torch.float32).view(B, H, R)
        elif d.read_fmt == RSSM_READ_NVFP4:
            codes = rc[: B * H * R * Cc // 2].view(B, H, R, Cc // 2)
            scales = rc[lay.rc_scales_off: lay.rc_scales_off + B * H * R * Cc // 16].view(B, H, R, Cc // 16)
        else:
            raise ValueError("layer has no read copy")
        return codes, scales
