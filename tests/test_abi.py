"""The C-ABI library loads, exports every function include/rssm.h declares, and
its host-side checks behave as documented (no GPU and no device memory used)."""
import ctypes as C
import os
import re

import pytest

from hybrid_ssm_decode_replayssm_b200 import rssm

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "rssm.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[a-z0-9_]+\s*\*?\s*(rssm_[a-z0-9_]+)\s*\(",
                                 src, flags=re.M)))


def test_header_and_binding_agree():
    assert declared_functions() == sorted(rssm.EXPORTED)


def test_library_exports_every_declared_symbol():
    L = rssm.lib()
    for name in declared_functions():
        assert hasattr(L, name), name


def _desc(**kw):
    base = dict(kind=rssm.RSSM_MAMBA2, batch=4, nheads=8, headdim=64, dstate=128, ngroups=2,
                window=16, max_draft=4, in_dtype=rssm.RSSM_BF16, read_fmt=rssm.RSSM_READ_FP32)
    base.update(kw)
    return rssm.make_desc(**base)


def _sizes(desc):
    s = [C.c_size_t() for _ in range(4)]
    lay = rssm.Layout()
    code = rssm.lib().rssm_workspace_size(C.byref(desc), *[C.byref(x) for x in s], C.byref(lay))
    return code, [x.value for x in s], lay


def test_workspace_layout_mamba2():
    code, (ck, buf, rc, meta), lay = _sizes(_desc())
    assert code == rssm.RSSM_OK
    B, H, P, N, G, cap = 4, 8, 64, 128, 2, 20
    assert lay.cap == cap and ck == B * H * P * N * 4 and rc == 0
    assert lay.buf_off[0] == 0
    assert lay.buf_off[1] >= B * H * cap * P * 2 and lay.buf_off[1] % 256 == 0
    assert lay.buf_off[2] >= lay.buf_off[1] + B * G * cap * N * 2
    assert buf >= lay.buf_off[2] + B * H * cap * 4
    assert meta >= lay.meta_status_off + 4


@pytest.mark.parametrize("fmt", [rssm.RSSM_READ_FP8_E4M3_ROW, rssm.RSSM_READ_NVFP4])
def test_workspace_layout_read_copy(fmt):
    code, (ck, buf, rc, meta), lay = _sizes(_desc(read_fmt=fmt))
    assert code == rssm.RSSM_OK
    rows, n = 4 * 8 * 64, 128
    if fmt == rssm.RSSM_READ_FP8_E4M3_ROW:
        codes_bytes, scale_bytes = rows * n, rows * 4            # 1 byte/elem, fp32 per row
    else:
        codes_bytes, scale_bytes = rows * n // 2, rows * n // 16  # 4 bits/elem, e4m3 per 16
    assert lay.rc_codes_off == 0 and lay.rc_scales_off >= codes_bytes
    assert lay.rc_scales_off % 256 == 0 and rc >= lay.rc_scales_off + scale_bytes


@pytest.mark.parametrize("kw,code", [
    (dict(kind=7), rssm.RSSM_ERR_INVALID_ARG),
    (dict(batch=0), rssm.RSSM_ERR_INVALID_ARG),
    (dict(ngroups=3), rssm.RSSM_ERR_INVALID_ARG),
    (dict(window=0), rssm.RSSM_ERR_INVALID_ARG),
    (dict(window=33), rssm.RSSM_ERR_INVALID_ARG),
    (dict(max_draft=9), rssm.RSSM_ERR_INVALID_ARG),
    (dict(window=2, max_draft=3), rssm.RSSM_ERR_INVALID_ARG),
    (dict(in_dtype=5), rssm.RSSM_ERR_INVALID_ARG),
    (dict(read_fmt=9), rssm.RSSM_ERR_INVALID_ARG),
    (dict(headdim=48), rssm.RSSM_ERR_UNSUPPORTED),
    (dict(dstate=96), rssm.RSSM_ERR_UNSUPPORTED),
])
def test_descriptor_validation(kw, code):
    got, _, _ = _sizes(_desc(**kw))
    assert got == code
    assert rssm.lib().rssm_last_error_string()


def test_create_checks_pointers_and_enqueues_nothing():
    L = rssm.lib()
    d = _desc()
    h = C.c_void_p()
    fake = 1 << 20                                          # never dereferenced by rssm_create
    assert L.rssm_create(C.byref(d), None, fake, None, fake, C.byref(h)) == rssm.RSSM_ERR_INVALID_ARG
    assert L.rssm_create(C.byref(d), fake + 16, fake, None, fake, C.byref(h)) == rssm.RSSM_ERR_INVALID_ARG
    d2 = _desc(read_fmt=rssm.RSSM_READ_NVFP4)
    assert L.rssm_create(C.byref(d2), fake, fake, None, fake, C.byref(h)) == rssm.RSSM_ERR_INVALID_ARG
    assert L.rssm_create(C.byref(d), fake, fake, None, fake, C.byref(h)) == rssm.RSSM_OK
    try:
        ins = (C.c_void_p * 4)(fake, fake, fake, fake)
        # parameters not set -> STATE, before anything is launched
        assert L.rssm_decode_step(h, ins, fake, None) == rssm.RSSM_ERR_STATE
        assert L.rssm_set_params(h, None, None) == rssm.RSSM_ERR_INVALID_ARG
        assert L.rssm_set_params(h, fake, fake) == rssm.RSSM_OK
        bad = (C.c_void_p * 4)(fake, None, fake, fake)
        assert L.rssm_decode_step(h, bad, fake, None) == rssm.RSSM_ERR_INVALID_ARG
        mis = (C.c_void_p * 4)(fake, fake + 2, fake, fake)
        assert L.rssm_decode_step(h, mis, fake, None) == rssm.RSSM_ERR_INVALID_ARG
        assert L.rssm_decode_step(h, ins, None, None) == rssm.RSSM_ERR_INVALID_ARG
        assert L.rssm_verify(h, 0, ins, fake, None) == rssm.RSSM_ERR_CAPACITY
        assert L.rssm_verify(h, 5, ins, fake, None) == rssm.RSSM_ERR_CAPACITY
        assert L.rssm_rollback(h, None, None) == rssm.RSSM_ERR_INVALID_ARG
        assert L.rssm_quantize_read_copy(h, None) == rssm.RSSM_ERR_STATE
        assert L.rssm_conventional_step(h, None, fake, ins, fake, None) == rssm.RSSM_ERR_INVALID_ARG
        # an fp32-read layer has no low-precision state format
        assert L.rssm_conventional_step_quantized(h, fake, fake, fake, fake, ins, fake, None) == rssm.RSSM_ERR_STATE
        assert L.rssm_get_bookkeeping(h, None, None) == rssm.RSSM_ERR_INVALID_ARG
        assert L.rssm_get_status(h, None, 0, None) == rssm.RSSM_ERR_INVALID_ARG
    finally:
        assert L.rssm_destroy(h) == rssm.RSSM_OK
    d0 = _desc(max_draft=0)
    assert L.rssm_create(C.byref(d0), fake, fake, None, fake, C.byref(h)) == rssm.RSSM_OK
    L.rssm_set_params(h, fake, fake)
    assert L.rssm_verify(h, 1, ins, fake, None) == rssm.RSSM_ERR_STATE
    L.rssm_destroy(h)


def test_quantized_state_step_checks_pointers():
    L = rssm.lib()
    fake = 1 << 20
    for fmt in (rssm.RSSM_READ_FP8_E4M3_ROW, rssm.RSSM_READ_NVFP4):
        d = _desc(read_fmt=fmt)
        h = C.c_void_p()
        assert L.rssm_create(C.byref(d), fake, fake, fake, fake, C.byref(h)) == rssm.RSSM_OK
        try:
            assert L.rssm_set_params(h, fake, fake) == rssm.RSSM_OK
            ins = (C.c_void_p * 4)(fake, fake, fake, fake)
            q = L.rssm_conventional_step_quantized
            assert q(h, None, fake, fake, fake, ins, fake, None) == rssm.RSSM_ERR_INVALID_ARG
            assert q(h, fake, fake, fake, None, ins, fake, None) == rssm.RSSM_ERR_INVALID_ARG
            assert q(h, fake + 8, fake, fake, fake, ins, fake, None) == rssm.RSSM_ERR_INVALID_ARG
            if fmt == rssm.RSSM_READ_FP8_E4M3_ROW:   # fp32 row scales: 4-byte aligned
                assert q(h, fake, fake + 2, fake, fake, ins, fake, None) == rssm.RSSM_ERR_INVALID_ARG
            assert q(h, fake, fake, fake, fake, ins, None, None) == rssm.RSSM_ERR_INVALID_ARG
        finally:
            assert L.rssm_destroy(h) == rssm.RSSM_OK
    assert L.rssm_conventional_step_quantized(None, None, None, None, None, None, None, None) == \
        rssm.RSSM_ERR_INVALID_ARG


def test_null_handle_everywhere():
    L = rssm.lib()
    for name in ["rssm_reset", "rssm_quantize_read_copy"]:
        assert getattr(L, name)(None, None) == rssm.RSSM_ERR_INVALID_ARG
    assert L.rssm_flush(None, None, None) == rssm.RSSM_ERR_INVALID_ARG
    assert L.rssm_decode_step(None, None, None, None) == rssm.RSSM_ERR_INVALID_ARG
    assert L.rssm_launch_count() >= 0


def test_workspace_layout_branching():
    """A branching layer doubles the checkpoint and read copy (2B slots) and adds the
    branch scratch (a copy of the ring regions) and the slot arrays."""
    for fmt in (rssm.RSSM_READ_FP32, rssm.RSSM_READ_NVFP4):
        code, (ck, buf, rc, meta), lay = _sizes(_desc(read_fmt=fmt))
        code2, (ck2, buf2, rc2, meta2), lay2 = _sizes(_desc(read_fmt=fmt, branching=True))
        assert code == code2 == rssm.RSSM_OK
        assert ck2 == 2 * ck and (rc2 >= 2 * rc - 512)
        assert lay2.branch_scratch_off >= lay2.buf_off[2] and lay2.branch_scratch_off % 256 == 0
        assert buf2 >= 2 * lay2.branch_scratch_off and lay.branch_scratch_off == 0
        B = 4
        offs = [lay2.meta_slot_off, lay2.meta_dst_off, lay2.meta_seen_off, lay2.meta_work_off]
        assert all(o % 256 == 0 for o in offs) and offs == sorted(offs)
        assert offs[0] > lay2.meta_status_off and meta2 >= offs[3] + 5 * B * 4
        assert lay.meta_slot_off == lay.meta_work_off == 0


def test_branch_calls_check_arguments():
    L = rssm.lib()
    fake = 1 << 20
    h = C.c_void_p()
    assert L.rssm_branch(None, fake, None) == rssm.RSSM_ERR_INVALID_ARG
    assert L.rssm_restore(None, fake, None) == rssm.RSSM_ERR_INVALID_ARG
    assert L.rssm_get_slots(None, fake, None) == rssm.RSSM_ERR_INVALID_ARG
    d = _desc()
    assert L.rssm_create(C.byref(d), fake, fake, None, fake, C.byref(h)) == rssm.RSSM_OK
    try:
        assert L.rssm_branch(h, fake, None) == rssm.RSSM_ERR_STATE       # created without branching
        assert L.rssm_get_slots(h, fake, None) == rssm.RSSM_ERR_STATE
        assert L.rssm_restore(h, None, None) == rssm.RSSM_ERR_INVALID_ARG
    finally:
        L.rssm_destroy(h)
    d = _desc(branching=True)
    assert L.rssm_create(C.byref(d), fake, fake, None, fake, C.byref(h)) == rssm.RSSM_OK
    try:
        assert L.rssm_branch(h, None, None) == rssm.RSSM_ERR_INVALID_ARG
        assert L.rssm_get_slots(h, None, None) == rssm.RSSM_ERR_INVALID_ARG
    finally:
        L.rssm_destroy(h)


def test_kda_descriptor_and_layout():
    base = dict(kind=rssm.RSSM_KDA, batch=2, nheads=4, headdim=128, dstate=128, window=8, max_draft=0)
    code, (ck, buf, rc, meta), lay = _sizes(_desc(**base))
    assert code == rssm.RSSM_OK and rc == 0 and ck == 2 * 4 * 128 * 128 * 4
    B, H, cap, d = 2, 4, 9, 128
    assert lay.cap == cap
    assert lay.buf_off[1] >= B * H * cap * d * 2                       # k ring (bf16)
    assert lay.buf_off[3] - lay.buf_off[2] >= B * H * cap * d * 4      # per-channel log gates (fp32)
    assert buf >= lay.buf_off[4] + B * H * cap * d * 4                 # w rows (fp32)
    code, (_, _, rc4, _), _ = _sizes(_desc(**dict(base, read_fmt=rssm.RSSM_READ_NVFP4)))
    assert code == rssm.RSSM_OK and rc4 == 2 * 4 * 128 * 64 + 2 * 4 * 128 * 8   # codes + E4M3 scales
    code, (_, _, rc8, _), _ = _sizes(_desc(**dict(base, read_fmt=rssm.RSSM_READ_FP8_E4M3_ROW)))
    assert code == rssm.RSSM_OK and rc8 == 2 * 4 * 128 * 128 + 2 * 4 * 128 * 4    # codes + fp32 row scales
    assert _sizes(_desc(**dict(base, headdim=64)))[0] == rssm.RSSM_ERR_UNSUPPORTED
    L = rssm.lib()
    fake = 1 << 20
    h = C.c_void_p()
    d_ = _desc(**dict(base, max_draft=2))
    assert L.rssm_create(C.byref(d_), fake, fake, None, fake, C.byref(h)) == rssm.RSSM_OK
    try:
        ins = (C.c_void_p * 5)(fake, fake, fake, fake, fake)
        assert L.rssm_verify(h, 3, ins, fake, None) == rssm.RSSM_ERR_CAPACITY   # k > max_draft
        assert L.rssm_verify(h, 0, ins, fake, None) == rssm.RSSM_ERR_CAPACITY
        assert L.rssm_arm_timeout_test(h) == rssm.RSSM_OK   # bf16: the serving kernel has waits
    finally:
        L.rssm_destroy(h)
    d_ = _desc(**dict(base, in_dtype=rssm.RSSM_F32))
    assert L.rssm_create(C.byref(d_), fake, fake, None, fake, C.byref(h)) == rssm.RSSM_OK
    try:
        assert L.rssm_arm_timeout_test(h) == rssm.RSSM_ERR_UNSUPPORTED
    finally:
        L.rssm_destroy(h)
    # a read copy: the create call needs its buffer; the serving kernel (fp32 reads only)
    # allocates no fold scratch, so the decode kernel has no waits to arm; the stored
    # low-precision state baseline is Mamba-2 / GDN only
    d_ = _desc(**dict(base, read_fmt=rssm.RSSM_READ_NVFP4))
    code, (ck4, buf4, rc4, meta4), lay4 = _sizes(d_)
    assert lay4.fold_scratch_off == 0
    assert L.rssm_create(C.byref(d_), fake, fake, None, fake, C.byref(h)) == rssm.RSSM_ERR_INVALID_ARG
    assert L.rssm_create(C.byref(d_), fake, fake, fake, fake, C.byref(h)) == rssm.RSSM_OK
    try:
        assert L.rssm_arm_timeout_test(h) == rssm.RSSM_ERR_UNSUPPORTED
        n = C.c_size_t()
        assert L.rssm_state_bytes(h, C.byref(n)) == rssm.RSSM_OK and n.value == ck4 + rc4 + buf4 + meta4
        ins = (C.c_void_p * 5)(fake, fake, fake, fake, fake)
        assert L.rssm_conventional_step_quantized(h, fake, fake, fake, fake, ins, fake, None) == \
            rssm.RSSM_ERR_UNSUPPORTED
    finally:
        L.rssm_destroy(h)


def test_state_io_checks_sizes():
    """rssm_state_bytes = checkpoint + read copy + ring buffers + meta (branch scratch
    excluded); export/import refuse a buffer of another size before any copy."""
    L = rssm.lib()
    fake = 1 << 20
    for kw in ({}, {"read_fmt": rssm.RSSM_READ_NVFP4, "branching": True}):
        d = _desc(**kw)
        code, (ck, buf, rc, meta), lay = _sizes(d)
        h = C.c_void_p()
        assert L.rssm_create(C.byref(d), fake, fake, fake, fake, C.byref(h)) == rssm.RSSM_OK
        try:
            n = C.c_size_t()
            assert L.rssm_state_bytes(h, C.byref(n)) == rssm.RSSM_OK
            ring = lay.branch_scratch_off if kw.get("branching") else (lay.fold_scratch_off or buf)
            assert n.value == ck + rc + ring + meta
            assert L.rssm_export_state(h, fake, n.value + 1, None) == rssm.RSSM_ERR_INVALID_ARG
            assert L.rssm_import_state(h, None, n.value, None) == rssm.RSSM_ERR_INVALID_ARG
            assert L.rssm_state_bytes(h, None) == rssm.RSSM_ERR_INVALID_ARG
        finally:
            L.rssm_destroy(h)
