"""The C-ABI library loads, exports every symbol include/qkn.h declares, and
rejects bad arguments on the host before touching a GPU (CPU only)."""
import ctypes
import re
import os

import pytest

import qk_normed_latent_qkn_b200 as qkn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    src = open(os.path.join(ROOT, "include", "qkn.h")).read()
    return sorted(set(re.findall(r"QKN_EXPORT\s+[\w\s\*]+?\b(qkn_\w+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    lib = qkn.raw_library()
    names = declared_symbols()
    assert names, "no declarations found"
    assert sorted(qkn.EXPORTED) == names
    for n in names:
        assert hasattr(lib, n), n


def test_version_and_status_strings():
    assert qkn.version() == 1
    for s in range(6):
        assert qkn.status_string(s)
    assert qkn.status_string(0) == "ok"


DIMS = qkn.Dims(num_heads=16, num_groups=1, r_kv=512, d_h=128, d_rope=64)


def _ws(dims, batch=4, s_q=1, sms=148):
    return qkn.decode_workspace_size(dims, batch, s_q, num_sms=sms)


def test_workspace_size_host_only():
    small = _ws(DIMS, 1)
    big = _ws(DIMS, 64)
    assert big > small > 256
    # enough room for one partial (rows x r fp32) per (segment, CTA) slot
    assert _ws(DIMS, 16, sms=148) >= (16 + 148) * 16 * 512 * 4


@pytest.mark.parametrize("bad", [
    dict(num_heads=0), dict(num_groups=3), dict(r_kv=12), dict(d_rope=7), dict(d_rope=256),
    dict(block_size=32), dict(eps=-1.0), dict(softmax_scale=-1.0), dict(dtype=7),
])
def test_bad_dims_rejected(bad):
    import dataclasses
    d = dataclasses.replace(DIMS, **bad)
    with pytest.raises(qkn.QknError) as e:
        _ws(d)
    assert e.value.status == qkn.ERR_INVALID_ARG


def test_default_softmax_scale_is_accepted():
    """softmax_scale = 0 asks the library for its default, 1/sqrt(d_h + d_rope); the binding passes 0
    when Dims.softmax_scale is None."""
    import dataclasses
    assert DIMS.softmax_scale is None and DIMS.c().softmax_scale == 0.0
    assert _ws(dataclasses.replace(DIMS, softmax_scale=0.0)) == _ws(DIMS)


def test_decode_rejects_null_pointers_before_any_launch():
    lib = qkn.raw_library()
    dims = DIMS.c()
    cache = qkn._Cache(None, None, None, 0)
    rc = lib.qkn_decode(ctypes.byref(dims), ctypes.byref(cache), 0, None, None, None, None, 1, None, 1, 1,
                        None, 0, None, None, None, None)
    assert rc == qkn.ERR_INVALID_ARG
    # a valid-looking cache but missing queries
    cache = qkn._Cache(0x1000, 0x2000, 0x3000, 4)
    rc = lib.qkn_decode(ctypes.byref(dims), ctypes.byref(cache), 0, None, None, None, None, 1, None, 1, 1,
                        None, 0, None, None, None, None)
    assert rc == qkn.ERR_INVALID_ARG
    # misaligned cache base
    cache = qkn._Cache(0x1001, 0x2000, 0x3000, 4)
    rc = lib.qkn_decode(ctypes.byref(dims), ctypes.byref(cache), 0, 0x100, 0x100, 0x100, 0x100, 1, 0x100, 1,
                        1, 0x100, 1 << 20, 0x100, 0x100, None, None)
    assert rc == qkn.ERR_INVALID_ARG


def test_decode_rejects_bad_options():
    lib = qkn.raw_library()
    dims = DIMS.c()
    cache = qkn._Cache(0x1000, 0x2000, 0x3000, 4)
    opts = qkn._Opts(qkn.KERNEL_AUTO, 0, 48, 0)     # head tile must be 16, 32 or 64
    rc = lib.qkn_decode(ctypes.byref(dims), ctypes.byref(cache), 0, 0x100, 0x100, 0x100, 0x100, 1, 0x100, 1,
                        1, 0x100, 1 << 30, 0x100, 0x100, ctypes.byref(opts), None)
    assert rc == qkn.ERR_INVALID_ARG
    rc = lib.qkn_decode(ctypes.byref(dims), ctypes.byref(cache), 5, 0x100, 0x100, 0x100, 0x100, 1, 0x100, 1,
                        1, 0x100, 1 << 30, 0x100, 0x100, None, None)
    assert rc == qkn.ERR_INVALID_ARG


def test_append_and_absorb_reject_bad_arguments():
    lib = qkn.raw_library()
    dims = DIMS.c()
    cache = qkn._Cache(0x1000, 0x2000, 0x3000, 4)
    assert lib.qkn_append(ctypes.byref(dims), ctypes.byref(cache), None, None, None, None, 0, None, None, None,
                          None) == qkn.OK          # n_tok == 0 is a no-op
    assert lib.qkn_append(ctypes.byref(dims), ctypes.byref(cache), None, None, None, None, 3, None, None, None,
                          None) == qkn.ERR_INVALID_ARG
    assert lib.qkn_append(ctypes.byref(dims), ctypes.byref(cache), 0x100, 0x100, 0x100, 0x100, -1, 0x100,
                          None, 0x100, None) == qkn.ERR_INVALID_ARG
    # neither w_k nor key_gram
    assert lib.qkn_append(ctypes.byref(dims), ctypes.byref(cache), 0x100, 0x100, 0x100, 0x100, 3, None,
                          None, 0x100, None) == qkn.ERR_INVALID_ARG
    # a misaligned Gram matrix
    assert lib.qkn_append(ctypes.byref(dims), ctypes.byref(cache), 0x100, 0x100, 0x100, 0x100, 3, 0x100,
                          0x102, 0x100, None) == qkn.ERR_INVALID_ARG
    assert lib.qkn_key_gram(ctypes.byref(dims), None, 0x100, None) == qkn.ERR_INVALID_ARG
    assert lib.qkn_key_gram(ctypes.byref(dims), 0x100, None, None) == qkn.ERR_INVALID_ARG
    assert lib.qkn_absorb_query(ctypes.byref(dims), None, None, None, 0, None, None, None, None, None, None,
                                None, None) == qkn.OK
    assert lib.qkn_absorb_query(ctypes.byref(dims), None, None, None, 2, None, None, None, None, None, None,
                                None, None) == qkn.ERR_INVALID_ARG


def test_kernel_choice_is_host_logic():
    f32 = qkn.Dims(num_heads=4, num_groups=1, r_kv=64, d_h=32, d_rope=16, dtype=qkn.F32)
    assert qkn.decode_kernel_for(f32, 1) == qkn.KERNEL_SIMT
    assert qkn.decode_kernel_for(f32, 1, kernel=qkn.KERNEL_TCGEN05) == -1


def test_append_absorb_validates_both_halves_before_any_launch():
    lib = qkn.raw_library()
    dims = DIMS.c()
    cache = qkn._Cache(0x1000, 0x2000, 0x3000, 4)
    P = 0x100
    # nothing to do: no tokens, no query rows
    assert lib.qkn_append_absorb(ctypes.byref(dims), ctypes.byref(cache), None, None, None, None, 0, None, None,
                                 None, 0, None, None, None, None, None, None, None, None, None, None) == qkn.OK
    # tokens without their arrays
    assert lib.qkn_append_absorb(ctypes.byref(dims), ctypes.byref(cache), None, None, None, None, 2, None, None,
                                 None, 0, P, None, P, P, P, P, None, None, None, None) == qkn.ERR_INVALID_ARG
    # query rows without their outputs
    assert lib.qkn_append_absorb(ctypes.byref(dims), ctypes.byref(cache), None, None, None, None, 0, P, P, P, 2,
                                 P, None, P, P, P, P, None, None, None, None) == qkn.ERR_INVALID_ARG
    # negative counts
    assert lib.qkn_append_absorb(ctypes.byref(dims), ctypes.byref(cache), P, P, P, P, -1, P, P, P, 1,
                                 P, None, P, P, P, P, P, P, P, None) == qkn.ERR_INVALID_ARG


def _decode_up(lib, dims, w_uv, d_v, out_v, batch=1):
    cache = qkn._Cache(0x1000, 0x2000, 0x3000, 4)
    return lib.qkn_decode_up(ctypes.byref(dims), ctypes.byref(cache), 0, 0x100, 0x100, 0x100, 0x100, 1, 0x100,
                             batch, 1, w_uv, d_v, 0x100, 1 << 30, out_v, 0x100, None, None)


def test_decode_up_validates_the_value_projection_before_any_launch():
    lib = qkn.raw_library()
    dims = DIMS.c()
    for d_v in (0, -16, 8, 100):                 # d_v must be a positive multiple of 16
        assert _decode_up(lib, dims, 0x100, d_v, 0x100) == qkn.ERR_INVALID_ARG
    assert _decode_up(lib, dims, None, 128, 0x100) == qkn.ERR_INVALID_ARG       # no W^UV
    assert _decode_up(lib, dims, 0x100, 128, None) == qkn.ERR_INVALID_ARG       # no output
    assert _decode_up(lib, dims, 0x108, 128, 0x100) == qkn.ERR_INVALID_ARG      # misaligned W^UV
    assert _decode_up(lib, dims, 0x100, 128, 0x104) == qkn.ERR_INVALID_ARG      # misaligned output
    assert _decode_up(lib, dims, 0x100, 128, 0x100, batch=0) == qkn.OK          # empty batch: no-op
    # W^UV_h and 32 merged rows must fit one CTA's shared memory: d_v = 176 is the widest at
    # r_kv = 512 in bf16; r_kv above 512 is not taken
    assert _decode_up(lib, dims, 0x100, 192, 0x100) == qkn.ERR_UNSUPPORTED
    import dataclasses
    wide = dataclasses.replace(DIMS, r_kv=1024).c()
    assert _decode_up(lib, wide, 0x100, 64, 0x100) == qkn.ERR_UNSUPPORTED


# ---------------------------------------------------------------- the GQA route
GQA_DIMS = qkn.Dims(num_heads=128, num_groups=8, r_kv=512, d_h=128, d_rope=64)


def _gqa_decode(lib, dims, cache, selection=None, sel_k=0, batch=1, q=0x100, out_v=0x100, ws=0x100):
    return lib.qkn_gqa_decode(ctypes.byref(dims), ctypes.byref(cache), q, 0x100, 0x100, 0x100, 0x100, 1, 0x100,
                              batch, 1, selection, sel_k, ws, 1 << 30, out_v, 0x100, 0, None)


def _gqa_append(lib, dims, cache, n_tok=4, c_new=0x100, w_uk=0x100):
    return lib.qkn_gqa_append(ctypes.byref(dims), ctypes.byref(cache), c_new, 0x100, 0x100, 0x100, n_tok, w_uk,
                              0x100, 0x100, 0x100, None)


def test_gqa_route_validates_before_any_launch():
    lib = qkn.raw_library()
    dims = GQA_DIMS.c()
    cache = qkn._GqaCache(0x1000, 0x2000, 0x3000, 4, 128)
    # widths the kernels take: (d_h, d_rope, d_v) = (128, 64, 128) or (64, 32, 64), bf16 only
    assert _gqa_decode(lib, dims, qkn._GqaCache(0x1000, 0x2000, 0x3000, 4, 96)) == qkn.ERR_UNSUPPORTED
    import dataclasses
    f32 = dataclasses.replace(GQA_DIMS, dtype=qkn.F32).c()
    assert _gqa_decode(lib, f32, cache) == qkn.ERR_UNSUPPORTED
    assert _gqa_append(lib, f32, cache) == qkn.ERR_UNSUPPORTED
    narrow = dataclasses.replace(GQA_DIMS, d_h=64, d_rope=32).c()
    assert _gqa_decode(lib, narrow, qkn._GqaCache(0x1000, 0x2000, 0x3000, 4, 64), batch=0) == qkn.OK
    # missing cache arrays, misaligned pointers, a selection without a length
    assert _gqa_decode(lib, dims, qkn._GqaCache(0x1000, None, 0x3000, 4, 128)) == qkn.ERR_INVALID_ARG
    assert _gqa_decode(lib, dims, qkn._GqaCache(0x1008, 0x2000, 0x3000, 4, 128)) == qkn.ERR_INVALID_ARG
    assert _gqa_decode(lib, dims, cache, q=None) == qkn.ERR_INVALID_ARG
    assert _gqa_decode(lib, dims, cache, q=0x104) == qkn.ERR_INVALID_ARG
    assert _gqa_decode(lib, dims, cache, out_v=0x108) == qkn.ERR_INVALID_ARG
    assert _gqa_decode(lib, dims, cache, ws=0x180) == qkn.ERR_INVALID_ARG       # workspace 256-byte aligned
    assert _gqa_decode(lib, dims, cache, selection=0x100, sel_k=0) == qkn.ERR_INVALID_ARG
    assert _gqa_decode(lib, dims, cache, batch=0) == qkn.OK                     # empty batch: no-op
    assert _gqa_append(lib, dims, cache, n_tok=-1) == qkn.ERR_INVALID_ARG
    assert _gqa_append(lib, dims, cache, n_tok=0) == qkn.OK
    assert _gqa_append(lib, dims, cache, c_new=None) == qkn.ERR_INVALID_ARG
    assert _gqa_append(lib, dims, cache, w_uk=0x104) == qkn.ERR_INVALID_ARG
    odd_r = dataclasses.replace(GQA_DIMS, r_kv=520).c()       # the expansion stages 32 latent columns at a time
    assert _gqa_append(lib, odd_r, cache) == qkn.ERR_UNSUPPORTED


def test_gqa_workspace_holds_one_partial_per_slot():
    # dense: 32 query rows per tile (s_q = 2, 16 heads per group), one tile per group, a partial
    # (rows x d_v fp32 + lse) per (sequence, tile) pair and per CTA of the schedule
    ws = qkn.gqa_workspace_size(GQA_DIMS, 128, 32, 2, num_sms=148)
    assert ws >= 256 + (32 * 8 + 148) * 32 * (128 * 4 + 4)
    assert qkn.gqa_workspace_size(GQA_DIMS, 128, 64, 2, num_sms=148) > ws

